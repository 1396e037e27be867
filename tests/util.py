"""Shared helpers for the test-suite (no method arithmetic here: conversions and
comparison metrics only)."""
import numpy as np
import torch


def f64(t):
    """torch tensor (any float dtype, any device) -> numpy float64."""
    return t.detach().float().cpu().numpy().astype(np.float64)


def rel_l2(got, want):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    den = np.linalg.norm(want)
    return float(np.linalg.norm(got - want) / (den if den > 0 else 1.0))


def u8(t):
    return t.detach().cpu().numpy().astype(np.uint8)


def to_cuda(d):
    return {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}

# Expert segments of the CUDA path start at multiples of 256 rows (its GEMM tile); the
# oracle's results do not depend on the alignment (pinned in test_oracle_moe.py).
SEG_ALIGN = 256
