"""GPU parity of the fused grouped-MLP forward and backward with the oracle.

Bar (the stated end-to-end tolerance): relative L2 <= 2e-2 for y, dx, dW1, dW2, dprobs against the
quantisation-emulating fp64 oracle; the routing maps saved by the forward are
bit-exact."""
import numpy as np
import pytest
import torch

import moe_workloads as wl
from oracle import moe as omoe
from tests.util import f64, rel_l2, SEG_ALIGN

pytestmark = pytest.mark.gpu
TOL_E2E = 2e-2


def _run(gpu_lib, cfg, d, backward=True):
    dev = {k: (v.cuda() if v is not None else None) for k, v in d.items()}
    layer = gpu_lib.GroupedMLP(cfg.T, cfg.k, cfg.E, cfg.H, cfg.F)
    gpu_lib.mxmoe_clear_device_status()
    layer.quantize_weights(dev["W1"], dev["W2"])
    y = layer.forward(dev["x"], dev["topk_idx"], dev["probs"])
    grads = layer.backward(dev["dy"]) if backward else None
    st, where = gpu_lib.mxmoe_get_device_status()
    assert st == 0, (st, where)
    return layer, y, grads


def _oracle(d, backward=True):
    x, W1, W2, probs = f64(d["x"]), f64(d["W1"]), f64(d["W2"]), f64(d["probs"])
    y, saved = omoe.mlp_fwd(x, d["topk_idx"].numpy(), probs, W1, W2)
    g = omoe.mlp_bwd(f64(d["dy"]), saved, probs, W1, W2) if backward else None
    return y, saved, g


@pytest.mark.parametrize("name", ["tiny_fb", "small"])
def test_fused_mlp_matches_oracle(gpu_lib, name):
    cfg = wl.CONFIGS["small"] if name == "small" else wl.custom(
        "tiny_fb", T=1024, H=256, F=512, E=4, k=2, seed=1)
    d = wl.make_all(cfg)
    layer, y, (dx, dW1, dW2, dprobs) = _run(gpu_lib, cfg, d)
    torch.cuda.synchronize()
    yo, saved, go = _oracle(d)
    # saved routing maps: bit-exact with the oracle's (128-aligned segments)
    r = omoe.route(d["topk_idx"].numpy(), cfg.E, align=SEG_ALIGN)
    np.testing.assert_array_equal(layer.saved_field("m_splits", torch.int32, cfg.E).cpu().numpy(), r["m_splits"])
    np.testing.assert_array_equal(layer.saved_field("seg_off", torch.int32, cfg.E + 1).cpu().numpy(), r["seg_off"])
    errs = dict(y=rel_l2(f64(y), yo), dx=rel_l2(f64(dx), go["dx"]), dW1=rel_l2(f64(dW1), go["dW1"]),
                dW2=rel_l2(f64(dW2), go["dW2"]), dprobs=rel_l2(f64(dprobs), go["dprobs"]))
    print(name, {k: f"{v:.2e}" for k, v in errs.items()})
    for k, v in errs.items():
        assert v <= TOL_E2E, (k, v)
    if name == "small":   # expert 7 has no tokens: zero weight gradients
        assert torch.all(dW1[cfg.E - 1] == 0) and torch.all(dW2[cfg.E - 1] == 0)
    else:                 # and directly against the expert-by-expert restatement of the backward
        ge = omoe.mlp_bwd_per_expert(f64(d["x"]), f64(d["dy"]), d["topk_idx"].numpy(), f64(d["probs"]),
                                     f64(d["W1"]), f64(d["W2"]))
        for k, got in (("dx", dx), ("dW1", dW1), ("dW2", dW2), ("dprobs", dprobs)):
            assert rel_l2(f64(got), ge[k]) <= TOL_E2E, (k, "per expert")


def test_fused_forward_tiny_config(gpu_lib):
    cfg = wl.CONFIGS["tiny"]
    d = wl.make_all(cfg)
    _, y, _ = _run(gpu_lib, cfg, d, backward=False)
    torch.cuda.synchronize()
    yo, _, _ = _oracle(d, backward=False)
    assert rel_l2(f64(y), yo) <= TOL_E2E


def test_fused_mlp_repeatable(gpu_lib):
    """Two runs give identical bytes (no atomics in the data path)."""
    cfg = wl.custom("rep", T=512, H=256, F=256, E=3, k=2, seed=4)
    d = wl.make_all(cfg)
    _, y1, g1 = _run(gpu_lib, cfg, d)
    _, y2, g2 = _run(gpu_lib, cfg, d)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    for a, b in zip(g1, g2):
        assert torch.equal(a, b)
