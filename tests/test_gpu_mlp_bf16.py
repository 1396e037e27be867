"""GPU parity of the bf16 grouped-MLP layer (the 16-bit comparison point of the MXFP8
layer) with the oracle run without quantisation.

Bar: relative L2 <= 1e-2 for y, dx, dW1, dW2, dprobs. Derivation: x, W1, W2, dy are bf16
on both sides; the kernels round Z, G/U, Yp, dGU and dXp to bf16 (unit roundoff 2^-9,
about 2e-3 relative each, about 1.1e-3 RMS), and no output passes through more than
four such roundings, so 4 * 2^-9 < 1e-2 bounds the relative L2 with margin; every GEMM
accumulates in fp32 (relative error far below that for K <= 28672)."""
import numpy as np
import pytest
import torch

import moe_workloads as wl
from oracle import moe as omoe
from tests.util import f64, rel_l2

pytestmark = pytest.mark.gpu
TOL_BF16 = 1e-2


def _run(gpu_lib, cfg, d):
    dev = {k: (v.cuda() if v is not None else None) for k, v in d.items()}
    layer = gpu_lib.GroupedMLP(cfg.T, cfg.k, cfg.E, cfg.H, cfg.F, precision="bf16")
    gpu_lib.mxmoe_clear_device_status()
    layer.quantize_weights(dev["W1"], dev["W2"])
    y = layer.forward(dev["x"], dev["topk_idx"], dev["probs"])
    grads = layer.backward(dev["dy"])
    torch.cuda.synchronize()
    st, where = gpu_lib.mxmoe_get_device_status()
    assert st == 0, (st, where)
    return y, grads


@pytest.mark.parametrize("name", ["tiny_fb", "small"])
def test_bf16_mlp_matches_oracle(gpu_lib, name):
    cfg = wl.CONFIGS["small"] if name == "small" else wl.custom(
        "tiny_fb", T=1024, H=256, F=512, E=4, k=2, seed=1)
    d = wl.make_all(cfg)
    y, (dx, dW1, dW2, dprobs) = _run(gpu_lib, cfg, d)
    x, W1, W2, probs = f64(d["x"]), f64(d["W1"]), f64(d["W2"]), f64(d["probs"])
    yo, saved = omoe.mlp_fwd(x, d["topk_idx"].numpy(), probs, W1, W2, quant=False)
    go = omoe.mlp_bwd(f64(d["dy"]), saved, probs, W1, W2, quant=False)
    errs = dict(y=rel_l2(f64(y), yo), dx=rel_l2(f64(dx), go["dx"]), dW1=rel_l2(f64(dW1), go["dW1"]),
                dW2=rel_l2(f64(dW2), go["dW2"]), dprobs=rel_l2(f64(dprobs), go["dprobs"]))
    print(name, {k: f"{v:.2e}" for k, v in errs.items()})
    for k, v in errs.items():
        assert v <= TOL_BF16, (k, v)
    if name == "small":   # the last expert has no tokens: zero weight gradients
        assert torch.all(dW1[cfg.E - 1] == 0) and torch.all(dW2[cfg.E - 1] == 0)


def test_bf16_mlp_ragged_and_repeatable(gpu_lib):
    """Ragged segments (T*k not a multiple of anything), one expert with a single row;
    two runs give identical bytes."""
    cfg = wl.custom("ragged", T=333, H=256, F=256, E=5, k=3, seed=11)
    d = wl.make_all(cfg)
    y1, g1 = _run(gpu_lib, cfg, d)
    y2, g2 = _run(gpu_lib, cfg, d)
    assert torch.equal(y1, y2)
    for a, b in zip(g1, g2):
        assert torch.equal(a, b)
    x, W1, W2, probs = f64(d["x"]), f64(d["W1"]), f64(d["W2"]), f64(d["probs"])
    yo, saved = omoe.mlp_fwd(x, d["topk_idx"].numpy(), probs, W1, W2, quant=False)
    go = omoe.mlp_bwd(f64(d["dy"]), saved, probs, W1, W2, quant=False)
    assert rel_l2(f64(y1), yo) <= TOL_BF16
    for name, got in zip(("dx", "dW1", "dW2", "dprobs"), g1):
        assert rel_l2(f64(got), go[name]) <= TOL_BF16, name


def test_bf16_mlp_zero_tokens(gpu_lib):
    """T = 0: the forward writes nothing, the backward zeroes the weight gradients."""
    E, H, F = 3, 256, 256
    layer = gpu_lib.GroupedMLP(0, 2, E, H, F, precision="bf16")
    W1 = torch.randn(E, 2 * F, H, device="cuda").bfloat16()
    W2 = torch.randn(E, H, F, device="cuda").bfloat16()
    layer.quantize_weights(W1, W2)
    x = torch.empty(0, H, dtype=torch.bfloat16, device="cuda")
    idx = torch.empty(0, 2, dtype=torch.int32, device="cuda")
    p = torch.empty(0, 2, dtype=torch.float32, device="cuda")
    y = layer.forward(x, idx, p)
    dW1 = torch.full((E, 2 * F, H), 7.0, device="cuda")
    dW2 = torch.full((E, H, F), 7.0, device="cuda")
    _, dW1, dW2, _ = layer.backward(torch.empty(0, H, dtype=torch.bfloat16, device="cuda"), dW1=dW1, dW2=dW2)
    torch.cuda.synchronize()
    assert y.shape == (0, H)
    assert torch.all(dW1 == 0) and torch.all(dW2 == 0)


def test_bf16_weights_prepare_layout(gpu_lib):
    """The weights buffer holds W1 rows gate/up interleaved in 64-row blocks, W1^T, W2 rows
    and W2^T: exact copies (bytes) of the bf16 inputs."""
    E, H, F = 2, 256, 512
    g = torch.Generator().manual_seed(5)
    W1 = torch.randn(E, 2 * F, H, generator=g).bfloat16()
    W2 = torch.randn(E, H, F, generator=g).bfloat16()
    wb = gpu_lib.mxmoe_weights_bf16_prepare(W1.cuda(), W2.cuda())
    torch.cuda.synchronize()
    raw = wb.cpu()

    def take(off, n):
        return raw[off:off + 2 * n].view(torch.bfloat16), (off + 2 * n + 255) // 256 * 256

    w1r, o = take(0, E * 2 * F * H)
    w1t, o = take(o, E * H * 2 * F)
    w2r, o = take(o, E * H * F)
    w2t, o = take(o, E * F * H)
    ilv = torch.empty_like(W1)
    for blk in range(F // 64):
        ilv[:, 128 * blk:128 * blk + 64] = W1[:, 64 * blk:64 * blk + 64]
        ilv[:, 128 * blk + 64:128 * blk + 128] = W1[:, F + 64 * blk:F + 64 * blk + 64]
    assert torch.equal(w1r.view(E, 2 * F, H), ilv)
    assert torch.equal(w1t.view(E, H, 2 * F), W1.transpose(1, 2))
    assert torch.equal(w2r.view(E, H, F), W2)
    assert torch.equal(w2t.view(E, F, H), W2.transpose(1, 2))
