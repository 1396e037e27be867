"""GPU parity of the per-tensor FP8 recipe with the oracle (moe.mlp_fwd_fp8_tensor /
mlp_bwd_fp8_tensor), through the C ABI.

Bars: the largest magnitudes the amax passes find and every E4M3 code of the weights and
of the permuted activations are bit-exact (both sides round fp32(v * m) to E4M3 with the
same correctly rounded multiplier); the fused layer's outputs reach relative L2 <= 2e-2
against the oracle run with the same delayed-scaling values for Z and dGU; the largest
|Z| the forward records agrees with the oracle's to 1e-3 (fp32 values on the GPU, fp64 in
the oracle), the largest |dGU| to 2^-7 (the backward reads G / U saved as bf16)."""
import numpy as np
import pytest
import torch

import moe_workloads as wl
from oracle import moe as omoe
from oracle import mxfp8 as omx
from tests.util import f64, rel_l2, u8, SEG_ALIGN

pytestmark = pytest.mark.gpu
TOL_E2E = 2e-2


def test_weights_per_tensor_codes_bit_exact(gpu_lib):
    E, H, F = 3, 256, 512
    W1 = wl.random_matrix(2 * F, H, seed=71, std=0.02, batch=E)
    W2 = wl.random_matrix(H, F, seed=72, std=0.02, batch=E)
    W2[1] *= 50.0                                    # experts with very different ranges
    wq = gpu_lib.mxmoe_weights_quantize_fp8(W1.cuda(), W2.cuda())
    torch.cuda.synchronize()
    v = [gpu_lib.mxmoe_weights_view(wq, E, H, F, w) for w in range(4)]
    r = np.arange(2 * F)
    hf, rr = (r >= F).astype(int), r - (r >= F) * F
    dst = (rr // 64) * 128 + hf * 64 + rr % 64       # gate / up interleave of the rowwise W1
    for e in range(E):
        w1, w2 = f64(W1[e]), f64(W2[e])
        m1, m2 = omx.tensor_multiplier(np.abs(w1).max()), omx.tensor_multiplier(np.abs(w2).max())
        q1, q2 = omx.quantize_tensor(w1, m1), omx.quantize_tensor(w2, m2)
        np.testing.assert_array_equal(u8(v[0].data)[e * 2 * F:(e + 1) * 2 * F][dst], q1)
        np.testing.assert_array_equal(u8(v[1].data)[e * H:(e + 1) * H], q1.T)
        np.testing.assert_array_equal(u8(v[2].data)[e * H:(e + 1) * H], q2)
        np.testing.assert_array_equal(u8(v[3].data)[e * F:(e + 1) * F], q2.T)
    for w in range(4):
        assert np.all(u8(v[w].scale) == 127)
    # the per-expert largest magnitudes, kept in the buffer's last 256-byte field: W1[e], then W2[e]
    am = wq[-256:].view(torch.float32)[:2 * E].cpu().numpy()
    want = [np.abs(f64(W1[e])).max() for e in range(E)] + [np.abs(f64(W2[e])).max() for e in range(E)]
    np.testing.assert_array_equal(am, np.array(want, dtype=np.float32))


def _layer_and_oracle(gpu_lib, cfg):
    d = wl.make_all(cfg)
    x, W1, W2, p = (f64(d[n]) for n in ("x", "W1", "W2", "probs"))
    idx, dy = d["topk_idx"].numpy(), f64(d["dy"])
    # delayed-scaling values: the largest |Z| and |dGU| of a first oracle pass
    _, s0 = omoe.mlp_fwd_fp8_tensor(x, idx, p, W1, W2, z_amax_in=1.0)
    g0 = omoe.mlp_bwd_fp8_tensor(dy, s0, dgu_amax_in=1.0)
    za, ga = np.float32(s0["z_amax"]), np.float32(g0["dgu_amax"])
    yo, so = omoe.mlp_fwd_fp8_tensor(x, idx, p, W1, W2, z_amax_in=float(za))
    go = omoe.mlp_bwd_fp8_tensor(dy, so, dgu_amax_in=float(ga))
    dev = {k: (v.cuda() if v is not None else None) for k, v in d.items()}
    layer = gpu_lib.GroupedMLP(cfg.T, cfg.k, cfg.E, cfg.H, cfg.F, precision="fp8")
    gpu_lib.mxmoe_clear_device_status()
    layer.quantize_weights(dev["W1"], dev["W2"])
    layer.set_amax(za, ga)
    y = layer.forward(dev["x"], dev["topk_idx"], dev["probs"])
    grads = layer.backward(dev["dy"])
    torch.cuda.synchronize()
    st, where = gpu_lib.mxmoe_get_device_status()
    assert st == 0, (st, where)
    return d, layer, y, grads, yo, so, go


@pytest.mark.parametrize("name", ["tiny_fb", "small"])
def test_fp8_tensor_layer_matches_oracle(gpu_lib, name):
    cfg = wl.CONFIGS["small"] if name == "small" else wl.custom("tiny_fb", T=1024, H=256, F=512, E=4, k=2, seed=1)
    d, layer, y, (dx, dW1, dW2, dprobs), yo, so, go = _layer_and_oracle(gpu_lib, cfg)
    errs = dict(y=rel_l2(f64(y), yo), dx=rel_l2(f64(dx), go["dx"]), dW1=rel_l2(f64(dW1), go["dW1"]),
                dW2=rel_l2(f64(dW2), go["dW2"]), dprobs=rel_l2(f64(dprobs), go["dprobs"]))
    print(name, {k: f"{v:.2e}" for k, v in errs.items()})
    for k, v in errs.items():
        assert v <= TOL_E2E, (k, v)
    # the saved amax field: largest |x| (exact) and the Z amax the forward used
    amax = layer.saved_field("amax", torch.float32, 2).cpu().numpy()
    assert amax[0] == np.float32(np.abs(f64(d["x"])).max())
    assert amax[1] == layer.amax_state[0].item()
    # the colwise copy of the permuted x saved for the weight gradient: bit-exact codes
    cap = layer.cap
    r = omoe.route(d["topk_idx"].numpy(), cfg.E, align=SEG_ALIGN)
    xc = u8(layer.saved_field("x_colT", torch.uint8, cfg.H * cap).view(cfg.H, cap))
    q = omx.quantize_tensor(f64(d["x"]), so["m"]["x"])
    live = r["token_of_row"] >= 0
    np.testing.assert_array_equal(xc[:, :r["Mp"]][:, live], q[r["token_of_row"][live]].T)
    assert np.all(xc[:, :r["Mp"]][:, ~live] == 0)
    # the largest |Z| and |dGU| recorded by the fused epilogues, then rolled into the inputs
    st = layer.amax_state.cpu().numpy()
    assert abs(st[1] - so["z_amax"]) <= 1e-3 * so["z_amax"], (st[1], so["z_amax"])
    # dGU comes from G / U saved as bf16 (each rounded by at most 2^-9), so its largest
    # magnitude may differ from the oracle's by up to about 2^-8 relative
    assert abs(st[3] - go["dgu_amax"]) <= 2.0 ** -7 * go["dgu_amax"], (st[3], go["dgu_amax"])
    layer.roll_amax()
    st2 = layer.amax_state.cpu().numpy()
    assert st2[0] == st[1] and st2[2] == st[3]
    if name == "small":   # expert 7 has no tokens: zero weight gradients
        assert torch.all(dW1[cfg.E - 1] == 0) and torch.all(dW2[cfg.E - 1] == 0)


def test_fp8_tensor_saturates_when_the_delayed_amax_is_small(gpu_lib):
    """A delayed Z amax a quarter of the real one: codes saturate at 448 on both sides and
    the layer still matches the oracle run with the same value."""
    cfg = wl.custom("sat", T=512, H=256, F=256, E=3, k=2, seed=73)
    d = wl.make_all(cfg)
    x, W1, W2, p = (f64(d[n]) for n in ("x", "W1", "W2", "probs"))
    idx, dy = d["topk_idx"].numpy(), f64(d["dy"])
    _, s0 = omoe.mlp_fwd_fp8_tensor(x, idx, p, W1, W2, z_amax_in=1.0)
    g0 = omoe.mlp_bwd_fp8_tensor(dy, s0, dgu_amax_in=1.0)
    za, ga = np.float32(s0["z_amax"] / 4), np.float32(g0["dgu_amax"] / 4)
    yo, so = omoe.mlp_fwd_fp8_tensor(x, idx, p, W1, W2, z_amax_in=float(za))
    go = omoe.mlp_bwd_fp8_tensor(dy, so, dgu_amax_in=float(ga))
    dev = {k: v.cuda() for k, v in d.items()}
    layer = gpu_lib.GroupedMLP(cfg.T, cfg.k, cfg.E, cfg.H, cfg.F, precision="fp8")
    layer.quantize_weights(dev["W1"], dev["W2"])
    layer.set_amax(za, ga)
    y = layer.forward(dev["x"], dev["topk_idx"], dev["probs"])
    dx, dW1, dW2, dprobs = layer.backward(dev["dy"])
    torch.cuda.synchronize()
    for got, want in ((y, yo), (dx, go["dx"]), (dW1, go["dW1"]), (dW2, go["dW2"]), (dprobs, go["dprobs"])):
        assert rel_l2(f64(got), want) <= TOL_E2E
    zc = u8(layer.saved_field("z_colT", torch.uint8, cfg.F * layer.cap))
    assert np.any((zc & 0x7F) == 0x7E)               # saturated codes are present
