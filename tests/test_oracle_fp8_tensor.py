"""Pins for the oracle's per-tensor FP8 recipe (one fp32 multiplier per tensor, E4M3
elements) -- the pages name FP8 beside MXFP8 ("MoE-Training für biologische
Grundmodelle optimieren", hyper.ai/de, precision passage) and fix nothing else, so the
multiplier, the rounding and the delayed scaling of Z / dGU are readings; these tests pin
the oracle against exact arithmetic and independent restatements (CPU only)."""
from fractions import Fraction

import numpy as np
import pytest

import moe_workloads as wl
from oracle import moe, mxfp8


def test_multiplier_is_the_nearest_fp32_to_448_over_amax():
    rng = np.random.default_rng(0)
    amaxes = np.concatenate([rng.lognormal(0, 6, 2000), [448.0, 1.0, 3.0, 2.0 ** -20, 1e6]]).astype(np.float32)
    for a in amaxes:
        m = mxfp8.tensor_multiplier(a)
        assert m.dtype == np.float32
        exact = Fraction(448) / Fraction(float(a))
        lo, hi = np.nextafter(m, np.float32(0)), np.nextafter(m, np.float32(np.inf))
        err = abs(Fraction(float(m)) - exact)
        assert err <= abs(Fraction(float(lo)) - exact) and err <= abs(Fraction(float(hi)) - exact)
    assert mxfp8.tensor_multiplier(0.0) == 1.0
    assert mxfp8.tensor_multiplier(448.0) == 1.0
    assert mxfp8.tensor_multiplier(1e-38) == np.finfo(np.float32).max      # quotient overflows


def test_largest_magnitude_maps_to_448():
    rng = np.random.default_rng(1)
    for a in rng.lognormal(0, 8, 500).astype(np.float32):
        m = mxfp8.tensor_multiplier(a)
        q = mxfp8.quantize_tensor(np.array([a, -a], dtype=np.float32), m)
        assert q.tolist() == [0x7E, 0xFE]


def test_unit_multiplier_is_the_plain_encoder_and_powers_of_two_shift():
    rng = np.random.default_rng(2)
    v = (rng.standard_normal(4096) * 40).astype(np.float32)
    v[0] = 448.0
    np.testing.assert_array_equal(mxfp8.quantize_tensor(v, mxfp8.tensor_multiplier(448.0)), mxfp8.e4m3_encode(v))
    # amax 224 -> m = 2: every code is the plain code of 2v
    v2 = (v / 2).astype(np.float32)
    np.testing.assert_array_equal(mxfp8.quantize_tensor(v2, mxfp8.tensor_multiplier(224.0)), mxfp8.e4m3_encode(v))
    assert mxfp8.quantize_tensor(np.float32(1.0), np.float32(2.0)) == 0x40               # 2.0


def test_product_is_rounded_to_fp32_before_e4m3():
    """v * m = 8.5000002 exactly, which rounds to the E4M3 value 9; in fp32 the product is
    8.5, the midpoint of 8 and 9, which goes to the even code (8): the code follows the
    fp32 product."""
    m = np.float32(5.941762924194336)
    v = np.float32(1.4305518865585327)
    assert float(v) * float(m) > 8.5 and float(np.float32(v * m)) == 8.5
    assert mxfp8.e4m3_encode(float(v) * float(m)) == 0x51                 # 9
    assert mxfp8.quantize_tensor(v, m) == 0x50                             # 8


def test_relative_error_bound_in_the_normal_range():
    rng = np.random.default_rng(3)
    v = (rng.standard_normal(100000) * rng.lognormal(0, 2, 100000)).astype(np.float32)
    m = mxfp8.tensor_multiplier(np.max(np.abs(v)))
    deq = mxfp8.fake_quant_tensor(v, m)
    normal = np.abs(v.astype(np.float64) * float(m)) >= 2.0 ** -6
    rel = np.abs(deq[normal] - v[normal]) / np.abs(v[normal])
    assert rel.max() <= 2.0 ** -4 * (1 + 1e-6)
    # below the normal range the error is at most half the subnormal step, in scaled units
    assert np.max(np.abs(deq[~normal] - v[~normal]) * float(m)) <= 2.0 ** -10 * (1 + 1e-6)


def _problem(seed=5, E=4, T=40):
    cfg = wl.custom("pt", T=T, H=64, F=96, E=E, k=2, seed=seed, routing="dead_last")
    d = wl.make_all(cfg)
    x, W1, W2, p = (d[n].double().numpy() for n in ("x", "W1", "W2", "probs"))
    return cfg, x, W1, W2, p, d["topk_idx"].numpy(), d["dy"].double().numpy()


def test_identity_quantiser_reduces_to_the_unquantised_layer(monkeypatch):
    """With the per-tensor quantiser replaced by the identity, the recipe's forward and
    backward equal the unquantised layer (whose backward is pinned by finite
    differences): the GEMM wiring of the recipe is the layer's."""
    cfg, x, W1, W2, p, idx, dy = _problem()
    monkeypatch.setattr(mxfp8, "fake_quant_tensor", lambda v, m: np.asarray(v, dtype=np.float64))
    monkeypatch.setattr(mxfp8, "dequantize_tensor", lambda c, m: np.asarray(c, dtype=np.float64) / np.float64(m))
    monkeypatch.setattr(mxfp8, "e4m3_encode", lambda v: np.asarray(v, dtype=np.float64))
    y, s = moe.mlp_fwd_fp8_tensor(x, idx, p, W1, W2, z_amax_in=1.0)
    g = moe.mlp_bwd_fp8_tensor(dy, s, dgu_amax_in=1.0)
    monkeypatch.undo()
    yu, su = moe.mlp_fwd(x, idx, p, W1, W2, quant=False)
    gu = moe.mlp_bwd(dy, su, p, W1, W2, quant=False)
    np.testing.assert_allclose(y, yu, rtol=1e-11, atol=1e-13)
    for n in ("dx", "dW1", "dW2", "dprobs"):
        np.testing.assert_allclose(g[n], gu[n], rtol=1e-10, atol=1e-12 * np.abs(gu[n]).max(), err_msg=n)


def _per_expert_restatement(x, dy, idx, p, W1, W2, z_amax_in, dgu_amax_in):
    """Token-by-token forward and expert-by-expert backward of the recipe, written from
    its definition: every operand is the elementwise per-tensor fake quantisation of its
    whole tensor (x, dY: all tokens; W1[e], W2[e]: per expert; Z, dGU: all routed rows with
    the given largest magnitudes)."""
    E, F2, H = W1.shape
    F = F2 // 2
    T, k = idx.shape
    fq = mxfp8.fake_quant_tensor
    mult = mxfp8.tensor_multiplier
    xq = fq(x, mult(np.abs(x).max()))
    dyq = fq(dy, mult(np.abs(dy).max()))
    w1q = [fq(W1[e], mult(np.abs(W1[e]).max())) for e in range(E)]
    w2q = [fq(W2[e], mult(np.abs(W2[e]).max())) for e in range(E)]
    mz, mg = np.float64(mult(z_amax_in)), np.float64(mult(dgu_amax_in))
    y = np.zeros((T, H))
    dx = np.zeros((T, H))
    dW1 = np.zeros((E, F2, H))
    dW2 = np.zeros((E, H, F))
    dprobs = np.zeros((T, k))
    for t in range(T):
        for j in range(k):
            e = idx[t, j]
            gu = w1q[e] @ xq[t]
            g_, u_ = gu[:F], gu[F:]
            a_ = moe.silu(g_) * u_
            zq = mxfp8.e4m3_decode(mxfp8.e4m3_encode(a_ * p[t, j] * mz)) / mz
            y[t] += w2q[e] @ zq
            dz = w2q[e].T @ dyq[t]
            dprobs[t, j] = np.sum(dz * a_)
            da = dz * p[t, j]
            dgu = np.concatenate([da * u_ * moe.dsilu(g_), da * moe.silu(g_)])
            dguq = mxfp8.e4m3_decode(mxfp8.e4m3_encode(dgu * mg)) / mg
            dx[t] += w1q[e].T @ dguq
            dW2[e] += np.outer(dyq[t], zq)
            dW1[e] += np.outer(dguq, xq[t])
    return y, dict(dx=dx, dW1=dW1, dW2=dW2, dprobs=dprobs)


@pytest.mark.parametrize("z_scale", [1.0, 0.5])     # 0.5: the delayed amax is too small, Z saturates
def test_recipe_equals_token_by_token_restatement(z_scale):
    cfg, x, W1, W2, p, idx, dy = _problem()
    _, s0 = moe.mlp_fwd_fp8_tensor(x, idx, p, W1, W2, z_amax_in=1.0)
    g0 = moe.mlp_bwd_fp8_tensor(dy, s0, dgu_amax_in=1.0)
    za, ga = s0["z_amax"] * z_scale, g0["dgu_amax"] * z_scale
    y, s = moe.mlp_fwd_fp8_tensor(x, idx, p, W1, W2, z_amax_in=za)
    g = moe.mlp_bwd_fp8_tensor(dy, s, dgu_amax_in=ga)
    yr, gr = _per_expert_restatement(x, dy, idx, p, W1, W2, za, ga)
    np.testing.assert_allclose(y, yr, rtol=1e-10, atol=1e-12 * np.abs(yr).max())
    for n in ("dx", "dW1", "dW2", "dprobs"):
        np.testing.assert_allclose(g[n], gr[n], rtol=1e-10, atol=1e-12 * np.abs(gr[n]).max(), err_msg=n)
    if z_scale < 1:   # saturation happened: the largest codes hit 448
        assert np.isclose(np.abs(s["Zq"]).max() * float(s["m"]["z"]), 448.0)
    assert np.all(g["dW1"][cfg.E - 1] == 0) and np.all(g["dW2"][cfg.E - 1] == 0)   # empty expert


def test_recipe_close_to_unquantised_and_amax_outputs():
    cfg, x, W1, W2, p, idx, dy = _problem(seed=6, T=96)
    _, s0 = moe.mlp_fwd_fp8_tensor(x, idx, p, W1, W2, z_amax_in=1.0)
    g0 = moe.mlp_bwd_fp8_tensor(dy, s0, dgu_amax_in=1.0)
    y, s = moe.mlp_fwd_fp8_tensor(x, idx, p, W1, W2, z_amax_in=s0["z_amax"])
    g = moe.mlp_bwd_fp8_tensor(dy, s, dgu_amax_in=g0["dgu_amax"])
    yu, su = moe.mlp_fwd(x, idx, p, W1, W2, quant=False)
    gu = moe.mlp_bwd(dy, su, p, W1, W2, quant=False)
    rel = lambda a, b: np.linalg.norm(a - b) / np.linalg.norm(b)  # noqa: E731
    assert rel(y, yu) < 0.1
    for n in ("dx", "dW1", "dW2", "dprobs"):
        assert rel(g[n], gu[n]) < 0.2, n
    # the recorded largest magnitudes are those of the unquantised-scale Z and dGU of the step
    assert s["z_amax"] == s0["z_amax"]
    Z = moe.silu(s["G"]) * s["U"] * s["p_row"][:, None]
    assert s["z_amax"] == np.abs(Z).max()
