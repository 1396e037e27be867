"""Pins for the oracle's routing, grouped GEMMs and MLP forward/backward (CPU only).

Grouping tokens by per-expert counts must not change the result of running each
expert on its own tokens ("MoE-Training für biologische Grundmodelle optimieren",
hyper.ai/de, GroupedLinear passage); the fused gate-up / ScaledSwiGLU / routing-scale
step has a forward and a backward (same page, GroupedMLP passage). These tests pin
the oracle against brute force, closed forms and finite differences."""
import itertools
import math

import numpy as np
import pytest
import torch

import moe_workloads as wl
from oracle import moe, mxfp8


def _tiny(T=8, H=32, F=32, E=3, k=2, seed=11, routing="softmax"):
    cfg = wl.custom(T=T, H=H, F=F, E=E, k=k, seed=seed, routing=routing)
    d = wl.make_all(cfg)
    return cfg, {n: (v.double().numpy() if isinstance(v, torch.Tensor) and v.is_floating_point()
                     else (v.numpy() if isinstance(v, torch.Tensor) else v)) for n, v in d.items()}


# ----------------------------------------------------------------------------- routing

def _route_brute(idx, E, align):
    T, k = idx.shape
    pairs = sorted((int(idx[t, j]), t, j) for t in range(T) for j in range(k))
    m = [sum(1 for p in pairs if p[0] == e) for e in range(E)]
    off = [0]
    for e in range(E):
        off.append(off[-1] + (m[e] + align - 1) // align * align)
    ros = {}
    cnt = [0] * E
    for e, t, j in pairs:
        ros[(t, j)] = off[e] + cnt[e]
        cnt[e] += 1
    return m, off, ros


@pytest.mark.parametrize("align", [32, 128])
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_route_matches_brute_force(seed, align):
    rng = np.random.default_rng(seed)
    T, E, k = 37, 5, 2
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)])
    r = moe.route(idx, E, align)
    m, off, ros = _route_brute(idx, E, align)
    assert r["m_splits"].tolist() == m
    assert r["seg_off"].tolist() == off
    for (t, j), row in ros.items():
        assert r["row_of_slot"][t, j] == row
        assert r["token_of_row"][row] == t
        assert r["slot_of_row"][row] == j
    live = r["token_of_row"] >= 0
    assert live.sum() == T * k


def test_route_invariants_and_empty_expert():
    cfg, d = _tiny(T=64, E=6, k=2, routing="dead_last")
    r = moe.route(d["topk_idx"], cfg.E, 32)
    assert r["m_splits"].sum() == cfg.T * cfg.k
    assert r["m_splits"][cfg.E - 1] == 0
    assert r["seg_off"][cfg.E] == r["seg_off"][cfg.E - 1]        # empty segment
    rows = r["row_of_slot"].reshape(-1)
    assert len(set(rows.tolist())) == rows.size                  # injective
    for t in range(cfg.T):
        for j in range(cfg.k):
            assert r["token_of_row"][r["row_of_slot"][t, j]] == t
    # within each segment, tokens strictly increase (stable by token)
    for e in range(cfg.E):
        seg = r["token_of_row"][r["seg_off"][e]:r["seg_off"][e] + r["m_splits"][e]]
        assert np.all(np.diff(seg) > 0)


def test_route_rejects_bad_ids():
    with pytest.raises(ValueError):
        moe.route(np.array([[0, 0]]), 3)
    with pytest.raises(ValueError):
        moe.route(np.array([[0, 3]]), 3)


# ----------------------------------------------------------------------------- SwiGLU

def test_silu_closed_forms():
    assert moe.silu(0.0) == 0.0
    assert moe.dsilu(0.0) == 0.5
    assert abs(moe.silu(1.0) - 1.0 / (1.0 + math.exp(-1.0))) < 1e-15
    assert abs(moe.silu(-2.0) - (-2.0) / (1.0 + math.exp(2.0))) < 1e-15
    assert abs(moe.silu(40.0) - 40.0) < 1e-12
    assert abs(moe.silu(-40.0)) < 1e-15
    # derivative against a central difference of silu
    for g in [-3.0, -0.7, 0.2, 1.5, 4.0]:
        h = 1e-6
        fd = (moe.silu(g + h) - moe.silu(g - h)) / (2 * h)
        assert abs(fd - moe.dsilu(g)) < 1e-9


# ----------------------------------------------------------------------------- grouped GEMMs

def test_grouped_gemm_integer_operands_exact():
    """Small integers are exact in MXFP8 (|v| <= 4 -> scaled values are multiples of 64
    below 256), so the grouped GEMM of quantised operands equals the int64 product."""
    rng = np.random.default_rng(3)
    E, N, K = 3, 8, 64
    idx = np.stack([rng.permutation(E)[:2] for _ in range(20)])
    r = moe.route(idx, E, 32)
    A = rng.integers(-4, 5, (r["Mp"], K)).astype(np.float64)
    A[r["token_of_row"] < 0] = 0
    B = rng.integers(-4, 5, (E, N, K)).astype(np.float64)
    Aq = mxfp8.fake_quant_rowwise(A)
    Bq = np.stack([mxfp8.fake_quant_rowwise(B[e]) for e in range(E)])
    np.testing.assert_array_equal(Aq, A)
    np.testing.assert_array_equal(Bq, B)
    C = moe.grouped_gemm(Aq, Bq, r["seg_off"])
    Ai, Bi = A.astype(np.int64), B.astype(np.int64)
    for e in range(E):
        s0, s1 = r["seg_off"][e], r["seg_off"][e + 1]
        np.testing.assert_array_equal(C[s0:s1], Ai[s0:s1] @ Bi[e].T)


def test_grouped_wgrad_per_expert_and_empty():
    rng = np.random.default_rng(4)
    E = 3
    seg_off = np.array([0, 64, 64, 96])         # expert 1 empty
    At = rng.standard_normal((5, 96))
    Bt = rng.standard_normal((7, 96))
    C = moe.grouped_gemm_wgrad(At, Bt, seg_off)
    assert C.shape == (E, 5, 7)
    np.testing.assert_array_equal(C[1], 0)
    for e in (0, 2):
        s0, s1 = seg_off[e], seg_off[e + 1]
        want = np.einsum("nm,km->nk", At[:, s0:s1], Bt[:, s0:s1])
        np.testing.assert_allclose(C[e], want, rtol=1e-12, atol=1e-12)


# ----------------------------------------------------------------------------- MLP forward

@pytest.mark.parametrize("quant", [True, False])
def test_forward_grouped_equals_per_token_loop(quant):
    cfg, d = _tiny(T=24, H=64, F=64, E=4, k=2, seed=5)
    y, _ = moe.mlp_fwd(d["x"], d["topk_idx"], d["probs"], d["W1"], d["W2"], quant=quant)
    y_ref = moe.mlp_per_token(d["x"], d["topk_idx"], d["probs"], d["W1"], d["W2"], quant=quant)
    np.testing.assert_allclose(y, y_ref, rtol=1e-11, atol=1e-13)


def test_forward_alignment_invariant():
    cfg, d = _tiny(T=40, H=64, F=96, E=3, k=2, seed=6)
    y32, s32 = moe.mlp_fwd(d["x"], d["topk_idx"], d["probs"], d["W1"], d["W2"], align=32)
    y128, s128 = moe.mlp_fwd(d["x"], d["topk_idx"], d["probs"], d["W1"], d["W2"], align=128)
    np.testing.assert_array_equal(y32, y128)
    g32 = moe.mlp_bwd(d["dy"], s32, d["probs"], d["W1"], d["W2"])
    g128 = moe.mlp_bwd(d["dy"], s128, d["probs"], d["W1"], d["W2"])
    for n in ("dx", "dW1", "dW2", "dprobs"):
        np.testing.assert_array_equal(g32[n], g128[n])


def test_dense_reduction_k1_e1():
    """E = 1, k = 1, p = 1, quantisation off: the layer is a textbook SwiGLU MLP."""
    rng = np.random.default_rng(7)
    T, H, F = 10, 32, 64
    x = rng.standard_normal((T, H))
    W1 = rng.standard_normal((1, 2 * F, H)) * 0.1
    W2 = rng.standard_normal((1, H, F)) * 0.1
    idx = np.zeros((T, 1), dtype=np.int64)
    p = np.ones((T, 1))
    y, _ = moe.mlp_fwd(x, idx, p, W1, W2, quant=False)
    g = x @ W1[0, :F].T
    u = x @ W1[0, F:].T
    want = ((g / (1 + np.exp(-g))) * u) @ W2[0].T
    np.testing.assert_allclose(y, want, rtol=1e-12, atol=1e-12)


def test_empty_expert_contributes_nothing():
    cfg, d = _tiny(T=32, H=64, F=64, E=4, k=2, seed=8, routing="dead_last")
    y, saved = moe.mlp_fwd(d["x"], d["topk_idx"], d["probs"], d["W1"], d["W2"])
    W1b, W2b = d["W1"].copy(), d["W2"].copy()
    W1b[cfg.E - 1] *= -3.0
    W2b[cfg.E - 1] += 1.0
    y2, _ = moe.mlp_fwd(d["x"], d["topk_idx"], d["probs"], W1b, W2b)
    np.testing.assert_array_equal(y, y2)
    g = moe.mlp_bwd(d["dy"], saved, d["probs"], d["W1"], d["W2"])
    assert np.all(g["dW1"][cfg.E - 1] == 0) and np.all(g["dW2"][cfg.E - 1] == 0)


def test_probability_scales_linearly():
    """Z carries p as a factor, so with quantisation off y is linear in each token's p."""
    cfg, d = _tiny(T=6, H=32, F=32, E=3, k=2, seed=9)
    y1, _ = moe.mlp_fwd(d["x"], d["topk_idx"], d["probs"], d["W1"], d["W2"], quant=False)
    p2 = d["probs"].copy()
    p2[:, 1] = 0.0
    y2, _ = moe.mlp_fwd(d["x"], d["topk_idx"], p2, d["W1"], d["W2"], quant=False)
    p3 = d["probs"].copy()
    p3[:, 1] *= 2.0
    y3, _ = moe.mlp_fwd(d["x"], d["topk_idx"], p3, d["W1"], d["W2"], quant=False)
    np.testing.assert_allclose(y3 - y1, y1 - y2, rtol=1e-10, atol=1e-12)


# ----------------------------------------------------------------------------- MLP backward

def _loss(x, probs, W1, W2, idx, dy):
    y, _ = moe.mlp_fwd(x, idx, probs, W1, W2, quant=False)
    return float(np.sum(y * dy))


@pytest.mark.parametrize("which", ["x", "probs", "W1", "W2"])
def test_backward_finite_differences(which):
    """Central differences in fp64 with quantisation off (the quantiser is piecewise
    constant, so differences through it say nothing)."""
    cfg, d = _tiny(T=8, H=32, F=32, E=3, k=2, seed=10)
    x, probs, W1, W2, idx, dy = d["x"], d["probs"], d["W1"], d["W2"], d["topk_idx"], d["dy"]
    _, saved = moe.mlp_fwd(x, idx, probs, W1, W2, quant=False)
    g = moe.mlp_bwd(dy, saved, probs, W1, W2, quant=False)
    ana = {"x": g["dx"], "probs": g["dprobs"], "W1": g["dW1"], "W2": g["dW2"]}[which]
    arrs = {"x": x, "probs": probs, "W1": W1, "W2": W2}
    base = arrs[which]
    rng = np.random.default_rng(0)
    flat = list(itertools.product(*[range(s) for s in base.shape]))
    picks = [flat[i] for i in rng.choice(len(flat), size=min(60, len(flat)), replace=False)]
    h = 1e-6
    num = []
    for pos in picks:
        a = {n: v.copy() for n, v in arrs.items()}
        a[which][pos] += h
        lp = _loss(a["x"], a["probs"], a["W1"], a["W2"], idx, dy)
        a[which][pos] -= 2 * h
        lm = _loss(a["x"], a["probs"], a["W1"], a["W2"], idx, dy)
        num.append((lp - lm) / (2 * h))
    num = np.array(num)
    an = np.array([ana[p] for p in picks])
    err = np.linalg.norm(num - an) / np.linalg.norm(an)
    assert err <= 1e-6, err


def test_quantised_backward_close_to_unquantised():
    """With MXFP8 on, gradients stay within a few percent of the unquantised ones
    (information: E4M3 keeps 3 mantissa bits)."""
    cfg, d = _tiny(T=64, H=64, F=64, E=3, k=2, seed=12)
    outs = {}
    for q in (True, False):
        _, saved = moe.mlp_fwd(d["x"], d["topk_idx"], d["probs"], d["W1"], d["W2"], quant=q)
        outs[q] = moe.mlp_bwd(d["dy"], saved, d["probs"], d["W1"], d["W2"], quant=q)
    for n in ("dx", "dW1", "dW2", "dprobs"):
        a, b = outs[True][n], outs[False][n]
        rel = np.linalg.norm(a - b) / np.linalg.norm(b)
        assert rel < 0.15, (n, rel)


def test_colwise_blocks_restart_at_segments():
    """A large value in an expert's first row must not change the scales of the
    previous expert's last block."""
    rng = np.random.default_rng(13)
    seg_off = np.array([0, 64, 128])
    m = np.array([40, 50])
    a = rng.standard_normal((128, 32))
    a[40:64] = 0
    a[114:128] = 0
    c1, s1 = moe.quantize_colwise_segments(a, seg_off, m)
    a2 = a.copy()
    a2[64] *= 1e6
    c2, s2 = moe.quantize_colwise_segments(a2, seg_off, m)
    np.testing.assert_array_equal(s1[:, :2], s2[:, :2])
    np.testing.assert_array_equal(c1[:, :64], c2[:, :64])
    assert np.any(s1[:, 2] != s2[:, 2])


def test_e5m2_gradients_variant():
    """Gradients in E5M2 (one mantissa bit fewer than E4M3): the backward stays close to the
    unquantised one, further from it than the all-E4M3 backward; the forward is unchanged
    and only the gradient outputs move."""
    cfg = wl.custom("e5", T=96, H=64, F=64, E=3, k=2, seed=9)
    d = wl.make_all(cfg)
    x, W1, W2, p = (d[n].double().numpy() for n in ("x", "W1", "W2", "probs"))
    idx, dy = d["topk_idx"].numpy(), d["dy"].double().numpy()
    _, sq = moe.mlp_fwd(x, idx, p, W1, W2)
    _, su = moe.mlp_fwd(x, idx, p, W1, W2, quant=False)
    g4 = moe.mlp_bwd(dy, sq, p, W1, W2)
    g5 = moe.mlp_bwd(dy, sq, p, W1, W2, grad_fmt="e5m2")
    gu = moe.mlp_bwd(dy, su, p, W1, W2, quant=False)
    rel = lambda a, b: np.linalg.norm(a - b) / np.linalg.norm(b)  # noqa: E731
    for n in ("dx", "dW1", "dW2"):
        assert rel(g5[n], gu[n]) < 0.15, n
        assert rel(g5[n], gu[n]) > rel(g4[n], gu[n]), n
    # dZ = dYq . W2q: only dY's format changed between the two
    assert not np.array_equal(g5["dZ"], g4["dZ"])


def test_ceil_scale_rule_variant():
    """The round-up scale rule changes only the blocks whose amax the OCP rule would
    saturate: the layer stays close to the unquantised one, and a block-wise comparison of
    the two rules' quantised inputs differs exactly where the OCP exponent is one lower."""
    cfg = wl.custom("ce", T=96, H=64, F=64, E=3, k=2, seed=10)
    d = wl.make_all(cfg)
    x, W1, W2, p = (d[n].double().numpy() for n in ("x", "W1", "W2", "probs"))
    idx, dy = d["topk_idx"].numpy(), d["dy"].double().numpy()
    yc, sc = moe.mlp_fwd(x, idx, p, W1, W2, scale_rule="ceil")
    yu, su = moe.mlp_fwd(x, idx, p, W1, W2, quant=False)
    gc = moe.mlp_bwd(dy, sc, p, W1, W2)
    gu = moe.mlp_bwd(dy, su, p, W1, W2, quant=False)
    rel = lambda a, b: np.linalg.norm(a - b) / np.linalg.norm(b)  # noqa: E731
    assert rel(yc, yu) < 0.1
    for n in ("dx", "dW1", "dW2", "dprobs"):
        assert rel(gc[n], gu[n]) < 0.15, n
    blocks = x.reshape(-1, 32)
    _, s_ocp = mxfp8.quantize_blocks(blocks)
    _, s_ceil = mxfp8.quantize_blocks(blocks, "e4m3", "ceil")
    amax = np.abs(blocks).max(axis=1)
    saturating = amax > 448.0 * np.exp2(s_ocp.astype(float) - 127)
    assert np.array_equal(s_ceil.astype(int) - s_ocp.astype(int), saturating.astype(int))
    assert saturating.any() and not saturating.all()


# ----------------------------------------------------------------------------- quantised backward pin

def _pin_problem():
    # H != F and 2F != H, so a transposed operand cannot pass for the right one; ragged
    # experts (about 47 rows each: a short last block of rows) and one expert with no tokens
    cfg = wl.custom("pin", T=70, H=64, F=96, E=4, k=2, seed=21, routing="dead_last")
    d = wl.make_all(cfg)
    x, W1, W2, p = (d[n].double().numpy() for n in ("x", "W1", "W2", "probs"))
    return cfg, x, W1, W2, p, d["topk_idx"].numpy(), d["dy"].double().numpy()


def _assert_same_grads(got, want, rtol=1e-11):
    for n in ("dx", "dW1", "dW2", "dprobs"):
        scale = np.max(np.abs(want[n]))
        np.testing.assert_allclose(got[n], want[n], rtol=rtol, atol=rtol * scale, err_msg=n)


@pytest.mark.parametrize("grad_fmt", ["e4m3", "e5m2"])
@pytest.mark.parametrize("rule", ["ocp", "ceil"])
def test_quantised_backward_equals_per_expert_restatement(grad_fmt, rule):
    """The grouped, padded backward equals the expert-by-expert restatement in which each
    backward GEMM quantises its two operands along its own contraction index (up to the
    order of fp64 sums)."""
    cfg, x, W1, W2, p, idx, dy = _pin_problem()
    m = moe.route(idx, cfg.E)["m_splits"]
    assert m[cfg.E - 1] == 0 and np.any(m % 32 != 0) and np.all(m[:-1] > 32)
    _, saved = moe.mlp_fwd(x, idx, p, W1, W2, scale_rule=rule)
    g = moe.mlp_bwd(dy, saved, p, W1, W2, grad_fmt=grad_fmt)
    ge = moe.mlp_bwd_per_expert(x, dy, idx, p, W1, W2, grad_fmt=grad_fmt, scale_rule=rule)
    _assert_same_grads(g, ge)
    assert np.all(ge["dW1"][cfg.E - 1] == 0) and np.all(ge["dW2"][cfg.E - 1] == 0)


def test_fake_quant_along_matches_blockwise_definition():
    """The restatement's block loop against the hand-built definition on one column: a
    short last block takes its scale over its own entries only."""
    a = np.zeros((40, 1))
    a[:32, 0] = 1.0
    a[5, 0] = 3.0           # first block: amax 3 -> scale 2^(1-8)
    a[32:, 0] = 0.0
    a[35, 0] = 0.75         # short block of 8: amax 0.75 -> its own scale, value exact
    a[36, 0] = 0.3          # 0.3 * 2^9 = 153.6; E4M3 steps by 16 in [128, 256) -> 160
    out = moe._fake_quant_along(a, 0)
    assert out[5, 0] == 3.0 and out[0, 0] == 1.0
    assert out[35, 0] == 0.75
    assert out[36, 0] == 160.0 * 2.0 ** -9
    np.testing.assert_array_equal(moe._fake_quant_along(a.T, 1), out.T)


def _mutated(monkeypatch, helper, call, replacement):
    """Replace call number ``call`` (0-based) of oracle helper ``helper`` inside the
    backward by ``replacement``; all other calls pass through."""
    orig = getattr(moe, helper)
    n = {"i": 0}

    def patched(*a, **kw):
        i = n["i"]
        n["i"] += 1
        return replacement(*a, **kw) if i in call else orig(*a, **kw)

    monkeypatch.setattr(moe, helper, patched)


def _rowwise(a, quant, fmt="e4m3", rule="ocp"):
    return mxfp8.fake_quant_rowwise(a, fmt, rule)


def _rowwise_seg(a, r, quant, fmt="e4m3", rule="ocp"):
    return mxfp8.fake_quant_rowwise(a, fmt, rule)


def _colwise(a, quant, fmt="e4m3", rule="ocp"):
    return mxfp8.fake_quant_colwise(a, fmt, rule)


# (helper, calls to replace, replacement): every operand of the four backward GEMMs given
# the other block direction. In the backward, _fq_row is called for dY then dGU;
# _fq_col_seg for dY, dGU, Z, Xp; _fq_col for W2[0..E) then W1[0..E).
_E_PIN = 4
MUTATIONS = {
    "fc2_dgrad_dY_colwise": ("_fq_row", {0}, _colwise),
    "fc1_dgrad_dGU_colwise": ("_fq_row", {1}, _colwise),
    "fc2_wgrad_dY_rowwise": ("_fq_col_seg", {0}, _rowwise_seg),
    "fc1_wgrad_dGU_rowwise": ("_fq_col_seg", {1}, _rowwise_seg),
    "fc2_wgrad_Z_rowwise": ("_fq_col_seg", {2}, _rowwise_seg),
    "fc1_wgrad_Xp_rowwise": ("_fq_col_seg", {3}, _rowwise_seg),
    "fc2_dgrad_W2_rowwise": ("_fq_col", set(range(_E_PIN)), lambda a, quant, rule="ocp": _rowwise(a, quant, "e4m3", rule)),
    "fc1_dgrad_W1_rowwise": ("_fq_col", set(range(_E_PIN, 2 * _E_PIN)),
                             lambda a, quant, rule="ocp": _rowwise(a, quant, "e4m3", rule)),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_per_expert_pin_catches_swapped_block_direction(monkeypatch, name):
    """A mistake planted in the oracle's backward -- one operand quantised with blocks
    along the wrong index -- makes it disagree with the restatement."""
    cfg, x, W1, W2, p, idx, dy = _pin_problem()
    assert cfg.E == _E_PIN
    _, saved = moe.mlp_fwd(x, idx, p, W1, W2)
    ge = moe.mlp_bwd_per_expert(x, dy, idx, p, W1, W2)
    helper, calls, repl = MUTATIONS[name]
    _mutated(monkeypatch, helper, calls, repl)
    g = moe.mlp_bwd(dy, saved, p, W1, W2)
    with pytest.raises(AssertionError):
        _assert_same_grads(g, ge)
