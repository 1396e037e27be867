"""Full-size parity of the fused layer (the launch configuration bench.py times) on the
workloads the oracle cannot run whole: Mixtral (8192 tokens, hidden 4096, FFN 14336, 8
experts, top-2), its Zipf-routed variant (one expert with 40 tokens) and the genomics
shape (32768 tokens, hidden 2048, FFN 5632, 64 experts, top-8).

The oracle quantises about a million values per second, so it cannot quantise a whole
expert's weights here; it checks what it can compute one value at a time:
  * routing maps (m_splits, segment offsets, row_of_slot, token_of_row, prob_of_row):
    bit-exact, whole arrays;
  * sampled MXFP8 blocks of every quantised copy -- the four weight copies (incl. the
    W1 gate/up interleave) and the saved colwise copy of the permuted activations:
    codes and scales bit-exact;
  * sampled gate/up entries (saved bf16): one quantised activation row times one
    quantised W1 row, rel. L2 <= 5e-3 (the GEMM-stage bar);
  * sampled colwise blocks of the saved MXFP8 Z = silu(G) * U * p over 32 rows of one
    expert, dequantised, rel. L2 <= 2e-2;
  * sampled fc2 weight-gradient entries dW2[e][h, f] over a whole expert's rows (its
    quantised activations, Z column and dY column), rel. L2 <= 5e-3.
The layer's own outputs, against the oracle's definition at the end-to-end bar (rel. L2
<= 2e-2, the same bar as the tiny and small workloads, where they are compared whole):
  * y[t, h] and dX[t, h] for sampled tokens and 128 sampled columns h, and dprobs[t, :],
    over tokens whose experts all lie in a small set S (two experts for the Mixtral shapes,
    the eight experts of one token for genomics): the oracle quantises the whole fc1
    weights (rowwise) and fc2 weights (colwise) of each expert in S -- the only parts
    that need a whole expert -- on a spawn-started process pool;
  * dW1[e][f, h] entries over a whole expert's rows (the fc1 weight gradient: colwise
    dGU column times colwise x column, dGU rebuilt from the quantised dY rows, the
    colwise W2 column and the gate / up entries of every row)."""
import concurrent.futures as cf
import multiprocessing as mp

import numpy as np
import pytest
import torch

import moe_workloads as wl
from oracle import moe as omoe
from oracle import mxfp8 as omx
from tests.util import f64, rel_l2, u8, SEG_ALIGN

pytestmark = pytest.mark.gpu
NSAMP = 24
TOL_E2E = 2e-2
NCOLS = 128          # sampled output columns of y and dX
NTOK = 16            # sampled tokens (at most)
CHUNK = 2048         # rows per oracle quantiser task


@pytest.fixture(scope="module")
def oracle_pool():
    with cf.ProcessPoolExecutor(max_workers=min(8, mp.cpu_count()), mp_context=mp.get_context("spawn")) as ex:
        yield ex


def _fq_rows_pooled(pool, a):
    """Oracle rowwise fake quantisation of a large fp64 matrix, CHUNK rows per task (the
    blocks lie within rows, so the split changes nothing)."""
    from tests import _oracle_pool
    parts = list(pool.map(_oracle_pool.fake_quant_rows, [a[i:i + CHUNK] for i in range(0, a.shape[0], CHUNK)]))
    return np.concatenate(parts, axis=0)


def _fq_vec(v):
    """Oracle MXFP8 of one 32-value block (as a 1 x 32 row): (codes, scale, dequantised)."""
    q, s = omx.quantize_rowwise(np.asarray(v, dtype=np.float64)[None, :])
    return q[0], int(s[0, 0]), omx.dequantize_rowwise(q, s)[0]


def _mx(data, sf, rows, cols, mx):
    return mx.MXFP8(data.view(rows, cols), sf, mx.SCALE_MMA)


def _run(gpu_lib, cfg):
    dev = "cuda"
    idx, probs = wl.make_routing(cfg)
    x, dy = wl.make_activations(cfg), wl.make_grad_output(cfg)
    W1, W2 = wl.make_weights_on(cfg, dev)
    layer = gpu_lib.GroupedMLP(cfg.T, cfg.k, cfg.E, cfg.H, cfg.F, device=dev)
    gpu_lib.mxmoe_clear_device_status()
    layer.quantize_weights(W1, W2)
    y = layer.forward(x.cuda(), idx.cuda(), probs.cuda())
    dx, dW1, dW2, dprobs = layer.backward(dy.cuda())
    torch.cuda.synchronize()
    st, where = gpu_lib.mxmoe_get_device_status()
    assert st == 0, (st, where)
    for t in (y, dx, dW1, dW2, dprobs):
        assert torch.isfinite(t).all()
    return idx, probs, x, dy, W1, W2, layer, (y, dx, dW1, dW2, dprobs)


def _expert_choice(cfg, r):
    if cfg.name == "mixtral_zipf":  # the 40-token expert and the largest one
        return [int(np.argmin(r["m_splits"])), int(np.argmax(r["m_splits"]))]
    return [0]


@pytest.mark.parametrize("name", ["mixtral", "mixtral_zipf", "genomics"])
def test_fullsize_sampled_parity(gpu_lib, oracle_pool, name):
    cfg = wl.CONFIGS[name]
    E, H, F, T, k = cfg.E, cfg.H, cfg.F, cfg.T, cfg.k
    idx, probs, x, dy, W1, W2, layer, outs = _run(gpu_lib, cfg)
    dW2 = outs[3]
    rng = np.random.default_rng(cfg.seed)
    cap = layer.cap
    mx = gpu_lib

    # ---- routing: bit-exact
    r = omoe.route(idx.numpy(), E, align=SEG_ALIGN)
    seg = r["seg_off"]
    np.testing.assert_array_equal(layer.saved_field("m_splits", torch.int32, E).cpu().numpy(), r["m_splits"])
    np.testing.assert_array_equal(layer.saved_field("seg_off", torch.int32, E + 1).cpu().numpy(), seg)
    np.testing.assert_array_equal(layer.saved_field("row_of_slot", torch.int32, T * k).cpu().numpy(),
                                  r["row_of_slot"].reshape(-1))
    tor = layer.saved_field("token_of_row", torch.int32, cap).cpu().numpy()
    np.testing.assert_array_equal(tor[:r["Mp"]], r["token_of_row"])
    por = layer.saved_field("prob_of_row", torch.float32, cap).cpu().numpy()
    live = r["token_of_row"] >= 0
    want_p = probs.numpy()[r["token_of_row"][live], r["slot_of_row"][live]]
    np.testing.assert_array_equal(por[:r["Mp"]][live], want_p)

    # ---- weight copies: sampled blocks bit-exact
    views = [mx.mxmoe_weights_view(layer.wq, E, H, F, w) for w in range(4)]
    codes = [u8(v.data) for v in views]
    scales = [u8(v.scale_plain()) for v in views]
    experts = _expert_choice(cfg, r)
    for e in experts:
        w1 = W1[e].float().cpu().numpy()
        w2 = W2[e].float().cpu().numpy()
        for _ in range(NSAMP):
            f, kb = int(rng.integers(2 * F)), int(rng.integers(H // 32))
            hf, rr = int(f >= F), f - int(f >= F) * F
            dst = e * 2 * F + (rr // 64) * 128 + hf * 64 + rr % 64  # gate/up interleave
            q, s, _ = _fq_vec(w1[f, 32 * kb:32 * kb + 32])
            np.testing.assert_array_equal(codes[0][dst, 32 * kb:32 * kb + 32], q)
            assert scales[0][dst, kb] == s
            h, fb = int(rng.integers(H)), int(rng.integers(2 * F // 32))
            q, s, _ = _fq_vec(w1[32 * fb:32 * fb + 32, h])
            np.testing.assert_array_equal(codes[1][e * H + h, 32 * fb:32 * fb + 32], q)
            assert scales[1][e * H + h, fb] == s
            h, fb = int(rng.integers(H)), int(rng.integers(F // 32))
            q, s, _ = _fq_vec(w2[h, 32 * fb:32 * fb + 32])
            np.testing.assert_array_equal(codes[2][e * H + h, 32 * fb:32 * fb + 32], q)
            assert scales[2][e * H + h, fb] == s
            f2, hb = int(rng.integers(F)), int(rng.integers(H // 32))
            q, s, _ = _fq_vec(w2[32 * hb:32 * hb + 32, f2])
            np.testing.assert_array_equal(codes[3][e * F + f2, 32 * hb:32 * hb + 32], q)
            assert scales[3][e * F + f2, hb] == s

    # ---- saved colwise copies and gate/up
    xcol = _mx(layer.saved_field("x_colT", torch.uint8, H * cap), layer.saved_field("x_colT_sf", torch.uint8,
               H * cap // 32), H, cap, mx)
    zcol = _mx(layer.saved_field("z_colT", torch.uint8, F * cap), layer.saved_field("z_colT_sf", torch.uint8,
               F * cap // 32), F, cap, mx)
    xc_codes, xc_sc = u8(xcol.data), u8(xcol.scale_plain())
    zc_codes, zc_sc = u8(zcol.data), u8(zcol.scale_plain())
    gu = f64(layer.saved_field("gu", torch.bfloat16, cap * 2 * F).view(cap, 2 * F))
    xf = f64(x)
    dyf = f64(dy)
    gu_got, gu_want, z_got, z_want, dw_got, dw_want = [], [], [], [], [], []
    for e in experts:
        s0, m = int(seg[e]), int(r["m_splits"][e])
        nblk = (m + 31) // 32
        w1 = W1[e].float().cpu().numpy().astype(np.float64)
        w2 = W2[e].float().cpu().numpy().astype(np.float64)
        rows = np.arange(s0, s0 + 32 * nblk)
        toks = r["token_of_row"][rows]
        xp = np.zeros((len(rows), H))
        xp[toks >= 0] = xf[toks[toks >= 0]]
        # x colT blocks
        for _ in range(NSAMP):
            h, b = int(rng.integers(H)), int(rng.integers(nblk))
            q, s, _ = _fq_vec(xp[32 * b:32 * b + 32, h])
            np.testing.assert_array_equal(xc_codes[h, s0 + 32 * b:s0 + 32 * b + 32], q)
            assert xc_sc[h, (s0 + 32 * b) // 32] == s
        # quantised activation rows of this expert (the fc1 operand) -- the expensive part
        xq = omx.fake_quant_rowwise(xp)
        p_row = np.zeros(len(rows))
        p_row[toks >= 0] = por[rows[toks >= 0]]
        fs = rng.integers(F, size=4)
        for f in fs:
            wg = omx.fake_quant_rowwise(w1[f][None])[0]
            wu = omx.fake_quant_rowwise(w1[F + f][None])[0]
            g_col, u_col = xq @ wg, xq @ wu                     # fp64 gate / up over the expert's rows
            for i in rng.integers(m, size=NSAMP // 4):
                gu_got += [gu[s0 + i, f], gu[s0 + i, F + f]]
                gu_want += [g_col[i], u_col[i]]
            z_col = omoe.silu(g_col) * u_col * p_row           # pad rows: p = 0
            for b in range(min(nblk, 4)):
                _, _, zd = _fq_vec(z_col[32 * b:32 * b + 32])
                z_got.append(omx.dequantize_rowwise(zc_codes[f:f + 1, s0 + 32 * b:s0 + 32 * b + 32],
                                                    zc_sc[f:f + 1, (s0 + 32 * b) // 32:(s0 + 32 * b) // 32 + 1])[0])
                z_want.append(zd)
            # dW2[e][h, f] = sum over the expert's rows of colwise-quantised dY[:, h] * Z[:, f]
            zq = np.concatenate([_fq_vec(z_col[32 * b:32 * b + 32])[2] for b in range(nblk)])
            for h in rng.integers(H, size=4):
                dyp = np.zeros(len(rows))
                dyp[toks >= 0] = dyf[toks[toks >= 0], h]
                dq = np.concatenate([_fq_vec(dyp[32 * b:32 * b + 32])[2] for b in range(nblk)])
                dw_want.append(float(dq @ zq))
                dw_got.append(float(dW2[e, h, f]))
        del w2
    assert rel_l2(np.array(gu_got), np.array(gu_want)) <= 5e-3
    assert rel_l2(np.concatenate(z_got), np.concatenate(z_want)) <= 2e-2
    assert rel_l2(np.array(dw_got), np.array(dw_want)) <= 5e-3
    _check_layer_outputs(cfg, r, idx.numpy(), probs.numpy(), xf, dyf, W1, W2, outs, experts, rng, oracle_pool)


def _expert_set(cfg, idx, experts):
    """A small set S of experts and the sampled tokens whose experts all lie in S."""
    if cfg.k == 2:
        S = sorted(set(experts) | ({1} if experts == [0] else set()))
    else:   # top-8 of 64: the experts of the first token routed to expert experts[0]
        t0 = int(np.nonzero((idx == experts[0]).any(axis=1))[0][0])
        S = sorted(set(idx[t0].tolist()))
    inside = np.nonzero(np.isin(idx, S).all(axis=1))[0]
    assert len(inside) > 0
    return S, inside[:NTOK]


def _check_layer_outputs(cfg, r, idx, probs, xf, dyf, W1, W2, outs, experts, rng, pool):
    """y, dprobs, dX on sampled tokens and columns, dW1 entries over one expert's rows,
    from the oracle's definition (fp64 over MXFP8-dequantised operands, blocks along each
    GEMM's contraction index), rel. L2 <= 2e-2."""
    H, F = cfg.H, cfg.F
    y, dx, dW1 = outs[0], outs[1], outs[2]
    dprobs = outs[4]
    S, toks = _expert_set(cfg, idx, experts)
    hs = np.sort(rng.choice(H, size=NCOLS, replace=False))
    y_want = np.zeros((len(toks), NCOLS))
    dx_want = np.zeros((len(toks), NCOLS))
    dp_want = np.zeros((len(toks), cfg.k))
    xq = _fq_rows_pooled(pool, xf[toks])                          # fc1 operand rows (blocks along H)
    dyq = _fq_rows_pooled(pool, dyf[toks])                        # fc2 data-gradient operand rows
    dw1_got, dw1_want = [], []
    for e in S:
        w1 = f64(W1[e])                                            # [2F, H]
        w2 = f64(W2[e])                                            # [H, F]
        w1q_row = _fq_rows_pooled(pool, w1)                        # blocks along H
        w2q_colT = _fq_rows_pooled(pool, np.ascontiguousarray(w2.T))   # [F, H], blocks along H
        w2q_row_h = omx.fake_quant_rowwise(w2[hs])                 # rows h of W2, blocks along F
        w1q_col_h = omx.fake_quant_rowwise(np.ascontiguousarray(w1[:, hs].T))   # [NCOLS, 2F], blocks along 2F
        for i, t in enumerate(toks):
            for j in range(cfg.k):
                if idx[t, j] != e:
                    continue
                p = float(probs[t, j])
                gu = w1q_row @ xq[i]
                g_, u_ = gu[:F], gu[F:]
                a_ = omoe.silu(g_) * u_
                zq = omx.fake_quant_rowwise((a_ * p)[None])[0]
                y_want[i] += w2q_row_h @ zq
                dz = w2q_colT @ dyq[i]
                dp_want[i, j] = float(np.sum(dz * a_))
                da = dz * p
                dgu = np.concatenate([da * u_ * omoe.dsilu(g_), da * omoe.silu(g_)])
                dx_want[i] += w1q_col_h @ omx.fake_quant_rowwise(dgu[None])[0]
        if e == S[0] or e in experts[:1]:
            dw1_got, dw1_want = _dw1_entries(cfg, r, e, probs, xf, dyf, w1q_row, w2q_colT, dW1, rng, pool,
                                             dw1_got, dw1_want)
        del w1, w2, w1q_row, w2q_colT
    assert len(dw1_want) > 0
    errs = dict(y=rel_l2(f64(y)[toks][:, hs], y_want), dx=rel_l2(f64(dx)[toks][:, hs], dx_want),
                dprobs=rel_l2(f64(dprobs)[toks], dp_want), dW1=rel_l2(np.array(dw1_got), np.array(dw1_want)))
    print(cfg.name, "experts", S, "tokens", len(toks), {n: f"{v:.2e}" for n, v in errs.items()})
    for n, v in errs.items():
        assert v <= TOL_E2E, (n, v)


def _dw1_entries(cfg, r, e, probs, xf, dyf, w1q_row, w2q_colT, dW1, rng, pool, got, want):
    """dW1[e][f, c] for 4 sampled FFN columns f (their gate and up rows of dW1) x 8 sampled
    hidden columns c: the sum over expert e's rows of the colwise-quantised dGU[:, f] times
    the colwise-quantised x[:, c]. dGU's column is rebuilt for every row of the expert from
    its quantised dY row, the colwise W2 column f and its gate / up entries."""
    H, F = cfg.H, cfg.F
    s0, m = int(r["seg_off"][e]), int(r["m_splits"][e])
    nblk = (m + 31) // 32
    rows = np.arange(s0, s0 + 32 * nblk)
    tk = r["token_of_row"][rows]
    sl = r["slot_of_row"][rows]
    live = tk >= 0
    p_row = np.zeros(len(rows))
    p_row[live] = probs[tk[live], sl[live]]
    xp = np.zeros((len(rows), H))
    xp[live] = xf[tk[live]]
    dyp = np.zeros((len(rows), H))
    dyp[live] = dyf[tk[live]]
    xq_r = _fq_rows_pooled(pool, xp)       # fc1 operand rows (blocks along H)
    dyq_r = _fq_rows_pooled(pool, dyp)     # fc2 data-gradient operand rows (blocks along H)

    def colq(v):                           # blocks of 32 rows of the expert's segment
        return np.concatenate([omx.fake_quant_rowwise(v[None, 32 * b:32 * b + 32])[0] for b in range(nblk)])

    cs = rng.integers(H, size=8)
    xq_cols = {int(c): colq(xp[:, c]) for c in cs}
    for f in rng.integers(F, size=4):
        g_ = xq_r @ w1q_row[f]
        u_ = xq_r @ w1q_row[F + f]
        da = (dyq_r @ w2q_colT[f]) * p_row
        for col, v in ((int(f), da * u_ * omoe.dsilu(g_)), (int(F + f), da * omoe.silu(g_))):
            vq = colq(v)
            for c in cs:
                want.append(float(vq @ xq_cols[int(c)]))
                got.append(float(dW1[e, col, c]))
    return got, want
