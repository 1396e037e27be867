"""Grouped expert MLP, forward and backward, fp64 (oracle; test infrastructure only).

Follows, in the pages' order, the steps the three pages name:
  1. tokens are grouped by expert using per-expert token counts ("MoE-Training für
     biologische Grundmodelle optimieren", hyper.ai/de, GroupedLinear passage);
  2. activations and weights are quantised to MXFP8 (same page, MXFP8 passage;
     "NVIDIA optimise l'entraînement MoE des modèles biologiques", hyper.ai/fr);
  3. the gate-up projection, the ScaledSwiGLU activation and the routing-weight
     scaling form one fused step, with a matching backward (hyper.ai/de, GroupedMLP
     passage; "NVIDIA apresenta técnicas ... arquitetura MoE", conexaotc.com.br,
     third optimisation);
  4. the down projection and the return to token order (the pages are silent on
     these; the plain reading: a second expert linear, and a sum over the k routed
     copies of each token).

Readings where the pages are silent (each is listed in the design notes):
  * rows are ordered by (expert ascending, token ascending); each expert segment
    starts at a multiple of ``align`` rows, pad rows are zero and ignored;
  * W1 is [E, 2F, H] (nn.Linear out x in) with gate rows first, up rows second;
    W2 is [E, H, F]; no biases;
  * Z = silu(G) * U * p, p the routed row's probability, applied before the down
    projection and quantised from its fp64 value;
  * backward uses the straight-through estimator (every quantiser passes the
    gradient unchanged) and quantises dY, dGU rowwise and colwise as the consuming
    GEMMs need; the activations saved for backward are kept in fp64 here;
  * gradients are E4M3 like everything else; ``grad_fmt="e5m2"`` is the variant that
    quantises dY and dGU to MXFP8 E5M2 instead (weights and activations stay E4M3);
  * every quantiser uses the OCP scale rule; ``scale_rule="ceil"`` is the variant whose
    scale is rounded up so that no element saturates (all quantisers of the layer).
Every GEMM is a library matmul over dequantised fp64 operands, one expert at a time.
"""
from __future__ import annotations

import numpy as np

from . import mxfp8

ALIGN_ORACLE = 32


def _roundup(x, a):
    return (x + a - 1) // a * a


# ----------------------------------------------------------------------------- routing

def route(topk_idx, E, align=ALIGN_ORACLE):
    """Counting sort of the (token, slot) pairs by expert, stable by token.

    Returns dict with m_splits int64[E], seg_off int64[E+1] (segment e starts at the
    sum of the earlier segments' counts rounded up to ``align``), row_of_slot
    int64[T,k], token_of_row int64[Mp] (-1 on pad rows), slot_of_row int64[Mp].
    Raises ValueError on an expert id out of range or repeated within a token."""
    idx = np.asarray(topk_idx, dtype=np.int64)
    T, k = idx.shape
    if np.any(idx < 0) or np.any(idx >= E):
        raise ValueError("expert id out of range")
    for t in range(T):
        if len(set(idx[t].tolist())) != k:
            raise ValueError("repeated expert within a token's top-k")
    tok = np.repeat(np.arange(T), k)
    slot = np.tile(np.arange(k), T)
    exp = idx.reshape(-1)
    order = np.lexsort((tok, exp))            # primary key: expert; secondary: token
    m_splits = np.bincount(exp, minlength=E).astype(np.int64)
    seg_off = np.zeros(E + 1, dtype=np.int64)
    seg_off[1:] = np.cumsum(_roundup(m_splits, align))
    Mp = int(seg_off[E])
    row_of_slot = np.zeros((T, k), dtype=np.int64)
    token_of_row = np.full(Mp, -1, dtype=np.int64)
    slot_of_row = np.full(Mp, -1, dtype=np.int64)
    pos = 0
    for e in range(E):
        for i in range(m_splits[e]):
            p = order[pos]
            pos += 1
            r = seg_off[e] + i
            row_of_slot[tok[p], slot[p]] = r
            token_of_row[r] = tok[p]
            slot_of_row[r] = slot[p]
    return dict(m_splits=m_splits, seg_off=seg_off, row_of_slot=row_of_slot,
                token_of_row=token_of_row, slot_of_row=slot_of_row, Mp=Mp)


def permute_rows(x, token_of_row):
    """Xp[r] = x[token_of_row[r]], zero where token_of_row == -1."""
    x = np.asarray(x, dtype=np.float64)
    out = np.zeros((len(token_of_row),) + x.shape[1:], dtype=np.float64)
    live = token_of_row >= 0
    out[live] = x[token_of_row[live]]
    return out


def unpermute_sum(yp, row_of_slot):
    """Y[t] = sum over slots j (in order) of Yp[row_of_slot[t, j]]."""
    yp = np.asarray(yp, dtype=np.float64)
    T, k = row_of_slot.shape
    out = np.zeros((T,) + yp.shape[1:], dtype=np.float64)
    for j in range(k):
        out += yp[row_of_slot[:, j]]
    return out


# ----------------------------------------------------------------------------- MXFP8 helpers

def quantize_colwise_segments(a, seg_off, m_splits, fmt="e4m3", rule="ocp"):
    """Colwise MXFP8 of a permuted [Mp, C] matrix: blocks of 32 rows that start at each
    expert segment's first row (segments are 32-aligned with zero pad rows), stored
    transposed -> (codes uint8[C, Mp], scales uint8[C, Mp/32])."""
    a = np.asarray(a, dtype=np.float64)
    Mp, C = a.shape
    codes = np.zeros((C, Mp), dtype=np.uint8)
    scales = np.zeros((C, Mp // mxfp8.BLOCK), dtype=np.uint8)
    for e in range(len(m_splits)):
        s0, s1 = int(seg_off[e]), int(seg_off[e + 1])
        if s1 == s0:
            continue
        assert s0 % mxfp8.BLOCK == 0 and s1 % mxfp8.BLOCK == 0
        c, s = mxfp8.quantize_colwise_t(a[s0:s1], fmt, rule)
        codes[:, s0:s1] = c
        scales[:, s0 // mxfp8.BLOCK:s1 // mxfp8.BLOCK] = s
    return codes, scales


def fake_quant_colwise_segments(a, seg_off, m_splits, fmt="e4m3", rule="ocp"):
    c, s = quantize_colwise_segments(a, seg_off, m_splits, fmt, rule)
    return mxfp8.dequantize_rowwise(c, s, fmt).T


def _fq_row(a, quant, fmt="e4m3", rule="ocp"):
    return mxfp8.fake_quant_rowwise(a, fmt, rule) if quant else np.asarray(a, dtype=np.float64)


def _fq_col(a, quant, rule="ocp"):
    return mxfp8.fake_quant_colwise(a, "e4m3", rule) if quant else np.asarray(a, dtype=np.float64)


def _fq_col_seg(a, r, quant, fmt="e4m3", rule="ocp"):
    if not quant:
        return np.asarray(a, dtype=np.float64)
    return fake_quant_colwise_segments(a, r["seg_off"], r["m_splits"], fmt, rule)


# ----------------------------------------------------------------------------- grouped GEMMs

def grouped_gemm(A, B, seg_off):
    """C[seg_e] = A[seg_e] @ B[e]^T for each expert e (A [Mp, K], B [E, N, K]), fp64;
    rows outside every segment are zero."""
    A = np.asarray(A, dtype=np.float64)
    E, N, _ = B.shape
    C = np.zeros((A.shape[0], N), dtype=np.float64)
    for e in range(E):
        s0, s1 = int(seg_off[e]), int(seg_off[e + 1])
        if s1 > s0:
            C[s0:s1] = A[s0:s1] @ np.asarray(B[e], dtype=np.float64).T
    return C


def grouped_gemm_wgrad(At, Bt, seg_off):
    """C[e] = At[:, seg_e] @ Bt[:, seg_e]^T (At [N, Mp], Bt [K', Mp]) -> [E, N, K'];
    an expert with no rows gets zeros."""
    E = len(seg_off) - 1
    At = np.asarray(At, dtype=np.float64)
    Bt = np.asarray(Bt, dtype=np.float64)
    C = np.zeros((E, At.shape[0], Bt.shape[0]), dtype=np.float64)
    for e in range(E):
        s0, s1 = int(seg_off[e]), int(seg_off[e + 1])
        if s1 > s0:
            C[e] = At[:, s0:s1] @ Bt[:, s0:s1].T
    return C


# ----------------------------------------------------------------------------- SwiGLU

def sigmoid(x):
    x = np.asarray(x, dtype=np.float64)
    return 1.0 / (1.0 + np.exp(-x))


def silu(x):
    """silu(g) = g / (1 + e^-g)."""
    x = np.asarray(x, dtype=np.float64)
    return x * sigmoid(x)


def dsilu(x):
    """d silu / dg = s(g) * (1 + g * (1 - s(g))), s the logistic function."""
    s = sigmoid(x)
    return s * (1.0 + x * (1.0 - s))


# ----------------------------------------------------------------------------- MLP

def mlp_fwd(x, topk_idx, probs, W1, W2, quant=True, align=ALIGN_ORACLE, scale_rule="ocp"):
    """Forward of the grouped expert MLP. Returns (y fp64[T,H], saved dict). scale_rule
    ("ocp" or "ceil") is the scale choice of every quantiser of the layer; the backward
    takes it from the saved dict."""
    x = np.asarray(x, dtype=np.float64)
    probs = np.asarray(probs, dtype=np.float64)
    E, F2, H = W1.shape
    F = F2 // 2
    r = route(topk_idx, E, align)
    Xp = permute_rows(x, r["token_of_row"])
    live = r["token_of_row"] >= 0
    p_row = np.zeros(r["Mp"], dtype=np.float64)
    p_row[live] = probs[r["token_of_row"][live], r["slot_of_row"][live]]
    sr = scale_rule
    Xq = _fq_row(Xp, quant, rule=sr)                                   # blocks along H
    W1q = np.stack([_fq_row(W1[e], quant, rule=sr) for e in range(E)])  # blocks along H
    GU = grouped_gemm(Xq, W1q, r["seg_off"])
    G, U = GU[:, :F], GU[:, F:]
    Z = silu(G) * U * p_row[:, None]
    Zq = _fq_row(Z, quant, rule=sr)                                    # blocks along F
    W2q = np.stack([_fq_row(W2[e], quant, rule=sr) for e in range(E)])  # blocks along F
    Yp = grouped_gemm(Zq, W2q, r["seg_off"])
    y = unpermute_sum(Yp, r["row_of_slot"])
    saved = dict(route=r, Xp=Xp, p_row=p_row, G=G, U=U, Z=Z, Yp=Yp, scale_rule=sr)
    return y, saved


def mlp_bwd(dy, saved, probs, W1, W2, quant=True, grad_fmt="e4m3"):
    """Backward (straight-through estimator for every quantiser). grad_fmt is the MXFP8
    element format of the gradients dY and dGU ("e4m3" or "e5m2").
    Returns dict dx fp64[T,H], dW1 fp64[E,2F,H], dW2 fp64[E,H,F], dprobs fp64[T,k]."""
    r = saved["route"]
    E, F2, H = W1.shape
    F = F2 // 2
    G, U, Z, p_row = saved["G"], saved["U"], saved["Z"], saved["p_row"]
    sr = saved.get("scale_rule", "ocp")
    dYp = permute_rows(dy, r["token_of_row"])
    dYq_row = _fq_row(dYp, quant, grad_fmt, sr)           # blocks along H (fc2 dgrad)
    dYq_col = _fq_col_seg(dYp, r, quant, grad_fmt, sr)    # blocks along M (fc2 wgrad)
    W2q_col = np.stack([_fq_col(W2[e], quant, sr) for e in range(E)])   # [H, F], blocks along H
    # fc2 dgrad: dZ = dYp . W2  (contract over H)
    dZ = grouped_gemm(dYq_row, np.transpose(W2q_col, (0, 2, 1)), r["seg_off"])
    A = silu(G) * U
    dprob_row = np.sum(dZ * A, axis=1)
    dA = dZ * p_row[:, None]
    dG = dA * U * dsilu(G)
    dU = dA * silu(G)
    dGU = np.concatenate([dG, dU], axis=1)
    dGUq_row = _fq_row(dGU, quant, grad_fmt, sr)          # blocks along 2F (fc1 dgrad)
    dGUq_col = _fq_col_seg(dGU, r, quant, grad_fmt, sr)   # blocks along M (fc1 wgrad)
    Zq_col = _fq_col_seg(Z, r, quant, rule=sr)
    Xq_col = _fq_col_seg(saved["Xp"], r, quant, rule=sr)
    # fc2 wgrad: dW2[e] = dYp_e^T . Z_e  (contract over the expert's rows)
    dW2 = grouped_gemm_wgrad(dYq_col.T, Zq_col.T, r["seg_off"])
    # fc1 dgrad: dXp = dGU . W1  (contract over 2F)
    W1q_col = np.stack([_fq_col(W1[e], quant, sr) for e in range(E)])   # [2F, H], blocks along 2F
    dXp = grouped_gemm(dGUq_row, np.transpose(W1q_col, (0, 2, 1)), r["seg_off"])
    # fc1 wgrad: dW1[e] = dGU_e^T . Xp_e
    dW1 = grouped_gemm_wgrad(dGUq_col.T, Xq_col.T, r["seg_off"])
    dx = unpermute_sum(dXp, r["row_of_slot"])
    dprobs = dprob_row[r["row_of_slot"]]
    return dict(dx=dx, dW1=dW1, dW2=dW2, dprobs=dprobs, dGU=dGU, dZ=dZ, dXp=dXp)


def mlp_per_token(x, topk_idx, probs, W1, W2, quant=True):
    """Forward written token by token: y[t] = sum_j W2q[e] . q(silu(g) * u * p) with
    g, u from W1q[e] . q(x[t]), e = topk_idx[t, j]. No grouping, no permutation."""
    x = np.asarray(x, dtype=np.float64)
    E, F2, H = W1.shape
    F = F2 // 2
    W1q = [_fq_row(W1[e], quant) for e in range(E)]
    W2q = [_fq_row(W2[e], quant) for e in range(E)]
    T, k = topk_idx.shape
    y = np.zeros((T, H), dtype=np.float64)
    for t in range(T):
        xq = _fq_row(x[t:t + 1], quant)[0]
        for j in range(k):
            e = int(topk_idx[t, j])
            gu = W1q[e] @ xq
            z = silu(gu[:F]) * gu[F:] * float(probs[t, j])
            zq = _fq_row(z[None, :], quant)[0]
            y[t] += W2q[e] @ zq
    return y


# ----------------------------------------------------------------------------- independent restatement

def _fake_quant_along(a, axis, fmt="e4m3", rule="ocp"):
    """Quantise then dequantise a 2-D fp64 matrix in blocks of 32 consecutive entries
    along ``axis`` (1: along each row; 0: down each column). When the axis length is not a
    multiple of 32 the last block is short: its scale is taken over the entries it has (as
    if zero-padded to 32) and only those entries are returned. Written as a plain loop over
    the blocks, each gathered into a [.., 32] array for ``mxfp8.quantize_blocks``."""
    a = np.asarray(a, dtype=np.float64)
    out = np.empty_like(a)
    n = a.shape[axis]
    for b0 in range(0, n, mxfp8.BLOCK):
        b1 = min(n, b0 + mxfp8.BLOCK)
        part = a[:, b0:b1] if axis == 1 else a[b0:b1, :].T        # [other, b1 - b0]
        blk = np.zeros((part.shape[0], mxfp8.BLOCK), dtype=np.float64)
        blk[:, :b1 - b0] = part
        codes, sb = mxfp8.quantize_blocks(blk, fmt, rule)
        deq = mxfp8.dequantize_blocks(codes, sb, fmt)[:, :b1 - b0]
        if axis == 1:
            out[:, b0:b1] = deq
        else:
            out[b0:b1, :] = deq.T
    return out


def mlp_bwd_per_expert(x, dy, topk_idx, probs, W1, W2, grad_fmt="e4m3", scale_rule="ocp"):
    """The quantised backward restated one expert at a time, without the routing tables,
    the padded permuted layout or any of the rowwise / colwise helpers above.

    For each expert e its rows are the (token, slot) pairs routed to it, in token order.
    The forward's fc1 is recomputed for those rows (x and W1 with blocks along H), then
    each of the four backward GEMMs quantises its two operands with 32-value blocks along
    THAT GEMM's contraction index -- the rule that lets a block's scale factor out of
    every partial dot product ("MoE-Training für biologische Grundmodelle optimieren",
    hyper.ai/de, MXFP8 passage: one scale per block of 32 values):
      fc2 data gradient   dZ    = dY_e . W2_e        contracts H:   dY along H, W2_e down H;
      fc2 weight gradient dW2_e = dY_e^T . Z_e       contracts rows: both down the rows;
      fc1 data gradient   dX_e  = dGU_e . W1_e       contracts 2F:  dGU along 2F, W1_e down 2F;
      fc1 weight gradient dW1_e = dGU_e^T . X_e      contracts rows: both down the rows.
    The expert's row blocks start at its first row and its last block may be short (the
    padded layout's zero rows change no scale). Gradients dY, dGU take ``grad_fmt``;
    weights, x and Z stay E4M3; every quantiser takes ``scale_rule``.
    Returns dict dx [T,H], dW1 [E,2F,H], dW2 [E,H,F], dprobs [T,k] (fp64)."""
    x = np.asarray(x, dtype=np.float64)
    dy = np.asarray(dy, dtype=np.float64)
    probs = np.asarray(probs, dtype=np.float64)
    idx = np.asarray(topk_idx, dtype=np.int64)
    E, F2, H = W1.shape
    F = F2 // 2
    T, k = idx.shape
    sr = scale_rule

    def q(a, axis, fmt="e4m3"):
        return _fake_quant_along(a, axis, fmt, sr)

    dx = np.zeros((T, H))
    dW1 = np.zeros((E, F2, H))
    dW2 = np.zeros((E, H, F))
    dprobs = np.zeros((T, k))
    for e in range(E):
        pairs = [(t, j) for t in range(T) for j in range(k) if idx[t, j] == e]
        if not pairs:
            continue                                   # no rows: zero weight gradients
        tok = np.array([t for t, _ in pairs])
        slot = np.array([j for _, j in pairs])
        p = probs[tok, slot]
        W1e = np.asarray(W1[e], dtype=np.float64)      # [2F, H]
        W2e = np.asarray(W2[e], dtype=np.float64)      # [H, F]
        Xe = x[tok]                                    # [m, H]
        GU = q(Xe, 1) @ q(W1e, 1).T                    # forward fc1, contracts H
        G, U = GU[:, :F], GU[:, F:]
        A = silu(G) * U
        Ze = A * p[:, None]
        dYe = dy[tok]                                  # [m, H]
        dZ = q(dYe, 1, grad_fmt) @ q(W2e, 0)           # contracts H
        dprob = np.sum(dZ * A, axis=1)
        dA = dZ * p[:, None]
        dGU = np.concatenate([dA * U * dsilu(G), dA * silu(G)], axis=1)   # [m, 2F]
        dW2[e] = q(dYe, 0, grad_fmt).T @ q(Ze, 0)      # contracts the expert's rows
        dXe = q(dGU, 1, grad_fmt) @ q(W1e, 0)          # contracts 2F
        dW1[e] = q(dGU, 0, grad_fmt).T @ q(Xe, 0)      # contracts the expert's rows
        for i, (t, j) in enumerate(pairs):
            dx[t] += dXe[i]
            dprobs[t, j] = dprob[i]
    return dict(dx=dx, dW1=dW1, dW2=dW2, dprobs=dprobs)


# ----------------------------------------------------------------------------- per-tensor FP8 recipe

def mlp_fwd_fp8_tensor(x, topk_idx, probs, W1, W2, z_amax_in, align=ALIGN_ORACLE):
    """Forward with per-tensor FP8 in place of MXFP8 (the pages' "FP8" beside "MXFP8":
    "MoE-Training für biologische Grundmodelle optimieren", hyper.ai/de, precision passage).

    Every operand is E4M3 under one fp32 multiplier per tensor (mxfp8.tensor_multiplier):
    x (all tokens), W1[e] and W2[e] (one per expert), from their own largest magnitude
    (current scaling). Z is produced tile by tile inside the fused step, so its multiplier
    comes from ``z_amax_in`` -- a largest magnitude known before the step (delayed scaling,
    e.g. the previous step's); values beyond it saturate. Returns (y, saved) where saved
    also holds ``z_amax`` (the largest |Z| over live rows, for the next step) and the
    multipliers."""
    x = np.asarray(x, dtype=np.float64)
    probs = np.asarray(probs, dtype=np.float64)
    E, F2, H = W1.shape
    F = F2 // 2
    r = route(topk_idx, E, align)
    live = r["token_of_row"] >= 0
    p_row = np.zeros(r["Mp"], dtype=np.float64)
    p_row[live] = probs[r["token_of_row"][live], r["slot_of_row"][live]]
    m_x = mxfp8.tensor_multiplier(np.max(np.abs(x)))
    m_w1 = [mxfp8.tensor_multiplier(np.max(np.abs(W1[e]))) for e in range(E)]
    m_w2 = [mxfp8.tensor_multiplier(np.max(np.abs(W2[e]))) for e in range(E)]
    m_z = mxfp8.tensor_multiplier(z_amax_in)
    Xq = permute_rows(mxfp8.fake_quant_tensor(x, m_x), r["token_of_row"])
    W1q = np.stack([mxfp8.fake_quant_tensor(W1[e], m_w1[e]) for e in range(E)])
    W2q = np.stack([mxfp8.fake_quant_tensor(W2[e], m_w2[e]) for e in range(E)])
    GU = grouped_gemm(Xq, W1q, r["seg_off"])
    G, U = GU[:, :F], GU[:, F:]
    Z = silu(G) * U * p_row[:, None]
    Zq = mxfp8.dequantize_tensor(mxfp8.e4m3_encode(Z * np.float64(m_z)), m_z)
    Yp = grouped_gemm(Zq, W2q, r["seg_off"])
    y = unpermute_sum(Yp, r["row_of_slot"])
    saved = dict(route=r, Xq=Xq, p_row=p_row, G=G, U=U, Zq=Zq, W1q=W1q, W2q=W2q,
                 z_amax=float(np.max(np.abs(Z[live]))) if live.any() else 0.0,
                 m=dict(x=m_x, w1=m_w1, w2=m_w2, z=m_z))
    return y, saved


def mlp_bwd_fp8_tensor(dy, saved, dgu_amax_in):
    """Backward of the per-tensor FP8 recipe (straight-through estimator). dY takes its
    multiplier from its own largest magnitude; dGU, produced inside the fused backward
    step, from ``dgu_amax_in`` (delayed scaling). A per-tensor quantiser has no block
    direction, so every GEMM reuses the one quantised copy of each operand (x, W1, W2 and
    Z from the forward, dY and dGU here). Returns dict dx, dW1, dW2, dprobs and dgu_amax
    (the largest |dGU| over live rows, for the next step)."""
    r = saved["route"]
    G, U, p_row = saved["G"], saved["U"], saved["p_row"]
    W1q, W2q = saved["W1q"], saved["W2q"]
    F = G.shape[1]
    live = r["token_of_row"] >= 0
    dy = np.asarray(dy, dtype=np.float64)
    m_dy = mxfp8.tensor_multiplier(np.max(np.abs(dy)))
    dYq = permute_rows(mxfp8.fake_quant_tensor(dy, m_dy), r["token_of_row"])
    dZ = grouped_gemm(dYq, np.transpose(W2q, (0, 2, 1)), r["seg_off"])      # contracts H
    A = silu(G) * U
    dprob_row = np.sum(dZ * A, axis=1)
    dA = dZ * p_row[:, None]
    dGU = np.concatenate([dA * U * dsilu(G), dA * silu(G)], axis=1)
    m_g = mxfp8.tensor_multiplier(dgu_amax_in)
    dGUq = mxfp8.dequantize_tensor(mxfp8.e4m3_encode(dGU * np.float64(m_g)), m_g)
    dW2 = grouped_gemm_wgrad(dYq.T, saved["Zq"].T, r["seg_off"])
    dXp = grouped_gemm(dGUq, np.transpose(W1q, (0, 2, 1)), r["seg_off"])    # contracts 2F
    dW1 = grouped_gemm_wgrad(dGUq.T, saved["Xq"].T, r["seg_off"])
    dx = unpermute_sum(dXp, r["row_of_slot"])
    dprobs = dprob_row[r["row_of_slot"]]
    del F
    return dict(dx=dx, dW1=dW1, dW2=dW2, dprobs=dprobs,
                dgu_amax=float(np.max(np.abs(dGU[live]))) if live.any() else 0.0, m_dy=m_dy, m_dgu=m_g)
