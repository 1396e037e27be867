"""Expert parallelism: the layer's experts spread over the ranks of a process group.

"MoE-Training für biologische Grundmodelle optimieren" (hyper.ai/de), expert-parallel
passage: expert parallelism combined with data parallelism, checked first on two GPUs and
then run with eight-way expert parallelism.

Rank r of G holds the contiguous experts [r*E_loc, (r+1)*E_loc), E_loc = E / G; every rank
brings its own tokens. One step on each rank:

  forward   plan: the rank's (token, slot) pairs sorted by destination rank (the rank of
            their expert), stable by pair index -> the G send counts travel by an
            all-to-all -> the pairs' rows x[t] (bf16), local expert ids and routing
            probabilities travel by all-to-all-v -> the local grouped MLP runs on the
            received rows, one row per pair (k = 1, E_loc experts) -> its output rows go
            back by the reversed all-to-all-v -> each token's k rows are summed in slot
            order (the combine of the single-GPU layer).
  backward  the same plan carries the rows of dY out and the rows of dX and the
            per-pair dprobs back; the weight gradients stay with each expert's owner.

Wire format of the dispatch direction (x out in the forward, dY out in the backward):
  wire="bf16"   rows travel as bf16, so every row's computation is the single-GPU layer's:
                a row's MXFP8 codes depend only on the row, and with ranks holding
                consecutive token ranges the rows of an expert arrive in global token
                order, so even the colwise blocks of the weight gradients match a
                single-GPU run on the whole batch;
  wire="mxfp8"  rows travel as their rowwise MXFP8 codes + E8M0 scales (1 + 1/32 bytes per
                value instead of 2) and are dequantised on arrival. The rowwise round trip
                is lossless, so the layer's rowwise operands are unchanged; its colwise
                copies (weight-gradient operands) are quantised from the dequantised
                rows: the layer computes exactly what the single-GPU layer computes for the
                inputs rounded to their MXFP8 rowwise grid.
The combine direction (y and dX back, dprobs back) stays bf16 / fp32: those rows are summed
over a token's slots, and quantising them would add a rounding the single-GPU layer does
not have. The exchanges are torch.distributed all-to-all calls (NCCL over NVLink /
NVSwitch on GPUs); nothing is multicast. The plan and the gathers are index plumbing
(torch), the layer's arithmetic -- quantisation and dequantisation included -- runs in
the library's kernels.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def plan_dispatch(topk_idx, E_loc, G):
    """Send plan of one rank: (counts, order, pos).

    counts  int64 [G]: pairs for each destination rank;
    order   int64 [T*k]: pair indices (t*k + j) sorted by destination rank, stable by pair
            index -- the send buffer's row i carries pair order[i];
    pos     int64 [T*k]: the inverse -- the send-buffer row of each pair."""
    dest = (topk_idx.reshape(-1).long() // E_loc)
    if dest.numel() and (int(dest.min()) < 0 or int(dest.max()) >= G):
        raise ValueError("expert id outside the group's experts")
    order = torch.argsort(dest, stable=True)
    counts = torch.bincount(dest, minlength=G)
    pos = torch.empty_like(order)
    pos[order] = torch.arange(order.numel(), device=order.device)
    return counts, order, pos


class LibraryLocalMLP:
    """The local grouped MLP of one rank on the library's kernels (MXFP8, fused forward and
    backward), with buffers for up to n_max received rows."""

    def __init__(self, n_max, E_loc, H, F, device):
        import mxfp8_grouped_gemm_moe_b200 as mx
        if not torch.cuda.is_available():
            raise RuntimeError("the library's local MLP needs a CUDA device")
        self.mx, self.E, self.H, self.F = mx, E_loc, H, F
        lib = mx.load()
        self.saved = torch.empty(lib.grouped_mlp_saved_size(n_max, 1, E_loc, H, F), dtype=torch.uint8, device=device)
        self.ws = torch.empty(lib.grouped_mlp_workspace_size(n_max, 1, E_loc, H, F), dtype=torch.uint8, device=device)
        self.wq = torch.empty(lib.mxmoe_weights_size(E_loc, H, F), dtype=torch.uint8, device=device)
        self.n = 0

    def quantize_weights(self, W1_loc, W2_loc):
        self.mx.mxmoe_weights_quantize(W1_loc, W2_loc, out=self.wq)

    def forward(self, x_rows, idx_rows, p_rows):
        self.n = x_rows.shape[0]
        return self.mx.grouped_mlp_fwd(x_rows, idx_rows, p_rows, self.wq, self.E, self.F, self.saved, self.ws)

    def backward(self, dy_rows):
        return self.mx.grouped_mlp_bwd(dy_rows, self.saved, self.wq, self.n, 1, self.E, self.H, self.F, self.ws)


class LibraryMXFP8Codec:
    """Rowwise MXFP8 (E4M3, plain scale layout) of gathered rows and its inverse, on the
    library's kernels."""

    def encode(self, x, idx):
        """(codes uint8 [n, H], scales uint8 [n, H/32]) of the rows x[idx]."""
        import mxfp8_grouped_gemm_moe_b200 as mx
        n, H = idx.numel(), x.shape[1]
        n32 = (n + 31) // 32 * 32                    # the quantiser's row granularity
        gather = torch.full((n32,), -1, dtype=torch.int32, device=x.device)
        gather[:n] = idx.to(torch.int32)
        r, _ = mx.mxfp8_quantize(x, colwise=False, layout=mx.SCALE_PLAIN, row_gather=gather, out_rows=n32)
        return r.data[:n], r.scale.view(n32, H // 32)[:n]

    def decode(self, codes, scales):
        """bf16 [n, H] rows from their codes and scales."""
        import mxfp8_grouped_gemm_moe_b200 as mx
        m = mx.MXFP8(codes.contiguous(), scales.contiguous().view(-1), mx.SCALE_PLAIN, mx.FMT_E4M3)
        return mx.mxfp8_dequantize(m)


def library_combine(rows, pos, T, k):
    """y[t] = sum over slots j (in order) of rows[pos[t*k + j]], fp32 sum rounded once to
    bf16 (the library's combine kernel)."""
    import mxfp8_grouped_gemm_moe_b200 as mx
    return mx.moe_unpermute(rows, pos.view(T, k).to(torch.int32))


class ExpertParallelMLP:
    """The grouped expert MLP with its E experts spread over the G ranks of `group`.

    local: the rank's local layer (forward(x_rows, idx_rows [n, 1] int32, p_rows [n, 1]
    fp32) -> y_rows; backward(dy_rows) -> (dx_rows, dW1_loc, dW2_loc, dprobs_rows [n, 1]));
    combine(rows, pos, T, k) -> [T, H]; wire "bf16" or "mxfp8" (the dispatch direction's
    format, see the module docstring) with codec (encode(x, idx) -> (codes, scales);
    decode(codes, scales) -> rows). All default to the library's kernels."""

    def __init__(self, T_max, k, E, H, F, group=None, device="cuda", local=None, combine=None, wire="bf16",
                 codec=None):
        self.group = group
        self.G = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        if E % self.G:
            raise ValueError("the experts must divide evenly over the ranks")
        self.k, self.E, self.H, self.F = k, E, H, F
        self.E_loc = E // self.G
        if wire not in ("bf16", "mxfp8"):
            raise ValueError("wire must be 'bf16' or 'mxfp8'")
        if wire == "mxfp8" and H % 32:
            raise ValueError("the MXFP8 wire needs H % 32 == 0")
        self.local = local if local is not None else LibraryLocalMLP(self.G * T_max * k, self.E_loc, H, F, device)
        self.combine = combine if combine is not None else library_combine
        self.wire = wire
        self.codec = codec if codec is not None else (LibraryMXFP8Codec() if wire == "mxfp8" else None)

    def experts(self):
        """The global ids of this rank's experts."""
        return range(self.rank * self.E_loc, (self.rank + 1) * self.E_loc)

    def _exchange(self, send, send_counts, recv_counts):
        out = send.new_empty((int(sum(recv_counts)),) + tuple(send.shape[1:]))
        dist.all_to_all_single(out, send.contiguous(), output_split_sizes=recv_counts,
                               input_split_sizes=send_counts, group=self.group)
        return out

    def _dispatch_rows(self, src, idx, sc, rc):
        """The rows src[idx], sent out by the plan's counts and received, in the wire format."""
        if self.wire == "bf16":
            return self._exchange(src[idx], sc, rc)
        codes, scales = self.codec.encode(src, idx)
        return self.codec.decode(self._exchange(codes, sc, rc), self._exchange(scales, sc, rc))

    def forward(self, x, topk_idx, probs):
        T, k = topk_idx.shape
        counts, order, pos = plan_dispatch(topk_idx, self.E_loc, self.G)
        recv = torch.empty_like(counts)
        dist.all_to_all_single(recv, counts, group=self.group)
        self._plan = (T, k, order, pos, counts.tolist(), recv.tolist())
        _, _, _, _, sc, rc = self._plan
        tok = order // k
        x_rows = self._dispatch_rows(x, tok, sc, rc)
        e_rows = self._exchange((topk_idx.reshape(-1)[order] % self.E_loc).to(torch.int32), sc, rc)
        p_rows = self._exchange(probs.reshape(-1)[order].float(), sc, rc)
        y_rows = self.local.forward(x_rows, e_rows.view(-1, 1), p_rows.view(-1, 1))
        back = self._exchange(y_rows, rc, sc)
        return self.combine(back, pos, T, k)

    def backward(self, dy):
        """(dx [T, H], dW1 of this rank's experts [E_loc, 2F, H], dW2 [E_loc, H, F],
        dprobs [T, k])."""
        T, k, order, pos, sc, rc = self._plan
        dy_rows = self._dispatch_rows(dy, order // k, sc, rc)
        dx_rows, dW1, dW2, dp_rows = self.local.backward(dy_rows)
        dx_back = self._exchange(dx_rows, rc, sc)
        dp_back = self._exchange(dp_rows.reshape(-1), rc, sc)
        dx = self.combine(dx_back, pos, T, k)
        dprobs = dp_back[pos].view(T, k)
        return dx, dW1, dW2, dprobs
