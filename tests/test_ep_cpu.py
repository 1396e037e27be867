"""Expert parallelism's exchange logic on the CPU (gloo, world size 2).

Each rank holds half the experts and its own tokens; the dispatch plan, the all-to-all
exchanges out and back and the slot-order combine run as in the layer, with the library's
local grouped MLP replaced by the oracle (the GPU kernels are tested elsewhere). The
result must equal the oracle run on the whole batch on one process: y, dX and dprobs of
each rank's tokens, and the weight gradients of each rank's experts (their rows arrive in
global token order, so even the colwise blocks match)."""
import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_plan_counts_order_and_inverse():
    from mxfp8_grouped_gemm_moe_b200.ep import plan_dispatch
    idx = torch.tensor([[3, 0], [1, 2], [0, 1], [2, 3], [3, 1]], dtype=torch.int32)
    counts, order, pos = plan_dispatch(idx, E_loc=2, G=2)
    dest = (idx.reshape(-1) // 2).tolist()
    assert counts.tolist() == [dest.count(0), dest.count(1)]
    assert order.tolist() == [i for i in range(10) if dest[i] == 0] + [i for i in range(10) if dest[i] == 1]
    assert torch.equal(order[pos], torch.arange(10))
    empty_counts, _, _ = plan_dispatch(torch.zeros((4, 1), dtype=torch.int32), E_loc=2, G=3)
    assert empty_counts.tolist() == [4, 0, 0]
    with pytest.raises(ValueError):
        plan_dispatch(torch.tensor([[5]]), E_loc=2, G=2)


def _problem():
    import moe_workloads as wl
    cfg = wl.custom("ep", T=96, H=64, F=96, E=4, k=2, seed=41)
    d = wl.make_all(cfg)
    return cfg, d


class _OracleLocal:
    """The oracle as a rank's local layer (rows with k = 1, the rank's experts)."""

    def __init__(self, W1, W2):
        self.W1, self.W2 = W1, W2

    def forward(self, x_rows, idx_rows, p_rows):
        from oracle import moe
        self.p = p_rows.double().numpy()
        y, self.saved = moe.mlp_fwd(x_rows.double().numpy(), idx_rows.numpy(), self.p, self.W1, self.W2)
        return torch.from_numpy(y)

    def backward(self, dy_rows):
        from oracle import moe
        g = moe.mlp_bwd(dy_rows.double().numpy(), self.saved, self.p, self.W1, self.W2)
        return (torch.from_numpy(g["dx"]), torch.from_numpy(g["dW1"]), torch.from_numpy(g["dW2"]),
                torch.from_numpy(g["dprobs"]))


class _OracleCodec:
    """The MXFP8 wire through the oracle's rowwise quantiser and dequantiser."""

    def encode(self, x, idx):
        from oracle import mxfp8 as omx
        q, sc = omx.quantize_rowwise(x[idx].double().numpy())
        return torch.from_numpy(np.ascontiguousarray(q, dtype=np.uint8)), \
            torch.from_numpy(np.ascontiguousarray(sc, dtype=np.uint8))

    def decode(self, codes, scales):
        from oracle import mxfp8 as omx
        return torch.from_numpy(omx.dequantize_rowwise(codes.numpy(), scales.numpy()))


def _combine(rows, pos, T, k):
    out = torch.zeros((T, rows.shape[1]), dtype=torch.float64)
    p = pos.view(T, k)
    for j in range(k):
        out += rows.double()[p[:, j]]
    return out


def _worker(rank, world, port, out, wire="bf16"):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from mxfp8_grouped_gemm_moe_b200.ep import ExpertParallelMLP
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        cfg, d = _problem()
        Tl = cfg.T // world
        sl = slice(rank * Tl, (rank + 1) * Tl)
        E_loc = cfg.E // world
        W1 = d["W1"].double().numpy()[rank * E_loc:(rank + 1) * E_loc]
        W2 = d["W2"].double().numpy()[rank * E_loc:(rank + 1) * E_loc]
        layer = ExpertParallelMLP(Tl, cfg.k, cfg.E, cfg.H, cfg.F, local=_OracleLocal(W1, W2), combine=_combine,
                                  wire=wire, codec=_OracleCodec() if wire == "mxfp8" else None)
        y = layer.forward(d["x"][sl], d["topk_idx"][sl], d["probs"][sl])
        dx, dW1, dW2, dprobs = layer.backward(d["dy"][sl])
        out[rank] = dict(y=y.numpy(), dx=dx.numpy(), dW1=dW1.numpy(), dW2=dW2.numpy(), dprobs=dprobs.numpy(),
                         experts=list(layer.experts()))
    finally:
        dist.destroy_process_group()


def test_expert_parallel_exchange_equals_single_process_oracle():
    world, port = 2, _free_port()
    out = mp.get_context("spawn").Manager().dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
    from oracle import moe
    cfg, d = _problem()
    x, W1, W2, p = (d[n].double().numpy() for n in ("x", "W1", "W2", "probs"))
    y, s = moe.mlp_fwd(x, d["topk_idx"].numpy(), p, W1, W2)
    g = moe.mlp_bwd(d["dy"].double().numpy(), s, p, W1, W2)
    Tl = cfg.T // world
    for r in range(world):
        o = out[r]
        sl = slice(r * Tl, (r + 1) * Tl)
        ex = o["experts"]
        np.testing.assert_allclose(o["y"], y[sl], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(o["dx"], g["dx"][sl], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(o["dprobs"], g["dprobs"][sl], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(o["dW1"], g["dW1"][ex[0]:ex[-1] + 1], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(o["dW2"], g["dW2"][ex[0]:ex[-1] + 1], rtol=1e-10, atol=1e-12)


def test_expert_parallel_mxfp8_wire_equals_oracle_on_rounded_inputs():
    """With rows travelling as MXFP8 codes + scales, the layer computes what the single-process
    oracle computes for x and dY rounded to their rowwise MXFP8 grid (the rowwise round trip
    is lossless; the colwise copies come from the rounded rows)."""
    from oracle import mxfp8 as omx
    from oracle import moe
    world, port = 2, _free_port()
    out = mp.get_context("spawn").Manager().dict()
    mp.start_processes(_worker, args=(world, port, out, "mxfp8"), nprocs=world, join=True, start_method="spawn")
    cfg, d = _problem()
    rnd = lambda a: omx.dequantize_rowwise(*omx.quantize_rowwise(a))  # noqa: E731
    x, dy = rnd(d["x"].double().numpy()), rnd(d["dy"].double().numpy())
    W1, W2, p = (d[n].double().numpy() for n in ("W1", "W2", "probs"))
    assert not np.array_equal(x, d["x"].double().numpy())      # the wire does round
    y, s = moe.mlp_fwd(x, d["topk_idx"].numpy(), p, W1, W2)
    g = moe.mlp_bwd(dy, s, p, W1, W2)
    Tl = cfg.T // world
    for r in range(world):
        o = out[r]
        sl = slice(r * Tl, (r + 1) * Tl)
        ex = o["experts"]
        np.testing.assert_allclose(o["y"], y[sl], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(o["dx"], g["dx"][sl], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(o["dprobs"], g["dprobs"][sl], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(o["dW1"], g["dW1"][ex[0]:ex[-1] + 1], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(o["dW2"], g["dW2"][ex[0]:ex[-1] + 1], rtol=1e-10, atol=1e-12)
