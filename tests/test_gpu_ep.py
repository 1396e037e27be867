"""Expert parallelism through the library's kernels on one GPU: a one-rank NCCL group
(the exchanges are copies to itself). Each routed pair becomes its own row (k = 1) of the
local layer, in the same per-expert order as the single-GPU layer, so the results must
be those of GroupedMLP bit for bit (same operands, same kernels, same combine)."""
import datetime

import pytest
import torch
import torch.distributed as dist

import moe_workloads as wl

pytestmark = pytest.mark.gpu


def test_one_rank_expert_parallel_equals_single_gpu_layer(gpu_lib):
    from mxfp8_grouped_gemm_moe_b200.ep import ExpertParallelMLP
    cfg = wl.custom("ep1", T=512, H=256, F=512, E=4, k=2, seed=43)
    d = {k: v.cuda() for k, v in wl.make_all(cfg).items()}
    ref = gpu_lib.GroupedMLP(cfg.T, cfg.k, cfg.E, cfg.H, cfg.F)
    ref.quantize_weights(d["W1"], d["W2"])
    y0 = ref.forward(d["x"], d["topk_idx"], d["probs"])
    g0 = ref.backward(d["dy"])
    dist.init_process_group("nccl", store=dist.HashStore(), rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60), device_id=torch.device("cuda", 0))
    try:
        ep = ExpertParallelMLP(cfg.T, cfg.k, cfg.E, cfg.H, cfg.F)
        ep.local.quantize_weights(d["W1"], d["W2"])
        y = ep.forward(d["x"], d["topk_idx"], d["probs"])
        dx, dW1, dW2, dprobs = ep.backward(d["dy"])
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    assert gpu_lib.mxmoe_get_device_status()[0] == 0
    assert torch.equal(y, y0)
    for got, want in zip((dx, dW1, dW2, dprobs), g0):
        assert torch.equal(got, want)


def test_one_rank_mxfp8_wire_equals_layer_on_rounded_inputs(gpu_lib):
    """Rows dispatched as MXFP8 codes + scales (quantised and dequantised by the library's
    kernels): the results equal GroupedMLP's on x and dY rounded to their rowwise MXFP8
    grid, bit for bit."""
    from mxfp8_grouped_gemm_moe_b200.ep import ExpertParallelMLP
    mx = gpu_lib
    cfg = wl.custom("ep1w", T=512, H=256, F=512, E=4, k=2, seed=47)
    d = {k: v.cuda() for k, v in wl.make_all(cfg).items()}

    def rnd(t):
        r, _ = mx.mxfp8_quantize(t, colwise=False, layout=mx.SCALE_PLAIN)
        return mx.mxfp8_dequantize(r)

    x1, dy1 = rnd(d["x"]), rnd(d["dy"])
    assert not torch.equal(x1, d["x"])
    ref = mx.GroupedMLP(cfg.T, cfg.k, cfg.E, cfg.H, cfg.F)
    ref.quantize_weights(d["W1"], d["W2"])
    y0 = ref.forward(x1, d["topk_idx"], d["probs"])
    g0 = ref.backward(dy1)
    dist.init_process_group("nccl", store=dist.HashStore(), rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60), device_id=torch.device("cuda", 0))
    try:
        ep = ExpertParallelMLP(cfg.T, cfg.k, cfg.E, cfg.H, cfg.F, wire="mxfp8")
        ep.local.quantize_weights(d["W1"], d["W2"])
        y = ep.forward(d["x"], d["topk_idx"], d["probs"])
        dx, dW1, dW2, dprobs = ep.backward(d["dy"])
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    assert mx.mxmoe_get_device_status()[0] == 0
    assert torch.equal(y, y0)
    for got, want in zip((dx, dW1, dW2, dprobs), g0):
        assert torch.equal(got, want)
