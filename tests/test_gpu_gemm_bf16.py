"""GPU parity of the bf16 grouped GEMMs (same scheduler and CTA-pair tiles as the MXFP8
path, tcgen05 kind::f16) with the oracle's grouped GEMMs in fp64 on the same bf16
operands. The products of bf16 values are exact in fp64, so the only difference is
the GPU's fp32 accumulation: relative L2 <= 5e-4 (fp32 out) / 5e-3 (bf16 out)."""
import numpy as np
import pytest
import torch

import moe_workloads as wl
from oracle import moe as omoe
from tests.util import f64, rel_l2, SEG_ALIGN

pytestmark = pytest.mark.gpu


def _routed(counts, seed):
    idx = []
    for e, c in enumerate(counts):
        idx += [e] * c
    idx = np.array(idx, dtype=np.int64).reshape(-1, 1)
    r = omoe.route(idx, len(counts), align=SEG_ALIGN)
    cap = (len(idx) + 255 * len(counts) + 255) // 256 * 256
    return r, cap


@pytest.mark.parametrize("counts,N,K", [
    ([300, 0, 129, 1, 640], 256, 64),
    ([1000, 500, 31, 33], 512, 1024),
    ([127, 129, 40, 700, 0, 0, 1, 255], 768, 192),
])
def test_grouped_gemm_bf16(gpu_lib, counts, N, K):
    r, cap = _routed(counts, seed=1)
    E = len(counts)
    T = sum(counts)
    x = wl.random_matrix(T, K, seed=T + K)
    Xp = torch.zeros((cap, K), dtype=torch.bfloat16)
    live = r["token_of_row"] >= 0
    Xp[:r["Mp"]][torch.from_numpy(live)] = x[torch.from_numpy(r["token_of_row"][live])]
    W = wl.random_matrix(N, K, seed=5, std=0.05, batch=E)
    seg = torch.tensor(r["seg_off"], dtype=torch.int32, device="cuda")
    want = omoe.grouped_gemm(f64(Xp[:r["Mp"]]), f64(W), r["seg_off"])
    for dt, tol in ((torch.float32, 5e-4), (torch.bfloat16, 5e-3)):
        C = gpu_lib.grouped_gemm_bf16(Xp.cuda(), W.cuda().reshape(E * N, K), seg, E, N, out_dtype=dt)
        torch.cuda.synchronize()
        got = f64(C)[:r["Mp"]]
        assert rel_l2(got, want) <= tol, dt
        for e in range(E):
            s0, s1 = r["seg_off"][e], r["seg_off"][e] + r["m_splits"][e]
            if s1 > s0:
                assert rel_l2(got[s0:s1], want[s0:s1]) <= tol, (dt, e)


@pytest.mark.parametrize("counts,N,K2", [
    ([300, 0, 129, 1, 640], 256, 256),
    ([1000, 500, 31, 33], 512, 768),
])
def test_grouped_gemm_bf16_wgrad(gpu_lib, counts, N, K2):
    r, cap = _routed(counts, seed=2)
    E = len(counts)
    T = sum(counts)
    a = wl.random_matrix(T, N, seed=21)
    b = wl.random_matrix(T, K2, seed=22)
    live = torch.from_numpy(r["token_of_row"] >= 0)
    tor = torch.from_numpy(r["token_of_row"][r["token_of_row"] >= 0])
    Ap = torch.zeros((cap, N), dtype=torch.bfloat16)
    Bp = torch.zeros((cap, K2), dtype=torch.bfloat16)
    Ap[:r["Mp"]][live] = a[tor]
    Bp[:r["Mp"]][live] = b[tor]
    seg = torch.tensor(r["seg_off"], dtype=torch.int32, device="cuda")
    C = torch.full((E, N, K2), float("nan"), device="cuda")
    gpu_lib.grouped_gemm_bf16_wgrad(Ap.t().contiguous().cuda(), Bp.t().contiguous().cuda(), seg, E, out=C)
    torch.cuda.synchronize()
    want = omoe.grouped_gemm_wgrad(f64(Ap[:r["Mp"]]).T, f64(Bp[:r["Mp"]]).T, r["seg_off"])
    got = f64(C)
    for e in range(E):
        if counts[e] == 0:
            assert np.all(got[e] == 0), e
        else:
            assert rel_l2(got[e], want[e]) <= 5e-4, e
