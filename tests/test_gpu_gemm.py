"""GPU parity of the MXFP8 grouped GEMMs (tcgen05 block-scaled) with the oracle.

Both sides quantise the same seeded bf16 inputs independently (bit-exact, pinned by
test_gpu_quantize); the oracle then multiplies the dequantised operands in fp64 one
expert at a time. Bar: relative L2 <= 5e-3 per GEMM stage."""
import numpy as np
import pytest
import torch

import moe_workloads as wl
from oracle import moe as omoe
from oracle import mxfp8 as omx
from tests.util import f64, rel_l2, SEG_ALIGN

pytestmark = pytest.mark.gpu
TOL_GEMM = 5e-3   # bf16 output: the stated bar per GEMM stage
TOL_F32 = 5e-4    # fp32 output: fp32 accumulation over K <= 4096 terms stays well inside K * 2^-24


@pytest.fixture(params=["pair", "single"])
def variant(request, monkeypatch):
    """Both kernel variants: CTA pairs (256-row tiles, default) and one CTA per tile."""
    monkeypatch.setenv("MXMOE_GEMM_PAIR", "2" if request.param == "pair" else "1")
    return request.param


def _segments(counts):
    E = len(counts)
    idx = []
    for e, c in enumerate(counts):
        idx += [e] * c
    idx = torch.tensor(idx, dtype=torch.int32).reshape(-1, 1)
    return idx, E


def _dense_perm_input(gpu_lib, counts, K, seed):
    """Permuted [cap, K] bf16 rows (pad rows zero) + the GPU routing maps for k = 1."""
    idx, E = _segments(counts)
    T = idx.shape[0]
    probs = torch.ones((T, 1))
    out = gpu_lib.moe_permute(idx.cuda(), probs.cuda(), E)
    x = wl.random_matrix(T, K, seed=seed)
    cap = gpu_lib.mxmoe_rows_capacity(T, 1, E)
    r = omoe.route(idx.numpy(), E, align=SEG_ALIGN)
    return x, out, cap, r, E


@pytest.mark.parametrize("N,K", [(256, 128), (256, 512), (512, 384)])
def test_single_tile_and_small(gpu_lib, variant, N, K):
    """One expert, one or two 256-column tiles: the tcgen05 path in isolation."""
    A = wl.random_matrix(256, K, seed=11)
    B = wl.random_matrix(N, K, seed=12, std=0.05)
    seg = torch.tensor([0, 256], dtype=torch.int32, device="cuda")
    ar, _ = gpu_lib.mxfp8_quantize(A.cuda(), colwise=False)
    br, _ = gpu_lib.mxfp8_quantize(B.cuda(), colwise=False)
    for dt in (torch.float32, torch.bfloat16):
        C = gpu_lib.grouped_gemm_mxfp8(ar, br, seg, 1, N, out_dtype=dt)
        torch.cuda.synchronize()
        want = omx.fake_quant_rowwise(f64(A)) @ omx.fake_quant_rowwise(f64(B)).T
        err = rel_l2(f64(C), want)
        assert err <= (TOL_F32 if dt == torch.float32 else TOL_GEMM), (dt, err)


@pytest.mark.parametrize("counts,N,K", [
    ([300, 0, 129, 1, 640], 256, 256),
    ([1000, 500, 31, 33], 512, 1024),
    ([127, 129, 40, 700, 0, 0, 1, 255], 768, 384),
])
def test_grouped_gemm_ragged(gpu_lib, variant, counts, N, K):
    x, out, cap, r, E = _dense_perm_input(gpu_lib, counts, K, seed=sum(counts))
    xr, _ = gpu_lib.mxfp8_quantize(x.cuda(), colwise=False, row_gather=out["token_of_row"],
                                   nrows=out["seg_off"][E:], out_rows=cap)
    W = wl.random_matrix(N, K, seed=7, std=0.05, batch=E)
    wr, _ = gpu_lib.mxfp8_quantize(W.cuda(), colwise=False)
    C = gpu_lib.grouped_gemm_mxfp8(xr, wr, out["seg_off"], E, N, out_dtype=torch.float32)
    torch.cuda.synchronize()
    Xp = omoe.permute_rows(f64(x), r["token_of_row"])
    Bq = np.stack([omx.fake_quant_rowwise(f64(W[e])) for e in range(E)])
    want = omoe.grouped_gemm(omx.fake_quant_rowwise(Xp), Bq, r["seg_off"])
    Mp = r["Mp"]
    got = f64(C)[:Mp]
    assert rel_l2(got, want) <= TOL_F32
    # per-expert check so a misrouted expert cannot hide in the global norm
    for e in range(E):
        s0, s1 = r["seg_off"][e], r["seg_off"][e] + r["m_splits"][e]
        if s1 > s0:
            assert rel_l2(got[s0:s1], want[s0:s1]) <= TOL_F32, e


@pytest.mark.parametrize("counts,N,K2", [
    ([300, 0, 129, 1, 640], 256, 256),
    ([1000, 500, 31, 33], 512, 768),
])
def test_grouped_wgrad_ragged(gpu_lib, variant, counts, N, K2):
    idx, E = _segments(counts)
    T = idx.shape[0]
    out = gpu_lib.moe_permute(idx.cuda(), torch.ones((T, 1)).cuda(), E)
    cap = gpu_lib.mxmoe_rows_capacity(T, 1, E)
    a = wl.random_matrix(T, N, seed=21)
    b = wl.random_matrix(T, K2, seed=22)
    _, ac = gpu_lib.mxfp8_quantize(a.cuda(), rowwise=False, row_gather=out["token_of_row"],
                                   nrows=out["seg_off"][E:], out_rows=cap)
    _, bc = gpu_lib.mxfp8_quantize(b.cuda(), rowwise=False, row_gather=out["token_of_row"],
                                   nrows=out["seg_off"][E:], out_rows=cap)
    C = torch.full((E, N, K2), float("nan"), device="cuda")
    gpu_lib.grouped_gemm_mxfp8_wgrad(ac, bc, out["seg_off"], E, out=C)
    torch.cuda.synchronize()
    r = omoe.route(idx.numpy(), E, align=SEG_ALIGN)
    Ap = omoe.permute_rows(f64(a), r["token_of_row"])
    Bp = omoe.permute_rows(f64(b), r["token_of_row"])
    Aq = omoe.fake_quant_colwise_segments(Ap, r["seg_off"], r["m_splits"])
    Bq = omoe.fake_quant_colwise_segments(Bp, r["seg_off"], r["m_splits"])
    want = omoe.grouped_gemm_wgrad(Aq.T, Bq.T, r["seg_off"])
    got = f64(C)
    for e in range(E):
        if counts[e] == 0:
            assert np.all(got[e] == 0), e
        else:
            assert rel_l2(got[e], want[e]) <= TOL_F32, e


@pytest.mark.parametrize("seg", [[0, 128, 256], [0, 512, 256], [0, 256, 4096]])
def test_bad_segments_reported(gpu_lib, variant, seg):
    """Segment offsets that are misaligned, decreasing or past the operand rows are
    caught on the device: nothing is written and the device status says so."""
    if variant == "single" and seg == [0, 128, 256]:
        pytest.skip("128-row segments are valid for single-CTA tiles")
    A = wl.random_matrix(512, 256, seed=31)
    B = wl.random_matrix(2 * 256, 256, seed=32, std=0.05)
    ar, _ = gpu_lib.mxfp8_quantize(A.cuda(), colwise=False)
    br, _ = gpu_lib.mxfp8_quantize(B.cuda(), colwise=False)
    gpu_lib.mxmoe_clear_device_status()
    C = torch.full((512, 256), 7.0, device="cuda")
    gpu_lib.grouped_gemm_mxfp8(ar, br, torch.tensor(seg, dtype=torch.int32, device="cuda"), 2, 256, out=C)
    torch.cuda.synchronize()
    st, _ = gpu_lib.mxmoe_get_device_status()
    gpu_lib.mxmoe_clear_device_status()
    assert st == 6  # MXMOE_ERR_DEVICE_CHECK
    assert torch.all(C == 7.0)
