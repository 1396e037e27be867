"""Failure detection on the device: a bounded wait that runs out ends the kernel with a
status, not a hang or a trap (no fault is provoked; the wait is made to expire by a flag
that withholds one signal).

grouped_gemm_mxfp8_debug_timeout runs the grouped GEMM with the first CTA pair's
accumulator-ready signal withheld. The call must return, the kernel must finish within a
few seconds (each wait gives up after 1 s), the device status word must read
MXMOE_ERR_DEVICE_TIMEOUT and clear on request, and the next normal call on the same
operands must be correct -- the context stays usable."""
import time

import numpy as np
import pytest
import torch

import moe_workloads as wl
from oracle import mxfp8 as omx
from tests.util import f64, rel_l2

pytestmark = pytest.mark.gpu
TOL_GEMM = 5e-3
WAIT_SITES = {1, 2, 3, 4, 7}   # producer, MMA (accumulator / operands), epilogue, scale copies


@pytest.fixture(params=["pair", "single"])
def variant(request, monkeypatch):
    monkeypatch.setenv("MXMOE_GEMM_PAIR", "2" if request.param == "pair" else "1")
    return request.param


@pytest.mark.parametrize("rows", [512, 256 * 160])   # one tile on the first CTA (pair), or several
def test_withheld_signal_times_out_and_context_recovers(gpu_lib, variant, rows):
    N, K = 256, 256
    A = wl.random_matrix(rows, K, seed=61)
    B = wl.random_matrix(N, K, seed=62, std=0.05)
    seg = torch.tensor([0, rows], dtype=torch.int32, device="cuda")
    ar, _ = gpu_lib.mxfp8_quantize(A.cuda(), colwise=False)
    br, _ = gpu_lib.mxfp8_quantize(B.cuda(), colwise=False)
    C = torch.zeros((rows, N), dtype=torch.bfloat16, device="cuda")
    torch.cuda.synchronize()
    gpu_lib.mxmoe_clear_device_status()
    t0 = time.monotonic()
    gpu_lib.grouped_gemm_mxfp8_debug_timeout(ar, br, seg, 1, N, C)
    torch.cuda.synchronize()
    dt = time.monotonic() - t0
    st, where = gpu_lib.mxmoe_get_device_status()
    assert st == 5, (st, where)                      # MXMOE_ERR_DEVICE_TIMEOUT
    assert where in WAIT_SITES, where
    assert 0.9 < dt < 10.0, dt                       # the 1 s limit ran out; nothing hung
    gpu_lib.mxmoe_clear_device_status()
    assert gpu_lib.mxmoe_get_device_status() == (0, 0)
    # the context is intact: the same GEMM, called normally, is right
    C2 = gpu_lib.grouped_gemm_mxfp8(ar, br, seg, 1, N, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert gpu_lib.mxmoe_get_device_status()[0] == 0
    want = omx.fake_quant_rowwise(f64(A[:1024])) @ omx.fake_quant_rowwise(f64(B)).T
    assert rel_l2(f64(C2[:1024]), want) <= TOL_GEMM
    assert np.isfinite(f64(C2)).all()
