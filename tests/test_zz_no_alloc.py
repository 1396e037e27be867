"""moe_permute_noalloc -- the routing index without a caller-provided scratch buffer.

For callers that cannot lend the library device memory per call (runtimes with a fixed
memory plan, plain C callers without an allocator). Checked through the C ABI against
moe_permute (which takes a workspace) on two calls in a row with different problems:
the outputs are indices and routing probabilities, so they must match exactly. The maps
are also compared with the oracle's routing directly. Kept in its own file, collected
last."""
import ctypes

import numpy as np
import pytest
import torch

import moe_workloads as wl
from oracle import moe as omoe
from tests.util import SEG_ALIGN

pytestmark = pytest.mark.gpu


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def _outputs(T, k, E, cap, dev):
    return dict(m_splits=torch.full((E,), -7, dtype=torch.int32, device=dev),
                seg_off=torch.full((E + 1,), -7, dtype=torch.int32, device=dev),
                row_of_slot=torch.full((T, k), -7, dtype=torch.int32, device=dev),
                token_of_row=torch.full((cap,), -7, dtype=torch.int32, device=dev),
                prob_of_row=torch.full((cap,), -7.0, dtype=torch.float32, device=dev))


def _call(lib, fn, idx, probs, E, ws=None):
    T, k = idx.shape
    cap = lib.mxmoe_rows_capacity(T, k, E)
    o = _outputs(T, k, E, cap, idx.device)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    args = [_ptr(idx), _ptr(probs), T, k, E, _ptr(o["m_splits"]), _ptr(o["seg_off"]), _ptr(o["row_of_slot"]),
            _ptr(o["token_of_row"]), _ptr(o["prob_of_row"])]
    if fn == "moe_permute":
        args += [_ptr(ws), ws.numel()]
    st = getattr(lib, fn)(*args, stream)
    assert st == 0, (fn, st)
    torch.cuda.synchronize()
    return o


def test_noalloc_matches_workspace_entry_point_twice(gpu_lib):
    lib = gpu_lib.load()
    problems = [wl.custom(T=3000, H=256, F=256, E=8, k=2, seed=51),
                wl.custom(T=5000, H=256, F=256, E=64, k=8, seed=52)]
    for cfg in problems:   # two calls in a row, different sizes, sharing the scratch array
        idx, probs = wl.make_routing(cfg)
        idx, probs = idx.cuda(), probs.cuda()
        ws = torch.empty(lib.moe_permute_workspace_size(cfg.T, cfg.k, cfg.E), dtype=torch.uint8, device="cuda")
        want = _call(lib, "moe_permute", idx, probs, cfg.E, ws)
        got = _call(lib, "moe_permute_noalloc", idx, probs, cfg.E)
        Mp = int(want["seg_off"][cfg.E])
        for name in ("m_splits", "seg_off", "row_of_slot"):
            assert torch.equal(got[name], want[name]), name
        assert torch.equal(got["token_of_row"][:Mp], want["token_of_row"][:Mp])
        assert torch.equal(got["prob_of_row"][:Mp], want["prob_of_row"][:Mp])
        assert int(got["m_splits"].sum()) == cfg.T * cfg.k
        # the oracle's counting sort (same 256-row segment alignment), bit for bit
        r = omoe.route(idx.cpu().numpy(), cfg.E, align=SEG_ALIGN)
        np.testing.assert_array_equal(got["m_splits"].cpu().numpy(), r["m_splits"])
        np.testing.assert_array_equal(got["seg_off"].cpu().numpy(), r["seg_off"])
        np.testing.assert_array_equal(got["row_of_slot"].cpu().numpy(), r["row_of_slot"])
        np.testing.assert_array_equal(got["token_of_row"][:Mp].cpu().numpy(), r["token_of_row"])
        live = r["token_of_row"] >= 0
        want_p = probs.cpu().numpy()[r["token_of_row"][live], r["slot_of_row"][live]]
        np.testing.assert_array_equal(got["prob_of_row"][:Mp].cpu().numpy()[live], want_p)


def test_noalloc_rejects_problems_beyond_its_scratch(gpu_lib):
    """A problem whose scratch exceeds the fixed array is refused before anything is
    enqueued: real device buffers are passed and stay untouched."""
    lib = gpu_lib.load()
    T, k, E = 70000, 2, 256            # needs 8 * 274 * 256 + 256 bytes > 256 KiB
    idx = torch.zeros((T, k), dtype=torch.int32, device="cuda")
    idx[:, 1] = 1
    probs = torch.full((T, k), 0.5, dtype=torch.float32, device="cuda")
    o = _outputs(T, k, E, lib.mxmoe_rows_capacity(T, k, E), "cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = lib.moe_permute_noalloc(_ptr(idx), _ptr(probs), T, k, E, _ptr(o["m_splits"]), _ptr(o["seg_off"]),
                                 _ptr(o["row_of_slot"]), _ptr(o["token_of_row"]), _ptr(o["prob_of_row"]), stream)
    assert st == 3                      # MXMOE_ERR_WORKSPACE_TOO_SMALL
    torch.cuda.synchronize()
    for name in ("m_splits", "seg_off", "row_of_slot", "token_of_row"):
        assert bool((o[name] == -7).all()), name
