"""GPU parity of moe_permute / moe_unpermute with the oracle (bit-exact indices)."""
import numpy as np
import pytest
import torch

import moe_workloads as wl
from oracle import moe as omoe
from tests.util import f64, SEG_ALIGN

pytestmark = pytest.mark.gpu


def _check_route(mx, idx, probs, E):
    out = mx.moe_permute(idx.cuda(), probs.cuda(), E)
    torch.cuda.synchronize()
    r = omoe.route(idx.numpy(), E, align=SEG_ALIGN)
    np.testing.assert_array_equal(out["m_splits"].cpu().numpy(), r["m_splits"])
    np.testing.assert_array_equal(out["seg_off"].cpu().numpy(), r["seg_off"])
    np.testing.assert_array_equal(out["row_of_slot"].cpu().numpy(), r["row_of_slot"])
    Mp = r["Mp"]
    np.testing.assert_array_equal(out["token_of_row"].cpu().numpy()[:Mp], r["token_of_row"])
    por = out["prob_of_row"].cpu().numpy()[:Mp]
    live = r["token_of_row"] >= 0
    want = np.zeros(Mp, dtype=np.float32)
    want[live] = probs.numpy()[r["token_of_row"][live], r["slot_of_row"][live]]
    np.testing.assert_array_equal(por, want)
    return out, r


@pytest.mark.parametrize("name", ["tiny", "small", "mixtral_zipf"])
def test_permute_configs(gpu_lib, name):
    cfg = wl.CONFIGS[name]
    idx, probs = wl.make_routing(cfg)
    out, r = _check_route(gpu_lib, idx, probs, cfg.E)
    if name == "small":
        assert r["m_splits"][cfg.E - 1] == 0
    if name == "mixtral_zipf":
        assert r["m_splits"][cfg.E - 1] == wl.ZIPF_SMALL_EXPERT_TOKENS


def test_permute_genomics_shape(gpu_lib):
    cfg = wl.custom(T=6000, H=256, F=256, E=64, k=8, seed=31)
    idx, probs = wl.make_routing(cfg)
    _check_route(gpu_lib, idx, probs, cfg.E)


def test_permute_ragged_counts(gpu_lib):
    """Experts with 0, 1, 31, 33, 127, 129, 40 and the rest of the tokens (k = 1)."""
    counts = [0, 1, 31, 33, 127, 129, 40]
    T = 700
    idx = []
    for e, c in enumerate(counts):
        idx += [e] * c
    idx += [7] * (T - len(idx))
    g = torch.Generator().manual_seed(5)
    perm = torch.randperm(T, generator=g)
    idx = torch.tensor(idx, dtype=torch.int32)[perm].reshape(T, 1)
    probs = torch.rand((T, 1), generator=g)
    out, r = _check_route(gpu_lib, idx, probs, 8)
    assert r["m_splits"].tolist() == counts + [T - sum(counts)]


def test_permute_all_on_one_expert(gpu_lib):
    T = 1000
    idx = torch.zeros((T, 1), dtype=torch.int32)
    probs = torch.ones((T, 1))
    out, r = _check_route(gpu_lib, idx, probs, 4)
    assert r["m_splits"].tolist() == [T, 0, 0, 0]


def test_permute_invalid_ids_flagged(gpu_lib):
    gpu_lib.mxmoe_clear_device_status()
    idx = torch.tensor([[0, 1], [2, 2], [1, 9]], dtype=torch.int32)
    probs = torch.ones((3, 2))
    out = gpu_lib.moe_permute(idx.cuda(), probs.cuda(), 4)
    st, where = gpu_lib.mxmoe_get_device_status()
    assert st == 6      # MXMOE_ERR_DEVICE_CHECK
    ros = out["row_of_slot"].cpu().numpy()
    assert ros[1, 1] == -1 and ros[2, 1] == -1 and ros[0, 0] >= 0
    gpu_lib.mxmoe_clear_device_status()
    assert gpu_lib.mxmoe_get_device_status()[0] == 0


@pytest.mark.parametrize("k,H,shift", [(2, 256, 0), (8, 2048, 0), (1, 1024, 0), (4, 264, 0), (3, 512, 8),
                                         (2, 1024, 8)])
def test_unpermute_matches_oracle(gpu_lib, k, H, shift):
    """Combine of the routed rows. H % 16 != 0, or a source only 16-byte aligned (`shift`
    bf16 elements into an aligned buffer), takes the 16-byte path; k = 3, 4 the four-slot
    variant."""
    E = 8
    T = 500
    cfg = wl.custom(T=T, H=H, F=256, E=E, k=k, seed=40 + k)
    idx, probs = wl.make_routing(cfg)
    out = gpu_lib.moe_permute(idx.cuda(), probs.cuda(), E)
    cap = gpu_lib.mxmoe_rows_capacity(T, k, E)
    yp = wl.random_matrix(cap, H, seed=3)
    buf = torch.zeros(cap * H + shift, dtype=torch.bfloat16, device="cuda")
    yp_dev = buf[shift:].view(cap, H)
    yp_dev.copy_(yp.cuda())
    y = gpu_lib.moe_unpermute(yp_dev, out["row_of_slot"])
    torch.cuda.synchronize()
    r = omoe.route(idx.numpy(), E, align=SEG_ALIGN)
    want = omoe.unpermute_sum(f64(yp), r["row_of_slot"])
    got = f64(y)
    # one rounding to bf16 of an fp32 sum: within one bf16 ulp of the exact sum
    ulp = np.maximum(np.abs(want), 1e-30) * 2.0 ** -8
    assert np.all(np.abs(got - want) <= ulp + 1e-30)
    # and bit-exact where the fp32 sum is exact (k <= 2 of bf16 values)
    if k <= 2:
        np.testing.assert_array_equal(got, f64(torch.from_numpy(want).to(torch.bfloat16)))
