"""GPU parity of the router (softmax over all experts, top-k, backward) with the oracle:
selected experts bit-exact (the decision is taken on the same fp32 logits), probabilities
and logit gradients within fp32 rounding of the fp64 oracle."""
import numpy as np
import pytest
import torch

from oracle import router as orouter
from tests.util import f64, rel_l2

pytestmark = pytest.mark.gpu


def _logits(T, E, seed, kind):
    g = torch.Generator().manual_seed(seed)
    l = torch.randn((T, E), generator=g)
    if kind == "ties":            # few distinct values: many equal logits per row
        l = torch.round(l * 1.5)
    elif kind == "dead":          # some experts forbidden for some tokens
        mask = torch.rand((T, E), generator=g) < 0.3
        mask[:, 0] = False        # keep one finite logit per row
        l[mask] = -float("inf")
    return l.float().contiguous()


@pytest.mark.parametrize("T,E,k,kind", [
    (1000, 8, 2, "randn"), (777, 64, 8, "randn"), (300, 256, 4, "randn"), (64, 5, 5, "randn"),
    (33, 1, 1, "randn"), (513, 8, 2, "ties"), (200, 100, 8, "ties"), (400, 32, 6, "dead"), (129, 256, 8, "dead"),
])
def test_router_matches_oracle(gpu_lib, T, E, k, kind):
    l = _logits(T, E, seed=T + E + k, kind=kind)
    gpu_lib.mxmoe_clear_device_status()
    idx, probs = gpu_lib.moe_router_topk(l.cuda(), k)
    torch.cuda.synchronize()
    assert gpu_lib.mxmoe_get_device_status()[0] == 0
    want_idx, want_p = orouter.topk(l.numpy(), k)
    np.testing.assert_array_equal(idx.cpu().numpy(), want_idx)
    np.testing.assert_allclose(f64(probs), want_p, rtol=4e-6, atol=1e-30)
    # backward of L = sum w * probs
    w = torch.randn((T, k), generator=torch.Generator().manual_seed(7)).float()
    dl = gpu_lib.moe_router_topk_bwd(l.cuda(), idx, w.cuda())
    torch.cuda.synchronize()
    want = orouter.topk_backward(l.numpy(), want_idx, w.numpy())
    assert rel_l2(f64(dl), want) <= 1e-5
    assert torch.isfinite(dl).all()


def test_router_rejects_rows_without_finite_logit(gpu_lib):
    l = torch.randn((40, 8))
    l[5] = -float("inf")
    l[9, 3] = float("nan")
    gpu_lib.mxmoe_clear_device_status()
    idx, probs = gpu_lib.moe_router_topk(l.cuda(), 2)
    torch.cuda.synchronize()
    st, _ = gpu_lib.mxmoe_get_device_status()
    gpu_lib.mxmoe_clear_device_status()
    assert st == 6  # MXMOE_ERR_DEVICE_CHECK
    idx = idx.cpu().numpy()
    assert (idx[5] == -1).all() and (idx[9] == -1).all()
    good = [t for t in range(40) if t not in (5, 9)]
    want_idx, _ = orouter.topk(l.numpy()[good], 2)
    np.testing.assert_array_equal(idx[good], want_idx)


def test_router_feeds_the_layer(gpu_lib):
    """Router output drives moe_permute directly: the routing maps equal the oracle's."""
    from oracle import moe as omoe
    from tests.util import SEG_ALIGN
    T, E, k = 2048, 16, 2
    l = _logits(T, E, seed=3, kind="randn")
    idx, probs = gpu_lib.moe_router_topk(l.cuda(), k)
    out = gpu_lib.moe_permute(idx, probs, E)
    torch.cuda.synchronize()
    want_idx, _ = orouter.topk(l.numpy(), k)
    r = omoe.route(want_idx, E, align=SEG_ALIGN)
    np.testing.assert_array_equal(out["m_splits"].cpu().numpy(), r["m_splits"])
    np.testing.assert_array_equal(out["seg_off"].cpu().numpy(), r["seg_off"])
