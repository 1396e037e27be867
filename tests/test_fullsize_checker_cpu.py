"""The sampled full-size parity checker of test_gpu_fullsize.py, run on the CPU against the
oracle's own whole-tensor outputs on small problems: the sampled y, dX, dprobs and dW1
values it rebuilds one token / one entry at a time must equal the oracle's forward and
backward (so the checker cannot pass a wrong layer by computing the same wrong thing)."""
import concurrent.futures as cf
import multiprocessing as mp

import numpy as np
import pytest
import torch

import moe_workloads as wl
from oracle import moe as omoe
from tests import test_gpu_fullsize as fs
from tests.util import SEG_ALIGN


@pytest.fixture(scope="module")
def pool():
    with cf.ProcessPoolExecutor(max_workers=2, mp_context=mp.get_context("spawn")) as ex:
        yield ex


@pytest.mark.parametrize("E,k", [(4, 2), (8, 4)])
def test_sampled_checker_agrees_with_oracle(pool, E, k, monkeypatch, capsys):
    cfg = wl.custom("chk", T=160, H=64, F=96, E=E, k=k, seed=31)
    d = wl.make_all(cfg)
    x, W1, W2, p = (d[n].double().numpy() for n in ("x", "W1", "W2", "probs"))
    idx, dy = d["topk_idx"].numpy(), d["dy"].double().numpy()
    y, saved = omoe.mlp_fwd(x, idx, p, W1, W2)
    g = omoe.mlp_bwd(dy, saved, p, W1, W2)
    outs = tuple(torch.from_numpy(v) for v in (y, g["dx"], g["dW1"], g["dW2"], g["dprobs"]))
    r = omoe.route(idx, E, align=SEG_ALIGN)
    monkeypatch.setattr(fs, "NCOLS", 32)
    # the same arithmetic, so agreement to rounding; the outputs pass through fp32 on the
    # way in (as the GPU's do), so the bar is fp32's relative precision with margin
    monkeypatch.setattr(fs, "TOL_E2E", 1e-6)
    fs._check_layer_outputs(cfg, r, idx, p, x, dy, torch.from_numpy(W1), torch.from_numpy(W2), outs, [0],
                            np.random.default_rng(0), pool)
    assert "tokens" in capsys.readouterr().out


@pytest.mark.parametrize("which", ["y", "dx", "dW1", "dprobs"])
def test_sampled_checker_catches_a_wrong_output(pool, monkeypatch, which):
    """A layer with one output off by 5 % fails the 2e-2 bar on that output."""
    cfg = wl.custom("chk", T=160, H=64, F=96, E=4, k=2, seed=32)
    d = wl.make_all(cfg)
    x, W1, W2, p = (d[n].double().numpy() for n in ("x", "W1", "W2", "probs"))
    idx, dy = d["topk_idx"].numpy(), d["dy"].double().numpy()
    y, saved = omoe.mlp_fwd(x, idx, p, W1, W2)
    g = omoe.mlp_bwd(dy, saved, p, W1, W2)
    vals = dict(y=y, dx=g["dx"], dW1=g["dW1"], dW2=g["dW2"], dprobs=g["dprobs"])
    vals[which] = 1.05 * vals[which]
    outs = tuple(torch.from_numpy(vals[n]) for n in ("y", "dx", "dW1", "dW2", "dprobs"))
    r = omoe.route(idx, cfg.E, align=SEG_ALIGN)
    monkeypatch.setattr(fs, "NCOLS", 32)
    with pytest.raises(AssertionError, match=which):
        fs._check_layer_outputs(cfg, r, idx, p, x, dy, torch.from_numpy(W1), torch.from_numpy(W2), outs, [0],
                                np.random.default_rng(0), pool)
