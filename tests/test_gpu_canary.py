"""Out-of-bounds writes on the device, caught without a sanitizer: every buffer the
library writes during a forward + backward (outputs, saved activations, workspace,
quantised weights) and during the standalone calls sits between guard regions of a known
byte pattern, which must be intact afterwards. Shapes with ragged experts and an empty
one, so that segment tails and pad rows are exercised."""
import ctypes

import pytest
import torch

import moe_workloads as wl

pytestmark = pytest.mark.gpu
GUARD = 4096
PATTERN = 0xA5


class Guarded:
    """A device byte buffer of n bytes with GUARD pattern bytes on each side."""

    def __init__(self, n, dev="cuda"):
        self.raw = torch.full((n + 2 * GUARD,), PATTERN, dtype=torch.uint8, device=dev)
        self.n = n

    def view(self, dtype=torch.uint8, shape=None):
        v = self.raw[GUARD:GUARD + self.n].view(dtype)
        return v.view(shape) if shape is not None else v

    def intact(self):
        return bool((self.raw[:GUARD] == PATTERN).all()) and bool((self.raw[GUARD + self.n:] == PATTERN).all())


def _nbytes(shape, dtype):
    n = torch.tensor([], dtype=dtype).element_size()
    for s in shape:
        n *= s
    return n


@pytest.mark.parametrize("recipe", ["mxfp8", "fp8", "bf16"])
def test_layer_writes_stay_inside_their_buffers(gpu_lib, recipe):
    mx = gpu_lib
    lib = mx.load()
    cfg = wl.custom("canary", T=700, H=256, F=512, E=5, k=2, seed=81, routing="dead_last")
    d = {k: v.cuda() for k, v in wl.make_all(cfg).items()}
    T, k, E, H, F = cfg.T, cfg.k, cfg.E, cfg.H, cfg.F
    if recipe == "bf16":
        sizes = (lib.grouped_mlp_bf16_saved_size(T, k, E, H, F), lib.grouped_mlp_bf16_workspace_size(T, k, E, H, F),
                 lib.mxmoe_weights_bf16_size(E, H, F))
    else:
        rc = mx.RECIPE_FP8_TENSOR if recipe == "fp8" else 0
        sizes = (lib.grouped_mlp_saved_size_ex(T, k, E, H, F, rc), lib.grouped_mlp_workspace_size_ex(T, k, E, H, F, rc),
                 lib.mxmoe_weights_size(E, H, F))
    saved, ws, wq = (Guarded(n) for n in sizes)
    outs = {n: Guarded(_nbytes(s, dt)) for n, s, dt in (
        ("y", (T, H), torch.bfloat16), ("dx", (T, H), torch.bfloat16), ("dW1", (E, 2 * F, H), torch.float32),
        ("dW2", (E, H, F), torch.float32), ("dprobs", (T, k), torch.float32))}
    o = {n: g.view(dt, s) for (n, g), (s, dt) in zip(outs.items(), (
        ((T, H), torch.bfloat16), ((T, H), torch.bfloat16), ((E, 2 * F, H), torch.float32),
        ((E, H, F), torch.float32), ((T, k), torch.float32)))}
    sv, w, q = saved.view(), ws.view(), wq.view()
    mx.mxmoe_clear_device_status()
    if recipe == "bf16":
        mx.mxmoe_weights_bf16_prepare(d["W1"], d["W2"], out=q)
        mx.grouped_mlp_bf16_fwd(d["x"], d["topk_idx"], d["probs"], q, E, F, sv, w, o["y"])
        mx.grouped_mlp_bf16_bwd(d["dy"], sv, q, T, k, E, H, F, w, o["dx"], o["dW1"], o["dW2"], o["dprobs"])
    elif recipe == "fp8":
        state = Guarded(16)
        st = state.view(torch.float32)
        st.fill_(1.0)
        mx.mxmoe_weights_quantize_fp8(d["W1"], d["W2"], out=q)
        mx.grouped_mlp_fp8_fwd(d["x"], d["topk_idx"], d["probs"], q, E, F, st, sv, w, o["y"])
        mx.grouped_mlp_fp8_bwd(d["dy"], sv, q, T, k, E, H, F, st, w, o["dx"], o["dW1"], o["dW2"], o["dprobs"])
        torch.cuda.synchronize()
        assert state.intact()
    else:
        mx.mxmoe_weights_quantize(d["W1"], d["W2"], out=q)
        mx.grouped_mlp_fwd(d["x"], d["topk_idx"], d["probs"], q, E, F, sv, w, o["y"])
        mx.grouped_mlp_bwd(d["dy"], sv, q, T, k, E, H, F, w, o["dx"], o["dW1"], o["dW2"], o["dprobs"])
    torch.cuda.synchronize()
    assert mx.mxmoe_get_device_status()[0] == 0
    for name, g in list(outs.items()) + [("saved", saved), ("workspace", ws), ("weights", wq)]:
        assert g.intact(), name
    assert torch.isfinite(o["y"].float()).all() and torch.isfinite(o["dx"].float()).all()


def test_standalone_calls_write_inside_their_buffers(gpu_lib):
    """Routing maps, the gathered quantiser, the grouped GEMMs and the combine, each into
    guarded outputs."""
    mx = gpu_lib
    lib = mx.load()
    T, k, E, H = 600, 2, 7, 256
    cfg = wl.custom("canary2", T=T, H=H, F=256, E=E, k=k, seed=82)
    idx, probs = (t.cuda() for t in wl.make_routing(cfg))
    x = wl.make_activations(cfg).cuda()
    cap = mx.mxmoe_rows_capacity(T, k, E)
    g = {n: Guarded(b) for n, b in (("m", E * 4), ("seg", (E + 1) * 4), ("ros", T * k * 4), ("tor", cap * 4),
                                    ("por", cap * 4), ("ws", lib.moe_permute_workspace_size(T, k, E)),
                                    ("xr", cap * H), ("xrs", cap * H // 32), ("xc", cap * H), ("xcs", cap * H // 32),
                                    ("y", T * H * 2))}
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    P = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    assert lib.moe_permute(P(idx), P(probs), T, k, E, P(g["m"].view()), P(g["seg"].view()), P(g["ros"].view()),
                           P(g["tor"].view()), P(g["por"].view()), P(g["ws"].view()), g["ws"].n, stream) == 0
    xr = mx.MXFP8(g["xr"].view().view(cap, H), g["xrs"].view(), mx.SCALE_MMA)
    xc = mx.MXFP8(g["xc"].view().view(H, cap), g["xcs"].view(), mx.SCALE_MMA)
    seg = g["seg"].view(torch.int32)
    st = lib.mxfp8_quantize(P(x), mx.DTYPE_BF16, 1, T, H, P(g["tor"].view()), ctypes.c_void_p(seg.data_ptr() + 4 * E),
                            cap, ctypes.byref(xr.as_struct()), ctypes.byref(xc.as_struct()), stream)
    assert st == 0
    yp = torch.randn((cap, H), device="cuda").to(torch.bfloat16)
    lib.moe_unpermute(P(yp), P(g["ros"].view()), T, k, H, P(g["y"].view()), stream)
    torch.cuda.synchronize()
    assert mx.mxmoe_get_device_status()[0] == 0
    for name, gg in g.items():
        assert gg.intact(), name
