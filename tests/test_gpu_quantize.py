"""GPU parity of mxfp8_quantize with the oracle's quantiser: bytes and scales bit-exact."""
import math
import os

import numpy as np
import pytest
import torch

import moe_workloads as wl
from oracle import moe as omoe
from oracle import mxfp8 as omx
from tests.util import f64, u8, SEG_ALIGN

pytestmark = pytest.mark.gpu
GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "mxfp8_blocks.txt")


def _golden():
    rows = []
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        name, vals, scale, codes = [f.strip() for f in line.split("|")]
        v = np.zeros(32)
        for it in vals.split(","):
            p, x = it.split(":")
            x = x.strip()
            v[int(p)] = float(x.split("*2^")[0]) * math.ldexp(1.0, int(x.split("*2^")[1])) if "*2^" in x else float(x)
        rows.append((name, v, int(scale, 16), {int(p): int(c, 16) for p, c in (i.split(":") for i in codes.split(","))}))
    return rows


def test_golden_blocks_on_gpu(gpu_lib):
    """The hand-built blocks, quantised by the GPU (fp32 input), rowwise and colwise."""
    blocks = _golden()
    n = len(blocks)
    src = np.zeros((max(32, n), 32), dtype=np.float32)
    for i, (_, v, _, _) in enumerate(blocks):
        src[i] = v
    t = torch.from_numpy(src).cuda()
    r, c = gpu_lib.mxfp8_quantize(t, layout=gpu_lib.SCALE_PLAIN)
    codes = u8(r.data)
    sc = u8(r.scale_plain())
    for i, (name, v, scale, exp) in enumerate(blocks):
        assert sc[i, 0] == scale, name
        for p, cc in exp.items():
            assert codes[i, p] == cc, (name, p, hex(codes[i, p]), hex(cc))
    # colwise of the transposed input gives the same bytes
    r2, c2 = gpu_lib.mxfp8_quantize(torch.from_numpy(np.ascontiguousarray(src.T)).cuda(), rowwise=False,
                                    layout=gpu_lib.SCALE_PLAIN)
    np.testing.assert_array_equal(u8(c2.data), codes)
    np.testing.assert_array_equal(u8(c2.scale_plain()), sc)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("layout", [0, 1])
@pytest.mark.parametrize("shape", [(256, 384), (384, 128), (128, 4096)])
def test_quantize_matches_oracle(gpu_lib, dtype, layout, shape):
    R, C = shape
    x = wl.random_matrix(R, C, seed=R + C, dtype=torch.float32)
    # widen the dynamic range: per-row powers of two from 2^-40 to 2^40
    g = torch.Generator().manual_seed(1)
    x = x * torch.exp2(torch.randint(-40, 40, (R, 1), generator=g).float())
    x[3, :40] = 0.0                      # an all-zero block
    x[5, 7] = -1e-30                     # tiny negative next to normal values
    x = x.to(dtype)
    r, c = gpu_lib.mxfp8_quantize(x.cuda(), layout=layout)
    torch.cuda.synchronize()
    qr, sr = omx.quantize_rowwise(f64(x))
    qc, sc = omx.quantize_colwise_t(f64(x))
    np.testing.assert_array_equal(u8(r.data), qr)
    np.testing.assert_array_equal(u8(r.scale_plain()), sr)
    np.testing.assert_array_equal(u8(c.data), qc)
    np.testing.assert_array_equal(u8(c.scale_plain()), sc)


@pytest.mark.parametrize("shape", [(96, 160), (224, 32)])
def test_quantize_untiled_shapes(gpu_lib, shape):
    """bf16 shapes that are not multiples of 128 take the per-tile kernel (the dense
    persistent kernel needs whole 128 x 128 tiles); same bytes as the oracle."""
    R, C = shape
    x = wl.random_matrix(R, C, seed=R * C, dtype=torch.float32).to(torch.bfloat16)
    r, c = gpu_lib.mxfp8_quantize(x.cuda(), layout=gpu_lib.SCALE_PLAIN)
    torch.cuda.synchronize()
    qr, sr = omx.quantize_rowwise(f64(x))
    qc, sc = omx.quantize_colwise_t(f64(x))
    np.testing.assert_array_equal(u8(r.data), qr)
    np.testing.assert_array_equal(u8(r.scale_plain()), sr)
    np.testing.assert_array_equal(u8(c.data), qc)
    np.testing.assert_array_equal(u8(c.scale_plain()), sc)


def test_gathered_quantize_16_byte_aligned_buffers(gpu_lib):
    """The per-tile kernel's 32-byte loads and stores need 32-byte aligned rows; a source
    and outputs that are only 16-byte aligned take the 16-byte loads and the two-store
    path, with the same bytes as the oracle (gathered rows, zero rows for index -1)."""
    import ctypes
    lib = gpu_lib.load()
    R, C, OR = 200, 160, 224
    x = wl.random_matrix(R, C, seed=77, dtype=torch.float32).to(torch.bfloat16)
    g = torch.Generator().manual_seed(5)
    gather = torch.randint(-1, R, (OR,), generator=g, dtype=torch.int32)
    sbuf = torch.zeros(R * C + 8, dtype=torch.bfloat16, device="cuda")
    src = sbuf[8:].view(R, C)                         # 16 bytes into the buffer
    src.copy_(x.cuda())
    rbuf = torch.zeros(OR * C + 16, dtype=torch.uint8, device="cuda")
    cbuf = torch.zeros(C * OR + 16, dtype=torch.uint8, device="cuda")
    r = gpu_lib.MXFP8(rbuf[16:].view(OR, C), torch.zeros(OR * C // 32, dtype=torch.uint8, device="cuda"),
                      gpu_lib.SCALE_PLAIN)
    c = gpu_lib.MXFP8(cbuf[16:].view(C, OR), torch.zeros(C * OR // 32, dtype=torch.uint8, device="cuda"),
                      gpu_lib.SCALE_PLAIN)
    assert src.data_ptr() % 32 == 16 and r.data.data_ptr() % 32 == 16 and c.data.data_ptr() % 32 == 16
    gdev = gather.cuda()
    rs, cs = r.as_struct(), c.as_struct()
    st = lib.mxfp8_quantize(gpu_lib._ptr(src), gpu_lib.DTYPE_BF16, 1, R, C, gpu_lib._ptr(gdev), None, OR,
                            ctypes.byref(rs), ctypes.byref(cs), gpu_lib._stream())
    assert st == 0, gpu_lib.status_string(st)
    torch.cuda.synchronize()
    xp = np.zeros((OR, C))
    live = gather.numpy() >= 0
    xp[live] = f64(x)[gather.numpy()[live]]
    qr, sr = omx.quantize_rowwise(xp)
    qc, sc = omx.quantize_colwise_t(xp)
    np.testing.assert_array_equal(u8(r.data), qr)
    np.testing.assert_array_equal(u8(r.scale_plain()), sr)
    np.testing.assert_array_equal(u8(c.data), qc)
    np.testing.assert_array_equal(u8(c.scale_plain()), sc)


def test_quantize_batched_weights(gpu_lib):
    E, N, K = 3, 256, 384
    W = wl.random_matrix(N, K, seed=9, std=0.02, batch=E)
    r, c = gpu_lib.mxfp8_quantize(W.cuda())
    torch.cuda.synchronize()
    rd, rs = u8(r.data), u8(r.scale_plain())
    cd, cs = u8(c.data), u8(c.scale_plain())
    for e in range(E):
        qr, sr = omx.quantize_rowwise(f64(W[e]))
        qc, sc = omx.quantize_colwise_t(f64(W[e]))
        np.testing.assert_array_equal(rd[e * N:(e + 1) * N], qr)
        np.testing.assert_array_equal(rs[e * N:(e + 1) * N], sr)
        np.testing.assert_array_equal(cd[e * K:(e + 1) * K], qc)
        np.testing.assert_array_equal(cs[e * K:(e + 1) * K], sc)


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_permute_quantize_matches_oracle(gpu_lib, name):
    """Fused gather + quantise of the routed activations: rowwise along H, colwise in
    32-row blocks of each 128-aligned expert segment."""
    cfg = wl.CONFIGS[name]
    idx, probs = wl.make_routing(cfg)
    x = wl.make_activations(cfg)
    out = gpu_lib.moe_permute(idx.cuda(), probs.cuda(), cfg.E)
    cap = gpu_lib.mxmoe_rows_capacity(cfg.T, cfg.k, cfg.E)
    r, c = gpu_lib.mxfp8_quantize(x.cuda(), row_gather=out["token_of_row"], nrows=out["seg_off"][cfg.E:],
                                  out_rows=cap)
    torch.cuda.synchronize()
    ro = omoe.route(idx.numpy(), cfg.E, align=SEG_ALIGN)
    Mp = ro["Mp"]
    Xp = omoe.permute_rows(f64(x), ro["token_of_row"])
    qr, sr = omx.quantize_rowwise(Xp)
    qc, sc = omoe.quantize_colwise_segments(Xp, ro["seg_off"], ro["m_splits"])
    np.testing.assert_array_equal(u8(r.data)[:Mp], qr)
    np.testing.assert_array_equal(u8(r.scale_plain())[:Mp], sr)
    np.testing.assert_array_equal(u8(c.data)[:, :Mp], qc)
    np.testing.assert_array_equal(u8(c.scale_plain())[:, :Mp // 32], sc)


def test_weights_buffer_layout(gpu_lib):
    """mxmoe_weights_quantize: the four copies match the oracle byte for byte, the W1
    rowwise copy with each expert's gate and up rows interleaved in 64-row blocks."""
    E, H, F = 2, 256, 512
    W1 = wl.random_matrix(2 * F, H, seed=41, std=0.02, batch=E)
    W2 = wl.random_matrix(H, F, seed=42, std=0.02, batch=E)
    wq = gpu_lib.mxmoe_weights_quantize(W1.cuda(), W2.cuda())
    torch.cuda.synchronize()
    views = [gpu_lib.mxmoe_weights_view(wq, E, H, F, w) for w in range(4)]
    # destination row of W1 row r of one expert (gate rows 0..F-1, up rows F..2F-1)
    r = np.arange(2 * F)
    hf, rr = (r >= F).astype(int), r - (r >= F) * F
    dst = (rr // 64) * 128 + hf * 64 + rr % 64
    for e in range(E):
        qr, sr = omx.quantize_rowwise(f64(W1[e]))
        got, gsc = u8(views[0].data)[e * 2 * F:(e + 1) * 2 * F], u8(views[0].scale_plain())[e * 2 * F:(e + 1) * 2 * F]
        np.testing.assert_array_equal(got[dst], qr)
        np.testing.assert_array_equal(gsc[dst], sr)
        qc, sc = omx.quantize_colwise_t(f64(W1[e]))
        np.testing.assert_array_equal(u8(views[1].data)[e * H:(e + 1) * H], qc)
        np.testing.assert_array_equal(u8(views[1].scale_plain())[e * H:(e + 1) * H], sc)
        qr2, sr2 = omx.quantize_rowwise(f64(W2[e]))
        np.testing.assert_array_equal(u8(views[2].data)[e * H:(e + 1) * H], qr2)
        np.testing.assert_array_equal(u8(views[2].scale_plain())[e * H:(e + 1) * H], sr2)
        qc2, sc2 = omx.quantize_colwise_t(f64(W2[e]))
        np.testing.assert_array_equal(u8(views[3].data)[e * F:(e + 1) * F], qc2)
        np.testing.assert_array_equal(u8(views[3].scale_plain())[e * F:(e + 1) * F], sc2)


@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
def test_dequantize_rows_matches_oracle(gpu_lib, fmt):
    """mxfp8_dequantize: every element equals the oracle's element(code) * 2^(scale - 127)
    (exact in bf16 for these scales); re-quantising the dequantised rows gives back the same
    codes and scales (the rowwise round trip is lossless, which expert parallelism relies on
    when rows travel as MXFP8)."""
    mx = gpu_lib
    f = mx.FMT_E4M3 if fmt == "e4m3" else mx.FMT_E5M2
    g = torch.Generator().manual_seed(91)
    x = (torch.randn((300, 512), generator=g) * torch.exp2(torch.randint(-20, 20, (300, 1), generator=g).float()))
    x = x.to(torch.bfloat16)
    x[7] = 0                                    # an all-zero row (scale byte 0)
    xr = torch.nn.functional.pad(x, (0, 0, 0, 20)).cuda()   # 320 rows (multiple of 32)
    r, _ = mx.mxfp8_quantize(xr, colwise=False, layout=mx.SCALE_PLAIN, fmt=f)
    y = mx.mxfp8_dequantize(r)
    torch.cuda.synchronize()
    want = omx.dequantize_rowwise(u8(r.data), u8(r.scale_plain()), fmt=fmt)
    np.testing.assert_array_equal(f64(y.cpu()), want)
    r2, _ = mx.mxfp8_quantize(y, colwise=False, layout=mx.SCALE_PLAIN, fmt=f)
    np.testing.assert_array_equal(u8(r2.data), u8(r.data))
    np.testing.assert_array_equal(u8(r2.scale_plain()), u8(r.scale_plain()))
