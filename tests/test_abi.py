"""The C-ABI library loads without a GPU, exports every entry point that
include/mxmoe.h declares, and rejects bad arguments on the host before touching the
device (CPU only)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mxmoe.h")


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    pat = re.compile(r"^\s*(?:const\s+)?(?:mxmoe_status|size_t|int64_t|int32_t|char\s*\*)\s*\*?\s*(\w+)\s*\(", re.M)
    return sorted(set(pat.findall(text)))


@pytest.fixture(scope="module")
def lib():
    import __graft_entry__
    __graft_entry__.build()
    import mxfp8_grouped_gemm_moe_b200 as mx
    return mx.load()


def test_header_declares_the_layer_entry_points():
    names = _declared_functions()
    for n in ["moe_permute", "moe_unpermute", "mxfp8_quantize", "grouped_gemm_mxfp8", "grouped_gemm_mxfp8_wgrad",
              "grouped_mlp_fwd", "grouped_mlp_bwd", "mxmoe_weights_quantize"]:
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    names = _declared_functions()
    assert len(names) >= 15
    for n in names:
        assert hasattr(lib, n), n


def test_checked_build_exports_the_same_symbols(lib):
    """The bounds-checked build (libmxmoe_checks.so, built by __graft_entry__.build()) is
    the same C ABI: every declared entry point is exported."""
    from mxfp8_grouped_gemm_moe_b200 import build as b
    assert os.path.exists(b.LIB_CHECKS)
    checked = ctypes.CDLL(b.LIB_CHECKS)
    for n in _declared_functions():
        assert hasattr(checked, n), n


def test_binding_signatures_cover_header(lib):
    import mxfp8_grouped_gemm_moe_b200 as mx
    assert set(_declared_functions()) == set(mx._SIGNATURES)


def test_status_strings(lib):
    import mxfp8_grouped_gemm_moe_b200 as mx
    for code, name in mx.STATUS_NAMES.items():
        assert lib.mxmoe_status_string(code).decode() == name


def test_sizes_are_host_only(lib):
    assert lib.mxmoe_rows_capacity(8192, 2, 8) == (8192 * 2 + 255 * 8 + 255) // 256 * 256
    assert lib.mxmoe_rows_capacity(0, 1, 1) == 256
    # weights: 4 copies of E*2F*H-ish bytes plus scales
    E, H, F = 8, 4096, 14336
    w = lib.mxmoe_weights_size(E, H, F)
    assert w >= 2 * (3 * E * H * F) * (1 + 1 / 32)
    s = lib.grouped_mlp_saved_size(8192, 2, 8, 4096, 14336)
    cap = lib.mxmoe_rows_capacity(8192, 2, 8)
    assert s >= cap * (4096 + 14336) * (1 + 1 / 32) + cap * 2 * 14336 * 2
    offs = [lib.grouped_mlp_saved_offset(f, 8192, 2, 8, 4096, 14336) for f in range(10)]
    assert offs == sorted(offs) and all(o % 256 == 0 for o in offs)
    assert lib.grouped_mlp_saved_offset(13, 1, 1, 1, 256, 256) == -1
    # per-tensor FP8: the saved amax field takes room only under that recipe; the recipe
    # combines with no other bit, and the MXFP8 _ex calls' sizes are unchanged by it
    fp8 = 8
    a = lib.grouped_mlp_saved_offset_ex(12, 8192, 2, 8, 4096, 14336, fp8)
    assert a >= 0 and a % 256 == 0
    assert lib.grouped_mlp_saved_size_ex(8192, 2, 8, 4096, 14336, fp8) == a + 256
    assert lib.grouped_mlp_saved_size_ex(8192, 2, 8, 4096, 14336, 0) == lib.grouped_mlp_saved_size(8192, 2, 8, 4096,
                                                                                                  14336)
    assert lib.grouped_mlp_saved_size_ex(8192, 2, 8, 4096, 14336, fp8 | 1) == 0
    assert lib.grouped_mlp_workspace_size_ex(8192, 2, 8, 4096, 14336, fp8) >= \
        lib.grouped_mlp_workspace_size_ex(8192, 2, 8, 4096, 14336, 0)


def test_host_argument_errors_enqueue_nothing(lib):
    """Every one of these is rejected before any CUDA call (so it runs without a GPU).
    The calls pass fake device addresses: should a check ever let one through, the call
    would reach a kernel launch, so the test refuses to run where a GPU is visible."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("passes fake device pointers; host-only test")
    import mxfp8_grouped_gemm_moe_b200 as mx
    P = ctypes.c_void_p
    bad = P(0)
    fake = P(1 << 20)             # never dereferenced: validation fails first
    S = P(0)
    # shapes
    assert lib.moe_permute(fake, fake, 10, 9, 4, fake, fake, fake, fake, fake, fake, 1 << 20, S) == 2
    assert lib.moe_permute(fake, fake, 10, 2, 300, fake, fake, fake, fake, fake, fake, 1 << 20, S) == 2
    assert lib.moe_permute(fake, fake, -1, 2, 4, fake, fake, fake, fake, fake, fake, 1 << 20, S) == 2
    # null pointers
    assert lib.moe_permute(bad, fake, 10, 2, 4, fake, fake, fake, fake, fake, fake, 1 << 20, S) == 1
    # workspace too small
    assert lib.moe_permute(fake, fake, 10, 2, 4, fake, fake, fake, fake, fake, fake, 4, S) == 3
    assert lib.moe_unpermute(fake, fake, 4, 2, 12, fake, S) == 2            # H % 8
    assert lib.moe_unpermute(bad, fake, 4, 2, 16, fake, S) == 1
    # router: k above E or 8, E out of range, missing outputs; T = 0 is a no-op
    assert lib.moe_router_topk(fake, 16, 4, 5, fake, fake, S) == 2
    assert lib.moe_router_topk(fake, 16, 300, 2, fake, fake, S) == 2
    assert lib.moe_router_topk(fake, 16, 64, 9, fake, fake, S) == 2
    assert lib.moe_router_topk(fake, 16, 8, 2, None, fake, S) == 1
    assert lib.moe_router_topk(None, 0, 8, 2, None, None, S) == 0
    assert lib.moe_router_topk_bwd(fake, fake, None, 16, 8, 2, fake, S) == 1
    assert lib.moe_router_topk_bwd(fake, fake, fake, 16, 0, 1, fake, S) == 2
    # quantize: bad dtype, bad shape, no outputs
    m = mx._MX(1 << 20, 1 << 20, 64, 64, 0, 0)
    assert lib.mxfp8_quantize(fake, 7, 1, 64, 64, None, None, 64, ctypes.byref(m), None, S) == 1
    assert lib.mxfp8_quantize(fake, 0, 1, 64, 48, None, None, 64, ctypes.byref(m), None, S) == 2
    assert lib.mxfp8_quantize(fake, 0, 1, 64, 64, None, None, 64, None, None, S) == 1
    m_bad_layout = mx._MX(1 << 20, 1 << 20, 64, 64, 1, 0)   # MMA layout needs multiples of 128
    assert lib.mxfp8_quantize(fake, 0, 1, 64, 64, None, None, 64, ctypes.byref(m_bad_layout), None, S) == 2
    # dequantise: MMA scale layout, null destination, cols not a multiple of 32; 0 rows is a no-op
    dq = mx._MX(1 << 20, 1 << 20, 64, 64, 0, 0)
    assert lib.mxfp8_dequantize(ctypes.byref(mx._MX(1 << 20, 1 << 20, 128, 128, 1, 0)), fake, S) == 1
    assert lib.mxfp8_dequantize(ctypes.byref(dq), None, S) == 1
    assert lib.mxfp8_dequantize(ctypes.byref(mx._MX(1 << 20, 1 << 20, 64, 48, 0, 0)), fake, S) == 2
    assert lib.mxfp8_dequantize(ctypes.byref(mx._MX(1 << 20, 1 << 20, 0, 64, 0, 0)), fake, S) == 0
    # grouped GEMM: N not a multiple of 128; A not in MMA layout
    A = mx._MX(1 << 20, 1 << 20, 256, 256, 1, 0)
    B = mx._MX(1 << 20, 1 << 20, 2 * 192, 256, 1, 0)
    assert lib.grouped_gemm_mxfp8(ctypes.byref(A), ctypes.byref(B), fake, 2, 192, 256, fake, 0, 192, S) == 2
    # weight-gradient GEMM: output rows must be a multiple of 256
    At = mx._MX(1 << 20, 1 << 20, 128, 256, 1, 0)
    Bt = mx._MX(1 << 20, 1 << 20, 128, 256, 1, 0)
    assert lib.grouped_gemm_mxfp8_wgrad(ctypes.byref(At), ctypes.byref(Bt), fake, 2, fake, S) == 2
    Ap = mx._MX(1 << 20, 1 << 20, 256, 256, 0, 0)
    B2 = mx._MX(1 << 20, 1 << 20, 512, 256, 1, 0)
    assert lib.grouped_gemm_mxfp8(ctypes.byref(Ap), ctypes.byref(B2), fake, 2, 256, 256, fake, 0, 256, S) == 1
    # fused MLP: F not a multiple of 256, workspace too small
    assert lib.grouped_mlp_fwd(fake, fake, fake, fake, 1 << 40, 16, 2, 4, 256, 384, fake, fake, 1 << 40, fake,
                               1 << 40, S) == 2
    assert lib.grouped_mlp_fwd(fake, fake, fake, fake, 1 << 40, 16, 2, 4, 256, 512, fake, fake, 1 << 40, fake,
                               16, S) == 3
    assert lib.grouped_mlp_bwd(fake, fake, 1 << 40, fake, 1 << 40, 16, 2, 4, 256, 512, fake, bad, fake, fake,
                               fake, 1 << 40, S) == 1
    # recipe flags: MXMOE_RECIPE_GRAD_E5M2 | _RECOMPUTE_GU | _SCALE_CEIL (1 | 2 | 4), or
    # _FP8_TENSOR (8) alone, which the _ex calls refuse (it runs through grouped_mlp_fp8_*)
    assert lib.grouped_mlp_bwd_ex(fake, fake, 1 << 40, fake, 1 << 40, 16, 2, 4, 256, 512, 8, fake, fake, fake, fake,
                                  fake, 1 << 40, S) == 1
    assert lib.grouped_mlp_fwd_ex(fake, fake, fake, fake, 1 << 40, 16, 2, 4, 256, 512, 16, fake, fake, 1 << 40, fake,
                                  1 << 40, S) == 1
    assert lib.grouped_mlp_fwd_ex(fake, fake, fake, fake, 1 << 40, 16, 2, 4, 256, 512, 8, fake, fake, 1 << 40, fake,
                                  1 << 40, S) == 1
    assert lib.grouped_mlp_saved_size_ex(16, 2, 4, 256, 512, 16) == 0
    assert lib.grouped_mlp_saved_size_ex(16, 2, 4, 256, 512, 8 | 4) == 0
    # per-tensor FP8: the delayed-scaling state must be given (16-byte aligned)
    assert lib.grouped_mlp_fp8_fwd(fake, fake, fake, fake, 1 << 40, 16, 2, 4, 256, 512, None, fake, fake, 1 << 40,
                                   fake, 1 << 40, S) == 1
    assert lib.grouped_mlp_fp8_bwd(fake, fake, 1 << 40, fake, 1 << 40, 16, 2, 4, 256, 512, P((1 << 20) + 4), fake,
                                   fake, fake, fake, fake, 1 << 40, S) == 1
    assert lib.mxmoe_weights_quantize_fp8(fake, fake, 4, 256, 384, fake, 1 << 40, S) == 2
    assert lib.grouped_mlp_saved_size_ex(16, 2, 4, 256, 512, 7) > 0
    # scale rules: only OCP (0) and CEIL (1)
    m_ok = mx._MX(1 << 20, 1 << 20, 64, 64, 0, 0)
    assert lib.mxfp8_quantize_ex(fake, 0, 1, 64, 64, None, None, 64, ctypes.byref(m_ok), None, 2, S) == 1
    assert lib.mxmoe_weights_quantize_ex(fake, fake, 2, 256, 512, -1, fake, 1 << 40, S) == 1
    # the recompute recipe saves the rowwise input instead of G / U: smaller saved buffer,
    # larger workspace (G / U recomputed there)
    a = (4096, 2, 8, 1024, 2816)
    assert lib.grouped_mlp_saved_size_ex(*a, 2) < lib.grouped_mlp_saved_size(*a)
    assert lib.grouped_mlp_workspace_size_ex(*a, 2) > lib.grouped_mlp_workspace_size(*a)
    assert lib.grouped_mlp_saved_size_ex(*a, 1) == lib.grouped_mlp_saved_size(*a)
    assert lib.grouped_mlp_saved_offset_ex(10, *a, 0) == lib.grouped_mlp_saved_offset_ex(11, *a, 0)  # empty x_row
    # an MXFP8 descriptor with an unknown element format; row / colT formats that disagree
    m_bad_fmt = mx._MX(1 << 20, 1 << 20, 64, 64, 0, 3)
    assert lib.mxfp8_quantize(fake, 0, 1, 64, 64, None, None, 64, ctypes.byref(m_bad_fmt), None, S) == 1
    r4 = mx._MX(1 << 20, 1 << 20, 64, 64, 0, 0)
    c5 = mx._MX(1 << 20, 1 << 20, 64, 64, 0, 1)
    assert lib.mxfp8_quantize(fake, 0, 1, 64, 64, None, None, 64, ctypes.byref(r4), ctypes.byref(c5), S) == 1
    # bf16 layer: same shape and size checks
    assert lib.grouped_mlp_bf16_fwd(fake, fake, fake, fake, 1 << 40, 16, 2, 4, 256, 384, fake, fake, 1 << 40, fake,
                                    1 << 40, S) == 2
    assert lib.grouped_mlp_bf16_bwd(fake, fake, 1 << 40, fake, 16, 16, 2, 4, 256, 512, fake, fake, fake, fake,
                                    fake, 1 << 40, S) == 3
    assert lib.mxmoe_weights_bf16_prepare(fake, fake, 2, 256, 384, fake, 1 << 40, S) == 2


def test_layer_arguments_checked_before_allocation(lib):
    """GroupedMLP rejects an unknown precision or a recipe the bf16 layer does not have,
    before any device memory is touched."""
    import mxfp8_grouped_gemm_moe_b200 as mx
    with pytest.raises(ValueError):
        mx.GroupedMLP(16, 2, 4, 256, 512, device="cpu", precision="fp4")
    with pytest.raises(ValueError):
        mx.GroupedMLP(16, 2, 4, 256, 512, device="cpu", precision="bf16", grad_format="e5m2")
    with pytest.raises(ValueError):
        mx.GroupedMLP(16, 2, 4, 256, 512, device="cpu", grad_format="e3m4")
    # sizes of a valid layer on the host (no kernel runs): the recompute recipe's saved
    # buffer holds the rowwise input instead of G / U
    a = mx.GroupedMLP(64, 2, 4, 256, 512, device="cpu")
    b = mx.GroupedMLP(64, 2, 4, 256, 512, device="cpu", recompute_gu=True)
    assert a.recipe == 0 and b.recipe == mx.RECIPE_RECOMPUTE_GU
    assert b.saved.numel() < a.saved.numel()
    c = mx.GroupedMLP(64, 2, 4, 256, 512, device="cpu", grad_format="e5m2", scale_rule="ceil")
    assert c.recipe == mx.RECIPE_GRAD_E5M2 | mx.RECIPE_SCALE_CEIL and c.scale_rule == mx.SCALE_RULE_CEIL
    assert c.saved.numel() == a.saved.numel()
    with pytest.raises(ValueError):
        mx.GroupedMLP(16, 2, 4, 256, 512, device="cpu", scale_rule="floor")
