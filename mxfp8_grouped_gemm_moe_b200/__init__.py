"""Python binding of libmxmoe.so -- the B200 MXFP8 grouped expert-MLP library.

Argument marshalling only: every function below forwards to the C entry point of the
same name (declared in include/mxmoe.h) and every step of the computation runs in the
library's CUDA kernels. PyTorch is used for device memory and the current stream. If
the shared library is missing or cannot be loaded, every call raises -- there is no
fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.environ.get("MXMOE_LIB") or os.path.join(_HERE, "libmxmoe.so")

MXMOE_OK = 0
STATUS_NAMES = {
    0: "MXMOE_OK", 1: "MXMOE_ERR_INVALID_ARG", 2: "MXMOE_ERR_UNSUPPORTED_SHAPE",
    3: "MXMOE_ERR_WORKSPACE_TOO_SMALL", 4: "MXMOE_ERR_CUDA", 5: "MXMOE_ERR_DEVICE_TIMEOUT",
    6: "MXMOE_ERR_DEVICE_CHECK",
}
DTYPE_BF16, DTYPE_F32 = 0, 1
SCALE_PLAIN, SCALE_MMA = 0, 1
FMT_E4M3, FMT_E5M2 = 0, 1
RECIPE_GRAD_E5M2, RECIPE_RECOMPUTE_GU, RECIPE_SCALE_CEIL, RECIPE_FP8_TENSOR = 1, 2, 4, 8
SCALE_RULE_OCP, SCALE_RULE_CEIL = 0, 1
_RULE = {"ocp": SCALE_RULE_OCP, "ceil": SCALE_RULE_CEIL}
_FMT = {"e4m3": FMT_E4M3, "e5m2": FMT_E5M2}
SAVED_FIELDS = ["m_splits", "seg_off", "row_of_slot", "token_of_row", "prob_of_row",
                "x_colT", "x_colT_sf", "z_colT", "z_colT_sf", "gu", "x_row", "x_row_sf", "amax"]


class MxmoeError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__(f"{fn} returned {STATUS_NAMES.get(status, status)}")


class _MX(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("scale", ctypes.c_void_p), ("rows", ctypes.c_int64),
                ("cols", ctypes.c_int64), ("scale_layout", ctypes.c_int32), ("elem_format", ctypes.c_int32)]


_lib = None

_P = ctypes.c_void_p
_I32 = ctypes.c_int32
_I64 = ctypes.c_int64
_SZ = ctypes.c_size_t
_PMX = ctypes.POINTER(_MX)

# name -> (restype, argtypes); the names and order follow include/mxmoe.h
_SIGNATURES = {
    "mxmoe_status_string": (ctypes.c_char_p, [_I32]),
    "mxmoe_get_device_status": (_I32, [ctypes.POINTER(_I32), ctypes.POINTER(_I32), _P]),
    "mxmoe_clear_device_status": (_I32, [_P]),
    "mxmoe_rows_capacity": (_I64, [_I32, _I32, _I32]),
    "moe_permute": (_I32, [_P, _P, _I32, _I32, _I32, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "moe_permute_workspace_size": (_SZ, [_I32, _I32, _I32]),
    "moe_permute_noalloc": (_I32, [_P, _P, _I32, _I32, _I32, _P, _P, _P, _P, _P, _P]),
    "moe_unpermute": (_I32, [_P, _P, _I32, _I32, _I32, _P, _P]),
    "moe_router_topk": (_I32, [_P, _I32, _I32, _I32, _P, _P, _P]),
    "grouped_gemm_bf16": (_I32, [_P, _I64, _P, _P, _I32, _I64, _I64, _P, _I32, _I64, _P]),
    "grouped_gemm_bf16_wgrad": (_I32, [_P, _P, _I64, _I64, _I64, _P, _I32, _P, _P]),
    "moe_router_topk_bwd": (_I32, [_P, _P, _P, _I32, _I32, _I32, _P, _P]),
    "mxfp8_quantize": (_I32, [_P, _I32, _I64, _I64, _I64, _P, _P, _I64, _PMX, _PMX, _P]),
    "mxfp8_quantize_ex": (_I32, [_P, _I32, _I64, _I64, _I64, _P, _P, _I64, _PMX, _PMX, _I32, _P]),
    "mxfp8_dequantize": (_I32, [_PMX, _P, _P]),
    "grouped_gemm_mxfp8": (_I32, [_PMX, _PMX, _P, _I32, _I64, _I64, _P, _I32, _I64, _P]),
    "grouped_gemm_mxfp8_debug_timeout": (_I32, [_PMX, _PMX, _P, _I32, _I64, _I64, _P, _I32, _I64, _P]),
    "grouped_gemm_mxfp8_wgrad": (_I32, [_PMX, _PMX, _P, _I32, _P, _P]),
    "mxmoe_weights_size": (_SZ, [_I32, _I32, _I32]),
    "mxmoe_weights_quantize": (_I32, [_P, _P, _I32, _I32, _I32, _P, _SZ, _P]),
    "mxmoe_weights_quantize_ex": (_I32, [_P, _P, _I32, _I32, _I32, _I32, _P, _SZ, _P]),
    "mxmoe_weights_view": (_I32, [_P, _I32, _I32, _I32, _I32, _PMX]),
    "grouped_mlp_saved_size": (_SZ, [_I32, _I32, _I32, _I32, _I32]),
    "grouped_mlp_saved_offset": (_I64, [_I32, _I32, _I32, _I32, _I32, _I32]),
    "grouped_mlp_workspace_size": (_SZ, [_I32, _I32, _I32, _I32, _I32]),
    "grouped_mlp_fwd": (_I32, [_P, _P, _P, _P, _SZ, _I32, _I32, _I32, _I32, _I32, _P, _P, _SZ, _P, _SZ, _P]),
    "grouped_mlp_bwd": (_I32, [_P, _P, _SZ, _P, _SZ, _I32, _I32, _I32, _I32, _I32, _P, _P, _P, _P, _P, _SZ, _P]),
    "grouped_mlp_saved_size_ex": (_SZ, [_I32, _I32, _I32, _I32, _I32, _I32]),
    "grouped_mlp_saved_offset_ex": (_I64, [_I32, _I32, _I32, _I32, _I32, _I32, _I32]),
    "grouped_mlp_workspace_size_ex": (_SZ, [_I32, _I32, _I32, _I32, _I32, _I32]),
    "grouped_mlp_fwd_ex": (_I32, [_P, _P, _P, _P, _SZ, _I32, _I32, _I32, _I32, _I32, _I32, _P, _P, _SZ, _P, _SZ, _P]),
    "mxmoe_weights_quantize_fp8": (_I32, [_P, _P, _I32, _I32, _I32, _P, _SZ, _P]),
    "grouped_mlp_fp8_fwd": (_I32, [_P, _P, _P, _P, _SZ, _I32, _I32, _I32, _I32, _I32, _P, _P, _P, _SZ, _P, _SZ, _P]),
    "grouped_mlp_fp8_bwd": (_I32, [_P, _P, _SZ, _P, _SZ, _I32, _I32, _I32, _I32, _I32, _P, _P, _P, _P, _P, _P, _SZ,
                                   _P]),
    "grouped_mlp_bwd_ex": (_I32, [_P, _P, _SZ, _P, _SZ, _I32, _I32, _I32, _I32, _I32, _I32, _P, _P, _P, _P, _P, _SZ,
                                  _P]),
    "mxmoe_weights_bf16_size": (_SZ, [_I32, _I32, _I32]),
    "mxmoe_weights_bf16_prepare": (_I32, [_P, _P, _I32, _I32, _I32, _P, _SZ, _P]),
    "grouped_mlp_bf16_saved_size": (_SZ, [_I32, _I32, _I32, _I32, _I32]),
    "grouped_mlp_bf16_workspace_size": (_SZ, [_I32, _I32, _I32, _I32, _I32]),
    "grouped_mlp_bf16_fwd": (_I32, [_P, _P, _P, _P, _SZ, _I32, _I32, _I32, _I32, _I32, _P, _P, _SZ, _P, _SZ, _P]),
    "grouped_mlp_bf16_bwd": (_I32, [_P, _P, _SZ, _P, _SZ, _I32, _I32, _I32, _I32, _I32, _P, _P, _P, _P, _P, _SZ,
                                    _P]),
    "mxmoe_profile_enable": (_I32, [_I32]),
    "mxmoe_profile_disable": (_I32, []),
    "mxmoe_profile_read": (_I32, [ctypes.POINTER(_I32), ctypes.POINTER(ctypes.c_float), _I32]),
    "mxmoe_launch_count": (_I64, []),
}

STAGE_NAMES = {1: "route", 2: "quant_x", 3: "fc1_swiglu", 4: "fc2", 5: "combine", 6: "quant_w1", 7: "quant_w2",
               8: "quant_dy", 9: "fc2_dgrad_swiglu_bwd", 10: "dprob", 11: "fc2_wgrad", 12: "fc1_dgrad",
               13: "fc1_wgrad", 14: "combine_dx", 15: "gemm", 16: "wgrad", 17: "quant", 18: "router",
               19: "router_bwd", 20: "fc1_recompute"}


def load(path: str | None = None):
    """Loads (once) and returns the ctypes handle of libmxmoe.so; raises if absent."""
    global _lib
    if _lib is not None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(f"libmxmoe.so not built ({p}); run __graft_entry__.build() first")
    lib = ctypes.CDLL(p)
    for name, (res, args) in _SIGNATURES.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    _lib = lib
    return lib


def _check(fn, st):
    if st != MXMOE_OK:
        raise MxmoeError(fn, st)


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


# ----------------------------------------------------------------------------- MXFP8 tensors
@dataclass
class MXFP8:
    """An MXFP8 matrix: data uint8 [rows, cols] (FP8 codes of `fmt`: FMT_E4M3 or FMT_E5M2),
    scale uint8 (E8M0), and the scale layout (SCALE_PLAIN = [rows, cols/32]; SCALE_MMA =
    tensor-core chunk order)."""
    data: torch.Tensor
    scale: torch.Tensor
    layout: int = SCALE_MMA
    fmt: int = FMT_E4M3

    @property
    def rows(self):
        return self.data.shape[0]

    @property
    def cols(self):
        return self.data.shape[1]

    @staticmethod
    def empty(rows, cols, layout=SCALE_MMA, device="cuda", fmt=FMT_E4M3):
        return MXFP8(torch.empty((rows, cols), dtype=torch.uint8, device=device),
                     torch.empty((rows * cols // 32,), dtype=torch.uint8, device=device), layout, fmt)

    def as_struct(self):
        return _MX(self.data.data_ptr(), self.scale.data_ptr(), self.rows, self.cols, self.layout, self.fmt)

    def scale_plain(self):
        """Scales as a [rows, cols/32] CPU tensor in plain order (index permutation only)."""
        s = self.scale.cpu()
        if self.layout == SCALE_PLAIN:
            return s.view(self.rows, self.cols // 32)
        return scales_mma_to_plain(s, self.rows, self.cols)


def scales_mma_to_plain(s, rows, cols):
    """Inverse of the MMA scale order: chunk (r//128, kb//4) of 512 bytes, inside it
    byte (r%32)*16 + ((r//32)%4)*4 + kb%4. Pure index permutation (CPU)."""
    s = torch.as_tensor(s).reshape(rows // 128, cols // 128, 32, 4, 4)   # [rg, kg, r%32, (r/32)%4, kb%4]
    s = s.permute(0, 3, 2, 1, 4)                                          # [rg, r/32%4, r%32, kg, kb%4]
    return s.reshape(rows, cols // 32).contiguous()


# ----------------------------------------------------------------------------- entry points
def status_string(s):
    return load().mxmoe_status_string(s).decode()


def mxmoe_get_device_status():
    v, w = _I32(0), _I32(0)
    _check("mxmoe_get_device_status", load().mxmoe_get_device_status(ctypes.byref(v), ctypes.byref(w), _stream()))
    return v.value, w.value


def mxmoe_clear_device_status():
    _check("mxmoe_clear_device_status", load().mxmoe_clear_device_status(_stream()))


def mxmoe_rows_capacity(T, k, E):
    return int(load().mxmoe_rows_capacity(T, k, E))


def moe_permute(topk_idx, probs, E):
    """-> dict(m_splits, seg_off, row_of_slot, token_of_row, prob_of_row) (device tensors)."""
    lib = load()
    T, k = topk_idx.shape
    cap = mxmoe_rows_capacity(T, k, E)
    dev = topk_idx.device
    out = dict(m_splits=torch.empty(E, dtype=torch.int32, device=dev),
               seg_off=torch.empty(E + 1, dtype=torch.int32, device=dev),
               row_of_slot=torch.empty((T, k), dtype=torch.int32, device=dev),
               token_of_row=torch.full((cap,), -2, dtype=torch.int32, device=dev),
               prob_of_row=torch.full((cap,), -1.0, dtype=torch.float32, device=dev))
    ws = torch.empty(lib.moe_permute_workspace_size(T, k, E), dtype=torch.uint8, device=dev)
    st = lib.moe_permute(_ptr(topk_idx), _ptr(probs), T, k, E, _ptr(out["m_splits"]), _ptr(out["seg_off"]),
                         _ptr(out["row_of_slot"]), _ptr(out["token_of_row"]), _ptr(out["prob_of_row"]),
                         _ptr(ws), ws.numel(), _stream())
    _check("moe_permute", st)
    return out


def moe_unpermute(y_perm, row_of_slot, out=None):
    T, k = row_of_slot.shape
    H = y_perm.shape[1]
    y = out if out is not None else torch.empty((T, H), dtype=torch.bfloat16, device=y_perm.device)
    _check("moe_unpermute", load().moe_unpermute(_ptr(y_perm), _ptr(row_of_slot), T, k, H, _ptr(y), _stream()))
    return y



def moe_router_topk(logits, k):
    """logits float32 [T, E] (cuda) -> (topk_idx int32 [T, k], probs float32 [T, k])."""
    T, E = logits.shape
    idx = torch.empty((T, k), dtype=torch.int32, device=logits.device)
    probs = torch.empty((T, k), dtype=torch.float32, device=logits.device)
    _check("moe_router_topk", load().moe_router_topk(_ptr(logits), T, E, k, _ptr(idx), _ptr(probs), _stream()))
    return idx, probs


def moe_router_topk_bwd(logits, topk_idx, dprobs):
    """-> dlogits float32 [T, E]."""
    T, E = logits.shape
    k = topk_idx.shape[1]
    dl = torch.empty((T, E), dtype=torch.float32, device=logits.device)
    _check("moe_router_topk_bwd", load().moe_router_topk_bwd(_ptr(logits), _ptr(topk_idx), _ptr(dprobs), T, E, k,
                                                                 _ptr(dl), _stream()))
    return dl


def mxfp8_quantize(src, rowwise=True, colwise=True, layout=SCALE_MMA, row_gather=None, nrows=None, out_rows=None,
                   fmt=FMT_E4M3, scale_rule=SCALE_RULE_OCP):
    """src [rows, cols] or [batch, rows, cols] bf16/fp32 -> (MXFP8 rowwise | None, MXFP8 colT | None);
    fmt FMT_E4M3 or FMT_E5M2 (element format of both outputs); scale_rule SCALE_RULE_OCP or
    SCALE_RULE_CEIL."""
    lib = load()
    dt = {torch.bfloat16: DTYPE_BF16, torch.float32: DTYPE_F32}[src.dtype]
    if src.dim() == 2:
        batch, (rows, cols) = 1, src.shape
    else:
        batch, rows, cols = src.shape
    orows = rows if out_rows is None else out_rows
    r = MXFP8.empty(batch * orows, cols, layout, src.device, fmt) if rowwise else None
    c = MXFP8.empty(batch * cols, orows, layout, src.device, fmt) if colwise else None
    rs = ctypes.byref(r.as_struct()) if r is not None else None
    cs = ctypes.byref(c.as_struct()) if c is not None else None
    if scale_rule == SCALE_RULE_OCP:
        st = lib.mxfp8_quantize(_ptr(src), dt, batch, rows, cols, _ptr(row_gather), _ptr(nrows), orows, rs, cs,
                                _stream())
        _check("mxfp8_quantize", st)
    else:
        st = lib.mxfp8_quantize_ex(_ptr(src), dt, batch, rows, cols, _ptr(row_gather), _ptr(nrows), orows, rs, cs,
                                   scale_rule, _stream())
        _check("mxfp8_quantize_ex", st)
    return r, c


def mxfp8_dequantize(m: MXFP8, out=None):
    """Rowwise MXFP8 with plain scales -> bf16 [rows, cols] (the library's kernel)."""
    lib = load()
    y = out if out is not None else torch.empty((m.rows, m.cols), dtype=torch.bfloat16, device=m.data.device)
    _check("mxfp8_dequantize", lib.mxfp8_dequantize(ctypes.byref(m.as_struct()), _ptr(y), _stream()))
    return y


def grouped_gemm_mxfp8(A: MXFP8, B: MXFP8, seg_off, E, N, out_dtype=torch.bfloat16, out=None):
    K = A.cols
    C = out if out is not None else torch.empty((A.rows, N), dtype=out_dtype, device=A.data.device)
    dt = DTYPE_BF16 if C.dtype == torch.bfloat16 else DTYPE_F32
    st = load().grouped_gemm_mxfp8(ctypes.byref(A.as_struct()), ctypes.byref(B.as_struct()), _ptr(seg_off), E, N,
                                   K, _ptr(C), dt, C.stride(0), _stream())
    _check("grouped_gemm_mxfp8", st)
    return C


def grouped_gemm_mxfp8_debug_timeout(A: MXFP8, B: MXFP8, seg_off, E, N, out):
    """Test hook of the device-timeout path: grouped_gemm_mxfp8 with the first CTA pair's
    accumulator-ready signal withheld. The kernel ends after about a second with the device
    status set to MXMOE_ERR_DEVICE_TIMEOUT and `out` only partly written."""
    dt = DTYPE_BF16 if out.dtype == torch.bfloat16 else DTYPE_F32
    st = load().grouped_gemm_mxfp8_debug_timeout(ctypes.byref(A.as_struct()), ctypes.byref(B.as_struct()),
                                                 _ptr(seg_off), E, N, A.cols, _ptr(out), dt, out.stride(0), _stream())
    _check("grouped_gemm_mxfp8_debug_timeout", st)
    return out


def grouped_gemm_mxfp8_wgrad(At: MXFP8, Bt: MXFP8, seg_off, E, out=None):
    C = out if out is not None else torch.empty((E, At.rows, Bt.rows), dtype=torch.float32, device=At.data.device)
    st = load().grouped_gemm_mxfp8_wgrad(ctypes.byref(At.as_struct()), ctypes.byref(Bt.as_struct()), _ptr(seg_off),
                                         E, _ptr(C), _stream())
    _check("grouped_gemm_mxfp8_wgrad", st)
    return C


def grouped_gemm_bf16(A, B, seg_off, E, N, out_dtype=torch.bfloat16, out=None):
    """A bf16 [rows_cap, K], B bf16 [E*N, K] (or [E, N, K]) -> C [rows_cap, N]."""
    rows, K = A.shape
    C = out if out is not None else torch.empty((rows, N), dtype=out_dtype, device=A.device)
    dt = DTYPE_BF16 if C.dtype == torch.bfloat16 else DTYPE_F32
    _check("grouped_gemm_bf16", load().grouped_gemm_bf16(_ptr(A), rows, _ptr(B), _ptr(seg_off), E, N, K, _ptr(C), dt,
                                                         C.stride(0), _stream()))
    return C


def grouped_gemm_bf16_wgrad(At, Bt, seg_off, E, out=None):
    """At bf16 [N, rows_cap], Bt bf16 [K2, rows_cap] -> C fp32 [E, N, K2]."""
    N, rows = At.shape
    K2 = Bt.shape[0]
    C = out if out is not None else torch.empty((E, N, K2), dtype=torch.float32, device=At.device)
    _check("grouped_gemm_bf16_wgrad", load().grouped_gemm_bf16_wgrad(_ptr(At), _ptr(Bt), N, K2, rows, _ptr(seg_off), E,
                                                                     _ptr(C), _stream()))
    return C


def mxmoe_weights_quantize(W1, W2, out=None, scale_rule=SCALE_RULE_OCP):
    lib = load()
    E, F2, H = W1.shape
    F = F2 // 2
    n = lib.mxmoe_weights_size(E, H, F)
    wq = out if out is not None else torch.empty(n, dtype=torch.uint8, device=W1.device)
    if scale_rule == SCALE_RULE_OCP:
        _check("mxmoe_weights_quantize",
               lib.mxmoe_weights_quantize(_ptr(W1), _ptr(W2), E, H, F, _ptr(wq), wq.numel(), _stream()))
    else:
        _check("mxmoe_weights_quantize_ex",
               lib.mxmoe_weights_quantize_ex(_ptr(W1), _ptr(W2), E, H, F, scale_rule, _ptr(wq), wq.numel(),
                                             _stream()))
    return wq


def mxmoe_weights_quantize_fp8(W1, W2, out=None):
    """Per-tensor FP8 weights buffer: per-expert amax of W1 / W2 and the four E4M3 copies
    (scale bytes 127)."""
    lib = load()
    E, F2, H = W1.shape
    F = F2 // 2
    wq = out if out is not None else torch.empty(lib.mxmoe_weights_size(E, H, F), dtype=torch.uint8,
                                                 device=W1.device)
    _check("mxmoe_weights_quantize_fp8",
           lib.mxmoe_weights_quantize_fp8(_ptr(W1), _ptr(W2), E, H, F, _ptr(wq), wq.numel(), _stream()))
    return wq


def grouped_mlp_fp8_fwd(x, topk_idx, probs, wq, E, F, amax_state, saved, ws, y=None):
    T, H = x.shape
    k = topk_idx.shape[1]
    y = y if y is not None else torch.empty((T, H), dtype=torch.bfloat16, device=x.device)
    st = load().grouped_mlp_fp8_fwd(_ptr(x), _ptr(topk_idx), _ptr(probs), _ptr(wq), wq.numel(), T, k, E, H, F,
                                    _ptr(amax_state), _ptr(y), _ptr(saved), saved.numel(), _ptr(ws), ws.numel(),
                                    _stream())
    _check("grouped_mlp_fp8_fwd", st)
    return y


def grouped_mlp_fp8_bwd(dy, saved, wq, T, k, E, H, F, amax_state, ws, dx=None, dW1=None, dW2=None, dprobs=None):
    dev = dy.device
    dx = dx if dx is not None else torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    dW1 = dW1 if dW1 is not None else torch.empty((E, 2 * F, H), dtype=torch.float32, device=dev)
    dW2 = dW2 if dW2 is not None else torch.empty((E, H, F), dtype=torch.float32, device=dev)
    dprobs = dprobs if dprobs is not None else torch.empty((T, k), dtype=torch.float32, device=dev)
    st = load().grouped_mlp_fp8_bwd(_ptr(dy), _ptr(saved), saved.numel(), _ptr(wq), wq.numel(), T, k, E, H, F,
                                    _ptr(amax_state), _ptr(dx), _ptr(dW1), _ptr(dW2), _ptr(dprobs), _ptr(ws),
                                    ws.numel(), _stream())
    _check("grouped_mlp_fp8_bwd", st)
    return dx, dW1, dW2, dprobs


def mxmoe_weights_view(wq, E, H, F, which):
    """MXFP8 view (0 W1 row, 1 W1 colT, 2 W2 row, 3 W2 colT) into a weights buffer."""
    m = _MX()
    _check("mxmoe_weights_view", load().mxmoe_weights_view(_ptr(wq), E, H, F, which, ctypes.byref(m)))
    base = wq.data_ptr()
    d0, s0 = m.data - base, m.scale - base
    n = m.rows * m.cols
    return MXFP8(wq[d0:d0 + n].view(m.rows, m.cols), wq[s0:s0 + n // 32], SCALE_MMA)


class GroupedMLP:
    """Buffers for one layer shape; forward/backward call the fused C entry points.

    precision "mxfp8" (default) runs the MXFP8 layer (grouped_mlp_fwd / _bwd); "bf16" runs
    the same steps on bf16 operands (grouped_mlp_bf16_fwd / _bwd); "fp8" runs per-tensor FP8
    (grouped_mlp_fp8_fwd / _bwd) with its delayed-scaling state in ``amax_state`` (fp32 [4]
    on the device: Z amax in / out, dGU amax in / out; ``roll_amax`` starts the next step
    with this step's values, ``set_amax`` sets the values to encode with). For the MXFP8 layer,
    grad_format "e4m3" (default) or "e5m2" picks the element format of the gradients (dY,
    dGU), recompute_gu=True saves the rowwise MXFP8 input instead of the bf16 gate/up
    pre-activations and recomputes those in the backward, and scale_rule "ocp" (default) or
    "ceil" picks the scale rule of every quantiser, the weights' included (the recipe flags
    of grouped_mlp_fwd_ex / _bwd_ex)."""

    def __init__(self, T, k, E, H, F, device="cuda", precision="mxfp8", grad_format="e4m3", recompute_gu=False,
                 scale_rule="ocp"):
        if precision not in ("mxfp8", "bf16", "fp8"):
            raise ValueError(f"unknown precision {precision!r}")
        if grad_format not in _FMT:
            raise ValueError(f"unknown grad_format {grad_format!r}")
        if scale_rule not in _RULE:
            raise ValueError(f"unknown scale_rule {scale_rule!r}")
        self.scale_rule = _RULE[scale_rule]
        self.recipe = ((RECIPE_GRAD_E5M2 if grad_format == "e5m2" else 0) |
                       (RECIPE_RECOMPUTE_GU if recompute_gu else 0) |
                       (RECIPE_SCALE_CEIL if scale_rule == "ceil" else 0))
        if precision != "mxfp8" and self.recipe:
            raise ValueError("grad_format / recompute_gu / scale_rule apply to the MXFP8 layer")
        if precision == "fp8":
            self.recipe = RECIPE_FP8_TENSOR
            self.amax_state = torch.zeros(4, dtype=torch.float32, device=device)
        lib = load()
        self.T, self.k, self.E, self.H, self.F = T, k, E, H, F
        self.precision = precision
        self.cap = mxmoe_rows_capacity(T, k, E)
        if precision == "bf16":
            saved = lib.grouped_mlp_bf16_saved_size(T, k, E, H, F)
            ws = lib.grouped_mlp_bf16_workspace_size(T, k, E, H, F)
            wsz = lib.mxmoe_weights_bf16_size(E, H, F)
        else:
            saved = lib.grouped_mlp_saved_size_ex(T, k, E, H, F, self.recipe)
            ws = lib.grouped_mlp_workspace_size_ex(T, k, E, H, F, self.recipe)
            wsz = lib.mxmoe_weights_size(E, H, F)
        if saved == 0 or ws == 0:
            raise MxmoeError("grouped_mlp sizes", 2)
        self.saved = torch.empty(saved, dtype=torch.uint8, device=device)
        self.ws = torch.empty(ws, dtype=torch.uint8, device=device)
        self.wq = torch.empty(wsz, dtype=torch.uint8, device=device)

    def quantize_weights(self, W1, W2):
        """Prepares the weights buffer: MXFP8 copies, or bf16 row / transposed copies."""
        if self.precision == "bf16":
            return mxmoe_weights_bf16_prepare(W1, W2, out=self.wq)
        if self.precision == "fp8":
            return mxmoe_weights_quantize_fp8(W1, W2, out=self.wq)
        return mxmoe_weights_quantize(W1, W2, out=self.wq, scale_rule=self.scale_rule)

    def set_amax(self, z_amax, dgu_amax):
        """Per-tensor FP8: the Z and dGU amax the next forward / backward encode with."""
        self.amax_state[0] = float(z_amax)
        self.amax_state[2] = float(dgu_amax)

    def roll_amax(self):
        """Per-tensor FP8 delayed scaling: the next step encodes Z and dGU with this step's
        largest magnitudes (device copies, no synchronisation)."""
        self.amax_state[0:4:2].copy_(self.amax_state[1:4:2])

    def forward(self, x, topk_idx, probs, y=None):
        if self.precision == "bf16":
            return grouped_mlp_bf16_fwd(x, topk_idx, probs, self.wq, self.E, self.F, self.saved, self.ws, y)
        if self.precision == "fp8":
            return grouped_mlp_fp8_fwd(x, topk_idx, probs, self.wq, self.E, self.F, self.amax_state, self.saved,
                                       self.ws, y)
        return grouped_mlp_fwd(x, topk_idx, probs, self.wq, self.E, self.F, self.saved, self.ws, y,
                               recipe=self.recipe)

    def backward(self, dy, dx=None, dW1=None, dW2=None, dprobs=None):
        if self.precision == "bf16":
            return grouped_mlp_bf16_bwd(dy, self.saved, self.wq, self.T, self.k, self.E, self.H, self.F, self.ws,
                                        dx, dW1, dW2, dprobs)
        if self.precision == "fp8":
            return grouped_mlp_fp8_bwd(dy, self.saved, self.wq, self.T, self.k, self.E, self.H, self.F,
                                       self.amax_state, self.ws, dx, dW1, dW2, dprobs)
        return grouped_mlp_bwd(dy, self.saved, self.wq, self.T, self.k, self.E, self.H, self.F, self.ws, dx, dW1,
                               dW2, dprobs, recipe=self.recipe)

    def saved_field(self, name, dtype=torch.uint8, count=None):
        """View of a named field of the saved buffer of the MXFP8 layer (inspection / tests)."""
        if self.precision == "bf16":
            raise ValueError("saved_field describes the MXFP8 / FP8 layers' saved buffer")
        lib = load()
        f = SAVED_FIELDS.index(name)
        off = lib.grouped_mlp_saved_offset_ex(f, self.T, self.k, self.E, self.H, self.F, self.recipe)
        esz = torch.tensor([], dtype=dtype).element_size()
        return self.saved[off:off + count * esz].view(dtype)


def mxmoe_weights_bf16_prepare(W1, W2, out=None):
    """bf16 W1 [E, 2F, H], W2 [E, H, F] -> the bf16 layer's weights buffer (uint8)."""
    E, F2, H = W1.shape
    F = F2 // 2
    lib = load()
    n = lib.mxmoe_weights_bf16_size(E, H, F)
    wb = out if out is not None else torch.empty(n, dtype=torch.uint8, device=W1.device)
    _check("mxmoe_weights_bf16_prepare",
           lib.mxmoe_weights_bf16_prepare(_ptr(W1), _ptr(W2), E, H, F, _ptr(wb), wb.numel(), _stream()))
    return wb


def grouped_mlp_fwd(x, topk_idx, probs, wq, E, F, saved, ws, y=None, recipe=0):
    T, H = x.shape
    k = topk_idx.shape[1]
    y = y if y is not None else torch.empty((T, H), dtype=torch.bfloat16, device=x.device)
    if recipe == 0:
        st = load().grouped_mlp_fwd(_ptr(x), _ptr(topk_idx), _ptr(probs), _ptr(wq), wq.numel(), T, k, E, H, F,
                                    _ptr(y), _ptr(saved), saved.numel(), _ptr(ws), ws.numel(), _stream())
        _check("grouped_mlp_fwd", st)
    else:
        st = load().grouped_mlp_fwd_ex(_ptr(x), _ptr(topk_idx), _ptr(probs), _ptr(wq), wq.numel(), T, k, E, H, F,
                                       recipe, _ptr(y), _ptr(saved), saved.numel(), _ptr(ws), ws.numel(), _stream())
        _check("grouped_mlp_fwd_ex", st)
    return y


def grouped_mlp_bwd(dy, saved, wq, T, k, E, H, F, ws, dx=None, dW1=None, dW2=None, dprobs=None, recipe=0):
    dev = dy.device
    dx = dx if dx is not None else torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    dW1 = dW1 if dW1 is not None else torch.empty((E, 2 * F, H), dtype=torch.float32, device=dev)
    dW2 = dW2 if dW2 is not None else torch.empty((E, H, F), dtype=torch.float32, device=dev)
    dprobs = dprobs if dprobs is not None else torch.empty((T, k), dtype=torch.float32, device=dev)
    if recipe == 0:
        st = load().grouped_mlp_bwd(_ptr(dy), _ptr(saved), saved.numel(), _ptr(wq), wq.numel(), T, k, E, H, F,
                                    _ptr(dx), _ptr(dW1), _ptr(dW2), _ptr(dprobs), _ptr(ws), ws.numel(), _stream())
        _check("grouped_mlp_bwd", st)
    else:
        st = load().grouped_mlp_bwd_ex(_ptr(dy), _ptr(saved), saved.numel(), _ptr(wq), wq.numel(), T, k, E, H, F,
                                       recipe, _ptr(dx), _ptr(dW1), _ptr(dW2), _ptr(dprobs), _ptr(ws), ws.numel(),
                                       _stream())
        _check("grouped_mlp_bwd_ex", st)
    return dx, dW1, dW2, dprobs


def grouped_mlp_bf16_fwd(x, topk_idx, probs, wb, E, F, saved, ws, y=None):
    T, H = x.shape
    k = topk_idx.shape[1]
    y = y if y is not None else torch.empty((T, H), dtype=torch.bfloat16, device=x.device)
    st = load().grouped_mlp_bf16_fwd(_ptr(x), _ptr(topk_idx), _ptr(probs), _ptr(wb), wb.numel(), T, k, E, H, F,
                                     _ptr(y), _ptr(saved), saved.numel(), _ptr(ws), ws.numel(), _stream())
    _check("grouped_mlp_bf16_fwd", st)
    return y


def grouped_mlp_bf16_bwd(dy, saved, wb, T, k, E, H, F, ws, dx=None, dW1=None, dW2=None, dprobs=None):
    dev = dy.device
    dx = dx if dx is not None else torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    dW1 = dW1 if dW1 is not None else torch.empty((E, 2 * F, H), dtype=torch.float32, device=dev)
    dW2 = dW2 if dW2 is not None else torch.empty((E, H, F), dtype=torch.float32, device=dev)
    dprobs = dprobs if dprobs is not None else torch.empty((T, k), dtype=torch.float32, device=dev)
    st = load().grouped_mlp_bf16_bwd(_ptr(dy), _ptr(saved), saved.numel(), _ptr(wb), wb.numel(), T, k, E, H, F,
                                     _ptr(dx), _ptr(dW1), _ptr(dW2), _ptr(dprobs), _ptr(ws), ws.numel(), _stream())
    _check("grouped_mlp_bf16_bwd", st)
    return dx, dW1, dW2, dprobs


# ----------------------------------------------------------------------------- instrumentation
def mxmoe_profile_enable(max_stages=4096):
    _check("mxmoe_profile_enable", load().mxmoe_profile_enable(max_stages))


def mxmoe_profile_disable():
    _check("mxmoe_profile_disable", load().mxmoe_profile_disable())


def mxmoe_profile_read(cap=4096):
    """-> list of (stage name, milliseconds) for the stages recorded since the last read."""
    tags = (_I32 * cap)()
    ms = (ctypes.c_float * cap)()
    n = load().mxmoe_profile_read(tags, ms, cap)
    return [(STAGE_NAMES.get(tags[i], str(tags[i])), ms[i]) for i in range(min(n, cap))]


def mxmoe_launch_count():
    return int(load().mxmoe_launch_count())
