// C ABI of the library: argument validation, buffer carving and the orchestration of
// the fused grouped-MLP forward and backward. Every step of the path runs in this
// library's kernels; nothing here allocates or synchronises (except the explicit
// status query).
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>

#include "../../include/mxmoe.h"
#include <nvtx3/nvToolsExt.h>

#include "mxmoe_launch.h"

#include "mxmoe_device.cuh"

using namespace mxmoe;

namespace {

inline size_t al256(size_t x) { return (x + 255) & ~size_t(255); }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline cudaStream_t S(void* s) { return reinterpret_cast<cudaStream_t>(s); }
inline mxmoe_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MXMOE_OK : MXMOE_ERR_CUDA; }


// Sub-buffers of a caller-provided byte buffer, each 256-byte aligned.
struct Carver {
  size_t off = 0;
  size_t take(size_t bytes) {
    const size_t o = off;
    off = al256(off + bytes);
    return o;
  }
};

bool valid_moe_shape(int32_t T, int32_t k, int32_t E) { return T >= 0 && k >= 1 && k <= 8 && E >= 1 && E <= 256; }
bool valid_mlp_shape(int32_t T, int32_t k, int32_t E, int32_t H, int32_t F) {
  return valid_moe_shape(T, k, E) && H > 0 && F > 0 && H % 256 == 0 && F % 256 == 0;
}

// ---------------------------------------------------------------- layouts
struct WeightsLayout {
  size_t d[4], s[4], amax, total;  // amax: per-tensor FP8 weights' largest magnitudes, W1 [E] then W2 [E]
  int64_t rows[4], cols[4];
};
WeightsLayout weights_layout(int64_t E, int64_t H, int64_t F) {
  WeightsLayout L;
  const int64_t r[4] = {E * 2 * F, E * H, E * H, E * F};
  const int64_t c[4] = {H, 2 * F, F, H};
  Carver cv;
  for (int i = 0; i < 4; ++i) {
    L.rows[i] = r[i];
    L.cols[i] = c[i];
    L.d[i] = cv.take((size_t)(r[i] * c[i]));
    L.s[i] = cv.take((size_t)(r[i] * c[i] / 32));
  }
  L.amax = cv.take((size_t)(2 * E * 4));
  L.total = cv.off;
  return L;
}

bool valid_recipe(int32_t recipe) {
  if (recipe == MXMOE_RECIPE_FP8_TENSOR) return true;  // per-tensor FP8 combines with no other bit
  return (recipe & ~(MXMOE_RECIPE_GRAD_E5M2 | MXMOE_RECIPE_RECOMPUTE_GU | MXMOE_RECIPE_SCALE_CEIL)) == 0;
}
bool fp8_tensor(int32_t recipe) { return recipe == MXMOE_RECIPE_FP8_TENSOR; }
int32_t recipe_scale_rule(int32_t recipe) {
  return (recipe & MXMOE_RECIPE_SCALE_CEIL) ? MXMOE_SCALE_RULE_CEIL : MXMOE_SCALE_RULE_OCP;
}
bool recomputes_gu(int32_t recipe) { return (recipe & MXMOE_RECIPE_RECOMPUTE_GU) != 0; }

struct SavedLayout {
  size_t off[13];
  size_t total;
};
// With MXMOE_RECIPE_RECOMPUTE_GU the gate/up pre-activations are not saved (zero bytes)
// and the rowwise MXFP8 copy of the permuted input is, for the backward's recompute.
SavedLayout saved_layout(int64_t T, int64_t k, int64_t E, int64_t H, int64_t F, int32_t recipe = 0) {
  const int64_t cap = rows_cap(T, k, E);
  const bool rc = recomputes_gu(recipe);
  SavedLayout L;
  Carver cv;
  L.off[MXMOE_SAVED_M_SPLITS] = cv.take(E * 4);
  L.off[MXMOE_SAVED_SEG_OFF] = cv.take((E + 1) * 4);
  L.off[MXMOE_SAVED_ROW_OF_SLOT] = cv.take(std::max<int64_t>(T * k, 1) * 4);
  L.off[MXMOE_SAVED_TOKEN_OF_ROW] = cv.take(cap * 4);
  L.off[MXMOE_SAVED_PROB_OF_ROW] = cv.take(cap * 4);
  L.off[MXMOE_SAVED_X_COLT] = cv.take(H * cap);
  L.off[MXMOE_SAVED_X_COLT_SF] = cv.take(H * cap / 32);
  L.off[MXMOE_SAVED_Z_COLT] = cv.take(F * cap);
  L.off[MXMOE_SAVED_Z_COLT_SF] = cv.take(F * cap / 32);
  L.off[MXMOE_SAVED_GU] = cv.take(rc ? 0 : cap * 2 * F * 2);
  L.off[MXMOE_SAVED_X_ROW] = cv.take(rc ? cap * H : 0);
  L.off[MXMOE_SAVED_X_ROW_SF] = cv.take(rc ? cap * H / 32 : 0);
  L.off[MXMOE_SAVED_AMAX] = cv.take(fp8_tensor(recipe) ? 2 * 4 : 0);  // largest |x|, Z's amax in use
  L.total = cv.off;
  return L;
}

struct FwdWs {
  size_t route, x_row, x_row_sf, z_row, z_row_sf, y_perm, total;
};
FwdWs fwd_ws(int64_t T, int64_t k, int64_t E, int64_t H, int64_t F) {
  const int64_t cap = rows_cap(T, k, E);
  FwdWs w;
  Carver cv;
  w.route = cv.take(route_workspace_bytes((int)T, (int)k, (int)E));
  w.x_row = cv.take(cap * H);
  w.x_row_sf = cv.take(cap * H / 32);
  w.z_row = cv.take(cap * F);
  w.z_row_sf = cv.take(cap * F / 32);
  w.y_perm = cv.take(cap * H * 2);
  w.total = cv.off;
  return w;
}

struct BwdWs {
  size_t dy_row, dy_row_sf, dy_colT, dy_colT_sf, dgu_row, dgu_row_sf, dgu_colT, dgu_colT_sf, dprob_part, dx_perm, gu,
      amax, total;
};
BwdWs bwd_ws(int64_t T, int64_t k, int64_t E, int64_t H, int64_t F, int32_t recipe = 0) {
  const int64_t cap = rows_cap(T, k, E);
  BwdWs w;
  Carver cv;
  w.dy_row = cv.take(cap * H);
  w.dy_row_sf = cv.take(cap * H / 32);
  w.dy_colT = cv.take(H * cap);
  w.dy_colT_sf = cv.take(H * cap / 32);
  w.dgu_row = cv.take(cap * 2 * F);
  w.dgu_row_sf = cv.take(cap * 2 * F / 32);
  w.dgu_colT = cv.take(2 * F * cap);
  w.dgu_colT_sf = cv.take(2 * F * cap / 32);
  w.dprob_part = cv.take(cap * (F / 128) * 4);
  w.dx_perm = cv.take(cap * H * 2);
  w.gu = cv.take(recomputes_gu(recipe) ? cap * 2 * F * 2 : 0);  // recomputed G / U (bf16)
  w.amax = cv.take(fp8_tensor(recipe) ? 2 * 4 : 0);               // largest |dY|, dGU's amax in use
  w.total = cv.off;
  return w;
}

bool valid_mx(const mxmoe_mxfp8* m) {
  return m && m->data && m->scale && aligned16(m->data) && aligned16(m->scale) && m->rows >= 0 && m->cols >= 0 &&
         (m->scale_layout == MXMOE_SCALE_PLAIN || m->scale_layout == MXMOE_SCALE_MMA) &&
         (m->elem_format == MXMOE_FMT_E4M3 || m->elem_format == MXMOE_FMT_E5M2);
}
bool mma_ready(const mxmoe_mxfp8* m) {
  return valid_mx(m) && m->scale_layout == MXMOE_SCALE_MMA && m->rows % 128 == 0 && m->cols % 128 == 0;
}

mxmoe_mxfp8 mk(uint8_t* base, size_t d, size_t s, int64_t rows, int64_t cols, int32_t fmt = MXMOE_FMT_E4M3) {
  mxmoe_mxfp8 m;
  m.data = base + d;
  m.scale = base + s;
  m.rows = rows;
  m.cols = cols;
  m.scale_layout = MXMOE_SCALE_MMA;
  m.elem_format = fmt;
  return m;
}

GemmArgs gemm_base(int mode, const mxmoe_mxfp8& A, const mxmoe_mxfp8& B, const int32_t* seg_off, int32_t E) {
  GemmArgs g;
  std::memset(&g, 0, sizeof(g));
  g.mode = mode;
  g.E = E;
  g.a_data = A.data;
  g.a_sf = A.scale;
  g.a_rows = A.rows;
  g.a_cols = A.cols;
  g.b_data = B.data;
  g.b_sf = B.scale;
  g.b_rows = B.rows;
  g.b_cols = B.cols;
  g.a_fmt = A.elem_format;
  g.b_fmt = B.elem_format;
  g.seg_off = seg_off;
  return g;
}


// ---------------------------------------------------------------- stage timing
// Host-side only: CUDA events around each stage, when enabled. Only the outermost
// stage scope records (a fused call's inner entry points are attributed to it).
struct Profiler {
  bool on = false;
  int cap = 0, n = 0, depth = 0;
  cudaEvent_t* ev = nullptr;
  int32_t* tags = nullptr;
};
Profiler g_prof;

// Stage names for NVTX ranges (index = MXMOE_STAGE_* tag).
const char* const kStageNames[] = {"",           "route",       "quant_x",       "fc1_swiglu",    "fc2",
                                   "combine",    "quant_w1",    "quant_w2",      "quant_dy",      "fc2_dgrad_swiglu_bwd",
                                   "dprob",      "fc2_wgrad",   "fc1_dgrad",     "fc1_wgrad",     "combine_dx",
                                   "gemm",       "wgrad",       "quant",         "router",        "router_bwd",
                                   "fc1_recompute"};

// One stage of the layer: an NVTX range on the host timeline (free unless a profiler
// such as Nsight Systems is attached) and, while mxmoe_profile_enable is on, a pair of
// CUDA events on the stage's stream (outermost stages only).
struct StageScope {
  cudaStream_t st;
  bool rec = false;
  StageScope(int32_t tag, cudaStream_t s) : st(s) {
    nvtxRangePushA(tag >= 0 && tag < (int32_t)(sizeof(kStageNames) / sizeof(kStageNames[0])) ? kStageNames[tag]
                                                                                              : "mxmoe");
    if (g_prof.on && g_prof.depth == 0 && g_prof.n < g_prof.cap) {
      cudaEventRecord(g_prof.ev[2 * g_prof.n], st);
      g_prof.tags[g_prof.n] = tag;
      rec = true;
    }
    ++g_prof.depth;
  }
  ~StageScope() {
    --g_prof.depth;
    if (rec) {
      cudaEventRecord(g_prof.ev[2 * g_prof.n + 1], st);
      ++g_prof.n;
    }
    nvtxRangePop();
  }
};

}  // namespace

// ============================================================================ C ABI
extern "C" {

const char* mxmoe_status_string(mxmoe_status s) {
  switch (s) {
    case MXMOE_OK: return "MXMOE_OK";
    case MXMOE_ERR_INVALID_ARG: return "MXMOE_ERR_INVALID_ARG";
    case MXMOE_ERR_UNSUPPORTED_SHAPE: return "MXMOE_ERR_UNSUPPORTED_SHAPE";
    case MXMOE_ERR_WORKSPACE_TOO_SMALL: return "MXMOE_ERR_WORKSPACE_TOO_SMALL";
    case MXMOE_ERR_CUDA: return "MXMOE_ERR_CUDA";
    case MXMOE_ERR_DEVICE_TIMEOUT: return "MXMOE_ERR_DEVICE_TIMEOUT";
    case MXMOE_ERR_DEVICE_CHECK: return "MXMOE_ERR_DEVICE_CHECK";
  }
  return "MXMOE_ERR_UNKNOWN";
}

mxmoe_status mxmoe_get_device_status(int32_t* out_host, int32_t* where_host, void* stream) {
  if (!out_host) return MXMOE_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(S(stream)) != cudaSuccess) return MXMOE_ERR_CUDA;
  int32_t v = 0, w = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(v)) != cudaSuccess) return MXMOE_ERR_CUDA;
  if (cudaMemcpyFromSymbol(&w, g_device_status_where, sizeof(w)) != cudaSuccess) return MXMOE_ERR_CUDA;
  *out_host = v;
  if (where_host) *where_host = w;
  return MXMOE_OK;
}

mxmoe_status mxmoe_clear_device_status(void* stream) {
  static const int32_t zero = 0;
  cudaError_t e = cudaMemcpyToSymbolAsync(g_device_status, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, S(stream));
  if (e == cudaSuccess)
    e = cudaMemcpyToSymbolAsync(g_device_status_where, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, S(stream));
  return cuda_status(e);
}

int64_t mxmoe_rows_capacity(int32_t T, int32_t k, int32_t E) { return rows_cap(T, k, E); }

size_t moe_permute_workspace_size(int32_t T, int32_t k, int32_t E) {
  return route_workspace_bytes(T, k, E);
}

mxmoe_status moe_permute(const int32_t* topk_idx_dev, const float* probs_dev, int32_t T, int32_t k, int32_t E,
                         int32_t* m_splits_dev, int32_t* seg_off_dev, int32_t* row_of_slot_dev,
                         int32_t* token_of_row_dev, float* prob_of_row_dev, void* ws_dev, size_t ws_bytes,
                         void* stream) {
  if (!valid_moe_shape(T, k, E)) return MXMOE_ERR_UNSUPPORTED_SHAPE;
  if ((T > 0 && (!topk_idx_dev || !row_of_slot_dev)) || !m_splits_dev || !seg_off_dev || !token_of_row_dev ||
      !ws_dev)
    return MXMOE_ERR_INVALID_ARG;
  if (prob_of_row_dev && T > 0 && !probs_dev) return MXMOE_ERR_INVALID_ARG;
  if (ws_bytes < moe_permute_workspace_size(T, k, E)) return MXMOE_ERR_WORKSPACE_TOO_SMALL;
  StageScope sc(MXMOE_STAGE_ROUTE, S(stream));
  return cuda_status(launch_route(topk_idx_dev, probs_dev, T, k, E, m_splits_dev, seg_off_dev, row_of_slot_dev,
                                  token_of_row_dev, prob_of_row_dev, ws_dev, S(stream)));
}

mxmoe_status moe_router_topk(const float* logits_dev, int32_t T, int32_t E, int32_t k, int32_t* topk_idx_dev,
                             float* probs_dev, void* stream) {
  if (T < 0 || E < 1 || E > 256 || k < 1 || k > 8 || k > E) return MXMOE_ERR_UNSUPPORTED_SHAPE;
  if (T == 0) return MXMOE_OK;
  if (!logits_dev || !topk_idx_dev || !probs_dev) return MXMOE_ERR_INVALID_ARG;
  StageScope sc(MXMOE_STAGE_ROUTER, S(stream));
  return cuda_status(launch_router_topk(logits_dev, T, E, k, topk_idx_dev, probs_dev, S(stream)));
}

mxmoe_status moe_router_topk_bwd(const float* logits_dev, const int32_t* topk_idx_dev, const float* dprobs_dev,
                                 int32_t T, int32_t E, int32_t k, float* dlogits_dev, void* stream) {
  if (T < 0 || E < 1 || E > 256 || k < 1 || k > 8 || k > E) return MXMOE_ERR_UNSUPPORTED_SHAPE;
  if (T == 0) return MXMOE_OK;
  if (!logits_dev || !topk_idx_dev || !dprobs_dev || !dlogits_dev) return MXMOE_ERR_INVALID_ARG;
  StageScope sc(MXMOE_STAGE_ROUTER_BWD, S(stream));
  return cuda_status(launch_router_topk_bwd(logits_dev, topk_idx_dev, dprobs_dev, T, E, k, dlogits_dev, S(stream)));
}

mxmoe_status moe_unpermute(const void* y_perm_dev, const int32_t* row_of_slot_dev, int32_t T, int32_t k, int32_t H,
                           void* y_dev, void* stream) {
  if (T < 0 || k < 1 || k > 8 || H <= 0 || H % 8 != 0) return MXMOE_ERR_UNSUPPORTED_SHAPE;
  if (T == 0) return MXMOE_OK;
  if (!y_perm_dev || !row_of_slot_dev || !y_dev || !aligned16(y_perm_dev) || !aligned16(y_dev))
    return MXMOE_ERR_INVALID_ARG;
  StageScope sc(MXMOE_STAGE_COMBINE, S(stream));
  return cuda_status(launch_unpermute(y_perm_dev, row_of_slot_dev, T, k, H, y_dev, S(stream)));
}

// mxfp8_quantize with an optional gate/up row interleave of the rowwise copy (row_ilv =
// half the rows of each batch matrix; the library uses it for the fc1 weight operand).
static mxmoe_status quantize_impl(const void* src_dev, int32_t src_dtype, int64_t batch, int64_t rows, int64_t cols,
                                  const int32_t* row_gather_dev, const int32_t* nrows_dev, int64_t out_rows,
                                  const mxmoe_mxfp8* out_row, const mxmoe_mxfp8* out_colT, int64_t row_ilv,
                                  int32_t scale_rule, void* stream, const float* tensor_amax = nullptr,
                                  int32_t tensor_per_batch = 0) {
  if (src_dtype != MXMOE_DTYPE_BF16 && src_dtype != MXMOE_DTYPE_F32) return MXMOE_ERR_INVALID_ARG;
  if (scale_rule != MXMOE_SCALE_RULE_OCP && scale_rule != MXMOE_SCALE_RULE_CEIL) return MXMOE_ERR_INVALID_ARG;
  if (!src_dev || !aligned16(src_dev) || (!out_row && !out_colT)) return MXMOE_ERR_INVALID_ARG;
  if (batch < 1 || rows < 0 || cols <= 0 || out_rows < 0) return MXMOE_ERR_UNSUPPORTED_SHAPE;
  if (row_gather_dev && batch != 1) return MXMOE_ERR_UNSUPPORTED_SHAPE;
  if (!row_gather_dev && out_rows != rows) return MXMOE_ERR_UNSUPPORTED_SHAPE;
  if (cols % 32 != 0 || out_rows % 32 != 0) return MXMOE_ERR_UNSUPPORTED_SHAPE;
  if (out_row) {
    if (!valid_mx(out_row)) return MXMOE_ERR_INVALID_ARG;
    if (out_row->rows != batch * out_rows || out_row->cols != cols) return MXMOE_ERR_UNSUPPORTED_SHAPE;
    if (out_row->scale_layout == MXMOE_SCALE_MMA && (out_rows % 128 != 0 || cols % 128 != 0))
      return MXMOE_ERR_UNSUPPORTED_SHAPE;
  }
  if (out_colT) {
    if (!valid_mx(out_colT)) return MXMOE_ERR_INVALID_ARG;
    if (out_colT->rows != batch * cols || out_colT->cols != out_rows) return MXMOE_ERR_UNSUPPORTED_SHAPE;
    if (out_colT->scale_layout == MXMOE_SCALE_MMA && (out_rows % 128 != 0 || cols % 128 != 0))
      return MXMOE_ERR_UNSUPPORTED_SHAPE;
  }
  if (out_row && out_colT && out_row->elem_format != out_colT->elem_format) return MXMOE_ERR_INVALID_ARG;
  if (out_rows == 0 || rows == 0) return MXMOE_OK;
  QuantArgs a;
  a.fmt = out_row ? out_row->elem_format : out_colT->elem_format;
  a.scale_rule = scale_rule;
  a.src = src_dev;
  a.src_dtype = src_dtype;
  a.batch = batch;
  a.rows = rows;
  a.cols = cols;
  a.gather = row_gather_dev;
  a.nrows = nrows_dev;
  a.out_rows = out_rows;
  a.row_data = out_row ? out_row->data : nullptr;
  a.row_sf = out_row ? out_row->scale : nullptr;
  a.row_layout = out_row ? out_row->scale_layout : 0;
  a.col_data = out_colT ? out_colT->data : nullptr;
  a.col_sf = out_colT ? out_colT->scale : nullptr;
  a.col_layout = out_colT ? out_colT->scale_layout : 0;
  a.row_ilv = row_ilv;
  a.tensor_amax = tensor_amax;
  a.tensor_per_batch = tensor_per_batch;
  if (tensor_amax && a.fmt != MXMOE_FMT_E4M3) return MXMOE_ERR_INVALID_ARG;
  StageScope sc(MXMOE_STAGE_QUANT, S(stream));
  return cuda_status(launch_quantize(a, S(stream)));
}

mxmoe_status mxfp8_quantize(const void* src_dev, int32_t src_dtype, int64_t batch, int64_t rows, int64_t cols,
                            const int32_t* row_gather_dev, const int32_t* nrows_dev, int64_t out_rows,
                            const mxmoe_mxfp8* out_row, const mxmoe_mxfp8* out_colT, void* stream) {
  return quantize_impl(src_dev, src_dtype, batch, rows, cols, row_gather_dev, nrows_dev, out_rows, out_row, out_colT, 0,
                       MXMOE_SCALE_RULE_OCP, stream);
}

mxmoe_status mxfp8_quantize_ex(const void* src_dev, int32_t src_dtype, int64_t batch, int64_t rows, int64_t cols,
                               const int32_t* row_gather_dev, const int32_t* nrows_dev, int64_t out_rows,
                               const mxmoe_mxfp8* out_row, const mxmoe_mxfp8* out_colT, int32_t scale_rule,
                               void* stream) {
  return quantize_impl(src_dev, src_dtype, batch, rows, cols, row_gather_dev, nrows_dev, out_rows, out_row, out_colT, 0,
                       scale_rule, stream);
}

mxmoe_status mxfp8_dequantize(const mxmoe_mxfp8* src_row, void* dst_dev, void* stream) {
  if (!src_row || !valid_mx(src_row) || !dst_dev || !aligned16(dst_dev)) return MXMOE_ERR_INVALID_ARG;
  if (src_row->scale_layout != MXMOE_SCALE_PLAIN) return MXMOE_ERR_INVALID_ARG;
  if (src_row->rows < 0 || src_row->cols <= 0 || src_row->cols % 32 != 0) return MXMOE_ERR_UNSUPPORTED_SHAPE;
  if (src_row->rows == 0) return MXMOE_OK;
  return cuda_status(launch_dequantize_rows(src_row->data, src_row->scale, src_row->rows, src_row->cols,
                                            src_row->elem_format, dst_dev, S(stream)));
}

static mxmoe_status grouped_gemm_impl(const mxmoe_mxfp8* A, const mxmoe_mxfp8* B, const int32_t* seg_off_dev,
                                      int32_t E, int64_t N, int64_t K, void* C_dev, int32_t c_dtype, int64_t ldc,
                                      int32_t debug_drop_commit, void* stream, const float* a_amax = nullptr,
                                      const float* b_amax = nullptr) {
  if (!A || !B || !seg_off_dev || !C_dev || !aligned16(C_dev)) return MXMOE_ERR_INVALID_ARG;
  if (c_dtype != MXMOE_DTYPE_BF16 && c_dtype != MXMOE_DTYPE_F32) return MXMOE_ERR_INVALID_ARG;
  if (!mma_ready(A) || !mma_ready(B)) return MXMOE_ERR_INVALID_ARG;
  if (E < 1 || E > 256 || N <= 0 || K <= 0 || N % 256 != 0 || K % 128 != 0) return MXMOE_ERR_UNSUPPORTED_SHAPE;
  if (A->rows % 256 != 0 || A->cols != K || B->cols != K || B->rows != (int64_t)E * N || ldc < N || ldc % 8 != 0)
    return MXMOE_ERR_UNSUPPORTED_SHAPE;
  if (A->rows == 0) return MXMOE_OK;
  GemmArgs g = gemm_base(kModeStore, *A, *B, seg_off_dev, E);
  g.N = N;
  g.K = K;
  g.c = C_dev;
  g.c_dtype = c_dtype;
  g.ldc = ldc;
  g.debug_drop_commit = debug_drop_commit;
  g.a_amax = a_amax;  // per-tensor FP8 operands (b: one value per expert)
  g.b_amax = b_amax;
  g.b_amax_per_expert = 1;
  StageScope sc(MXMOE_STAGE_GEMM, S(stream));
  return cuda_status(launch_gemm(g, S(stream)));
}

mxmoe_status grouped_gemm_mxfp8(const mxmoe_mxfp8* A, const mxmoe_mxfp8* B, const int32_t* seg_off_dev,
                                int32_t E, int64_t N, int64_t K, void* C_dev, int32_t c_dtype, int64_t ldc,
                                void* stream) {
  return grouped_gemm_impl(A, B, seg_off_dev, E, N, K, C_dev, c_dtype, ldc, 0, stream);
}

mxmoe_status grouped_gemm_mxfp8_debug_timeout(const mxmoe_mxfp8* A, const mxmoe_mxfp8* B,
                                              const int32_t* seg_off_dev, int32_t E, int64_t N, int64_t K,
                                              void* C_dev, int32_t c_dtype, int64_t ldc, void* stream) {
  return grouped_gemm_impl(A, B, seg_off_dev, E, N, K, C_dev, c_dtype, ldc, 1, stream);
}

static mxmoe_status grouped_wgrad_impl(const mxmoe_mxfp8* At, const mxmoe_mxfp8* Bt, const int32_t* seg_off_dev,
                                       int32_t E, float* C_dev, void* stream, const float* a_amax,
                                       const float* b_amax);
mxmoe_status grouped_gemm_mxfp8_wgrad(const mxmoe_mxfp8* At, const mxmoe_mxfp8* Bt, const int32_t* seg_off_dev,
                                      int32_t E, float* C_dev, void* stream) {
  return grouped_wgrad_impl(At, Bt, seg_off_dev, E, C_dev, stream, nullptr, nullptr);
}
static mxmoe_status grouped_wgrad_impl(const mxmoe_mxfp8* At, const mxmoe_mxfp8* Bt, const int32_t* seg_off_dev,
                                       int32_t E, float* C_dev, void* stream, const float* a_amax,
                                       const float* b_amax) {
  if (!At || !Bt || !seg_off_dev || !C_dev || !aligned16(C_dev)) return MXMOE_ERR_INVALID_ARG;
  if (!mma_ready(At) || !mma_ready(Bt)) return MXMOE_ERR_INVALID_ARG;
  if (E < 1 || E > 256 || At->cols != Bt->cols || At->rows <= 0 || At->rows % 256 != 0 || Bt->rows % 256 != 0 ||
      Bt->rows <= 0 || At->cols % 256 != 0)
    return MXMOE_ERR_UNSUPPORTED_SHAPE;
  GemmArgs g = gemm_base(kModeWgrad, *At, *Bt, seg_off_dev, E);
  g.N = At->rows;
  g.K2 = Bt->rows;
  g.c = C_dev;
  g.c_dtype = MXMOE_DTYPE_F32;
  g.ldc = Bt->rows;
  g.a_amax = a_amax;  // per-tensor FP8 operands (one value each)
  g.b_amax = b_amax;
  StageScope sc(MXMOE_STAGE_WGRAD, S(stream));
  return cuda_status(launch_gemm(g, S(stream)));
}

mxmoe_status grouped_gemm_bf16(const void* A_dev, int64_t rows_cap, const void* B_dev, const int32_t* seg_off_dev,
                               int32_t E, int64_t N, int64_t K, void* C_dev, int32_t c_dtype, int64_t ldc,
                               void* stream) {
  if (!A_dev || !B_dev || !seg_off_dev || !C_dev || !aligned16(A_dev) || !aligned16(B_dev) || !aligned16(C_dev))
    return MXMOE_ERR_INVALID_ARG;
  if (c_dtype != MXMOE_DTYPE_BF16 && c_dtype != MXMOE_DTYPE_F32) return MXMOE_ERR_INVALID_ARG;
  if (E < 1 || E > 256 || N <= 0 || K <= 0 || rows_cap < 0 || N % 256 != 0 || K % 64 != 0 || rows_cap % 256 != 0 ||
      ldc < N || ldc % 8 != 0)
    return MXMOE_ERR_UNSUPPORTED_SHAPE;
  if (rows_cap == 0) return MXMOE_OK;
  GemmArgs g;
  std::memset(&g, 0, sizeof(g));
  g.mode = kModeStore;
  g.bf16_operands = 1;
  g.E = E;
  g.a_data = static_cast<const uint8_t*>(A_dev);
  g.a_rows = rows_cap;
  g.a_cols = K;
  g.b_data = static_cast<const uint8_t*>(B_dev);
  g.b_rows = (int64_t)E * N;
  g.b_cols = K;
  g.seg_off = seg_off_dev;
  g.N = N;
  g.K = K;
  g.c = C_dev;
  g.c_dtype = c_dtype;
  g.ldc = ldc;
  StageScope sc(MXMOE_STAGE_GEMM, S(stream));
  return cuda_status(launch_gemm(g, S(stream)));
}

mxmoe_status grouped_gemm_bf16_wgrad(const void* At_dev, const void* Bt_dev, int64_t N, int64_t K2, int64_t rows_cap,
                                     const int32_t* seg_off_dev, int32_t E, float* C_dev, void* stream) {
  if (!At_dev || !Bt_dev || !seg_off_dev || !C_dev || !aligned16(At_dev) || !aligned16(Bt_dev) || !aligned16(C_dev))
    return MXMOE_ERR_INVALID_ARG;
  if (E < 1 || E > 256 || N <= 0 || K2 <= 0 || rows_cap <= 0 || N % 256 != 0 || K2 % 256 != 0 || rows_cap % 256 != 0)
    return MXMOE_ERR_UNSUPPORTED_SHAPE;
  GemmArgs g;
  std::memset(&g, 0, sizeof(g));
  g.mode = kModeWgrad;
  g.bf16_operands = 1;
  g.E = E;
  g.a_data = static_cast<const uint8_t*>(At_dev);
  g.a_rows = N;
  g.a_cols = rows_cap;
  g.b_data = static_cast<const uint8_t*>(Bt_dev);
  g.b_rows = K2;
  g.b_cols = rows_cap;
  g.seg_off = seg_off_dev;
  g.N = N;
  g.K2 = K2;
  g.c = C_dev;
  g.c_dtype = MXMOE_DTYPE_F32;
  g.ldc = K2;
  StageScope sc(MXMOE_STAGE_WGRAD, S(stream));
  return cuda_status(launch_gemm(g, S(stream)));
}

size_t mxmoe_weights_size(int32_t E, int32_t H, int32_t F) { return weights_layout(E, H, F).total; }

mxmoe_status mxmoe_weights_view(void* wq_dev, int32_t E, int32_t H, int32_t F, int32_t which, mxmoe_mxfp8* out) {
  if (!wq_dev || !out || which < 0 || which > 3) return MXMOE_ERR_INVALID_ARG;
  const WeightsLayout L = weights_layout(E, H, F);
  *out = mk(reinterpret_cast<uint8_t*>(wq_dev), L.d[which], L.s[which], L.rows[which], L.cols[which]);
  return MXMOE_OK;
}

mxmoe_status mxmoe_weights_quantize(const void* W1_dev, const void* W2_dev, int32_t E, int32_t H, int32_t F,
                                    void* wq_dev, size_t wq_bytes, void* stream) {
  return mxmoe_weights_quantize_ex(W1_dev, W2_dev, E, H, F, MXMOE_SCALE_RULE_OCP, wq_dev, wq_bytes, stream);
}

mxmoe_status mxmoe_weights_quantize_ex(const void* W1_dev, const void* W2_dev, int32_t E, int32_t H, int32_t F,
                                       int32_t scale_rule, void* wq_dev, size_t wq_bytes, void* stream) {
  if (scale_rule != MXMOE_SCALE_RULE_OCP && scale_rule != MXMOE_SCALE_RULE_CEIL) return MXMOE_ERR_INVALID_ARG;
  if (E < 1 || E > 256 || H <= 0 || F <= 0 || H % 256 != 0 || F % 256 != 0) return MXMOE_ERR_UNSUPPORTED_SHAPE;
  if (!W1_dev || !W2_dev || !wq_dev || !aligned16(W1_dev) || !aligned16(W2_dev) || !aligned16(wq_dev))
    return MXMOE_ERR_INVALID_ARG;
  const WeightsLayout L = weights_layout(E, H, F);
  if (wq_bytes < L.total) return MXMOE_ERR_WORKSPACE_TOO_SMALL;
  uint8_t* b = reinterpret_cast<uint8_t*>(wq_dev);
  mxmoe_mxfp8 w1r = mk(b, L.d[0], L.s[0], L.rows[0], L.cols[0]);
  mxmoe_mxfp8 w1c = mk(b, L.d[1], L.s[1], L.rows[1], L.cols[1]);
  mxmoe_mxfp8 w2r = mk(b, L.d[2], L.s[2], L.rows[2], L.cols[2]);
  mxmoe_mxfp8 w2c = mk(b, L.d[3], L.s[3], L.rows[3], L.cols[3]);
  mxmoe_status s;
  {
    StageScope sc(MXMOE_STAGE_QUANT_W1, S(stream));
    s = quantize_impl(W1_dev, MXMOE_DTYPE_BF16, E, 2 * (int64_t)F, H, nullptr, nullptr, 2 * (int64_t)F, &w1r, &w1c,
                      F, scale_rule, stream);
  }
  if (s != MXMOE_OK) return s;
  StageScope sc(MXMOE_STAGE_QUANT_W2, S(stream));
  return mxfp8_quantize_ex(W2_dev, MXMOE_DTYPE_BF16, E, H, F, nullptr, nullptr, H, &w2r, &w2c, scale_rule, stream);
}

mxmoe_status mxmoe_weights_quantize_fp8(const void* W1_dev, const void* W2_dev, int32_t E, int32_t H, int32_t F,
                                        void* wq_dev, size_t wq_bytes, void* stream) {
  if (E < 1 || E > 256 || H <= 0 || F <= 0 || H % 256 != 0 || F % 256 != 0) return MXMOE_ERR_UNSUPPORTED_SHAPE;
  if (!W1_dev || !W2_dev || !wq_dev || !aligned16(W1_dev) || !aligned16(W2_dev) || !aligned16(wq_dev))
    return MXMOE_ERR_INVALID_ARG;
  const WeightsLayout L = weights_layout(E, H, F);
  if (wq_bytes < L.total) return MXMOE_ERR_WORKSPACE_TOO_SMALL;
  uint8_t* b = reinterpret_cast<uint8_t*>(wq_dev);
  mxmoe_mxfp8 w1r = mk(b, L.d[0], L.s[0], L.rows[0], L.cols[0]);
  mxmoe_mxfp8 w1c = mk(b, L.d[1], L.s[1], L.rows[1], L.cols[1]);
  mxmoe_mxfp8 w2r = mk(b, L.d[2], L.s[2], L.rows[2], L.cols[2]);
  mxmoe_mxfp8 w2c = mk(b, L.d[3], L.s[3], L.rows[3], L.cols[3]);
  float* am = reinterpret_cast<float*>(b + L.amax);  // W1[e] then W2[e]
  cudaStream_t st = S(stream);
  mxmoe_status s;
  {
    StageScope sc(MXMOE_STAGE_QUANT_W1, st);
    if (launch_amax_bf16(W1_dev, 2 * (int64_t)F * H, E, am, st) != cudaSuccess) return MXMOE_ERR_CUDA;
    s = quantize_impl(W1_dev, MXMOE_DTYPE_BF16, E, 2 * (int64_t)F, H, nullptr, nullptr, 2 * (int64_t)F, &w1r, &w1c,
                      F, MXMOE_SCALE_RULE_OCP, stream, am, 1);
  }
  if (s != MXMOE_OK) return s;
  StageScope sc(MXMOE_STAGE_QUANT_W2, st);
  if (launch_amax_bf16(W2_dev, (int64_t)H * F, E, am + E, st) != cudaSuccess) return MXMOE_ERR_CUDA;
  return quantize_impl(W2_dev, MXMOE_DTYPE_BF16, E, H, F, nullptr, nullptr, H, &w2r, &w2c, 0, MXMOE_SCALE_RULE_OCP,
                       stream, am + E, 1);
}

size_t grouped_mlp_saved_size(int32_t T, int32_t k, int32_t E, int32_t H, int32_t F) {
  return grouped_mlp_saved_size_ex(T, k, E, H, F, 0);
}
size_t grouped_mlp_saved_size_ex(int32_t T, int32_t k, int32_t E, int32_t H, int32_t F, int32_t recipe) {
  if (!valid_recipe(recipe)) return 0;
  return saved_layout(T, k, E, H, F, recipe).total;
}

int64_t grouped_mlp_saved_offset(int32_t field, int32_t T, int32_t k, int32_t E, int32_t H, int32_t F) {
  return grouped_mlp_saved_offset_ex(field, T, k, E, H, F, 0);
}
int64_t grouped_mlp_saved_offset_ex(int32_t field, int32_t T, int32_t k, int32_t E, int32_t H, int32_t F,
                                    int32_t recipe) {
  if (field < 0 || field > 12 || !valid_recipe(recipe)) return -1;
  return (int64_t)saved_layout(T, k, E, H, F, recipe).off[field];
}

size_t grouped_mlp_workspace_size(int32_t T, int32_t k, int32_t E, int32_t H, int32_t F) {
  return grouped_mlp_workspace_size_ex(T, k, E, H, F, 0);
}
size_t grouped_mlp_workspace_size_ex(int32_t T, int32_t k, int32_t E, int32_t H, int32_t F, int32_t recipe) {
  if (!valid_recipe(recipe)) return 0;
  return std::max(fwd_ws(T, k, E, H, F).total, bwd_ws(T, k, E, H, F, recipe).total);
}

mxmoe_status grouped_mlp_fwd(const void* x_dev, const int32_t* topk_idx_dev, const float* probs_dev,
                             const void* wq_dev, size_t wq_bytes, int32_t T, int32_t k, int32_t E, int32_t H,
                             int32_t F, void* y_dev, void* saved_dev, size_t saved_bytes, void* ws_dev,
                             size_t ws_bytes, void* stream) {
  return grouped_mlp_fwd_ex(x_dev, topk_idx_dev, probs_dev, wq_dev, wq_bytes, T, k, E, H, F, 0, y_dev, saved_dev,
                            saved_bytes, ws_dev, ws_bytes, stream);
}

static mxmoe_status fwd_impl(const void* x_dev, const int32_t* topk_idx_dev, const float* probs_dev,
                             const void* wq_dev, size_t wq_bytes, int32_t T, int32_t k, int32_t E, int32_t H,
                             int32_t F, int32_t recipe, float* amax_state, void* y_dev, void* saved_dev,
                             size_t saved_bytes, void* ws_dev, size_t ws_bytes, void* stream);

mxmoe_status grouped_mlp_fwd_ex(const void* x_dev, const int32_t* topk_idx_dev, const float* probs_dev,
                                const void* wq_dev, size_t wq_bytes, int32_t T, int32_t k, int32_t E, int32_t H,
                                int32_t F, int32_t recipe, void* y_dev, void* saved_dev, size_t saved_bytes,
                                void* ws_dev, size_t ws_bytes, void* stream) {
  if (fp8_tensor(recipe)) return MXMOE_ERR_INVALID_ARG;  // per-tensor FP8: grouped_mlp_fp8_fwd
  return fwd_impl(x_dev, topk_idx_dev, probs_dev, wq_dev, wq_bytes, T, k, E, H, F, recipe, nullptr, y_dev, saved_dev,
                  saved_bytes, ws_dev, ws_bytes, stream);
}

mxmoe_status grouped_mlp_fp8_fwd(const void* x_dev, const int32_t* topk_idx_dev, const float* probs_dev,
                                 const void* wq_dev, size_t wq_bytes, int32_t T, int32_t k, int32_t E, int32_t H,
                                 int32_t F, float* amax_state_dev, void* y_dev, void* saved_dev, size_t saved_bytes,
                                 void* ws_dev, size_t ws_bytes, void* stream) {
  if (!amax_state_dev || !aligned16(amax_state_dev)) return MXMOE_ERR_INVALID_ARG;
  return fwd_impl(x_dev, topk_idx_dev, probs_dev, wq_dev, wq_bytes, T, k, E, H, F, MXMOE_RECIPE_FP8_TENSOR,
                  amax_state_dev, y_dev, saved_dev, saved_bytes, ws_dev, ws_bytes, stream);
}

static mxmoe_status fwd_impl(const void* x_dev, const int32_t* topk_idx_dev, const float* probs_dev,
                             const void* wq_dev, size_t wq_bytes, int32_t T, int32_t k, int32_t E, int32_t H,
                             int32_t F, int32_t recipe, float* amax_state, void* y_dev, void* saved_dev,
                             size_t saved_bytes, void* ws_dev, size_t ws_bytes, void* stream) {
  if (!valid_recipe(recipe)) return MXMOE_ERR_INVALID_ARG;
  if (!valid_mlp_shape(T, k, E, H, F)) return MXMOE_ERR_UNSUPPORTED_SHAPE;
  if (!wq_dev || !saved_dev || !ws_dev || !aligned16(wq_dev) || !aligned16(saved_dev) || !aligned16(ws_dev))
    return MXMOE_ERR_INVALID_ARG;
  if (T > 0 && (!x_dev || !topk_idx_dev || !probs_dev || !y_dev || !aligned16(x_dev) || !aligned16(y_dev)))
    return MXMOE_ERR_INVALID_ARG;
  if (wq_bytes < mxmoe_weights_size(E, H, F) || saved_bytes < grouped_mlp_saved_size_ex(T, k, E, H, F, recipe) ||
      ws_bytes < grouped_mlp_workspace_size_ex(T, k, E, H, F, recipe))
    return MXMOE_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = S(stream);
  const int64_t cap = rows_cap(T, k, E);
  const bool rc = recomputes_gu(recipe);
  const SavedLayout SL = saved_layout(T, k, E, H, F, recipe);
  const FwdWs W = fwd_ws(T, k, E, H, F);
  const WeightsLayout WL = weights_layout(E, H, F);
  uint8_t* sv = reinterpret_cast<uint8_t*>(saved_dev);
  uint8_t* ws = reinterpret_cast<uint8_t*>(ws_dev);
  uint8_t* wq = reinterpret_cast<uint8_t*>(const_cast<void*>(wq_dev));
  int32_t* m_splits = reinterpret_cast<int32_t*>(sv + SL.off[MXMOE_SAVED_M_SPLITS]);
  int32_t* seg_off = reinterpret_cast<int32_t*>(sv + SL.off[MXMOE_SAVED_SEG_OFF]);
  int32_t* ros = reinterpret_cast<int32_t*>(sv + SL.off[MXMOE_SAVED_ROW_OF_SLOT]);
  int32_t* tor = reinterpret_cast<int32_t*>(sv + SL.off[MXMOE_SAVED_TOKEN_OF_ROW]);
  float* por = reinterpret_cast<float*>(sv + SL.off[MXMOE_SAVED_PROB_OF_ROW]);

  // 1. route
  cudaError_t e;
  {
    StageScope sc(MXMOE_STAGE_ROUTE, st);
    e = launch_route(topk_idx_dev, probs_dev, T, k, E, m_splits, seg_off, ros, tor, por, ws + W.route, st);
  }
  if (e != cudaSuccess) return MXMOE_ERR_CUDA;
  // per-tensor FP8: largest |x| and the Z amax this forward encodes with (both kept in the
  // saved buffer for the backward); this step's largest |Z| is recorded into amax_state[1]
  const bool pt = fp8_tensor(recipe);
  float* x_amax = pt ? reinterpret_cast<float*>(sv + SL.off[MXMOE_SAVED_AMAX]) : nullptr;
  float* z_used = pt ? x_amax + 1 : nullptr;
  const float* w1_amax = pt ? reinterpret_cast<const float*>(wq + WL.amax) : nullptr;
  const float* w2_amax = pt ? w1_amax + E : nullptr;
  if (pt && (cudaMemcpyAsync(z_used, amax_state, 4, cudaMemcpyDeviceToDevice, st) != cudaSuccess ||
             cudaMemsetAsync(amax_state + 1, 0, 4, st) != cudaSuccess))
    return MXMOE_ERR_CUDA;
  if (T == 0) return MXMOE_OK;
  // 2. permute + quantise x (rowwise for fc1 -- saved when the backward recomputes G / U --
  // and colwise, saved for fc1 wgrad)
  mxmoe_mxfp8 x_row = rc ? mk(sv, SL.off[MXMOE_SAVED_X_ROW], SL.off[MXMOE_SAVED_X_ROW_SF], cap, H)
                         : mk(ws, W.x_row, W.x_row_sf, cap, H);
  mxmoe_mxfp8 x_col = mk(sv, SL.off[MXMOE_SAVED_X_COLT], SL.off[MXMOE_SAVED_X_COLT_SF], H, cap);
  mxmoe_status s;
  {
    StageScope sc(MXMOE_STAGE_QUANT_X, st);
    if (pt && launch_amax_bf16(x_dev, (int64_t)T * H, 1, x_amax, st) != cudaSuccess) return MXMOE_ERR_CUDA;
    s = quantize_impl(x_dev, MXMOE_DTYPE_BF16, 1, T, H, tor, seg_off + E, cap, &x_row, &x_col, 0,
                      recipe_scale_rule(recipe), stream, x_amax, 0);
  }
  if (s != MXMOE_OK) return s;
  // 3. fc1 + SwiGLU x prob -> Z (MXFP8 row + colT), G/U saved unless recomputed
  mxmoe_mxfp8 w1r = mk(wq, WL.d[0], WL.s[0], WL.rows[0], WL.cols[0]);
  GemmArgs g = gemm_base(kModeSwigluFwd, x_row, w1r, seg_off, E);
  g.K = H;
  g.F = F;
  g.N = 2 * (int64_t)F;
  g.rows_cap = cap;
  g.prob_of_row = por;
  g.z_row = ws + W.z_row;
  g.z_row_sf = ws + W.z_row_sf;
  g.z_colT = sv + SL.off[MXMOE_SAVED_Z_COLT];
  g.z_colT_sf = sv + SL.off[MXMOE_SAVED_Z_COLT_SF];
  g.scale_rule = recipe_scale_rule(recipe);
  g.gu = rc ? nullptr : reinterpret_cast<uint16_t*>(sv + SL.off[MXMOE_SAVED_GU]);
  g.a_amax = x_amax;
  g.b_amax = w1_amax;
  g.b_amax_per_expert = 1;
  g.out_amax_in = z_used;
  g.out_amax_rec = pt ? amax_state + 1 : nullptr;
  {
    StageScope sc(MXMOE_STAGE_FC1_SWIGLU, st);
    e = launch_gemm(g, st);
  }
  if (e != cudaSuccess) return MXMOE_ERR_CUDA;
  // 4. fc2 -> Yp bf16
  mxmoe_mxfp8 z_row = mk(ws, W.z_row, W.z_row_sf, cap, F);
  mxmoe_mxfp8 w2r = mk(wq, WL.d[2], WL.s[2], WL.rows[2], WL.cols[2]);
  {
    StageScope sc(MXMOE_STAGE_FC2, st);
    s = grouped_gemm_impl(&z_row, &w2r, seg_off, E, H, F, ws + W.y_perm, MXMOE_DTYPE_BF16, H, 0, stream, z_used,
                          w2_amax);
  }
  if (s != MXMOE_OK) return s;
  // 5. combine
  StageScope sc(MXMOE_STAGE_COMBINE, st);
  return moe_unpermute(ws + W.y_perm, ros, T, k, H, y_dev, stream);
}

mxmoe_status grouped_mlp_bwd(const void* dy_dev, const void* saved_dev, size_t saved_bytes, const void* wq_dev,
                             size_t wq_bytes, int32_t T, int32_t k, int32_t E, int32_t H, int32_t F, void* dx_dev,
                             float* dW1_dev, float* dW2_dev, float* dprobs_dev, void* ws_dev, size_t ws_bytes,
                             void* stream) {
  return grouped_mlp_bwd_ex(dy_dev, saved_dev, saved_bytes, wq_dev, wq_bytes, T, k, E, H, F, 0, dx_dev, dW1_dev,
                            dW2_dev, dprobs_dev, ws_dev, ws_bytes, stream);
}

static mxmoe_status bwd_impl(const void* dy_dev, const void* saved_dev, size_t saved_bytes, const void* wq_dev,
                             size_t wq_bytes, int32_t T, int32_t k, int32_t E, int32_t H, int32_t F, int32_t recipe,
                             float* amax_state, void* dx_dev, float* dW1_dev, float* dW2_dev, float* dprobs_dev,
                             void* ws_dev, size_t ws_bytes, void* stream);

mxmoe_status grouped_mlp_bwd_ex(const void* dy_dev, const void* saved_dev, size_t saved_bytes, const void* wq_dev,
                                size_t wq_bytes, int32_t T, int32_t k, int32_t E, int32_t H, int32_t F,
                                int32_t recipe, void* dx_dev, float* dW1_dev, float* dW2_dev, float* dprobs_dev,
                                void* ws_dev, size_t ws_bytes, void* stream) {
  if (fp8_tensor(recipe)) return MXMOE_ERR_INVALID_ARG;  // per-tensor FP8: grouped_mlp_fp8_bwd
  return bwd_impl(dy_dev, saved_dev, saved_bytes, wq_dev, wq_bytes, T, k, E, H, F, recipe, nullptr, dx_dev, dW1_dev,
                  dW2_dev, dprobs_dev, ws_dev, ws_bytes, stream);
}

mxmoe_status grouped_mlp_fp8_bwd(const void* dy_dev, const void* saved_dev, size_t saved_bytes, const void* wq_dev,
                                 size_t wq_bytes, int32_t T, int32_t k, int32_t E, int32_t H, int32_t F,
                                 float* amax_state_dev, void* dx_dev, float* dW1_dev, float* dW2_dev,
                                 float* dprobs_dev, void* ws_dev, size_t ws_bytes, void* stream) {
  if (!amax_state_dev || !aligned16(amax_state_dev)) return MXMOE_ERR_INVALID_ARG;
  return bwd_impl(dy_dev, saved_dev, saved_bytes, wq_dev, wq_bytes, T, k, E, H, F, MXMOE_RECIPE_FP8_TENSOR,
                  amax_state_dev, dx_dev, dW1_dev, dW2_dev, dprobs_dev, ws_dev, ws_bytes, stream);
}

static mxmoe_status bwd_impl(const void* dy_dev, const void* saved_dev, size_t saved_bytes, const void* wq_dev,
                             size_t wq_bytes, int32_t T, int32_t k, int32_t E, int32_t H, int32_t F, int32_t recipe,
                             float* amax_state, void* dx_dev, float* dW1_dev, float* dW2_dev, float* dprobs_dev,
                             void* ws_dev, size_t ws_bytes, void* stream) {
  if (!valid_recipe(recipe)) return MXMOE_ERR_INVALID_ARG;
  const int32_t grad_format = (recipe & MXMOE_RECIPE_GRAD_E5M2) ? MXMOE_FMT_E5M2 : MXMOE_FMT_E4M3;
  if (!valid_mlp_shape(T, k, E, H, F)) return MXMOE_ERR_UNSUPPORTED_SHAPE;
  if (!wq_dev || !saved_dev || !ws_dev || !dW1_dev || !dW2_dev || !aligned16(wq_dev) || !aligned16(saved_dev) ||
      !aligned16(ws_dev) || !aligned16(dW1_dev) || !aligned16(dW2_dev))
    return MXMOE_ERR_INVALID_ARG;
  if (T > 0 && (!dy_dev || !dx_dev || !dprobs_dev || !aligned16(dy_dev) || !aligned16(dx_dev)))
    return MXMOE_ERR_INVALID_ARG;
  if (wq_bytes < mxmoe_weights_size(E, H, F) || saved_bytes < grouped_mlp_saved_size_ex(T, k, E, H, F, recipe) ||
      ws_bytes < grouped_mlp_workspace_size_ex(T, k, E, H, F, recipe))
    return MXMOE_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = S(stream);
  const int64_t cap = rows_cap(T, k, E);
  const bool rc = recomputes_gu(recipe);
  const SavedLayout SL = saved_layout(T, k, E, H, F, recipe);
  const BwdWs W = bwd_ws(T, k, E, H, F, recipe);
  const WeightsLayout WL = weights_layout(E, H, F);
  uint8_t* sv = reinterpret_cast<uint8_t*>(const_cast<void*>(saved_dev));
  uint8_t* ws = reinterpret_cast<uint8_t*>(ws_dev);
  uint8_t* wq = reinterpret_cast<uint8_t*>(const_cast<void*>(wq_dev));
  const int32_t* seg_off = reinterpret_cast<const int32_t*>(sv + SL.off[MXMOE_SAVED_SEG_OFF]);
  const int32_t* ros = reinterpret_cast<const int32_t*>(sv + SL.off[MXMOE_SAVED_ROW_OF_SLOT]);
  const int32_t* tor = reinterpret_cast<const int32_t*>(sv + SL.off[MXMOE_SAVED_TOKEN_OF_ROW]);
  const float* por = reinterpret_cast<const float*>(sv + SL.off[MXMOE_SAVED_PROB_OF_ROW]);

  // per-tensor FP8: the forward's largest |x| and Z amax (saved), largest |dY| and the dGU
  // amax this backward encodes with (workspace); this step's largest |dGU| is recorded into
  // amax_state[3]
  const bool pt = fp8_tensor(recipe);
  const float* x_amax = pt ? reinterpret_cast<const float*>(sv + SL.off[MXMOE_SAVED_AMAX]) : nullptr;
  const float* z_used = pt ? x_amax + 1 : nullptr;
  float* dy_amax = pt ? reinterpret_cast<float*>(ws + W.amax) : nullptr;
  float* dgu_used = pt ? dy_amax + 1 : nullptr;
  const float* w1_amax = pt ? reinterpret_cast<const float*>(wq + WL.amax) : nullptr;
  const float* w2_amax = pt ? w1_amax + E : nullptr;
  if (pt && (cudaMemcpyAsync(dgu_used, amax_state + 2, 4, cudaMemcpyDeviceToDevice, st) != cudaSuccess ||
             cudaMemsetAsync(amax_state + 3, 0, 4, st) != cudaSuccess))
    return MXMOE_ERR_CUDA;
  // 1. permute + quantise dy: rowwise (fc2 dgrad) and colwise (fc2 wgrad)
  mxmoe_mxfp8 dy_row = mk(ws, W.dy_row, W.dy_row_sf, cap, H, grad_format);
  mxmoe_mxfp8 dy_col = mk(ws, W.dy_colT, W.dy_colT_sf, H, cap, grad_format);
  mxmoe_status s;
  if (T > 0) {
    StageScope sc(MXMOE_STAGE_QUANT_DY, st);
    if (pt && launch_amax_bf16(dy_dev, (int64_t)T * H, 1, dy_amax, st) != cudaSuccess) return MXMOE_ERR_CUDA;
    s = quantize_impl(dy_dev, MXMOE_DTYPE_BF16, 1, T, H, tor, seg_off + E, cap, &dy_row, &dy_col, 0,
                      recipe_scale_rule(recipe), stream, dy_amax, 0);
    if (s != MXMOE_OK) return s;
  }
  // 1b. G / U recomputed from the saved rowwise x (the fc1 GEMM again, epilogue writing
  // only G / U) when the forward did not save them
  if (rc && T > 0) {
    mxmoe_mxfp8 x_row = mk(sv, SL.off[MXMOE_SAVED_X_ROW], SL.off[MXMOE_SAVED_X_ROW_SF], cap, H);
    mxmoe_mxfp8 w1r = mk(wq, WL.d[0], WL.s[0], WL.rows[0], WL.cols[0]);
    GemmArgs g = gemm_base(kModeSwigluFwd, x_row, w1r, seg_off, E);
    g.K = H;
    g.F = F;
    g.N = 2 * (int64_t)F;
    g.rows_cap = cap;
    g.prob_of_row = por;
    g.gu = reinterpret_cast<uint16_t*>(ws + W.gu);
    StageScope sc(MXMOE_STAGE_FC1_RECOMPUTE, st);
    if (launch_gemm(g, st) != cudaSuccess) return MXMOE_ERR_CUDA;
  }
  const uint16_t* gu = reinterpret_cast<const uint16_t*>(rc ? ws + W.gu : sv + SL.off[MXMOE_SAVED_GU]);
  // 2. fc2 dgrad + SwiGLU/prob backward -> dGU (MXFP8 row + colT), dprob partials
  mxmoe_mxfp8 w2c = mk(wq, WL.d[3], WL.s[3], WL.rows[3], WL.cols[3]);
  {
    GemmArgs g = gemm_base(kModeSwigluBwd, dy_row, w2c, seg_off, E);
    g.K = H;
    g.N = F;
    g.F = F;
    g.rows_cap = cap;
    g.prob_of_row = por;
    g.gu_in = gu;
    g.dgu_row = ws + W.dgu_row;
    g.dgu_row_sf = ws + W.dgu_row_sf;
    g.dgu_colT = ws + W.dgu_colT;
    g.dgu_colT_sf = ws + W.dgu_colT_sf;
    g.dprob_part = reinterpret_cast<float*>(ws + W.dprob_part);
    g.out_fmt = grad_format;
    g.scale_rule = recipe_scale_rule(recipe);
    g.a_amax = dy_amax;
    g.b_amax = w2_amax;
    g.b_amax_per_expert = 1;
    g.out_amax_in = dgu_used;
    g.out_amax_rec = pt ? amax_state + 3 : nullptr;
    StageScope sc(MXMOE_STAGE_FC2_DGRAD, st);
    if (T > 0 && launch_gemm(g, st) != cudaSuccess) return MXMOE_ERR_CUDA;
  }
  // 3. dprobs
  {
    StageScope sc(MXMOE_STAGE_DPROB, st);
    if (launch_dprob_reduce(reinterpret_cast<const float*>(ws + W.dprob_part), F / 128, ros, (int64_t)T * k,
                            dprobs_dev, st) != cudaSuccess)
      return MXMOE_ERR_CUDA;
  }
  // 4. fc2 wgrad: dW2[e] = dYp_e^T . Z_e
  mxmoe_mxfp8 z_col = mk(sv, SL.off[MXMOE_SAVED_Z_COLT], SL.off[MXMOE_SAVED_Z_COLT_SF], F, cap);
  {
    StageScope sc(MXMOE_STAGE_FC2_WGRAD, st);
    s = grouped_wgrad_impl(&dy_col, &z_col, seg_off, E, dW2_dev, stream, dy_amax, z_used);
  }
  if (s != MXMOE_OK) return s;
  // 5. fc1 dgrad: dXp = dGU . W1 (contract 2F)
  mxmoe_mxfp8 dgu_row = mk(ws, W.dgu_row, W.dgu_row_sf, cap, 2 * (int64_t)F, grad_format);
  mxmoe_mxfp8 w1c = mk(wq, WL.d[1], WL.s[1], WL.rows[1], WL.cols[1]);
  if (T > 0) {
    StageScope sc(MXMOE_STAGE_FC1_DGRAD, st);
    s = grouped_gemm_impl(&dgu_row, &w1c, seg_off, E, H, 2 * (int64_t)F, ws + W.dx_perm, MXMOE_DTYPE_BF16, H, 0,
                          stream, dgu_used, w1_amax);
    if (s != MXMOE_OK) return s;
  }
  // 6. fc1 wgrad: dW1[e] = dGU_e^T . Xp_e
  mxmoe_mxfp8 dgu_col = mk(ws, W.dgu_colT, W.dgu_colT_sf, 2 * (int64_t)F, cap, grad_format);
  mxmoe_mxfp8 x_col = mk(sv, SL.off[MXMOE_SAVED_X_COLT], SL.off[MXMOE_SAVED_X_COLT_SF], H, cap);
  {
    StageScope sc(MXMOE_STAGE_FC1_WGRAD, st);
    s = grouped_wgrad_impl(&dgu_col, &x_col, seg_off, E, dW1_dev, stream, dgu_used, x_amax);
  }
  if (s != MXMOE_OK) return s;
  // 7. combine dX
  StageScope sc(MXMOE_STAGE_COMBINE_DX, st);
  return moe_unpermute(ws + W.dx_perm, ros, T, k, H, dx_dev, stream);
}

mxmoe_status mxmoe_profile_enable(int32_t max_stages) {
  if (max_stages <= 0 || g_prof.on) return MXMOE_ERR_INVALID_ARG;
  g_prof.ev = new cudaEvent_t[2 * (size_t)max_stages];
  g_prof.tags = new int32_t[max_stages];
  for (int i = 0; i < 2 * max_stages; ++i)
    if (cudaEventCreate(&g_prof.ev[i]) != cudaSuccess) return MXMOE_ERR_CUDA;
  g_prof.cap = max_stages;
  g_prof.n = 0;
  g_prof.depth = 0;
  g_prof.on = true;
  return MXMOE_OK;
}

mxmoe_status mxmoe_profile_disable(void) {
  if (!g_prof.ev) return MXMOE_OK;
  for (int i = 0; i < 2 * g_prof.cap; ++i) cudaEventDestroy(g_prof.ev[i]);
  delete[] g_prof.ev;
  delete[] g_prof.tags;
  g_prof = Profiler();
  return MXMOE_OK;
}

int32_t mxmoe_profile_read(int32_t* tags_host, float* ms_host, int32_t cap) {
  if (!g_prof.on) return 0;
  const int n = g_prof.n;
  for (int i = 0; i < n && i < cap; ++i) {
    cudaEventSynchronize(g_prof.ev[2 * i + 1]);
    float ms = 0.f;
    cudaEventElapsedTime(&ms, g_prof.ev[2 * i], g_prof.ev[2 * i + 1]);
    if (tags_host) tags_host[i] = g_prof.tags[i];
    if (ms_host) ms_host[i] = ms;
  }
  g_prof.n = 0;
  return n;
}

int64_t mxmoe_launch_count(void) { return g_launch_count.load(); }

}  // extern "C"
