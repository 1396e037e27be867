// The bf16 grouped expert MLP: the same steps, scheduler and fused epilogues as the MXFP8
// layer in api.cu, on bf16 operands (no quantisation) -- the 16-bit comparison point the
// pages set MXFP8 against ("MoE-Training für biologische Grundmodelle optimieren", MXFP8
// passage: 8 instead of 16 bits per value). The operands that the MXFP8 path quantises
// rowwise / colwise are here bf16 row copies and transposed copies.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>

#include "mxmoe_launch.h"

namespace mxmoe {
namespace bf16path {

struct WeightsLayout {
  size_t w1r, w1t, w2r, w2t, total;  // W1 rows (gate/up interleaved), W1^T, W2 rows, W2^T
};
WeightsLayout weights_layout(int64_t E, int64_t H, int64_t F) {
  WeightsLayout L;
  Carver cv;
  L.w1r = cv.take(E * 2 * F * H * 2);
  L.w1t = cv.take(E * H * 2 * F * 2);
  L.w2r = cv.take(E * H * F * 2);
  L.w2t = cv.take(E * F * H * 2);
  L.total = cv.off;
  return L;
}

struct SavedLayout {
  size_t m_splits, seg_off, ros, tor, por, x_colT, z_colT, gu, total;
};
SavedLayout saved_layout(int64_t T, int64_t k, int64_t E, int64_t H, int64_t F) {
  const int64_t cap = rows_cap(T, k, E);
  SavedLayout L;
  Carver cv;
  L.m_splits = cv.take(E * 4);
  L.seg_off = cv.take((E + 1) * 4);
  L.ros = cv.take(std::max<int64_t>(T * k, 1) * 4);
  L.tor = cv.take(cap * 4);
  L.por = cv.take(cap * 4);
  L.x_colT = cv.take(H * cap * 2);
  L.z_colT = cv.take(F * cap * 2);
  L.gu = cv.take(cap * 2 * F * 2);
  L.total = cv.off;
  return L;
}

struct FwdWs {
  size_t route, x_row, z_row, y_perm, total;
};
FwdWs fwd_ws(int64_t T, int64_t k, int64_t E, int64_t H, int64_t F) {
  const int64_t cap = rows_cap(T, k, E);
  FwdWs w;
  Carver cv;
  w.route = cv.take(route_workspace_bytes((int)T, (int)k, (int)E));
  w.x_row = cv.take(cap * H * 2);
  w.z_row = cv.take(cap * F * 2);
  w.y_perm = cv.take(cap * H * 2);
  w.total = cv.off;
  return w;
}

struct BwdWs {
  size_t dy_row, dy_colT, dgu_row, dgu_colT, dprob_part, dx_perm, total;
};
BwdWs bwd_ws(int64_t T, int64_t k, int64_t E, int64_t H, int64_t F) {
  const int64_t cap = rows_cap(T, k, E);
  BwdWs w;
  Carver cv;
  w.dy_row = cv.take(cap * H * 2);
  w.dy_colT = cv.take(H * cap * 2);
  w.dgu_row = cv.take(cap * 2 * F * 2);
  w.dgu_colT = cv.take(2 * F * cap * 2);
  w.dprob_part = cv.take(cap * (F / 128) * 4);
  w.dx_perm = cv.take(cap * H * 2);
  w.total = cv.off;
  return w;
}

// bf16 row copy (optionally gathered / interleaved) and transposed copy of a bf16 source.
cudaError_t copy(const void* src, int64_t batch, int64_t rows, int64_t cols, const int32_t* gather,
                 const int32_t* nrows, int64_t out_rows, void* row_out, void* col_out, int64_t row_ilv,
                 cudaStream_t st) {
  QuantArgs a;
  std::memset(&a, 0, sizeof(a));
  a.src = src;
  a.src_dtype = MXMOE_DTYPE_BF16;
  a.batch = batch;
  a.rows = rows;
  a.cols = cols;
  a.gather = gather;
  a.nrows = nrows;
  a.out_rows = out_rows;
  a.row_data = static_cast<uint8_t*>(row_out);
  a.col_data = static_cast<uint8_t*>(col_out);
  a.row_ilv = row_ilv;
  return launch_bf16_copy(a, st);
}

GemmArgs gemm(int mode, const void* a, int64_t a_rows, int64_t a_cols, const void* b, int64_t b_rows, int64_t b_cols,
              const int32_t* seg_off, int32_t E) {
  GemmArgs g;
  std::memset(&g, 0, sizeof(g));
  g.mode = mode;
  g.bf16_operands = 1;
  g.E = E;
  g.a_data = static_cast<const uint8_t*>(a);
  g.a_rows = a_rows;
  g.a_cols = a_cols;
  g.b_data = static_cast<const uint8_t*>(b);
  g.b_rows = b_rows;
  g.b_cols = b_cols;
  g.seg_off = seg_off;
  return g;
}

}  // namespace bf16path
}  // namespace mxmoe

using namespace mxmoe;

extern "C" {

size_t mxmoe_weights_bf16_size(int32_t E, int32_t H, int32_t F) { return bf16path::weights_layout(E, H, F).total; }

mxmoe_status mxmoe_weights_bf16_prepare(const void* W1_dev, const void* W2_dev, int32_t E, int32_t H, int32_t F,
                                        void* wb_dev, size_t wb_bytes, void* stream) {
  if (E < 1 || E > 256 || H <= 0 || F <= 0 || H % 256 != 0 || F % 256 != 0) return MXMOE_ERR_UNSUPPORTED_SHAPE;
  if (!W1_dev || !W2_dev || !wb_dev || !aligned16(W1_dev) || !aligned16(W2_dev) || !aligned16(wb_dev))
    return MXMOE_ERR_INVALID_ARG;
  const bf16path::WeightsLayout L = bf16path::weights_layout(E, H, F);
  if (wb_bytes < L.total) return MXMOE_ERR_WORKSPACE_TOO_SMALL;
  uint8_t* wb = static_cast<uint8_t*>(wb_dev);
  cudaStream_t st = S(stream);
  {
    StageScope sc(MXMOE_STAGE_QUANT_W1, st);
    if (bf16path::copy(W1_dev, E, 2 * (int64_t)F, H, nullptr, nullptr, 2 * (int64_t)F, wb + L.w1r, wb + L.w1t, F,
                       st) != cudaSuccess)
      return MXMOE_ERR_CUDA;
  }
  StageScope sc(MXMOE_STAGE_QUANT_W2, st);
  return cuda_status(bf16path::copy(W2_dev, E, H, F, nullptr, nullptr, H, wb + L.w2r, wb + L.w2t, 0, st));
}

size_t grouped_mlp_bf16_saved_size(int32_t T, int32_t k, int32_t E, int32_t H, int32_t F) {
  if (!valid_mlp_shape(T, k, E, H, F)) return 0;
  return bf16path::saved_layout(T, k, E, H, F).total;
}

size_t grouped_mlp_bf16_workspace_size(int32_t T, int32_t k, int32_t E, int32_t H, int32_t F) {
  if (!valid_mlp_shape(T, k, E, H, F)) return 0;
  return std::max(bf16path::fwd_ws(T, k, E, H, F).total, bf16path::bwd_ws(T, k, E, H, F).total);
}

mxmoe_status grouped_mlp_bf16_fwd(const void* x_dev, const int32_t* topk_idx_dev, const float* probs_dev,
                                  const void* wb_dev, size_t wb_bytes, int32_t T, int32_t k, int32_t E, int32_t H,
                                  int32_t F, void* y_dev, void* saved_dev, size_t saved_bytes, void* ws_dev,
                                  size_t ws_bytes, void* stream) {
  if (!valid_mlp_shape(T, k, E, H, F)) return MXMOE_ERR_UNSUPPORTED_SHAPE;
  if (!wb_dev || !saved_dev || !ws_dev || !aligned16(wb_dev) || !aligned16(saved_dev) || !aligned16(ws_dev))
    return MXMOE_ERR_INVALID_ARG;
  if (T > 0 && (!x_dev || !topk_idx_dev || !probs_dev || !y_dev || !aligned16(x_dev) || !aligned16(y_dev)))
    return MXMOE_ERR_INVALID_ARG;
  if (wb_bytes < mxmoe_weights_bf16_size(E, H, F) || saved_bytes < grouped_mlp_bf16_saved_size(T, k, E, H, F) ||
      ws_bytes < grouped_mlp_bf16_workspace_size(T, k, E, H, F))
    return MXMOE_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = S(stream);
  const int64_t cap = rows_cap(T, k, E);
  const bf16path::SavedLayout SL = bf16path::saved_layout(T, k, E, H, F);
  const bf16path::FwdWs W = bf16path::fwd_ws(T, k, E, H, F);
  const bf16path::WeightsLayout WL = bf16path::weights_layout(E, H, F);
  uint8_t* sv = static_cast<uint8_t*>(saved_dev);
  uint8_t* ws = static_cast<uint8_t*>(ws_dev);
  const uint8_t* wb = static_cast<const uint8_t*>(wb_dev);
  int32_t* seg_off = reinterpret_cast<int32_t*>(sv + SL.seg_off);
  int32_t* ros = reinterpret_cast<int32_t*>(sv + SL.ros);
  int32_t* tor = reinterpret_cast<int32_t*>(sv + SL.tor);
  float* por = reinterpret_cast<float*>(sv + SL.por);
  cudaError_t e;
  {
    StageScope sc(MXMOE_STAGE_ROUTE, st);
    e = launch_route(topk_idx_dev, probs_dev, T, k, E, reinterpret_cast<int32_t*>(sv + SL.m_splits), seg_off, ros, tor,
                     por, ws + W.route, st);
  }
  if (e != cudaSuccess) return MXMOE_ERR_CUDA;
  if (T == 0) return MXMOE_OK;
  {  // permuted x rows (fc1 operand) and their transpose (saved: fc1 weight-gradient operand)
    StageScope sc(MXMOE_STAGE_QUANT_X, st);
    e = bf16path::copy(x_dev, 1, T, H, tor, seg_off + E, cap, ws + W.x_row, sv + SL.x_colT, 0, st);
  }
  if (e != cudaSuccess) return MXMOE_ERR_CUDA;
  {  // fc1 + SwiGLU x prob -> Z bf16 rows + transposed (saved), G/U saved
    GemmArgs g = bf16path::gemm(kModeSwigluFwd, ws + W.x_row, cap, H, wb + WL.w1r, (int64_t)E * 2 * F, H, seg_off, E);
    g.K = H;
    g.F = F;
    g.N = 2 * (int64_t)F;
    g.rows_cap = cap;
    g.prob_of_row = por;
    g.z_row = ws + W.z_row;
    g.z_colT = sv + SL.z_colT;
    g.gu = reinterpret_cast<uint16_t*>(sv + SL.gu);
    StageScope sc(MXMOE_STAGE_FC1_SWIGLU, st);
    e = launch_gemm(g, st);
  }
  if (e != cudaSuccess) return MXMOE_ERR_CUDA;
  mxmoe_status s;
  {
    StageScope sc(MXMOE_STAGE_FC2, st);
    s = grouped_gemm_bf16(ws + W.z_row, cap, wb + WL.w2r, seg_off, E, H, F, ws + W.y_perm, MXMOE_DTYPE_BF16, H,
                          stream);
  }
  if (s != MXMOE_OK) return s;
  StageScope sc(MXMOE_STAGE_COMBINE, st);
  return moe_unpermute(ws + W.y_perm, ros, T, k, H, y_dev, stream);
}

mxmoe_status grouped_mlp_bf16_bwd(const void* dy_dev, const void* saved_dev, size_t saved_bytes, const void* wb_dev,
                                  size_t wb_bytes, int32_t T, int32_t k, int32_t E, int32_t H, int32_t F,
                                  void* dx_dev, float* dW1_dev, float* dW2_dev, float* dprobs_dev, void* ws_dev,
                                  size_t ws_bytes, void* stream) {
  if (!valid_mlp_shape(T, k, E, H, F)) return MXMOE_ERR_UNSUPPORTED_SHAPE;
  if (!wb_dev || !saved_dev || !ws_dev || !dW1_dev || !dW2_dev || !aligned16(wb_dev) || !aligned16(saved_dev) ||
      !aligned16(ws_dev) || !aligned16(dW1_dev) || !aligned16(dW2_dev))
    return MXMOE_ERR_INVALID_ARG;
  if (T > 0 && (!dy_dev || !dx_dev || !dprobs_dev || !aligned16(dy_dev) || !aligned16(dx_dev)))
    return MXMOE_ERR_INVALID_ARG;
  if (wb_bytes < mxmoe_weights_bf16_size(E, H, F) || saved_bytes < grouped_mlp_bf16_saved_size(T, k, E, H, F) ||
      ws_bytes < grouped_mlp_bf16_workspace_size(T, k, E, H, F))
    return MXMOE_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = S(stream);
  const int64_t cap = rows_cap(T, k, E);
  const bf16path::SavedLayout SL = bf16path::saved_layout(T, k, E, H, F);
  const bf16path::BwdWs W = bf16path::bwd_ws(T, k, E, H, F);
  const bf16path::WeightsLayout WL = bf16path::weights_layout(E, H, F);
  const uint8_t* sv = static_cast<const uint8_t*>(saved_dev);
  uint8_t* ws = static_cast<uint8_t*>(ws_dev);
  const uint8_t* wb = static_cast<const uint8_t*>(wb_dev);
  const int32_t* seg_off = reinterpret_cast<const int32_t*>(sv + SL.seg_off);
  const int32_t* ros = reinterpret_cast<const int32_t*>(sv + SL.ros);
  const int32_t* tor = reinterpret_cast<const int32_t*>(sv + SL.tor);
  const float* por = reinterpret_cast<const float*>(sv + SL.por);
  cudaError_t e = cudaSuccess;
  if (T > 0) {  // permuted dY rows (fc2 dgrad operand) and transpose (fc2 wgrad operand)
    StageScope sc(MXMOE_STAGE_QUANT_DY, st);
    e = bf16path::copy(dy_dev, 1, T, H, tor, seg_off + E, cap, ws + W.dy_row, ws + W.dy_colT, 0, st);
  }
  if (e != cudaSuccess) return MXMOE_ERR_CUDA;
  {  // fc2 dgrad + SwiGLU / prob backward -> dGU bf16 rows + transposed, dprob partials
    GemmArgs g = bf16path::gemm(kModeSwigluBwd, ws + W.dy_row, cap, H, wb + WL.w2t, (int64_t)E * F, H, seg_off, E);
    g.K = H;
    g.N = F;
    g.F = F;
    g.rows_cap = cap;
    g.prob_of_row = por;
    g.gu_in = reinterpret_cast<const uint16_t*>(sv + SL.gu);
    g.dgu_row = ws + W.dgu_row;
    g.dgu_colT = ws + W.dgu_colT;
    g.dprob_part = reinterpret_cast<float*>(ws + W.dprob_part);
    StageScope sc(MXMOE_STAGE_FC2_DGRAD, st);
    if (T > 0 && launch_gemm(g, st) != cudaSuccess) return MXMOE_ERR_CUDA;
  }
  {
    StageScope sc(MXMOE_STAGE_DPROB, st);
    if (launch_dprob_reduce(reinterpret_cast<const float*>(ws + W.dprob_part), F / 128, ros, (int64_t)T * k,
                            dprobs_dev, st) != cudaSuccess)
      return MXMOE_ERR_CUDA;
  }
  mxmoe_status s;
  {
    StageScope sc(MXMOE_STAGE_FC2_WGRAD, st);
    s = grouped_gemm_bf16_wgrad(ws + W.dy_colT, sv + SL.z_colT, H, F, cap, seg_off, E, dW2_dev, stream);
  }
  if (s != MXMOE_OK) return s;
  if (T > 0) {
    StageScope sc(MXMOE_STAGE_FC1_DGRAD, st);
    s = grouped_gemm_bf16(ws + W.dgu_row, cap, wb + WL.w1t, seg_off, E, H, 2 * (int64_t)F, ws + W.dx_perm,
                          MXMOE_DTYPE_BF16, H, stream);
    if (s != MXMOE_OK) return s;
  }
  {
    StageScope sc(MXMOE_STAGE_FC1_WGRAD, st);
    s = grouped_gemm_bf16_wgrad(ws + W.dgu_colT, sv + SL.x_colT, 2 * (int64_t)F, H, cap, seg_off, E, dW1_dev, stream);
  }
  if (s != MXMOE_OK) return s;
  StageScope sc(MXMOE_STAGE_COMBINE_DX, st);
  return moe_unpermute(ws + W.dx_perm, ros, T, k, H, dx_dev, stream);
}

}  // extern "C"
