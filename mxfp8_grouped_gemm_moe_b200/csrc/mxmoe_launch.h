// Internal host-side launch interface between the C ABI (api.cu) and the kernels.
#pragma once
#include <cuda_runtime.h>

#include <atomic>
#include <cstddef>
#include <cstdint>

#include "../../include/mxmoe.h"

namespace mxmoe {

// Kernels launched by this library since load (reported by mxmoe_launch_count).
inline std::atomic<int64_t> g_launch_count{0};

// Rows of the permuted buffers (live + pad) for T tokens, top-k, E experts:
// roundup(T*k + 255*E, 256) -- every expert segment starts on a 256-row boundary.
inline int64_t rows_cap(int64_t T, int64_t k, int64_t E) { return (T * k + 255 * E + 255) / 256 * 256; }

// ---------------------------------------------------------------- routing / combine
size_t route_workspace_bytes(int T, int k, int E);
cudaError_t launch_route(const int32_t* idx, const float* probs, int T, int k, int E, int32_t* m_splits,
                         int32_t* seg_off, int32_t* row_of_slot, int32_t* token_of_row, float* prob_of_row,
                         void* ws, cudaStream_t st);
cudaError_t launch_unpermute(const void* yp, const int32_t* ros, int T, int k, int H, void* y, cudaStream_t st);
cudaError_t launch_dprob_reduce(const float* part, int nparts, const int32_t* ros, int64_t n, float* dprobs,
                                cudaStream_t st);

// ---------------------------------------------------------------- router
cudaError_t launch_router_topk(const float* logits, int T, int E, int k, int32_t* idx, float* probs,
                               cudaStream_t st);
cudaError_t launch_router_topk_bwd(const float* logits, const int32_t* idx, const float* dprobs, int T, int E, int k,
                                   float* dlogits, cudaStream_t st);

// ---------------------------------------------------------------- quantisation
struct QuantArgs {
  const void* src;
  int32_t src_dtype;
  int64_t batch, rows, cols;
  const int32_t* gather;  // nullable
  const int32_t* nrows;   // nullable (device)
  int64_t out_rows;
  uint8_t* row_data;  // nullable
  uint8_t* row_sf;
  int32_t row_layout;
  uint8_t* col_data;  // nullable
  uint8_t* col_sf;
  int32_t col_layout;
  // > 0: the rowwise copy of each [2*row_ilv, cols] batch matrix stores its rows in
  // 64-row blocks interleaved [first half 0..63, second half 0..63, first 64..127, ...]
  int64_t row_ilv;
  int32_t fmt;         // element format of both outputs: MXMOE_FMT_E4M3 or MXMOE_FMT_E5M2
  int32_t scale_rule;  // MXMOE_SCALE_RULE_OCP or MXMOE_SCALE_RULE_CEIL
  // per-tensor FP8 (E4M3 only): when set, every element is encoded under the multiplier
  // m = 448 / amax of its tensor (tensor_amax[batch index] when tensor_per_batch, else
  // tensor_amax[0]) and every scale byte is 127 (2^0); null: MXFP8 block scales
  const float* tensor_amax;
  int32_t tensor_per_batch;
};
cudaError_t launch_quantize(const QuantArgs& a, cudaStream_t st);
// Largest magnitude of each of `groups` consecutive bf16 arrays of n elements
// (n % 8 == 0, 16-byte aligned) into out[groups] (fp32; cleared first).
// Rowwise MXFP8 with plain scales [rows, cols/32] -> bf16 [rows, cols] (cols % 32 == 0).
cudaError_t launch_dequantize_rows(const uint8_t* codes, const uint8_t* scales, int64_t rows, int64_t cols, int fmt,
                                   void* out, cudaStream_t st);
cudaError_t launch_amax_bf16(const void* src, int64_t n, int32_t groups, float* out, cudaStream_t st);
// bf16 -> bf16 copies with the same row gather / valid-row count / gate-up interleave as
// launch_quantize: row_data receives the (permuted) rows, col_data the transposed matrix
// [batch*cols, out_rows]; the scale fields are ignored. bf16 sources only.
cudaError_t launch_bf16_copy(const QuantArgs& a, cudaStream_t st);

// ---------------------------------------------------------------- grouped GEMM
enum GemmMode : int32_t {
  kModeStore = 0,       // C = A . B_e^T, bf16 or fp32 out (M grouped by expert segments)
  kModeSwigluFwd = 1,   // fc1 + SwiGLU x prob -> MXFP8 Z (row + colT) and / or G, U bf16 (each optional)
  kModeSwigluBwd = 2,   // fc2 dgrad + SwiGLU/prob backward -> MXFP8 dGU (row + colT), dprob partials
  kModeWgrad = 3,       // C[e] = At_e . Bt_e^T, fp32, contraction over the expert's rows
};

struct GemmArgs {
  int32_t mode;
  int32_t E;
  int32_t bf16_operands;  // 0: MXFP8 E4M3 operands with E8M0 scales; 1: bf16 operands, no scales
  // operands (MMA scale layout); a_cols / b_cols count elements
  const uint8_t* a_data;
  const uint8_t* a_sf;
  int64_t a_rows, a_cols;
  const uint8_t* b_data;
  const uint8_t* b_sf;
  int64_t b_rows, b_cols;
  int32_t a_fmt, b_fmt;    // element formats of the MXFP8 operands (MXMOE_FMT_*)
  const int32_t* seg_off;  // device [E+1]
  int64_t N;               // per-expert B rows (store/bwd), F (fwd), output rows per expert (wgrad)
  int64_t K;               // contraction length (not used by wgrad)
  // plain output
  void* c;
  int32_t c_dtype;
  int64_t ldc;
  int64_t K2;  // wgrad: output columns per expert
  // SwiGLU forward epilogue
  const float* prob_of_row;
  int64_t F;
  int64_t rows_cap;
  uint8_t* z_row;
  uint8_t* z_row_sf;
  uint8_t* z_colT;
  uint8_t* z_colT_sf;
  uint16_t* gu;  // bf16 [rows_cap, 2F]
  // SwiGLU backward epilogue
  const uint16_t* gu_in;
  uint8_t* dgu_row;
  uint8_t* dgu_row_sf;
  uint8_t* dgu_colT;
  uint8_t* dgu_colT_sf;
  float* dprob_part;  // [rows_cap, F/128]
  int32_t out_fmt;    // element format of the fused epilogues' MXFP8 outputs (Z / dGU)
  int32_t scale_rule; // scale rule of the fused epilogues' quantisers (MXMOE_SCALE_RULE_*)
  // per-tensor FP8 (null for MXFP8): the operands' largest magnitudes (fp32); b_amax holds
  // one value per expert when b_amax_per_expert. Every output is scaled by
  // 1 / (m(a_amax) * m(b_amax)), m(amax) = 448 / amax (the operands' scale bytes are 127).
  const float* a_amax;
  const float* b_amax;
  int32_t b_amax_per_expert;
  // per-tensor FP8 outputs of the fused epilogues (Z, dGU): encoded under m(*out_amax_in);
  // the largest |output| over the launch is recorded into *out_amax_rec (atomic max)
  const float* out_amax_in;
  float* out_amax_rec;
  // debug: if non-zero, the MMA warp withholds its first accumulator-ready signal so
  // that the epilogue's bounded wait expires (tests the timeout path; never set in
  // normal use)
  int32_t debug_drop_commit;
  // checked build only: if non-zero, the bounds checks of the dprob partials use half the
  // real extent, so that valid writes are flagged and skipped (tests the check path)
  int32_t debug_check_shrink;
};
cudaError_t launch_gemm(const GemmArgs& g, cudaStream_t st);
int gemm_num_sms();

}  // namespace mxmoe
