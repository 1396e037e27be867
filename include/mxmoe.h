/*
 * mxmoe.h -- C ABI of the B200 (sm_100a) MXFP8 grouped expert-MLP library.
 *
 * What the library computes (sources: three short web pages on one NVIDIA tutorial;
 * they give no formulas, so the exact conventions below are this library's stated
 * readings):
 *   - "MoE-Training für biologische Grundmodelle optimieren" (hyper.ai/de): grouping
 *     of tokens by per-expert token counts so that all expert GEMMs run in one call
 *     (GroupedLinear passage); MXFP8 with one scale factor per block of 32 values
 *     (MXFP8 passage); a fused gate-up / ScaledSwiGLU / routing-scale kernel with a
 *     matching backward (GroupedMLP passage);
 *   - "NVIDIA apresenta técnicas para tornar mais eficiente o treinamento de modelos
 *     biológicos baseados em arquitetura MoE" (conexaotc.com.br): the fused kernel
 *     covers quantisation, SwiGLU and routing-weight scaling (third optimisation);
 *   - "NVIDIA optimise l'entraînement MoE des modèles biologiques" (hyper.ai/fr):
 *     expert GEMMs in one GPU call; MXFP8 halves the footprint; SwiGLU and
 *     quantisation fused, forward and backward.
 *
 * Conventions (all entry points):
 *   - Every pointer argument named *_dev or documented "device" is CUDA device memory
 *     owned by the caller; the library never allocates, frees or synchronises, and
 *     enqueues all work asynchronously on `stream` (a cudaStream_t; NULL = legacy
 *     default stream).
 *   - Device pointers must be 16-byte aligned; byte sizes documented per argument.
 *   - Host-detectable errors (bad pointer, shape, size) return a non-zero status and
 *     enqueue nothing. Errors found on the device (an expert id out of range or
 *     repeated within a token, a wait that timed out) are recorded in a per-device
 *     status word read with mxmoe_get_device_status(); kernels never trap.
 *   - bf16 is IEEE bfloat16 stored as uint16; E4M3 is OCP FP8 E4M3 (bias 7, max 448,
 *     no infinities); E8M0 is an unsigned power-of-two exponent byte (bias 127).
 *   - MXFP8 rule (OCP Microscaling v1.0): for a block of 32 values with largest
 *     magnitude amax, X = clamp(floor(log2(amax)) - 8, -127, 127) (amax == 0 gives
 *     -127), scale byte = X + 127, element = E4M3(v * 2^-X) rounded to nearest-even
 *     and saturated to +-448.
 *   - Routed rows are ordered by (expert ascending, token ascending). Expert e's
 *     segment of rows starts at seg_off[e], a multiple of 256; its first m_splits[e]
 *     rows are live, the rest up to seg_off[e+1] are zero pad rows. The buffers of
 *     permuted rows hold mxmoe_rows_capacity(T, k, E) rows.
 */
#ifndef MXMOE_H_
#define MXMOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t mxmoe_status;

#define MXMOE_OK 0
#define MXMOE_ERR_INVALID_ARG 1          /* null / misaligned pointer, bad enum, negative size */
#define MXMOE_ERR_UNSUPPORTED_SHAPE 2    /* shape outside what the kernels handle */
#define MXMOE_ERR_WORKSPACE_TOO_SMALL 3  /* ws_bytes / saved_bytes / wq_bytes below the query */
#define MXMOE_ERR_CUDA 4                 /* a CUDA runtime call failed (launch, attribute) */
#define MXMOE_ERR_DEVICE_TIMEOUT 5       /* device: a bounded wait gave up */
#define MXMOE_ERR_DEVICE_CHECK 6         /* device: invalid routing input */

/* dtypes */
#define MXMOE_DTYPE_BF16 0
#define MXMOE_DTYPE_F32 1

/* scale rules of a quantisation (mxfp8_quantize_ex, mxmoe_weights_quantize_ex) */
#define MXMOE_SCALE_RULE_OCP 0  /* X = clamp(floor(log2(amax)) - emax, -127, 127); elements saturate */
#define MXMOE_SCALE_RULE_CEIL 1 /* smallest X with amax <= max * 2^X (the OCP X, or one more): nothing
                                   saturates (a variant; the pages give no rule) */

/* element formats of an mxmoe_mxfp8 matrix */
#define MXMOE_FMT_E4M3 0 /* OCP FP8 E4M3: bias 7, max 448 (activations, weights; gradients by default) */
#define MXMOE_FMT_E5M2 1 /* OCP FP8 E5M2: bias 15, max 57344, saturating (the gradient variant) */

/* scale-factor layouts of an mxmoe_mxfp8 matrix */
#define MXMOE_SCALE_PLAIN 0 /* row-major [rows][cols/32] */
#define MXMOE_SCALE_MMA 1   /* rows, cols multiples of 128: [rows/128][cols/128] chunks of 512 bytes;
                               inside a chunk the scale of (row r, block kb) is at byte
                               (r%32)*16 + ((r/32)%4)*4 + kb%4 -- the tensor cores' scale-factor order */

/*
 * One MXFP8 matrix: `rows` x `cols` FP8 codes of `elem_format`, row-major (row stride
 * `cols` bytes), quantised in blocks of 32 consecutive elements along each row, plus
 * rows*cols/32 E8M0 scale bytes laid out as `scale_layout` says. A "colwise"
 * quantisation of a source matrix S [R, C] (blocks of 32 consecutive rows of S) is
 * stored transposed: rows = C, cols = R. Both pointers are device memory owned by the
 * caller. The scale rule of an E5M2 matrix is the MXFP8 rule below with 15 (the largest
 * exponent of E5M2) in place of 8.
 */
typedef struct mxmoe_mxfp8 {
  uint8_t* data;
  uint8_t* scale;
  int64_t rows;
  int64_t cols;
  int32_t scale_layout;
  int32_t elem_format; /* MXMOE_FMT_E4M3 (0) or MXMOE_FMT_E5M2 */
} mxmoe_mxfp8;

/* ------------------------------------------------------------------ status / sizes */

/* Human-readable name of a status code (static string; never NULL). */
const char* mxmoe_status_string(mxmoe_status s);

/* Copies the current device's status word (MXMOE_OK or the first device error since
 * the last clear) to *out_host and the tag of the site that set it to *where_host
 * (nullable). Synchronises `stream`. */
mxmoe_status mxmoe_get_device_status(int32_t* out_host, int32_t* where_host, void* stream);

/* Resets the current device's status word to MXMOE_OK (enqueued on `stream`). */
mxmoe_status mxmoe_clear_device_status(void* stream);

/* Upper bound on the number of permuted rows (live + pad) for T tokens, top-k and E
 * experts: roundup(T*k + 255*E, 256). Every [Mp, *] buffer below has this many rows. */
int64_t mxmoe_rows_capacity(int32_t T, int32_t k, int32_t E);

/* ------------------------------------------------------------------ router (upstream of the path) */

/*
 * moe_router_topk -- the router step ahead of the expert MLP ("MoE-Training für
 * biologische Grundmodelle optimieren", routing passage: a router assigns every token to
 * its experts). The pages give no formula; readings: probabilities are a softmax over all
 * E experts (not renormalised over the k selected), the k largest are selected in
 * descending order, equal logits keep the lower expert index first, and a logit of -inf
 * marks an expert the token may not use (probability 0; selected last).
 *   logits_dev    float [T, E]  row-major, finite or -inf, at least one finite per row.
 *   topk_idx_dev  int32 [T, k]  out: selected experts, descending probability.
 *   probs_dev     float [T, k]  out: their softmax probabilities (fp32).
 * A row with NaN or no finite logit sets MXMOE_ERR_DEVICE_CHECK and gets ids -1 and
 * probabilities 0 (moe_permute then rejects those pairs).
 * Limits: 1 <= E <= 256, 1 <= k <= min(E, 8), T >= 0.
 */
mxmoe_status moe_router_topk(const float* logits_dev, int32_t T, int32_t E, int32_t k, int32_t* topk_idx_dev,
                             float* probs_dev, void* stream);

/*
 * moe_router_topk_bwd -- gradient of a loss that depends on the selected probabilities:
 *   dlogits[t, e] = P[t, e] * (g[t, e] - sum_j dprobs[t, j] * P[t, idx[t, j]]),
 * P the softmax of the row, g[t, e] = dprobs[t, j] for e = idx[t, j] (0 otherwise).
 * The softmax is recomputed from the logits (nothing is saved by the forward).
 *   logits_dev [T, E], topk_idx_dev [T, k] (as returned by moe_router_topk),
 *   dprobs_dev float [T, k], dlogits_dev float [T, E] (out).
 * Same limits and device checks as the forward.
 */
mxmoe_status moe_router_topk_bwd(const float* logits_dev, const int32_t* topk_idx_dev, const float* dprobs_dev,
                                 int32_t T, int32_t E, int32_t k, float* dlogits_dev, void* stream);

/* ------------------------------------------------------------------ routing (GroupedLinear input) */

/*
 * moe_permute -- groups the routed (token, slot) pairs by expert: a counting sort,
 * stable by token ("MoE-Training für biologische Grundmodelle optimieren", GroupedLinear
 * passage: the per-expert token counts drive the gather of the expert matrices).
 *   topk_idx_dev  int32 [T, k]  expert id of each token's k choices; distinct within a
 *                 token and in [0, E). Violations set MXMOE_ERR_DEVICE_CHECK and the
 *                 offending pair is dropped.
 *   probs_dev     float [T, k]  routing probabilities (nullable if prob_of_row_dev is).
 *   Outputs (device, caller-owned):
 *   m_splits_dev     int32 [E]     tokens per expert
 *   seg_off_dev      int32 [E+1]   start row of each expert segment (multiples of 256);
 *                                  seg_off[E] = Mp, the padded row count
 *   row_of_slot_dev  int32 [T, k]  permuted row of each (token, slot)
 *   token_of_row_dev int32 [mxmoe_rows_capacity]  token of each row, -1 on pad rows
 *                                  (rows >= Mp are left untouched)
 *   prob_of_row_dev  float [mxmoe_rows_capacity]  probability of each row, 0 on pad rows
 *                                  (nullable)
 *   ws_dev / ws_bytes  scratch of at least moe_permute_workspace_size(T, k, E) bytes.
 * Limits: 1 <= k <= 8, 1 <= E <= 256, T >= 0.
 */
mxmoe_status moe_permute(const int32_t* topk_idx_dev, const float* probs_dev, int32_t T, int32_t k, int32_t E,
                         int32_t* m_splits_dev, int32_t* seg_off_dev, int32_t* row_of_slot_dev,
                         int32_t* token_of_row_dev, float* prob_of_row_dev, void* ws_dev, size_t ws_bytes,
                         void* stream);
size_t moe_permute_workspace_size(int32_t T, int32_t k, int32_t E);

/*
 * moe_permute_noalloc -- the same routing index as moe_permute, for callers that cannot
 * provide a scratch buffer (no counterpart in the pages: it is a calling convenience).
 * Such callers include serving runtimes that plan all device memory ahead of time and
 * have no free buffer to lend per call, and plain C callers without a device allocator.
 * It allocates nothing and takes no workspace: its scratch is a fixed 256 KiB array in
 * the library's own device memory, present on every GPU that loads the library until
 * the process exits.
 *   Arguments and outputs: as moe_permute.
 *   Limit: 8 * ceil(T / 256) * E + 256 bytes of scratch must fit in 256 KiB (e.g.
 *   T = 65536 with E = 128, or T = 32768 with E = 256); larger problems return
 *   MXMOE_ERR_WORKSPACE_TOO_SMALL and enqueue nothing.
 *   The first call on a device looks up the array's device address (once per device,
 *   with that device current); make that first call before any stream capture. The
 *   address is kept for the life of the process: calls after cudaDeviceReset (which
 *   reloads the library's device code and may move the array) are not supported.
 *   All calls on a device share the one array: calls that may overlap on the GPU (for
 *   example on two streams without ordering between them) race and must be serialised
 *   by the caller. Nothing in the array needs clearing between calls: every word a call
 *   reads, it has written first.
 */
mxmoe_status moe_permute_noalloc(const int32_t* topk_idx_dev, const float* probs_dev, int32_t T, int32_t k,
                                 int32_t E, int32_t* m_splits_dev, int32_t* seg_off_dev, int32_t* row_of_slot_dev,
                                 int32_t* token_of_row_dev, float* prob_of_row_dev, void* stream);

/*
 * moe_unpermute -- returns routed rows to token order and sums the k copies of each
 * token: y[t] = sum_{j<k} y_perm[row_of_slot[t, j]], accumulated in fp32 in slot order
 * and rounded once to bf16 (the pages are silent on the combine; this is the plain
 * reading). y_perm_dev bf16 [rows, H]; y_dev bf16 [T, H]. H % 8 == 0; both pointers
 * 16-byte aligned (MXMOE_ERR_INVALID_ARG otherwise). When both are 32-byte aligned and
 * H % 16 == 0 the kernel moves 32 bytes per access (same results either way).
 */
mxmoe_status moe_unpermute(const void* y_perm_dev, const int32_t* row_of_slot_dev, int32_t T, int32_t k,
                           int32_t H, void* y_dev, void* stream);

/* ------------------------------------------------------------------ MXFP8 quantisation */

/*
 * mxfp8_quantize -- MXFP8 quantisation, rowwise and/or colwise, optionally fused with a
 * row gather ("MoE-Training für biologische Grundmodelle optimieren", MXFP8 passage:
 * 8-bit values with one scale per 32-value block; GroupedMLP passage: the conversions
 * between 16-bit and 8-bit are fused instead of run as separate operations).
 *   src_dev      [batch, rows, cols] of src_dtype (MXMOE_DTYPE_BF16 or _F32), row-major.
 *   row_gather_dev  nullable int32 [out_rows]: if given (batch must be 1), output row r
 *                is src row row_gather[r], or zeros where row_gather[r] < 0.
 *   nrows_dev    nullable int32 (one value, device): only output rows < *nrows_dev are
 *                written (e.g. &seg_off[E]); must be a multiple of 128 if given.
 *   out_rows     rows of each output matrix (== rows when there is no gather).
 *   out_row      nullable: rowwise result, rows = batch*out_rows, cols = cols.
 *   out_colT     nullable: colwise result (blocks of 32 consecutive output rows within
 *                each batch matrix), stored transposed: rows = batch*cols, cols = out_rows;
 *                batch b's matrix occupies rows [b*cols, (b+1)*cols).
 * Shapes: cols % 32 == 0, out_rows % 32 == 0 (both % 128 == 0 for MXMOE_SCALE_MMA).
 * Element format: each output's elem_format (E4M3 or E5M2); when both outputs are given
 * their formats must agree (else MXMOE_ERR_INVALID_ARG).
 */
mxmoe_status mxfp8_quantize(const void* src_dev, int32_t src_dtype, int64_t batch, int64_t rows, int64_t cols,
                            const int32_t* row_gather_dev, const int32_t* nrows_dev, int64_t out_rows,
                            const mxmoe_mxfp8* out_row, const mxmoe_mxfp8* out_colT, void* stream);
/*
 * mxfp8_dequantize -- the inverse of the rowwise quantisation, for MXFP8 rows that travel
 * between devices ("MoE-Training für biologische Grundmodelle optimieren", expert-parallel
 * passage: the experts spread over GPUs; the routed rows can travel as codes + scales): every
 * element becomes element(code) * 2^(scale - 127), rounded once to bf16 (exact whenever
 * the block's scale is at least 2^-124, i.e. for every block quantised from bf16 values
 * of magnitude above about 2^-115).
 *   src_row  rowwise MXFP8 [rows, cols], MXMOE_SCALE_PLAIN scales; cols % 32 == 0;
 *            either element format.
 *   dst_dev  bf16 [rows, cols], 16-byte aligned.
 * Errors: MXMOE_ERR_INVALID_ARG for a null / unaligned pointer or an MMA scale layout,
 * MXMOE_ERR_UNSUPPORTED_SHAPE for cols % 32 != 0.
 */
mxmoe_status mxfp8_dequantize(const mxmoe_mxfp8* src_row, void* dst_dev, void* stream);

/* mxfp8_quantize with the scale rule chosen (MXMOE_SCALE_RULE_OCP, the rule above, or
 * MXMOE_SCALE_RULE_CEIL: the OCP exponent plus one for the blocks whose amax lies above
 * the format's largest value times the OCP scale, so that no element saturates). Any
 * other rule returns MXMOE_ERR_INVALID_ARG. */
mxmoe_status mxfp8_quantize_ex(const void* src_dev, int32_t src_dtype, int64_t batch, int64_t rows, int64_t cols,
                               const int32_t* row_gather_dev, const int32_t* nrows_dev, int64_t out_rows,
                               const mxmoe_mxfp8* out_row, const mxmoe_mxfp8* out_colT, int32_t scale_rule,
                               void* stream);

/* ------------------------------------------------------------------ grouped GEMMs (GroupedLinear) */

/*
 * grouped_gemm_mxfp8 -- one launch for all experts ("MoE-Training für biologische
 * Grundmodelle optimieren", GroupedLinear passage; "NVIDIA optimise l'entraînement MoE
 * des modèles biologiques", first improvement): for every expert e,
 *     C[seg_e, :] = dequant(A)[seg_e, :] . dequant(B_e)^T,   seg_e = [seg_off[e], seg_off[e+1])
 * with fp32 accumulation on the tensor cores. A and B may each be E4M3 or E5M2 (their
 * elem_format; e.g. an E5M2 gradient times an E4M3 weight).
 *   A   MXFP8 [rows_cap, K], MXMOE_SCALE_MMA; rows_cap % 256 == 0.
 *   B   MXFP8 [E*N, K], MXMOE_SCALE_MMA (expert e's rows are [e*N, (e+1)*N)).
 *   seg_off_dev  int32 [E+1], multiples of 256, read on the device (no host sync).
 *   C_dev [rows_cap, ldc] of c_dtype (MXMOE_DTYPE_BF16 or _F32); rows >= seg_off[E]
 *         are not written.
 * Shapes: N % 256 == 0, K % 128 == 0, ldc >= N, ldc % 8 == 0.
 * Errors: host-checkable argument and shape errors are returned; segment offsets that
 * are not non-decreasing multiples of 256 starting at 0 and ending at most at rows_cap
 * are caught on the device (nothing is computed; mxmoe_get_device_status then reports
 * MXMOE_ERR_DEVICE_CHECK).
 */
mxmoe_status grouped_gemm_mxfp8(const mxmoe_mxfp8* A, const mxmoe_mxfp8* B, const int32_t* seg_off_dev,
                                int32_t E, int64_t N, int64_t K, void* C_dev, int32_t c_dtype, int64_t ldc,
                                void* stream);

/*
 * grouped_gemm_mxfp8_debug_timeout -- test hook for the device-timeout path (failure
 * detection; no counterpart in the pages). The same call as grouped_gemm_mxfp8, except
 * that the first CTA pair's MMA issuer withholds its first accumulator-ready signal: that
 * pair's epilogue warps wait for it until the wait limit (1 s) runs out, record
 * MXMOE_ERR_DEVICE_TIMEOUT in the device status word and stop (the first wait of the pair
 * to run out records its site: normally the epilogue's, possibly the scale-copy thread's,
 * which stalls behind it); the pair's other roles stop at their own limits, wait for
 * their issued copies, scale copies and MMAs, release TMEM and return. The
 * kernel ends (no hang, no trap) with C only partly written; the context stays usable.
 * Arguments, checks and errors as grouped_gemm_mxfp8. Never use it for results.
 */
mxmoe_status grouped_gemm_mxfp8_debug_timeout(const mxmoe_mxfp8* A, const mxmoe_mxfp8* B,
                                              const int32_t* seg_off_dev, int32_t E, int64_t N, int64_t K,
                                              void* C_dev, int32_t c_dtype, int64_t ldc, void* stream);

/*
 * grouped_gemm_mxfp8_wgrad -- weight-gradient form, contracting over each expert's
 * (ragged) rows: C[e] = dequant(At)[:, seg_e] . dequant(Bt)[:, seg_e]^T, fp32, [E, N, K2].
 * An expert with no rows gets zeros.
 *   At  MXFP8 [N, rows_cap] (colwise-transposed activations/gradients), MXMOE_SCALE_MMA.
 *   Bt  MXFP8 [K2, rows_cap], MXMOE_SCALE_MMA.
 *   C_dev float [E, N, K2].
 * Shapes: N % 256 == 0, K2 % 256 == 0, rows_cap % 256 == 0. Segment offsets are
 * checked on the device as for grouped_gemm_mxfp8.
 */
mxmoe_status grouped_gemm_mxfp8_wgrad(const mxmoe_mxfp8* At, const mxmoe_mxfp8* Bt, const int32_t* seg_off_dev,
                                      int32_t E, float* C_dev, void* stream);

/*
 * grouped_gemm_bf16 / grouped_gemm_bf16_wgrad -- the same grouped GEMMs on bf16 operands
 * (no quantisation; the 16-bit comparison point the pages set MXFP8 against: "MoE-Training
 * für biologische Grundmodelle optimieren", MXFP8 passage), on the same persistent
 * scheduler and CTA-pair tiles, fp32 accumulation (tcgen05 kind::f16).
 *   grouped_gemm_bf16: C[seg_e, :] = A[seg_e, :] . B_e^T
 *     A_dev  bf16 [rows_cap, K] row-major; B_dev bf16 [E*N, K]; seg_off_dev as above;
 *     C_dev  [rows_cap, ldc] of c_dtype (MXMOE_DTYPE_BF16 or _F32).
 *     Shapes: rows_cap % 256 == 0, N % 256 == 0, K % 64 == 0, ldc >= N, ldc % 8 == 0.
 *   grouped_gemm_bf16_wgrad: C[e] = At[:, seg_e] . Bt[:, seg_e]^T, fp32 [E, N, K2]
 *     At_dev bf16 [N, rows_cap]; Bt_dev bf16 [K2, rows_cap] (transposed activations /
 *     gradients). Shapes: N % 256 == 0, K2 % 256 == 0, rows_cap % 256 == 0.
 * All pointers 16-byte aligned; segment offsets are checked on the device as above.
 */
mxmoe_status grouped_gemm_bf16(const void* A_dev, int64_t rows_cap, const void* B_dev, const int32_t* seg_off_dev,
                               int32_t E, int64_t N, int64_t K, void* C_dev, int32_t c_dtype, int64_t ldc,
                               void* stream);
mxmoe_status grouped_gemm_bf16_wgrad(const void* At_dev, const void* Bt_dev, int64_t N, int64_t K2, int64_t rows_cap,
                                     const int32_t* seg_off_dev, int32_t E, float* C_dev, void* stream);

/* ------------------------------------------------------------------ fused grouped MLP (GroupedMLP) */

/*
 * Quantised weights: one opaque device buffer of mxmoe_weights_size(E, H, F) bytes that
 * holds four MXFP8 copies (MMA scale layout):
 *   W1 rowwise  [E*2F, H]  (fc1 forward operand; blocks along H)
 *   W1 colwise  [E*H, 2F]  (fc1 data-gradient operand; blocks along 2F)
 *   W2 rowwise  [E*H, F]   (fc2 forward operand; blocks along F)
 *   W2 colwise  [E*F, H]   (fc2 data-gradient operand; blocks along H)
 * The W1 rowwise copy keeps each expert's rows in 64-row blocks interleaved gate / up
 * (gate 0..63, up 0..63, gate 64..127, ...), so that one 128-row operand tile holds
 * matching gate and up columns; the other three copies keep the natural row order.
 * W1_dev bf16 [E, 2F, H] (rows 0..F-1 gate, F..2F-1 up; nn.Linear out x in),
 * W2_dev bf16 [E, H, F]. Requires H % 256 == 0, F % 256 == 0.
 */
size_t mxmoe_weights_size(int32_t E, int32_t H, int32_t F);
mxmoe_status mxmoe_weights_quantize(const void* W1_dev, const void* W2_dev, int32_t E, int32_t H, int32_t F,
                                    void* wq_dev, size_t wq_bytes, void* stream);
/* The same with the scale rule chosen (MXMOE_SCALE_RULE_*); a layer run with
 * MXMOE_RECIPE_SCALE_CEIL takes weights quantised with MXMOE_SCALE_RULE_CEIL. */
mxmoe_status mxmoe_weights_quantize_ex(const void* W1_dev, const void* W2_dev, int32_t E, int32_t H, int32_t F,
                                       int32_t scale_rule, void* wq_dev, size_t wq_bytes, void* stream);
/* View of one of the four copies inside a weights buffer (which: 0 W1 row, 1 W1 col,
 * 2 W2 row, 3 W2 col). Host-only pointer arithmetic. */
mxmoe_status mxmoe_weights_view(void* wq_dev, int32_t E, int32_t H, int32_t F, int32_t which, mxmoe_mxfp8* out);

/*
 * Activations saved by the forward for the backward: one opaque device buffer of
 * grouped_mlp_saved_size(...) bytes (routing maps, colwise MXFP8 copies of the permuted
 * input and of Z, and the gate/up pre-activations in bf16). Named fields can be located
 * with grouped_mlp_saved_offset for inspection.
 */
#define MXMOE_SAVED_M_SPLITS 0     /* int32 [E] */
#define MXMOE_SAVED_SEG_OFF 1      /* int32 [E+1] */
#define MXMOE_SAVED_ROW_OF_SLOT 2  /* int32 [T*k] */
#define MXMOE_SAVED_TOKEN_OF_ROW 3 /* int32 [cap] */
#define MXMOE_SAVED_PROB_OF_ROW 4  /* float [cap] */
#define MXMOE_SAVED_X_COLT 5       /* e4m3 [H, cap] */
#define MXMOE_SAVED_X_COLT_SF 6    /* e8m0, MMA layout */
#define MXMOE_SAVED_Z_COLT 7       /* e4m3 [F, cap] */
#define MXMOE_SAVED_Z_COLT_SF 8    /* e8m0, MMA layout */
#define MXMOE_SAVED_GU 9           /* bf16 [cap, 2F] (gate | up); 0 bytes with MXMOE_RECIPE_RECOMPUTE_GU */
#define MXMOE_SAVED_X_ROW 10       /* e4m3 [cap, H], only with MXMOE_RECIPE_RECOMPUTE_GU (else 0 bytes) */
#define MXMOE_SAVED_X_ROW_SF 11    /* e8m0, MMA layout, likewise */
#define MXMOE_SAVED_AMAX 12        /* float [2]: largest |x|, and the Z amax the forward encoded Z with;
                                      only with MXMOE_RECIPE_FP8_TENSOR (else 0 bytes) */
size_t grouped_mlp_saved_size(int32_t T, int32_t k, int32_t E, int32_t H, int32_t F);
int64_t grouped_mlp_saved_offset(int32_t field, int32_t T, int32_t k, int32_t E, int32_t H, int32_t F);

/* Scratch for one forward or backward call (the larger of the two). */
size_t grouped_mlp_workspace_size(int32_t T, int32_t k, int32_t E, int32_t H, int32_t F);

/*
 * grouped_mlp_fwd -- forward of the MoE expert MLP as one grouped computation
 * ("MoE-Training für biologische Grundmodelle optimieren", GroupedLinear, MXFP8 and
 * GroupedMLP passages; "NVIDIA apresenta técnicas ... arquitetura MoE", third
 * optimisation):
 *   route -> permute + quantise x -> fc1 grouped GEMM whose epilogue computes
 *   Z = silu(G) * U * p (p = the row's routing probability) and quantises Z to MXFP8
 *   (Z never reaches memory in 16-bit) -> fc2 grouped GEMM -> combine.
 *   x_dev bf16 [T, H]; topk_idx_dev int32 [T, k]; probs_dev float [T, k];
 *   wq_dev from mxmoe_weights_quantize; y_dev bf16 [T, H].
 * Limits: as moe_permute, plus H % 256 == 0, F % 256 == 0.
 */
mxmoe_status grouped_mlp_fwd(const void* x_dev, const int32_t* topk_idx_dev, const float* probs_dev,
                             const void* wq_dev, size_t wq_bytes, int32_t T, int32_t k, int32_t E, int32_t H,
                             int32_t F, void* y_dev, void* saved_dev, size_t saved_bytes, void* ws_dev,
                             size_t ws_bytes, void* stream);

/*
 * grouped_mlp_bwd -- the matching backward (straight-through for every quantiser):
 *   permute + quantise dy -> fc2 data-gradient GEMM whose epilogue applies the SwiGLU
 *   and probability-scale backward (dA = dZ*p, dG = dA*U*silu'(G), dU = dA*silu(G),
 *   dprob = sum_f dZ*A) and quantises dGU rowwise and colwise -> fc2 weight-gradient
 *   GEMM -> fc1 data-gradient GEMM -> fc1 weight-gradient GEMM -> combine.
 *   dy_dev bf16 [T, H]; outputs dx_dev bf16 [T, H], dW1_dev float [E, 2F, H],
 *   dW2_dev float [E, H, F], dprobs_dev float [T, k] (all overwritten; experts with
 *   no tokens get zero weight gradients).
 */
mxmoe_status grouped_mlp_bwd(const void* dy_dev, const void* saved_dev, size_t saved_bytes, const void* wq_dev,
                             size_t wq_bytes, int32_t T, int32_t k, int32_t E, int32_t H, int32_t F, void* dx_dev,
                             float* dW1_dev, float* dW2_dev, float* dprobs_dev, void* ws_dev, size_t ws_bytes,
                             void* stream);

/*
 * Recipes of the fused layer (bit flags; 0 = the default above). The forward and the
 * backward of one step take the same recipe; the saved-buffer and workspace sizes depend
 * on it (query them with the _ex size functions).
 *   MXMOE_RECIPE_GRAD_E5M2      the gradients dY and dGU are quantised to MXFP8 E5M2
 *                               (wider range, one mantissa bit fewer; the pages name FP8
 *                               beside MXFP8 and fix no element format): every backward
 *                               GEMM multiplies an E5M2 gradient by an E4M3 weight or
 *                               activation. Backward only.
 *   MXMOE_RECIPE_RECOMPUTE_GU   the forward saves the rowwise MXFP8 copy of the permuted
 *                               input (cap*H*(1+1/32) bytes) instead of the bf16 gate/up
 *                               pre-activations (cap*2F*2 bytes), and the backward first
 *                               recomputes G / U with the fc1 GEMM ("MoE-Training für
 *                               biologische Grundmodelle optimieren": activation memory
 *                               is the pressure MXFP8 and the fused kernel relieve). The
 *                               recomputed G / U live in the workspace for the call.
 *   MXMOE_RECIPE_SCALE_CEIL     every quantiser of the call (x, Z; dY, dGU) uses
 *                               MXMOE_SCALE_RULE_CEIL; quantise the weights with
 *                               mxmoe_weights_quantize_ex(..., MXMOE_SCALE_RULE_CEIL, ...).
 *   MXMOE_RECIPE_FP8_TENSOR     per-tensor FP8 in place of MXFP8 (see grouped_mlp_fp8_fwd);
 *                               it combines with no other bit, is run only through
 *                               grouped_mlp_fp8_fwd / _bwd (the _ex calls refuse it) and is
 *                               passed to the _ex size queries for that layer's sizes.
 * A recipe with any other bit set returns MXMOE_ERR_INVALID_ARG (sizes: 0 / -1).
 */
#define MXMOE_RECIPE_GRAD_E5M2 1
#define MXMOE_RECIPE_RECOMPUTE_GU 2
#define MXMOE_RECIPE_SCALE_CEIL 4
#define MXMOE_RECIPE_FP8_TENSOR 8
size_t grouped_mlp_saved_size_ex(int32_t T, int32_t k, int32_t E, int32_t H, int32_t F, int32_t recipe);
int64_t grouped_mlp_saved_offset_ex(int32_t field, int32_t T, int32_t k, int32_t E, int32_t H, int32_t F,
                                    int32_t recipe);
size_t grouped_mlp_workspace_size_ex(int32_t T, int32_t k, int32_t E, int32_t H, int32_t F, int32_t recipe);
mxmoe_status grouped_mlp_fwd_ex(const void* x_dev, const int32_t* topk_idx_dev, const float* probs_dev,
                                const void* wq_dev, size_t wq_bytes, int32_t T, int32_t k, int32_t E, int32_t H,
                                int32_t F, int32_t recipe, void* y_dev, void* saved_dev, size_t saved_bytes,
                                void* ws_dev, size_t ws_bytes, void* stream);
mxmoe_status grouped_mlp_bwd_ex(const void* dy_dev, const void* saved_dev, size_t saved_bytes, const void* wq_dev,
                                size_t wq_bytes, int32_t T, int32_t k, int32_t E, int32_t H, int32_t F,
                                int32_t recipe, void* dx_dev, float* dW1_dev, float* dW2_dev, float* dprobs_dev,
                                void* ws_dev, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------ per-tensor FP8 grouped MLP */

/*
 * The same layer with per-tensor FP8 in place of MXFP8 -- the pages name "FP8" beside
 * "MXFP8" ("MoE-Training für biologische Grundmodelle optimieren", precision passage) and
 * fix nothing else; the rule below is this library's reading.
 * Every operand is OCP E4M3 under one fp32 multiplier per tensor, m = 448 / amax rounded
 * to nearest (1 when amax == 0; the largest finite fp32 if the quotient overflows); an
 * element's code is E4M3(fp32(v * m)) (nearest, ties to even, saturating), its value
 * code / m. The tensors: x and dY (all tokens), W1[e] and W2[e] (one multiplier per
 * expert), Z and dGU (all routed rows). x, dY and the weights use their own amax (current
 * scaling: an extra read pass each). Z and dGU are produced tile by tile inside the fused
 * GEMM epilogues, so their multipliers come from an amax known before the call (delayed
 * scaling): the caller-owned device array amax_state_dev, fp32 [4], 16-byte aligned:
 *   [0] Z amax the forward encodes Z with (read);  [1] largest |Z| of this forward (written);
 *   [2] dGU amax the backward encodes dGU with (read); [3] largest |dGU| of this backward
 *   (written).
 * Values beyond the given amax saturate to +-448. A training loop copies [1] -> [0] and
 * [3] -> [2] between steps (the first step needs a starting value, e.g. from a forward /
 * backward run for that purpose). The operands' MXFP8 scale bytes are all 127 (2^0), so
 * the grouped GEMMs run the same block-scaled tensor-core instruction; each GEMM output is
 * scaled by 1 / (m_a * m_b) in its epilogue.
 *
 * mxmoe_weights_quantize_fp8: the per-expert amax of W1 and W2 (kept in the weights
 *   buffer) and the four copies of mxmoe_weights_quantize, per-tensor encoded. Same
 *   arguments, buffer size and limits as mxmoe_weights_quantize.
 * grouped_mlp_fp8_fwd / grouped_mlp_fp8_bwd: the steps, arguments, limits and outputs of
 *   grouped_mlp_fwd / _bwd, with weights from mxmoe_weights_quantize_fp8, saved-buffer and
 *   workspace sizes from the _ex queries with MXMOE_RECIPE_FP8_TENSOR, and amax_state_dev as
 *   above (null or misaligned: MXMOE_ERR_INVALID_ARG). The backward takes the saved buffer
 *   of a per-tensor forward.
 */
mxmoe_status mxmoe_weights_quantize_fp8(const void* W1_dev, const void* W2_dev, int32_t E, int32_t H, int32_t F,
                                        void* wq_dev, size_t wq_bytes, void* stream);
mxmoe_status grouped_mlp_fp8_fwd(const void* x_dev, const int32_t* topk_idx_dev, const float* probs_dev,
                                 const void* wq_dev, size_t wq_bytes, int32_t T, int32_t k, int32_t E, int32_t H,
                                 int32_t F, float* amax_state_dev, void* y_dev, void* saved_dev, size_t saved_bytes,
                                 void* ws_dev, size_t ws_bytes, void* stream);
mxmoe_status grouped_mlp_fp8_bwd(const void* dy_dev, const void* saved_dev, size_t saved_bytes, const void* wq_dev,
                                 size_t wq_bytes, int32_t T, int32_t k, int32_t E, int32_t H, int32_t F,
                                 float* amax_state_dev, void* dx_dev, float* dW1_dev, float* dW2_dev,
                                 float* dprobs_dev, void* ws_dev, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------ bf16 grouped MLP */

/*
 * The same expert MLP in bf16: the 16-bit comparison point the pages set MXFP8 against
 * ("MoE-Training für biologische Grundmodelle optimieren", MXFP8 passage: MXFP8 halves the
 * bits of the 16-bit operands). Every step of grouped_mlp_fwd / grouped_mlp_bwd runs with
 * the quantisers replaced by bf16 copies (the permuted rows and their transposes) and the
 * GEMMs on tcgen05 kind::f16 with fp32 accumulation; the fused epilogues write Z and dGU
 * in bf16. Same argument meaning, limits and error behaviour as the MXFP8 layer.
 *
 * Weights: one opaque device buffer of mxmoe_weights_bf16_size(E, H, F) bytes holding
 *   W1 rows [E*2F, H] (gate / up interleaved in 64-row blocks, as the MXFP8 copy),
 *   W1^T [E*H, 2F], W2 rows [E*H, F], W2^T [E*F, H], all bf16,
 * written by mxmoe_weights_bf16_prepare from W1_dev bf16 [E, 2F, H], W2_dev bf16 [E, H, F].
 * Saved activations: grouped_mlp_bf16_saved_size bytes (routing maps, the transposed
 * permuted input [H, cap] and Z^T [F, cap], gate/up pre-activations [cap, 2F], bf16).
 * Scratch: grouped_mlp_bf16_workspace_size bytes for either call.
 */
size_t mxmoe_weights_bf16_size(int32_t E, int32_t H, int32_t F);
mxmoe_status mxmoe_weights_bf16_prepare(const void* W1_dev, const void* W2_dev, int32_t E, int32_t H, int32_t F,
                                        void* wb_dev, size_t wb_bytes, void* stream);
size_t grouped_mlp_bf16_saved_size(int32_t T, int32_t k, int32_t E, int32_t H, int32_t F);
size_t grouped_mlp_bf16_workspace_size(int32_t T, int32_t k, int32_t E, int32_t H, int32_t F);
mxmoe_status grouped_mlp_bf16_fwd(const void* x_dev, const int32_t* topk_idx_dev, const float* probs_dev,
                                  const void* wb_dev, size_t wb_bytes, int32_t T, int32_t k, int32_t E, int32_t H,
                                  int32_t F, void* y_dev, void* saved_dev, size_t saved_bytes, void* ws_dev,
                                  size_t ws_bytes, void* stream);
mxmoe_status grouped_mlp_bf16_bwd(const void* dy_dev, const void* saved_dev, size_t saved_bytes, const void* wb_dev,
                                  size_t wb_bytes, int32_t T, int32_t k, int32_t E, int32_t H, int32_t F,
                                  void* dx_dev, float* dW1_dev, float* dW2_dev, float* dprobs_dev, void* ws_dev,
                                  size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------ instrumentation */

/* Stage tags reported by mxmoe_profile_read (one per enqueued stage). */
#define MXMOE_STAGE_ROUTE 1          /* moe_permute (3 small kernels) */
#define MXMOE_STAGE_QUANT_X 2        /* permute + quantise x (rowwise + colwise) */
#define MXMOE_STAGE_FC1_SWIGLU 3     /* fc1 grouped GEMM + SwiGLU x prob -> MXFP8 epilogue */
#define MXMOE_STAGE_FC2 4            /* fc2 grouped GEMM */
#define MXMOE_STAGE_COMBINE 5        /* moe_unpermute of y */
#define MXMOE_STAGE_QUANT_W1 6       /* W1 rowwise + colwise */
#define MXMOE_STAGE_QUANT_W2 7       /* W2 rowwise + colwise */
#define MXMOE_STAGE_QUANT_DY 8       /* permute + quantise dy */
#define MXMOE_STAGE_FC2_DGRAD 9      /* fc2 data-gradient GEMM + SwiGLU backward epilogue */
#define MXMOE_STAGE_DPROB 10         /* dprob reduction */
#define MXMOE_STAGE_FC2_WGRAD 11     /* fc2 weight-gradient GEMM */
#define MXMOE_STAGE_FC1_DGRAD 12     /* fc1 data-gradient GEMM */
#define MXMOE_STAGE_FC1_WGRAD 13     /* fc1 weight-gradient GEMM */
#define MXMOE_STAGE_COMBINE_DX 14    /* moe_unpermute of dx */
#define MXMOE_STAGE_GEMM 15          /* standalone grouped_gemm_mxfp8 */
#define MXMOE_STAGE_WGRAD 16         /* standalone grouped_gemm_mxfp8_wgrad */
#define MXMOE_STAGE_QUANT 17         /* standalone mxfp8_quantize */
#define MXMOE_STAGE_ROUTER 18        /* moe_router_topk */
#define MXMOE_STAGE_ROUTER_BWD 19    /* moe_router_topk_bwd */
#define MXMOE_STAGE_FC1_RECOMPUTE 20 /* backward: fc1 GEMM recomputing G / U (MXMOE_RECIPE_RECOMPUTE_GU) */

/* Host-side stage timing, off by default: while enabled, every stage the library
 * enqueues is bracketed by two CUDA events recorded on that stage's stream (up to
 * max_stages stages; later ones are not recorded). Creates 2*max_stages events on the
 * current device. Not thread-safe; for benchmarks. */
mxmoe_status mxmoe_profile_enable(int32_t max_stages);
mxmoe_status mxmoe_profile_disable(void);
/* Waits for the recorded events, writes up to `cap` (tag, milliseconds) pairs, returns
 * how many stages were recorded (and clears the record). */
int32_t mxmoe_profile_read(int32_t* tags_host, float* ms_host, int32_t cap);
/* Number of CUDA kernels this library has launched since it was loaded. */
int64_t mxmoe_launch_count(void);

#ifdef __cplusplus
}
#endif
#endif /* MXMOE_H_ */
