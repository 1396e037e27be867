// MXFP8 quantisation of activations and weights, rowwise and colwise from one read,
// optionally fused with the expert permutation (row gather).
//
// "MoE-Training für biologische Grundmodelle optimieren" (hyper.ai/de), MXFP8 passage:
// 8-bit values with one scale per block of 32; GroupedMLP passage: the 16-bit -> 8-bit
// conversions are fused rather than run as separate operations. Element / scale rule:
// OCP MX (E4M3 elements, E8M0 scale, X = clamp(floor(log2 amax) - 8, -127, 127),
// round-to-nearest-even with saturation); E5M2 elements (largest exponent 15 in place of
// 8) for the gradient variant, on the per-tile path; either scale rule (OCP, or the
// exponent rounded up so that nothing saturates) on both paths.
//
// One CTA quantises a 128 x 128 tile staged in shared memory: rowwise blocks (32
// consecutive columns of a row) and colwise blocks (32 consecutive rows of a column,
// written transposed) come from the same HBM read. bf16 rows are read 32 bytes per load,
// and the 32 codes of a block leave in one 256-bit store (a whole 32-byte sector) when the
// destination is 32-byte aligned: half as many load and store requests as 16-byte vectors,
// and no half-sector writes.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "mxmoe_device.cuh"
#include "mxmoe_launch.h"
#include "ptx_sm100.cuh"
#include "tensor_map.h"

namespace mxmoe {

constexpr int kQTile = 128;
constexpr int kQThreads = 256;
// 32 code bytes at p: one 256-bit store when p is 32-byte aligned, else two 16-byte stores
__device__ __forceinline__ void st_codes32(uint8_t* p, const uint32_t (&q)[8]) {
  if ((reinterpret_cast<uintptr_t>(p) & 31) == 0) {
    asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(q[0]), "r"(q[1]),
                 "r"(q[2]), "r"(q[3]), "r"(q[4]), "r"(q[5]), "r"(q[6]), "r"(q[7])
                 : "memory");
  } else {
    uint4* d = reinterpret_cast<uint4*>(p);
    d[0] = make_uint4(q[0], q[1], q[2], q[3]);
    d[1] = make_uint4(q[4], q[5], q[6], q[7]);
  }
}

template <typename T>
struct SrcTraits;
// Shared tile layout: each 32-element block of a row is followed by 16 bytes of padding
// (block stride kBS elements, row stride 4 * kBS). With 4 lanes per row (one per block)
// the rowwise 16-byte loads, and with consecutive column pairs per warp the colwise
// 4-/8-byte loads, hit distinct banks.
template <>
struct SrcTraits<__nv_bfloat16> {
  static constexpr int kVec = 8;   // elements per 16-byte vector
  static constexpr int kBS = 40;   // 32 elements + 16 bytes
};
template <>
struct SrcTraits<float> {
  static constexpr int kVec = 4;
  static constexpr int kBS = 36;
};
template <typename T>
__device__ __forceinline__ int tile_off(int row, int col) {
  using Tr = SrcTraits<T>;
  return row * (4 * Tr::kBS) + (col >> 5) * Tr::kBS + (col & 31);
}

__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }
__device__ __forceinline__ float to_f32(float v) { return v; }

// 32 consecutive elements of a shared-memory row -> fp32 (16-byte loads).
__device__ __forceinline__ void load32_row(const __nv_bfloat16* p, float (&v)[32]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 w = reinterpret_cast<const uint4*>(p)[i];
    v[8 * i + 0] = bf16_lo(w.x); v[8 * i + 1] = bf16_hi(w.x);
    v[8 * i + 2] = bf16_lo(w.y); v[8 * i + 3] = bf16_hi(w.y);
    v[8 * i + 4] = bf16_lo(w.z); v[8 * i + 5] = bf16_hi(w.z);
    v[8 * i + 6] = bf16_lo(w.w); v[8 * i + 7] = bf16_hi(w.w);
  }
}
__device__ __forceinline__ void load32_row(const float* p, float (&v)[32]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 w = reinterpret_cast<const float4*>(p)[i];
    v[4 * i + 0] = w.x; v[4 * i + 1] = w.y; v[4 * i + 2] = w.z; v[4 * i + 3] = w.w;
  }
}
// Two adjacent elements of a shared-memory row -> fp32.
__device__ __forceinline__ void load_pair(const __nv_bfloat16* p, float& a, float& b) {
  const uint32_t w = *reinterpret_cast<const uint32_t*>(p);
  a = bf16_lo(w);
  b = bf16_hi(w);
}
__device__ __forceinline__ void load_pair(const float* p, float& a, float& b) {
  const float2 w = *reinterpret_cast<const float2*>(p);
  a = w.x;
  b = w.y;
}

// Largest magnitudes of packed bf16 pairs: one bf16x2 max-of-magnitudes per pair of
// words (the signs of partial results are meaningless and are cleared at the end); a
// pairwise tree keeps the dependent chain short. A NaN gives the canonical NaN, whose
// all-ones exponent yields the same block scale as any other NaN.
__device__ __forceinline__ uint32_t bmax2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.NaN.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
template <int N>
__device__ __forceinline__ uint32_t bmax_tree(const uint32_t (&w)[N]) {
  uint32_t t[N / 2];
#pragma unroll
  for (int i = 0; i < N / 2; ++i) t[i] = bmax2(w[2 * i], w[2 * i + 1]);
#pragma unroll
  for (int s = N / 4; s >= 1; s >>= 1)
#pragma unroll
    for (int i = 0; i < s; ++i) t[i] = bmax2(t[i], t[i + s]);
  return t[0] & 0x7FFF7FFFu;
}
// MXFP8 of 32 bf16 values given as 16 packed words (element 2k in the low half of w[k],
// 2k+1 in the high half). The block amax of the bf16 values equals that of the values
// widened to fp32 (widening is exact), hence the same scale as quant_block32; the scaled
// values are formed two per instruction (packed fp32x2 multiply, each lane rounded as the
// scalar multiply). tm != 0: per-tensor FP8 under the multiplier tm (scale byte 127).
template <int FMT = MXMOE_FMT_E4M3>
__device__ __forceinline__ uint8_t quant_block32_bf16(const uint32_t (&w)[16], uint32_t (&out)[8],
                                                      bool ceil_rule = false, float tm = 0.f) {
  int32_t X = 0;
  float s = tm;
  if (tm == 0.f) {
    const uint32_t m = bmax_tree(w);
    const uint32_t amax = max(m << 16, m & 0xFFFF0000u);
    X = mx_scale_exp_from_amax_bits<FMT>(amax, ceil_rule);
    s = mx_inv_scale(X);
  }
  const float2 s2 = make_float2(s, s);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float2 a = __fmul2_rn(make_float2(bf16_lo(w[2 * i]), bf16_hi(w[2 * i])), s2);
    const float2 c = __fmul2_rn(make_float2(bf16_lo(w[2 * i + 1]), bf16_hi(w[2 * i + 1])), s2);
    out[i] = (uint32_t)fp8x2<FMT>(a.x, a.y) | ((uint32_t)fp8x2<FMT>(c.x, c.y) << 16);
  }
  return (uint8_t)(X + 127);
}

// Colwise MXFP8 of two adjacent columns over 32 rows: w[r] holds (column c, row r) in
// its low half and (column c+1, row r) in its high half.
template <int FMT = MXMOE_FMT_E4M3>
__device__ __forceinline__ void quant_colpair_bf16(const uint32_t (&w)[32], uint32_t (&o0)[8], uint32_t (&o1)[8],
                                                   uint8_t& sb0, uint8_t& sb1, bool ceil_rule = false,
                                                   float tm = 0.f) {
  int32_t X0 = 0, X1 = 0;
  float s0 = tm, s1 = tm;
  if (tm == 0.f) {
    const uint32_t m = bmax_tree(w);
    X0 = mx_scale_exp_from_amax_bits<FMT>(m << 16, ceil_rule);
    X1 = mx_scale_exp_from_amax_bits<FMT>(m & 0xFFFF0000u, ceil_rule);
    s0 = mx_inv_scale(X0);
    s1 = mx_inv_scale(X1);
  }
  const float2 s02 = make_float2(s0, s0), s12 = make_float2(s1, s1);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float2 a0 = __fmul2_rn(make_float2(bf16_lo(w[4 * i]), bf16_lo(w[4 * i + 1])), s02);
    const float2 b0 = __fmul2_rn(make_float2(bf16_lo(w[4 * i + 2]), bf16_lo(w[4 * i + 3])), s02);
    const float2 a1 = __fmul2_rn(make_float2(bf16_hi(w[4 * i]), bf16_hi(w[4 * i + 1])), s12);
    const float2 b1 = __fmul2_rn(make_float2(bf16_hi(w[4 * i + 2]), bf16_hi(w[4 * i + 3])), s12);
    o0[i] = (uint32_t)fp8x2<FMT>(a0.x, a0.y) | ((uint32_t)fp8x2<FMT>(b0.x, b0.y) << 16);
    o1[i] = (uint32_t)fp8x2<FMT>(a1.x, a1.y) | ((uint32_t)fp8x2<FMT>(b1.x, b1.y) << 16);
  }
  sb0 = (uint8_t)(X0 + 127);
  sb1 = (uint8_t)(X1 + 127);
}

template <int FMT>
__device__ __forceinline__ uint8_t quant_row_block(const __nv_bfloat16* p, uint32_t (&q)[8], bool ceil_rule,
                                                   float tm) {
  uint32_t w[16];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 v = reinterpret_cast<const uint4*>(p)[i];
    w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
  }
  return quant_block32_bf16<FMT>(w, q, ceil_rule, tm);
}
template <int FMT>
__device__ __forceinline__ uint8_t quant_row_block(const float* p, uint32_t (&q)[8], bool ceil_rule, float tm) {
  float v[32];
  load32_row(p, v);
  return quant_block32<FMT>(v, q, ceil_rule, tm);
}

template <int FMT>
__device__ __forceinline__ void quant_col_pair(const __nv_bfloat16* p, int ld, uint32_t (&q0)[8], uint32_t (&q1)[8],
                                               uint8_t& s0, uint8_t& s1, bool ceil_rule, float tm) {
  uint32_t w[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) w[i] = *reinterpret_cast<const uint32_t*>(p + i * ld);
  quant_colpair_bf16<FMT>(w, q0, q1, s0, s1, ceil_rule, tm);
}
template <int FMT>
__device__ __forceinline__ void quant_col_pair(const float* p, int ld, uint32_t (&q0)[8], uint32_t (&q1)[8],
                                               uint8_t& s0, uint8_t& s1, bool ceil_rule, float tm) {
  float v[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = p[i * ld];
  s0 = quant_block32<FMT>(v, q0, ceil_rule, tm);
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = p[i * ld + 1];
  s1 = quant_block32<FMT>(v, q1, ceil_rule, tm);
}

// One CTA per 128 x 128 tile (many resident per SM to overlap load latency).
template <typename T, int FMT>
__global__ void __launch_bounds__(kQThreads, sizeof(T) == 2 ? 4 : 2) mxfp8_quantize_kernel(QuantArgs a) {
  using Tr = SrcTraits<T>;
  extern __shared__ __align__(16) uint8_t q_smem_raw[];
  T* tile = reinterpret_cast<T*>(q_smem_raw);
  // the tile's scale bytes, four per row (rowwise) / per transposed row (colwise)
  __shared__ uint32_t s_rsc[kQTile], s_csc[kQTile];

  const int64_t c0 = (int64_t)blockIdx.x * kQTile;
  const int64_t r0 = (int64_t)blockIdx.y * kQTile;
  const int64_t b = blockIdx.z;
  // elements per load: 32 bytes for bf16 (one 256-bit load), 16 bytes for fp32
  constexpr int LV = sizeof(T) == 2 ? 16 : Tr::kVec;
  constexpr int VPR = kQTile / LV;              // vectors per tile row
  constexpr int NL = kQTile * VPR / kQThreads;  // vectors per thread
  constexpr int RSTEP = kQThreads / VPR;        // tile rows between a thread's vectors
  const int row_t = threadIdx.x / VPR, cv = threadIdx.x % VPR;
  // the valid-row count and this thread's gather indices are read together: the index
  // array holds out_rows entries, so reading them before the count is known stays in bounds
  int32_t gidx[NL];
#pragma unroll
  for (int k = 0; k < NL; ++k) {
    const int64_t orow = r0 + row_t + k * RSTEP;
    gidx[k] = (a.gather && orow < a.out_rows) ? __ldg(a.gather + orow) : -1;
  }
  int64_t nvalid = a.out_rows;
  if (a.nrows) {
    const int64_t nv = __ldg(a.nrows);
    nvalid = nv < nvalid ? nv : nvalid;
  }
  if (r0 >= nvalid) return;
  const T* src = reinterpret_cast<const T*>(a.src);
  const float tm = a.tensor_amax ? tensor_multiplier(a.tensor_amax[a.tensor_per_batch ? b : 0]) : 0.f;

  // ---- load the tile (gathered rows, zero outside the matrix / for pad rows); all of a
  // thread's loads (32 bytes per bf16 vector, 16 per fp32 vector) are issued before any use
  {
    const int64_t col = c0 + (int64_t)cv * LV;
    int64_t srow[NL];
#pragma unroll
    for (int k = 0; k < NL; ++k) {
      const int64_t orow = r0 + row_t + k * RSTEP;
      srow[k] = -1;
      if (orow < nvalid && col < a.cols) srow[k] = a.gather ? (int64_t)gidx[k] : b * a.rows + orow;
      // checked build: a gathered row outside the source matrix reads as a zero row
      if (a.gather && srow[k] >= 0 && !check_index(srow[k], a.rows, 67)) srow[k] = -1;
    }
    constexpr int HV = LV / Tr::kVec;  // 16-byte halves per load
    uint4 buf[NL][HV];
    // a 256-bit load needs a 32-byte aligned address: rows are 64-byte multiples (cols % 32
    // == 0) and vectors start at 32-byte offsets, so the base pointer decides
    const bool v8 = (reinterpret_cast<uintptr_t>(src) & 31) == 0;
#pragma unroll
    for (int k = 0; k < NL; ++k) {
      const uint4* p = reinterpret_cast<const uint4*>(src + srow[k] * a.cols + col);
      if (srow[k] < 0) {
#pragma unroll
        for (int hv = 0; hv < HV; ++hv) buf[k][hv] = make_uint4(0, 0, 0, 0);
      } else if constexpr (HV == 2) {
        if (v8) {
          asm volatile("ld.global.nc.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                       : "=r"(buf[k][0].x), "=r"(buf[k][0].y), "=r"(buf[k][0].z), "=r"(buf[k][0].w),
                         "=r"(buf[k][1].x), "=r"(buf[k][1].y), "=r"(buf[k][1].z), "=r"(buf[k][1].w)
                       : "l"(p));
        } else {
          buf[k][0] = __ldg(p);
          buf[k][1] = __ldg(p + 1);
        }
      } else {
        buf[k][0] = __ldg(p);
      }
    }
#pragma unroll
    for (int k = 0; k < NL; ++k)
#pragma unroll
      for (int hv = 0; hv < HV; ++hv)
        *reinterpret_cast<uint4*>(tile + tile_off<T>(row_t + k * RSTEP, cv * LV + hv * Tr::kVec)) = buf[k][hv];
  }
  __syncthreads();

  // ---- rowwise: item = (row, 32-column block); 4 lanes cover a row, so a warp stores 8
  // whole 128-byte lines
  if (a.row_data) {
#pragma unroll 1
    for (int it = threadIdx.x; it < kQTile * 4; it += kQThreads) {
      const int row = it >> 2, blk = it & 3;
      const int64_t orow = r0 + row;
      const int64_t col = c0 + 32 * blk;
      if (orow >= nvalid || col >= a.cols) continue;
      uint32_t q[8];
      const uint8_t sb = quant_row_block<FMT>(tile + tile_off<T>(row, 32 * blk), q, a.scale_rule != 0, tm);
      int64_t drow = orow;
      if (a.row_ilv > 0) {  // gate / up interleave of the fc1 operand
        const int64_t hf = orow >= a.row_ilv, rr = orow - hf * a.row_ilv;
        drow = (rr >> 6) * 128 + hf * 64 + (rr & 63);
      }
      const int64_t grow = b * a.out_rows + drow;
      st_codes32(a.row_data + grow * a.cols + col, q);
      reinterpret_cast<uint8_t*>(s_rsc)[row * 4 + blk] = sb;
    }
  }
  // ---- colwise: item = (pair of adjacent columns, 32-row block), one per thread; a warp
  // reads 32 consecutive column pairs of a row per load (conflict free); stored transposed
  if (a.col_data) {
    const int pcol = threadIdx.x & 63, rb = threadIdx.x >> 6;
    const int64_t col = c0 + 2 * pcol;
    const int64_t orow = r0 + 32 * rb;
    if (orow < nvalid && col < a.cols) {
      uint32_t q0[8], q1[8];
      uint8_t s0, s1;
      quant_col_pair<FMT>(tile + tile_off<T>(32 * rb, 2 * pcol), 4 * Tr::kBS, q0, q1, s0, s1, a.scale_rule != 0,
                          tm);
      const int64_t grow = b * a.cols + col;  // row of the transposed matrix
      st_codes32(a.col_data + grow * a.out_rows + orow, q0);
      st_codes32(a.col_data + (grow + 1) * a.out_rows + orow, q1);
      reinterpret_cast<uint8_t*>(s_csc)[(2 * pcol) * 4 + rb] = s0;
      reinterpret_cast<uint8_t*>(s_csc)[(2 * pcol + 1) * 4 + rb] = s1;
    }
  }
  __syncthreads();
  // ---- scale bytes: a row's four blocks of this tile are adjacent in both scale layouts
  // (one 32-bit store); threads 0-127 store the rowwise scales, 128-255 the colwise ones.
  // In the MMA layout the tile's 128 x 4 bytes of a copy form one 512-byte chunk, and
  // thread t stores its word t (row (t % 4) * 32 + t / 4), so a warp writes 128
  // consecutive bytes.
  {
    const bool rowwise = threadIdx.x < kQTile;
    const int t = threadIdx.x & (kQTile - 1);
    const int32_t layout = rowwise ? a.row_layout : a.col_layout;
    const int r = layout == MXMOE_SCALE_MMA ? (t & 3) * 32 + (t >> 2) : t;
    uint8_t* sf = rowwise ? a.row_sf : a.col_sf;
    bool ok;
    int64_t grow, kb0, srows, scols;
    int nb;
    if (rowwise) {
      const int64_t orow = r0 + r;
      int64_t drow = orow;
      if (a.row_ilv > 0) {  // gate / up interleave of the fc1 operand
        const int64_t hf = orow >= a.row_ilv, rr = orow - hf * a.row_ilv;
        drow = (rr >> 6) * 128 + hf * 64 + (rr & 63);
      }
      ok = a.row_data != nullptr && orow < nvalid;
      grow = b * a.out_rows + drow;
      kb0 = c0 / 32;
      nb = (int)((a.cols - c0) / 32 < 4 ? (a.cols - c0) / 32 : 4);
      srows = a.batch * a.out_rows;
      scols = a.cols;
    } else {
      ok = a.col_data != nullptr && c0 + r < a.cols;
      grow = b * a.cols + c0 + r;
      kb0 = r0 / 32;
      nb = (int)((nvalid - r0 + 31) / 32 < 4 ? (nvalid - r0 + 31) / 32 : 4);
      srows = a.batch * a.cols;
      scols = a.out_rows;
    }
    if (ok) {
      const uint32_t w = rowwise ? s_rsc[r] : s_csc[r];
      uint8_t* p = sf + sf_offset(layout, srows, scols, grow, kb0);
      if (nb == 4 && (reinterpret_cast<uintptr_t>(p) & 3) == 0) {
        *reinterpret_cast<uint32_t*>(p) = w;
      } else {
        for (int j = 0; j < nb; ++j) sf[sf_offset(layout, srows, scols, grow, kb0 + j)] = (uint8_t)(w >> (8 * j));
      }
    }
  }
}

// ----------------------------------------------------------------------------- dense bf16 path
// Persistent variant for dense (ungathered) bf16 matrices whose rows and columns are
// multiples of 128 -- the expert weights. Each CTA walks a strided list of 128 x 128
// tiles. Tiles arrive by TMA into a 2-stage ring (the next tile is read while this one is
// quantised); a stage holds the tile as two 64-column halves of [128 rows][128 bytes] in
// the TMA 128-byte swizzle (16-byte chunk j of row r at chunk j ^ (r % 8)). The E4M3
// codes of both copies are assembled in shared memory in the same swizzled layout and
// leave by TMA stores of whole 128-byte lines; only the scale bytes are stored directly.
constexpr int kQtStages = 2;
constexpr uint32_t kQtStageBytes = 2 * 128 * 128;   // 32 KB of bf16
constexpr uint32_t kQtOutBytes = 128 * 128;         // 16 KB of codes per copy
constexpr uint32_t kQtOffOut = kQtStages * kQtStageBytes;
constexpr uint32_t kQtOffBar = kQtOffOut + 2 * kQtOutBytes;
constexpr uint32_t kQtSmem = kQtOffBar + 64 + 1024;

// Byte offset of (row, 16-byte chunk j) in a [rows][128 bytes] 128-byte-swizzled region.
__device__ __forceinline__ uint32_t sw128(int row, int j) {
  return (uint32_t)row * 128u + ((uint32_t)(j ^ (row & 7)) << 4);
}
// Byte offset of (row, col) of a bf16 tile inside its stage.
__device__ __forceinline__ uint32_t qt_off(int row, int col) {
  const uint32_t half = (uint32_t)col >> 6, byte = ((uint32_t)col & 63) * 2;
  return half * 16384u + sw128(row, (int)(byte >> 4)) + (byte & 15);
}

__global__ void __launch_bounds__(kQThreads, 2)
    mxfp8_quantize_tma_kernel(const __grid_constant__ CUtensorMap tm, const __grid_constant__ CUtensorMap tm_row,
                              const __grid_constant__ CUtensorMap tm_col, const __grid_constant__ QuantArgs a,
                              int32_t tiles_c, int32_t tiles_per_batch, int32_t ntiles) {
  extern __shared__ uint8_t qt_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(qt_smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* out_row = smem + kQtOffOut;
  uint8_t* out_col = out_row + kQtOutBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kQtOffBar);
  volatile int32_t* s_abort = reinterpret_cast<volatile int32_t*>(full + kQtStages);

  const int32_t first = (int32_t)blockIdx.x, stride = (int32_t)gridDim.x;
  const int32_t mine = first < ntiles ? (ntiles - 1 - first) / stride + 1 : 0;
  auto tile_of = [&](int32_t i, int64_t& b, int64_t& r0, int64_t& c0) {
    const int32_t t = first + i * stride;
    b = t / tiles_per_batch;
    const int32_t rem = t % tiles_per_batch;
    r0 = (int64_t)(rem / tiles_c) * kQTile;
    c0 = (int64_t)(rem % tiles_c) * kQTile;
  };
  auto issue = [&](int32_t i) {  // thread 0: TMA loads of my i-th tile into stage i % S
    int64_t b, r0, c0;
    tile_of(i, b, r0, c0);
    uint8_t* st = smem + (i % kQtStages) * kQtStageBytes;
    uint64_t* bar = &full[i % kQtStages];
    ptx::mbar_arrive_expect_tx(bar, kQtStageBytes);
    const int32_t y = (int32_t)(b * a.rows + r0);
    ptx::tma_load_2d(st, &tm, (int32_t)c0, y, bar);
    ptx::tma_load_2d(st + 16384, &tm, (int32_t)c0 + 64, y, bar);
  };
  if (threadIdx.x == 0) {
    for (int s = 0; s < kQtStages; ++s) ptx::mbar_init(&full[s], 1);
    *s_abort = 0;
    ptx::fence_mbar_init();
    ptx::prefetch_tensormap(&tm);
    ptx::prefetch_tensormap(&tm_row);
    ptx::prefetch_tensormap(&tm_col);
    for (int32_t i = 0; i < kQtStages && i < mine; ++i) issue(i);
  }
  __syncthreads();

  for (int32_t i = 0; i < mine; ++i) {
    const bool ok = ptx::mbar_wait(&full[i % kQtStages], (uint32_t)(i / kQtStages) & 1u, 30);
    if (!ok) *s_abort = 1;
    // the previous tile's output stores have read the staging buffers
    if (threadIdx.x == 0) ptx::bulk_wait_group_read<0>();
    __syncthreads();
    if (*s_abort) break;
    const uint8_t* st = smem + (i % kQtStages) * kQtStageBytes;
    int64_t b, r0, c0;
    tile_of(i, b, r0, c0);
    const float tm = a.tensor_amax ? tensor_multiplier(a.tensor_amax[a.tensor_per_batch ? b : 0]) : 0.f;

    // rowwise: 512 items (row, 32-column block), 2 per thread; a warp takes 8 rows and
    // lanes l, l + 8, l + 16, l + 24 share a row, so each 8-lane phase of a 16-byte shared
    // access touches 8 distinct chunk positions (conflict free)
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int it = threadIdx.x + k * kQThreads;
      const int l = it & 31;
      const int row = 8 * (it >> 5) + (l & 7), blk = l >> 3;
      uint32_t w[16];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const uint4 v = *reinterpret_cast<const uint4*>(st + qt_off(row, 32 * blk + 8 * t));
        w[4 * t] = v.x; w[4 * t + 1] = v.y; w[4 * t + 2] = v.z; w[4 * t + 3] = v.w;
      }
      uint32_t q[8];
      const uint8_t sb = quant_block32_bf16(w, q, a.scale_rule != 0, tm);
      *reinterpret_cast<uint4*>(out_row + sw128(row, 2 * blk)) = make_uint4(q[0], q[1], q[2], q[3]);
      *reinterpret_cast<uint4*>(out_row + sw128(row, 2 * blk + 1)) = make_uint4(q[4], q[5], q[6], q[7]);
      const int64_t orow = r0 + row;
      int64_t drow = orow;
      if (a.row_ilv > 0) {  // gate / up interleave of the fc1 operand
        const int64_t hf = orow >= a.row_ilv, rr = orow - hf * a.row_ilv;
        drow = (rr >> 6) * 128 + hf * 64 + (rr & 63);
      }
      a.row_sf[sf_offset(a.row_layout, a.batch * a.out_rows, a.cols, b * a.out_rows + drow, (c0 >> 5) + blk)] = sb;
    }
    // colwise: item = (pair of adjacent columns, 32-row block), one per thread; a warp
    // reads 32 consecutive column pairs (one 128-byte half-row) per load, conflict free.
    // Codes go to rows 2p, 2p + 1 of the transposed [128 columns][128 rows] output tile.
    {
      const int pcol = threadIdx.x & 63, rb = threadIdx.x >> 6;
      uint32_t w[32];
#pragma unroll
      for (int r = 0; r < 32; ++r) w[r] = *reinterpret_cast<const uint32_t*>(st + qt_off(32 * rb + r, 2 * pcol));
      uint32_t q0[8], q1[8];
      uint8_t s0, s1;
      quant_colpair_bf16(w, q0, q1, s0, s1, a.scale_rule != 0, tm);
      *reinterpret_cast<uint4*>(out_col + sw128(2 * pcol, 2 * rb)) = make_uint4(q0[0], q0[1], q0[2], q0[3]);
      *reinterpret_cast<uint4*>(out_col + sw128(2 * pcol, 2 * rb + 1)) = make_uint4(q0[4], q0[5], q0[6], q0[7]);
      *reinterpret_cast<uint4*>(out_col + sw128(2 * pcol + 1, 2 * rb)) = make_uint4(q1[0], q1[1], q1[2], q1[3]);
      *reinterpret_cast<uint4*>(out_col + sw128(2 * pcol + 1, 2 * rb + 1)) = make_uint4(q1[4], q1[5], q1[6], q1[7]);
      const int64_t grow = b * a.cols + c0 + 2 * pcol;  // row of the transposed matrix
      const int64_t kb = (r0 >> 5) + rb;
      a.col_sf[sf_offset(a.col_layout, a.batch * a.cols, a.out_rows, grow, kb)] = s0;
      a.col_sf[sf_offset(a.col_layout, a.batch * a.cols, a.out_rows, grow + 1, kb)] = s1;
    }
    ptx::fence_proxy_async_shared();  // this thread's staging writes before the TMA stores
    __syncthreads();                  // stage i fully read, staging fully written
    if (threadIdx.x == 0) {
      // rowwise copy: two 64-row boxes (the fc1 interleave moves 64-row blocks)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        int64_t drow = r0 + 64 * hh;
        if (a.row_ilv > 0) {
          const int64_t hf = drow >= a.row_ilv, rr = drow - hf * a.row_ilv;
          drow = (rr >> 6) * 128 + hf * 64;
        }
        ptx::tma_store_2d(&tm_row, out_row + hh * 8192, (int32_t)c0, (int32_t)(b * a.out_rows + drow));
      }
      // colwise copy: the transposed tile, [128 columns][128 rows]
      ptx::tma_store_2d(&tm_col, out_col, (int32_t)r0, (int32_t)(b * a.cols + c0));
      ptx::bulk_commit_group();
      if (i + kQtStages < mine) issue(i + kQtStages);
    }
  }
  if (threadIdx.x == 0) ptx::bulk_wait_group<0>();
}

// ----------------------------------------------------------------------------- bf16 operand copies
// Operands of the bf16 grouped MLP: the same tiles, gather and interleave as the
// quantiser, but the outputs are plain bf16 -- the (permuted) rows and the transposed
// matrix (K-major operand of the weight-gradient GEMMs).
__global__ void __launch_bounds__(kQThreads, 4) bf16_copy_kernel(QuantArgs a) {
  using T = __nv_bfloat16;
  using Tr = SrcTraits<T>;
  extern __shared__ __align__(16) uint8_t q_smem_raw[];
  T* tile = reinterpret_cast<T*>(q_smem_raw);
  const int64_t c0 = (int64_t)blockIdx.x * kQTile;
  const int64_t r0 = (int64_t)blockIdx.y * kQTile;
  const int64_t b = blockIdx.z;
  int64_t nvalid = a.out_rows;
  if (a.nrows) {
    const int64_t nv = *a.nrows;
    nvalid = nv < nvalid ? nv : nvalid;
  }
  if (r0 >= nvalid) return;
  const T* src = reinterpret_cast<const T*>(a.src);
  constexpr int VPR = kQTile / Tr::kVec;
  constexpr int NL = kQTile * VPR / kQThreads;
  constexpr int RSTEP = kQThreads / VPR;
  const int row_t = threadIdx.x / VPR, cv = threadIdx.x % VPR;
  {
    const int64_t col = c0 + (int64_t)cv * Tr::kVec;
    uint4 buf[NL];
#pragma unroll
    for (int k = 0; k < NL; ++k) {
      const int64_t orow = r0 + row_t + k * RSTEP;
      int64_t srow = -1;
      if (orow < nvalid && col < a.cols) srow = a.gather ? (int64_t)__ldg(a.gather + orow) : b * a.rows + orow;
      buf[k] = srow >= 0 ? __ldg(reinterpret_cast<const uint4*>(src + srow * a.cols + col)) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int k = 0; k < NL; ++k)
      *reinterpret_cast<uint4*>(tile + tile_off<T>(row_t + k * RSTEP, cv * Tr::kVec)) = buf[k];
  }
  __syncthreads();
  uint16_t* rout = reinterpret_cast<uint16_t*>(a.row_data);
  uint16_t* cout = reinterpret_cast<uint16_t*>(a.col_data);
  if (rout) {
#pragma unroll 1
    for (int it = threadIdx.x; it < kQTile * 4; it += kQThreads) {
      const int row = it >> 2, blk = it & 3;
      const int64_t orow = r0 + row, col = c0 + 32 * blk;
      if (orow >= nvalid || col >= a.cols) continue;
      int64_t drow = orow;
      if (a.row_ilv > 0) {
        const int64_t hf = orow >= a.row_ilv, rr = orow - hf * a.row_ilv;
        drow = (rr >> 6) * 128 + hf * 64 + (rr & 63);
      }
      const uint4* sp = reinterpret_cast<const uint4*>(tile + tile_off<T>(row, 32 * blk));
      uint4* dp = reinterpret_cast<uint4*>(rout + (b * a.out_rows + drow) * a.cols + col);
#pragma unroll
      for (int i = 0; i < 4; ++i) dp[i] = sp[i];
    }
  }
  if (cout) {
    // a thread transposes a pair of adjacent columns over 32 rows
    const int pcol = threadIdx.x & 63, rb = threadIdx.x >> 6;
    const int64_t col = c0 + 2 * pcol, orow = r0 + 32 * rb;
    if (orow < nvalid && col < a.cols) {
      uint32_t w[32];
      const T* p = tile + tile_off<T>(32 * rb, 2 * pcol);
#pragma unroll
      for (int r = 0; r < 32; ++r) w[r] = *reinterpret_cast<const uint32_t*>(p + r * 4 * Tr::kBS);
      uint32_t lo[16], hi[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        lo[j] = __byte_perm(w[2 * j], w[2 * j + 1], 0x5410);  // column col, rows 2j, 2j+1
        hi[j] = __byte_perm(w[2 * j], w[2 * j + 1], 0x7632);  // column col + 1
      }
      uint4* d0 = reinterpret_cast<uint4*>(cout + (b * a.cols + col) * a.out_rows + orow);
      uint4* d1 = reinterpret_cast<uint4*>(cout + (b * a.cols + col + 1) * a.out_rows + orow);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        d0[i] = make_uint4(lo[4 * i], lo[4 * i + 1], lo[4 * i + 2], lo[4 * i + 3]);
        d1[i] = make_uint4(hi[4 * i], hi[4 * i + 1], hi[4 * i + 2], hi[4 * i + 3]);
      }
    }
  }
}

cudaError_t launch_bf16_copy(const QuantArgs& a, cudaStream_t st) {
  if (a.src_dtype != MXMOE_DTYPE_BF16) return cudaErrorInvalidValue;
  const size_t smem = (size_t)kQTile * 4 * SrcTraits<__nv_bfloat16>::kBS * sizeof(__nv_bfloat16);
  cudaError_t e = cudaFuncSetAttribute(bf16_copy_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)((a.cols + kQTile - 1) / kQTile), (unsigned)((a.out_rows + kQTile - 1) / kQTile),
            (unsigned)a.batch);
  if (grid.x == 0 || grid.y == 0 || grid.z == 0) return cudaSuccess;
  bf16_copy_kernel<<<grid, kQThreads, smem, st>>>(a);
  ++g_launch_count;
  return cudaGetLastError();
}

static bool qt_applies(const QuantArgs& a) {
  return a.src_dtype == MXMOE_DTYPE_BF16 && a.fmt == MXMOE_FMT_E4M3 && !a.gather && !a.nrows && a.out_rows == a.rows && a.rows % kQTile == 0 &&
         a.cols % kQTile == 0 && a.batch * a.rows < (int64_t)1 << 31 && a.batch * a.cols < (int64_t)1 << 31 &&
         a.row_data && a.col_data && (reinterpret_cast<uintptr_t>(a.row_data) & 15) == 0 &&
         (reinterpret_cast<uintptr_t>(a.col_data) & 15) == 0;
}

// 2-D uint8 map over [rows, 128 * k] codes for the TMA stores: box `box_rows` x 128 bytes,
// 128-byte swizzle (the staging layout).
static bool make_code_map(CUtensorMap* m, void* base, int64_t rows, int64_t cols, uint32_t box_rows) {
  auto fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols};
  cuuint32_t box[2] = {128, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static cudaError_t launch_qt(const QuantArgs& a, cudaStream_t st) {
  auto fn = get_encode_fn();
  if (!fn) return cudaErrorInvalidValue;
  CUtensorMap tm, tm_row, tm_col;
  cuuint64_t dims[2] = {(cuuint64_t)a.cols, (cuuint64_t)(a.batch * a.rows)};
  cuuint64_t strides[1] = {(cuuint64_t)(a.cols * 2)};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t estr[2] = {1, 1};
  if (fn(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(a.src), dims, strides, box, estr,
         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  if (!make_code_map(&tm_row, a.row_data, a.batch * a.out_rows, a.cols, 64) ||
      !make_code_map(&tm_col, a.col_data, a.batch * a.cols, a.out_rows, 128))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(mxfp8_quantize_tma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kQtSmem);
  if (e != cudaSuccess) return e;
  const int32_t tiles_c = (int32_t)(a.cols / kQTile);
  const int32_t tiles_per_batch = (int32_t)(a.rows / kQTile) * tiles_c;
  const int32_t ntiles = tiles_per_batch * (int32_t)a.batch;
  if (ntiles == 0) return cudaSuccess;
  int dev = 0, nsm = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  const int grid = std::min<int64_t>(ntiles, (int64_t)(nsm > 0 ? nsm : 148) * 2);
  mxfp8_quantize_tma_kernel<<<grid, kQThreads, kQtSmem, st>>>(tm, tm_row, tm_col, a, tiles_c, tiles_per_batch,
                                                               ntiles);
  ++g_launch_count;
  return cudaGetLastError();
}

template <typename T, int FMT>
static cudaError_t launch_q(const QuantArgs& a, cudaStream_t st) {
  using Tr = SrcTraits<T>;
  const size_t smem = (size_t)kQTile * 4 * Tr::kBS * sizeof(T);
  cudaError_t e =
      cudaFuncSetAttribute(mxfp8_quantize_kernel<T, FMT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)((a.cols + kQTile - 1) / kQTile), (unsigned)((a.out_rows + kQTile - 1) / kQTile),
            (unsigned)a.batch);
  if (grid.x == 0 || grid.y == 0 || grid.z == 0) return cudaSuccess;
  mxfp8_quantize_kernel<T, FMT><<<grid, kQThreads, smem, st>>>(a);
  ++g_launch_count;
  return cudaGetLastError();
}

// ----------------------------------------------------------------------------- dequantisation
// Rowwise MXFP8 (plain scale layout) -> bf16: value = element(code) * 2^(scale - 127). Each
// thread turns 16 codes (one 16-byte load, within one 32-element block) into 16 bf16. The
// codes decode exactly to fp16 (E4M3 and E5M2 are subsets of it), the power-of-two scaling
// is exact in fp32, and the product rounds once to bf16 -- exact for every block whose
// scale is at least 2^-124 (smaller scales can give values below bf16's subnormal step).
template <int FMT>
__global__ void __launch_bounds__(256) mxfp8_dequant_rows_kernel(const uint4* __restrict__ codes,
                                                                 const uint8_t* __restrict__ scales, int64_t n16,
                                                                 uint4* __restrict__ out) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n16) return;
  const uint4 c = __ldg(codes + i);
  const uint32_t sb = __ldg(scales + (i >> 1));
  const float s = __uint_as_float(sb ? sb << 23 : 0x00400000u);  // 2^(byte - 127) (byte 0: the subnormal 2^-127)
  const uint32_t w[4] = {c.x, c.y, c.z, c.w};
  uint32_t o[8];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w[k] >> (16 * hh)),
                                                        FMT == MXMOE_FMT_E4M3 ? __NV_E4M3 : __NV_E5M2);
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h));
      o[2 * k + hh] = pack_bf16x2(f.x * s, f.y * s);
    }
  }
  out[2 * i] = make_uint4(o[0], o[1], o[2], o[3]);
  out[2 * i + 1] = make_uint4(o[4], o[5], o[6], o[7]);
}

cudaError_t launch_dequantize_rows(const uint8_t* codes, const uint8_t* scales, int64_t rows, int64_t cols, int fmt,
                                   void* out, cudaStream_t st) {
  const int64_t n16 = rows * cols / 16;
  if (n16 == 0) return cudaSuccess;
  const int64_t blocks = (n16 + 255) / 256;
  const uint4* c = reinterpret_cast<const uint4*>(codes);
  uint4* o = reinterpret_cast<uint4*>(out);
  if (fmt == MXMOE_FMT_E5M2) mxfp8_dequant_rows_kernel<MXMOE_FMT_E5M2><<<(unsigned)blocks, 256, 0, st>>>(c, scales, n16, o);
  else mxfp8_dequant_rows_kernel<MXMOE_FMT_E4M3><<<(unsigned)blocks, 256, 0, st>>>(c, scales, n16, o);
  ++g_launch_count;
  return cudaGetLastError();
}

// ----------------------------------------------------------------------------- per-tensor amax
// Largest magnitude of each group (blockIdx.y) of a bf16 array: a grid-stride pass of
// 16-byte loads per group, a SIMD max over the magnitude bits (|bf16| patterns order like
// unsigned integers), a warp max, one atomic per warp on the group's fp32 word (non-negative
// fp32 bit patterns also order like unsigned integers). HBM-bound: n * 2 bytes per group.
__global__ void __launch_bounds__(256) amax_bf16_kernel(const uint4* __restrict__ src, int64_t nvec,
                                                        float* __restrict__ out) {
  const uint4* p = src + (int64_t)blockIdx.y * nvec;
  uint32_t m = 0;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nvec; i += (int64_t)gridDim.x * blockDim.x) {
    const uint4 v = __ldg(p + i);
    m = __vmaxu2(m, v.x & 0x7FFF7FFFu);
    m = __vmaxu2(m, v.y & 0x7FFF7FFFu);
    m = __vmaxu2(m, v.z & 0x7FFF7FFFu);
    m = __vmaxu2(m, v.w & 0x7FFF7FFFu);
  }
  uint32_t am = max(m << 16, m & 0xFFFF0000u);
  am = __reduce_max_sync(0xffffffffu, am);
  if ((threadIdx.x & 31) == 0 && am != 0) atomicMax(reinterpret_cast<unsigned int*>(out + blockIdx.y), am);
}

cudaError_t launch_amax_bf16(const void* src, int64_t n, int32_t groups, float* out, cudaStream_t st) {
  if (n <= 0 || n % 8 != 0 || groups < 1 || groups > 65535) return cudaErrorInvalidValue;
  cudaError_t e = cudaMemsetAsync(out, 0, sizeof(float) * (size_t)groups, st);
  if (e != cudaSuccess) return e;
  const int64_t nvec = n / 8;
  int64_t gx = (int64_t)gemm_num_sms() * 8 / groups;
  const int64_t need = (nvec + 255) / 256;
  gx = gx < 1 ? 1 : (gx > need ? need : gx);
  amax_bf16_kernel<<<dim3((unsigned)gx, (unsigned)groups), 256, 0, st>>>(reinterpret_cast<const uint4*>(src), nvec,
                                                                        out);
  ++g_launch_count;
  return cudaGetLastError();
}

cudaError_t launch_quantize(const QuantArgs& a, cudaStream_t st) {
  if (a.fmt != MXMOE_FMT_E4M3 && a.fmt != MXMOE_FMT_E5M2) return cudaErrorInvalidValue;
  if (a.tensor_amax && a.fmt != MXMOE_FMT_E4M3) return cudaErrorInvalidValue;
  if (qt_applies(a)) return launch_qt(a, st);
  if (a.fmt == MXMOE_FMT_E5M2)
    return a.src_dtype == MXMOE_DTYPE_BF16 ? launch_q<__nv_bfloat16, MXMOE_FMT_E5M2>(a, st)
                                           : launch_q<float, MXMOE_FMT_E5M2>(a, st);
  return a.src_dtype == MXMOE_DTYPE_BF16 ? launch_q<__nv_bfloat16, MXMOE_FMT_E4M3>(a, st)
                                         : launch_q<float, MXMOE_FMT_E4M3>(a, st);
}

}  // namespace mxmoe
