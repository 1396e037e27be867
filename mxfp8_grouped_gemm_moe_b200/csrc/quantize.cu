// MXFP8 quantisation of activations and weights, rowwise and colwise from one read,
// optionally fused with the expert permutation (row gather).
//
// "MoE-Training für biologische Grundmodelle optimieren" (hyper.ai/de), MXFP8 passage:
// 8-bit values with one scale per block of 32; GroupedMLP passage: the 16-bit -> 8-bit
// conversions are fused rather than run as separate operations. Element / scale rule:
// OCP MX (E4M3 elements, E8M0 scale, X = clamp(floor(log2 amax) - 8, -127, 127),
// round-to-nearest-even with saturation).
//
// One CTA quantises a 128 x 128 tile staged in shared memory: rowwise blocks (32
// consecutive columns of a row) and colwise blocks (32 consecutive rows of a column,
// written transposed) come from the same HBM read. Loads and stores are 16-byte
// vectors; a warp's rowwise / colwise stores cover whole 32-byte sectors.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "mxmoe_device.cuh"
#include "mxmoe_launch.h"

namespace mxmoe {

constexpr int kQTile = 128;
constexpr int kQThreads = 256;

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

// MXFP8 of 32 bf16 values given as 16 packed words (element 2k in the low half of w[k],
// 2k+1 in the high half). |bf16| bit patterns order like unsigned 16-bit integers, so
// the block amax is a SIMD max over the masked words; the result equals the amax of the
// values widened to fp32 (widening is exact), hence the same scale as quant_block32.
__device__ __forceinline__ uint8_t quant_block32_bf16(const uint32_t (&w)[16], uint32_t (&out)[8]) {
  uint32_t m = 0;
#pragma unroll
  for (int i = 0; i < 16; ++i) m = __vmaxu2(m, w[i] & 0x7FFF7FFFu);
  const uint32_t amax = max(m << 16, m & 0xFFFF0000u);
  const int32_t X = mx_scale_exp_from_amax_bits(amax);
  const float s = mx_inv_scale(X);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t lo = e4m3x2(bf16_lo(w[2 * i]) * s, bf16_hi(w[2 * i]) * s);
    const uint32_t hi = e4m3x2(bf16_lo(w[2 * i + 1]) * s, bf16_hi(w[2 * i + 1]) * s);
    out[i] = lo | (hi << 16);
  }
  return (uint8_t)(X + 127);
}

// Colwise MXFP8 of two adjacent columns over 32 rows: w[r] holds (column c, row r) in
// its low half and (column c+1, row r) in its high half.
__device__ __forceinline__ void quant_colpair_bf16(const uint32_t (&w)[32], uint32_t (&o0)[8], uint32_t (&o1)[8],
                                                   uint8_t& sb0, uint8_t& sb1) {
  uint32_t m = 0;
#pragma unroll
  for (int i = 0; i < 32; ++i) m = __vmaxu2(m, w[i] & 0x7FFF7FFFu);
  const int32_t X0 = mx_scale_exp_from_amax_bits(m << 16);
  const int32_t X1 = mx_scale_exp_from_amax_bits(m & 0xFFFF0000u);
  const float s0 = mx_inv_scale(X0), s1 = mx_inv_scale(X1);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    o0[i] = (uint32_t)e4m3x2(bf16_lo(w[4 * i]) * s0, bf16_lo(w[4 * i + 1]) * s0) |
            ((uint32_t)e4m3x2(bf16_lo(w[4 * i + 2]) * s0, bf16_lo(w[4 * i + 3]) * s0) << 16);
    o1[i] = (uint32_t)e4m3x2(bf16_hi(w[4 * i]) * s1, bf16_hi(w[4 * i + 1]) * s1) |
            ((uint32_t)e4m3x2(bf16_hi(w[4 * i + 2]) * s1, bf16_hi(w[4 * i + 3]) * s1) << 16);
  }
  sb0 = (uint8_t)(X0 + 127);
  sb1 = (uint8_t)(X1 + 127);
}

template <typename T>
__device__ __forceinline__ uint8_t quant_row_block(const T* p, uint32_t (&q)[8]);
template <>
__device__ __forceinline__ uint8_t quant_row_block<__nv_bfloat16>(const __nv_bfloat16* p, uint32_t (&q)[8]) {
  uint32_t w[16];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 v = reinterpret_cast<const uint4*>(p)[i];
    w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
  }
  return quant_block32_bf16(w, q);
}
template <>
__device__ __forceinline__ uint8_t quant_row_block<float>(const float* p, uint32_t (&q)[8]) {
  float v[32];
  load32_row(p, v);
  return quant_block32(v, q);
}

template <typename T>
__device__ __forceinline__ void quant_col_pair(const T* p, int ld, uint32_t (&q0)[8], uint32_t (&q1)[8], uint8_t& s0,
                                               uint8_t& s1);
template <>
__device__ __forceinline__ void quant_col_pair<__nv_bfloat16>(const __nv_bfloat16* p, int ld, uint32_t (&q0)[8],
                                                              uint32_t (&q1)[8], uint8_t& s0, uint8_t& s1) {
  uint32_t w[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) w[i] = *reinterpret_cast<const uint32_t*>(p + i * ld);
  quant_colpair_bf16(w, q0, q1, s0, s1);
}
template <>
__device__ __forceinline__ void quant_col_pair<float>(const float* p, int ld, uint32_t (&q0)[8], uint32_t (&q1)[8],
                                                      uint8_t& s0, uint8_t& s1) {
  float v[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = p[i * ld];
  s0 = quant_block32(v, q0);
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = p[i * ld + 1];
  s1 = quant_block32(v, q1);
}

// One CTA per 128 x 128 tile (many resident per SM to overlap load latency).
template <typename T>
__global__ void __launch_bounds__(kQThreads, sizeof(T) == 2 ? 4 : 2) mxfp8_quantize_kernel(QuantArgs a) {
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

  // ---- load the tile (gathered rows, zero outside the matrix / for pad rows); all of a
  // thread's row indices, then all of its 16-byte loads, are issued before any use
  constexpr int VPR = kQTile / Tr::kVec;        // vectors per tile row
  constexpr int NL = kQTile * VPR / kQThreads;  // vectors per thread
  constexpr int RSTEP = kQThreads / VPR;        // tile rows between a thread's vectors
  const int row_t = threadIdx.x / VPR, cv = threadIdx.x % VPR;
  {
    const int64_t col = c0 + (int64_t)cv * Tr::kVec;
    int64_t srow[NL];
#pragma unroll
    for (int k = 0; k < NL; ++k) {
      const int64_t orow = r0 + row_t + k * RSTEP;
      srow[k] = -1;
      if (orow < nvalid && col < a.cols) srow[k] = a.gather ? (int64_t)__ldg(a.gather + orow) : b * a.rows + orow;
    }
    uint4 buf[NL];
#pragma unroll
    for (int k = 0; k < NL; ++k)
      buf[k] = srow[k] >= 0 ? __ldg(reinterpret_cast<const uint4*>(src + srow[k] * a.cols + col))
                            : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int k = 0; k < NL; ++k)
      *reinterpret_cast<uint4*>(tile + tile_off<T>(row_t + k * RSTEP, cv * Tr::kVec)) = buf[k];
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
      const uint8_t sb = quant_row_block<T>(tile + tile_off<T>(row, 32 * blk), q);
      int64_t drow = orow;
      if (a.row_ilv > 0) {  // gate / up interleave of the fc1 operand
        const int64_t hf = orow >= a.row_ilv, rr = orow - hf * a.row_ilv;
        drow = (rr >> 6) * 128 + hf * 64 + (rr & 63);
      }
      const int64_t grow = b * a.out_rows + drow;
      uint4* dst = reinterpret_cast<uint4*>(a.row_data + grow * a.cols + col);
      dst[0] = make_uint4(q[0], q[1], q[2], q[3]);
      dst[1] = make_uint4(q[4], q[5], q[6], q[7]);
      a.row_sf[sf_offset(a.row_layout, a.batch * a.out_rows, a.cols, grow, col / 32)] = sb;
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
      quant_col_pair<T>(tile + tile_off<T>(32 * rb, 2 * pcol), 4 * Tr::kBS, q0, q1, s0, s1);
      const int64_t grow = b * a.cols + col;  // row of the transposed matrix
      uint4* d0 = reinterpret_cast<uint4*>(a.col_data + grow * a.out_rows + orow);
      uint4* d1 = reinterpret_cast<uint4*>(a.col_data + (grow + 1) * a.out_rows + orow);
      d0[0] = make_uint4(q0[0], q0[1], q0[2], q0[3]);
      d0[1] = make_uint4(q0[4], q0[5], q0[6], q0[7]);
      d1[0] = make_uint4(q1[0], q1[1], q1[2], q1[3]);
      d1[1] = make_uint4(q1[4], q1[5], q1[6], q1[7]);
      a.col_sf[sf_offset(a.col_layout, a.batch * a.cols, a.out_rows, grow, orow / 32)] = s0;
      a.col_sf[sf_offset(a.col_layout, a.batch * a.cols, a.out_rows, grow + 1, orow / 32)] = s1;
    }
  }
}

template <typename T>
static cudaError_t launch_q(const QuantArgs& a, cudaStream_t st) {
  using Tr = SrcTraits<T>;
  const size_t smem = (size_t)kQTile * 4 * Tr::kBS * sizeof(T);
  cudaError_t e =
      cudaFuncSetAttribute(mxfp8_quantize_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)((a.cols + kQTile - 1) / kQTile), (unsigned)((a.out_rows + kQTile - 1) / kQTile),
            (unsigned)a.batch);
  if (grid.x == 0 || grid.y == 0 || grid.z == 0) return cudaSuccess;
  mxfp8_quantize_kernel<T><<<grid, kQThreads, smem, st>>>(a);
  ++g_launch_count;
  return cudaGetLastError();
}

cudaError_t launch_quantize(const QuantArgs& a, cudaStream_t st) {
  if (a.src_dtype == MXMOE_DTYPE_BF16) return launch_q<__nv_bfloat16>(a, st);
  return launch_q<float>(a, st);
}

}  // namespace mxmoe
