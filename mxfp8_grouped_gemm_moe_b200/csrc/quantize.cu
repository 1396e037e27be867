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
template <>
struct SrcTraits<__nv_bfloat16> {
  static constexpr int kPad = 8;  // elements of row padding in shared memory (16 bytes)
  static constexpr int kVec = 8;  // elements per 16-byte vector
};
template <>
struct SrcTraits<float> {
  static constexpr int kPad = 4;
  static constexpr int kVec = 4;
};

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

// 16-byte asynchronous global -> shared copy (zero-filled when src_bytes == 0).
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"((uint32_t)__cvta_generic_to_shared(smem)),
               "l"(gmem), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

// Persistent over 128 x 128 tiles (tile t: batch, row tile, column tile), two shared
// buffers: tile t+1 is in flight while tile t is quantised.
template <typename T>
__global__ void __launch_bounds__(kQThreads) mxfp8_quantize_kernel(QuantArgs a) {
  using Tr = SrcTraits<T>;
  constexpr int LD = kQTile + Tr::kPad;
  constexpr int VPR = kQTile / Tr::kVec;        // 16-byte vectors per tile row
  constexpr int NL = kQTile * VPR / kQThreads;  // vectors per thread
  constexpr int RSTEP = kQThreads / VPR;        // tile rows between a thread's vectors
  extern __shared__ __align__(16) uint8_t q_smem_raw[];
  T* bufs[2] = {reinterpret_cast<T*>(q_smem_raw), reinterpret_cast<T*>(q_smem_raw) + kQTile * LD};

  int64_t nvalid = a.out_rows;
  if (a.nrows) {
    const int64_t nv = *a.nrows;
    nvalid = nv < nvalid ? nv : nvalid;
  }
  const int64_t ct = (a.cols + kQTile - 1) / kQTile;
  const int64_t rt = (nvalid + kQTile - 1) / kQTile;   // row tiles that hold valid rows
  const int64_t ntiles = a.batch * rt * ct;
  const T* src = reinterpret_cast<const T*>(a.src);
  const int row_t = threadIdx.x / VPR, cv = threadIdx.x % VPR;

  auto issue = [&](int64_t tile, T* dst) {
    const int64_t b = tile / (rt * ct), rem = tile % (rt * ct);
    const int64_t r0 = (rem / ct) * kQTile, c0 = (rem % ct) * kQTile;
    const int64_t col = c0 + (int64_t)cv * Tr::kVec;
#pragma unroll
    for (int k = 0; k < NL; ++k) {
      const int64_t orow = r0 + row_t + k * RSTEP;
      int64_t srow = -1;
      if (orow < nvalid && col < a.cols) srow = a.gather ? (int64_t)__ldg(a.gather + orow) : b * a.rows + orow;
      const T* g = srow >= 0 ? src + srow * a.cols + col : src;
      cp_async16(dst + (row_t + k * RSTEP) * LD + cv * Tr::kVec, g, srow >= 0 ? 16u : 0u);
    }
  };

  int64_t tile = blockIdx.x;
  if (tile < ntiles) issue(tile, bufs[0]);
  cp_async_commit();
  for (int it = 0; tile < ntiles; ++it, tile += gridDim.x) {
    T* cur = bufs[it & 1];
    if (tile + gridDim.x < ntiles) issue(tile + gridDim.x, bufs[(it + 1) & 1]);
    cp_async_commit();
    cp_async_wait_1();
    __syncthreads();

    const int64_t b = tile / (rt * ct), rem = tile % (rt * ct);
    const int64_t r0 = (rem / ct) * kQTile, c0 = (rem % ct) * kQTile;
    // ---- rowwise: item = (32-column block, row); a warp takes 32 consecutive rows of one
    // block, so its 16-byte shared loads hit distinct banks (row stride = 4 banks mod 32)
    if (a.row_data) {
#pragma unroll 1
      for (int i2 = threadIdx.x; i2 < kQTile * 4; i2 += kQThreads) {
        const int row = i2 & (kQTile - 1), blk = i2 >> 7;
        const int64_t orow = r0 + row;
        const int64_t col = c0 + 32 * blk;
        if (orow >= nvalid || col >= a.cols) continue;
        float v[32];
        load32_row(cur + row * LD + 32 * blk, v);
        uint32_t q[8];
        const uint8_t sb = quant_block32(v, q);
        const int64_t grow = b * a.out_rows + orow;
        uint4* dst = reinterpret_cast<uint4*>(a.row_data + grow * a.cols + col);
        dst[0] = make_uint4(q[0], q[1], q[2], q[3]);
        dst[1] = make_uint4(q[4], q[5], q[6], q[7]);
        a.row_sf[sf_offset(a.row_layout, a.batch * a.out_rows, a.cols, grow, col / 32)] = sb;
      }
    }
    // ---- colwise: item = (column, 32-row block); a warp reads 32 consecutive columns of
    // a row per load (conflict free); stored transposed
    if (a.col_data) {
#pragma unroll 1
      for (int i2 = threadIdx.x; i2 < kQTile * 4; i2 += kQThreads) {
        const int cc = i2 & (kQTile - 1), rb = i2 >> 7;
        const int64_t col = c0 + cc;
        const int64_t orow = r0 + 32 * rb;
        if (orow >= nvalid || col >= a.cols) continue;
        float v[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = to_f32(cur[(32 * rb + i) * LD + cc]);
        uint32_t q[8];
        const uint8_t sb = quant_block32(v, q);
        const int64_t grow = b * a.cols + col;  // row of the transposed matrix
        uint4* dst = reinterpret_cast<uint4*>(a.col_data + grow * a.out_rows + orow);
        dst[0] = make_uint4(q[0], q[1], q[2], q[3]);
        dst[1] = make_uint4(q[4], q[5], q[6], q[7]);
        a.col_sf[sf_offset(a.col_layout, a.batch * a.cols, a.out_rows, grow, orow / 32)] = sb;
      }
    }
    __syncthreads();  // `cur` is refilled two tiles from now
  }
}

template <typename T>
static cudaError_t launch_q(const QuantArgs& a, cudaStream_t st) {
  using Tr = SrcTraits<T>;
  const size_t smem = 2 * (size_t)kQTile * (kQTile + Tr::kPad) * sizeof(T);
  cudaError_t e =
      cudaFuncSetAttribute(mxfp8_quantize_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int64_t tiles = a.batch * ((a.out_rows + kQTile - 1) / kQTile) * ((a.cols + kQTile - 1) / kQTile);
  if (tiles == 0) return cudaSuccess;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, mxfp8_quantize_kernel<T>, kQThreads, smem);
  if (e != cudaSuccess) return e;
  const int64_t grid = std::min<int64_t>(tiles, (int64_t)gemm_num_sms() * std::max(per_sm, 1));
  mxfp8_quantize_kernel<T><<<(unsigned)grid, kQThreads, smem, st>>>(a);
  ++g_launch_count;
  return cudaGetLastError();
}

cudaError_t launch_quantize(const QuantArgs& a, cudaStream_t st) {
  if (a.src_dtype == MXMOE_DTYPE_BF16) return launch_q<__nv_bfloat16>(a, st);
  return launch_q<float>(a, st);
}

}  // namespace mxmoe
