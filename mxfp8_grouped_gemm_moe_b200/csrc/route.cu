// Routing index (counting sort of (token, slot) pairs by expert, stable by token),
// combine (unpermute + sum of the k copies) and the routing-probability gradient
// reduction.
//
// "MoE-Training für biologische Grundmodelle optimieren" (hyper.ai/de), GroupedLinear
// passage: the expert matrices are gathered from per-expert token counts. Order of rows
// within an expert and the 256-row segment alignment are this library's reading.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "mxmoe_device.cuh"
#include "mxmoe_launch.h"

namespace mxmoe {

constexpr int kRouteTokensPerBlock = 256;
constexpr int kMaxExperts = 256;
constexpr int kMaxTopK = 8;
constexpr int kSegAlign = 256;  // expert segments start at multiples of the GEMM's 256-row tile

// Pass 1: per-block expert histogram; validates ids (out of range or repeated within a
// token -> device check error, pair dropped).
__global__ void __launch_bounds__(kRouteTokensPerBlock) route_count_kernel(const int32_t* __restrict__ idx, int T,
                                                                           int k, int E,
                                                                           int32_t* __restrict__ block_counts) {
  __shared__ int32_t cnt[kMaxExperts];
  for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  const int t = blockIdx.x * kRouteTokensPerBlock + threadIdx.x;
  if (t < T) {
    int32_t mine[kMaxTopK];
    for (int j = 0; j < k; ++j) mine[j] = idx[(int64_t)t * k + j];
    for (int j = 0; j < k; ++j) {
      const int32_t e = mine[j];
      bool ok = (e >= 0 && e < E);
      for (int i = 0; i < j; ++i) ok = ok && (mine[i] != e);
      if (ok) {
        atomicAdd(&cnt[e], 1);
      } else {
        record_error(MXMOE_ERR_DEVICE_CHECK, 100);
      }
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) block_counts[(int64_t)blockIdx.x * E + e] = cnt[e];
}

// Pass 2 (one block): m_splits, 256-aligned segment offsets, per-(block, expert) base
// rows; marks pad rows (token -1, prob 0).
__global__ void __launch_bounds__(1024) route_scan_kernel(const int32_t* __restrict__ block_counts, int nblocks,
                                                          int E, int32_t* __restrict__ block_base,
                                                          int32_t* __restrict__ m_splits,
                                                          int32_t* __restrict__ seg_off,
                                                          int32_t* __restrict__ token_of_row,
                                                          float* __restrict__ prob_of_row) {
  __shared__ int32_t s_m[kMaxExperts];
  __shared__ int32_t s_off[kMaxExperts + 1];
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int32_t s = 0;
    for (int b = 0; b < nblocks; ++b) s += block_counts[(int64_t)b * E + e];
    s_m[e] = s;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int32_t o = 0;
    for (int e = 0; e < E; ++e) {
      s_off[e] = o;
      o += (s_m[e] + kSegAlign - 1) / kSegAlign * kSegAlign;
    }
    s_off[E] = o;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    m_splits[e] = s_m[e];
    int32_t base = s_off[e];
    for (int b = 0; b < nblocks; ++b) {
      block_base[(int64_t)b * E + e] = base;
      base += block_counts[(int64_t)b * E + e];
    }
  }
  for (int e = threadIdx.x; e <= E; e += blockDim.x) seg_off[e] = s_off[e];
  // pad rows of every segment
  for (int e = 0; e < E; ++e) {
    const int32_t p0 = s_off[e] + s_m[e], p1 = s_off[e + 1];
    for (int r = p0 + threadIdx.x; r < p1; r += blockDim.x) {
      token_of_row[r] = -1;
      if (prob_of_row) prob_of_row[r] = 0.f;
    }
  }
}

// Pass 3: stable scatter. Rank of token t among this block's tokens routed to expert e
// = number of earlier tokens of the block whose top-k contains e (bitmask popcount).
__global__ void __launch_bounds__(kRouteTokensPerBlock) route_scatter_kernel(
    const int32_t* __restrict__ idx, const float* __restrict__ probs, int T, int k, int E,
    const int32_t* __restrict__ block_base, int32_t* __restrict__ row_of_slot, int32_t* __restrict__ token_of_row,
    float* __restrict__ prob_of_row, int64_t cap) {
  constexpr int W = kRouteTokensPerBlock / 32;
  __shared__ uint32_t mask[kMaxExperts * W];
  for (int i = threadIdx.x; i < E * W; i += blockDim.x) mask[i] = 0u;
  __syncthreads();
  const int t = blockIdx.x * kRouteTokensPerBlock + threadIdx.x;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int32_t mine[kMaxTopK];
  bool valid[kMaxTopK];
  if (t < T) {
    for (int j = 0; j < k; ++j) mine[j] = idx[(int64_t)t * k + j];
    for (int j = 0; j < k; ++j) {
      const int32_t e = mine[j];
      bool ok = (e >= 0 && e < E);
      for (int i = 0; i < j; ++i) ok = ok && (mine[i] != e);
      valid[j] = ok;
      if (ok) atomicOr(&mask[e * W + w], 1u << lane);
    }
  }
  __syncthreads();
  if (t < T) {
    for (int j = 0; j < k; ++j) {
      if (!valid[j]) {
        row_of_slot[(int64_t)t * k + j] = -1;
        continue;
      }
      const int32_t e = mine[j];
      int32_t rank = __popc(mask[e * W + w] & ((1u << lane) - 1u));
      for (int ww = 0; ww < w; ++ww) rank += __popc(mask[e * W + ww]);
      const int32_t row = block_base[(int64_t)blockIdx.x * E + e] + rank;
      const bool in = check_index(row, cap, 68);  // checked build: inside the row buffers
      row_of_slot[(int64_t)t * k + j] = in ? row : -1;
      if (!in) continue;
      token_of_row[row] = t;
      if (prob_of_row) prob_of_row[row] = probs[(int64_t)t * k + j];
    }
  }
}

// y[t] = sum_j y_perm[row_of_slot[t, j]] (fp32 in slot order, bf16 out). One block per
// token; each thread issues the loads of all k routed rows of its vector before the first
// sum (KMAX >= k slots, unrouted ones skipped), VW 16-byte words per vector: 2 (256-bit
// loads and stores) when both buffers are 32-byte aligned, else 1.
template <int KMAX, int VW>
__global__ void __launch_bounds__(256) unpermute_kernel(const uint4* __restrict__ yp, const int32_t* __restrict__ ros,
                                                        int T, int k, int H, uint4* __restrict__ y) {
  const int t = blockIdx.x;
  const int nvec = H / (8 * VW);
  int32_t rows[KMAX];
#pragma unroll
  for (int j = 0; j < KMAX; ++j) rows[j] = j < k ? __ldg(ros + (int64_t)t * k + j) : -1;
  for (int v = threadIdx.x; v < nvec; v += blockDim.x) {
    uint4 q[KMAX][VW];
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      if (rows[j] < 0) continue;
      const uint4* p = yp + ((int64_t)rows[j] * nvec + v) * VW;
      if constexpr (VW == 2) {
        asm volatile("ld.global.nc.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                     : "=r"(q[j][0].x), "=r"(q[j][0].y), "=r"(q[j][0].z), "=r"(q[j][0].w), "=r"(q[j][1].x),
                       "=r"(q[j][1].y), "=r"(q[j][1].z), "=r"(q[j][1].w)
                     : "l"(p));
      } else {
        q[j][0] = __ldg(p);
      }
    }
    float acc[8 * VW];
#pragma unroll
    for (int i = 0; i < 8 * VW; ++i) acc[i] = 0.f;
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      if (rows[j] < 0) continue;
#pragma unroll
      for (int w = 0; w < VW; ++w) {
        float* a = acc + 8 * w;
        a[0] += bf16_lo(q[j][w].x); a[1] += bf16_hi(q[j][w].x);
        a[2] += bf16_lo(q[j][w].y); a[3] += bf16_hi(q[j][w].y);
        a[4] += bf16_lo(q[j][w].z); a[5] += bf16_hi(q[j][w].z);
        a[6] += bf16_lo(q[j][w].w); a[7] += bf16_hi(q[j][w].w);
      }
    }
    uint32_t o[4 * VW];
#pragma unroll
    for (int i = 0; i < 4 * VW; ++i) o[i] = pack_bf16x2(acc[2 * i], acc[2 * i + 1]);
    uint4* d = y + ((int64_t)t * nvec + v) * VW;
    if constexpr (VW == 2) {
      asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(d), "r"(o[0]), "r"(o[1]),
                   "r"(o[2]), "r"(o[3]), "r"(o[4]), "r"(o[5]), "r"(o[6]), "r"(o[7])
                   : "memory");
    } else {
      *d = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
}

// dprobs[t, j] = sum over p of part[row, p], row = row_of_slot[t, j]. G lanes per (t, j):
// lane l of the group adds partials l, l + G, ... in order (coalesced reads), then the G
// lane sums are combined by a fixed butterfly, so the result is deterministic. Every lane
// of a warp takes part in the shuffles; groups past n add nothing and store nothing.
template <int G>
__global__ void __launch_bounds__(256) dprob_reduce_kernel(const float* __restrict__ part, int nparts,
                                                           const int32_t* __restrict__ ros, int64_t n,
                                                           float* __restrict__ dprobs) {
  const int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / G;
  const int sub = threadIdx.x & (G - 1);
  float s = 0.f;
  if (i < n) {
    const int32_t row = ros[i];
    if (row >= 0)
      for (int p = sub; p < nparts; p += G) s += part[(int64_t)row * nparts + p];
  }
#pragma unroll
  for (int o = G / 2; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (i < n && sub == 0) dprobs[i] = s;
}

// ----------------------------------------------------------------------------- launchers
size_t route_workspace_bytes(int T, int k, int E) {
  (void)k;
  const int64_t nb = ((int64_t)T + kRouteTokensPerBlock - 1) / kRouteTokensPerBlock;
  return (size_t)(2 * std::max<int64_t>(nb, 1) * E * sizeof(int32_t)) + 256;
}

cudaError_t launch_route(const int32_t* idx, const float* probs, int T, int k, int E, int32_t* m_splits,
                         int32_t* seg_off, int32_t* row_of_slot, int32_t* token_of_row, float* prob_of_row,
                         void* ws, cudaStream_t st) {
  const int nb = (T + kRouteTokensPerBlock - 1) / kRouteTokensPerBlock;
  const int nbl = nb > 0 ? nb : 1;
  int32_t* counts = reinterpret_cast<int32_t*>(ws);
  int32_t* base = counts + (int64_t)nbl * E;
  if (nb == 0) cudaMemsetAsync(counts, 0, sizeof(int32_t) * E, st);
  else route_count_kernel<<<nb, kRouteTokensPerBlock, 0, st>>>(idx, T, k, E, counts);
  route_scan_kernel<<<1, 1024, 0, st>>>(counts, nbl, E, base, m_splits, seg_off, token_of_row, prob_of_row);
  if (nb > 0)
    route_scatter_kernel<<<nb, kRouteTokensPerBlock, 0, st>>>(idx, probs, T, k, E, base, row_of_slot, token_of_row,
                                                              prob_of_row, rows_cap(T, k, E));
  g_launch_count += (nb > 0) ? 3 : 1;
  return cudaGetLastError();
}

cudaError_t launch_unpermute(const void* yp, const int32_t* ros, int T, int k, int H, void* y, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  const bool v32 = H % 16 == 0 && (reinterpret_cast<uintptr_t>(yp) & 31) == 0 && (reinterpret_cast<uintptr_t>(y) & 31) == 0;
  const int nvec = H / (v32 ? 16 : 8);
  const int threads = std::min(256, std::max(32, (nvec + 31) / 32 * 32));
  const uint4* src = reinterpret_cast<const uint4*>(yp);
  uint4* dst = reinterpret_cast<uint4*>(y);
#define MXMOE_UNPERMUTE(KM)                                                               \
  do {                                                                                    \
    if (v32) unpermute_kernel<KM, 2><<<T, threads, 0, st>>>(src, ros, T, k, H, dst);      \
    else unpermute_kernel<KM, 1><<<T, threads, 0, st>>>(src, ros, T, k, H, dst);          \
  } while (0)
  if (k <= 1) MXMOE_UNPERMUTE(1);
  else if (k <= 2) MXMOE_UNPERMUTE(2);
  else if (k <= 4) MXMOE_UNPERMUTE(4);
  else MXMOE_UNPERMUTE(kMaxTopK);
#undef MXMOE_UNPERMUTE
  ++g_launch_count;
  return cudaGetLastError();
}

cudaError_t launch_dprob_reduce(const float* part, int nparts, const int32_t* ros, int64_t n, float* dprobs,
                                cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  // a warp per output for long partial rows, a quarter warp for short ones
  if (nparts >= 96)
    dprob_reduce_kernel<32><<<(unsigned)((n * 32 + 255) / 256), 256, 0, st>>>(part, nparts, ros, n, dprobs);
  else
    dprob_reduce_kernel<8><<<(unsigned)((n * 8 + 255) / 256), 256, 0, st>>>(part, nparts, ros, n, dprobs);
  ++g_launch_count;
  return cudaGetLastError();
}

}  // namespace mxmoe
