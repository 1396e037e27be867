// Router: softmax over all experts, top-k selection, and its backward.
//
// "MoE-Training für biologische Grundmodelle optimieren" (hyper.ai/de), routing passage:
// a router assigns every token to its experts ahead of the expert MLP. Readings (the
// pages give no formula): probabilities are a softmax over all E experts (not
// renormalised over the selected k); the k largest are selected in descending order,
// equal logits keep the lower expert index first (softmax is monotone, so the selection
// is made on the fp32 logits themselves, exactly); -inf marks an expert a token may not
// use.
//
// One warp per token, E <= 256: lane l holds the logits of experts l, l + 32, ... in
// registers; max, sum and the k argmax rounds are warp shuffles. The kernels read the
// logits once (T * E * 4 bytes) and write T * k * 8 bytes (forward) or T * E * 4 bytes
// (backward): latency-bound for small E, bandwidth-bound for large E.
#include <cuda_runtime.h>

#include <cstdint>

#include "mxmoe_device.cuh"
#include "mxmoe_launch.h"

namespace mxmoe {

constexpr int kRouterWarps = 8;  // tokens per 256-thread block

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Loads token t's logits (lane-strided), returns false (warp-uniform) unless the row has
// a finite maximum and no NaN; m = max, s = sum of exp(l - m).
template <int EPL>
__device__ __forceinline__ bool load_softmax(const float* logits, int64_t t, int E, int lane, float (&v)[EPL],
                                             float& m, float& s) {
  const float* row = logits + t * E;
  bool nan = false;
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    const int e = lane + 32 * i;
    v[i] = e < E ? row[e] : -INFINITY;
    nan |= v[i] != v[i];
  }
  float lm = -INFINITY;
#pragma unroll
  for (int i = 0; i < EPL; ++i) lm = fmaxf(lm, v[i]);
  m = warp_max(lm);
  if (__any_sync(0xffffffffu, nan) || !(m > -INFINITY && m < INFINITY)) return false;
  float ls = 0.f;
#pragma unroll
  for (int i = 0; i < EPL; ++i) ls += expf(v[i] - m);
  s = warp_sum(ls);
  return true;
}

template <int EPL>
__global__ void __launch_bounds__(32 * kRouterWarps)
    router_topk_kernel(const float* __restrict__ logits, int T, int E, int k, int32_t* __restrict__ idx,
                       float* __restrict__ probs) {
  const int lane = threadIdx.x & 31;
  const int64_t t = (int64_t)blockIdx.x * kRouterWarps + (threadIdx.x >> 5);
  if (t >= T) return;
  float v[EPL], m, s;
  if (!load_softmax<EPL>(logits, t, E, lane, v, m, s)) {
    if (lane == 0) record_error(MXMOE_ERR_DEVICE_CHECK, 40);
    if (lane < k) {
      idx[t * k + lane] = -1;
      probs[t * k + lane] = 0.f;
    }
    return;
  }
  uint32_t taken = 0;
  for (int j = 0; j < k; ++j) {
    // this lane's best untaken expert: larger logit, then lower index
    float bv = -INFINITY;
    int be = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int e = lane + 32 * i;
      if (e < E && !((taken >> i) & 1u) && (v[i] > bv || (v[i] == bv && e < be))) {
        bv = v[i];
        be = e;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oe = __shfl_xor_sync(0xffffffffu, be, o);
      if (ov > bv || (ov == bv && oe < be)) {
        bv = ov;
        be = oe;
      }
    }
    if ((be & 31) == lane) taken |= 1u << (be >> 5);
    if (lane == 0) {
      idx[t * k + j] = be;
      probs[t * k + j] = expf(bv - m) / s;
    }
  }
}

template <int EPL>
__global__ void __launch_bounds__(32 * kRouterWarps)
    router_topk_bwd_kernel(const float* __restrict__ logits, const int32_t* __restrict__ idx,
                           const float* __restrict__ dprobs, int T, int E, int k, float* __restrict__ dlogits) {
  const int lane = threadIdx.x & 31;
  const int64_t t = (int64_t)blockIdx.x * kRouterWarps + (threadIdx.x >> 5);
  if (t >= T) return;
  float v[EPL], m, s;
  if (!load_softmax<EPL>(logits, t, E, lane, v, m, s)) {
    if (lane == 0) record_error(MXMOE_ERR_DEVICE_CHECK, 41);
    return;
  }
  // g[e] = upstream gradient of the selected probability of expert e (0 if unselected)
  float g[EPL];
#pragma unroll
  for (int i = 0; i < EPL; ++i) g[i] = 0.f;
  for (int j = 0; j < k; ++j) {
    const int e = idx[t * k + j];
    const float d = dprobs[t * k + j];
    if (e < 0 || e >= E) {
      if (lane == 0) record_error(MXMOE_ERR_DEVICE_CHECK, 42);
      continue;
    }
#pragma unroll
    for (int i = 0; i < EPL; ++i)
      if (lane + 32 * i == e) g[i] += d;
  }
  // dl_e = P_e (g_e - sum_i g_i P_i)
  const float inv = 1.0f / s;
  float p[EPL], gp = 0.f;
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    p[i] = expf(v[i] - m) * inv;
    gp += g[i] * p[i];
  }
  gp = warp_sum(gp);
  float* out = dlogits + t * E;
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    const int e = lane + 32 * i;
    if (e < E) out[e] = p[i] * (g[i] - gp);
  }
}

cudaError_t launch_router_topk(const float* logits, int T, int E, int k, int32_t* idx, float* probs,
                               cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  const dim3 grid((unsigned)((T + kRouterWarps - 1) / kRouterWarps)), block(32 * kRouterWarps);
  if (E <= 32) router_topk_kernel<1><<<grid, block, 0, st>>>(logits, T, E, k, idx, probs);
  else if (E <= 64) router_topk_kernel<2><<<grid, block, 0, st>>>(logits, T, E, k, idx, probs);
  else if (E <= 128) router_topk_kernel<4><<<grid, block, 0, st>>>(logits, T, E, k, idx, probs);
  else router_topk_kernel<8><<<grid, block, 0, st>>>(logits, T, E, k, idx, probs);
  ++g_launch_count;
  return cudaGetLastError();
}

cudaError_t launch_router_topk_bwd(const float* logits, const int32_t* idx, const float* dprobs, int T, int E, int k,
                                   float* dlogits, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  const dim3 grid((unsigned)((T + kRouterWarps - 1) / kRouterWarps)), block(32 * kRouterWarps);
  if (E <= 32) router_topk_bwd_kernel<1><<<grid, block, 0, st>>>(logits, idx, dprobs, T, E, k, dlogits);
  else if (E <= 64) router_topk_bwd_kernel<2><<<grid, block, 0, st>>>(logits, idx, dprobs, T, E, k, dlogits);
  else if (E <= 128) router_topk_bwd_kernel<4><<<grid, block, 0, st>>>(logits, idx, dprobs, T, E, k, dlogits);
  else router_topk_bwd_kernel<8><<<grid, block, 0, st>>>(logits, idx, dprobs, T, E, k, dlogits);
  ++g_launch_count;
  return cudaGetLastError();
}

}  // namespace mxmoe
