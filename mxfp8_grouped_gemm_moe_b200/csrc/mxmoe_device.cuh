// Device-side helpers shared by the library's kernels: the device status word, the
// MXFP8 block quantiser (OCP MX: E4M3 or E5M2 elements, E8M0 power-of-two scale per 32
// values) and the scale-factor layouts.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "../../include/mxmoe.h"

namespace mxmoe {

// Longest time any single wait in a kernel may take before the kernel gives up and
// reports MXMOE_ERR_DEVICE_TIMEOUT (1 s; a healthy wait lasts microseconds).
constexpr uint64_t kWaitLimitNs = 1000000000ull;

// One status word per device (first error wins); read with mxmoe_get_device_status.
// Defined here: the library is built as a single translation unit.
__device__ int32_t g_device_status = 0;
__device__ int32_t g_device_status_where = 0;

__device__ __forceinline__ void record_error(int32_t code, int32_t where) {
  if (atomicCAS(&g_device_status, 0, code) == 0) g_device_status_where = where;
}
__device__ __forceinline__ void record_timeout(int32_t where) { record_error(MXMOE_ERR_DEVICE_TIMEOUT, where); }

// Bounds checks of the checked build (compiled with -DMXMOE_CHECKS=1 into
// libmxmoe_checks.so): an index computed from device data (segment offsets, gathers,
// routing counts) that falls outside [0, n) records MXMOE_ERR_DEVICE_CHECK with the site's
// tag (60..69) and the caller skips the access -- no trap, no out-of-bounds access. The
// release build compiles every check to `true`.
#ifndef MXMOE_CHECKS
#define MXMOE_CHECKS 0
#endif
__device__ __forceinline__ bool check_index(int64_t i, int64_t n, int32_t site) {
#if MXMOE_CHECKS
  if (i < 0 || i >= n) {
    record_error(MXMOE_ERR_DEVICE_CHECK, site);
    return false;
  }
#else
  (void)i;
  (void)n;
  (void)site;
#endif
  return true;
}

// ----------------------------------------------------------------------------- quantiser
// Scale exponent X = clamp(floor(log2(amax)) - emax, -127, 127) from the bit pattern of a
// non-negative fp32 amax (emax = 8 for E4M3 elements, 15 for E5M2); zero or subnormal
// amax gives the lower clamp (-127).
// With ceil_rule the exponent is one higher when amax's significand exceeds 1.75 (both
// formats' largest value is 1.75 * 2^emax): the smallest power-of-two scale under which no
// element saturates.
template <int FMT = MXMOE_FMT_E4M3>
__device__ __forceinline__ int32_t mx_scale_exp_from_amax_bits(uint32_t amax_bits, bool ceil_rule = false) {
  constexpr int32_t kEmax = FMT == MXMOE_FMT_E4M3 ? 8 : 15;  // largest exponent of the element format
  const int32_t ef = (int32_t)((amax_bits >> 23) & 0xFFu);
  if (ef == 0) return -127;
  int32_t X = ef - 127 - kEmax;
  if (ceil_rule && (amax_bits & 0x7FFFFFu) > 0x600000u) ++X;
  return X < -127 ? -127 : (X > 127 ? 127 : X);
}

// 2^-X as an fp32 (X in [-127, 119] for fp32 inputs, so 127 - X is a normal exponent).
__device__ __forceinline__ float mx_inv_scale(int32_t X) {
  return __uint_as_float((uint32_t)(127 - X) << 23);
}

// Two fp32 -> two FP8 codes of the element format (round to nearest even, saturate to
// the largest finite value: +-448 for E4M3, +-57344 for E5M2), low byte = a.
template <int FMT = MXMOE_FMT_E4M3>
__device__ __forceinline__ uint16_t fp8x2(float a, float b) {
  return (uint16_t)__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE,
                                            FMT == MXMOE_FMT_E4M3 ? __NV_E4M3 : __NV_E5M2);
}
__device__ __forceinline__ uint16_t e4m3x2(float a, float b) { return fp8x2<MXMOE_FMT_E4M3>(a, b); }

// Per-tensor FP8: the fp32 multiplier m = 448 / amax, rounded to nearest (IEEE
// division), 1 when amax == 0 and the largest finite fp32 when the quotient overflows. An
// element's code is E4M3(fp32(v * m)).
__device__ __forceinline__ float tensor_multiplier(float amax) {
  if (!(amax > 0.f)) return 1.f;
  return fminf(__fdiv_rn(448.f, amax), 3.40282346638528859812e38f);
}
// Dequantisation factor of a product of two per-tensor operands: 1 / (m_a * m_b).
__device__ __forceinline__ float tensor_alpha(float amax_a, float amax_b) {
  return __frcp_rn(tensor_multiplier(amax_a) * tensor_multiplier(amax_b));
}

// Quantise 32 fp32 values held by one thread -> 32 codes packed in 8 words; returns the
// E8M0 scale byte. tm != 0: per-tensor FP8 under the multiplier tm (scale byte 127).
template <int FMT = MXMOE_FMT_E4M3>
__device__ __forceinline__ uint8_t quant_block32(const float (&v)[32], uint32_t (&out)[8], bool ceil_rule = false,
                                                 float tm = 0.f) {
  int32_t X = 0;
  float s = tm;
  if (tm == 0.f) {
    uint32_t amax = 0;
#pragma unroll
    for (int i = 0; i < 32; ++i) amax = max(amax, __float_as_uint(fabsf(v[i])));
    X = mx_scale_exp_from_amax_bits<FMT>(amax, ceil_rule);
    s = mx_inv_scale(X);
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t lo = fp8x2<FMT>(v[4 * i + 0] * s, v[4 * i + 1] * s);
    const uint32_t hi = fp8x2<FMT>(v[4 * i + 2] * s, v[4 * i + 3] * s);
    out[i] = lo | (hi << 16);
  }
  return (uint8_t)(X + 127);
}

// ----------------------------------------------------------------------------- layouts
// Byte offset of the scale of (row r, 32-column block kb) of a rows x cols matrix.
// PLAIN: row-major [rows, cols/32].
// MMA:   [rows/128][cols/128] chunks of 512 bytes; inside a chunk the scale of row r and
//        block kb (mod 4) sits at (r%32)*16 + ((r/32)%4)*4 + kb%4, i.e. 32 rows of 16
//        bytes, the layout the tensor core's scale-factor copy into TMEM expects.
__host__ __device__ __forceinline__ int64_t sf_offset(int32_t layout, int64_t rows, int64_t cols, int64_t r,
                                                      int64_t kb) {
  if (layout == MXMOE_SCALE_PLAIN) return r * (cols / 32) + kb;
  const int64_t chunk = (r >> 7) * (cols >> 7) + (kb >> 2);
  return chunk * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (kb & 3);
  (void)rows;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);  // .x = a (low half)
  return *reinterpret_cast<uint32_t*>(&h);
}

}  // namespace mxmoe
