// Persistent MXFP8 grouped GEMM for sm_100a (tcgen05 block-scaled MMA, TMEM
// accumulators, TMA operand loads), with the fused epilogues of the expert MLP.
//
// "MoE-Training für biologische Grundmodelle optimieren" (hyper.ai/de): GroupedLinear
// runs every expert's GEMM in one call driven by per-expert token counts; Blackwell
// tensor cores run MXFP8 natively; the GroupedMLP kernel fuses the gate-up projection,
// the ScaledSwiGLU activation and the routing-weight scaling, forward and backward,
// without keeping the intermediates in memory. "NVIDIA apresenta técnicas ...
// arquitetura MoE" (conexaotc.com.br) adds that quantisation is part of that fusion.
//
// Design (B200):
//  * one CTA per SM, persistent over a linear tile list; expert segments are 128-row
//    aligned, so an M tile never straddles two experts and its expert is found from
//    the device-side segment offsets (no host synchronisation on m_splits);
//  * tile 128 x 256 x 128 (M x N x K), 4-stage TMA -> shared-memory ring; operand
//    tiles use the 128-byte swizzle; the E8M0 scales arrive with plain bulk copies in
//    the tensor cores' scale order and are moved to TMEM with tcgen05.cp;
//  * warp 0 issues the copies, warp 1 issues tcgen05.mma (kind::mxf8f6f4, block32
//    scales), warps 2..9 are the epilogue: they drain the 128 x 256 fp32 accumulator
//    from TMEM into registers, hand TMEM back to the MMA warp at once, then run the
//    epilogue math and stores while the next tile's MMAs proceed;
//  * every wait is bounded (1 s) and reports MXMOE_ERR_DEVICE_TIMEOUT instead of
//    hanging; no cluster, no multicast.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <cstring>
#include <mutex>

#include "mxmoe_device.cuh"
#include "mxmoe_launch.h"
#include "ptx_sm100.cuh"

namespace mxmoe {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 128;
#ifndef MXMOE_STAGES
#define MXMOE_STAGES 4
#endif
constexpr int STAGES = MXMOE_STAGES;
constexpr int kThreads = 320;  // 10 warps
constexpr int kEpiWarps = 8;

constexpr uint32_t kABytes = BM * BK;       // 16 KB
constexpr uint32_t kBBytes = BN * BK;       // 32 KB
constexpr uint32_t kSfaBytes = 512;         // 128 rows x 4 scale bytes
constexpr uint32_t kSfbBytes = 1024;        // 256 rows x 4 scale bytes
constexpr uint32_t kStageBytes = 51200;     // A + B + SFA + SFB, padded to 1 KB
constexpr uint32_t kTxBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes;
constexpr uint32_t kStagingPerWarp = 2048;  // colwise transpose staging
constexpr uint32_t kOffStaging = STAGES * kStageBytes;
constexpr uint32_t kOffBars = kOffStaging + kEpiWarps * kStagingPerWarp;
constexpr int kMaxE = 256;
constexpr uint32_t kOffSeg = kOffBars + 256;
constexpr uint32_t kOffOrder = kOffSeg + (kMaxE + 1) * 4 + 12;
constexpr uint32_t kSmemUsed = kOffOrder + kMaxE * 4;
constexpr uint32_t kSmemBytes = kSmemUsed + 1024;  // slack for 1 KB alignment
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemSfa = 256;  // two buffers of 4 columns
constexpr uint32_t kTmemSfb = 264;  // two buffers of 8 columns
constexpr uint32_t kTmemStash = 384;  // epilogue scratch: 64 columns per (lane quadrant, half)
constexpr int GROUP_M = 16;         // m tiles per raster group (L2 reuse of B)

static_assert(kStageBytes >= kTxBytes && kStageBytes % 1024 == 0, "stage layout");
static_assert(kSmemBytes <= 232448, "shared memory budget");

struct TileInfo {
  int32_t e;
  int32_t k_iters;
  int32_t a_y, a_x0;
  int32_t b_y0, b_y1, b_x0;
  int32_t n_tile;
  int64_t row0;  // output row base
};

template <int MODE>
__device__ __forceinline__ int32_t n_tiles_of(const GemmArgs& g) {
  if (MODE == kModeStore) return (int32_t)(g.N / BN);
  if (MODE == kModeSwigluFwd) return (int32_t)(g.F / 128);
  if (MODE == kModeSwigluBwd) return (int32_t)(g.F / BN);
  return (int32_t)((g.N / BM) * (g.K2 / BN));  // per expert, wgrad
}

template <int MODE>
__device__ __forceinline__ int64_t total_tiles(const GemmArgs& g, const int32_t* s_seg) {
  if (MODE == kModeWgrad) return (int64_t)g.E * n_tiles_of<MODE>(g);
  return (int64_t)(s_seg[g.E] / BM) * n_tiles_of<MODE>(g);
}

template <int MODE>
__device__ __forceinline__ TileInfo get_tile(const GemmArgs& g, int64_t idx, const int32_t* s_seg,
                                             const int32_t* s_order) {
  TileInfo t;
  if (MODE == kModeWgrad) {
    const int32_t per = n_tiles_of<MODE>(g);
    const int32_t nk2 = (int32_t)(g.K2 / BN);
    const int32_t pos = (int32_t)(idx / per), r = (int32_t)(idx % per);
    const int32_t e = s_order[pos];
    const int32_t n_t = r / nk2, k2_t = r % nk2;
    t.e = e;
    t.k_iters = (s_seg[e + 1] - s_seg[e]) / BK;
    t.a_y = n_t * BM;
    t.a_x0 = s_seg[e];
    t.b_y0 = k2_t * BN;
    t.b_y1 = t.b_y0 + 128;
    t.b_x0 = s_seg[e];
    t.n_tile = k2_t;
    t.row0 = (int64_t)e * g.N + (int64_t)n_t * BM;
    return t;
  }
  const int32_t ntn = n_tiles_of<MODE>(g);
  const int32_t num_m = s_seg[g.E] / BM;
  const int64_t group_size = (int64_t)GROUP_M * ntn;
  const int32_t grp = (int32_t)(idx / group_size);
  const int32_t r = (int32_t)(idx % group_size);
  const int32_t m0 = grp * GROUP_M;
  const int32_t gm = min(GROUP_M, num_m - m0);
  const int32_t m_t = m0 + r % gm;
  const int32_t n_t = r / gm;
  const int32_t row = m_t * BM;
  // expert = the e with s_seg[e] <= row < s_seg[e+1] (segments of empty experts have
  // zero length and are skipped by the search)
  int32_t lo = 0, hi = g.E - 1;
  while (lo < hi) {
    const int32_t mid = (lo + hi) >> 1;
    if (s_seg[mid + 1] > row) hi = mid;
    else lo = mid + 1;
  }
  const int32_t e = lo;
  t.e = e;
  t.k_iters = (int32_t)(g.K / BK);
  t.a_y = row;
  t.a_x0 = 0;
  t.b_x0 = 0;
  t.n_tile = n_t;
  t.row0 = row;
  if (MODE == kModeSwigluFwd) {
    t.b_y0 = (int32_t)(e * 2 * g.F + (int64_t)n_t * 128);
    t.b_y1 = (int32_t)(e * 2 * g.F + g.F + (int64_t)n_t * 128);
  } else {
    t.b_y0 = (int32_t)((int64_t)e * g.N + (int64_t)n_t * BN);
    t.b_y1 = t.b_y0 + 128;
  }
  return t;
}

// Logistic function from the hardware tanh: s(x) = (1 + tanh(x/2)) / 2 -- one special-
// function-unit op and no division (the epilogues are bound by that unit). Its error
// (about 2^-11 relative to 1) sits far below the E4M3 rounding that follows.
__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float sigmoid_f(float x) { return fmaf(0.5f, tanh_approx(0.5f * x), 0.5f); }
__device__ __forceinline__ float silu_f(float x) { return x * sigmoid_f(x); }

// Warp-wide colwise MXFP8 of a 32 x 32 fp32 block held one row per lane (lane = row,
// v[i] = column i): blocks of 32 rows of one column, written transposed (column i ->
// 32 consecutive bytes at dst + i*ld) with one scale byte per column.
// The block is transposed through the warp's 2 KB staging buffer in two rounds of 16
// columns. Staging layout (fp32 words): row r = 16*h + i (i < 16) lives in line i (32
// words), half h; its four 16-byte chunks are XOR-swizzled by (i & 7), so both the
// row-wise 16-byte stores and the column-wise 4-byte loads are bank-conflict free.
// After the transpose, lane (c = lane % 16, h = lane / 16) holds rows [16h, 16h+16) of
// column c; the two halves combine their amax with one shuffle.
__device__ __forceinline__ void colwise_quant_store(const float (&v)[32], float* stg, int lane, uint8_t* dst,
                                                    int64_t ld, uint8_t* sf_base, int64_t sf_rows, int64_t sf_cols,
                                                    int64_t col_row0, int64_t kb) {
  const int wi = lane & 15, wh = lane >> 4;  // this lane's row as (line, half) when writing
  const int c = lane & 15, rh = lane >> 4;   // column and row half this lane reads
#pragma unroll
  for (int r = 0; r < 2; ++r) {
#pragma unroll
    for (int qd = 0; qd < 4; ++qd) {
      const int phys = ((wh << 2) | qd) ^ (wi & 7);
      *reinterpret_cast<float4*>(stg + wi * 32 + phys * 4) =
          make_float4(v[16 * r + 4 * qd], v[16 * r + 4 * qd + 1], v[16 * r + 4 * qd + 2], v[16 * r + 4 * qd + 3]);
    }
    __syncwarp();
    float w[16];
    uint32_t amax = 0;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int phys = ((rh << 2) | (c >> 2)) ^ (j & 7);
      w[j] = stg[j * 32 + phys * 4 + (c & 3)];
      amax = max(amax, __float_as_uint(fabsf(w[j])));
    }
    __syncwarp();
    amax = max(amax, __shfl_xor_sync(0xffffffffu, amax, 16));
    const int32_t X = mx_scale_exp_from_amax_bits(amax);
    const float sc = mx_inv_scale(X);
    uint32_t q[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t lo = e4m3x2(w[4 * i] * sc, w[4 * i + 1] * sc);
      const uint32_t hi = e4m3x2(w[4 * i + 2] * sc, w[4 * i + 3] * sc);
      q[i] = lo | (hi << 16);
    }
    const int col = 16 * r + c;
    *reinterpret_cast<uint4*>(dst + (int64_t)col * ld + 16 * rh) = make_uint4(q[0], q[1], q[2], q[3]);
    if (rh == 0) sf_base[sf_offset(MXMOE_SCALE_MMA, sf_rows, sf_cols, col_row0 + col, kb)] = (uint8_t)(X + 127);
  }
}

__device__ __forceinline__ void rowwise_quant_store(const float (&v)[32], uint8_t* dst, uint8_t* sf, int64_t rows,
                                                    int64_t cols, int64_t row, int64_t kb) {
  uint32_t q[8];
  const uint8_t sb = quant_block32(v, q);
  uint4* d = reinterpret_cast<uint4*>(dst);
  d[0] = make_uint4(q[0], q[1], q[2], q[3]);
  d[1] = make_uint4(q[4], q[5], q[6], q[7]);
  sf[sf_offset(MXMOE_SCALE_MMA, rows, cols, row, kb)] = sb;
}

// Hands the accumulator back to the MMA warp once this warp's TMEM reads (and writes
// to its spare columns) have completed.
__device__ __forceinline__ void release_accumulator(uint64_t* bar_acc_empty, int lane) {
  ptx::tc_fence_before();
  __syncwarp();
  if (lane == 0) ptx::mbar_arrive(bar_acc_empty);
}

// 8 fp32 (bit patterns) starting at v[i0] -> 8 bf16 in one 16-byte vector.
template <int N>
__device__ __forceinline__ uint4 pack8_bf16(const uint32_t (&v)[N], int i0) {
  uint4 o;
  o.x = pack_bf16x2(__uint_as_float(v[i0 + 0]), __uint_as_float(v[i0 + 1]));
  o.y = pack_bf16x2(__uint_as_float(v[i0 + 2]), __uint_as_float(v[i0 + 3]));
  o.z = pack_bf16x2(__uint_as_float(v[i0 + 4]), __uint_as_float(v[i0 + 5]));
  o.w = pack_bf16x2(__uint_as_float(v[i0 + 6]), __uint_as_float(v[i0 + 7]));
  return o;
}

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    mxgemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                  const __grid_constant__ GemmArgs g) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bar_full = reinterpret_cast<uint64_t*>(smem + kOffBars);
  uint64_t* bar_empty = bar_full + STAGES;
  uint64_t* bar_acc_full = bar_empty + STAGES;
  uint64_t* bar_acc_empty = bar_acc_full + 1;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bar_acc_empty + 1);
  volatile int32_t* s_abort = reinterpret_cast<volatile int32_t*>(s_tmem + 1);
  int32_t* s_seg = reinterpret_cast<int32_t*>(smem + kOffSeg);
  int32_t* s_order = reinterpret_cast<int32_t*>(smem + kOffOrder);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- setup
  for (int i = threadIdx.x; i <= g.E; i += blockDim.x) s_seg[i] = g.seg_off[i];
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      ptx::mbar_init(&bar_full[s], 1);
      ptx::mbar_init(&bar_empty[s], 1);
    }
    ptx::mbar_init(bar_acc_full, 1);
    ptx::mbar_init(bar_acc_empty, kEpiWarps);
    *s_abort = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    ptx::prefetch_tensormap(&tmA);
    ptx::prefetch_tensormap(&tmB);
  }
  if (warp == 1) {
    ptx::tmem_alloc(s_tmem, kTmemCols);
    ptx::tmem_relinquish();
  }
  __syncthreads();
  if (MODE == kModeWgrad) {
    // experts in decreasing size (largest first), ties by index
    for (int e = threadIdx.x; e < g.E; e += blockDim.x) {
      const int32_t me = s_seg[e + 1] - s_seg[e];
      int32_t rank = 0;
      for (int f = 0; f < g.E; ++f) {
        const int32_t mf = s_seg[f + 1] - s_seg[f];
        rank += (mf > me) || (mf == me && f < e);
      }
      s_order[rank] = e;
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = *s_tmem;
  const int64_t ntiles = total_tiles<MODE>(g, s_seg);

  if (warp == 0) {
    // ===================================================== TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t ph = 0;
      const int64_t a_kchunks = g.a_cols / 128, b_kchunks = g.b_cols / 128;
      for (int64_t tile = blockIdx.x; tile < ntiles && !*s_abort; tile += gridDim.x) {
        const TileInfo t = get_tile<MODE>(g, tile, s_seg, s_order);
        for (int kb = 0; kb < t.k_iters; ++kb) {
          if (!ptx::mbar_wait(&bar_empty[stage], ph ^ 1u, 1)) {
            *s_abort = 1;
            break;
          }
          uint8_t* sb = smem + stage * kStageBytes;
          ptx::mbar_arrive_expect_tx(&bar_full[stage], kTxBytes);
          const int32_t kx_a = t.a_x0 + kb * BK, kx_b = t.b_x0 + kb * BK;
          ptx::tma_load_2d(sb, &tmA, kx_a, t.a_y, &bar_full[stage]);
          ptx::tma_load_2d(sb + kABytes, &tmB, kx_b, t.b_y0, &bar_full[stage]);
          ptx::tma_load_2d(sb + kABytes + kBBytes / 2, &tmB, kx_b, t.b_y1, &bar_full[stage]);
          const int64_t ca = (int64_t)(t.a_y / 128) * a_kchunks + kx_a / 128;
          const int64_t cb0 = (int64_t)(t.b_y0 / 128) * b_kchunks + kx_b / 128;
          const int64_t cb1 = (int64_t)(t.b_y1 / 128) * b_kchunks + kx_b / 128;
          ptx::bulk_load(sb + kABytes + kBBytes, g.a_sf + ca * 512, 512, &bar_full[stage]);
          ptx::bulk_load(sb + kABytes + kBBytes + kSfaBytes, g.b_sf + cb0 * 512, 512, &bar_full[stage]);
          ptx::bulk_load(sb + kABytes + kBBytes + kSfaBytes + 512, g.b_sf + cb1 * 512, 512, &bar_full[stage]);
          if (++stage == STAGES) {
            stage = 0;
            ph ^= 1u;
          }
        }
      }
    }
  } else if (warp == 1) {
    // ===================================================== MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t ph = 0, acc_ph = 0;
      bool dropped = false;
      for (int64_t tile = blockIdx.x; tile < ntiles && !*s_abort; tile += gridDim.x) {
        const TileInfo t = get_tile<MODE>(g, tile, s_seg, s_order);
        if (t.k_iters == 0) continue;
        if (!ptx::mbar_wait(bar_acc_empty, acc_ph ^ 1u, 2)) {
          *s_abort = 1;
          break;
        }
        ptx::tc_fence_after();
        bool ok = true;
        for (int kb = 0; kb < t.k_iters; ++kb) {
          if (!ptx::mbar_wait(&bar_full[stage], ph, 3)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t sbase = ptx::smem_u32(smem + stage * kStageBytes);
          const uint32_t buf = (uint32_t)(stage & 1);
          const uint32_t t_sfa = tmem_base + kTmemSfa + buf * 4;
          const uint32_t t_sfb = tmem_base + kTmemSfb + buf * 8;
          const uint32_t sfa_s = sbase + kABytes + kBBytes;
          ptx::tmem_cp_32x128b_warpx4(t_sfa, ptx::make_smem_desc(sfa_s, 0, 128, ptx::kLayoutSwizzleNone));
          ptx::tmem_cp_32x128b_warpx4(t_sfb, ptx::make_smem_desc(sfa_s + kSfaBytes, 0, 128, ptx::kLayoutSwizzleNone));
          ptx::tmem_cp_32x128b_warpx4(t_sfb + 4,
                                      ptx::make_smem_desc(sfa_s + kSfaBytes + 512, 0, 128, ptx::kLayoutSwizzleNone));
          const uint64_t adesc = ptx::make_smem_desc(sbase, 16, 1024, ptx::kLayoutSwizzle128B);
          const uint64_t bdesc = ptx::make_smem_desc(sbase + kABytes, 16, 1024, ptx::kLayoutSwizzle128B);
#pragma unroll
          for (int kk = 0; kk < BK / 32; ++kk) {
            const uint32_t idesc = ptx::make_idesc_mxf8(BM, BN, (uint32_t)kk, (uint32_t)kk);
            ptx::mma_mxf8(tmem_base, adesc + (uint64_t)(2 * kk), bdesc + (uint64_t)(2 * kk), idesc, t_sfa, t_sfb,
                          (kb | kk) != 0 ? 1u : 0u);
          }
          ptx::tc_commit(&bar_empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            ph ^= 1u;
          }
        }
        if (!ok) {
          *s_abort = 1;
          break;
        }
        if (g.debug_drop_commit && !dropped && blockIdx.x == 0) {
          dropped = true;  // withhold the signal (timeout-path test)
        } else {
          ptx::tc_commit(bar_acc_full);
        }
        acc_ph ^= 1u;
      }
    }
  } else {
    // ===================================================== epilogue warps 2..9
    const int ew = warp - 2;
    const int q = warp & 3;  // TMEM lane quadrant this warp may access
    const int h = ew >> 2;   // column half
    float* stg = reinterpret_cast<float*>(smem + kOffStaging + ew * kStagingPerWarp);
    uint32_t acc_ph = 0;
    const uint32_t t_lane = tmem_base + ((uint32_t)(32 * q) << 16);
    const uint32_t t_stash = t_lane + kTmemStash + 64 * h;  // this warp's 64 spare TMEM columns
    for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
      // warp-uniform abort check (the TMEM loads below are warp-collective)
      if (__any_sync(0xffffffffu, *s_abort != 0)) break;
      const TileInfo t = get_tile<MODE>(g, tile, s_seg, s_order);
      const int64_t mrow0 = t.row0 + 32 * q;  // first row of this warp's 32-row block
      const int64_t row = mrow0 + lane;
      const bool have_acc = t.k_iters > 0;
      if (have_acc) {
        const bool ok = ptx::mbar_wait(bar_acc_full, acc_ph, 4);
        if (!__all_sync(0xffffffffu, ok)) {
          *s_abort = 1;
          break;
        }
        __syncwarp();
        acc_ph ^= 1u;
        ptx::tc_fence_after();
      }

      if (MODE == kModeStore || MODE == kModeWgrad) {
        uint32_t acc[128];
        if (have_acc) {
#pragma unroll
          for (int c = 0; c < 4; ++c)
            ptx::tmem_ld_32x32b_x32(t_lane + 128 * h + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&acc[32 * c]));
          ptx::tmem_wait_ld();
          release_accumulator(bar_acc_empty, lane);
        } else {
#pragma unroll
          for (int i = 0; i < 128; ++i) acc[i] = 0u;
        }
        const int64_t col0 = (int64_t)t.n_tile * BN + 128 * h;
        if (MODE == kModeWgrad || g.c_dtype == MXMOE_DTYPE_F32) {
          float* c = reinterpret_cast<float*>(g.c) + row * g.ldc + col0;
#pragma unroll
          for (int i = 0; i < 32; ++i)
            reinterpret_cast<uint4*>(c)[i] = make_uint4(acc[4 * i], acc[4 * i + 1], acc[4 * i + 2], acc[4 * i + 3]);
        } else {
          uint16_t* c = reinterpret_cast<uint16_t*>(g.c) + row * g.ldc + col0;
#pragma unroll
          for (int i = 0; i < 16; ++i) reinterpret_cast<uint4*>(c)[i] = pack8_bf16(acc, 8 * i);
        }
      } else if (MODE == kModeSwigluFwd) {
        const int64_t F = g.F, F2 = 2 * g.F;
        const float p = g.prob_of_row[row];
        const int64_t f0 = (int64_t)t.n_tile * 128 + 64 * h;  // this warp's 64 Z columns
        // phase 1 (the MMA warp waits for it): drain gate / up (TMEM columns [64h, +64) and
        // [128 + 64h, +64)), keep them as packed bf16 for the backward's saved copy, form
        // Z = silu(G) * U * p in fp32 and park Z in this warp's spare TMEM columns
        uint4 gsave[8], usave[8];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t gr[32], ur[32];
          ptx::tmem_ld_32x32b_x32(t_lane + 64 * h + 32 * c, gr);
          ptx::tmem_ld_32x32b_x32(t_lane + 128 + 64 * h + 32 * c, ur);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            gsave[4 * c + i] = pack8_bf16(gr, 8 * i);
            usave[4 * c + i] = pack8_bf16(ur, 8 * i);
          }
#pragma unroll
          for (int i = 0; i < 32; ++i)
            gr[i] = __float_as_uint(silu_f(__uint_as_float(gr[i])) * __uint_as_float(ur[i]) * p);
          ptx::tmem_st_32x32b_x16(t_stash + 32 * c, *reinterpret_cast<uint32_t(*)[16]>(&gr[0]));
          ptx::tmem_st_32x32b_x16(t_stash + 32 * c + 16, *reinterpret_cast<uint32_t(*)[16]>(&gr[16]));
        }
        ptx::tmem_wait_st();
        release_accumulator(bar_acc_empty, lane);
        {
          uint4* gd = reinterpret_cast<uint4*>(g.gu + row * F2 + f0);
          uint4* ud = reinterpret_cast<uint4*>(g.gu + row * F2 + F + f0);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            gd[i] = gsave[i];
            ud[i] = usave[i];
          }
        }
        // phase 2: MXFP8 of Z, rowwise (fc2 operand) and colwise (fc2 weight-gradient operand)
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
          uint32_t zr[32];
          ptx::tmem_ld_32x32b_x32(t_stash + 32 * c, zr);
          ptx::tmem_wait_ld();
          float z[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) z[i] = __uint_as_float(zr[i]);
          const int64_t fc = f0 + 32 * c;
          rowwise_quant_store(z, g.z_row + row * F + fc, g.z_row_sf, g.rows_cap, F, row, fc / 32);
          colwise_quant_store(z, stg, lane, g.z_colT + fc * g.rows_cap + mrow0, g.rows_cap, g.z_colT_sf, F,
                              g.rows_cap, fc, mrow0 / 32);
        }
      } else if (MODE == kModeSwigluBwd) {
        const int64_t F = g.F, F2 = 2 * g.F;
        const float p = g.prob_of_row[row];
        const int64_t f0 = (int64_t)t.n_tile * BN + 128 * h;  // this warp's 128 dZ columns
        // phase 1: drain dZ, park it in TMEM as packed bf16 pairs (the E4M3 rounding that
        // follows is 2^5 coarser than that rounding)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t tmp[32], pk[16];
          ptx::tmem_ld_32x32b_x32(t_lane + 128 * h + 32 * c, tmp);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(__uint_as_float(tmp[2 * i]), __uint_as_float(tmp[2 * i + 1]));
          ptx::tmem_st_32x32b_x16(t_stash + 16 * c, pk);
        }
        ptx::tmem_wait_st();
        release_accumulator(bar_acc_empty, lane);
        // phase 2: SwiGLU / probability backward, 32 columns at a time; G and U of the next
        // chunk are fetched while this one is processed
        const uint4* gsrc = reinterpret_cast<const uint4*>(g.gu_in + row * F2 + f0);
        const uint4* usrc = reinterpret_cast<const uint4*>(g.gu_in + row * F2 + F + f0);
        uint4 gq[4], uq[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          gq[i] = gsrc[i];
          uq[i] = usrc[i];
        }
        float dprob = 0.f;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t dzw[16];
          ptx::tmem_ld_32x32b_x16(t_stash + 16 * c, dzw);
          const uint32_t gw[16] = {gq[0].x, gq[0].y, gq[0].z, gq[0].w, gq[1].x, gq[1].y, gq[1].z, gq[1].w,
                                   gq[2].x, gq[2].y, gq[2].z, gq[2].w, gq[3].x, gq[3].y, gq[3].z, gq[3].w};
          const uint32_t uw[16] = {uq[0].x, uq[0].y, uq[0].z, uq[0].w, uq[1].x, uq[1].y, uq[1].z, uq[1].w,
                                   uq[2].x, uq[2].y, uq[2].z, uq[2].w, uq[3].x, uq[3].y, uq[3].z, uq[3].w};
          if (c < 3) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              gq[i] = gsrc[4 * (c + 1) + i];
              uq[i] = usrc[4 * (c + 1) + i];
            }
          }
          ptx::tmem_wait_ld();
          float vg[32], vu[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float gg = (i & 1) ? bf16_hi(gw[i >> 1]) : bf16_lo(gw[i >> 1]);
            const float uu = (i & 1) ? bf16_hi(uw[i >> 1]) : bf16_lo(uw[i >> 1]);
            const float dz = (i & 1) ? bf16_hi(dzw[i >> 1]) : bf16_lo(dzw[i >> 1]);
            const float sg = sigmoid_f(gg);                  // sigmoid(G)
            const float sl = gg * sg;                        // silu(G)
            const float da = dz * p;                         // dA = dZ * p
            dprob += dz * sl * uu;                           // dprob += dZ * A
            vg[i] = da * uu * (sg * (1.0f + gg * (1.0f - sg)));
            vu[i] = da * sl;
          }
          const int64_t fg = f0 + 32 * c;
          rowwise_quant_store(vg, g.dgu_row + row * F2 + fg, g.dgu_row_sf, g.rows_cap, F2, row, fg / 32);
          colwise_quant_store(vg, stg, lane, g.dgu_colT + fg * g.rows_cap + mrow0, g.rows_cap, g.dgu_colT_sf, F2,
                              g.rows_cap, fg, mrow0 / 32);
          rowwise_quant_store(vu, g.dgu_row + row * F2 + F + fg, g.dgu_row_sf, g.rows_cap, F2, row, (F + fg) / 32);
          colwise_quant_store(vu, stg, lane, g.dgu_colT + (F + fg) * g.rows_cap + mrow0, g.rows_cap,
                              g.dgu_colT_sf, F2, g.rows_cap, F + fg, mrow0 / 32);
        }
        g.dprob_part[row * (F / 128) + t.n_tile * 2 + h] = dprob;
      }
    }
  }

  // ---- teardown: every role has finished issuing; the epilogue has drained the last
  // accumulator, so every MMA has completed before TMEM is released.
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem_base, kTmemCols);
  }
}

// ----------------------------------------------------------------------------- host side
static PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D uint8 tensor map over a row-major [rows, cols] matrix, box 128 x 128, 128-byte swizzle.
static bool make_map(CUtensorMap* m, const void* base, int64_t rows, int64_t cols) {
  auto fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols};
  cuuint32_t box[2] = {128, 128};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int gemm_num_sms() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

template <int MODE>
static cudaError_t launch_mode(const CUtensorMap& ma, const CUtensorMap& mb, const GemmArgs& g, int64_t tiles_ub,
                               cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(mxgemm_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  const int nsm = gemm_num_sms();
  const int grid = (int)(tiles_ub < nsm ? (tiles_ub > 0 ? tiles_ub : 1) : nsm);
  mxgemm_kernel<MODE><<<grid, kThreads, kSmemBytes, st>>>(ma, mb, g);
  ++g_launch_count;
  return cudaGetLastError();
}

cudaError_t launch_gemm(const GemmArgs& g, cudaStream_t st) {
  CUtensorMap ma, mb;
  if (!make_map(&ma, g.a_data, g.a_rows, g.a_cols) || !make_map(&mb, g.b_data, g.b_rows, g.b_cols))
    return cudaErrorInvalidValue;
  int64_t tiles_ub;
  switch (g.mode) {
    case kModeStore:
      tiles_ub = (g.a_rows / BM) * (g.N / BN);
      return launch_mode<kModeStore>(ma, mb, g, tiles_ub, st);
    case kModeSwigluFwd:
      tiles_ub = (g.a_rows / BM) * (g.F / 128);
      return launch_mode<kModeSwigluFwd>(ma, mb, g, tiles_ub, st);
    case kModeSwigluBwd:
      tiles_ub = (g.a_rows / BM) * (g.F / BN);
      return launch_mode<kModeSwigluBwd>(ma, mb, g, tiles_ub, st);
    case kModeWgrad:
      tiles_ub = (int64_t)g.E * (g.N / BM) * (g.K2 / BN);
      return launch_mode<kModeWgrad>(ma, mb, g, tiles_ub, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace mxmoe
