// moe_permute_noalloc: the routing index of moe_permute with its scratch memory held by
// the library instead of passed in by the caller.
//
// Some callers cannot hand the library a scratch buffer: a serving runtime that plans
// every device byte ahead of time and has no free buffer for a helper call, or a plain C
// caller with no device allocator of its own. This entry point needs nothing beyond the
// caller's inputs and outputs: its scratch lives in a fixed-size array in the library's
// device memory (allocated when the library's device code is loaded, kept until exit,
// on every GPU that loads the library).
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "mxmoe_launch.h"

namespace mxmoe {

// Capacity of the scratch array (bytes). moe_permute needs 8 * ceil(T / 256) * E bytes
// (+256), so this covers, e.g., T = 65536 with E = 128, or T = 32768 with E = 256.
constexpr size_t kNoallocScratchBytes = 256 * 1024;

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoallocScratchBytes];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once per device
// (the array's name in host code is only a host-side stand-in, never a device address).
cudaError_t noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) {
      cudaGetLastError();  // clear the runtime's error slot: later calls must not report it
      return e;
    }
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return cudaSuccess;
}
}  // namespace

}  // namespace mxmoe

extern "C" mxmoe_status moe_permute_noalloc(const int32_t* topk_idx_dev, const float* probs_dev, int32_t T,
                                            int32_t k, int32_t E, int32_t* m_splits_dev, int32_t* seg_off_dev,
                                            int32_t* row_of_slot_dev, int32_t* token_of_row_dev,
                                            float* prob_of_row_dev, void* stream) {
  using namespace mxmoe;
  if (T < 0 || k < 1 || k > 8 || E < 1 || E > 256) return MXMOE_ERR_UNSUPPORTED_SHAPE;
  if ((T > 0 && (!topk_idx_dev || !row_of_slot_dev)) || !m_splits_dev || !seg_off_dev || !token_of_row_dev)
    return MXMOE_ERR_INVALID_ARG;
  if (prob_of_row_dev && T > 0 && !probs_dev) return MXMOE_ERR_INVALID_ARG;
  if (route_workspace_bytes(T, k, E) > kNoallocScratchBytes) return MXMOE_ERR_WORKSPACE_TOO_SMALL;
  void* ws = nullptr;
  if (noalloc_scratch(&ws) != cudaSuccess) return MXMOE_ERR_CUDA;
  // Every scratch word the routing kernels read is written earlier in the same call
  // (per-block counts, then per-block bases), so no clearing is needed.
  const cudaError_t e = launch_route(topk_idx_dev, probs_dev, T, k, E, m_splits_dev, seg_off_dev, row_of_slot_dev,
                                     token_of_row_dev, prob_of_row_dev, ws, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MXMOE_OK : MXMOE_ERR_CUDA;
}
