// bitnet_linear_noalloc: BitLinear for callers that must not allocate device
// memory (see include/bitnet.h).  The scratch that bitnet_linear takes from a
// caller workspace lives here in a fixed file-scope device array instead.
#include <mutex>

#include <cuda_runtime.h>

#include "bitnet.h"

namespace {

constexpr size_t kNoAllocScratchBytes = (size_t)BITNET_NOALLOC_SCRATCH_BYTES;

// One copy per device that loads the library, held until the process exits.
// Host code must not use this name as a device address (it is a host-side
// stand-in); the real address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device; resolved once
// per device (with that device current) and cached.
bitnet_status noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BITNET_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return BITNET_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p)
      return BITNET_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return BITNET_OK;
}

}  // namespace

extern "C" bitnet_status bitnet_linear_noalloc(const uint8_t* packed, const float* gamma,
                                               int64_t N, int64_t K, const uint16_t* x,
                                               int64_t M, uint16_t* y, void* stream) {
  if (!packed || !gamma || !x || !y) return BITNET_ERR_INVALID_ARG;
  if (M < 1 || N < 1 || K < 4 || K % 4 != 0 || K > 524288 || M > 0x7fffffff || N > 0x7fffffff)
    return BITNET_ERR_SHAPE;
  // the shape's scratch must fit the fixed array
  if (bitnet_linear_workspace_size(M, N, K) > kNoAllocScratchBytes) return BITNET_ERR_WORKSPACE;
  void* scratch = nullptr;
  const bitnet_status st = noalloc_scratch(&scratch);
  if (st != BITNET_OK) return st;
  return bitnet_linear(packed, gamma, N, K, x, M, y, nullptr, nullptr, scratch,
                       kNoAllocScratchBytes, stream);
}
