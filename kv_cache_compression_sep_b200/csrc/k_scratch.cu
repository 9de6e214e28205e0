// Fixed device scratch behind sep_attn_fwd_noalloc: a file-scope __device__ array in this
// module's image, so that the call needs no buffer from its caller and no allocation. The array
// only holds the compacted anchor K / V that the forward workspace would otherwise hold.
#include <cuda_runtime.h>

#include <atomic>

#include "../../include/sepattn.h"
#include "sep_launch.h"

namespace sep {

static __device__ __align__(256) unsigned char g_fwd_scratch[SEP_NOALLOC_SCRATCH_BYTES];

// Device address of the array on the current device. The first call per device looks it up
// (cudaGetSymbolAddress also loads this module there); later calls reuse the cached address.
void* noalloc_fwd_scratch(cudaError_t* err) {
  static std::atomic<void*> cache[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    *err = e;
    return nullptr;
  }
  const bool cached = dev >= 0 && dev < 64;
  void* p = cached ? cache[dev].load(std::memory_order_acquire) : nullptr;
  if (!p) {
    e = cudaGetSymbolAddress(&p, g_fwd_scratch);
    if (e != cudaSuccess || !p) {
      *err = (e != cudaSuccess) ? e : cudaErrorInvalidSymbol;
      return nullptr;
    }
    if (cached) cache[dev].store(p, std::memory_order_release);
  }
  *err = cudaSuccess;
  return p;
}

}  // namespace sep
