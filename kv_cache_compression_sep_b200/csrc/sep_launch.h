// Host-side interface between the C-ABI layer (api.cpp) and the kernel launchers (*.cu).
// Plain C++ types only; every pointer is a device pointer owned by the caller.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/sepattn.h"

namespace sep {

// Launch with programmatic stream serialisation: the kernel may start while the previous kernel
// of the stream finishes (it waits for it in grid_dep_wait before touching global memory), so
// that its launch and prologue overlap the other's tail. Every kernel of the library's training
// and decode steps is started this way.
template <typename... KArgs, typename... Args>
cudaError_t launch_chained(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                           cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// Device address of the sticky error word on the current device (nullptr on failure).
unsigned* device_error_word();
// Wall-clock limit of each pipeline wait of the attention forward kernel (sep_set_wait_limit_ns);
// by default the same 1.5 s as every other bounded wait.
constexpr unsigned long long kDefaultPipelineWaitNs = 1500ull * 1000ull * 1000ull;
unsigned long long pipeline_wait_limit_ns();
// Fixed scratch of sep_attn_fwd_noalloc on the current device (first call per device: setup).
void* noalloc_fwd_scratch(cudaError_t* err);

cudaError_t launch_mask_build(const uint8_t* sep, int B, int L, int a, int n, int bm, int bn,
                              int32_t* anchor_idx, int32_t* anchor_cnt, uint32_t* anchor_bits,
                              int32_t* gather_end, int8_t* tile_map, int64_t* kept,
                              cudaStream_t stream);

// Stage bits of launch_attn_bwd.
constexpr int kBwdPrep = 1, kBwdDq = 2, kBwdDkv = 4, kBwdAll = 7;

// Copies the K/V rows of every anchor to rows 0..anchor_cnt[b]-1 of kc/vc ([B, L, Hkv, d]).
cudaError_t launch_compact_anchors(const void* k, const void* v, const int32_t* anchor_idx,
                                   const int32_t* anchor_cnt, int B, int L, int Hkv, int d,
                                   void* kc, void* vc, cudaStream_t stream);

struct AttnMaps {
  CUtensorMap q, k, v, kc, vc;  // 4-D {d, H, L, B}, box {64, 1, 128, 1}, 128-byte swizzle
  CUtensorMap o, dout, dq, dk, dv;  // O store (forward); dO load, dQ/dK/dV stores (backward)
  CUtensorMap k64, v64, kc64, vc64;  // the same tensors with 64-row boxes (forward half tiles)
};

struct AttnShape {
  int B, L, Hq, Hkv, d, a, n;
  float scale;
};

cudaError_t launch_attn_fwd(const AttnMaps& maps, const AttnShape& s, const uint32_t* anchor_bits,
                            const int32_t* gather_end, const int8_t* tile_map, void* o,
                            float* lse, cudaStream_t stream);

cudaError_t launch_attn_bwd(const AttnMaps& maps, const AttnShape& s, const uint32_t* anchor_bits,
                            const int32_t* anchor_idx, const int32_t* anchor_cnt,
                            const int32_t* gather_end, const int8_t* tile_map, const void* o,
                            const float* lse, const void* dout, const void* q, const void* k,
                            const void* v, void* dq, void* dk, void* dv, void* kc, void* vc,
                            float* delta, float* dka, float* dva, void* sched, int stages,
                            cudaStream_t stream);

// Bytes of the backward work-list region inside the workspace.
size_t bwd_sched_bytes(int B, int L);

cudaError_t launch_sepcache_init(const SepCacheState& st, cudaStream_t stream);
cudaError_t launch_sepcache_update(const SepCacheState& st, const void* k_new,
                                   const void* v_new, const uint8_t* sep_new,
                                   cudaStream_t stream);
cudaError_t launch_sepcache_prefill(const SepCacheState& st, const void* k, const void* v,
                                    const uint8_t* sep, int L, cudaStream_t stream);
cudaError_t launch_sepcache_decode(const SepCacheState& st, const void* q, void* o, float* lse,
                                   float scale, cudaStream_t stream);
cudaError_t launch_sepcache_export(const SepCacheState& st, int32_t* pos_out, int32_t* count,
                                   cudaStream_t stream);

}  // namespace sep
