// C ABI of libsepattn.so: argument validation, workspace layout, TMA descriptor encoding and
// kernel launch. See include/sepattn.h for the contract of every entry point.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstring>

#include "../../include/sepattn.h"
#include "sep_launch.h"

namespace sep {
static std::atomic<unsigned long long> g_pipeline_wait_ns{kDefaultPipelineWaitNs};
unsigned long long pipeline_wait_limit_ns() { return g_pipeline_wait_ns.load(); }
}  // namespace sep

namespace {

using sep::AttnMaps;
using sep::AttnShape;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// [B, L, H, d] bf16 token-major tensor as a 4-D map {d, H, L, B}; box {64, 1, rows, 1} with the
// 128-byte swizzle (one 128-byte row of 64 bf16 per key/query, 128 or 64 rows per box).
bool encode_map(CUtensorMap* m, const void* base, int B, int L, int H, int d, int rows = 128) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)L, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)H * d * 2, (cuuint64_t)L * H * d * 2};
  cuuint32_t box[4] = {64, 1, (cuuint32_t)rows, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int check_attn_args(const void* q, const void* k, const void* v, int B, int L, int Hq, int Hkv,
                    int d, int a, int n, const SepMask* mask) {
  if (!q || !k || !v || !mask) return SEP_ERR_INVALID_ARG;
  if (B < 1 || L < 1 || Hq < 1 || Hkv < 1 || a < 0 || n < 1) return SEP_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return SEP_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return SEP_ERR_UNSUPPORTED;
  if (mask->B != B || mask->L != L || mask->a != a || mask->n != n) return SEP_ERR_INVALID_ARG;
  if (!mask->sep || !mask->anchor_idx || !mask->anchor_cnt || !mask->anchor_bits ||
      !mask->gather_end || !mask->tile_map)
    return SEP_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v)) return SEP_ERR_MISALIGNED;
  return SEP_OK;
}

// Workspace pieces (each 256-byte aligned, in this order).
struct FwdWs {
  size_t kc, vc, total;
};
FwdWs fwd_ws(int B, int L, int Hkv, int d) {
  FwdWs w;
  const size_t kv = round_up((size_t)B * L * Hkv * d * 2, 256);
  w.kc = 0;
  w.vc = kv;
  w.total = 2 * kv;
  return w;
}
struct BwdWs {
  size_t kc, vc, delta, dka, dva, sched, total;
};
BwdWs bwd_ws(int B, int L, int Hq, int Hkv, int d) {
  BwdWs w;
  const size_t kv = round_up((size_t)B * L * Hkv * d * 2, 256);
  const size_t kvf = round_up((size_t)B * L * Hkv * d * 4, 256);
  const size_t dl = round_up((size_t)B * Hq * L * 4, 256);
  w.kc = 0;
  w.vc = kv;
  w.delta = 2 * kv;
  w.dka = w.delta + dl;
  w.dva = w.dka + kvf;
  w.sched = w.dva + kvf;
  w.total = w.sched + round_up(sep::bwd_sched_bytes(B, L), 256);
  return w;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? SEP_OK : SEP_ERR_CUDA; }

}  // namespace

extern "C" {

int sep_mask_build(const uint8_t* sep, int B, int L, int a, int n, int bm, int bn,
                   int32_t* anchor_idx, int32_t* anchor_cnt, uint32_t* anchor_bits,
                   int32_t* gather_end, int8_t* tile_map, int64_t* kept_pairs,
                   sep_stream_t stream) {
  if (!sep || !anchor_idx || !anchor_cnt || !anchor_bits || !gather_end || !tile_map)
    return SEP_ERR_INVALID_ARG;
  if (B < 1 || L < 1 || a < 0 || n < 1 || bm < 1 || bn < 1) return SEP_ERR_INVALID_ARG;
  if (L > (1 << 30)) return SEP_ERR_UNSUPPORTED;
  return cuda_status(sep::launch_mask_build(sep, B, L, a, n, bm, bn, anchor_idx, anchor_cnt,
                                            anchor_bits, gather_end, tile_map, kept_pairs,
                                            reinterpret_cast<cudaStream_t>(stream)));
}

size_t sep_attn_fwd_workspace_size(int B, int L, int Hkv, int d) {
  if (B < 1 || L < 1 || Hkv < 1 || d < 1) return 0;
  return fwd_ws(B, L, Hkv, d).total;
}

static int attn_fwd_impl(int stages, const sep_bf16* q, const sep_bf16* k, const sep_bf16* v,
                         int B, int L, int Hq, int Hkv, int d, float scale, int a, int n,
                         const SepMask* mask, sep_bf16* o, float* lse, void* workspace,
                         size_t workspace_bytes, sep_stream_t stream) {
  int st = check_attn_args(q, k, v, B, L, Hq, Hkv, d, a, n, mask);
  if (st != SEP_OK) return st;
  if (!o || !lse) return SEP_ERR_INVALID_ARG;
  if (!aligned16(o)) return SEP_ERR_MISALIGNED;
  const FwdWs w = fwd_ws(B, L, Hkv, d);
  if (!workspace || workspace_bytes < w.total) return SEP_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return SEP_ERR_MISALIGNED;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  void* kc = ws + w.kc;
  void* vc = ws + w.vc;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (stages & 1) {
    cudaError_t e = sep::launch_compact_anchors(k, v, mask->anchor_idx, mask->anchor_cnt, B, L,
                                                Hkv, d, kc, vc, s);
    if (e != cudaSuccess) return SEP_ERR_CUDA;
  }
  if (stages & 2) {
    AttnMaps maps;
    std::memset(&maps, 0, sizeof(maps));
    if (!encode_map(&maps.q, q, B, L, Hq, d) || !encode_map(&maps.k, k, B, L, Hkv, d) ||
        !encode_map(&maps.v, v, B, L, Hkv, d) || !encode_map(&maps.kc, kc, B, L, Hkv, d) ||
        !encode_map(&maps.vc, vc, B, L, Hkv, d) || !encode_map(&maps.o, o, B, L, Hq, d) ||
        !encode_map(&maps.k64, k, B, L, Hkv, d, 64) || !encode_map(&maps.v64, v, B, L, Hkv, d, 64) ||
        !encode_map(&maps.kc64, kc, B, L, Hkv, d, 64) ||
        !encode_map(&maps.vc64, vc, B, L, Hkv, d, 64))
      return SEP_ERR_CUDA;
    AttnShape sh{B, L, Hq, Hkv, d, a, n, scale};
    return cuda_status(
        sep::launch_attn_fwd(maps, sh, mask->anchor_bits, mask->gather_end, mask->tile_map, o, lse, s));
  }
  return SEP_OK;
}

int sep_attn_fwd(const sep_bf16* q, const sep_bf16* k, const sep_bf16* v, int B, int L, int Hq,
                 int Hkv, int d, float scale, int a, int n, const SepMask* mask, sep_bf16* o,
                 float* lse, void* workspace, size_t workspace_bytes, sep_stream_t stream) {
  return attn_fwd_impl(3, q, k, v, B, L, Hq, Hkv, d, scale, a, n, mask, o, lse, workspace,
                       workspace_bytes, stream);
}

int sep_attn_fwd_stage(int stage, const sep_bf16* q, const sep_bf16* k, const sep_bf16* v, int B,
                       int L, int Hq, int Hkv, int d, float scale, int a, int n,
                       const SepMask* mask, sep_bf16* o, float* lse, void* workspace,
                       size_t workspace_bytes, sep_stream_t stream) {
  if (stage != 0 && stage != 1) return SEP_ERR_INVALID_ARG;
  return attn_fwd_impl(1 << stage, q, k, v, B, L, Hq, Hkv, d, scale, a, n, mask, o, lse,
                       workspace, workspace_bytes, stream);
}

size_t sep_attn_bwd_workspace_size(int B, int L, int Hq, int Hkv, int d) {
  if (B < 1 || L < 1 || Hq < 1 || Hkv < 1 || d < 1) return 0;
  return bwd_ws(B, L, Hq, Hkv, d).total;
}

static int attn_bwd_impl(int stages, const sep_bf16* q, const sep_bf16* k, const sep_bf16* v,
                         const sep_bf16* o, const float* lse, const sep_bf16* dout, int B, int L,
                         int Hq, int Hkv, int d, float scale, int a, int n, const SepMask* mask,
                         sep_bf16* dq, sep_bf16* dk, sep_bf16* dv, void* workspace,
                         size_t workspace_bytes, sep_stream_t stream) {
  int st = check_attn_args(q, k, v, B, L, Hq, Hkv, d, a, n, mask);
  if (st != SEP_OK) return st;
  if (!o || !lse || !dout || !dq || !dk || !dv) return SEP_ERR_INVALID_ARG;
  if (!aligned16(o) || !aligned16(dout) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return SEP_ERR_MISALIGNED;
  const BwdWs w = bwd_ws(B, L, Hq, Hkv, d);
  if (!workspace || workspace_bytes < w.total) return SEP_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return SEP_ERR_MISALIGNED;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  void* kc = ws + w.kc;
  void* vc = ws + w.vc;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);

  AttnMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  if (!encode_map(&maps.q, q, B, L, Hq, d) || !encode_map(&maps.k, k, B, L, Hkv, d) ||
      !encode_map(&maps.v, v, B, L, Hkv, d) || !encode_map(&maps.kc, kc, B, L, Hkv, d) ||
      !encode_map(&maps.vc, vc, B, L, Hkv, d) || !encode_map(&maps.o, o, B, L, Hq, d) ||
      !encode_map(&maps.dout, dout, B, L, Hq, d) || !encode_map(&maps.dq, dq, B, L, Hq, d) ||
      !encode_map(&maps.dk, dk, B, L, Hkv, d) || !encode_map(&maps.dv, dv, B, L, Hkv, d) ||
      !encode_map(&maps.k64, k, B, L, Hkv, d, 64) || !encode_map(&maps.v64, v, B, L, Hkv, d, 64) ||
      !encode_map(&maps.kc64, kc, B, L, Hkv, d, 64) ||
      !encode_map(&maps.vc64, vc, B, L, Hkv, d, 64))
    return SEP_ERR_CUDA;
  AttnShape sh{B, L, Hq, Hkv, d, a, n, scale};
  return cuda_status(sep::launch_attn_bwd(
      maps, sh, mask->anchor_bits, mask->anchor_idx, mask->anchor_cnt, mask->gather_end, mask->tile_map,
      o, lse, dout, q, k, v, dq, dk, dv, kc, vc, reinterpret_cast<float*>(ws + w.delta),
      reinterpret_cast<float*>(ws + w.dka), reinterpret_cast<float*>(ws + w.dva), ws + w.sched,
      stages, s));
}

int sep_attn_bwd(const sep_bf16* q, const sep_bf16* k, const sep_bf16* v, const sep_bf16* o,
                 const float* lse, const sep_bf16* dout, int B, int L, int Hq, int Hkv, int d,
                 float scale, int a, int n, const SepMask* mask, sep_bf16* dq, sep_bf16* dk,
                 sep_bf16* dv, void* workspace, size_t workspace_bytes, sep_stream_t stream) {
  return attn_bwd_impl(sep::kBwdAll, q, k, v, o, lse, dout, B, L, Hq, Hkv, d, scale, a, n, mask,
                       dq, dk, dv, workspace, workspace_bytes, stream);
}

int sep_attn_bwd_stage(int stage, const sep_bf16* q, const sep_bf16* k, const sep_bf16* v,
                       const sep_bf16* o, const float* lse, const sep_bf16* dout, int B, int L,
                       int Hq, int Hkv, int d, float scale, int a, int n, const SepMask* mask,
                       sep_bf16* dq, sep_bf16* dk, sep_bf16* dv, void* workspace,
                       size_t workspace_bytes, sep_stream_t stream) {
  if (stage < 0 || stage > 2) return SEP_ERR_INVALID_ARG;
  return attn_bwd_impl(1 << stage, q, k, v, o, lse, dout, B, L, Hq, Hkv, d, scale, a, n, mask, dq,
                       dk, dv, workspace, workspace_bytes, stream);
}

static int check_cache(const SepCacheState* st) {
  if (!st) return SEP_ERR_INVALID_ARG;
  if (st->S < 1 || st->Hq < 1 || st->Hkv < 1 || st->a < 0 || st->s < 0 || st->w < 1)
    return SEP_ERR_INVALID_ARG;
  if (st->Hq % st->Hkv != 0) return SEP_ERR_INVALID_ARG;
  const int G = st->Hq / st->Hkv;
  if (st->d != 64 && st->d != 128) return SEP_ERR_UNSUPPORTED;
  if (G > 8) return SEP_ERR_UNSUPPORTED;
  if (!st->k_slots || !st->v_slots || !st->slot_pos || !st->slot_sep || !st->meta ||
      !st->rope_freq)
    return SEP_ERR_INVALID_ARG;
  if (!aligned16(st->k_slots) || !aligned16(st->v_slots) || !aligned16(st->rope_freq))
    return SEP_ERR_MISALIGNED;
  if (!(st->rope_theta > 0.f)) return SEP_ERR_INVALID_ARG;
  // usage threshold of the Past Window: 0 (none) or above the three fixed blocks
  if (st->c < 0 || (st->c > 0 && st->c <= st->a + st->s + st->w)) return SEP_ERR_INVALID_ARG;
  if (st->c > 0 && std::min(st->s, st->c - st->a - st->w) > 4096) return SEP_ERR_UNSUPPORTED;
  return SEP_OK;
}

int sepcache_state_init(const SepCacheState* st, sep_stream_t stream) {
  int e = check_cache(st);
  if (e != SEP_OK) return e;
  return cuda_status(sep::launch_sepcache_init(*st, reinterpret_cast<cudaStream_t>(stream)));
}

int sepcache_update(const SepCacheState* st, const sep_bf16* k_new, const sep_bf16* v_new,
                    const uint8_t* sep_new, sep_stream_t stream) {
  int e = check_cache(st);
  if (e != SEP_OK) return e;
  if (!k_new || !v_new || !sep_new) return SEP_ERR_INVALID_ARG;
  if (!aligned16(k_new) || !aligned16(v_new)) return SEP_ERR_MISALIGNED;
  return cuda_status(sep::launch_sepcache_update(*st, k_new, v_new, sep_new,
                                                 reinterpret_cast<cudaStream_t>(stream)));
}

int sepcache_prefill(const SepCacheState* st, const sep_bf16* k, const sep_bf16* v,
                     const uint8_t* sep, int L, sep_stream_t stream) {
  int e = check_cache(st);
  if (e != SEP_OK) return e;
  if (!k || !v || !sep || L < 1) return SEP_ERR_INVALID_ARG;
  if (st->s > 16384) return SEP_ERR_UNSUPPORTED;
  if (!aligned16(k) || !aligned16(v)) return SEP_ERR_MISALIGNED;
  return cuda_status(sep::launch_sepcache_prefill(*st, k, v, sep, L,
                                                  reinterpret_cast<cudaStream_t>(stream)));
}

int sepcache_decode(const SepCacheState* st, const sep_bf16* q, sep_bf16* o, float* lse,
                    float scale, sep_stream_t stream) {
  int e = check_cache(st);
  if (e != SEP_OK) return e;
  if (!q || !o) return SEP_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(o)) return SEP_ERR_MISALIGNED;
  return cuda_status(
      sep::launch_sepcache_decode(*st, q, o, lse, scale, reinterpret_cast<cudaStream_t>(stream)));
}

int sepcache_export_order(const SepCacheState* st, int32_t* pos_out, int32_t* count,
                          sep_stream_t stream) {
  int e = check_cache(st);
  if (e != SEP_OK) return e;
  if (!pos_out || !count) return SEP_ERR_INVALID_ARG;
  return cuda_status(
      sep::launch_sepcache_export(*st, pos_out, count, reinterpret_cast<cudaStream_t>(stream)));
}

int sep_last_device_error(void) {
  unsigned* p = sep::device_error_word();
  if (!p) return SEP_ERR_CUDA;
  if (cudaDeviceSynchronize() != cudaSuccess) return SEP_ERR_CUDA;
  unsigned v = 0;
  if (cudaMemcpy(&v, p, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return SEP_ERR_CUDA;
  if (v != 0) {
    const unsigned zero = 0;
    if (cudaMemcpy(p, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
      return SEP_ERR_CUDA;
  }
  return (int)v;
}

int sep_attn_fwd_noalloc(const sep_bf16* q, const sep_bf16* k, const sep_bf16* v, int B, int L,
                         int Hq, int Hkv, int d, float scale, int a, int n, const SepMask* mask,
                         sep_bf16* o, float* lse, sep_stream_t stream) {
  // host checks first, so that an oversized problem is refused before any device work
  int st = check_attn_args(q, k, v, B, L, Hq, Hkv, d, a, n, mask);
  if (st != SEP_OK) return st;
  if (!o || !lse) return SEP_ERR_INVALID_ARG;
  if (fwd_ws(B, L, Hkv, d).total > (size_t)SEP_NOALLOC_SCRATCH_BYTES) return SEP_ERR_SCRATCH_LIMIT;
  cudaError_t e = cudaSuccess;
  void* scratch = sep::noalloc_fwd_scratch(&e);
  if (!scratch) return SEP_ERR_CUDA;
  return attn_fwd_impl(3, q, k, v, B, L, Hq, Hkv, d, scale, a, n, mask, o, lse, scratch,
                       (size_t)SEP_NOALLOC_SCRATCH_BYTES, stream);
}

int sep_set_wait_limit_ns(unsigned long long ns) {
  sep::g_pipeline_wait_ns.store(ns ? ns : sep::kDefaultPipelineWaitNs);
  return SEP_OK;
}

const char* sep_status_string(int status) {
  switch (status) {
    case SEP_OK: return "ok";
    case SEP_ERR_INVALID_ARG: return "invalid argument";
    case SEP_ERR_UNSUPPORTED: return "unsupported size";
    case SEP_ERR_MISALIGNED: return "misaligned pointer";
    case SEP_ERR_CUDA: return "CUDA error";
    case SEP_ERR_TIMEOUT: return "device pipeline wait timed out";
    case SEP_ERR_WORKSPACE: return "workspace missing or too small";
    case SEP_ERR_SCRATCH_LIMIT:
      return "problem needs more than the fixed scratch of sep_attn_fwd_noalloc";
    default: return "unknown status";
  }
}

}  // extern "C"
