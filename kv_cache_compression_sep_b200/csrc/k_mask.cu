// sep_mask_build kernels: the separator-sparse mask M_b in compressed form.
//
// Keep rule (SepLLM, atlas.scime.ai summary, section "Approach"): query i keeps key j <= i when
// j is an initial token (j < a), a separator, or one of the n most recent neighbours
// (i - j < n). With the anchor flag f[j] = (j < a) || sep[j] this is
//     keep(i, j) = j <= i && (i - j < n || f[j]).
//
// Kernel 1 (one CTA per batch element): block-wide exclusive scan of f, compaction of the
// anchor positions, and the kept-pair count sum_i min(i+1, n) + C(i-n) with C the inclusive
// anchor count. Kernel 2 (one CTA per query tile): gather_end and one row of the tile map, each
// tile classified in O(log L) from anchor counts (binary search over the sorted anchor list).
#include <cuda_runtime.h>

#include "sep_common.cuh"
#include "sep_launch.h"

namespace sep {

__device__ unsigned g_device_error_word;

constexpr int kScanThreads = 1024;
constexpr int kScanItems = 16;

__global__ void __launch_bounds__(kScanThreads) mask_scan_kernel(const uint8_t* __restrict__ sep,
                                                                 int L, int a, int n,
                                                                 int32_t* __restrict__ anchor_idx,
                                                                 int32_t* __restrict__ anchor_cnt,
                                                                 uint32_t* __restrict__ anchor_bits,
                                                                 int64_t* __restrict__ kept) {
  const int b = blockIdx.x;
  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  sep += (size_t)b * L;
  anchor_idx += (size_t)b * L;
  anchor_bits += (size_t)b * ((L + 31) / 32);

  __shared__ int s_warp[32];
  __shared__ long long s_red[32];
  __shared__ int s_total;

  int carry = 0;           // anchors before this pass
  long long csum = 0;      // sum over x <= L-1-n of C(x), this thread's share
  const long long last_x = (long long)L - 1 - n;

  for (int base = 0; base < L; base += kScanThreads * kScanItems) {
    const int j0 = base + tid * kScanItems;
    uint32_t bits = 0;
#pragma unroll
    for (int k = 0; k < kScanItems; ++k) {
      const int j = j0 + k;
      if (j < L && (j < a || sep[j] != 0)) bits |= 1u << k;
    }
    // packed flags: lanes 2k and 2k+1 hold the two 16-position halves of word j0 / 32
    {
      const uint32_t hi = __shfl_down_sync(0xffffffffu, bits, 1);
      if ((lane & 1) == 0 && j0 < L) anchor_bits[j0 / 32] = bits | (hi << 16);
    }
    const int cnt = __popc(bits);
    // block exclusive scan of cnt
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      int w = (lane < kScanThreads / 32) ? s_warp[lane] : 0;
      int wi = w;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, wi, o);
        if (lane >= o) wi += y;
      }
      if (lane < kScanThreads / 32) s_warp[lane] = wi - w;  // exclusive warp offsets
      if (lane == 31) s_total = wi;
    }
    __syncthreads();
    int run = carry + s_warp[warp] + incl - cnt;  // anchors before j0
#pragma unroll
    for (int k = 0; k < kScanItems; ++k) {
      const int j = j0 + k;
      if (bits & (1u << k)) anchor_idx[run++] = j;
      if ((long long)j <= last_x) csum += run;  // run = C(j), inclusive
    }
    carry += s_total;
    __syncthreads();
  }
  for (int j = carry + tid; j < L; j += kScanThreads) anchor_idx[j] = -1;

  // block reduction of csum
  long long v = csum;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_down_sync(0xffffffffu, v, o);
  if (lane == 0) s_red[warp] = v;
  __syncthreads();
  if (tid == 0) {
    long long tot = 0;
    for (int w = 0; w < kScanThreads / 32; ++w) tot += s_red[w];
    const long long Ln = L, nn = n;
    const long long win = (Ln <= nn) ? Ln * (Ln + 1) / 2 : nn * (nn + 1) / 2 + (Ln - nn) * nn;
    anchor_cnt[b] = carry;
    if (kept) kept[b] = win + tot;
  }
}

// Number of anchors at positions < x (lower bound in the sorted list).
__device__ __forceinline__ int count_lt(const int32_t* __restrict__ idx, int cnt, long long x) {
  int lo = 0, hi = cnt;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if ((long long)idx[mid] < x)
      lo = mid + 1;
    else
      hi = mid;
  }
  return lo;
}

__global__ void __launch_bounds__(256) mask_tiles_kernel(const int32_t* __restrict__ anchor_idx,
                                                         const int32_t* __restrict__ anchor_cnt,
                                                         int L, int n, int bm, int bn, int T,
                                                         int U, int32_t* __restrict__ gather_end,
                                                         int8_t* __restrict__ tile_map) {
  const int t = blockIdx.x, b = blockIdx.y;
  const int cnt = anchor_cnt[b];
  const int32_t* idx = anchor_idx + (size_t)b * L;
  const long long r0 = (long long)t * bm;
  const long long r1 = min((long long)L, r0 + bm) - 1;
  if (threadIdx.x == 0) {
    const long long lo_key = max(0ll, r0 - n + 1);
    const long long lo_tile = lo_key / bn;
    gather_end[(size_t)b * T + t] = count_lt(idx, cnt, lo_tile * bn);
  }
  for (int u = threadIdx.x; u < U; u += blockDim.x) {
    const long long k0 = (long long)u * bn;
    const long long k1 = min((long long)L, k0 + bn) - 1;
    int8_t cls;
    if (k0 > r1) {
      cls = SEP_TILE_SKIP;  // every key is after every row
    } else {
      // a window pair exists if the blocks overlap or the closest pair is < n apart
      const bool win = (k1 >= r0) || (r0 - k1 < n);
      const long long hi_a = min(k1, r1);
      const bool anc = count_lt(idx, cnt, hi_a + 1) - count_lt(idx, cnt, k0) > 0;
      if (!win && !anc) {
        cls = SEP_TILE_SKIP;
      } else {
        bool full = false;
        if (k1 <= r0) {  // every pair causal; keys the last row sees beyond n back must be anchors
          const long long x = min(k1, r1 - n);
          full = (x < k0) ||
                 (count_lt(idx, cnt, x + 1) - count_lt(idx, cnt, k0) == (int)(x - k0 + 1));
        }
        cls = full ? SEP_TILE_FULL : SEP_TILE_PARTIAL;
      }
    }
    tile_map[((size_t)b * T + t) * U + u] = cls;
  }
}

unsigned* device_error_word() {
  static unsigned* cache[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  if (!cache[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error_word) != cudaSuccess) return nullptr;
    cache[dev] = static_cast<unsigned*>(p);
  }
  return cache[dev];
}

cudaError_t launch_mask_build(const uint8_t* sep, int B, int L, int a, int n, int bm, int bn,
                              int32_t* anchor_idx, int32_t* anchor_cnt, uint32_t* anchor_bits,
                              int32_t* gather_end, int8_t* tile_map, int64_t* kept,
                              cudaStream_t stream) {
  mask_scan_kernel<<<B, kScanThreads, 0, stream>>>(sep, L, a, n, anchor_idx, anchor_cnt,
                                                   anchor_bits, kept);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int T = (L + bm - 1) / bm, U = (L + bn - 1) / bn;
  mask_tiles_kernel<<<dim3(T, B), 256, 0, stream>>>(anchor_idx, anchor_cnt, L, n, bm, bn, T, U,
                                                     gather_end, tile_map);
  return cudaGetLastError();
}

}  // namespace sep
