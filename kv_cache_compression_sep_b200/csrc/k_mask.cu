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
// tile classified from anchor counts C(x) = #anchors < x: in O(1) from the anchor flag words up
// to the tile's last row, staged in shared memory with their exclusive popcount prefix; for
// sequences whose words do not fit there, in O(log L) by binary search over the anchor list.
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
  grid_dep_wait();
  grid_dep_launch_next();
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

// Class of block (query rows r0..r1, key tile u) and the gather end of the query tile, from an
// anchor counter C(x) = #anchors at positions < x (0 <= x <= L).
template <class Count>
__device__ __forceinline__ void classify_tiles(Count C, int L, int n, int bn, int T, int U, int b,
                                               int t, long long r0, long long r1,
                                               int32_t* __restrict__ gather_end,
                                               int8_t* __restrict__ tile_map) {
  if (threadIdx.x == 0) {
    const long long lo_key = max(0ll, r0 - n + 1);
    const long long lo_tile = lo_key / bn;
    gather_end[(size_t)b * T + t] = C(lo_tile * bn);
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
      const int c0 = C(k0);
      const bool anc = C(hi_a + 1) - c0 > 0;
      if (!win && !anc) {
        cls = SEP_TILE_SKIP;
      } else {
        bool full = false;
        if (k1 <= r0) {  // every pair causal; keys the last row sees beyond n back must be anchors
          const long long x = min(k1, r1 - n);
          full = (x < k0) || (C(x + 1) - c0 == (int)(x - k0 + 1));
        }
        cls = full ? SEP_TILE_FULL : SEP_TILE_PARTIAL;
      }
    }
    tile_map[((size_t)b * T + t) * U + u] = cls;
  }
}

// O(log L) counts: binary search over the sorted anchor list (long sequences).
__global__ void __launch_bounds__(256) mask_tiles_kernel(const int32_t* __restrict__ anchor_idx,
                                                         const int32_t* __restrict__ anchor_cnt,
                                                         int L, int n, int bm, int bn, int T,
                                                         int U, int32_t* __restrict__ gather_end,
                                                         int8_t* __restrict__ tile_map) {
  grid_dep_wait();
  grid_dep_launch_next();
  const int t = blockIdx.x, b = blockIdx.y;
  const int cnt = anchor_cnt[b];
  const int32_t* idx = anchor_idx + (size_t)b * L;
  const long long r0 = (long long)t * bm;
  const long long r1 = min((long long)L, r0 + bm) - 1;
  classify_tiles([&](long long x) { return count_lt(idx, cnt, x); }, L, n, bn, T, U, b, t, r0, r1,
                 gather_end, tile_map);
}

constexpr int kTileWordsMax = 6000;  // flag words staged by mask_tiles_words_kernel (< 48 KB)

// O(1) counts: the CTA stages the anchor flag words 0 .. r1 / 32 of its sequence and their
// exclusive popcount prefix in shared memory; C(x) = pre[x / 32] + popc(word & (bit x%32 - 1)).
__global__ void __launch_bounds__(256) mask_tiles_words_kernel(
    const uint32_t* __restrict__ anchor_bits, int L, int n, int bm, int bn, int T, int U,
    int32_t* __restrict__ gather_end, int8_t* __restrict__ tile_map) {
  extern __shared__ uint32_t s_words[];  // [nw] flag words, then [nw + 1] prefix counts
  __shared__ int s_warp[8];
  grid_dep_wait();
  grid_dep_launch_next();
  const int t = blockIdx.x, b = blockIdx.y;
  const int W = (L + 31) / 32;
  const long long r0 = (long long)t * bm;
  const long long r1 = min((long long)L, r0 + bm) - 1;
  // counts are asked for x <= r1 + 1: words 0 .. (r1 + 1) / 32, those inside the sequence
  const int nw = min(W, (int)((r1 + 1) / 32) + 1);
  uint32_t* words = s_words;
  int* pre = reinterpret_cast<int*>(s_words + nw);
  const uint32_t* src = anchor_bits + (size_t)b * W;
  // each thread sums a run of consecutive words, then an exclusive scan over the runs
  const int per = (nw + blockDim.x - 1) / blockDim.x;
  const int w0 = min(nw, (int)threadIdx.x * per), w1 = min(nw, w0 + per);
  int run = 0;
  for (int w = w0; w < w1; ++w) {
    const uint32_t v = __ldg(src + w);
    words[w] = v;
    run += __popc(v);
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = run;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  int base = 0;
  for (int k = 0; k < warp; ++k) base += s_warp[k];
  int acc = base + incl - run;  // anchors in words < w0
  for (int w = w0; w < w1; ++w) {
    pre[w] = acc;
    acc += __popc(words[w]);
  }
  if ((int)threadIdx.x == (int)blockDim.x - 1) {
    int tot = 0;
    for (int k = 0; k < 8; ++k) tot += s_warp[k];
    pre[nw] = tot;  // anchors in all staged words
  }
  __syncthreads();
  auto C = [&](long long x) -> int {
    const int w = (int)(x >> 5);
    if (w >= nw) return pre[nw];
    return pre[w] + __popc(words[w] & ((1u << (x & 31)) - 1u));
  };
  classify_tiles(C, L, n, bn, T, U, b, t, r0, r1, gather_end, tile_map);
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
  cudaError_t e = launch_chained(mask_scan_kernel, dim3(B), dim3(kScanThreads), 0, stream, sep, L,
                                 a, n, anchor_idx, anchor_cnt, anchor_bits, kept);
  if (e != cudaSuccess) return e;
  const int T = (L + bm - 1) / bm, U = (L + bn - 1) / bn;
  const int W = (L + 31) / 32;
  if (W <= kTileWordsMax) {
    const size_t smem = (2 * (size_t)W + 1) * sizeof(uint32_t);
    return launch_chained(mask_tiles_words_kernel, dim3(T, B), dim3(256), smem, stream,
                          anchor_bits, L, n, bm, bn, T, U, gather_end, tile_map);
  }
  return launch_chained(mask_tiles_kernel, dim3(T, B), dim3(256), 0, stream, anchor_idx,
                        anchor_cnt, L, n, bm, bn, T, U, gather_end, tile_map);
}

}  // namespace sep
