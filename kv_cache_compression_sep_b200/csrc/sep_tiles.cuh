// Tile schedule and keep-mask helpers shared by the forward and backward attention kernels.
//
// keep(i, j) = j <= i && (i - j < n || f[j]) with f[j] = (j < a) || sep[j] (SepLLM, atlas.scime.ai
// summary, section "Approach"). Query tile t (rows 128t..128t+127) reads whole key tiles
// lo(t)..t, lo(t) = max(0, 128t - n + 1) / 128, and the anchors left of tile lo(t) (the first
// gather_end[t] entries of the sorted anchor list), which every row of the tile keeps.
#pragma once

#include <stdint.h>

namespace sep {

// Row i of batch b of the compacted anchor K / V (one warp; kv_ch = 16-byte chunks per row):
// the K / V row of the i-th anchor when i < cnt, zeros for the padding rows after the last
// anchor (how many is the caller's choice).
__device__ __forceinline__ void compact_anchor_row(const uint4* __restrict__ k,
                                                   const uint4* __restrict__ v,
                                                   const int32_t* __restrict__ anchor_idx,
                                                   int cnt, int L, int b, int i, int kv_ch,
                                                   uint4* __restrict__ kc, uint4* __restrict__ vc,
                                                   int lane) {
  const size_t row = (size_t)b * L + i;
  uint4* dk = kc + row * kv_ch;
  uint4* dv = vc + row * kv_ch;
  if (i < cnt) {
    const size_t src = ((size_t)b * L + __ldg(anchor_idx + row)) * kv_ch;
    for (int c = lane; c < kv_ch; c += 32) {
      const uint4 x = __ldg(k + src + c), y = __ldg(v + src + c);
      dk[c] = x;
      dv[c] = y;
    }
  } else {
    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
    for (int c = lane; c < kv_ch; c += 32) {
      dk[c] = z;
      dv[c] = z;
    }
  }
}

__host__ __device__ __forceinline__ int window_lo_tile(int t, int n) {
  const long long k = (long long)t * 128 - n + 1;
  return k > 0 ? (int)(k / 128) : 0;
}

// Bits of one 32-column word (columns 32w..32w+31 of a 128-column tile) that lie in [lo, hi].
__device__ __forceinline__ uint32_t range_word(long long lo, long long hi, int w) {
  const long long l = lo - 32 * w, h = hi - 32 * w;
  if (h < 0 || l > 31 || h < l) return 0u;
  const uint32_t le = (h >= 31) ? 0xffffffffu : ((2u << h) - 1u);
  const uint32_t ge = (l <= 0) ? 0xffffffffu : ~((1u << l) - 1u);
  return le & ge;
}

// Keep bits of one 32-column word of key tile k0..k0+127 for query row i (row-major view: the
// thread owns a query row, the columns are keys). fbits = anchor flags of the word's keys.
__device__ __forceinline__ uint32_t window_keep_word(int w, long long i, long long k0, int n,
                                                     int L, uint32_t fbits) {
  const long long hi = (i < (long long)L - 1 ? i : (long long)L - 1) - k0;  // causal, in bounds
  const long long lo = i - n + 1 - k0;                                     // inside the band
  return range_word(lo > 0 ? lo : 0, hi, w) | (fbits & range_word(0, hi, w));
}

}  // namespace sep
