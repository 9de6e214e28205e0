// sep_attn_bwd: backward of separator-sparse attention on sm_100a (tcgen05 + TMEM + TMA).
//
// Gradients of sum(O * dO) over the kept pairs of the SepLLM mask (the same mask is used when
// training from scratch: "How SepLLM reorchestrates the language model...", section "The
// Mechanics of Compression"; "SepLLM: Accelerate Large Language Models ...", atlas.scime.ai,
// "Key results"). With P = exp(S - lse) on kept pairs:
//   dV = P^T dO, dP = dO V^T, Delta_i = sum_c dO_ic O_ic, dS = P (dP - Delta),
//   dQ = scale dS K, dK = scale dS^T Q,
// dK, dV summed over the query heads of a KV head.
//
// Kernels, in stream order:
//   1. prep: compacted anchor K/V rows (shared with the forward), zeroed fp32 anchor partials,
//      Delta = rowsum(dO * O).
//   2. dQ (query-major, one CTA per (query tile, query head, batch); same key tiles as the
//      forward): S = Q K^T and dP = dO V^T into TMEM, dS = P (dP - Delta) written back to TMEM
//      as bf16, dQ += dS K (A from TMEM, B = K MN-major).
//   3. dK/dV (key-major): one CTA per window key tile u (query tiles t with lo(t) <= u <= t) or
//      per (anchor chunk c, segment of query tiles that gather it). Per (query tile, query head):
//      S^T = K Q^T, dP^T = V dO^T into TMEM; P^T and dS^T back to TMEM as bf16;
//      dV += P^T dO, dK += dS^T Q. Non-anchor keys of a window tile get their complete gradient
//      and are written as bf16; anchor keys are summed in fp32 (window part + every gathered
//      part) in a compact [B, anchors, Hkv, d] buffer.
//   4. combine: anchor partials to bf16 dK/dV at the anchors' positions.
#include <cuda_runtime.h>

#include "sep_common.cuh"
#include "sep_launch.h"
#include "sep_tiles.cuh"

namespace sep {

constexpr int kBoxBytes = 128 * 64 * 2;
constexpr int kAnchorSeg = 16;  // query tiles per anchor-chunk CTA of the dK/dV kernel

// ------------------------------------------------------------------ prep kernels
__global__ void __launch_bounds__(256) zero_anchor_partials_kernel(
    const int32_t* __restrict__ anchor_cnt, int L, int rowvec, int rows_per_cta,
    float4* __restrict__ dka, float4* __restrict__ dva) {
  const int b = blockIdx.y;
  const int cnt = anchor_cnt[b];
  const int r0 = blockIdx.x * rows_per_cta;
  if (r0 >= cnt) return;
  const int rows = min(rows_per_cta, cnt - r0);
  const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int e = threadIdx.x; e < rows * rowvec; e += blockDim.x) {
    const size_t dst = ((size_t)b * L + r0 + e / rowvec) * rowvec + e % rowvec;
    dka[dst] = z;
    dva[dst] = z;
  }
}

// Delta[b][h][i] = sum_c dO[b,i,h,c] * O[b,i,h,c]; one thread per (b, i, h) row, 16-byte loads.
template <int D>
__global__ void __launch_bounds__(256) delta_kernel(const __nv_bfloat16* __restrict__ o,
                                                    const __nv_bfloat16* __restrict__ dout,
                                                    int B, int L, int Hq, float* __restrict__ delta) {
  // consecutive threads take consecutive positions i of one (b, h): coalesced Delta stores
  const long long id = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (id >= (long long)B * L * Hq) return;
  const int i = (int)(id % L);
  const long long bh = id / L;
  const int h = (int)(bh % Hq), b = (int)(bh / Hq);
  const long long row = ((long long)b * L + i) * Hq + h;
  const uint4* po = reinterpret_cast<const uint4*>(o + row * D);
  const uint4* pd = reinterpret_cast<const uint4*>(dout + row * D);
  float acc = 0.f;
#pragma unroll
  for (int q = 0; q < D / 8; ++q) {
    const uint4 x = __ldg(po + q), y = __ldg(pd + q);
    const uint32_t xs[4] = {x.x, x.y, x.z, x.w}, ys[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
    for (int z = 0; z < 4; ++z) {
      const __nv_bfloat162 a2 = *reinterpret_cast<const __nv_bfloat162*>(&xs[z]);
      const __nv_bfloat162 b2 = *reinterpret_cast<const __nv_bfloat162*>(&ys[z]);
      acc = fmaf(__low2float(a2), __low2float(b2), acc);
      acc = fmaf(__high2float(a2), __high2float(b2), acc);
    }
  }
  delta[((size_t)b * Hq + h) * L + i] = acc;
}

// ------------------------------------------------------------------ shared parameter block
struct BwdParams {
  CUtensorMap tmQ, tmK, tmV, tmKc, tmVc, tmdO;
  const uint32_t* anchor_bits;  // [B, W] packed anchor flags
  const int32_t* anchor_idx;
  const int32_t* anchor_cnt;
  const int32_t* gather_end;
  const int8_t* tile_map;
  const float* lse;    // [B, Hq, L] natural log
  const float* delta;  // [B, Hq, L]
  __nv_bfloat16* dq;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  float* dka;  // [B, L, Hkv, D] fp32 anchor partials (rows < anchor_cnt)
  float* dva;
  unsigned* err;
  int B, L, Hq, Hkv, T, W, a, n;
  float scale, scale_log2;
};

// ------------------------------------------------------------------ dQ kernel
template <int D>
struct DqCfg {
  static constexpr int KB = D / 64;
  static constexpr int TILE = KB * kBoxBytes;
  static constexpr int NST = (D == 128) ? 2 : 4;
  static constexpr int SMEM_TILES = TILE * (2 + 2 * NST);  // Q, dO, NST x (K, V)
  static constexpr int COL_S = 0, COL_DP = 256, COL_DQ = 384;
};

template <int NST>
struct DqBar {
  uint64_t q_full;
  uint64_t k_full[NST], k_empty[NST], v_full[NST], v_empty[NST];
  uint64_t s_full[2], ds_ready[2], dq_done[2];
  uint64_t dp_free;
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

template <int D>
constexpr size_t dq_smem_bytes() {
  return 1024 + DqCfg<D>::SMEM_TILES + sizeof(DqBar<DqCfg<D>::NST>);
}

template <int D>
__global__ void __launch_bounds__(192, 1) sep_attn_bwd_dq_kernel(const __grid_constant__ BwdParams p) {
  using C = DqCfg<D>;
  constexpr int NST = C::NST;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sdO = sQ + C::TILE;
  uint8_t* sK = sdO + C::TILE;
  uint8_t* sV = sK + NST * C::TILE;
  DqBar<NST>* bar = reinterpret_cast<DqBar<NST>*>(sV + NST * C::TILE);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = p.T - 1 - (int)blockIdx.x;
  const int h = blockIdx.y, b = blockIdx.z;
  const int kvh = h / (p.Hq / p.Hkv);
  const int lo_tile = window_lo_tile(t, p.n);
  const int nwin = t - lo_tile + 1;
  const int ge = p.gather_end[(size_t)b * p.T + t];
  const int N = nwin + (ge + 127) / 128;
  volatile int* abort_flag = &bar->abort_flag;

  if (threadIdx.x == 0) {
    mbar_init(&bar->q_full, 1);
    for (int s = 0; s < NST; ++s) {
      mbar_init(&bar->k_full[s], 1);
      mbar_init(&bar->k_empty[s], 1);
      mbar_init(&bar->v_full[s], 1);
      mbar_init(&bar->v_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar->s_full[s], 1);
      mbar_init(&bar->ds_ready[s], 128);
      mbar_init(&bar->dq_done[s], 1);
    }
    mbar_init(&bar->dp_free, 128);
    mbar_init(&bar->drain, 1);
    bar->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(&bar->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar->tmem_base;

  if (warp == 4) {
    if (lane == 0) {
      mbar_arrive_expect_tx(&bar->q_full, 2 * C::TILE);
      for (int kb = 0; kb < C::KB; ++kb) {
        tma_load_4d(sQ + kb * kBoxBytes, &p.tmQ, &bar->q_full, kb * 64, h, t * 128, b);
        tma_load_4d(sdO + kb * kBoxBytes, &p.tmdO, &bar->q_full, kb * 64, h, t * 128, b);
      }
      for (int j = 0; j < N; ++j) {
        const int st = j % NST, r = j / NST;
        const bool win = j < nwin;
        const int row0 = win ? (t - j) * 128 : (j - nwin) * 128;
        if (r > 0 && !mbar_wait(&bar->k_empty[st], (r - 1) & 1, p.err, abort_flag)) break;
        mbar_arrive_expect_tx(&bar->k_full[st], C::TILE);
        for (int kb = 0; kb < C::KB; ++kb)
          tma_load_4d(sK + st * C::TILE + kb * kBoxBytes, win ? &p.tmK : &p.tmKc,
                      &bar->k_full[st], kb * 64, kvh, row0, b);
        if (r > 0 && !mbar_wait(&bar->v_empty[st], (r - 1) & 1, p.err, abort_flag)) {
          mbar_wait(&bar->k_full[st], r & 1, nullptr, nullptr);
          break;
        }
        mbar_arrive_expect_tx(&bar->v_full[st], C::TILE);
        for (int kb = 0; kb < C::KB; ++kb)
          tma_load_4d(sV + st * C::TILE + kb * kBoxBytes, win ? &p.tmV : &p.tmVc,
                      &bar->v_full[st], kb * 64, kvh, row0, b);
      }
      if (*abort_flag) {
        mbar_wait(&bar->q_full, 0, nullptr, nullptr);
        for (int j = max(0, N - NST); j < N; ++j) {
          mbar_wait(&bar->k_full[j % NST], (j / NST) & 1, nullptr, nullptr);
          mbar_wait(&bar->v_full[j % NST], (j / NST) & 1, nullptr, nullptr);
        }
      }
    }
  } else if (warp == 5) {
    if (lane == 0) {
      constexpr uint32_t idS = make_idesc_bf16(128, 128, false, false);
      constexpr uint32_t idQ = make_idesc_bf16(128, D, false, true);
      const uint32_t sQa = smem_u32(sQ), sdOa = smem_u32(sdO);
      const uint32_t sKa = smem_u32(sK), sVa = smem_u32(sV);
      bool ok = mbar_wait(&bar->q_full, 0, p.err, abort_flag);
      auto issue_SdP = [&](int j) -> bool {
        const int st = j % NST;
        if (!mbar_wait(&bar->k_full[st], (j / NST) & 1, p.err, abort_flag)) return false;
        if (!mbar_wait(&bar->v_full[st], (j / NST) & 1, p.err, abort_flag)) return false;
        // S[j%2] held dS_{j-2}, read by dQ_{j-2}
        if (j >= 2 && !mbar_wait(&bar->dq_done[j & 1], ((j - 2) >> 1) & 1, p.err, abort_flag))
          return false;
        // dP was read by the softmax warps for tile j-1
        if (j >= 1 && !mbar_wait(&bar->dp_free, (j - 1) & 1, p.err, abort_flag)) return false;
        tc_fence_after();
        const uint32_t dS = tmem + C::COL_S + (j & 1) * 128;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kBoxBytes + (kk & 3) * 32;
          mma_ss(dS, make_sdesc_sw128(sQa + off, 16, 1024),
                 make_sdesc_sw128(sKa + st * C::TILE + off, 16, 1024), idS, kk > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kBoxBytes + (kk & 3) * 32;
          mma_ss(tmem + C::COL_DP, make_sdesc_sw128(sdOa + off, 16, 1024),
                 make_sdesc_sw128(sVa + st * C::TILE + off, 16, 1024), idS, kk > 0 ? 1u : 0u);
        }
        tc_commit(&bar->s_full[j & 1]);
        tc_commit(&bar->v_empty[st]);
        return true;
      };
      auto issue_dQ = [&](int j) -> bool {
        const int st = j % NST;
        if (!mbar_wait(&bar->ds_ready[j & 1], (j >> 1) & 1, p.err, abort_flag)) return false;
        tc_fence_after();
        const uint32_t aS = tmem + C::COL_S + (j & 1) * 128;
#pragma unroll
        for (int kk = 0; kk < 128 / 16; ++kk) {
          mma_ts(tmem + C::COL_DQ, aS + kk * 8,
                 make_sdesc_sw128(sKa + st * C::TILE + kk * 2048, kBoxBytes, 1024), idQ,
                 (j > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(&bar->dq_done[j & 1]);
        tc_commit(&bar->k_empty[st]);
        return true;
      };
      if (ok) ok = issue_SdP(0);
      for (int j = 0; ok && j < N; ++j) {
        if (j + 1 < N && !issue_SdP(j + 1)) break;
        if (!issue_dQ(j)) break;
      }
      tc_commit(&bar->drain);
      mbar_wait(&bar->drain, 0, nullptr, nullptr);
    }
  } else {
    const int row = threadIdx.x;
    const long long i = (long long)t * 128 + row;
    const bool valid = i < p.L;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const uint32_t* bits_row = p.anchor_bits + (size_t)b * p.W;
    const int8_t* tmap = p.tile_map + ((size_t)b * p.T + t) * p.T;
    const float sl2 = p.scale_log2;
    const size_t rowstat = ((size_t)b * p.Hq + h) * p.L + (valid ? i : 0);
    const float lse2 = valid ? p.lse[rowstat] * 1.4426950408889634f : INFINITY;
    const float dlt = valid ? p.delta[rowstat] : 0.f;
    bool ok = true;
    for (int j = 0; j < N; ++j) {
      const int sb = j & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&bar->s_full[sb], (j >> 1) & 1, p.err, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t keep[4] = {0xffffffffu, 0xffffffffu, 0xffffffffu, 0xffffffffu};
      if (j < nwin) {
        const int u = t - j;
        const long long k0 = (long long)u * 128;
        if (tmap[u] != SEP_TILE_FULL) {
#pragma unroll
          for (int w = 0; w < 4; ++w)
            keep[w] = window_keep_word(w, i, k0, p.n, p.L,
                                       (u * 4 + w < p.W) ? __ldg(bits_row + u * 4 + w) : 0u);
        } else if (k0 + 128 > p.L) {
#pragma unroll
          for (int w = 0; w < 4; ++w) keep[w] = range_word(0, (long long)p.L - 1 - k0, w);
        }
      } else {
        const int rem = ge - (j - nwin) * 128;
        if (rem < 128) {
#pragma unroll
          for (int w = 0; w < 4; ++w) keep[w] = range_word(0, rem - 1, w);
        }
      }
      const uint32_t aS = tmem + lane_off + C::COL_S + sb * 128;
      const uint32_t aP = tmem + lane_off + C::COL_DP;
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t s[32], dp[32];
        tmem_ld32(aS + ch * 32, s);
        tmem_ld32(aP + ch * 32, dp);
        tmem_ld_wait();
        if (ch == 3) {
          tc_fence_before();
          mbar_arrive(&bar->dp_free);
        }
        uint32_t ds[16];
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          float v[2];
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            const bool kp = (keep[ch] >> (c + q)) & 1u;
            const float pr = kp ? ex2(fmaf(__uint_as_float(s[c + q]), sl2, -lse2)) : 0.f;
            v[q] = pr * (__uint_as_float(dp[c + q]) - dlt);
          }
          ds[c >> 1] = pack_bf16x2(v[0], v[1]);
        }
        // dS chunk ch lands in columns 16ch..16ch+15 of the S buffer (already read)
        uint32_t (&d16)[16] = ds;
        asm volatile(
            "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, "
            "%10, %11, %12, %13, %14, %15, %16};" ::"r"(aS + ch * 16),
            "r"(d16[0]), "r"(d16[1]), "r"(d16[2]), "r"(d16[3]), "r"(d16[4]), "r"(d16[5]),
            "r"(d16[6]), "r"(d16[7]), "r"(d16[8]), "r"(d16[9]), "r"(d16[10]), "r"(d16[11]),
            "r"(d16[12]), "r"(d16[13]), "r"(d16[14]), "r"(d16[15])
            : "memory");
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bar->ds_ready[sb]);
    }
    if (ok && __all_sync(0xffffffffu, mbar_wait(&bar->dq_done[(N - 1) & 1], ((N - 1) >> 1) & 1,
                                                p.err, abort_flag))) {
      tc_fence_after();
      __nv_bfloat16* drow = p.dq + (((size_t)b * p.L + (valid ? i : 0)) * p.Hq + h) * D;
#pragma unroll 1
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_off + C::COL_DQ + cc * 32, v);
        tmem_ld_wait();
        if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(drow + cc * 32);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint32_t w4[4];
#pragma unroll
            for (int z = 0; z < 4; ++z)
              w4[z] = pack_bf16x2(__uint_as_float(v[8 * q + 2 * z]) * p.scale,
                                  __uint_as_float(v[8 * q + 2 * z + 1]) * p.scale);
            dst[q] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
          }
        }
      }
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ dK/dV kernel
template <int D>
struct DkvCfg {
  static constexpr int KB = D / 64;
  static constexpr int TILE = KB * kBoxBytes;
  static constexpr int NST = 2;
  static constexpr int SMEM_TILES = TILE * (2 + 2 * NST);  // K, V, NST x (Q, dO)
  static constexpr int COL_S = 0, COL_DP = 128, COL_DV = 256, COL_DK = 256 + D;
};

template <int NST>
struct DkvBar {
  uint64_t kv_full;
  uint64_t q_full[NST], q_empty[NST];
  uint64_t s_full, pds_ready, mm_done;
  uint64_t drain;
  float lse2[NST][128];
  float delta[NST][128];
  int anchor_before;  // anchors at positions < 128u (window items)
  int warp_anchor[4];
  uint32_t tmem_base;
  int abort_flag;
};

template <int D>
constexpr size_t dkv_smem_bytes() {
  return 1024 + DkvCfg<D>::SMEM_TILES + sizeof(DkvBar<DkvCfg<D>::NST>);
}

__device__ __forceinline__ int count_lt_dev(const int32_t* __restrict__ idx, int cnt, long long x) {
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

template <int D>
__global__ void __launch_bounds__(192, 1) sep_attn_bwd_dkv_kernel(const __grid_constant__ BwdParams p,
                                                                 int nseg) {
  using C = DkvCfg<D>;
  constexpr int NST = C::NST;
  const int G = p.Hq / p.Hkv;
  const int kvh = blockIdx.y, b = blockIdx.z;
  const int item = blockIdx.x;
  const int cnt = p.anchor_cnt[b];
  const int32_t* ge_row = p.gather_end + (size_t)b * p.T;

  // ---- which key rows and which query tiles this CTA handles
  bool window;
  int u = 0, c = 0, t_begin, t_end;
  if (item < p.T) {
    window = true;
    u = p.T - 1 - item;
    t_begin = u;
    t_end = u;
    while (t_end + 1 < p.T && window_lo_tile(t_end + 1, p.n) <= u) ++t_end;
    ++t_end;
  } else {
    window = false;
    const int x = item - p.T;
    c = x / nseg;
    const int sg = x % nseg;
    if (c * 128 >= cnt) return;
    // first query tile that gathers anchor 128c: gather_end is non-decreasing in t
    int lo = 0, hi = p.T;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (ge_row[mid] > c * 128)
        hi = mid;
      else
        lo = mid + 1;
    }
    t_begin = lo + sg * kAnchorSeg;
    t_end = min(p.T, t_begin + kAnchorSeg);
    if (t_begin >= p.T) return;
  }
  const int npairs = (t_end - t_begin) * G;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sK = smem;
  uint8_t* sV = sK + C::TILE;
  uint8_t* sQ = sV + C::TILE;
  uint8_t* sdO = sQ + NST * C::TILE;
  DkvBar<NST>* bar = reinterpret_cast<DkvBar<NST>*>(sdO + NST * C::TILE);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort_flag = &bar->abort_flag;

  if (threadIdx.x == 0) {
    mbar_init(&bar->kv_full, 1);
    for (int s = 0; s < NST; ++s) {
      mbar_init(&bar->q_full[s], 1 + 32);
      mbar_init(&bar->q_empty[s], 1);
    }
    mbar_init(&bar->s_full, 1);
    mbar_init(&bar->pds_ready, 128);
    mbar_init(&bar->mm_done, 1);
    mbar_init(&bar->drain, 1);
    bar->abort_flag = 0;
    bar->anchor_before = window ? count_lt_dev(p.anchor_idx + (size_t)b * p.L, cnt, (long long)u * 128) : 0;
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(&bar->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar->tmem_base;

  if (warp == 4) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      mbar_arrive_expect_tx(&bar->kv_full, 2 * C::TILE);
      const int krow = window ? u * 128 : c * 128;
      for (int kb = 0; kb < C::KB; ++kb) {
        tma_load_4d(sK + kb * kBoxBytes, window ? &p.tmK : &p.tmKc, &bar->kv_full, kb * 64, kvh,
                    krow, b);
        tma_load_4d(sV + kb * kBoxBytes, window ? &p.tmV : &p.tmVc, &bar->kv_full, kb * 64, kvh,
                    krow, b);
      }
    }
    for (int q = 0; q < npairs; ++q) {
      const int st = q % NST, r = q / NST;
      const int t = t_begin + q / G, h = kvh * G + q % G;
      bool okw = true;
      if (r > 0) okw = mbar_wait(&bar->q_empty[st], (r - 1) & 1, p.err, abort_flag);
      if (!__all_sync(0xffffffffu, okw)) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(&bar->q_full[st], 2 * C::TILE);
        for (int kb = 0; kb < C::KB; ++kb) {
          tma_load_4d(sQ + st * C::TILE + kb * kBoxBytes, &p.tmQ, &bar->q_full[st], kb * 64, h,
                      t * 128, b);
          tma_load_4d(sdO + st * C::TILE + kb * kBoxBytes, &p.tmdO, &bar->q_full[st], kb * 64, h,
                      t * 128, b);
        }
      }
      // per-query statistics of this tile: log2-domain lse (+inf past L) and Delta
      const size_t base = ((size_t)b * p.Hq + h) * p.L;
#pragma unroll
      for (int z = 0; z < 4; ++z) {
        const int col = lane * 4 + z;
        const long long i = (long long)t * 128 + col;
        const bool v = i < p.L;
        bar->lse2[st][col] = v ? p.lse[base + i] * 1.4426950408889634f : INFINITY;
        bar->delta[st][col] = v ? p.delta[base + i] : 0.f;
      }
      mbar_arrive(&bar->q_full[st]);
    }
    if (lane == 0 && *abort_flag) {
      mbar_wait(&bar->kv_full, 0, nullptr, nullptr);
      for (int q = max(0, npairs - NST); q < npairs; ++q)
        mbar_wait(&bar->q_full[q % NST], (q / NST) & 1, nullptr, nullptr);
    }
  } else if (warp == 5) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = make_idesc_bf16(128, 128, false, false);
      constexpr uint32_t idG = make_idesc_bf16(128, D, false, true);
      const uint32_t sKa = smem_u32(sK), sVa = smem_u32(sV);
      const uint32_t sQa = smem_u32(sQ), sdOa = smem_u32(sdO);
      bool ok = mbar_wait(&bar->kv_full, 0, p.err, abort_flag);
      for (int q = 0; ok && q < npairs; ++q) {
        const int st = q % NST;
        if (!mbar_wait(&bar->q_full[st], (q / NST) & 1, p.err, abort_flag)) break;
        // S^T / dP^T columns are read (as P^T / dS^T) by the previous pair's gradient MMAs
        if (q > 0 && !mbar_wait(&bar->mm_done, (q - 1) & 1, p.err, abort_flag)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kBoxBytes + (kk & 3) * 32;
          mma_ss(tmem + C::COL_S, make_sdesc_sw128(sKa + off, 16, 1024),
                 make_sdesc_sw128(sQa + st * C::TILE + off, 16, 1024), idS, kk > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kBoxBytes + (kk & 3) * 32;
          mma_ss(tmem + C::COL_DP, make_sdesc_sw128(sVa + off, 16, 1024),
                 make_sdesc_sw128(sdOa + st * C::TILE + off, 16, 1024), idS, kk > 0 ? 1u : 0u);
        }
        tc_commit(&bar->s_full);
        if (!mbar_wait(&bar->pds_ready, q & 1, p.err, abort_flag)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 128 / 16; ++kk) {
          mma_ts(tmem + C::COL_DV, tmem + C::COL_S + kk * 8,
                 make_sdesc_sw128(sdOa + st * C::TILE + kk * 2048, kBoxBytes, 1024), idG,
                 (q > 0 || kk > 0) ? 1u : 0u);
          mma_ts(tmem + C::COL_DK, tmem + C::COL_DP + kk * 8,
                 make_sdesc_sw128(sQa + st * C::TILE + kk * 2048, kBoxBytes, 1024), idG,
                 (q > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(&bar->mm_done);
        tc_commit(&bar->q_empty[st]);
      }
      tc_commit(&bar->drain);
      mbar_wait(&bar->drain, 0, nullptr, nullptr);
    }
  } else {
    // ---------------------------------------------------------------- softmax warps (thread = key)
    const int krow = threadIdx.x;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const float sl2 = p.scale_log2;
    // this thread's key: position j (window) or compact anchor row r (gathered)
    const long long j = window ? (long long)u * 128 + krow : -1;
    const int r = window ? -1 : c * 128 + krow;
    bool fj = false;
    if (window && j < p.L) fj = (__ldg(p.anchor_bits + (size_t)b * p.W + (j >> 5)) >> (j & 31)) & 1u;
    bool ok = true;
    for (int q = 0; q < npairs; ++q) {
      const int st = q % NST;
      const int t = t_begin + q / G;
      if (!__all_sync(0xffffffffu, mbar_wait(&bar->s_full, q & 1, p.err, abort_flag))) {
        ok = false;
        break;
      }
      // q_full also covers the per-query statistics written by the producer warp
      if (!__all_sync(0xffffffffu, mbar_wait(&bar->q_full[st], (q / NST) & 1, p.err, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
      // keep bits over the 128 query columns of tile t for this key
      uint32_t keep[4];
      const long long q0 = (long long)t * 128;
      if (window) {
        const int cls = p.tile_map[((size_t)b * p.T + t) * p.T + u];
        if (j >= p.L) {
#pragma unroll
          for (int w = 0; w < 4; ++w) keep[w] = 0u;
        } else if (cls == SEP_TILE_FULL) {
#pragma unroll
          for (int w = 0; w < 4; ++w) keep[w] = 0xffffffffu;
        } else {
          // query i keeps j iff i >= j and (i - j < n or f[j])
          const long long lo = j - q0;
          const long long hi = fj ? 127 : j + p.n - 1 - q0;
#pragma unroll
          for (int w = 0; w < 4; ++w) keep[w] = range_word(lo, hi, w);
        }
      } else {
        const uint32_t all = (r < ge_row[t]) ? 0xffffffffu : 0u;
#pragma unroll
        for (int w = 0; w < 4; ++w) keep[w] = all;
      }
      const float* lse2 = bar->lse2[st];
      const float* dl = bar->delta[st];
      const uint32_t aS = tmem + lane_off + C::COL_S;
      const uint32_t aP = tmem + lane_off + C::COL_DP;
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t s[32], dp[32];
        tmem_ld32(aS + ch * 32, s);
        tmem_ld32(aP + ch * 32, dp);
        tmem_ld_wait();
        uint32_t pk[16], dk16[16];
#pragma unroll
        for (int cc = 0; cc < 32; cc += 2) {
          float pv[2], dv2[2];
#pragma unroll
          for (int z = 0; z < 2; ++z) {
            const int col = ch * 32 + cc + z;
            const bool kp = (keep[ch] >> (cc + z)) & 1u;
            const float pr = kp ? ex2(fmaf(__uint_as_float(s[cc + z]), sl2, -lse2[col])) : 0.f;
            pv[z] = pr;
            dv2[z] = pr * (__uint_as_float(dp[cc + z]) - dl[col]);
          }
          pk[cc >> 1] = pack_bf16x2(pv[0], pv[1]);
          dk16[cc >> 1] = pack_bf16x2(dv2[0], dv2[1]);
        }
        asm volatile(
            "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, "
            "%10, %11, %12, %13, %14, %15, %16};" ::"r"(aS + ch * 16),
            "r"(pk[0]), "r"(pk[1]), "r"(pk[2]), "r"(pk[3]), "r"(pk[4]), "r"(pk[5]), "r"(pk[6]),
            "r"(pk[7]), "r"(pk[8]), "r"(pk[9]), "r"(pk[10]), "r"(pk[11]), "r"(pk[12]),
            "r"(pk[13]), "r"(pk[14]), "r"(pk[15])
            : "memory");
        asm volatile(
            "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, "
            "%10, %11, %12, %13, %14, %15, %16};" ::"r"(aP + ch * 16),
            "r"(dk16[0]), "r"(dk16[1]), "r"(dk16[2]), "r"(dk16[3]), "r"(dk16[4]), "r"(dk16[5]),
            "r"(dk16[6]), "r"(dk16[7]), "r"(dk16[8]), "r"(dk16[9]), "r"(dk16[10]),
            "r"(dk16[11]), "r"(dk16[12]), "r"(dk16[13]), "r"(dk16[14]), "r"(dk16[15])
            : "memory");
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bar->pds_ready);
    }
    // ---- epilogue: dV and dK rows of this key
    // compact index of this key if it is an anchor (window items): anchors before the tile plus
    // anchors before it inside the tile
    const unsigned ball = __ballot_sync(0xffffffffu, fj);
    if (lane == 0) bar->warp_anchor[warp] = __popc(ball);
    asm volatile("bar.sync 1, 128;" ::: "memory");
    int cidx = -1;
    if (window && fj) {
      int before = bar->anchor_before + __popc(ball & ((1u << lane) - 1u));
      for (int w = 0; w < warp; ++w) before += bar->warp_anchor[w];
      cidx = before;
    } else if (!window && r < cnt) {
      cidx = r;
    }
    if (ok && npairs > 0 &&
        __all_sync(0xffffffffu, mbar_wait(&bar->mm_done, (npairs - 1) & 1, p.err, abort_flag))) {
      tc_fence_after();
      const bool write_direct = window && j < p.L && !fj;
#pragma unroll 1
      for (int part = 0; part < 2; ++part) {  // 0: dV, 1: dK
        const float mul = part ? p.scale : 1.f;
        const uint32_t col0 = part ? C::COL_DK : C::COL_DV;
#pragma unroll 1
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t v[32];
          tmem_ld32(tmem + lane_off + col0 + cc * 32, v);
          tmem_ld_wait();
          if (write_direct) {
            __nv_bfloat16* dst = (part ? p.dk : p.dv) + (((size_t)b * p.L + j) * p.Hkv + kvh) * D + cc * 32;
            uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
            for (int z = 0; z < 4; ++z) {
              uint32_t w4[4];
#pragma unroll
              for (int y = 0; y < 4; ++y)
                w4[y] = pack_bf16x2(__uint_as_float(v[8 * z + 2 * y]) * mul,
                                    __uint_as_float(v[8 * z + 2 * y + 1]) * mul);
              d4[z] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
            }
          } else if (cidx >= 0) {
            float* dst = (part ? p.dka : p.dva) + (((size_t)b * p.L + cidx) * p.Hkv + kvh) * D + cc * 32;
#pragma unroll
            for (int z = 0; z < 8; ++z) {
              atomicAdd(reinterpret_cast<float4*>(dst) + z,
                        make_float4(__uint_as_float(v[4 * z]) * mul, __uint_as_float(v[4 * z + 1]) * mul,
                                    __uint_as_float(v[4 * z + 2]) * mul, __uint_as_float(v[4 * z + 3]) * mul));
            }
          }
        }
      }
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ anchor combine
// dK/dV rows of the anchors: the fp32 sums of every part, rounded once to bf16.
__global__ void __launch_bounds__(256) anchor_combine_kernel(
    const int32_t* __restrict__ anchor_idx, const int32_t* __restrict__ anchor_cnt, int L,
    int rowlen, int rows_per_cta, const float* __restrict__ dka, const float* __restrict__ dva,
    __nv_bfloat16* __restrict__ dk, __nv_bfloat16* __restrict__ dv) {
  const int b = blockIdx.y;
  const int cnt = anchor_cnt[b];
  const int r0 = blockIdx.x * rows_per_cta;
  if (r0 >= cnt) return;
  const int rows = min(rows_per_cta, cnt - r0);
  const int q4 = rowlen / 4;
  for (int e = threadIdx.x; e < rows * q4; e += blockDim.x) {
    const int r = r0 + e / q4, z = e % q4;
    const size_t src = ((size_t)b * L + r) * rowlen + z * 4;
    const size_t dst = ((size_t)b * L + anchor_idx[(size_t)b * L + r]) * rowlen + z * 4;
    const float4 x = *reinterpret_cast<const float4*>(dka + src);
    const float4 y = *reinterpret_cast<const float4*>(dva + src);
    *reinterpret_cast<uint2*>(dk + dst) = make_uint2(pack_bf16x2(x.x, x.y), pack_bf16x2(x.z, x.w));
    *reinterpret_cast<uint2*>(dv + dst) = make_uint2(pack_bf16x2(y.x, y.y), pack_bf16x2(y.z, y.w));
  }
}

cudaError_t launch_attn_bwd(const AttnMaps& maps, const AttnShape& s, const uint32_t* anchor_bits,
                            const int32_t* anchor_idx, const int32_t* anchor_cnt,
                            const int32_t* gather_end, const int8_t* tile_map, const void* o,
                            const float* lse, const void* dout, const void* q, const void* k,
                            const void* v, void* dq, void* dk, void* dv, void* kc, void* vc,
                            float* delta, float* dka, float* dva, int stages,
                            cudaStream_t stream) {
  (void)q;
  cudaError_t e = cudaSuccess;
  if (stages & kBwdPrep) {
  e = launch_compact_anchors(k, v, anchor_idx, anchor_cnt, s.B, s.L, s.Hkv, s.d, kc, vc, stream);
  if (e != cudaSuccess) return e;
  {
    const int rowvec = s.Hkv * s.d / 4;
    dim3 grid((s.L + 31) / 32, s.B);
    zero_anchor_partials_kernel<<<grid, 256, 0, stream>>>(anchor_cnt, s.L, rowvec, 32,
                                                          reinterpret_cast<float4*>(dka),
                                                          reinterpret_cast<float4*>(dva));
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  {
    const long long rows = (long long)s.B * s.L * s.Hq;
    const unsigned blocks = (unsigned)((rows + 255) / 256);
    if (s.d == 128)
      delta_kernel<128><<<blocks, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(o),
                                                    static_cast<const __nv_bfloat16*>(dout), s.B,
                                                    s.L, s.Hq, delta);
    else
      delta_kernel<64><<<blocks, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(o),
                                                   static_cast<const __nv_bfloat16*>(dout), s.B,
                                                   s.L, s.Hq, delta);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  }
  if (!(stages & (kBwdDq | kBwdDkv))) return cudaSuccess;
  BwdParams prm;
  prm.tmQ = maps.q;
  prm.tmK = maps.k;
  prm.tmV = maps.v;
  prm.tmKc = maps.kc;
  prm.tmVc = maps.vc;
  prm.tmdO = maps.dout;
  prm.anchor_bits = anchor_bits;
  prm.anchor_idx = anchor_idx;
  prm.anchor_cnt = anchor_cnt;
  prm.gather_end = gather_end;
  prm.tile_map = tile_map;
  prm.lse = lse;
  prm.delta = delta;
  prm.dq = static_cast<__nv_bfloat16*>(dq);
  prm.dk = static_cast<__nv_bfloat16*>(dk);
  prm.dv = static_cast<__nv_bfloat16*>(dv);
  prm.dka = dka;
  prm.dva = dva;
  prm.err = device_error_word();
  prm.B = s.B;
  prm.L = s.L;
  prm.Hq = s.Hq;
  prm.Hkv = s.Hkv;
  prm.T = (s.L + 127) / 128;
  prm.W = (s.L + 31) / 32;
  prm.a = s.a;
  prm.n = s.n;
  prm.scale = s.scale;
  prm.scale_log2 = s.scale * 1.4426950408889634f;
  const int nseg = (prm.T + kAnchorSeg - 1) / kAnchorSeg;
  const int nchunks = prm.T;  // anchor chunks of 128 rows: at most ceil(L / 128)
  dim3 grid_q(prm.T, s.Hq, s.B);
  dim3 grid_kv(prm.T + nchunks * nseg, s.Hkv, s.B);
  if (s.d == 128) {
    constexpr size_t smq = dq_smem_bytes<128>(), smkv = dkv_smem_bytes<128>();
    static_assert(smq <= 227 * 1024 && smkv <= 227 * 1024, "shared memory budget");
    static bool attr_set[64] = {false};  // per device: set once, outside any stream capture
    int dev = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if (dev < 0 || dev >= 64 || !attr_set[dev]) {
      if ((e = cudaFuncSetAttribute(sep_attn_bwd_dq_kernel<128>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smq)) != cudaSuccess)
        return e;
      if ((e = cudaFuncSetAttribute(sep_attn_bwd_dkv_kernel<128>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smkv)) != cudaSuccess)
        return e;
      if (dev >= 0 && dev < 64) attr_set[dev] = true;
    }
    if (stages & kBwdDq) sep_attn_bwd_dq_kernel<128><<<grid_q, 192, smq, stream>>>(prm);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (stages & kBwdDkv) sep_attn_bwd_dkv_kernel<128><<<grid_kv, 192, smkv, stream>>>(prm, nseg);
  } else {
    constexpr size_t smq = dq_smem_bytes<64>(), smkv = dkv_smem_bytes<64>();
    static_assert(smq <= 227 * 1024 && smkv <= 227 * 1024, "shared memory budget");
    static bool attr_set[64] = {false};  // per device: set once, outside any stream capture
    int dev = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if (dev < 0 || dev >= 64 || !attr_set[dev]) {
      if ((e = cudaFuncSetAttribute(sep_attn_bwd_dq_kernel<64>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smq)) != cudaSuccess)
        return e;
      if ((e = cudaFuncSetAttribute(sep_attn_bwd_dkv_kernel<64>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smkv)) != cudaSuccess)
        return e;
      if (dev >= 0 && dev < 64) attr_set[dev] = true;
    }
    if (stages & kBwdDq) sep_attn_bwd_dq_kernel<64><<<grid_q, 192, smq, stream>>>(prm);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (stages & kBwdDkv) sep_attn_bwd_dkv_kernel<64><<<grid_kv, 192, smkv, stream>>>(prm, nseg);
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (stages & kBwdDkv) {
    dim3 grid((s.L + 31) / 32, s.B);
    anchor_combine_kernel<<<grid, 256, 0, stream>>>(anchor_idx, anchor_cnt, s.L, s.Hkv * s.d, 32,
                                                    dka, dva, static_cast<__nv_bfloat16*>(dk),
                                                    static_cast<__nv_bfloat16*>(dv));
  }
  return cudaGetLastError();
}

}  // namespace sep
