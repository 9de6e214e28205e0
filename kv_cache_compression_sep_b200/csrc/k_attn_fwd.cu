// sep_attn_fwd: separator-sparse causal attention forward on sm_100a (tcgen05 + TMEM + TMA).
//
// Computes O = M(A, V, M_b) ("How SepLLM reorchestrates the language model...", section
// "SepLLM's Architecture: Composing Efficiency"): softmax attention where query i keeps key j
// iff j <= i && (i - j < n || f[j]), f = initial-or-separator ("SepLLM: Accelerate Large
// Language Models ...", atlas.scime.ai summary, "Approach").
//
// One CTA per (query tile t of 128 rows, query head h, batch b). Its keys are split in two
// disjoint parts that together hold every kept key exactly once:
//   * window tiles u = t, t-1, ..., lo(t), lo(t) = max(0, 128t - n + 1) / 128: whole 128-key
//     tiles loaded by TMA in tile mode; FULL tiles need no mask, PARTIAL tiles apply keep()
//     element-wise;
//   * anchors left of tile lo(t): the first gather_end[t] anchors, kept by every row of the
//     tile, read in chunks of 128 from a compacted copy (rows 0..cnt-1 of kc/vc) so that they
//     too arrive as TMA tiles.
// Skipped tiles are never loaded.
//
// Warp roles (192 threads): warps 0-3 softmax (thread = query row = TMEM lane), warp 4 TMA
// producer, warp 5 TMEM allocator + MMA issuer (one thread). Per key tile j:
//   S_j = Q K_j^T                  (tcgen05.mma, A and B K-major in smem, D in TMEM S[j%2])
//   P_j = exp2(S_j*c - m)          (softmax warps: tcgen05.ld S, online max with lazy
//                                   rescale of O, tcgen05.st of bf16 P into TMEM P[j%2])
//   O  += P_j V_j                  (tcgen05.mma, A = P from TMEM, B = V MN-major in smem)
// S_{j+1} is issued before PV_j so the tensor core works while softmax runs.
#include <cuda_runtime.h>

#include "sep_common.cuh"
#include "sep_launch.h"
#include "sep_tiles.cuh"

namespace sep {

struct FwdParams {
  CUtensorMap tmQ, tmK, tmV, tmKc, tmVc;
  const uint8_t* sep;
  const int32_t* gather_end;
  const int8_t* tile_map;
  __nv_bfloat16* o;
  float* lse;
  unsigned* err;
  int B, L, Hq, Hkv, T, a, n;
  float scale_log2;
};

template <int D>
struct FwdCfg {
  static constexpr int BM = 128, BN = 128;
  static constexpr int KB = D / 64;                 // 128-byte column boxes per row
  static constexpr int BOX_BYTES = 128 * 64 * 2;    // one [128 rows][64 cols] bf16 box
  static constexpr int TILE_BYTES = KB * BOX_BYTES; // one [128][D] tile
  static constexpr int NST = (D == 128) ? 2 : 4;    // K/V pipeline stages (1 CTA per SM)
  static constexpr int SMEM_TILES = TILE_BYTES * (1 + 2 * NST);
  static constexpr int TMEM_COLS = 512;
  static constexpr int COL_S = 0;      // S[0], S[1]: 128 fp32 columns each
  static constexpr int COL_O = 256;    // O: D fp32 columns
  static constexpr int COL_P = 384;    // P[0], P[1]: 64 columns each (bf16 pairs)
};

template <int NST>
struct FwdBar {
  uint64_t q_full;
  uint64_t k_full[NST], k_empty[NST], v_full[NST], v_empty[NST];
  uint64_t s_full[2], p_ready[2], pv_done[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

template <int D>
constexpr size_t fwd_smem_bytes() {
  return 1024 /*alignment slack*/ + FwdCfg<D>::SMEM_TILES + sizeof(FwdBar<FwdCfg<D>::NST>);
}

template <int D>
__global__ void __launch_bounds__(192, 1) sep_attn_fwd_kernel(const __grid_constant__ FwdParams p) {
  using C = FwdCfg<D>;
  constexpr int NST = C::NST;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + C::TILE_BYTES;
  uint8_t* sV = sK + NST * C::TILE_BYTES;
  FwdBar<NST>* bar = reinterpret_cast<FwdBar<NST>*>(sV + NST * C::TILE_BYTES);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = p.T - 1 - (int)blockIdx.x;  // heaviest query tiles first
  const int h = blockIdx.y, b = blockIdx.z;
  const int kvh = h / (p.Hq / p.Hkv);
  const int lo_tile = window_lo_tile(t, p.n);
  const int nwin = t - lo_tile + 1;
  const int ge = p.gather_end[(size_t)b * p.T + t];
  const int ngat = (ge + C::BN - 1) / C::BN;
  const int N = nwin + ngat;
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
      mbar_init(&bar->p_ready[s], 128);
      mbar_init(&bar->pv_done[s], 1);
    }
    mbar_init(&bar->drain, 1);
    bar->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(&bar->tmem_base, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar->tmem_base;

  if (warp == 4) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&p.tmQ);
      tma_prefetch_desc(&p.tmK);
      tma_prefetch_desc(&p.tmV);
      mbar_arrive_expect_tx(&bar->q_full, C::TILE_BYTES);
      for (int kb = 0; kb < C::KB; ++kb)
        tma_load_4d(sQ + kb * C::BOX_BYTES, &p.tmQ, &bar->q_full, kb * 64, h, t * C::BM, b);
      for (int j = 0; j < N; ++j) {
        const int st = j % NST, r = j / NST;
        const bool win = j < nwin;
        const CUtensorMap* mk = win ? &p.tmK : &p.tmKc;
        const CUtensorMap* mv = win ? &p.tmV : &p.tmVc;
        const int row0 = win ? (t - j) * C::BN : (j - nwin) * C::BN;
        if (r > 0 && !mbar_wait(&bar->k_empty[st], (r - 1) & 1, p.err, abort_flag)) break;
        mbar_arrive_expect_tx(&bar->k_full[st], C::TILE_BYTES);
        for (int kb = 0; kb < C::KB; ++kb)
          tma_load_4d(sK + st * C::TILE_BYTES + kb * C::BOX_BYTES, mk, &bar->k_full[st], kb * 64,
                      kvh, row0, b);
        if (r > 0 && !mbar_wait(&bar->v_empty[st], (r - 1) & 1, p.err, abort_flag)) {
          // K of this tile is in flight: let it land before leaving
          mbar_wait(&bar->k_full[st], r & 1, nullptr, nullptr);
          break;
        }
        mbar_arrive_expect_tx(&bar->v_full[st], C::TILE_BYTES);
        for (int kb = 0; kb < C::KB; ++kb)
          tma_load_4d(sV + st * C::TILE_BYTES + kb * C::BOX_BYTES, mv, &bar->v_full[st], kb * 64,
                      kvh, row0, b);
      }
      if (*abort_flag) {
        // drain: wait (bounded) until every issued load has landed
        mbar_wait(&bar->q_full, 0, nullptr, nullptr);
        for (int j = max(0, N - NST); j < N; ++j) {
          mbar_wait(&bar->k_full[j % NST], (j / NST) & 1, nullptr, nullptr);
          mbar_wait(&bar->v_full[j % NST], (j / NST) & 1, nullptr, nullptr);
        }
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = make_idesc_bf16(128, 128, false, false);
      constexpr uint32_t idO = make_idesc_bf16(128, D, false, true);
      const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK), sVa = smem_u32(sV);
      bool ok = mbar_wait(&bar->q_full, 0, p.err, abort_flag);
      auto issue_S = [&](int j) -> bool {
        const int st = j % NST;
        if (!mbar_wait(&bar->k_full[st], (j / NST) & 1, p.err, abort_flag)) return false;
        tc_fence_after();
        const uint32_t dS = tmem + C::COL_S + (j & 1) * 128;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::BOX_BYTES + (kk & 3) * 32;
          const uint64_t ad = make_sdesc_sw128(sQa + off, 16, 1024);
          const uint64_t bd = make_sdesc_sw128(sKa + st * C::TILE_BYTES + off, 16, 1024);
          mma_ss(dS, ad, bd, idS, kk > 0 ? 1u : 0u);
        }
        tc_commit(&bar->s_full[j & 1]);
        tc_commit(&bar->k_empty[st]);
        return true;
      };
      auto issue_PV = [&](int j) -> bool {
        const int st = j % NST;
        if (!mbar_wait(&bar->p_ready[j & 1], (j >> 1) & 1, p.err, abort_flag)) return false;
        if (!mbar_wait(&bar->v_full[st], (j / NST) & 1, p.err, abort_flag)) return false;
        tc_fence_after();
        const uint32_t aP = tmem + C::COL_P + (j & 1) * 64;
#pragma unroll
        for (int kk = 0; kk < 128 / 16; ++kk) {
          const uint64_t bd =
              make_sdesc_sw128(sVa + st * C::TILE_BYTES + kk * 2048, C::BOX_BYTES, 1024);
          mma_ts(tmem + C::COL_O, aP + kk * 8, bd, idO, (j > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(&bar->pv_done[j & 1]);
        tc_commit(&bar->v_empty[st]);
        return true;
      };
      if (ok) ok = issue_S(0);
      for (int j = 0; ok && j < N; ++j) {
        if (j + 1 < N && !issue_S(j + 1)) break;
        if (!issue_PV(j)) break;
      }
      // make sure every MMA issued has completed before TMEM is released
      tc_commit(&bar->drain);
      mbar_wait(&bar->drain, 0, nullptr, nullptr);
    }
  } else {
    // ------------------------------------------------------------ softmax warpgroup
    const int row = threadIdx.x;  // 0..127 = TMEM lane
    const long long i = (long long)t * C::BM + row;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const uint8_t* sep_row = p.sep + (size_t)b * p.L;
    const int8_t* tmap = p.tile_map + ((size_t)b * p.T + t) * p.T;
    const float sl2 = p.scale_log2;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < N; ++j) {
      const int sb = j & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&bar->s_full[sb], (j >> 1) & 1, p.err, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t s[128];
      {
        uint32_t (&c0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&s[0]);
        uint32_t (&c1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&s[32]);
        uint32_t (&c2)[32] = *reinterpret_cast<uint32_t(*)[32]>(&s[64]);
        uint32_t (&c3)[32] = *reinterpret_cast<uint32_t(*)[32]>(&s[96]);
        const uint32_t a0 = tmem + lane_off + C::COL_S + sb * 128;
        tmem_ld32(a0, c0);
        tmem_ld32(a0 + 32, c1);
        tmem_ld32(a0 + 64, c2);
        tmem_ld32(a0 + 96, c3);
        tmem_ld_wait();
      }
      // ---- mask
      uint32_t keep[4] = {0xffffffffu, 0xffffffffu, 0xffffffffu, 0xffffffffu};
      bool masked = false;
      if (j < nwin) {
        const int u = t - j;
        const long long k0 = (long long)u * C::BN;
        const int cls = tmap[u];
        if (cls != SEP_TILE_FULL) {
          masked = true;
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            const uint32_t fb = anchor_bits32(sep_row, k0 + 32 * w, p.L, p.a);
            keep[w] = window_keep_word(w, i, k0, p.n, p.L, fb);
          }
        } else if (k0 + C::BN > p.L) {
          masked = true;
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            const long long hi = (long long)p.L - 1 - (k0 + 32 * w);
            keep[w] = (hi < 0) ? 0u : (hi >= 31 ? 0xffffffffu : ((2u << hi) - 1u));
          }
        }
      } else {
        const int rem = ge - (j - nwin) * C::BN;  // valid anchors in this chunk
        if (rem < C::BN) {
          masked = true;
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            const int hi = rem - 1 - 32 * w;
            keep[w] = (hi < 0) ? 0u : (hi >= 31 ? 0xffffffffu : ((2u << hi) - 1u));
          }
        }
      }
      float mx = -INFINITY;
      if (masked) {
#pragma unroll
        for (int c = 0; c < 128; ++c) {
          const float v = ((keep[c >> 5] >> (c & 31)) & 1u) ? __uint_as_float(s[c]) : -INFINITY;
          s[c] = __float_as_uint(v);
          mx = fmaxf(mx, v);
        }
      } else {
#pragma unroll
        for (int c = 0; c < 128; ++c) mx = fmaxf(mx, __uint_as_float(s[c]));
      }
      // ---- online max with lazy rescale (only when the max grows by more than 2^8)
      const float m_tile = mx * sl2;
      if (j == 0) {
        m_run = m_tile;
      } else {
        const bool need = m_tile > m_run + 8.0f;
        if (__any_sync(0xffffffffu, need)) {
          if (!__all_sync(0xffffffffu, mbar_wait(&bar->pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1,
                                                 p.err, abort_flag))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const float alpha = need ? ex2(m_run - m_tile) : 1.0f;
#pragma unroll 1
          for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t ov[32];
            const uint32_t ao = tmem + lane_off + C::COL_O + cc * 32;
            tmem_ld32(ao, ov);
            tmem_ld_wait();
#pragma unroll
            for (int q = 0; q < 32; ++q) ov[q] = __float_as_uint(__uint_as_float(ov[q]) * alpha);
            tmem_st32(ao, ov);
          }
          tmem_st_wait();
          if (need) {
            l_run *= alpha;
            m_run = m_tile;
          }
        }
      }
      const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
      // ---- P = exp2(S * scale*log2e - m), row sum, pack to bf16 pairs
      uint32_t pk[64];
      float sum = 0.f;
#pragma unroll
      for (int c = 0; c < 128; c += 2) {
        const float e0 = ex2(fmaf(__uint_as_float(s[c]), sl2, -m_use));
        const float e1 = ex2(fmaf(__uint_as_float(s[c + 1]), sl2, -m_use));
        sum += e0 + e1;
        pk[c >> 1] = pack_bf16x2(e0, e1);
      }
      l_run += sum;
      // P[j%2] was read by PV_{j-2}: wait for it before overwriting
      if (j >= 2 && !__all_sync(0xffffffffu, mbar_wait(&bar->pv_done[sb], ((j - 2) >> 1) & 1,
                                                     p.err, abort_flag))) {
        ok = false;
        break;
      }
      {
        const uint32_t ap = tmem + lane_off + C::COL_P + sb * 64;
        tmem_st32(ap, *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
        tmem_st32(ap + 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[32]));
        tmem_st_wait();
      }
      tc_fence_before();
      mbar_arrive(&bar->p_ready[sb]);
    }
    // ---- epilogue: O / l, LSE
    if (ok && __all_sync(0xffffffffu, mbar_wait(&bar->pv_done[(N - 1) & 1], ((N - 1) >> 1) & 1,
                                                p.err, abort_flag))) {
      tc_fence_after();
      const float inv_l = 1.0f / l_run;
      const bool valid = i < p.L;
      __nv_bfloat16* orow = p.o + (((size_t)b * p.L + (valid ? i : 0)) * p.Hq + h) * D;
#pragma unroll 1
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t ov[32];
        tmem_ld32(tmem + lane_off + C::COL_O + cc * 32, ov);
        tmem_ld_wait();
        uint32_t pkd[16];
#pragma unroll
        for (int q = 0; q < 16; ++q)
          pkd[q] = pack_bf16x2(__uint_as_float(ov[2 * q]) * inv_l,
                               __uint_as_float(ov[2 * q + 1]) * inv_l);
        if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(orow + cc * 32);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            dst[q] = make_uint4(pkd[4 * q], pkd[4 * q + 1], pkd[4 * q + 2], pkd[4 * q + 3]);
        }
      }
      if (valid)
        p.lse[((size_t)b * p.Hq + h) * p.L + i] = (m_run + __log2f(l_run)) * 0.69314718055994531f;
    }
    tc_fence_before();
  }

  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------------ anchor compaction
// Row r < anchor_cnt[b] of kc/vc receives the K/V row of anchor r; rows from anchor_cnt[b] up to
// the next multiple of 128 are zeroed so that the last (partly valid) anchor chunk holds finite
// values (masked scores still multiply V in the P*V product).
__global__ void __launch_bounds__(256) compact_anchors_kernel(
    const uint4* __restrict__ k, const uint4* __restrict__ v, const int32_t* __restrict__ anchor_idx,
    const int32_t* __restrict__ anchor_cnt, int L, int rowvec, int rows_per_cta,
    uint4* __restrict__ kc, uint4* __restrict__ vc) {
  const int b = blockIdx.y;
  const int cnt = anchor_cnt[b];
  const int pad_end = min(L, (cnt + 127) / 128 * 128);
  const int r0 = blockIdx.x * rows_per_cta;
  if (r0 >= pad_end) return;
  const int rows = min(rows_per_cta, pad_end - r0);
  const int32_t* idx = anchor_idx + (size_t)b * L;
  for (int e = threadIdx.x; e < rows * rowvec; e += blockDim.x) {
    const int r = r0 + e / rowvec, c = e % rowvec;
    const size_t dst = ((size_t)b * L + r) * rowvec + c;
    if (r < cnt) {
      const size_t src = ((size_t)b * L + idx[r]) * rowvec + c;
      kc[dst] = __ldg(k + src);
      vc[dst] = __ldg(v + src);
    } else {
      kc[dst] = make_uint4(0, 0, 0, 0);
      vc[dst] = make_uint4(0, 0, 0, 0);
    }
  }
}

cudaError_t launch_compact_anchors(const void* k, const void* v, const int32_t* anchor_idx,
                                   const int32_t* anchor_cnt, int B, int L, int Hkv, int d,
                                   void* kc, void* vc, cudaStream_t stream) {
  const int rowvec = Hkv * d * 2 / 16;
  const int rows_per_cta = 32;
  dim3 grid((L + rows_per_cta - 1) / rows_per_cta, B);
  compact_anchors_kernel<<<grid, 256, 0, stream>>>(
      static_cast<const uint4*>(k), static_cast<const uint4*>(v), anchor_idx, anchor_cnt, L,
      rowvec, rows_per_cta, static_cast<uint4*>(kc), static_cast<uint4*>(vc));
  return cudaGetLastError();
}

template <int D>
static cudaError_t launch_fwd_t(const FwdParams& prm, int T, int Hq, int B, cudaStream_t stream) {
  constexpr size_t smem = fwd_smem_bytes<D>();
  static_assert(smem <= 227 * 1024, "shared memory budget");
  static bool attr_set[64] = {false};  // per device: set once, outside any stream capture
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    e = cudaFuncSetAttribute(sep_attn_fwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  sep_attn_fwd_kernel<D><<<dim3(T, Hq, B), 192, smem, stream>>>(prm);
  return cudaGetLastError();
}

cudaError_t launch_attn_fwd(const AttnMaps& maps, const AttnShape& s, const uint8_t* sep,
                            const int32_t* gather_end, const int8_t* tile_map, void* o,
                            float* lse, cudaStream_t stream) {
  FwdParams prm;
  prm.tmQ = maps.q;
  prm.tmK = maps.k;
  prm.tmV = maps.v;
  prm.tmKc = maps.kc;
  prm.tmVc = maps.vc;
  prm.sep = sep;
  prm.gather_end = gather_end;
  prm.tile_map = tile_map;
  prm.o = static_cast<__nv_bfloat16*>(o);
  prm.lse = lse;
  prm.err = device_error_word();
  prm.B = s.B;
  prm.L = s.L;
  prm.Hq = s.Hq;
  prm.Hkv = s.Hkv;
  prm.T = (s.L + 127) / 128;
  prm.a = s.a;
  prm.n = s.n;
  prm.scale_log2 = s.scale * 1.4426950408889634f;
  if (s.d == 128) return launch_fwd_t<128>(prm, prm.T, s.Hq, s.B, stream);
  if (s.d == 64) return launch_fwd_t<64>(prm, prm.T, s.Hq, s.B, stream);
  return cudaErrorInvalidValue;
}

}  // namespace sep
