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
//   1. prep (one warp per position): compacted anchor K/V rows (as the forward), zeroed fp32
//      anchor partials, Delta = rowsum(dO * O); then the dK/dV work list (bwd_schedule_kernel).
//   2. dQ (query-major, persistent over the forward's item order and key tiles): S = Q K^T and
//      dP = dO V^T into TMEM, dS = P (dP - Delta) written back to TMEM as bf16,
//      dQ += dS K (A from TMEM, B = K MN-major); a storer warp writes the dQ tile.
//   3. dK/dV (key-major, persistent, items fetched dynamically, heaviest first): work items
//      are window key tiles u (all query tiles t with lo(t) <= u <= t) and (anchor chunk c,
//      segment of query tiles that gather it). Per (query tile, query head), in two 64-row query halves:
//      S^T = K Q^T, dP^T = V dO^T into TMEM; P^T and dS^T back to TMEM as bf16;
//      dV += P^T dO, dK += dS^T Q. Non-anchor keys of a window tile get their complete gradient
//      and leave as bf16 through a storer warp's TMA store; anchor keys are summed in fp32
//      (window part + every gathered part) in a compact [B, anchors, Hkv, d] buffer.
//   4. combine: anchor partials to bf16 dK/dV at the anchors' positions.
#include <cuda_runtime.h>
#include <cstddef>
#include <type_traits>

#include "sep_common.cuh"
#include "sep_launch.h"
#include "sep_tiles.cuh"

namespace sep {

constexpr int kBoxBytes = 128 * 64 * 2;

// ------------------------------------------------------------------ prep kernel
// One warp per position i of one sequence b (8 per CTA), all in one pass:
//   Delta[b][h][i] = sum_c dO[b,i,h,c] * O[b,i,h,c] for every query head h (the O and dO rows of
//   position i are Hq * d contiguous bf16: 16-byte chunks, D / 8 consecutive chunks per head,
//   summed over the D / 8 lanes that hold them);
//   row i of the compacted anchor K / V (i < cnt + 128: the 128 rows after the last anchor are
//   zeros, for the anchor chunks of the dQ pass that start at 64 + a multiple of 128);
//   zero row i of the compact fp32 anchor partials (i < cnt);
//   and the four work-list counters (block 0).
template <int D>
__global__ void __launch_bounds__(256) bwd_prep_kernel(
    const uint4* __restrict__ o, const uint4* __restrict__ dout, const uint4* __restrict__ k,
    const uint4* __restrict__ v, const int32_t* __restrict__ anchor_idx,
    const int32_t* __restrict__ anchor_cnt, int L, int Hq, int Hkv,
    uint4* __restrict__ kc, uint4* __restrict__ vc, float4* __restrict__ dka,
    float4* __restrict__ dva, float* __restrict__ delta, int32_t* __restrict__ counters) {
  grid_dep_wait();
  grid_dep_launch_next();
  constexpr int CPH = D / 8;  // 16-byte chunks per head; divides 32
  const int b = blockIdx.y;
  const int lane = threadIdx.x & 31;
  const int i = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (blockIdx.x == 0 && b == 0 && threadIdx.x < 4) counters[threadIdx.x] = 0;
  if (i >= L) return;
  const size_t row = (size_t)b * L + i;
  const int nch = Hq * CPH;
  const uint4* po = o + row * nch;
  const uint4* pd = dout + row * nch;
  // groups of up to kRounds 32-chunk rounds: every load of a group is issued before any of
  // its reductions, so a warp keeps several 16-byte loads of O and dO in flight
  constexpr int kRounds = 4;
  for (int g0 = 0; g0 < nch; g0 += 32 * kRounds) {
    uint4 xv[kRounds], yv[kRounds];
#pragma unroll
    for (int r = 0; r < kRounds; ++r) {
      const int c = g0 + 32 * r + lane;
      if (c < nch) {
        xv[r] = __ldg(po + c);
        yv[r] = __ldg(pd + c);
      } else {
        xv[r] = yv[r] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
#pragma unroll
    for (int r = 0; r < kRounds; ++r) {
      const int c = g0 + 32 * r + lane;
      if (g0 + 32 * r >= nch) break;  // warp-uniform
      const uint32_t xs[4] = {xv[r].x, xv[r].y, xv[r].z, xv[r].w};
      const uint32_t ys[4] = {yv[r].x, yv[r].y, yv[r].z, yv[r].w};
      float acc = 0.f;
#pragma unroll
      for (int z = 0; z < 4; ++z) {
        const __nv_bfloat162 a2 = *reinterpret_cast<const __nv_bfloat162*>(&xs[z]);
        const __nv_bfloat162 b2 = *reinterpret_cast<const __nv_bfloat162*>(&ys[z]);
        acc = fmaf(__low2float(a2), __low2float(b2), acc);
        acc = fmaf(__high2float(a2), __high2float(b2), acc);
      }
#pragma unroll
      for (int off = CPH / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
      if (c < nch && (lane % CPH) == 0) delta[((size_t)b * Hq + c / CPH) * L + i] = acc;
    }
  }
  const int cnt = __ldg(anchor_cnt + b);
  if (i < min(L, cnt + 128))
    compact_anchor_row(k, v, anchor_idx, cnt, L, b, i, Hkv * D / 8, kc, vc, lane);
  if (i < cnt) {
    const int pc = Hkv * D / 4;
    const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int c = lane; c < pc; c += 32) {
      dka[row * pc + c] = z;
      dva[row * pc + c] = z;
    }
  }
}

// ------------------------------------------------------------------ shared parameter block
struct BwdParams {
  CUtensorMap tmQ, tmK, tmV, tmKc, tmVc, tmdO, tmdQ, tmdK, tmdV;
  CUtensorMap tmK64, tmV64, tmKc64, tmVc64;  // 64-row boxes: the halves of a merged tile (dQ)
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
// Query-major, persistent over a flattened key-tile stream (same item order and key tiles as
// the forward). Per key tile: S = Q K^T and dP = dO V^T into TMEM; the softmax warpgroups
// (two per row: key columns 64wg..64wg+63) form dS = P (dP - Delta) with P = exp2(S c - lse2)
// and store it to TMEM as bf16; dQ += dS K (A from TMEM, B = K MN-major). The scaled dQ tile
// leaves through shared memory and one TMA store.
template <int D>
struct DqCfg {
  static constexpr int KB = D / 64;
  static constexpr int TILE = KB * kBoxBytes;
  static constexpr int NST = 2;
  static constexpr int DOB = (D == 128) ? 1 : 2;               // dO buffers
  static constexpr int SMEM_TILES = TILE * (2 + DOB + 2 * NST);  // Q x2, dO, NST x (K, V)
  static constexpr int COL_S = 0, COL_DP = 128, COL_DQ = 256, COL_DS = 256 + D;
  static constexpr int THREADS = 352;  // 8 softmax warps, producer, MMA issuer, dQ storer
};

template <int NST, int DOB>
struct DqBar {
  uint64_t q_full[2], q_empty[2], q_staged[2], do_full[DOB], do_empty[DOB];
  uint64_t k_full[NST], k_empty[NST], v_full[NST], v_empty[NST];
  uint64_t s_full, s_free, ds_ready, dq_done;
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

template <int D>
constexpr size_t dq_smem_bytes() {
  return 1024 + DqCfg<D>::SMEM_TILES + sizeof(DqBar<DqCfg<D>::NST, DqCfg<D>::DOB>);
}

// Items of the dQ pass, with the forward's half-window rule: when the lower 64 keys of the
// oldest window tile lo lie outside every row's band (128 t - n + 1 >= 128 lo + 64), their
// anchors join the gathered ones (ge counts both), the oldest window tile is merged (lower half:
// compacted anchors 0..63; upper half: keys 128 lo + 64 ..) and the anchor chunks start at
// compacted row arow0 = 64.
struct BwdItem {
  int t, h, b, nwin, ge, N, arow0;
  bool half;
};
__device__ __forceinline__ BwdItem bwd_item_base(const BwdParams& p, int x) {
  BwdItem it;
  const int per_t = p.Hq * p.B;
  it.t = p.T - 1 - x / per_t;
  const int rem = x % per_t;
  it.h = rem % p.Hq;
  it.b = rem / p.Hq;
  const int lo = window_lo_tile(it.t, p.n);
  it.nwin = it.t - lo + 1;
  it.half = lo < it.t && (long long)it.t * 128 - p.n + 1 >= (long long)lo * 128 + 64;
  it.arow0 = it.half ? 64 : 0;
  it.ge = 0;
  it.N = it.nwin;
  return it;
}
__device__ __forceinline__ int bwd_item_ge(const BwdParams& p, int x) {
  const BwdItem it = bwd_item_base(p, x);
  int ge = p.gather_end[(size_t)it.b * p.T + it.t];
  if (it.half) {
    const uint32_t* w = p.anchor_bits + (size_t)it.b * p.W + (size_t)(it.t - it.nwin + 1) * 4;
    ge += __popc(__ldg(w)) + __popc(__ldg(w + 1));
  }
  return ge;
}
__device__ __forceinline__ BwdItem bwd_item_with(const BwdParams& p, int x, int ge) {
  BwdItem it = bwd_item_base(p, x);
  it.ge = ge;
  it.N = it.nwin + (max(0, ge - it.arow0) + 127) / 128;
  return it;
}
struct BwdTileRaw {
  uint32_t fb[4];
  int cls;
};
__device__ __forceinline__ BwdTileRaw bwd_tile_raw(const BwdParams& p, int b, int t, int u) {
  BwdTileRaw r;
  r.cls = p.tile_map[((size_t)b * p.T + t) * p.T + u];
  const uint32_t* w = p.anchor_bits + (size_t)b * p.W + (size_t)u * 4;
#pragma unroll
  for (int q = 0; q < 4; ++q) r.fb[q] = (u * 4 + q < p.W) ? __ldg(w + q) : 0u;
  return r;
}

template <int D>
__global__ void __launch_bounds__(DqCfg<D>::THREADS, 1)
    sep_attn_bwd_dq_kernel(const __grid_constant__ BwdParams p, int nitems) {
  using C = DqCfg<D>;
  constexpr int NST = C::NST, DOB = C::DOB;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ = smem;                 // 2 buffers (item parity), reused to stage dQ
  uint8_t* sdO = sQ + 2 * C::TILE;    // DOB buffers (item % DOB)
  uint8_t* sK = sdO + DOB * C::TILE;
  uint8_t* sV = sK + NST * C::TILE;
  DqBar<NST, DOB>* bar = reinterpret_cast<DqBar<NST, DOB>*>(sV + NST * C::TILE);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort_flag = &bar->abort_flag;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar->q_full[s], 1);
      mbar_init(&bar->q_empty[s], 1);
      mbar_init(&bar->q_staged[s], 256);
    }
    for (int s = 0; s < DOB; ++s) {
      mbar_init(&bar->do_full[s], 1);
      mbar_init(&bar->do_empty[s], 1);
    }
    for (int s = 0; s < NST; ++s) {
      mbar_init(&bar->k_full[s], 1);
      mbar_init(&bar->k_empty[s], 1);
      mbar_init(&bar->v_full[s], 1);
      mbar_init(&bar->v_empty[s], 1);
    }
    mbar_init(&bar->s_full, 1);
    mbar_init(&bar->s_free, 256);
    mbar_init(&bar->ds_ready, 256);
    mbar_init(&bar->dq_done, 1);
    mbar_init(&bar->drain, 1);
    bar->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc(&bar->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar->tmem_base;
  grid_dep_wait();

  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int g = 0;
      int kq = 0, kd = 0;  // items whose Q / dO load was issued
      bool ok = true;
      int ge_cur = bwd_item_ge(p, blockIdx.x);
      for (int k = 0, x = blockIdx.x; ok && x < nitems; ++k, x += gridDim.x) {
        const BwdItem it = bwd_item_with(p, x, ge_cur);
        if (x + (int)gridDim.x < nitems) ge_cur = bwd_item_ge(p, x + gridDim.x);
        const int kvh = it.h / (p.Hq / p.Hkv);
        const int qb = k & 1;
        if (k >= 2 && !mbar_wait(&bar->q_empty[qb], ((k - 2) >> 1) & 1, p.err, abort_flag)) {
          ok = false;
          break;
        }
        kq = k + 1;
        mbar_arrive_expect_tx(&bar->q_full[qb], C::TILE);
        for (int kb = 0; kb < C::KB; ++kb)
          tma_load_4d(sQ + qb * C::TILE + kb * kBoxBytes, &p.tmQ, &bar->q_full[qb], kb * 64, it.h,
                      it.t * 128, it.b);
        const int db = k % DOB;
        for (int j = 0; j < it.N; ++j, ++g) {
          if (j == 1 || (j == 0 && it.N == 1)) {
            // dO of this item: after the first K/V tile is on its way (its buffer frees when the
            // dP products of item k - DOB are done)
            if (k >= DOB &&
                !mbar_wait(&bar->do_empty[db], ((k - DOB) / DOB) & 1, p.err, abort_flag)) {
              ok = false;
              break;
            }
            kd = k + 1;
            mbar_arrive_expect_tx(&bar->do_full[db], C::TILE);
            for (int kb = 0; kb < C::KB; ++kb)
              tma_load_4d(sdO + db * C::TILE + kb * kBoxBytes, &p.tmdO, &bar->do_full[db],
                          kb * 64, it.h, it.t * 128, it.b);
          }
          const int st = g % NST, r = g / NST;
          const bool win = j < it.nwin;
          const bool merged = it.half && j == it.nwin - 1;
          const int row0 = win ? (it.t - j) * 128 : it.arow0 + (j - it.nwin) * 128;
          if (r > 0 && !mbar_wait(&bar->k_empty[st], (r - 1) & 1, p.err, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bar->k_full[st], C::TILE);
          for (int kb = 0; kb < C::KB; ++kb) {
            uint8_t* dst = sK + st * C::TILE + kb * kBoxBytes;
            if (merged) {  // compacted anchors 0..63, then keys 128 lo + 64 ..
              tma_load_4d(dst, &p.tmKc64, &bar->k_full[st], kb * 64, kvh, 0, it.b);
              tma_load_4d(dst + 64 * 128, &p.tmK64, &bar->k_full[st], kb * 64, kvh, row0 + 64, it.b);
            } else {
              tma_load_4d(dst, win ? &p.tmK : &p.tmKc, &bar->k_full[st], kb * 64, kvh, row0, it.b);
            }
          }
          if (r > 0 && !mbar_wait(&bar->v_empty[st], (r - 1) & 1, p.err, abort_flag)) {
            mbar_wait(&bar->k_full[st], r & 1, nullptr, nullptr);
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bar->v_full[st], C::TILE);
          for (int kb = 0; kb < C::KB; ++kb) {
            uint8_t* dst = sV + st * C::TILE + kb * kBoxBytes;
            if (merged) {
              tma_load_4d(dst, &p.tmVc64, &bar->v_full[st], kb * 64, kvh, 0, it.b);
              tma_load_4d(dst + 64 * 128, &p.tmV64, &bar->v_full[st], kb * 64, kvh, row0 + 64, it.b);
            } else {
              tma_load_4d(dst, win ? &p.tmV : &p.tmVc, &bar->v_full[st], kb * 64, kvh, row0, it.b);
            }
          }
        }
      }
      if (!ok) {
        // drain: the loads of the last NST key tiles, Q and dO tiles that may be in flight
        // (older phases completed already, so their waits return at once)
        for (int gg = max(0, g - NST); gg < g; ++gg) {
          mbar_wait(&bar->k_full[gg % NST], (gg / NST) & 1, nullptr, nullptr);
          mbar_wait(&bar->v_full[gg % NST], (gg / NST) & 1, nullptr, nullptr);
        }
        for (int kk = max(0, kq - 2); kk < kq; ++kk)
          mbar_wait(&bar->q_full[kk & 1], (kk >> 1) & 1, nullptr, nullptr);
        for (int kk = max(0, kd - DOB); kk < kd; ++kk)
          mbar_wait(&bar->do_full[kk % DOB], (kk / DOB) & 1, nullptr, nullptr);
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = make_idesc_bf16(128, 128, false, false);
      constexpr uint32_t idQ = make_idesc_bf16(128, D, false, true);
      const uint32_t sQa = smem_u32(sQ), sdOa = smem_u32(sdO);
      const uint32_t sKa = smem_u32(sK), sVa = smem_u32(sV);
      bool ok = true;
      int g = 0, pend = -1, pend_first = 0;
      auto issue_dQ = [&](int gg, int first) -> bool {
        const int st = gg % NST;
        if (!mbar_wait(&bar->ds_ready, gg & 1, p.err, abort_flag)) return false;
        tc_fence_after();
        const uint32_t klo = sdesc_lo(sKa + st * C::TILE, kBoxBytes);
#pragma unroll
        for (int kk = 0; kk < 128 / 16; ++kk)
          mma_ts(tmem + C::COL_DQ, tmem + C::COL_DS + kk * 8,
                 sdesc_join(klo + kk * (2048 >> 4), kDescHi), idQ, (!first || kk > 0) ? 1u : 0u);
        tc_commit(&bar->dq_done);
        tc_commit(&bar->k_empty[st]);
        return true;
      };
      int ge_cur = bwd_item_ge(p, blockIdx.x);
      for (int k = 0, x = blockIdx.x; ok && x < nitems; ++k, x += gridDim.x) {
        const BwdItem it = bwd_item_with(p, x, ge_cur);
        if (x + (int)gridDim.x < nitems) ge_cur = bwd_item_ge(p, x + gridDim.x);
        const int qb = k & 1, db = k % DOB;
        if (!mbar_wait(&bar->q_full[qb], (k >> 1) & 1, p.err, abort_flag)) { ok = false; break; }
        const uint32_t sQb = sQa + qb * C::TILE, sdOb = sdOa + db * C::TILE;
        for (int j = 0; j < it.N; ++j, ++g) {
          const int st = g % NST;
          // at an item boundary the previous item's last dQ product goes first: the next item's
          // S waits for its Q / dO tiles, and that item's epilogue waits for this product
          if (j == 0 && pend >= 0) {
            if (!issue_dQ(pend, pend_first)) { ok = false; break; }
            pend = -1;
          }
          if (!mbar_wait(&bar->k_full[st], (g / NST) & 1, p.err, abort_flag)) { ok = false; break; }
          if (!mbar_wait(&bar->v_full[st], (g / NST) & 1, p.err, abort_flag)) { ok = false; break; }
          if (g > 0 && !mbar_wait(&bar->s_free, (g - 1) & 1, p.err, abort_flag)) { ok = false; break; }
          if (j == 0 && !mbar_wait(&bar->do_full[db], (k / DOB) & 1, p.err, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t qlo = sdesc_lo(sQb, 16), klo = sdesc_lo(sKa + st * C::TILE, 16);
          const uint32_t dlo = sdesc_lo(sdOb, 16), vlo = sdesc_lo(sVa + st * C::TILE, 16);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = ((kk >> 2) * kBoxBytes + (kk & 3) * 32) >> 4;
            mma_ss(tmem + C::COL_S, sdesc_join(qlo + off, kDescHi), sdesc_join(klo + off, kDescHi),
                   idS, kk > 0 ? 1u : 0u);
          }
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = ((kk >> 2) * kBoxBytes + (kk & 3) * 32) >> 4;
            mma_ss(tmem + C::COL_DP, sdesc_join(dlo + off, kDescHi),
                   sdesc_join(vlo + off, kDescHi), idS, kk > 0 ? 1u : 0u);
          }
          tc_commit(&bar->s_full);
          tc_commit(&bar->v_empty[st]);
          if (j == it.N - 1) tc_commit(&bar->do_empty[db]);
          if (pend >= 0 && !issue_dQ(pend, pend_first)) { ok = false; break; }
          pend = g;
          pend_first = (j == 0);
        }
      }
      if (ok && pend >= 0) issue_dQ(pend, pend_first);
      tc_commit(&bar->drain);
      mbar_wait(&bar->drain, 0, nullptr, nullptr);
    }
  } else if (warp == 10) {
    // ------------------------------------------------------------ dQ tile storer
    if (lane == 0) {
      bool ok = true;
      for (int k = 0, x = blockIdx.x; ok && x < nitems; ++k, x += gridDim.x) {
        const BwdItem it = bwd_item_base(p, x);
        if (!mbar_wait(&bar->q_staged[k & 1], (k >> 1) & 1, p.err, abort_flag)) {
          ok = false;
          break;
        }
        const uint8_t* stage = sQ + (k & 1) * C::TILE;
        for (int kb = 0; kb < C::KB; ++kb)
          tma_store_4d(&p.tmdQ, stage + kb * kBoxBytes, kb * 64, it.h, it.t * 128, it.b);
        bulk_commit_group();
        bulk_wait_read_all();
        mbar_arrive(&bar->q_empty[k & 1]);
      }
      bulk_wait_all();
    }
  } else {
    // ------------------------------------------------------------ softmax warpgroups
    const int row = threadIdx.x & 127;
    const int wg = threadIdx.x >> 7;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const float sl2 = p.scale_log2;
    bool ok = true;
    int g = 0, k_item = 0;
    int ge_cur = bwd_item_ge(p, blockIdx.x);
    BwdTileRaw cur;
    {
      const BwdItem f0 = bwd_item_base(p, blockIdx.x);
      cur = bwd_tile_raw(p, f0.b, f0.t, f0.t);
    }
    for (int x = blockIdx.x; ok && x < nitems; x += gridDim.x) {
      const BwdItem it = bwd_item_with(p, x, ge_cur);
      const int xn = x + gridDim.x;
      if (xn < nitems) ge_cur = bwd_item_ge(p, xn);
      const long long i = (long long)it.t * 128 + row;
      const bool valid = i < p.L;
      const size_t rowstat = ((size_t)it.b * p.Hq + it.h) * p.L + (valid ? i : 0);
      const float lse2 = valid ? p.lse[rowstat] * 1.4426950408889634f : INFINITY;
      const float dlt = valid ? p.delta[rowstat] : 0.f;
      for (int j = 0; j < it.N; ++j, ++g) {
        const BwdTileRaw raw = cur;
        if (j + 1 < it.nwin) {
          cur = bwd_tile_raw(p, it.b, it.t, it.t - (j + 1));
        } else if (j + 1 == it.N && xn < nitems) {
          const BwdItem fn = bwd_item_base(p, xn);
          cur = bwd_tile_raw(p, fn.b, fn.t, fn.t);
        }
        uint32_t keep[2] = {0xffffffffu, 0xffffffffu};
        if (it.half && j == it.nwin - 1 && wg == 0) {
          // lower half of the merged tile: gathered anchors 0..63, kept by every row
          const int cnt = min(it.ge, 64);
#pragma unroll
          for (int w = 0; w < 2; ++w) keep[w] = range_word(0, cnt - 1, w);
        } else if (j < it.nwin) {
          const int u = it.t - j;
          const long long k0 = (long long)u * 128;
          if (raw.cls != SEP_TILE_FULL) {
#pragma unroll
            for (int w = 0; w < 2; ++w)
              keep[w] = window_keep_word(2 * wg + w, i, k0, p.n, p.L, raw.fb[2 * wg + w]);
          } else if (k0 + 128 > p.L) {
#pragma unroll
            for (int w = 0; w < 2; ++w) keep[w] = range_word(0, (long long)p.L - 1 - k0, 2 * wg + w);
          }
        } else {
          const int rem = it.ge - it.arow0 - (j - it.nwin) * 128;
          if (rem < 128) {
#pragma unroll
            for (int w = 0; w < 2; ++w) keep[w] = range_word(0, rem - 1, 2 * wg + w);
          }
        }
        if (!__all_sync(0xffffffffu, mbar_wait(&bar->s_full, g & 1, p.err, abort_flag))) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t sv[64], dp[64];
        {
          const uint32_t aS = tmem + lane_off + C::COL_S + wg * 64;
          const uint32_t aP = tmem + lane_off + C::COL_DP + wg * 64;
          tmem_ld32(aS, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
          tmem_ld32(aS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
          tmem_ld32(aP, *reinterpret_cast<uint32_t(*)[32]>(&dp[0]));
          tmem_ld32(aP + 32, *reinterpret_cast<uint32_t(*)[32]>(&dp[32]));
          tmem_ld_wait();
        }
        tc_fence_before();
        mbar_arrive(&bar->s_free);  // S and dP may be overwritten by the next tile's MMAs
        // two columns per packed fp32x2 instruction: x = S * scale*log2(e) - lse2, P = exp2(x)
        // on kept pairs, dS = P (dP - Delta)
        const float2 sl2x2 = make_float2(sl2, sl2), nl2 = make_float2(-lse2, -lse2);
        const float2 ndl2 = make_float2(-dlt, -dlt);
#pragma unroll
        for (int c = 0; c < 64; c += 2) {
          const float2 x = f2_fma(make_float2(__uint_as_float(sv[c]), __uint_as_float(sv[c + 1])),
                                  sl2x2, nl2);
          const float2 dd = f2_add(make_float2(__uint_as_float(dp[c]), __uint_as_float(dp[c + 1])),
                                   ndl2);
          const float p0 = ((keep[c >> 5] >> (c & 31)) & 1u) ? ex2(x.x) : 0.f;
          const float p1 = ((keep[(c + 1) >> 5] >> ((c + 1) & 31)) & 1u) ? ex2(x.y) : 0.f;
          const float2 v = f2_mul(make_float2(p0, p1), dd);
          sv[c >> 1] = pack_bf16x2(v.x, v.y);
        }
        // dS has one buffer: the previous tile's dQ MMA must have read it
        if (g > 0 &&
            !__all_sync(0xffffffffu, mbar_wait(&bar->dq_done, (g - 1) & 1, p.err, abort_flag))) {
          ok = false;
          break;
        }
        tc_fence_after();
        tmem_st32(tmem + lane_off + C::COL_DS + wg * 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&bar->ds_ready);
      }
      if (!ok) break;
      // ---- epilogue: scale * dQ as bf16 through the item's (free) Q buffer, one TMA store
      if (!__all_sync(0xffffffffu, mbar_wait(&bar->dq_done, (g - 1) & 1, p.err, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint8_t* stage = sQ + (k_item & 1) * C::TILE;
#pragma unroll 1
      for (int cc = 0; cc < D / 64; ++cc) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_off + C::COL_DQ + wg * (D / 2) + cc * 32, v);
        tmem_ld_wait();
        uint32_t pkd[16];
#pragma unroll
        for (int q = 0; q < 16; ++q)
          pkd[q] = pack_bf16x2(__uint_as_float(v[2 * q]) * p.scale,
                               __uint_as_float(v[2 * q + 1]) * p.scale);
        const int col0 = wg * (D / 2) + cc * 32;
        uint8_t* box = stage + (col0 >> 6) * kBoxBytes;
#pragma unroll
        for (int q = 0; q < 4; ++q)
          *reinterpret_cast<uint4*>(box + sw128_offset(row, ((col0 & 63) >> 3) + q)) =
              make_uint4(pkd[4 * q], pkd[4 * q + 1], pkd[4 * q + 2], pkd[4 * q + 3]);
      }
      fence_proxy_async_smem();
      mbar_arrive(&bar->q_staged[k_item & 1]);  // the storer warp writes the tile out
      ++k_item;
    }
    tc_fence_before();
  }
  grid_dep_launch_next();  // the next kernel of the stream may start its prologue
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ dK/dV work list
// Items of the key-major pass, one per (key unit, segment of query tiles):
//   window item: key tile u of batch b with every query tile t whose window key tiles lo(t)..t
//                contain u (t_begin = u .. t_end - 1), so that its non-anchor keys get their
//                complete gradient in one item; at position u * B + b, so that the list runs
//                from the largest key range (u = 0 under dense causal) to the smallest;
//   anchor item: compacted anchor chunk c (anchors 128c..128c+127) with the query tiles that
//                gather it (gather_end[t] > 128c), in segments of kSegT tiles (their fp32 partial
//                sums are added atomically).
// Every kv head processes every item. Built on the device by bwd_schedule_kernel.
constexpr int kSegT = 16;

struct WorkItem {
  int b, unit, t_begin, t_end;  // unit: key tile u (window) or anchor chunk c
};

// One CTA per batch element: per-key-tile anchor prefix counts, then the anchor and window items.
__global__ void __launch_bounds__(1024) bwd_schedule_kernel(
    const int32_t* __restrict__ anchor_cnt, const int32_t* __restrict__ gather_end,
    const uint32_t* __restrict__ anchor_bits, int L, int n, int T, int W, int32_t* __restrict__ tile_prefix,
    WorkItem* __restrict__ anchor_items, WorkItem* __restrict__ window_items,
    int32_t* __restrict__ counters /* [0] anchor items, [1] window items; [2], [3] dK/dV pass */) {
  grid_dep_wait();
  grid_dep_launch_next();
  const int b = blockIdx.x;
  const int tid = threadIdx.x;
  __shared__ int s_warp[32];
  __shared__ int s_carry;
  if (tid == 0) s_carry = 0;
  __syncthreads();
  // ---- exclusive prefix over key tiles of the anchor counts
  for (int base = 0; base < T; base += blockDim.x) {
    const int u = base + tid;
    int c = 0;
    if (u < T) {
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (u * 4 + q < W) c += __popc(anchor_bits[(size_t)b * W + u * 4 + q]);
    }
    int incl = c;
    const int lane = tid & 31, warp = tid >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      const int wv = (lane < (int)(blockDim.x >> 5)) ? s_warp[lane] : 0;
      int wi = wv;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, wi, o);
        if (lane >= o) wi += y;
      }
      if (lane < (int)(blockDim.x >> 5)) s_warp[lane] = wi - wv;
    }
    __syncthreads();
    const int carry = s_carry;
    if (u < T) tile_prefix[(size_t)b * T + u] = carry + s_warp[warp] + incl - c;
    __syncthreads();
    if (tid == blockDim.x - 1) s_carry = carry + s_warp[warp] + incl;
    __syncthreads();
  }
  // ---- anchor items
  const int cnt = anchor_cnt[b];
  const int nch = (cnt + 127) / 128;
  const int32_t* ge = gather_end + (size_t)b * T;
  for (int c = tid; c < nch; c += blockDim.x) {
    int lo = 0, hi = T;  // first query tile that gathers anchor 128c
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (ge[mid] > c * 128) hi = mid; else lo = mid + 1;
    }
    const int nseg = (T - lo + kSegT - 1) / kSegT;
    if (nseg > 0) {
      const int at = atomicAdd(&counters[0], nseg);
      for (int sg = 0; sg < nseg; ++sg) {
        const int t0 = lo + sg * kSegT;
        anchor_items[at + sg] = WorkItem{b, c, t0, min(T, t0 + kSegT)};
      }
    }
  }
  // ---- window items: query tiles t with lo(t) <= u <= t; lo is non-decreasing in t, so the
  // last such t is found by binary search
  for (int u = tid; u < T; u += blockDim.x) {
    int lo = u + 1, hi = T;  // first t > u with lo(t) > u
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (window_lo_tile(mid, n) > u) hi = mid; else lo = mid + 1;
    }
    window_items[(size_t)u * gridDim.x + b] = WorkItem{b, u, u, lo};
  }
  if (tid == 0) atomicAdd(&counters[1], T);
}

// ------------------------------------------------------------------ dK/dV kernel
// Key-major, persistent over the work list (anchor items first, then window items; every kv
// head of an item in turn). Per (query tile, query head) pair the query tile is split in two
// 64-row halves h = 0, 1, each owned by one softmax warpgroup (thread = key row = TMEM lane):
//   S^T_h = K Q_h^T, dP^T_h = V dO_h^T            (M = 128 keys, N = 64 queries)
//   P^T = exp2(S^T c - lse2), dS^T = P^T (dP^T - Delta), written over S^T_h / dP^T_h as bf16
//   dV += P^T_h dO_h, dK += dS^T_h Q_h             (A from TMEM, B MN-major in smem)
// The MMA warp issues one half's S^T/dP^T while the other half's softmax runs. dV and dK stay
// in TMEM for the whole item. Epilogue: every window item covers all query tiles of its key
// tile, so its non-anchor rows are final and leave as bf16 through shared memory and a TMA
// store; anchor rows add their fp32 window part into the compact anchor partials, and anchor
// items add into the compact partials too.
template <int D>
struct DkvCfg {
  static constexpr int KB = D / 64;
  static constexpr int TILE = KB * kBoxBytes;
  static constexpr int KVB = (D == 128) ? 1 : 2;  // K/V buffers (items in flight)
  static constexpr int NST = (D == 128) ? 2 : 3;  // Q/dO stages (pairs in flight)
  static constexpr int SMEM_TILES = TILE * (2 * KVB + 2 * NST);
  // d = 64 ("wide"): S^T and dP^T of a whole pair (128 keys x 128 queries, N = 128 products),
  // P^T and dS^T as bf16 in columns of their own, so that the next pair's S^T / dP^T may be
  // issued as soon as the softmax warps have read these; both softmax warpgroups work on the
  // same pair (query columns 64 wg ..). TMEM: S^T 0, dP^T 128, P^T 256, dS^T 320, dV 384, dK 448.
  // d = 128: the accumulators take 256 columns, so S^T / dP^T are formed per 64-query half in
  // two buffers (half-pair k = 2 P + h uses buffer k % 2: S^T at 128 b, dP^T at 128 b + 64, then
  // P^T / dS^T written over them).
  static constexpr bool WIDE = (D == 64);
  static constexpr int NB = 2;
  static constexpr int COL_S = 0, COL_DPW = 128, COL_P = 256, COL_DS = 320;
  static constexpr int COL_DV = WIDE ? 384 : 256, COL_DK = COL_DV + D;
  static_assert(COL_DK + D <= 512, "TMEM columns");
  static constexpr int THREADS = 352;  // 8 softmax warps, producer, MMA issuer, storer
};

// One entry of the item ring: the work item and the mask inputs every role needs, loaded once
// from global memory by the producer and read by the other roles from shared memory.
struct ItemSlot {
  int x;                   // item index (>= nitems: no more items)
  int b, unit, t_begin, t_end, window;
  int pre_tile;            // anchors left of key tile `unit` (window items)
  int cnt_b;               // anchors of batch b
  uint32_t tile_words[4];  // anchor flags of key tile `unit` (window items)
};

template <int NST, int KVB, int NB>
struct DkvBar {
  uint64_t kv_full[KVB], kv_empty[KVB];
  uint64_t q_full[NST], q_empty[NST];
  // per S^T / dP^T buffer (wide: index 0 only): S^T / dP^T ready, P^T / dS^T written, products
  // done; wide: S^T / dP^T read by both warpgroups (s_free)
  uint64_t s_full[NB], pds_ready[NB], mm_done[NB], s_free;
  uint64_t acc_full, acc_free;
  uint64_t acc_dv;        // wide: the item's dV products are done (its dK products may still run)
  uint64_t staged[KVB];   // the item's dK/dV rows are in the K/V buffer (softmax -> storer)
  uint64_t drain;
  uint64_t item_full[4];  // ring of fetched work items (producer -> MMA, softmax, storer)
  ItemSlot item[4];
  alignas(16) float nlse2[NST][128];  // -log2-domain LSE of each query of the stage (-inf past L)
  alignas(16) float delta[NST][128];
  int pin[NST];           // mask input of the stage's pair: tile class (window) or gather_end
  uint32_t tmem_base;
  int abort_flag;
};

// the softmax reads the per-query statistics four at a time (16-byte shared-memory loads)
using DkvBar128 = DkvBar<DkvCfg<128>::NST, DkvCfg<128>::KVB, DkvCfg<128>::NB>;
using DkvBar64 = DkvBar<DkvCfg<64>::NST, DkvCfg<64>::KVB, DkvCfg<64>::NB>;
static_assert(offsetof(DkvBar128, nlse2) % 16 == 0 && offsetof(DkvBar128, delta) % 16 == 0,
              "16-byte aligned statistics");
static_assert(offsetof(DkvBar64, nlse2) % 16 == 0 && offsetof(DkvBar64, delta) % 16 == 0,
              "16-byte aligned statistics");
template <int D>
constexpr size_t dkv_smem_bytes() {
  return 1024 + DkvCfg<D>::SMEM_TILES +
         sizeof(DkvBar<DkvCfg<D>::NST, DkvCfg<D>::KVB, DkvCfg<D>::NB>);
}

struct DkvItem {
  int b, unit, t_begin, t_end;
  bool window;
  int kvh, npairs;
};

__device__ __forceinline__ DkvItem dkv_item(const BwdParams& p, const WorkItem* aitems,
                                           const WorkItem* witems, int n_anchor, int x, int G) {
  DkvItem it;
  it.kvh = x % p.Hkv;
  const int e = x / p.Hkv;
  const WorkItem w = (e < n_anchor) ? aitems[e] : witems[e - n_anchor];
  it.window = e >= n_anchor;
  it.b = w.b;
  it.unit = w.unit;
  it.t_begin = w.t_begin;
  it.t_end = w.t_end;
  it.npairs = (w.t_end - w.t_begin) * G;
  return it;
}
__device__ __forceinline__ DkvItem slot_item(const ItemSlot& sl, int Hkv, int G) {
  DkvItem it;
  it.kvh = sl.x % Hkv;
  it.window = sl.window != 0;
  it.b = sl.b;
  it.unit = sl.unit;
  it.t_begin = sl.t_begin;
  it.t_end = sl.t_end;
  it.npairs = (sl.t_end - sl.t_begin) * G;
  return it;
}

template <int D>
__global__ void __launch_bounds__(DkvCfg<D>::THREADS, 1)
    sep_attn_bwd_dkv_kernel(const __grid_constant__ BwdParams p, const WorkItem* __restrict__ aitems,
                            const WorkItem* __restrict__ witems, int32_t* __restrict__ counters,
                            const int32_t* __restrict__ tile_prefix) {
  using C = DkvCfg<D>;
  constexpr int NST = C::NST, KVB = C::KVB, NB = C::NB;
  const int G = p.Hq / p.Hkv;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sK = smem;                       // KVB buffers
  uint8_t* sV = sK + KVB * C::TILE;         // KVB buffers
  uint8_t* sQ = sV + KVB * C::TILE;         // NST stages
  uint8_t* sdO = sQ + NST * C::TILE;        // NST stages
  DkvBar<NST, KVB, NB>* bar = reinterpret_cast<DkvBar<NST, KVB, NB>*>(sdO + NST * C::TILE);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort_flag = &bar->abort_flag;

  if (threadIdx.x == 0) {
    for (int s = 0; s < KVB; ++s) {
      mbar_init(&bar->kv_full[s], 1);
      mbar_init(&bar->kv_empty[s], 1);
    }
    for (int s = 0; s < NST; ++s) {
      mbar_init(&bar->q_full[s], 1 + 32);
      mbar_init(&bar->q_empty[s], 1);
    }
    for (int bb = 0; bb < NB; ++bb) {
      mbar_init(&bar->s_full[bb], 1);
      mbar_init(&bar->pds_ready[bb], C::WIDE ? 256 : 128);
      mbar_init(&bar->mm_done[bb], 1);
    }
    mbar_init(&bar->s_free, 256);
    mbar_init(&bar->acc_full, 1);
    mbar_init(&bar->acc_dv, 1);
    mbar_init(&bar->acc_free, 256);
    for (int s = 0; s < KVB; ++s) mbar_init(&bar->staged[s], 256);
    mbar_init(&bar->drain, 1);
    for (int s = 0; s < 4; ++s) mbar_init(&bar->item_full[s], 1);
    bar->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc(&bar->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar->tmem_base;
  grid_dep_wait();
  const int n_anchor = counters[0];
  const int nitems = (n_anchor + counters[1]) * p.Hkv;

  if (warp == 8) {
    // ---------------------------------------------------------------- producer (whole warp)
    int P = 0;
    int nkv = 0;  // items whose K/V load was issued
    bool ok = true;
    // Items are taken one at a time from the global counter (counters[2]) once the K/V buffer
    // they will use is free, and published to the other roles through the item ring; the
    // first index >= nitems ends every role.
    for (int I = 0; ok; ++I) {
      const int kb = I % KVB;
      bool okw = true;
      if (I >= KVB) okw = mbar_wait(&bar->kv_empty[kb], ((I - KVB) / KVB) & 1, p.err, abort_flag);
      if (!__all_sync(0xffffffffu, okw)) { ok = false; break; }
      int x = 0;
      if (lane == 0) {
        // fetch the item, start its K/V loads, then load its mask inputs and publish it all
        x = min(atomicAdd(&counters[2], 1), nitems);
        ItemSlot& sl = bar->item[I & 3];
        sl.x = x;
        if (x < nitems) {
          const DkvItem w = dkv_item(p, aitems, witems, n_anchor, x, G);
          mbar_arrive_expect_tx(&bar->kv_full[kb], 2 * C::TILE);
          const int krow = w.unit * 128;
          for (int q = 0; q < C::KB; ++q) {
            tma_load_4d(sK + kb * C::TILE + q * kBoxBytes, w.window ? &p.tmK : &p.tmKc,
                        &bar->kv_full[kb], q * 64, w.kvh, krow, w.b);
            tma_load_4d(sV + kb * C::TILE + q * kBoxBytes, w.window ? &p.tmV : &p.tmVc,
                        &bar->kv_full[kb], q * 64, w.kvh, krow, w.b);
          }
          nkv = I + 1;
          sl.b = w.b;
          sl.unit = w.unit;
          sl.t_begin = w.t_begin;
          sl.t_end = w.t_end;
          sl.window = w.window ? 1 : 0;
#pragma unroll
          for (int q = 0; q < 4; ++q)
            sl.tile_words[q] = (w.window && w.unit * 4 + q < p.W)
                                   ? __ldg(p.anchor_bits + (size_t)w.b * p.W + w.unit * 4 + q)
                                   : 0u;
          sl.pre_tile = w.window ? __ldg(tile_prefix + (size_t)w.b * p.T + w.unit) : 0;
          sl.cnt_b = __ldg(p.anchor_cnt + w.b);
        }
        mbar_arrive(&bar->item_full[I & 3]);
      }
      x = __shfl_sync(0xffffffffu, x, 0);
      if (x >= nitems) break;
      __syncwarp();
      const DkvItem it = slot_item(bar->item[I & 3], p.Hkv, G);
      for (int q = 0; q < it.npairs; ++q, ++P) {
        const int st = P % NST, r = P / NST;
        const int t = it.t_begin + q / G, h = it.kvh * G + q % G;
        okw = true;
        if (r > 0) okw = mbar_wait(&bar->q_empty[st], (r - 1) & 1, p.err, abort_flag);
        if (!__all_sync(0xffffffffu, okw)) { ok = false; break; }
        if (lane == 0) {
          mbar_arrive_expect_tx(&bar->q_full[st], 2 * C::TILE);
          for (int z = 0; z < C::KB; ++z) {
            tma_load_4d(sQ + st * C::TILE + z * kBoxBytes, &p.tmQ, &bar->q_full[st], z * 64, h,
                        t * 128, it.b);
            tma_load_4d(sdO + st * C::TILE + z * kBoxBytes, &p.tmdO, &bar->q_full[st], z * 64, h,
                        t * 128, it.b);
          }
          // the pair's mask input: class of block (t, unit), or the anchors tile t gathers
          bar->pin[st] = it.window ? (int)__ldg(p.tile_map + ((size_t)it.b * p.T + t) * p.T + it.unit)
                                   : __ldg(p.gather_end + (size_t)it.b * p.T + t);
        }
        // per-query statistics: log2-domain lse (+inf past L: P = 0 there) and Delta
        const size_t base = ((size_t)it.b * p.Hq + h) * p.L;
#pragma unroll
        for (int z = 0; z < 4; ++z) {
          const int col = lane * 4 + z;
          const long long i = (long long)t * 128 + col;
          const bool v = i < p.L;
          bar->nlse2[st][col] = v ? -__ldg(p.lse + base + i) * 1.4426950408889634f : -INFINITY;
          bar->delta[st][col] = v ? __ldg(p.delta + base + i) : 0.f;
        }
        mbar_arrive(&bar->q_full[st]);
      }
    }
    if (lane == 0 && !ok) {
      // drain: the Q/dO loads of the last NST pairs and the K/V loads of the last KVB items
      for (int pp = max(0, P - NST); pp < P; ++pp)
        mbar_wait(&bar->q_full[pp % NST], (pp / NST) & 1, nullptr, nullptr);
      for (int ii = max(0, nkv - KVB); ii < nkv; ++ii)
        mbar_wait(&bar->kv_full[ii % KVB], (ii / KVB) & 1, nullptr, nullptr);
    }
  } else if (warp == 9) {
    // ---------------------------------------------------------------- MMA issuer
    // Over the flattened sequence of half-pairs k = 2 P + h (pair P, query half h): S^T/dP^T of
    // the first NB half-pairs, then for every k its dV/dK products G(k) followed by S(k + NB),
    // which reuses the buffer of k once G(k) has read it. With one K/V buffer the next item is
    // published only after this item's epilogue, so every G of the item goes out before its
    // first S.
    if (lane == 0) {
      constexpr uint32_t idS = make_idesc_bf16(128, 64, false, false);
      constexpr uint32_t idG = make_idesc_bf16(128, D, false, true);
      const uint32_t sKa = smem_u32(sK), sVa = smem_u32(sV);
      const uint32_t sQa = smem_u32(sQ), sdOa = smem_u32(sdO);
      bool ok = true;
      // cursor over (item, pair): local item count I, its index x, pair q within it, the
      // CTA-wide pair count P, and the query half h
      struct Cur {
        int I, x, q, P, h;
        DkvItem it;
      };
      auto load_item = [&](Cur& c) -> bool {  // c.I set: wait for the producer to publish it
        if (!mbar_wait(&bar->item_full[c.I & 3], (c.I >> 2) & 1, p.err, abort_flag)) return false;
        c.x = bar->item[c.I & 3].x;
        c.q = 0;
        if (c.x < nitems) c.it = slot_item(bar->item[c.I & 3], p.Hkv, G);
        return true;
      };
      auto issue_S = [&](const Cur& c) -> bool {
        const int h = c.h, k = 2 * c.P + h, bb = k % NB;
        const int kb = c.I % KVB, st = c.P % NST;
        if (h == 0) {
          if (c.q == 0 && !mbar_wait(&bar->kv_full[kb], (c.I / KVB) & 1, p.err, abort_flag)) return false;
          if (!mbar_wait(&bar->q_full[st], (c.P / NST) & 1, p.err, abort_flag)) return false;
        }
        // the buffer holds the P^T / dS^T of half-pair k - NB until its products are done
        if (k >= NB && !mbar_wait(&bar->mm_done[bb], ((k / NB) - 1) & 1, p.err, abort_flag))
          return false;
        tc_fence_after();
        const uint32_t kA = sKa + kb * C::TILE, vA = sVa + kb * C::TILE;
        const uint32_t qA = sQa + st * C::TILE, dA = sdOa + st * C::TILE;
        const uint32_t cS = tmem + 128 * bb, cP = cS + 64;
        const uint32_t klo = sdesc_lo(kA, 16), vlo = sdesc_lo(vA, 16);
        const uint32_t qlo = sdesc_lo(qA + h * 64 * 128, 16), dlo = sdesc_lo(dA + h * 64 * 128, 16);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk >> 2) * kBoxBytes + (kk & 3) * 32) >> 4;
          mma_ss(cS, sdesc_join(klo + off, kDescHi), sdesc_join(qlo + off, kDescHi), idS,
                 kk > 0 ? 1u : 0u);
          mma_ss(cP, sdesc_join(vlo + off, kDescHi), sdesc_join(dlo + off, kDescHi), idS,
                 kk > 0 ? 1u : 0u);
        }
        tc_commit(&bar->s_full[bb]);
        return true;
      };
      auto issue_G = [&](const Cur& c) -> bool {
        const int h = c.h, k = 2 * c.P + h, bb = k % NB;
        const int st = c.P % NST;
        // the first dV/dK product of an item overwrites the accumulators: the previous item's
        // epilogue must have read them
        if (h == 0 && c.q == 0 && c.I > 0 &&
            !mbar_wait(&bar->acc_free, (c.I - 1) & 1, p.err, abort_flag))
          return false;
        if (!mbar_wait(&bar->pds_ready[bb], (k / NB) & 1, p.err, abort_flag)) return false;
        tc_fence_after();
        const uint32_t qA = sQa + st * C::TILE, dA = sdOa + st * C::TILE;
        const uint32_t cS = tmem + 128 * bb, cP = cS + 64;
        const uint32_t dlo = sdesc_lo(dA + h * 64 * 128, kBoxBytes);
        const uint32_t qlo = sdesc_lo(qA + h * 64 * 128, kBoxBytes);
#pragma unroll
        for (int kk = 0; kk < 64 / 16; ++kk) {
          const uint32_t roff = (kk * 16 * 128) >> 4;
          const uint32_t acc = (c.q > 0 || h > 0 || kk > 0) ? 1u : 0u;
          mma_ts(tmem + C::COL_DV, cS + kk * 8, sdesc_join(dlo + roff, kDescHi), idG, acc);
          mma_ts(tmem + C::COL_DK, cP + kk * 8, sdesc_join(qlo + roff, kDescHi), idG, acc);
        }
        tc_commit(&bar->mm_done[bb]);
        if (h == 1) {
          tc_commit(&bar->q_empty[st]);
          if (c.q == c.it.npairs - 1) tc_commit(&bar->acc_full);
        }
        return true;
      };
      if constexpr (C::WIDE) {
        // S^T / dP^T of the whole pair (N = 128), then, once the softmax warps have read them,
        // the next pair's; dV / dK products of a pair once its P^T / dS^T are in TMEM
        constexpr uint32_t idSW = make_idesc_bf16(128, 128, false, false);
        auto issue_SW = [&](const Cur& c) -> bool {
          const int kb = c.I % KVB, st = c.P % NST;
          if (c.q == 0 && !mbar_wait(&bar->kv_full[kb], (c.I / KVB) & 1, p.err, abort_flag)) return false;
          if (!mbar_wait(&bar->q_full[st], (c.P / NST) & 1, p.err, abort_flag)) return false;
          tc_fence_after();
          const uint32_t klo = sdesc_lo(sKa + kb * C::TILE, 16), vlo = sdesc_lo(sVa + kb * C::TILE, 16);
          const uint32_t qlo = sdesc_lo(sQa + st * C::TILE, 16), dlo = sdesc_lo(sdOa + st * C::TILE, 16);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = ((kk >> 2) * kBoxBytes + (kk & 3) * 32) >> 4;
            mma_ss(tmem + C::COL_S, sdesc_join(klo + off, kDescHi), sdesc_join(qlo + off, kDescHi),
                   idSW, kk > 0 ? 1u : 0u);
            mma_ss(tmem + C::COL_DPW, sdesc_join(vlo + off, kDescHi),
                   sdesc_join(dlo + off, kDescHi), idSW, kk > 0 ? 1u : 0u);
          }
          tc_commit(&bar->s_full[0]);
          return true;
        };
        auto issue_GW = [&](const Cur& c) -> bool {
          const int st = c.P % NST;
          if (c.q == 0 && c.I > 0 && !mbar_wait(&bar->acc_free, (c.I - 1) & 1, p.err, abort_flag))
            return false;
          if (!mbar_wait(&bar->pds_ready[0], c.P & 1, p.err, abort_flag)) return false;
          tc_fence_after();
          const uint32_t dlo = sdesc_lo(sdOa + st * C::TILE, kBoxBytes);
          const uint32_t qlo = sdesc_lo(sQa + st * C::TILE, kBoxBytes);
          if (c.q < c.it.npairs - 1) {
#pragma unroll
            for (int kk = 0; kk < 128 / 16; ++kk) {
              const uint32_t roff = (kk * 16 * 128) >> 4;
              const uint32_t acc = (c.q > 0 || kk > 0) ? 1u : 0u;
              mma_ts(tmem + C::COL_DV, tmem + C::COL_P + kk * 8, sdesc_join(dlo + roff, kDescHi),
                     idG, acc);
              mma_ts(tmem + C::COL_DK, tmem + C::COL_DS + kk * 8, sdesc_join(qlo + roff, kDescHi),
                     idG, acc);
            }
          } else {
            // the item's last pair: every dV product, then every dK product, so that the
            // epilogue's dV half starts while the dK products run
#pragma unroll
            for (int kk = 0; kk < 128 / 16; ++kk)
              mma_ts(tmem + C::COL_DV, tmem + C::COL_P + kk * 8,
                     sdesc_join(dlo + ((kk * 16 * 128) >> 4), kDescHi), idG,
                     (c.q > 0 || kk > 0) ? 1u : 0u);
            tc_commit(&bar->acc_dv);
#pragma unroll
            for (int kk = 0; kk < 128 / 16; ++kk)
              mma_ts(tmem + C::COL_DK, tmem + C::COL_DS + kk * 8,
                     sdesc_join(qlo + ((kk * 16 * 128) >> 4), kDescHi), idG,
                     (c.q > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit(&bar->mm_done[0]);
          tc_commit(&bar->q_empty[st]);
          if (c.q == c.it.npairs - 1) tc_commit(&bar->acc_full);
          return true;
        };
        Cur c;
        c.I = 0;
        c.P = 0;
        c.h = 0;
        ok = load_item(c);
        if (ok && c.x < nitems) ok = issue_SW(c);
        while (ok && c.x < nitems) {
          Cur n = c;
          ++n.P;
          bool more = true;
          if (++n.q >= n.it.npairs) {
            // the next item: published once the epilogue of item I + 1 - KVB has freed its K/V
            // buffer, which needs no product of this item
            ++n.I;
            ok = load_item(n);
            more = ok && n.x < nitems;
          }
          if (!ok) break;
          // at the last pair of an item its products go first, so that the epilogue (which
          // runs before the next item's first softmax) starts as early as possible
          const bool gfirst = n.q == 0;
          if (gfirst) {
            ok = issue_GW(c);
            if (!ok) break;
          }
          if (more) {
            if (!mbar_wait(&bar->s_free, c.P & 1, p.err, abort_flag)) { ok = false; break; }
            ok = issue_SW(n);
            if (!ok) break;
          }
          if (!gfirst) ok = issue_GW(c);
          c = n;
        }
      } else {
        // per 64-query half h: G(P, A), S(P+1, A), G(P, B), S(P+1, B), so that half A's next
        // softmax can run while half B's is still working; with one K/V buffer the next item
        // is published only after this item's epilogue, so both G of an item's last pair come
        // before the next item's S
        auto S_h = [&](Cur c, int h) { c.h = h; return issue_S(c); };
        auto G_h = [&](Cur c, int h) { c.h = h; return issue_G(c); };
        Cur c;
        c.I = 0;
        c.P = 0;
        c.h = 0;
        ok = load_item(c);
        if (ok && c.x < nitems) ok = S_h(c, 0) && S_h(c, 1);
        while (ok && c.x < nitems) {
          Cur n = c;
          ++n.P;
          if (c.q + 1 < c.it.npairs) {
            ++n.q;
            ok = G_h(c, 0) && S_h(n, 0) && G_h(c, 1) && S_h(n, 1);
          } else if (KVB == 1) {
            ++n.I;
            ok = G_h(c, 0) && G_h(c, 1) && load_item(n);
            if (ok && n.x < nitems) ok = S_h(n, 0) && S_h(n, 1);
          } else {
            ++n.I;
            ok = load_item(n);
            const bool more = ok && n.x < nitems;
            ok = ok && G_h(c, 0) && (!more || S_h(n, 0)) && G_h(c, 1) && (!more || S_h(n, 1));
          }
          c = n;
        }
      }
      tc_commit(&bar->drain);
      mbar_wait(&bar->drain, 0, nullptr, nullptr);
    }
  } else if (warp == 10) {
    // ---------------------------------------------------------------- dK/dV storer
    // Per item, once the softmax warps have staged it: the bf16 rows of a window
    // item leave by TMA store from the item's K/V buffer; then the buffer is released.
    if (lane == 0) {
      for (int I = 0;; ++I) {
        if (!mbar_wait(&bar->item_full[I & 3], (I >> 2) & 1, p.err, abort_flag)) break;
        const int x = bar->item[I & 3].x;
        if (x >= nitems) break;
        const DkvItem it = slot_item(bar->item[I & 3], p.Hkv, G);
        const int kb = I % KVB;
        if (!mbar_wait(&bar->staged[kb], (I / KVB) & 1, p.err, abort_flag)) break;
        if (it.window) {
          for (int z = 0; z < C::KB; ++z) {
            tma_store_4d(&p.tmdV, sV + kb * C::TILE + z * kBoxBytes, z * 64, it.kvh, it.unit * 128, it.b);
            tma_store_4d(&p.tmdK, sK + kb * C::TILE + z * kBoxBytes, z * 64, it.kvh, it.unit * 128, it.b);
          }
          bulk_commit_group();
          bulk_wait_read_all();  // the buffer may now take a later item's K / V
        }
        mbar_arrive(&bar->kv_empty[kb]);
      }
      bulk_wait_all();  // dK / dV stores complete before the CTA exits
    }
  } else if (warp < 8) {
    // ---------------------------------------------------------------- softmax warpgroups
    const int h = threadIdx.x >> 7;      // query half owned by this warpgroup
    const int krow = threadIdx.x & 127;  // key row = TMEM lane
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const float sl2 = p.scale_log2;
    bool ok = true;
    int P = 0;
    for (int I = 0; ok; ++I) {
      if (!__all_sync(0xffffffffu, mbar_wait(&bar->item_full[I & 3], (I >> 2) & 1, p.err, abort_flag))) {
        ok = false;
        break;
      }
      const ItemSlot& sl = bar->item[I & 3];
      const int x = sl.x;
      if (x >= nitems) break;
      const DkvItem it = slot_item(sl, p.Hkv, G);
      const int kb = I % KVB;
      long long j = -1;  // key position (window items)
      bool fj = false;
      int r = -1;        // compact anchor row (anchor items)
      uint32_t tile_words[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) tile_words[q] = sl.tile_words[q];
      if (it.window) {
        j = (long long)it.unit * 128 + krow;
        fj = j < p.L && ((tile_words[krow >> 5] >> (krow & 31)) & 1u);
      } else {
        r = it.unit * 128 + krow;
      }
      // used at the epilogue
      const int pre_tile = sl.pre_tile;
      const int cnt_b = sl.cnt_b;
      for (int q = 0; q < it.npairs; ++q, ++P) {
        const int st = P % NST;
        const int t = it.t_begin + q / G;
        // half-pair index and its S^T / dP^T buffer (wide: the pair, buffer 0)
        const int kk2 = C::WIDE ? P : 2 * P + h, bb = C::WIDE ? 0 : kk2 % NB;
        const int sbuf_use = C::WIDE ? P : kk2 / NB;
        if (!__all_sync(0xffffffffu,
                        mbar_wait(&bar->s_full[bb], sbuf_use & 1, p.err, abort_flag))) {
          ok = false;
          break;
        }
        // q_full also covers the per-query statistics and the mask input of the pair, written
        // by the producer warp
        if (!__all_sync(0xffffffffu, mbar_wait(&bar->q_full[st], (P / NST) & 1, p.err, abort_flag))) {
          ok = false;
          break;
        }
        const int cur = bar->pin[st];
        // keep bits over the 64 query columns of this half
        uint32_t keep[2];
        const long long q0 = (long long)t * 128 + 64 * h;
        if (it.window) {
          const int cls = cur;
          if (j >= p.L) {
            keep[0] = keep[1] = 0u;
          } else if (cls == SEP_TILE_FULL) {
            keep[0] = keep[1] = 0xffffffffu;
          } else {  // query i keeps j iff i >= j and (i - j < n or f[j])
            const long long lo = j - q0;
            const long long hi = fj ? 63 : j + p.n - 1 - q0;
            keep[0] = range_word(lo, hi, 0);
            keep[1] = range_word(lo, hi, 1);
          }
        } else {
          const uint32_t all = (r < cur) ? 0xffffffffu : 0u;
          keep[0] = keep[1] = all;
        }
        tc_fence_after();
        const float* nlse2 = &bar->nlse2[st][64 * h];
        const float* dl = &bar->delta[st][64 * h];
        // one 32-column chunk: x = S * scale*log2(e) - lse2 (two queries per packed fp32x2
        // instruction), P = exp2(x) on kept pairs, dS = P (dP - Delta), both packed to bf16
        auto pds_chunk = [&](auto all_kept, int ch, const uint32_t(&sv)[32],
                             const uint32_t(&dp)[32], uint32_t(&pk)[16], uint32_t(&dk16)[16]) {
          constexpr bool kAll = decltype(all_kept)::value;
          const float2 sl2x2 = make_float2(sl2, sl2);
          float4 nl4 = make_float4(0.f, 0.f, 0.f, 0.f), dl4 = nl4;
#pragma unroll
          for (int c = 0; c < 32; c += 2) {
            const int col = 32 * ch + c;
            if ((c & 3) == 0) {
              nl4 = *reinterpret_cast<const float4*>(nlse2 + col);
              dl4 = *reinterpret_cast<const float4*>(dl + col);
            }
            const float2 nlp = (c & 3) ? make_float2(nl4.z, nl4.w) : make_float2(nl4.x, nl4.y);
            const float2 dlp = (c & 3) ? make_float2(dl4.z, dl4.w) : make_float2(dl4.x, dl4.y);
            const float2 x = f2_fma(make_float2(__uint_as_float(sv[c]), __uint_as_float(sv[c + 1])),
                                    sl2x2, nlp);
            const float2 dd = f2_sub(make_float2(__uint_as_float(dp[c]), __uint_as_float(dp[c + 1])), dlp);
            const float p0 = (kAll || ((keep[ch] >> c) & 1u)) ? ex2(x.x) : 0.f;
            const float p1 = (kAll || ((keep[ch] >> (c + 1)) & 1u)) ? ex2(x.y) : 0.f;
            const float2 ds = f2_mul(make_float2(p0, p1), dd);
            pk[c >> 1] = pack_bf16x2(p0, p1);
            dk16[c >> 1] = pack_bf16x2(ds.x, ds.y);
          }
        };
        if constexpr (C::WIDE) {
          // this warpgroup's 64 query columns of the pair's S^T / dP^T; P^T / dS^T go to their
          // own columns once the previous pair's products have read them
          const uint32_t aS = tmem + lane_off + C::COL_S + 64 * h;
          const uint32_t aD = tmem + lane_off + C::COL_DPW + 64 * h;
          uint32_t pk[2][16], dk16[2][16];
          // every row of the warp keeps all 64 query columns (e.g. anchor items): no selects
          const bool all_kept = __all_sync(0xffffffffu, (keep[0] & keep[1]) == 0xffffffffu);
#pragma unroll
          for (int ch = 0; ch < 2; ++ch) {
            uint32_t sv[32], dp[32];
            tmem_ld32(aS + 32 * ch, sv);
            tmem_ld32(aD + 32 * ch, dp);
            tmem_ld_wait();
            if (ch == 1) {
              tc_fence_before();
              mbar_arrive(&bar->s_free);  // the next pair's S^T / dP^T may overwrite them
            }
            if (all_kept)
              pds_chunk(std::true_type{}, ch, sv, dp, pk[ch], dk16[ch]);
            else
              pds_chunk(std::false_type{}, ch, sv, dp, pk[ch], dk16[ch]);
          }
          if (P > 0 && !__all_sync(0xffffffffu,
                                   mbar_wait(&bar->mm_done[0], (P - 1) & 1, p.err, abort_flag))) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int ch = 0; ch < 2; ++ch) {
            tmem_st16(tmem + lane_off + C::COL_P + 32 * h + 16 * ch, pk[ch]);
            tmem_st16(tmem + lane_off + C::COL_DS + 32 * h + 16 * ch, dk16[ch]);
          }
        } else {
          // two 32-column chunks; packed chunk c lands in columns 16c..16c+15, already read
          const uint32_t aS = tmem + lane_off + 128 * bb, aP = aS + 64;
#pragma unroll
          for (int ch = 0; ch < 2; ++ch) {
            uint32_t sv[32], dp[32];
            tmem_ld32(aS + 32 * ch, sv);
            tmem_ld32(aP + 32 * ch, dp);
            tmem_ld_wait();
            uint32_t pk[16], dk16[16];
            pds_chunk(std::false_type{}, ch, sv, dp, pk, dk16);
            tmem_st16(aS + 16 * ch, pk);
            tmem_st16(aP + 16 * ch, dk16);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&bar->pds_ready[bb]);
      }
      if (!ok) break;
      // ---------------------------------------------------------------- item epilogue
      if constexpr (C::WIDE) {
        // warpgroup h finishes columns 32 h .. 32 h + 31 of dV (once the item's dV products are
        // done), then the same columns of dK (row krow of the key unit)
        long long dst_row = -1;
        const bool stage_row = it.window;
        if (it.window) {
          if (fj) {
            int before = pre_tile;
#pragma unroll
            for (int q = 0; q < 4; ++q)
              if (q < (krow >> 5)) before += __popc(tile_words[q]);
            before += __popc(tile_words[krow >> 5] & ((1u << (krow & 31)) - 1u));
            dst_row = before;
          }
        } else if (r < cnt_b) {
          dst_row = r;
        }
#pragma unroll
        for (int m = 0; m < 2; ++m) {  // 0: dV, 1: dK
          if (!__all_sync(0xffffffffu, mbar_wait(m ? &bar->acc_full : &bar->acc_dv, I & 1, p.err,
                                                 abort_flag))) {
            ok = false;
            break;
          }
          tc_fence_after();
          uint32_t acc[32];
          tmem_ld32(tmem + lane_off + (m ? C::COL_DK : C::COL_DV) + 32 * h, acc);
          tmem_ld_wait();
          const float mul = m ? p.scale : 1.f;
          if (dst_row >= 0) {
            float* dst = (m ? p.dka : p.dva) +
                         (((size_t)it.b * p.L + dst_row) * p.Hkv + it.kvh) * D + 32 * h;
#pragma unroll
            for (int z = 0; z < 8; ++z)
              atomicAdd(reinterpret_cast<float4*>(dst) + z,
                        make_float4(__uint_as_float(acc[4 * z]) * mul, __uint_as_float(acc[4 * z + 1]) * mul,
                                    __uint_as_float(acc[4 * z + 2]) * mul, __uint_as_float(acc[4 * z + 3]) * mul));
          }
          if (stage_row) {
            // bf16 into this item's K (dK) or V (dV) buffer, swizzled box layout
            uint8_t* stage = (m ? sK : sV) + kb * C::TILE;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint4 v4 = make_uint4(
                  pack_bf16x2(__uint_as_float(acc[8 * q]) * mul, __uint_as_float(acc[8 * q + 1]) * mul),
                  pack_bf16x2(__uint_as_float(acc[8 * q + 2]) * mul, __uint_as_float(acc[8 * q + 3]) * mul),
                  pack_bf16x2(__uint_as_float(acc[8 * q + 4]) * mul, __uint_as_float(acc[8 * q + 5]) * mul),
                  pack_bf16x2(__uint_as_float(acc[8 * q + 6]) * mul, __uint_as_float(acc[8 * q + 7]) * mul));
              *reinterpret_cast<uint4*>(stage + sw128_offset(krow, 4 * h + q)) = v4;
            }
          }
        }
        if (!ok) break;
        tc_fence_before();
        mbar_arrive(&bar->acc_free);  // the next item may overwrite dV / dK
        if (stage_row) fence_proxy_async_smem();
        mbar_arrive(&bar->staged[kb]);  // the storer writes the rows out and frees the buffer
        continue;
      }
      if (!__all_sync(0xffffffffu, mbar_wait(&bar->acc_full, I & 1, p.err, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
      // warpgroup 0 finishes dV, warpgroup 1 finishes dK (row krow of the key unit)
      const float mul = h ? p.scale : 1.f;
      const uint32_t col0 = h ? C::COL_DK : C::COL_DV;
      float* part = h ? p.dka : p.dva;
      // compact anchor row that takes this row's fp32 sums, or -1; non-anchor rows of a window
      // item are final and are staged for the TMA store
      long long dst_row = -1;
      const bool stage_row = it.window;
      if (it.window) {
        if (fj) {
          int before = pre_tile;
#pragma unroll
          for (int q = 0; q < 4; ++q)
            if (q < (krow >> 5)) before += __popc(tile_words[q]);
          before += __popc(tile_words[krow >> 5] & ((1u << (krow & 31)) - 1u));
          dst_row = before;
        }
      } else if (r < cnt_b) {
        dst_row = r;
      }
      float* dst = dst_row >= 0 ? part + (((size_t)it.b * p.L + dst_row) * p.Hkv + it.kvh) * D : nullptr;
      uint8_t* stage = (h ? sK : sV) + kb * C::TILE;
      // every accumulator column of the row in one round trip, then the writes
      uint32_t accs[D / 32][32];
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) tmem_ld32(tmem + lane_off + col0 + cc * 32, accs[cc]);
      tmem_ld_wait();
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        const uint32_t(&acc)[32] = accs[cc];
        if (dst) {
#pragma unroll
          for (int z = 0; z < 8; ++z)
            atomicAdd(reinterpret_cast<float4*>(dst + cc * 32) + z,
                      make_float4(__uint_as_float(acc[4 * z]) * mul, __uint_as_float(acc[4 * z + 1]) * mul,
                                  __uint_as_float(acc[4 * z + 2]) * mul, __uint_as_float(acc[4 * z + 3]) * mul));
        }
        if (stage_row) {
          // bf16 row into this item's K (dK) or V (dV) buffer, swizzled box layout
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint4 v4 = make_uint4(
                pack_bf16x2(__uint_as_float(acc[8 * q]) * mul, __uint_as_float(acc[8 * q + 1]) * mul),
                pack_bf16x2(__uint_as_float(acc[8 * q + 2]) * mul, __uint_as_float(acc[8 * q + 3]) * mul),
                pack_bf16x2(__uint_as_float(acc[8 * q + 4]) * mul, __uint_as_float(acc[8 * q + 5]) * mul),
                pack_bf16x2(__uint_as_float(acc[8 * q + 6]) * mul, __uint_as_float(acc[8 * q + 7]) * mul));
            const int chunk16 = cc * 4 + q;  // 16-byte chunk of the row
            *reinterpret_cast<uint4*>(stage + (chunk16 >> 3) * kBoxBytes +
                                      sw128_offset(krow, chunk16 & 7)) = v4;
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&bar->acc_free);  // the next item may overwrite dV / dK
      if (stage_row) fence_proxy_async_smem();
      mbar_arrive(&bar->staged[kb]);  // the storer writes the rows out and frees the buffer
    }
    tc_fence_before();
  }
  grid_dep_launch_next();  // the next kernel of the stream may start its prologue
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  // the last CTA out rewinds the item counter, so that a later launch over the same work list
  // (the staged form run again) starts from item 0
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(&counters[3], 1) == (int)gridDim.x - 1) {
      atomicExch(&counters[2], 0);
      atomicExch(&counters[3], 0);
    }
  }
}

// ------------------------------------------------------------------ anchor combine
// dK/dV rows of the anchors: the fp32 sums of every part, rounded once to bf16. One warp per
// compact anchor row (8 per CTA); q4 = float4 chunks per row.
__global__ void __launch_bounds__(256) anchor_combine_kernel(
    const int32_t* __restrict__ anchor_idx, const int32_t* __restrict__ anchor_cnt, int L, int q4,
    const float4* __restrict__ dka, const float4* __restrict__ dva, uint2* __restrict__ dk,
    uint2* __restrict__ dv) {
  grid_dep_wait();
  grid_dep_launch_next();
  const int b = blockIdx.y;
  const int r = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (r >= __ldg(anchor_cnt + b)) return;
  const size_t src = ((size_t)b * L + r) * q4;
  const size_t dst = ((size_t)b * L + __ldg(anchor_idx + (size_t)b * L + r)) * q4;
  for (int c = threadIdx.x & 31; c < q4; c += 32) {
    const float4 x = dka[src + c], y = dva[src + c];
    dk[dst + c] = make_uint2(pack_bf16x2(x.x, x.y), pack_bf16x2(x.z, x.w));
    dv[dst + c] = make_uint2(pack_bf16x2(y.x, y.y), pack_bf16x2(y.z, y.w));
  }
}

size_t bwd_sched_bytes(int B, int L) {
  const size_t T = (L + 127) / 128;
  const size_t cap = (size_t)B * T * ((T + kSegT - 1) / kSegT);
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  return up(4 * sizeof(int32_t)) + up((size_t)B * T * sizeof(int32_t)) + 2 * up(cap * sizeof(WorkItem));
}

static int sm_count_dev() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!cache[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

template <int D>
static cudaError_t set_bwd_attrs() {
  static bool attr_set[64] = {false};  // per device: set once, outside any stream capture
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < 64 && attr_set[dev]) return cudaSuccess;
  constexpr size_t smq = dq_smem_bytes<D>(), smkv = dkv_smem_bytes<D>();
  static_assert(smq <= 227 * 1024 && smkv <= 227 * 1024, "shared memory budget");
  if ((e = cudaFuncSetAttribute(sep_attn_bwd_dq_kernel<D>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smq)) != cudaSuccess)
    return e;
  if ((e = cudaFuncSetAttribute(sep_attn_bwd_dkv_kernel<D>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smkv)) != cudaSuccess)
    return e;
  if (dev >= 0 && dev < 64) attr_set[dev] = true;
  return cudaSuccess;
}

cudaError_t launch_attn_bwd(const AttnMaps& maps, const AttnShape& s, const uint32_t* anchor_bits,
                            const int32_t* anchor_idx, const int32_t* anchor_cnt,
                            const int32_t* gather_end, const int8_t* tile_map, const void* o,
                            const float* lse, const void* dout, const void* q, const void* k,
                            const void* v, void* dq, void* dk, void* dv, void* kc, void* vc,
                            float* delta, float* dka, float* dva, void* sched, int stages,
                            cudaStream_t stream) {
  (void)q;
  (void)tile_map;
  cudaError_t e = cudaSuccess;
  const int T = (s.L + 127) / 128, W = (s.L + 31) / 32;
  // schedule region: counters, tile prefix counts, anchor items, window items
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  const size_t cap = (size_t)s.B * T * ((T + kSegT - 1) / kSegT);
  uint8_t* sw = static_cast<uint8_t*>(sched);
  int32_t* counters = reinterpret_cast<int32_t*>(sw);
  int32_t* tile_prefix = reinterpret_cast<int32_t*>(sw + up(4 * sizeof(int32_t)));
  WorkItem* aitems = reinterpret_cast<WorkItem*>(sw + up(4 * sizeof(int32_t)) + up((size_t)s.B * T * sizeof(int32_t)));
  WorkItem* witems = aitems + up(cap * sizeof(WorkItem)) / sizeof(WorkItem);

  if (stages & kBwdPrep) {
    const dim3 pgrid((s.L + 7) / 8, s.B);
    auto prep = (s.d == 128) ? bwd_prep_kernel<128> : bwd_prep_kernel<64>;
    e = launch_chained(prep, pgrid, dim3(256), 0, stream, static_cast<const uint4*>(o),
                       static_cast<const uint4*>(dout), static_cast<const uint4*>(k),
                       static_cast<const uint4*>(v), anchor_idx, anchor_cnt, s.L, s.Hq, s.Hkv,
                       static_cast<uint4*>(kc), static_cast<uint4*>(vc),
                       reinterpret_cast<float4*>(dka), reinterpret_cast<float4*>(dva), delta,
                       counters);
    if (e != cudaSuccess) return e;
    e = launch_chained(bwd_schedule_kernel, dim3(s.B), dim3(1024), 0, stream, anchor_cnt,
                       gather_end, anchor_bits, s.L, s.n, T, W, tile_prefix, aitems, witems,
                       counters);
    if (e != cudaSuccess) return e;
  }
  if (!(stages & (kBwdDq | kBwdDkv))) return cudaSuccess;
  BwdParams prm;
  prm.tmQ = maps.q;
  prm.tmK = maps.k;
  prm.tmV = maps.v;
  prm.tmKc = maps.kc;
  prm.tmVc = maps.vc;
  prm.tmdO = maps.dout;
  prm.tmK64 = maps.k64;
  prm.tmV64 = maps.v64;
  prm.tmKc64 = maps.kc64;
  prm.tmVc64 = maps.vc64;
  prm.tmdQ = maps.dq;
  prm.tmdK = maps.dk;
  prm.tmdV = maps.dv;
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
  prm.T = T;
  prm.W = W;
  prm.a = s.a;
  prm.n = s.n;
  prm.scale = s.scale;
  prm.scale_log2 = s.scale * 1.4426950408889634f;
  const int nsm = sm_count_dev();
  const int dq_items = T * s.Hq * s.B;
  const int grid_q = dq_items < nsm ? dq_items : nsm;
  if (s.d == 128) {
    if ((e = set_bwd_attrs<128>()) != cudaSuccess) return e;
    if ((stages & kBwdDq) &&
        (e = launch_chained(sep_attn_bwd_dq_kernel<128>, dim3(grid_q), dim3(DqCfg<128>::THREADS),
                            dq_smem_bytes<128>(), stream, prm, dq_items)) != cudaSuccess)
      return e;
    if ((stages & kBwdDkv) &&
        (e = launch_chained(sep_attn_bwd_dkv_kernel<128>, dim3(nsm), dim3(DkvCfg<128>::THREADS),
                            dkv_smem_bytes<128>(), stream, prm, aitems, witems, counters,
                            tile_prefix)) != cudaSuccess)
      return e;
  } else {
    if ((e = set_bwd_attrs<64>()) != cudaSuccess) return e;
    if ((stages & kBwdDq) &&
        (e = launch_chained(sep_attn_bwd_dq_kernel<64>, dim3(grid_q), dim3(DqCfg<64>::THREADS),
                            dq_smem_bytes<64>(), stream, prm, dq_items)) != cudaSuccess)
      return e;
    if ((stages & kBwdDkv) &&
        (e = launch_chained(sep_attn_bwd_dkv_kernel<64>, dim3(nsm), dim3(DkvCfg<64>::THREADS),
                            dkv_smem_bytes<64>(), stream, prm, aitems, witems, counters,
                            tile_prefix)) != cudaSuccess)
      return e;
  }
  if (stages & kBwdDkv) {
    dim3 grid((s.L + 7) / 8, s.B);
    return launch_chained(anchor_combine_kernel, grid, dim3(256), 0, stream, anchor_idx,
                          anchor_cnt, s.L, s.Hkv * s.d / 4, reinterpret_cast<const float4*>(dka),
                          reinterpret_cast<const float4*>(dva), static_cast<uint2*>(dk),
                          static_cast<uint2*>(dv));
  }
  return cudaSuccess;
}

}  // namespace sep
