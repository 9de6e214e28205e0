// sep_attn_fwd: separator-sparse causal attention forward on sm_100a (tcgen05 + TMEM + TMA).
//
// Computes O = M(A, V, M_b) ("How SepLLM reorchestrates the language model...", section
// "SepLLM's Architecture: Composing Efficiency"): softmax attention where query i keeps key j
// iff j <= i && (i - j < n || f[j]), f = initial-or-separator ("SepLLM: Accelerate Large
// Language Models ...", atlas.scime.ai summary, "Approach").
//
// Work item = (query tile t of 128 rows, query head h, batch b). Its keys are split in two
// disjoint parts that together hold every kept key exactly once:
//   * window tiles u = t, t-1, ..., lo(t), lo(t) = max(0, 128t - n + 1) / 128: whole 128-key
//     tiles loaded by TMA in tile mode; FULL tiles need no mask, PARTIAL tiles apply keep()
//     element-wise;
//   * anchors left of tile lo(t): the first gather_end[t] anchors, kept by every row of the
//     tile, read in chunks of 128 from a compacted copy (rows 0..cnt-1 of kc/vc) so that they
//     too arrive as TMA tiles.
// Skipped tiles are never loaded.
//
// Persistent CTAs, one per SM, 352 threads: warps 0-7 softmax (two warps per query row, each
// owning 64 key columns; thread = row = TMEM lane), warp 8 TMA producer, warp 9 TMEM allocator
// and MMA issuer (one thread), warp 10 O storer. Per key tile j:
//   S_j = Q K_j^T                  (tcgen05.mma, A and B K-major in smem, D in TMEM)
//   P_j = exp2(S_j*c - m)          (softmax warps: tcgen05.ld S, online max with lazy
//                                   rescale of O, tcgen05.st of bf16 P into TMEM)
//   O  += P_j V_j                  (tcgen05.mma, A = P from TMEM, B = V MN-major in smem)
// S_{j+1} is issued before PV_j so the tensor core works while the softmax runs.
#include <cuda_runtime.h>

#include <algorithm>

#include "sep_common.cuh"
#include "sep_launch.h"
#include "sep_tiles.cuh"

namespace sep {

struct FwdParams {
  CUtensorMap tmQ, tmK, tmV, tmKc, tmVc, tmO;
  CUtensorMap tmK64, tmV64, tmKc64, tmVc64;  // 64-row boxes: the two halves of a merged tile
  const uint32_t* anchor_bits;  // [B, W] packed anchor flags
  const int32_t* gather_end;
  const int8_t* tile_map;
  __nv_bfloat16* o;
  float* lse;
  unsigned* err;
  unsigned long long wait_ns;  // limit of each pipeline wait (drain waits keep kWaitLimitNs)
  int B, L, Hq, Hkv, T, W, a, n;
  float scale_log2;
};

// Every kFwdEx2FmaPeriod-th pair of scores of the softmax takes its exp2 on the FMA pipe
// (ex2_fma2) instead of the XU pipe: 74.7 -> 71.3 us for the Pythia-160m forward with a quarter
// moved (a third: 72.2 us, a half: 73.9 us).
#ifndef SEP_FWD_EX2_FMA_PERIOD
#define SEP_FWD_EX2_FMA_PERIOD 4
#endif
constexpr int kFwdEx2FmaPeriod = SEP_FWD_EX2_FMA_PERIOD;

template <int D>
struct FwdCfg {
  static constexpr int BM = 128, BN = 128;
  static constexpr int KB = D / 64;                 // 128-byte column boxes per row
  static constexpr int BOX_BYTES = 128 * 64 * 2;    // one [128 rows][64 cols] bf16 box
  static constexpr int TILE_BYTES = KB * BOX_BYTES; // one [128][D] tile
  static constexpr int NST = (D == 128) ? 2 : 4;    // K/V pipeline stages
  static constexpr int SMEM_TILES = TILE_BYTES * (2 + 2 * NST);  // Q x2, NST x (K, V)
  static constexpr int COL_S = 0;  // S: 128 fp32 columns
  // O in two accumulators, one per key half (softmax warpgroup): O_wg = sum over the tile's keys
  // 64 wg .. 64 wg + 63 of P V, each scaled by its own warpgroup's running row max
  static constexpr int COL_O0 = 128, COL_O1 = 128 + D;
  static constexpr int COL_P = 128 + 2 * D;  // P: 64 columns (bf16 pairs)
  static constexpr int TMEM_COLS = 512;
  static_assert(COL_P + 64 <= TMEM_COLS, "TMEM columns");
  static constexpr int THREADS = 352;  // 8 softmax warps, producer, MMA issuer, O storer
};

template <int NST>
struct FwdBar {
  uint64_t q_full[2], q_empty[2], o_staged[2];
  uint64_t k_full[NST], k_empty[NST], v_full[NST], v_empty[NST];
  uint64_t s_full, s_free, p_ready, pv_done;
  uint64_t drain;
  uint64_t pair[4];  // exchange barrier of softmax warps w and w + 4 (64 arrivals)
  float xm[2][128];  // running row max of each warpgroup's key half, exchanged once per item
  float xl[2][128];  // and its row sum
  uint32_t tmem_base;
  int abort_flag;
};

template <int D>
constexpr size_t fwd_smem_bytes() {
  return 1024 /*alignment slack*/ + FwdCfg<D>::SMEM_TILES + sizeof(FwdBar<FwdCfg<D>::NST>);
}

// Work item x (heaviest query tiles first): query tile t, head h, batch b, and its key tiles.
// Half window: when the lower 64 keys of the oldest window tile lo lie outside every row's band
// (128 t - n + 1 >= 128 lo + 64, e.g. any n <= 64), every row keeps exactly the anchors among
// them, like the anchors left of tile lo; they join the gathered anchors (ge counts both), and
// the oldest window tile becomes a merged tile: its lower half holds compacted anchors 0..63,
// its upper half the keys 128 lo + 64 .. 128 lo + 127. The remaining anchors follow in chunks of
// 128 from compacted row arow0 = 64. This saves the key tile that anchors up to 64 would
// otherwise take, and half of the padding of the gathered part.
struct FwdItem {
  int t, h, b, nwin, ge, N, arow0;
  bool half;
};
__device__ __forceinline__ FwdItem fwd_item_base(const FwdParams& p, int x) {
  FwdItem it;
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
// Gathered anchors of item x: gather_end (anchors left of tile lo), plus those in the lower half
// of tile lo for a half-window item.
__device__ __forceinline__ int fwd_item_ge(const FwdParams& p, int x) {
  const FwdItem it = fwd_item_base(p, x);
  int ge = p.gather_end[(size_t)it.b * p.T + it.t];
  if (it.half) {
    const uint32_t* w = p.anchor_bits + (size_t)it.b * p.W + (size_t)(it.t - it.nwin + 1) * 4;
    ge += __popc(__ldg(w)) + __popc(__ldg(w + 1));
  }
  return ge;
}
__device__ __forceinline__ FwdItem fwd_item_with(const FwdParams& p, int x, int ge) {
  FwdItem it = fwd_item_base(p, x);
  it.ge = ge;
  it.N = it.nwin + (max(0, ge - it.arow0) + 127) / 128;
  return it;
}

// Raw mask inputs of one window key tile: its tile-map class and 128 anchor-flag bits.
struct TileRaw {
  uint32_t fb[4];
  int cls;
};
__device__ __forceinline__ TileRaw load_tile_raw(const FwdParams& p, int b, int t, int u) {
  TileRaw r;
  r.cls = p.tile_map[((size_t)b * p.T + t) * p.T + u];
  const uint32_t* w = p.anchor_bits + (size_t)b * p.W + (size_t)u * 4;
#pragma unroll
  for (int q = 0; q < 4; ++q) r.fb[q] = (u * 4 + q < p.W) ? __ldg(w + q) : 0u;
  return r;
}

// Persistent: CTA c handles items c, c + gridDim.x, ... Every role walks the same flattened
// sequence of key tiles (g = 0, 1, ... over all its items), so pipeline phases carry across
// item boundaries and the next item's loads and first MMA overlap the current item's tail.
// Warps 0-7 run the softmax: warpgroup wg = 0, 1 handles key columns 64wg..64wg+63 of every
// query row (thread = row = TMEM lane), so two warps per SM sub-partition share the
// exponentials; warp 8 is the TMA producer, warp 9 the MMA issuer.
template <int D>
__global__ void __launch_bounds__(FwdCfg<D>::THREADS, 1)
    sep_attn_fwd_kernel(const __grid_constant__ FwdParams p, int nitems) {
  using C = FwdCfg<D>;
  constexpr int NST = C::NST;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ = smem;                       // 2 buffers (item parity)
  uint8_t* sK = sQ + 2 * C::TILE_BYTES;
  uint8_t* sV = sK + NST * C::TILE_BYTES;
  FwdBar<NST>* bar = reinterpret_cast<FwdBar<NST>*>(sV + NST * C::TILE_BYTES);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort_flag = &bar->abort_flag;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar->q_full[s], 1);
      mbar_init(&bar->q_empty[s], 1);
      mbar_init(&bar->o_staged[s], 256);
    }
    for (int s = 0; s < NST; ++s) {
      mbar_init(&bar->k_full[s], 1);
      mbar_init(&bar->k_empty[s], 1);
      mbar_init(&bar->v_full[s], 1);
      mbar_init(&bar->v_empty[s], 1);
    }
    mbar_init(&bar->s_full, 1);
    mbar_init(&bar->s_free, 256);
    mbar_init(&bar->p_ready, 256);
    mbar_init(&bar->pv_done, 1);
    mbar_init(&bar->drain, 1);
    for (int s = 0; s < 4; ++s) mbar_init(&bar->pair[s], 64);
    bar->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc(&bar->tmem_base, C::TMEM_COLS);
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
      tma_prefetch_desc(&p.tmQ);
      tma_prefetch_desc(&p.tmK);
      tma_prefetch_desc(&p.tmV);
      tma_prefetch_desc(&p.tmKc);
      tma_prefetch_desc(&p.tmVc);
      tma_prefetch_desc(&p.tmK64);
      tma_prefetch_desc(&p.tmV64);
      tma_prefetch_desc(&p.tmKc64);
      tma_prefetch_desc(&p.tmVc64);
      int g = 0;
      int kq = 0;  // items whose Q load was issued
      bool ok = true;
      int ge_cur = fwd_item_ge(p, blockIdx.x);
      for (int k = 0, x = blockIdx.x; ok && x < nitems; ++k, x += gridDim.x) {
        const FwdItem it = fwd_item_with(p, x, ge_cur);
        if (x + (int)gridDim.x < nitems) ge_cur = fwd_item_ge(p, x + gridDim.x);  // prefetch
        const int kvh = it.h / (p.Hq / p.Hkv);
        const int qb = k & 1;
        if (k >= 2 &&
            !mbar_wait(&bar->q_empty[qb], ((k - 2) >> 1) & 1, p.err, abort_flag, p.wait_ns)) {
          ok = false;
          break;
        }
        kq = k + 1;
        mbar_arrive_expect_tx(&bar->q_full[qb], C::TILE_BYTES);
        for (int kb = 0; kb < C::KB; ++kb)
          tma_load_4d(sQ + qb * C::TILE_BYTES + kb * C::BOX_BYTES, &p.tmQ, &bar->q_full[qb],
                      kb * 64, it.h, it.t * C::BM, it.b);
        for (int j = 0; j < it.N; ++j, ++g) {
          const int st = g % NST, r = g / NST;
          const bool win = j < it.nwin;
          const bool merged = it.half && j == it.nwin - 1;
          const CUtensorMap* mk = win ? &p.tmK : &p.tmKc;
          const CUtensorMap* mv = win ? &p.tmV : &p.tmVc;
          const int row0 = win ? (it.t - j) * C::BN : it.arow0 + (j - it.nwin) * C::BN;
          if (r > 0 && !mbar_wait(&bar->k_empty[st], (r - 1) & 1, p.err, abort_flag, p.wait_ns)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bar->k_full[st], C::TILE_BYTES);
          for (int kb = 0; kb < C::KB; ++kb) {
            uint8_t* dst = sK + st * C::TILE_BYTES + kb * C::BOX_BYTES;
            if (merged) {  // compacted anchors 0..63, then keys 128 lo + 64 ..
              tma_load_4d(dst, &p.tmKc64, &bar->k_full[st], kb * 64, kvh, 0, it.b);
              tma_load_4d(dst + 64 * 128, &p.tmK64, &bar->k_full[st], kb * 64, kvh, row0 + 64, it.b);
            } else {
              tma_load_4d(dst, mk, &bar->k_full[st], kb * 64, kvh, row0, it.b);
            }
          }
          if (r > 0 && !mbar_wait(&bar->v_empty[st], (r - 1) & 1, p.err, abort_flag, p.wait_ns)) {
            mbar_wait(&bar->k_full[st], r & 1, nullptr, nullptr);
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bar->v_full[st], C::TILE_BYTES);
          for (int kb = 0; kb < C::KB; ++kb) {
            uint8_t* dst = sV + st * C::TILE_BYTES + kb * C::BOX_BYTES;
            if (merged) {
              tma_load_4d(dst, &p.tmVc64, &bar->v_full[st], kb * 64, kvh, 0, it.b);
              tma_load_4d(dst + 64 * 128, &p.tmV64, &bar->v_full[st], kb * 64, kvh, row0 + 64, it.b);
            } else {
              tma_load_4d(dst, mv, &bar->v_full[st], kb * 64, kvh, row0, it.b);
            }
          }
        }
      }
      if (!ok) {
        // drain: let every load issued for the last NST tiles and the last two Q tiles land
        // (older phases completed already, so their waits return at once)
        for (int gg = max(0, g - NST); gg < g; ++gg) {
          mbar_wait(&bar->k_full[gg % NST], (gg / NST) & 1, nullptr, nullptr);
          mbar_wait(&bar->v_full[gg % NST], (gg / NST) & 1, nullptr, nullptr);
        }
        for (int kk = max(0, kq - 2); kk < kq; ++kk)
          mbar_wait(&bar->q_full[kk & 1], (kk >> 1) & 1, nullptr, nullptr);
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = make_idesc_bf16(128, 128, false, false);
      constexpr uint32_t idO = make_idesc_bf16(128, D, false, true);
      const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK), sVa = smem_u32(sV);
      bool ok = true;
      int g = 0;           // global index of the next S tile
      int pv_pending = -1; // global index of the tile whose PV is still to issue
      int pv_first = 0;    // that tile is the first of its item (overwrite O)
      auto issue_PV = [&](int gg, int first) -> bool {
        const int st = gg % NST;
        if (!mbar_wait(&bar->p_ready, gg & 1, p.err, abort_flag, p.wait_ns)) return false;
        if (!mbar_wait(&bar->v_full[st], (gg / NST) & 1, p.err, abort_flag, p.wait_ns)) return false;
        tc_fence_after();
        const uint32_t aP = tmem + C::COL_P;
        const uint32_t vlo = sdesc_lo(sVa + st * C::TILE_BYTES, C::BOX_BYTES);
#pragma unroll
        for (int kk = 0; kk < 128 / 16; ++kk)
          mma_ts(tmem + (kk < 4 ? C::COL_O0 : C::COL_O1), aP + kk * 8,
                 sdesc_join(vlo + kk * (2048 >> 4), kDescHi), idO,
                 (!first || (kk & 3) > 0) ? 1u : 0u);
        tc_commit(&bar->pv_done);
        tc_commit(&bar->v_empty[st]);
        return true;
      };
      int ge_cur = fwd_item_ge(p, blockIdx.x);
      for (int k = 0, x = blockIdx.x; ok && x < nitems; ++k, x += gridDim.x) {
        const FwdItem it = fwd_item_with(p, x, ge_cur);
        if (x + (int)gridDim.x < nitems) ge_cur = fwd_item_ge(p, x + gridDim.x);  // prefetch
        const int qb = k & 1;
        if (!mbar_wait(&bar->q_full[qb], (k >> 1) & 1, p.err, abort_flag, p.wait_ns)) {
          ok = false;
          break;
        }
        const uint32_t sQb = sQa + qb * C::TILE_BYTES;
        for (int j = 0; j < it.N; ++j, ++g) {
          const int st = g % NST;
          if (!mbar_wait(&bar->k_full[st], (g / NST) & 1, p.err, abort_flag, p.wait_ns)) {
            ok = false;
            break;
          }
          // S has one buffer: the softmax warps must have loaded S_{g-1}
          if (g > 0 && !mbar_wait(&bar->s_free, (g - 1) & 1, p.err, abort_flag, p.wait_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t qlo = sdesc_lo(sQb, 16), klo = sdesc_lo(sKa + st * C::TILE_BYTES, 16);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = ((kk >> 2) * C::BOX_BYTES + (kk & 3) * 32) >> 4;
            mma_ss(tmem + C::COL_S, sdesc_join(qlo + off, kDescHi), sdesc_join(klo + off, kDescHi),
                   idS, kk > 0 ? 1u : 0u);
          }
          tc_commit(&bar->s_full);
          tc_commit(&bar->k_empty[st]);
          // P V of the previous tile, while the softmax warps work on this one
          if (pv_pending >= 0 && !issue_PV(pv_pending, pv_first)) { ok = false; break; }
          pv_pending = g;
          pv_first = (j == 0);
        }
      }
      if (ok && pv_pending >= 0) issue_PV(pv_pending, pv_first);
      tc_commit(&bar->drain);
      mbar_wait(&bar->drain, 0, nullptr, nullptr);
    }
  } else if (warp == 10) {
    // ------------------------------------------------------------ O tile storer
    if (lane == 0) {
      bool ok = true;
      for (int k = 0, x = blockIdx.x; ok && x < nitems; ++k, x += gridDim.x) {
        const FwdItem it = fwd_item_base(p, x);
        if (!mbar_wait(&bar->o_staged[k & 1], (k >> 1) & 1, p.err, abort_flag, p.wait_ns)) {
          ok = false;
          break;
        }
        const uint8_t* stage = sQ + (k & 1) * C::TILE_BYTES;
        for (int kb = 0; kb < C::KB; ++kb)
          tma_store_4d(&p.tmO, stage + kb * C::BOX_BYTES, kb * 64, it.h, it.t * C::BM, it.b);
        bulk_commit_group();
        bulk_wait_read_all();  // the staging buffer may now take a later item's Q
        mbar_arrive(&bar->q_empty[k & 1]);
      }
      bulk_wait_all();  // O stores complete before the CTA exits
    }
  } else {
    // ------------------------------------------------------------ softmax warpgroups
    const int row = threadIdx.x & 127;  // query row = TMEM lane
    const int wg = threadIdx.x >> 7;    // column half
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    // Warps w and w + 4 (the two halves of the same rows) exchange row statistics through an
    // mbarrier with a bounded wait, so that when one of them gives up the other cannot block
    // on the exchange.
    int xph = 0;  // exchanges done
    auto pair_sync = [&]() -> bool {
      mbar_arrive(&bar->pair[warp & 3]);
      const bool r = mbar_wait(&bar->pair[warp & 3], xph & 1, p.err, abort_flag, p.wait_ns);
      ++xph;
      return __all_sync(0xffffffffu, r);
    };
    const float sl2 = p.scale_log2;
    bool ok = true;
    int g = 0;
    int k_item = 0;  // this CTA's item counter (Q buffer parity)
    int ge_cur = fwd_item_ge(p, blockIdx.x);
    TileRaw cur;  // mask inputs of the next tile to process, loaded one tile ahead
    {
      const FwdItem f0 = fwd_item_base(p, blockIdx.x);
      cur = load_tile_raw(p, f0.b, f0.t, f0.t);
    }
    for (int x = blockIdx.x; ok && x < nitems; x += gridDim.x) {
      const FwdItem it = fwd_item_with(p, x, ge_cur);
      const int xn = x + gridDim.x;
      if (xn < nitems) ge_cur = fwd_item_ge(p, xn);  // prefetch the next item's gather count
      const long long i = (long long)it.t * C::BM + row;
      float m_run = -INFINITY, l_run = 0.f;
      for (int j = 0; j < it.N; ++j, ++g) {
        const TileRaw raw = cur;
        // prefetch the next tile's mask inputs (next window tile of this item, or the
        // diagonal tile of the next item)
        if (j + 1 < it.nwin) {
          cur = load_tile_raw(p, it.b, it.t, it.t - (j + 1));
        } else if (j + 1 == it.N && xn < nitems) {
          const FwdItem fn = fwd_item_base(p, xn);
          cur = load_tile_raw(p, fn.b, fn.t, fn.t);
        }
        if (!__all_sync(0xffffffffu, mbar_wait(&bar->s_full, g & 1, p.err, abort_flag, p.wait_ns))) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t s[64];
        {
          const uint32_t a0 = tmem + lane_off + C::COL_S + wg * 64;
          tmem_ld32(a0, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
          tmem_ld32(a0 + 32, *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
          tmem_ld_wait();
        }
        tc_fence_before();
        mbar_arrive(&bar->s_free);  // S may be overwritten by the next tile's MMA
        // ---- mask of this thread's 64 columns (words 2wg, 2wg+1 of the tile)
        uint32_t keep[2] = {0xffffffffu, 0xffffffffu};
        bool masked = false;
        if (it.half && j == it.nwin - 1 && wg == 0) {
          // lower half of the merged tile: gathered anchors 0..63, kept by every row
          const int cnt = min(it.ge, 64);
          if (cnt < 64) {
            masked = true;
#pragma unroll
            for (int w = 0; w < 2; ++w) keep[w] = range_word(0, cnt - 1, w);
          }
        } else if (j < it.nwin) {
          const int u = it.t - j;
          const long long k0 = (long long)u * C::BN;
          if (raw.cls != SEP_TILE_FULL) {
            masked = true;
#pragma unroll
            for (int w = 0; w < 2; ++w)
              keep[w] = window_keep_word(2 * wg + w, i, k0, p.n, p.L, raw.fb[2 * wg + w]);
          } else if (k0 + C::BN > p.L) {
            masked = true;
#pragma unroll
            for (int w = 0; w < 2; ++w) keep[w] = range_word(0, (long long)p.L - 1 - k0, 2 * wg + w);
          }
        } else {
          const int rem = it.ge - it.arow0 - (j - it.nwin) * C::BN;  // valid anchors in this chunk
          if (rem < C::BN) {
            masked = true;
#pragma unroll
            for (int w = 0; w < 2; ++w) keep[w] = range_word(0, rem - 1, 2 * wg + w);
          }
        }
        // ---- row max of this warpgroup's 64 key columns (three-input max, 4 chains); the two
        // halves keep separate running statistics and accumulators until the item's epilogue
        if (masked) {
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (!((keep[c >> 5] >> (c & 31)) & 1u)) s[c] = __float_as_uint(-INFINITY);
        }
        float mx4[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) mx4[q] = -INFINITY;
#pragma unroll
        for (int c = 0; c < 64; c += 2)
          mx4[(c >> 1) & 3] =
              fmax3(mx4[(c >> 1) & 3], __uint_as_float(s[c]), __uint_as_float(s[c + 1]));
        const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
        // ---- online max with lazy rescale (only when the max grows by more than 2^8)
        const float m_tile = mx * sl2;
        float alpha = 1.0f;
        bool any_rescale = false;
        if (j == 0) {
          m_run = m_tile;
        } else {
          const bool need = m_tile > m_run + 8.0f;
          any_rescale = __any_sync(0xffffffffu, need);
          if (need) {
            alpha = ex2(m_run - m_tile);
            l_run *= alpha;
            m_run = m_tile;
          }
        }
        const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
        // ---- P = exp2(S * scale*log2e - m), partial row sum (8 chains), packed to bf16 pairs
        // in place over the already consumed S registers (pair c/2 <= c)
        // two columns per packed fp32x2 instruction (scale and subtract, and the row sums)
        float2 sum4[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) sum4[q] = make_float2(0.f, 0.f);
        const float2 sl2x2 = make_float2(sl2, sl2), nm2 = make_float2(-m_use, -m_use);
#pragma unroll
        for (int c = 0; c < 64; c += 2) {
          const float2 x = f2_fma(make_float2(__uint_as_float(s[c]), __uint_as_float(s[c + 1])),
                                  sl2x2, nm2);
          // every kFwdEx2FmaPeriod-th pair on the FMA pipe, the rest on the XU pipe
          const float2 e = (kFwdEx2FmaPeriod > 0 &&
                            (c >> 1) % (kFwdEx2FmaPeriod > 0 ? kFwdEx2FmaPeriod : 1) ==
                                kFwdEx2FmaPeriod - 1)
                               ? ex2_fma2(x)
                               : make_float2(ex2(x.x), ex2(x.y));
          sum4[(c >> 1) & 3] = f2_add(sum4[(c >> 1) & 3], e);
          s[c >> 1] = pack_bf16x2(e.x, e.y);
        }
        l_run += ((sum4[0].x + sum4[0].y) + (sum4[1].x + sum4[1].y)) +
                 ((sum4[2].x + sum4[2].y) + (sum4[3].x + sum4[3].y));
        // P and O: the previous tile's P V must be complete (it read P and accumulated O)
        if (g > 0 &&
            !__all_sync(0xffffffffu,
                        mbar_wait(&bar->pv_done, (g - 1) & 1, p.err, abort_flag, p.wait_ns))) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (any_rescale) {
#pragma unroll 1
          for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t ov[32];
            const uint32_t ao = tmem + lane_off + (wg ? C::COL_O1 : C::COL_O0) + cc * 32;
            tmem_ld32(ao, ov);
            tmem_ld_wait();
#pragma unroll
            for (int q = 0; q < 32; ++q) ov[q] = __float_as_uint(__uint_as_float(ov[q]) * alpha);
            tmem_st32(ao, ov);
          }
        }
        tmem_st32(tmem + lane_off + C::COL_P + wg * 32, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&bar->p_ready);
      }
      if (!ok) break;
      // ---- epilogue of this item: the two halves' running max and row sum are exchanged and
      // combined, O = (O0 2^(m0-m) + O1 2^(m1-m)) / (l0 2^(m0-m) + l1 2^(m1-m)), LSE (O0 / O1
      // are reused by the next item's first P V, which the MMA warp issues only after this
      // thread's next p_ready; the other half reads these slots before its next p_ready, so
      // they are not rewritten before being read)
      bar->xm[wg][row] = m_run;
      bar->xl[wg][row] = l_run;
      if (!pair_sync()) {
        ok = false;
        break;
      }
      const float m_o = bar->xm[wg ^ 1][row], l_o = bar->xl[wg ^ 1][row];
      const float m0 = wg ? m_o : m_run, m1 = wg ? m_run : m_o;
      const float l0 = wg ? l_o : l_run, l1 = wg ? l_run : l_o;
      const float m_max = fmaxf(m0, m1);
      const float m_row = (m_max == -INFINITY) ? 0.f : m_max;
      const float a0 = ex2(m0 - m_row), a1 = ex2(m1 - m_row);
      const float l_tot = l0 * a0 + l1 * a1;
      if (!__all_sync(0xffffffffu,
                      mbar_wait(&bar->pv_done, (g - 1) & 1, p.err, abort_flag, p.wait_ns))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const float inv_l = 1.0f / l_tot;
      const float c0 = a0 * inv_l, c1 = a1 * inv_l;
      const bool valid = i < p.L;
      // O / l as bf16 into the item's Q buffer (every S MMA of the item has completed, so Q is
      // no longer read), in the swizzled box layout, then one TMA store of the whole tile
      uint8_t* stage = sQ + (k_item & 1) * C::TILE_BYTES;
#pragma unroll 1
      for (int cc = 0; cc < D / 64; ++cc) {
        uint32_t ov0[32], ov1[32];
        tmem_ld32(tmem + lane_off + C::COL_O0 + wg * (D / 2) + cc * 32, ov0);
        tmem_ld32(tmem + lane_off + C::COL_O1 + wg * (D / 2) + cc * 32, ov1);
        tmem_ld_wait();
        uint32_t pkd[16];
#pragma unroll
        for (int q = 0; q < 16; ++q)
          pkd[q] = pack_bf16x2(
              fmaf(__uint_as_float(ov0[2 * q]), c0, __uint_as_float(ov1[2 * q]) * c1),
              fmaf(__uint_as_float(ov0[2 * q + 1]), c0, __uint_as_float(ov1[2 * q + 1]) * c1));
        const int col0 = wg * (D / 2) + cc * 32;  // first column of these 32
        uint8_t* box = stage + (col0 >> 6) * C::BOX_BYTES;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int chunk = ((col0 & 63) >> 3) + q;
          *reinterpret_cast<uint4*>(box + sw128_offset(row, chunk)) =
              make_uint4(pkd[4 * q], pkd[4 * q + 1], pkd[4 * q + 2], pkd[4 * q + 3]);
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(&bar->o_staged[k_item & 1]);  // the storer warp writes the tile out
      if (valid && wg == 0)
        p.lse[((size_t)it.b * p.Hq + it.h) * p.L + i] =
            (m_row + __log2f(l_tot)) * 0.69314718055994531f;
      ++k_item;
    }
    tc_fence_before();
  }

  grid_dep_launch_next();  // the next kernel of the stream may start its prologue
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------------ anchor compaction
// Row r < anchor_cnt[b] of kc/vc receives the K/V row of anchor r; the 128 rows after the last
// anchor are zeroed, so that the last (partly valid) anchor chunk holds finite values wherever
// it starts (at a multiple of 128, or at 64 + a multiple of 128 after a merged tile): masked
// scores still multiply V in the P*V product.
// One warp per compacted row (8 rows per CTA); CTAs past the last anchor tile exit at once.
__global__ void __launch_bounds__(256) compact_anchors_kernel(
    const uint4* __restrict__ k, const uint4* __restrict__ v, const int32_t* __restrict__ anchor_idx,
    const int32_t* __restrict__ anchor_cnt, int L, int kv_ch, uint4* __restrict__ kc,
    uint4* __restrict__ vc) {
  grid_dep_wait();
  grid_dep_launch_next();
  const int b = blockIdx.y;
  const int cnt = __ldg(anchor_cnt + b);
  const int pad_end = min(L, cnt + 128);
  const int i = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (i >= pad_end) return;
  compact_anchor_row(k, v, anchor_idx, cnt, L, b, i, kv_ch, kc, vc, threadIdx.x & 31);
}

cudaError_t launch_compact_anchors(const void* k, const void* v, const int32_t* anchor_idx,
                                   const int32_t* anchor_cnt, int B, int L, int Hkv, int d,
                                   void* kc, void* vc, cudaStream_t stream) {
  const int kv_ch = Hkv * d * 2 / 16;
  dim3 grid((L + 7) / 8, B);
  return launch_chained(compact_anchors_kernel, grid, dim3(256), 0, stream,
                        static_cast<const uint4*>(k), static_cast<const uint4*>(v), anchor_idx,
                        anchor_cnt, L, kv_ch, static_cast<uint4*>(kc), static_cast<uint4*>(vc));
}

static int sm_count() {
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
  const int nitems = T * Hq * B;
  const int grid = std::min(nitems, sm_count());
  return launch_chained(sep_attn_fwd_kernel<D>, dim3(grid), dim3(FwdCfg<D>::THREADS), smem, stream,
                        prm, nitems);
}

cudaError_t launch_attn_fwd(const AttnMaps& maps, const AttnShape& s, const uint32_t* anchor_bits,
                            const int32_t* gather_end, const int8_t* tile_map, void* o,
                            float* lse, cudaStream_t stream) {
  FwdParams prm;
  prm.tmQ = maps.q;
  prm.tmK = maps.k;
  prm.tmV = maps.v;
  prm.tmKc = maps.kc;
  prm.tmVc = maps.vc;
  prm.tmO = maps.o;
  prm.tmK64 = maps.k64;
  prm.tmV64 = maps.v64;
  prm.tmKc64 = maps.kc64;
  prm.tmVc64 = maps.vc64;
  prm.anchor_bits = anchor_bits;
  prm.gather_end = gather_end;
  prm.tile_map = tile_map;
  prm.o = static_cast<__nv_bfloat16*>(o);
  prm.lse = lse;
  prm.err = device_error_word();
  prm.wait_ns = pipeline_wait_limit_ns();
  prm.B = s.B;
  prm.L = s.L;
  prm.Hq = s.Hq;
  prm.Hkv = s.Hkv;
  prm.T = (s.L + 127) / 128;
  prm.W = (s.L + 31) / 32;
  prm.a = s.a;
  prm.n = s.n;
  prm.scale_log2 = s.scale * 1.4426950408889634f;
  if (s.d == 128) return launch_fwd_t<128>(prm, prm.T, s.Hq, s.B, stream);
  if (s.d == 64) return launch_fwd_t<64>(prm, prm.T, s.Hq, s.B, stream);
  return cudaErrorInvalidValue;
}

}  // namespace sep
