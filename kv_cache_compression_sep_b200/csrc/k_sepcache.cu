// SepCache streaming decode on sm_100a: cache update (append / compress), prefill from a prompt
// and single-query attention with positional-encoding shifting.
//
// Cache blocks ("How SepLLM reorchestrates the language model...", beiduofen.top, section
// "SepLLM's Architecture: Composing Efficiency"): a initial slots, a separator FIFO of s slots,
// a local-window FIFO of w slots and, with a usage threshold c > 0, a Past Window of
// P = c - a - w slots. When the window overflows, its oldest token leaves: with c = 0 it moves
// to the separator FIFO if it is a separator and is dropped otherwise; with c > 0 it goes to
// the Past Window, which is compressed (its separators to the FIFO, the rest dropped) by the
// step that makes the total usage reach c. The separator FIFO drops its oldest entries when
// full. Positions are ranks inside the cache (SepLLM project card, "Limitations & Caveats":
// streaming needs positional-encoding shifting): the key of rank p is seen at RoPE(p) and the
// query at RoPE(occupied - 1).
//
// Slot storage per (sequence, KV head) is [n][d], n = a + s + P + w: initial slots, the
// separator ring, the past window (a plain array, emptied by each compression), the window
// ring.
//
// Rotation storage. Inside each block the rank of a key is its own counter plus one offset that
// the whole block shares: initial, past-window and window keys hold consecutive original
// positions t, and the separators in the FIFO hold consecutive admission indices A (the A-th
// separator ever admitted; the FIFO keeps the newest, oldest first). So every key is stored
// rotated once by RoPE(counter), counter = t or A, and since RoPE(m)q . RoPE(p)k =
// RoPE(m - p + u)q . RoPE(u)k, the query is rotated once per block by RoPE(m - offset) instead of
// rotating every key at every step. A key is rotated by RoPE(t) when it is appended and, when it
// enters the separator FIFO, re-rotated by RoPE(A - t). Without positional shifting
// (original_positions) keys stay at RoPE(t) and every block's query angle is its own position.
// Angles are formed and reduced in fp64 (position x inverse frequency), rotations are rounded to
// bf16.
//
// Decode: one CTA per (sequence, KV head), all resident in one wave. Bulk copies stream the
// retained K/V rows in rank order through a shared-memory ring; a group of D/8 lanes takes one
// key row (8 contiguous elements per lane, one 16-byte load of K and one of V), forms the
// partial dot products with the block's rotated queries, reduces them across the group so that
// each lane is left the score of one query, keeps that query's online softmax, and accumulates
// the V rows of every query. Groups are combined through shared memory. No global scratch.
#include <cuda_runtime.h>

#include <type_traits>

#include "sep_common.cuh"
#include "sep_launch.h"

namespace sep {

// ------------------------------------------------------------------ RoPE of stored keys
// (cos, sin) of the angle pos * f: the angle is formed in fp64 and reduced to [-pi, pi] by
// subtracting the nearest multiple of 2 pi (fp64), then the fp32 sincosf of the reduced angle is
// taken. The error (about 1e-7 absolute, from rounding the reduced angle to fp32) is far below the
// bf16 rounding of the rotated keys, and positions up to 2^31 keep full precision.
__device__ __forceinline__ void rope_cos_sin(long long pos, double f, float* cs, float* sn) {
  constexpr double kTwoPi = 6.283185307179586, kInvTwoPi = 0.15915494309189535;
  const double x = __dmul_rn((double)pos, f);
  const double r = __fma_rn(-rint(__dmul_rn(x, kInvTwoPi)), kTwoPi, x);
  sincosf((float)r, sn, cs);
}

// Rotate-half pairs (k, k + d/2), angle pos * freq[k], freq[k] = theta^(-2k/d) (fp64 table).
// x holds dims k0..k0+7, y dims k0+d/2..k0+d/2+7 of one key row. The (cos, sin) of the 8 pairs
// come from rope_cos_sin (rope_chunk_cs); the rotation is fp32 arithmetic with the operations
// spelled out (no contraction choices left to the compiler), rounded to bf16, so that every
// kernel that rotates the same row by the same angle produces the same bits.
struct ChunkCS {
  float c[8], s[8];
};
__device__ __forceinline__ ChunkCS rope_chunk_cs(int k0, long long pos,
                                                 const double* __restrict__ freq) {
  ChunkCS r;
#pragma unroll
  for (int z = 0; z < 8; ++z) rope_cos_sin(pos, __ldg(freq + k0 + z), &r.c[z], &r.s[z]);
  return r;
}
__device__ __forceinline__ void rope_apply_chunks(uint4& x, uint4& y, const ChunkCS& r) {
  uint32_t xs[4] = {x.x, x.y, x.z, x.w}, ys[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const __nv_bfloat162 xa = *reinterpret_cast<const __nv_bfloat162*>(&xs[q]);
    const __nv_bfloat162 ya = *reinterpret_cast<const __nv_bfloat162*>(&ys[q]);
    const float xv[2] = {__low2float(xa), __high2float(xa)};
    const float yv[2] = {__low2float(ya), __high2float(ya)};
    __nv_bfloat16 xo[2], yo[2];
#pragma unroll
    for (int z = 0; z < 2; ++z) {
      const float cs = r.c[2 * q + z], sn = r.s[2 * q + z];
      xo[z] = __float2bfloat16_rn(__fmaf_rn(xv[z], cs, -__fmul_rn(yv[z], sn)));
      yo[z] = __float2bfloat16_rn(__fmaf_rn(yv[z], cs, __fmul_rn(xv[z], sn)));
    }
    const __nv_bfloat162 xp = __halves2bfloat162(xo[0], xo[1]);
    const __nv_bfloat162 yp = __halves2bfloat162(yo[0], yo[1]);
    xs[q] = *reinterpret_cast<const uint32_t*>(&xp);
    ys[q] = *reinterpret_cast<const uint32_t*>(&yp);
  }
  x = make_uint4(xs[0], xs[1], xs[2], xs[3]);
  y = make_uint4(ys[0], ys[1], ys[2], ys[3]);
}
__device__ __forceinline__ void rope_rotate_chunks(uint4& x, uint4& y, int k0, long long pos,
                                                   const double* __restrict__ freq) {
  if (pos == 0) return;
  rope_apply_chunks(x, y, rope_chunk_cs(k0, pos, freq));
}

// ------------------------------------------------------------------ init
__global__ void sepcache_init_kernel(int S, int c, int d, double theta, int32_t* meta,
                                     int32_t* slot_pos, uint8_t* slot_sep, double* freq) {
  const int tid = blockIdx.x * blockDim.x + threadIdx.x;
  const int nthr = gridDim.x * blockDim.x;
  for (int e = tid; e < S * SEPCACHE_META; e += nthr) meta[e] = 0;
  for (int e = tid; e < S * c; e += nthr) {
    slot_pos[e] = -1;
    slot_sep[e] = 0;
  }
  for (int k = tid; k < d / 2; k += nthr) freq[k] = pow(theta, -2.0 * (double)k / (double)d);
}

// ------------------------------------------------------------------ update
// One CTA per sequence. Thread 0 plans the step, all threads copy rows (16-byte vectors). With a
// Past Window (P > 0) the step that makes the usage reach c then compresses it: a block-wide
// scan numbers the past window's separators k = 0, 1, ... (oldest first); the FIFO keeps the
// last s of its current entries followed by them, so separator k lands at ring index
// (sep_head + sep_cnt + k) mod s, gets admission index admit + k, and is kept when it is among
// the last s (k >= nnew - s).
constexpr int kUpdateThreads = 128;

struct CacheDims {
  int Hkv, d, a, s, w, P, c, orig;
};

__global__ void __launch_bounds__(kUpdateThreads) sepcache_update_kernel(
    CacheDims cd, const double* __restrict__ freq, uint4* __restrict__ k_slots,
    uint4* __restrict__ v_slots, int32_t* __restrict__ slot_pos, uint8_t* __restrict__ slot_sep,
    int32_t* __restrict__ meta, const uint4* __restrict__ k_new, const uint4* __restrict__ v_new,
    const uint8_t* __restrict__ sep_new) {
  grid_dep_wait();
  grid_dep_launch_next();
  extern __shared__ int2 s_moves[];  // compression: (past slot, separator slot), min(s, P) at most
  const int Hkv = cd.Hkv, d = cd.d, a = cd.a, s = cd.s, w = cd.w, P = cd.P;
  const int seq = blockIdx.x;
  const int ns = a + s + P + w;  // slots per sequence
  const int win_base = a + s + P;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int32_t* m = meta + (size_t)seq * SEPCACHE_META;
  // slot_new, move_from, move_to, t, compress, past_cnt, sep_head, sep_cnt, move_angle, admit
  __shared__ int plan[10];
  __shared__ int s_warp[kUpdateThreads / 32];
  // the metadata and the window's oldest slot (flag, position), loaded in parallel
  __shared__ int s_meta[SEPCACHE_META];
  __shared__ int s_oldsep, s_oldpos;
  if (tid < SEPCACHE_META) s_meta[tid] = m[tid];
  if (tid == 32) {
    const int wh = m[SEPCACHE_META_WIN_HEAD];
    s_oldsep = slot_sep[(size_t)seq * ns + win_base + wh];
    s_oldpos = slot_pos[(size_t)seq * ns + win_base + wh];
  }
  // this thread's first share of the new token (K rotated at its position t, V), fetched and
  // rotated while the step is planned: it depends on t only, not on the plan
  const int vec = d / 8;   // 16-byte vectors per row
  const int hv = vec / 2;  // vectors per RoPE half
  uint4 nkx = make_uint4(0u, 0u, 0u, 0u), nky = nkx, nv = nkx;
  {
    const int t_new = m[SEPCACHE_META_T];
    if (tid < Hkv * hv) {
      const size_t src = ((size_t)seq * Hkv + tid / hv) * vec + tid % hv;
      nkx = k_new[src];
      nky = k_new[src + hv];
      rope_rotate_chunks(nkx, nky, 8 * (tid % hv), t_new, freq);
    }
    if (tid < Hkv * vec) nv = v_new[(size_t)seq * Hkv * vec + tid];
  }
  __syncthreads();
  if (tid == 0) {
    const int t = s_meta[SEPCACHE_META_T];
    int slot_new, move_from = -1, move_to = -1, move_angle = 0;
    int ninit = s_meta[SEPCACHE_META_NINIT];
    int sep_head = s_meta[SEPCACHE_META_SEP_HEAD], sep_cnt = s_meta[SEPCACHE_META_SEP_CNT];
    int win_head = s_meta[SEPCACHE_META_WIN_HEAD], win_cnt = s_meta[SEPCACHE_META_WIN_CNT];
    int past_cnt = (P > 0) ? s_meta[SEPCACHE_META_PAST_CNT] : 0;
    int admit = s_meta[SEPCACHE_META_SEP_ADMIT];
    if (t < a) {
      slot_new = t;
      ninit = t + 1;
    } else if (win_cnt < w) {
      slot_new = win_base + (win_head + win_cnt) % w;
      ++win_cnt;
    } else {
      // window full: its oldest token leaves and the new token takes its slot
      const int old_slot = win_base + win_head;
      if (P > 0) {
        move_from = old_slot;
        move_to = a + s + past_cnt;
        ++past_cnt;
      } else if (s_oldsep && s > 0) {  // the flag of old_slot = win_base + win_head
        if (sep_cnt < s) {
          move_to = a + (sep_head + sep_cnt) % s;
          ++sep_cnt;
        } else {  // separator FIFO full: the oldest separator is dropped
          move_to = a + sep_head;
          sep_head = (sep_head + 1) % s;
        }
        move_from = old_slot;
        // stored at RoPE(t_old); in the FIFO it is seen at RoPE(admission index)
        move_angle = cd.orig ? 0 : admit - s_oldpos;
        ++admit;
      }
      slot_new = old_slot;
      win_head = (win_head + 1) % w;
    }
    const bool compress = P > 0 && ninit + sep_cnt + past_cnt + win_cnt >= cd.c;
    m[SEPCACHE_META_T] = t + 1;
    m[SEPCACHE_META_NINIT] = ninit;
    m[SEPCACHE_META_SEP_HEAD] = sep_head;
    m[SEPCACHE_META_SEP_CNT] = sep_cnt;
    m[SEPCACHE_META_WIN_HEAD] = win_head;
    m[SEPCACHE_META_WIN_CNT] = win_cnt;
    if (P > 0) m[SEPCACHE_META_PAST_CNT] = past_cnt;
    m[SEPCACHE_META_SEP_ADMIT] = admit;
    plan[0] = slot_new;
    plan[1] = move_from;
    plan[2] = move_to;
    plan[3] = t;
    plan[4] = compress ? 1 : 0;
    plan[5] = past_cnt;
    plan[6] = sep_head;
    plan[7] = sep_cnt;
    plan[8] = move_angle;
    plan[9] = admit;
  }
  __syncthreads();
  const int slot_new = plan[0], move_from = plan[1], move_to = plan[2], t = plan[3];
  const size_t seq_rows = (size_t)seq * Hkv * ns;
  // move a row (all heads, all threads): V copied, K re-rotated by `angle` on the way
  auto move_row = [&](int from, int to, int angle) {
    for (int e = tid; e < Hkv * hv; e += kUpdateThreads) {
      const int hh = e / hv, q = e % hv;
      const size_t src = (seq_rows + (size_t)hh * ns + from) * vec + q;
      const size_t dst = (seq_rows + (size_t)hh * ns + to) * vec + q;
      uint4 x = k_slots[src], y = k_slots[src + hv];
      rope_rotate_chunks(x, y, 8 * q, angle, freq);
      k_slots[dst] = x;
      k_slots[dst + hv] = y;
    }
    for (int e = tid; e < Hkv * vec; e += kUpdateThreads) {
      const int hh = e / vec, q = e % vec;
      v_slots[(seq_rows + (size_t)hh * ns + to) * vec + q] =
          v_slots[(seq_rows + (size_t)hh * ns + from) * vec + q];
    }
  };
  if (move_from >= 0) {
    move_row(move_from, move_to, plan[8]);
    if (tid == 0) {
      slot_pos[(size_t)seq * ns + move_to] = slot_pos[(size_t)seq * ns + move_from];
      slot_sep[(size_t)seq * ns + move_to] = slot_sep[(size_t)seq * ns + move_from];
    }
    __syncthreads();
  }
  // the new token: K rotated at its original position t (the first share was prepared above)
  for (int e = tid; e < Hkv * hv; e += kUpdateThreads) {
    const int hh = e / hv, q = e % hv;
    const size_t dst = (seq_rows + (size_t)hh * ns + slot_new) * vec + q;
    uint4 x = nkx, y = nky;
    if (e != tid) {
      const size_t src = ((size_t)seq * Hkv + hh) * vec + q;
      x = k_new[src];
      y = k_new[src + hv];
      rope_rotate_chunks(x, y, 8 * q, t, freq);
    }
    k_slots[dst] = x;
    k_slots[dst + hv] = y;
  }
  for (int e = tid; e < Hkv * vec; e += kUpdateThreads) {
    const int hh = e / vec, q = e % vec;
    v_slots[(seq_rows + (size_t)hh * ns + slot_new) * vec + q] =
        (e == tid) ? nv : v_new[((size_t)seq * Hkv + hh) * vec + q];
  }
  if (tid == 0) {
    slot_pos[(size_t)seq * ns + slot_new] = t;
    slot_sep[(size_t)seq * ns + slot_new] = sep_new[seq] != 0;
  }
  if (!plan[4]) return;

  // ---- compression of the past window [a + s, a + s + past_cnt)
  __syncthreads();
  const int past_cnt = plan[5], sep_head = plan[6], sep_cnt = plan[7], admit = plan[9];
  const uint8_t* pflag = slot_sep + (size_t)seq * ns + a + s;
  int cnt = 0;
  for (int i = tid; i < past_cnt; i += kUpdateThreads) cnt += pflag[i] != 0;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) cnt += __shfl_down_sync(0xffffffffu, cnt, o);
  if (lane == 0) s_warp[warp] = cnt;
  __syncthreads();
  int nnew = 0;
  for (int x = 0; x < kUpdateThreads / 32; ++x) nnew += s_warp[x];
  const int kfirst = (s > 0) ? max(0, nnew - s) : nnew;  // the first new separator kept
  int carry = 0;
  for (int base = 0; base < past_cnt; base += kUpdateThreads) {
    const int i = base + tid;
    const int f = (i < past_cnt && pflag[i] != 0) ? 1 : 0;
    int incl = f;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    __syncthreads();
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    int k = carry + incl - f;
    for (int x = 0; x < warp; ++x) k += s_warp[x];
    if (f && k >= kfirst)
      s_moves[k - kfirst] = make_int2(a + s + i, a + (sep_head + sep_cnt + k) % s);
    for (int x = 0; x < kUpdateThreads / 32; ++x) carry += s_warp[x];
  }
  __syncthreads();
  const int nkept = nnew - kfirst;
  for (int j = 0; j < nkept; ++j) {
    const int2 mv = s_moves[j];
    const int tp = slot_pos[(size_t)seq * ns + mv.x];
    // admission index of new separator k = kfirst + j is admit + k
    move_row(mv.x, mv.y, cd.orig ? 0 : admit + kfirst + j - tp);
    if (tid == 0) {
      slot_pos[(size_t)seq * ns + mv.y] = tp;
      slot_sep[(size_t)seq * ns + mv.y] = 1;
    }
  }
  __syncthreads();
  for (int i = tid; i < past_cnt; i += kUpdateThreads) {  // the past window is empty again
    slot_pos[(size_t)seq * ns + a + s + i] = -1;
    slot_sep[(size_t)seq * ns + a + s + i] = 0;
  }
  if (tid == 0) {
    const int total = sep_cnt + nnew;
    if (s > 0) {
      m[SEPCACHE_META_SEP_HEAD] = (total > s) ? (sep_head + total - s) % s : sep_head;
      m[SEPCACHE_META_SEP_CNT] = min(total, s);
    }
    m[SEPCACHE_META_PAST_CNT] = 0;
    m[SEPCACHE_META_SEP_ADMIT] = admit + nnew;
  }
}

// ------------------------------------------------------------------ prefill
// State after appending the L prompt tokens of every sequence one at a time to an empty cache,
// in one pass (the rule of sepcache_update solved in closed form):
//   initial slots 0..min(a, L)-1 hold tokens 0..min(a, L)-1;
//   the window ring holds the last nwin = min(w, L - a) tokens, token u at ring index
//   (u - a) mod w, its head at (L - a) mod w once the ring has wrapped;
//   tokens u in [a, e_end) were compressed: the A-th separator among them (A = 0, 1, ...) was
//   admitted to the FIFO at ring index A mod s, so the ring keeps the last min(s, count) of
//   them, its head at (count - kept) mod s;
//   with c = 0, e_end = L - nwin (every token that left the window was compressed at once) and
//   the past window is empty; with c > 0 the past window is compressed in runs: after the
//   window is full every step moves one token into it, and a run of need = c - a - w - sep_cnt
//   tokens triggers a compression, so run boundaries follow the recurrence
//   e <- e + need(sep_cnt), sep_cnt <- min(s, sep_cnt + separators in the run), as long as a
//   run has left the window entirely; tokens [e_end, L - nwin) are the past window.
// kPrefillSplit CTAs per sequence, each for a run of slots: each finds e_end and the separator
// count (block-wide counts), scans the flags to place the kept separators, writes the slot maps
// of its slots and copies and rotates their K/V rows of every KV head (the cos/sin of a slot's
// pairs are formed once and applied to all heads); the first CTA writes the metadata. K/V rows
// of unused slots are left as they are. Keys get exactly the rotations the single-token updates
// give them: RoPE(t) on entry and, for separators with shifting, RoPE(A - t) on admission.
constexpr int kPrefillThreads = 256;
constexpr int kPrefillItems = 16;
constexpr int kPrefillSplit = 8;

__device__ __forceinline__ int block_count_flags(const uint8_t* flags, int lo, int hi,
                                                 int* s_warp) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int cnt = 0;
  for (int u = lo + tid; u < hi; u += kPrefillThreads) cnt += flags[u] != 0;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) cnt += __shfl_down_sync(0xffffffffu, cnt, o);
  __syncthreads();  // s_warp free (an earlier call may still be reading it)
  if (lane == 0) s_warp[warp] = cnt;
  __syncthreads();
  int tot = 0;
  for (int x = 0; x < kPrefillThreads / 32; ++x) tot += s_warp[x];
  return tot;
}

__global__ void __launch_bounds__(kPrefillThreads) sepcache_prefill_kernel(
    int L, CacheDims cd, const double* __restrict__ freq, const uint4* __restrict__ k_in,
    const uint4* __restrict__ v_in, const uint8_t* __restrict__ sep_in, uint4* __restrict__ k_slots,
    uint4* __restrict__ v_slots, int32_t* __restrict__ slot_pos, uint8_t* __restrict__ slot_sep,
    int32_t* __restrict__ meta) {
  extern __shared__ int s_seppos[];  // [s]: position of the separator at each ring index
  __shared__ int s_warp[kPrefillThreads / 32];
  const int Hkv = cd.Hkv, d = cd.d, a = cd.a, s = cd.s, w = cd.w, P = cd.P;
  const int seq = blockIdx.x, split = blockIdx.y;
  const int ns = a + s + P + w;
  const int slots_per = (ns + kPrefillSplit - 1) / kPrefillSplit;
  const int slot_lo = split * slots_per, slot_hi = min(ns, slot_lo + slots_per);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint8_t* flags = sep_in + (size_t)seq * L;
  const int ninit = min(a, L);
  const int nwin = max(0, min(w, L - a));
  const int win_first = L - nwin;  // oldest token in the window (>= a)

  // ---- compressed range [a, e_end) and the number of separators admitted from it
  int e_end, count;
  if (P == 0) {
    e_end = max(a, win_first);
    count = (s > 0) ? block_count_flags(flags, a, e_end, s_warp) : 0;
  } else {
    e_end = a;
    count = 0;
    int kept = 0;
    for (;;) {
      const int need = cd.c - a - w - kept;  // >= 1 since c > a + s + w
      if (nwin < w || e_end + need > win_first) break;  // the run has not left the window
      const int nsep = block_count_flags(flags, e_end, e_end + need, s_warp);
      count += nsep;
      kept = min(s, kept + nsep);
      e_end += need;
    }
  }
  const int sep_cnt = min(s, count);
  const int first_kept = count - sep_cnt;
  const int past_cnt = (P > 0) ? max(0, win_first - e_end) : 0;

  // ---- exclusive scan over [a, e_end); the kept separators record their positions by ring index
  if (sep_cnt > 0) {
    int carry = 0;
    for (int base = a; base < e_end; base += kPrefillThreads * kPrefillItems) {
      const int u0 = base + tid * kPrefillItems;
      uint32_t bits = 0;
#pragma unroll
      for (int q = 0; q < kPrefillItems; ++q)
        if (u0 + q < e_end && flags[u0 + q] != 0) bits |= 1u << q;
      const int n = __popc(bits);
      int incl = n;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      __syncthreads();
      if (lane == 31) s_warp[warp] = incl;
      __syncthreads();
      int before = carry;
      for (int x = 0; x < warp; ++x) before += s_warp[x];
      int k = before + incl - n;  // index of this thread's first separator
#pragma unroll
      for (int q = 0; q < kPrefillItems; ++q) {
        if (bits & (1u << q)) {
          if (k >= first_kept) s_seppos[k % s] = u0 + q;
          ++k;
        }
      }
      int blk = 0;
      for (int x = 0; x < kPrefillThreads / 32; ++x) blk += s_warp[x];
      carry += blk;
    }
  }
  __syncthreads();

  // slot -> original position (-1: unused); for separator slots also the admission index
  auto pos_of = [&](int slot, int* admit_idx) -> int {
    if (slot < a) return slot < ninit ? slot : -1;
    if (slot < a + s) {
      const int r = slot - a;
      if (!(count >= s || r < count)) return -1;
      // kept admission indices are first_kept..count-1, one per residue mod s
      *admit_idx = first_kept + (((r - first_kept) % s) + s) % s;
      return s_seppos[r];
    }
    if (slot < a + s + P) {
      const int r = slot - a - s;
      return r < past_cnt ? e_end + r : -1;
    }
    const int r = slot - a - s - P;
    if (nwin == w || r < nwin) {
      const int r0 = (win_first - a) % w;
      return win_first + (r - r0 + w) % w;
    }
    return -1;
  };

  // ---- slot maps of this CTA's slots, metadata once per sequence
  for (int slot = slot_lo + tid; slot < slot_hi; slot += kPrefillThreads) {
    int A = 0;
    const int pos = pos_of(slot, &A);
    slot_pos[(size_t)seq * ns + slot] = pos;
    slot_sep[(size_t)seq * ns + slot] = (pos >= 0 && flags[pos] != 0) ? 1 : 0;
  }
  if (split == 0) {
    if (tid == 0) {
      int32_t* m = meta + (size_t)seq * SEPCACHE_META;
      m[SEPCACHE_META_T] = L;
      m[SEPCACHE_META_NINIT] = ninit;
      m[SEPCACHE_META_SEP_HEAD] = (s > 0) ? first_kept % s : 0;
      m[SEPCACHE_META_SEP_CNT] = sep_cnt;
      m[SEPCACHE_META_WIN_HEAD] = (L - a >= w) ? (L - a) % w : 0;
      m[SEPCACHE_META_WIN_CNT] = nwin;
      m[SEPCACHE_META_PAST_CNT] = past_cnt;
      m[SEPCACHE_META_SEP_ADMIT] = count;
    }
  }
  // ---- K/V rows of this CTA's occupied slots, every head (one warp per slot): lane l rotates
  // pair chunk l % hv of heads l / hv, l / hv + 32 / hv, ... with the chunk's cos/sin formed once
  const int vec = d / 8;
  const int hv = vec / 2;         // pair chunks per row (8 at d = 128, 4 at d = 64)
  const int hstep = 32 / hv;      // heads one warp pass covers
  const int e = lane % hv;
  for (int slot = slot_lo + warp; slot < slot_hi; slot += kPrefillThreads / 32) {
    int A = 0;
    const int pos = pos_of(slot, &A);
    if (pos < 0) continue;
    const bool rerotate = slot >= a && slot < a + s && !cd.orig;
    const ChunkCS cs1 = rope_chunk_cs(8 * e, pos, freq);
    ChunkCS cs2 = cs1;
    if (rerotate) cs2 = rope_chunk_cs(8 * e, (long long)A - pos, freq);
    for (int head = lane / hv; head < Hkv; head += hstep) {
      const size_t src = (((size_t)seq * L + pos) * Hkv + head) * vec;
      const size_t dst = (((size_t)seq * Hkv + head) * ns + slot) * vec;
      uint4 x = __ldg(k_in + src + e), y = __ldg(k_in + src + e + hv);
      if (pos != 0) rope_apply_chunks(x, y, cs1);
      if (rerotate && A != pos) rope_apply_chunks(x, y, cs2);
      k_slots[dst + e] = x;
      k_slots[dst + e + hv] = y;
    }
    for (int c = lane; c < Hkv * vec; c += 32) {
      const int head = c / vec, q = c % vec;
      v_slots[(((size_t)seq * Hkv + head) * ns + slot) * vec + q] =
          __ldg(v_in + (((size_t)seq * L + pos) * Hkv + head) * vec + q);
    }
  }
}

// ------------------------------------------------------------------ decode
// Lane groups: LPK = D / 8 lanes per key row, 8 contiguous elements per lane; NG = 128 / LPK
// groups per CTA, each taking kDecRows rows of every KC = kDecRows NG row chunk (four
// independent rows per group and stage give each warp enough work between ring waits), in a
// ring of three chunks.
constexpr int kDecThreads = 128;
constexpr int kDecStages = 3;
constexpr int kDecRows = 4;
constexpr int kDecWarps = kDecThreads / 32;

template <int N>
__host__ __device__ constexpr int ilog2() {
  return N >= 32 ? 5 : N >= 16 ? 4 : N >= 8 ? 3 : N >= 4 ? 2 : N >= 2 ? 1 : 0;
}

// Reduction over the LPK lanes of a group of GP per-query partial sums: the first log2(GP)
// butterfly levels halve what a lane holds (it keeps one half, adding its partner's copy of it,
// and sends the other half); the remaining levels sum one value. Afterwards lane l of the group
// holds the full score of query own_query(l).
template <int GP, int LPK>
__device__ __forceinline__ float group_reduce_own(float (&v)[GP], int l) {
  constexpr int LG = ilog2<GP>(), LL = ilog2<LPK>();
  static_assert((1 << LG) == GP && (1 << LL) == LPK && GP <= LPK, "group shape");
#pragma unroll
  for (int lv = 0; lv < LG; ++lv) {
    const int off = LPK >> (lv + 1), h = (GP >> lv) >> 1;
    const bool upper = (l & off) != 0;
#pragma unroll
    for (int i = 0; i < h; ++i) {
      const float send = upper ? v[i] : v[i + h];
      const float keep = upper ? v[i + h] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
    }
  }
  float r = v[0];
#pragma unroll
  for (int lv = LG; lv < LL; ++lv) r += __shfl_xor_sync(0xffffffffu, r, LPK >> (lv + 1));
  return r;
}
template <int GP, int LPK>
__device__ __forceinline__ int own_query(int l) {
  int g = 0;
#pragma unroll
  for (int lv = 0; lv < ilog2<GP>(); ++lv)
    if (l & (LPK >> (lv + 1))) g += GP >> (lv + 1);
  return g;
}
template <int GP, int LPK>
__device__ __forceinline__ int lane_of_query(int g) {
  int src = 0;
#pragma unroll
  for (int lv = 0; lv < ilog2<GP>(); ++lv)
    if (g & (GP >> (lv + 1))) src |= LPK >> (lv + 1);
  return src;
}

__device__ __forceinline__ float2 bf16x2_to_float2(uint32_t u) {
  return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
}

template <int D, int GP>
struct DecCfg {
  static constexpr int LPK = D / 8;
  static constexpr int NG = kDecThreads / LPK;
  static constexpr int KC = kDecRows * NG;  // rows per ring stage
  static constexpr int RING_BYTES = kDecStages * KC * D * 2 * 2;
  static constexpr int COMB_BYTES = kDecWarps * GP * D * 4;  // per-warp V sums at the end
  static constexpr int BUF_BYTES = RING_BYTES > COMB_BYTES ? RING_BYTES : COMB_BYTES;
};

template <int D, int GP>
struct DecSmem {
  alignas(128) uint8_t buf[DecCfg<D, GP>::BUF_BYTES];  // K/V ring, later the combine buffer
  alignas(16) float qrot[3][GP][D];  // the queries rotated for each block, x scale*log2(e)
  uint64_t full[kDecStages];
  int done[kDecStages];  // warps finished with the stage's current chunk
  int issued;            // chunks whose copies were issued (0..issued-1)
  float wm[kDecWarps][GP], wl[kDecWarps][GP];
  int abort_flag;
};

// Block of logical rank r: 0 initial, 1 separator FIFO, 2 past window and window.
__device__ __forceinline__ int rank_block(int r, int ninit, int sep_cnt) {
  return (r < ninit) ? 0 : (r < ninit + sep_cnt) ? 1 : 2;
}

struct DecodeArgs {
  int Hq, Hkv, G, a, s, P, w;
  const __nv_bfloat16* k_slots;
  const __nv_bfloat16* v_slots;
  const int32_t* meta;
  const double* freq;
  const __nv_bfloat16* q;
  __nv_bfloat16* o;
  float* lse;
  float scale_log2;
  unsigned* err;
};

template <int D, int GP, bool ORIG>
__global__ void __launch_bounds__(kDecThreads, (GP >= 8) ? 2 : 4)
    sepcache_decode_kernel(const __grid_constant__ DecodeArgs p) {
  using C = DecCfg<D, GP>;
  constexpr int LPK = C::LPK, NG = C::NG, KC = C::KC;
  constexpr int HALF = D / 2;
  grid_dep_wait();
  const int kvh = blockIdx.x, seq = blockIdx.y;
  const int ns = p.a + p.s + p.P + p.w;
  const int tid = threadIdx.x, warp = tid >> 5, grp = tid / LPK, l = tid % LPK;
  extern __shared__ __align__(128) uint8_t dsm_raw[];
  DecSmem<D, GP>& sm = *reinterpret_cast<DecSmem<D, GP>*>(dsm_raw);
  __nv_bfloat16* ring = reinterpret_cast<__nv_bfloat16*>(sm.buf);
  auto ring_k = [&](int st, int row) { return ring + ((size_t)(st * 2 + 0) * KC + row) * D; };
  auto ring_v = [&](int st, int row) { return ring + ((size_t)(st * 2 + 1) * KC + row) * D; };

  const int32_t* m = p.meta + (size_t)seq * SEPCACHE_META;
  const int T = m[SEPCACHE_META_T];
  const int ninit = m[SEPCACHE_META_NINIT];
  const int sep_head = m[SEPCACHE_META_SEP_HEAD], sep_cnt = m[SEPCACHE_META_SEP_CNT];
  const int win_head = m[SEPCACHE_META_WIN_HEAD], win_cnt = m[SEPCACHE_META_WIN_CNT];
  const int past_cnt = (p.P > 0) ? m[SEPCACHE_META_PAST_CNT] : 0;
  const int admit = m[SEPCACHE_META_SEP_ADMIT];
  const int occ = ninit + sep_cnt + past_cnt + win_cnt;
  const int mq = occ - 1;  // the query's own rank
  const int nchunks = (occ + KC - 1) / KC;
  const size_t row_base = ((size_t)seq * p.Hkv + kvh) * ns;
  volatile int* abort_flag = &sm.abort_flag;

  auto issue_chunk = [&](int ch) {  // one thread: bulk copies of chunk ch into its stage
    const int st = ch % kDecStages;
    const int c0 = ch * KC;
    const int rows = min(KC, occ - c0);
    mbar_arrive_expect_tx(&sm.full[st], (uint32_t)(rows * D * 2 * 2));
    // ranks map to slots piecewise contiguously: initial block, the separator ring, the past
    // window, the window ring; a run ends at a block boundary or a ring wrap
    int r = c0;
    const int end = c0 + rows;
    while (r < end) {
      int slot, len;
      if (r < ninit) {
        slot = r;
        len = min(end, ninit) - r;
      } else if (r < ninit + sep_cnt) {
        const int x = (sep_head + (r - ninit)) % p.s;
        slot = p.a + x;
        len = min(min(end, ninit + sep_cnt) - r, p.s - x);
      } else if (r < ninit + sep_cnt + past_cnt) {
        slot = p.a + p.s + (r - ninit - sep_cnt);
        len = min(end, ninit + sep_cnt + past_cnt) - r;
      } else {
        const int x = (win_head + (r - ninit - sep_cnt - past_cnt)) % p.w;
        slot = p.a + p.s + p.P + x;
        len = min(end - r, p.w - x);
      }
      const size_t src = (row_base + slot) * D;
      bulk_load(ring_k(st, r - c0), p.k_slots + src, (uint32_t)(len * D * 2), &sm.full[st]);
      bulk_load(ring_v(st, r - c0), p.v_slots + src, (uint32_t)(len * D * 2), &sm.full[st]);
      r += len;
    }
    atomicMax(&sm.issued, ch + 1);  // warps may refill different stages at the same time
  };
  if (tid == 0) {
    for (int st = 0; st < kDecStages; ++st) {
      mbar_init(&sm.full[st], 1);
      sm.done[st] = 0;
    }
    sm.abort_flag = 0;
    sm.issued = 0;
    fence_barrier_init();
    for (int ch = 0; ch < min(kDecStages, nchunks); ++ch) issue_chunk(ch);
  }

  // ---- the G queries of this KV head rotated once per block (while the first chunks load):
  // block 0 = initial keys (stored at RoPE(rank)), 1 = separators (stored at RoPE(admission
  // index), rank = ninit + index - oldest index), 2 = past window and window (stored at
  // RoPE(original position), query at T - 1). Without shifting every block uses T - 1.
  {
    long long qpos[3];
    qpos[0] = ORIG ? (long long)T - 1 : (long long)mq;
    qpos[1] = ORIG ? (long long)T - 1 : (long long)mq - ninit + (admit - sep_cnt);
    qpos[2] = (long long)T - 1;
    for (int e = tid; e < 3 * HALF; e += kDecThreads) {
      const int blk = e / HALF, k = e % HALF;
      float sn, cs;
      rope_cos_sin(qpos[blk], __ldg(p.freq + k), &cs, &sn);
#pragma unroll
      for (int g = 0; g < GP; ++g) {
        float r1 = 0.f, r2 = 0.f;
        if (g < p.G) {
          const __nv_bfloat16* qh = p.q + ((size_t)seq * p.Hq + kvh * p.G + g) * D;
          const float x1 = __bfloat162float(qh[k]);
          const float x2 = __bfloat162float(qh[k + HALF]);
          r1 = (x1 * cs - x2 * sn) * p.scale_log2;
          r2 = (x2 * cs + x1 * sn) * p.scale_log2;
        }
        sm.qrot[blk][g][k] = r1;
        sm.qrot[blk][g][k + HALF] = r2;
      }
    }
  }
  __syncthreads();

  // ---- consumers: group grp takes rows grp, grp + NG, ... of every chunk
  float2 qr[GP][4];   // this lane's 8 query elements (as pairs) of the current block
  float2 acc[GP][4];  // V sums of every query over this lane's 8 elements
  float m_own = -INFINITY, l_own = 0.f;  // softmax state of this lane's own query
  int cur_blk = -1;
#pragma unroll
  for (int g = 0; g < GP; ++g)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[g][i] = make_float2(0.f, 0.f);

  // this lane's 8 query elements of every query, rotated for block blk
  auto load_q = [&](int blk) {
    cur_blk = blk;
#pragma unroll
    for (int g = 0; g < GP; ++g) {
      const float4 a0 = *reinterpret_cast<const float4*>(&sm.qrot[blk][g][l * 8]);
      const float4 a1 = *reinterpret_cast<const float4*>(&sm.qrot[blk][g][l * 8 + 4]);
      qr[g][0] = make_float2(a0.x, a0.y);
      qr[g][1] = make_float2(a0.z, a0.w);
      qr[g][2] = make_float2(a1.x, a1.y);
      qr[g][3] = make_float2(a1.z, a1.w);
    }
  };

  bool ok = true;
  for (int ch = 0; ch < nchunks && ok; ++ch) {
    const int st = ch % kDecStages;
    if (!__all_sync(0xffffffffu, mbar_wait(&sm.full[st], (ch / kDecStages) & 1, p.err, abort_flag))) {
      ok = false;
      break;
    }
    const int c0 = ch * KC;
    // one key row of the group: scores against the block's rotated queries, online softmax of
    // this lane's query, V sums of every query; CHECKED rows test their rank (block boundary,
    // rows past the occupancy). A chunk that lies in one block entirely takes the path below
    // without them, where the group's rows are scored independently and enter the online
    // softmax together (one maximum and one rescale test per kDecRows rows).
    auto process_row = [&](auto checked, int sub) {
      constexpr bool CHECKED = decltype(checked)::value;
      const int row = sub * NG + grp;
      const int r = c0 + row;
      const bool valid = !CHECKED || r < occ;
      if (CHECKED) {
        const int blk = rank_block(r, ninit, sep_cnt);
        if (blk != cur_blk) load_q(blk);
      }
      uint4 kk = make_uint4(0u, 0u, 0u, 0u), vv = make_uint4(0u, 0u, 0u, 0u);
      if (valid) {
        kk = *reinterpret_cast<const uint4*>(ring_k(st, row) + l * 8);
        vv = *reinterpret_cast<const uint4*>(ring_v(st, row) + l * 8);
      }
      const float2 k2[4] = {bf16x2_to_float2(kk.x), bf16x2_to_float2(kk.y),
                            bf16x2_to_float2(kk.z), bf16x2_to_float2(kk.w)};
      float part[GP];
#pragma unroll
      for (int g = 0; g < GP; ++g) {
        float2 s2 = f2_mul(qr[g][0], k2[0]);
        s2 = f2_fma(qr[g][1], k2[1], s2);
        s2 = f2_fma(qr[g][2], k2[2], s2);
        s2 = f2_fma(qr[g][3], k2[3], s2);
        part[g] = s2.x + s2.y;
      }
      const float sc = group_reduce_own<GP, LPK>(part, l);
      // online softmax of this lane's query, lazy rescale (only when the max grows by > 2^8)
      const bool need = valid && sc > m_own + 8.0f;
      if (__any_sync(0xffffffffu, need)) {
        const float alpha = need ? ex2(m_own - sc) : 1.0f;
        if (need) {
          l_own *= alpha;
          m_own = sc;
        }
#pragma unroll
        for (int g = 0; g < GP; ++g) {
          const float ag = __shfl_sync(0xffffffffu, alpha, lane_of_query<GP, LPK>(g), LPK);
          const float2 ag2 = make_float2(ag, ag);
#pragma unroll
          for (int i = 0; i < 4; ++i) acc[g][i] = f2_mul(acc[g][i], ag2);
        }
      }
      const float p_own = valid ? ex2(sc - m_own) : 0.f;
      l_own += p_own;
      const float2 v2[4] = {bf16x2_to_float2(vv.x), bf16x2_to_float2(vv.y),
                            bf16x2_to_float2(vv.z), bf16x2_to_float2(vv.w)};
#pragma unroll
      for (int g = 0; g < GP; ++g) {
        const float pg = __shfl_sync(0xffffffffu, p_own, lane_of_query<GP, LPK>(g), LPK);
        const float2 pg2 = make_float2(pg, pg);
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[g][i] = f2_fma(pg2, v2[i], acc[g][i]);
      }
    };
    const int blk0 = rank_block(c0, ninit, sep_cnt);
    if (c0 + KC <= occ && blk0 == rank_block(c0 + KC - 1, ninit, sep_cnt)) {
      if (blk0 != cur_blk) load_q(blk0);
      // the group's rows scored independently, entering the online softmax together
      float sc[kDecRows];
      uint4 vv[kDecRows];
#pragma unroll
      for (int sub = 0; sub < kDecRows; ++sub) {
        const int row = sub * NG + grp;
        const uint4 kk = *reinterpret_cast<const uint4*>(ring_k(st, row) + l * 8);
        vv[sub] = *reinterpret_cast<const uint4*>(ring_v(st, row) + l * 8);
        const float2 k2[4] = {bf16x2_to_float2(kk.x), bf16x2_to_float2(kk.y),
                              bf16x2_to_float2(kk.z), bf16x2_to_float2(kk.w)};
        float part[GP];
#pragma unroll
        for (int g = 0; g < GP; ++g) {
          float2 s2 = f2_mul(qr[g][0], k2[0]);
          s2 = f2_fma(qr[g][1], k2[1], s2);
          s2 = f2_fma(qr[g][2], k2[2], s2);
          s2 = f2_fma(qr[g][3], k2[3], s2);
          part[g] = s2.x + s2.y;
        }
        sc[sub] = group_reduce_own<GP, LPK>(part, l);
      }
      float mx = sc[0];
#pragma unroll
      for (int sub = 1; sub < kDecRows; ++sub) mx = fmaxf(mx, sc[sub]);
      const bool need = mx > m_own + 8.0f;
      if (__any_sync(0xffffffffu, need)) {
        const float alpha = need ? ex2(m_own - mx) : 1.0f;
        if (need) {
          l_own *= alpha;
          m_own = mx;
        }
#pragma unroll
        for (int g = 0; g < GP; ++g) {
          const float ag = __shfl_sync(0xffffffffu, alpha, lane_of_query<GP, LPK>(g), LPK);
          const float2 ag2 = make_float2(ag, ag);
#pragma unroll
          for (int i = 0; i < 4; ++i) acc[g][i] = f2_mul(acc[g][i], ag2);
        }
      }
#pragma unroll
      for (int sub = 0; sub < kDecRows; ++sub) {
        const float p_own = ex2(sc[sub] - m_own);
        l_own += p_own;
        const float2 v2[4] = {bf16x2_to_float2(vv[sub].x), bf16x2_to_float2(vv[sub].y),
                              bf16x2_to_float2(vv[sub].z), bf16x2_to_float2(vv[sub].w)};
#pragma unroll
        for (int g = 0; g < GP; ++g) {
          const float pg = __shfl_sync(0xffffffffu, p_own, lane_of_query<GP, LPK>(g), LPK);
          const float2 pg2 = make_float2(pg, pg);
#pragma unroll
          for (int i = 0; i < 4; ++i) acc[g][i] = f2_fma(pg2, v2[i], acc[g][i]);
        }
      }
    } else {
#pragma unroll
      for (int sub = 0; sub < kDecRows; ++sub) process_row(std::true_type(), sub);
    }
    // the last warp done with this stage refills it (its reads all precede the atomic)
    __syncwarp();
    if ((tid & 31) == 0) {
      __threadfence_block();
      if (atomicAdd(&sm.done[st], 1) == kDecWarps - 1) {
        sm.done[st] = 0;
        if (ch + kDecStages < nchunks) {
          fence_proxy_async_smem();
          issue_chunk(ch + kDecStages);
        }
      }
    }
  }
  if (__syncthreads_or(!ok)) {
    // a wait ran out: let the copies of the last issued chunks land before the CTA leaves
    // (no chunk is issued any more: every warp has left the loop)
    if (tid == 0) {
      const int n_is = *reinterpret_cast<volatile int*>(&sm.issued);
      for (int ch = max(0, n_is - kDecStages); ch < n_is; ++ch)
        mbar_wait(&sm.full[ch % kDecStages], (ch / kDecStages) & 1, nullptr, nullptr);
    }
  }
  grid_dep_launch_next();  // the cache is read: the next kernel of the stream may start

  // ---- every query's softmax state from the lanes that own it
  float mrun[GP], lrun[GP];
#pragma unroll
  for (int g = 0; g < GP; ++g) {
    mrun[g] = __shfl_sync(0xffffffffu, m_own, lane_of_query<GP, LPK>(g), LPK);
    lrun[g] = __shfl_sync(0xffffffffu, l_own, lane_of_query<GP, LPK>(g), LPK);
  }
  // ---- combine the groups of each warp (lanes l and l ^ LPK, l ^ 2 LPK, ... hold the same
  // elements)
#pragma unroll
  for (int off = LPK; off < 32; off <<= 1) {
#pragma unroll
    for (int g = 0; g < GP; ++g) {
      const float mo = __shfl_xor_sync(0xffffffffu, mrun[g], off);
      const float lo = __shfl_xor_sync(0xffffffffu, lrun[g], off);
      const float M = fmaxf(mrun[g], mo);
      const float Mu = (M == -INFINITY) ? 0.f : M;
      const float fs = ex2(mrun[g] - Mu), fo = ex2(mo - Mu);
      const float2 fs2 = make_float2(fs, fs), fo2 = make_float2(fo, fo);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float2 ao;
        ao.x = __shfl_xor_sync(0xffffffffu, acc[g][i].x, off);
        ao.y = __shfl_xor_sync(0xffffffffu, acc[g][i].y, off);
        acc[g][i] = f2_fma(acc[g][i], fs2, f2_mul(ao, fo2));
      }
      lrun[g] = lrun[g] * fs + lo * fo;
      mrun[g] = M;
    }
  }
  // ---- combine the warps of this CTA through shared memory (the ring is no longer used)
  __syncthreads();
  float* s_acc = reinterpret_cast<float*>(sm.buf);  // [kDecWarps][GP][D]
  if ((tid & 31) < LPK) {
    if (l == 0) {
#pragma unroll
      for (int g = 0; g < GP; ++g) {
        sm.wm[warp][g] = mrun[g];
        sm.wl[warp][g] = lrun[g];
      }
    }
#pragma unroll
    for (int g = 0; g < GP; ++g) {
      float4* dst = reinterpret_cast<float4*>(s_acc + ((size_t)warp * GP + g) * D + l * 8);
      dst[0] = make_float4(acc[g][0].x, acc[g][0].y, acc[g][1].x, acc[g][1].y);
      dst[1] = make_float4(acc[g][2].x, acc[g][2].y, acc[g][3].x, acc[g][3].y);
    }
  }
  __syncthreads();
  for (int e = tid; e < p.G * D; e += kDecThreads) {
    const int g = e / D, col = e % D;
    float M = -INFINITY;
    for (int x = 0; x < kDecWarps; ++x) M = fmaxf(M, sm.wm[x][g]);
    const float Mu = (M == -INFINITY) ? 0.f : M;
    float sum = 0.f, lsum = 0.f;
    for (int x = 0; x < kDecWarps; ++x) {
      const float f = ex2(sm.wm[x][g] - Mu);
      sum += s_acc[((size_t)x * GP + g) * D + col] * f;
      lsum += sm.wl[x][g] * f;
    }
    const int hq = kvh * p.G + g;
    p.o[((size_t)seq * p.Hq + hq) * D + col] = __float2bfloat16(lsum > 0.f ? sum / lsum : 0.f);
    if (col == 0 && p.lse)
      p.lse[(size_t)seq * p.Hq + hq] =
          lsum > 0.f ? (M + __log2f(lsum)) * 0.69314718055994531f : -INFINITY;
  }
}

// ------------------------------------------------------------------ export order
// Slot holding logical rank r (r < occupied).
__device__ __forceinline__ int rank_to_slot(int r, int ninit, int sep_head, int sep_cnt,
                                            int past_cnt, int win_head, int a, int s, int P,
                                            int w) {
  if (r < ninit) return r;
  r -= ninit;
  if (r < sep_cnt) return a + (sep_head + r) % s;
  r -= sep_cnt;
  if (r < past_cnt) return a + s + r;
  r -= past_cnt;
  return a + s + P + (win_head + r) % w;
}

__global__ void sepcache_export_kernel(int a, int s, int P, int w,
                                       const int32_t* __restrict__ meta,
                                       const int32_t* __restrict__ slot_pos,
                                       int32_t* __restrict__ pos_out, int32_t* __restrict__ count) {
  const int seq = blockIdx.x;
  const int c = a + s + P + w;
  const int32_t* m = meta + (size_t)seq * SEPCACHE_META;
  const int ninit = m[SEPCACHE_META_NINIT];
  const int sep_head = m[SEPCACHE_META_SEP_HEAD], sep_cnt = m[SEPCACHE_META_SEP_CNT];
  const int win_head = m[SEPCACHE_META_WIN_HEAD], win_cnt = m[SEPCACHE_META_WIN_CNT];
  const int past_cnt = (P > 0) ? m[SEPCACHE_META_PAST_CNT] : 0;
  const int occ = ninit + sep_cnt + past_cnt + win_cnt;
  for (int r = threadIdx.x; r < c; r += blockDim.x) {
    pos_out[(size_t)seq * c + r] =
        r < occ ? slot_pos[(size_t)seq * c + rank_to_slot(r, ninit, sep_head, sep_cnt, past_cnt,
                                                          win_head, a, s, P, w)]
                : -1;
  }
  if (threadIdx.x == 0) count[seq] = occ;
}

// ------------------------------------------------------------------ launchers
// Past Window slots and slots per sequence of a cache state.
static int past_slots(const SepCacheState& st) { return st.c > 0 ? st.c - st.a - st.w : 0; }
static int cache_slots(const SepCacheState& st) { return st.a + st.s + past_slots(st) + st.w; }
static CacheDims cache_dims(const SepCacheState& st) {
  return CacheDims{st.Hkv, st.d, st.a, st.s, st.w, past_slots(st), st.c, st.original_positions};
}

cudaError_t launch_sepcache_init(const SepCacheState& st, cudaStream_t stream) {
  const int c = cache_slots(st);
  sepcache_init_kernel<<<64, 256, 0, stream>>>(st.S, c, st.d, (double)st.rope_theta, st.meta,
                                               st.slot_pos, st.slot_sep, st.rope_freq);
  return cudaGetLastError();
}

cudaError_t launch_sepcache_update(const SepCacheState& st, const void* k_new, const void* v_new,
                                   const uint8_t* sep_new, cudaStream_t stream) {
  const int P = past_slots(st);
  const size_t smem = (size_t)max(1, min(st.s, P)) * sizeof(int2);  // compression moves
  return launch_chained(sepcache_update_kernel, dim3(st.S), dim3(kUpdateThreads), smem, stream,
                        cache_dims(st), st.rope_freq, reinterpret_cast<uint4*>(st.k_slots),
                        reinterpret_cast<uint4*>(st.v_slots), st.slot_pos, st.slot_sep, st.meta,
                        static_cast<const uint4*>(k_new), static_cast<const uint4*>(v_new),
                        sep_new);
}

cudaError_t launch_sepcache_prefill(const SepCacheState& st, const void* k, const void* v,
                                    const uint8_t* sep, int L, cudaStream_t stream) {
  const size_t smem = (size_t)max(st.s, 1) * sizeof(int);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(sepcache_prefill_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  sepcache_prefill_kernel<<<dim3(st.S, kPrefillSplit), kPrefillThreads, smem, stream>>>(
      L, cache_dims(st), st.rope_freq, static_cast<const uint4*>(k),
      static_cast<const uint4*>(v), sep, reinterpret_cast<uint4*>(st.k_slots),
      reinterpret_cast<uint4*>(st.v_slots), st.slot_pos, st.slot_sep, st.meta);
  return cudaGetLastError();
}

template <int D, int GP, bool ORIG>
static cudaError_t launch_decode_t(const SepCacheState& st, const void* q, void* o, float* lse,
                                   float scale, cudaStream_t stream) {
  constexpr size_t smem = sizeof(DecSmem<D, GP>);
  static bool attr_set[64] = {false};  // per device: set once, outside any stream capture
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    e = cudaFuncSetAttribute(sepcache_decode_kernel<D, GP, ORIG>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  DecodeArgs a;
  a.Hq = st.Hq;
  a.Hkv = st.Hkv;
  a.G = st.Hq / st.Hkv;
  a.a = st.a;
  a.s = st.s;
  a.P = past_slots(st);
  a.w = st.w;
  a.k_slots = reinterpret_cast<const __nv_bfloat16*>(st.k_slots);
  a.v_slots = reinterpret_cast<const __nv_bfloat16*>(st.v_slots);
  a.meta = st.meta;
  a.freq = st.rope_freq;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.o = static_cast<__nv_bfloat16*>(o);
  a.lse = lse;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.err = device_error_word();
  dim3 grid(st.Hkv, st.S);
  return launch_chained(sepcache_decode_kernel<D, GP, ORIG>, grid, dim3(kDecThreads), smem, stream,
                        a);
}

template <int D, int GP>
static cudaError_t launch_decode_d(const SepCacheState& st, const void* q, void* o, float* lse,
                                   float scale, cudaStream_t stream) {
  return st.original_positions ? launch_decode_t<D, GP, true>(st, q, o, lse, scale, stream)
                               : launch_decode_t<D, GP, false>(st, q, o, lse, scale, stream);
}

cudaError_t launch_sepcache_decode(const SepCacheState& st, const void* q, void* o, float* lse,
                                   float scale, cudaStream_t stream) {
  const int G = st.Hq / st.Hkv;  // padded to the next power of two (zero queries)
  const int GP = G <= 1 ? 1 : G <= 2 ? 2 : G <= 4 ? 4 : 8;
  if (G < 1 || G > 8) return cudaErrorInvalidValue;
  if (st.d == 128) {
    switch (GP) {
      case 1: return launch_decode_d<128, 1>(st, q, o, lse, scale, stream);
      case 2: return launch_decode_d<128, 2>(st, q, o, lse, scale, stream);
      case 4: return launch_decode_d<128, 4>(st, q, o, lse, scale, stream);
      default: return launch_decode_d<128, 8>(st, q, o, lse, scale, stream);
    }
  }
  if (st.d == 64) {
    switch (GP) {
      case 1: return launch_decode_d<64, 1>(st, q, o, lse, scale, stream);
      case 2: return launch_decode_d<64, 2>(st, q, o, lse, scale, stream);
      case 4: return launch_decode_d<64, 4>(st, q, o, lse, scale, stream);
      default: return launch_decode_d<64, 8>(st, q, o, lse, scale, stream);
    }
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_sepcache_export(const SepCacheState& st, int32_t* pos_out, int32_t* count,
                                   cudaStream_t stream) {
  sepcache_export_kernel<<<st.S, 256, 0, stream>>>(st.a, st.s, past_slots(st), st.w, st.meta,
                                                   st.slot_pos, pos_out, count);
  return cudaGetLastError();
}

}  // namespace sep
