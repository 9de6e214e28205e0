// SepCache streaming decode on sm_100a: cache update (append / compress) and single-query
// attention with positional-encoding shifting.
//
// Cache blocks ("How SepLLM reorchestrates the language model...", beiduofen.top, section
// "SepLLM's Architecture: Composing Efficiency"): a initial slots, a separator FIFO of s slots,
// a local-window FIFO of w slots and, with a usage threshold c > 0, a Past Window of
// P = c - a - w slots. When the window overflows, its oldest token leaves: with c = 0 it moves
// to the separator FIFO if it is a separator and is dropped otherwise; with c > 0 it goes to
// the Past Window, which is compressed (its separators to the FIFO, the rest dropped) by the
// step that makes the total usage reach c. The separator FIFO drops its oldest entries when
// full. Positions are ranks inside the cache (SepLLM project card, "Limitations & Caveats":
// streaming needs positional-encoding shifting), so a key is rotated by RoPE(rank) at every
// step and the query by RoPE(occupied - 1).
//
// Slot storage per (sequence, KV head) is [n][d], n = a + s + P + w: initial slots, the
// separator ring, the past window (a plain array, emptied by each compression), the window
// ring. Keys are stored without rotation.
//
// Decode: one CTA per (sequence, KV head), all of them resident at once (4 per SM), so the
// whole cache streams in a single wave. Each CTA streams its ranks through a shared-memory ring
// filled by bulk copies, with 8 half-warps (one key per half-warp per step, the row spread over
// 16 lanes), rotates keys in registers (cos/sin advanced by a complex recurrence from the table
// row of the first rank), keeps an online softmax per query head, and combines its half-warps
// through shared memory. No global scratch is used.
#include <cuda_runtime.h>

#include "sep_common.cuh"
#include "sep_launch.h"

namespace sep {

constexpr int kDecThreads = 128;   // 8 half-warps per CTA; one CTA per (sequence, KV head)
constexpr int kHalfWarps = kDecThreads / 16;

// ------------------------------------------------------------------ init
__global__ void sepcache_init_kernel(int S, int c, int d, double theta, int32_t* meta,
                                     int32_t* slot_pos, uint8_t* slot_sep, float* rope_cs) {
  const int tid = blockIdx.x * blockDim.x + threadIdx.x;
  const int nthr = gridDim.x * blockDim.x;
  for (int e = tid; e < S * SEPCACHE_META; e += nthr) meta[e] = 0;
  for (int e = tid; e < S * c; e += nthr) {
    slot_pos[e] = -1;
    slot_sep[e] = 0;
  }
  const int h = d / 2;
  for (int e = tid; e < c * h; e += nthr) {
    const int p = e / h, k = e % h;
    const double ang = (double)p * pow(theta, -2.0 * (double)k / (double)d);
    double sn, cs;
    sincos(ang, &sn, &cs);
    rope_cs[2 * e] = (float)cs;
    rope_cs[2 * e + 1] = (float)sn;
  }
}

// Key rotation for a cache without positional shifting: the 16-byte chunks x (dims k0..k0+7)
// and y (dims k0+d/2..k0+d/2+7) of one key row rotated at original position pos, the angle of
// pair k being pos * theta^(-2k/d) as in the cos/sin table; fp64 arithmetic, rounded to bf16.
__device__ __forceinline__ void rope_rotate_chunks(uint4& x, uint4& y, int k0, int pos, int d,
                                                   double theta) {
  uint32_t xs[4] = {x.x, x.y, x.z, x.w}, ys[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const __nv_bfloat162 xa = *reinterpret_cast<const __nv_bfloat162*>(&xs[q]);
    const __nv_bfloat162 ya = *reinterpret_cast<const __nv_bfloat162*>(&ys[q]);
    double xv[2] = {(double)__low2float(xa), (double)__high2float(xa)};
    double yv[2] = {(double)__low2float(ya), (double)__high2float(ya)};
    __nv_bfloat16 xo[2], yo[2];
#pragma unroll
    for (int z = 0; z < 2; ++z) {
      const int k = k0 + 2 * q + z;
      double sn, cs;
      sincos((double)pos * pow(theta, -2.0 * (double)k / (double)d), &sn, &cs);
      xo[z] = __double2bfloat16(xv[z] * cs - yv[z] * sn);
      yo[z] = __double2bfloat16(yv[z] * cs + xv[z] * sn);
    }
    const __nv_bfloat162 xp = __halves2bfloat162(xo[0], xo[1]);
    const __nv_bfloat162 yp = __halves2bfloat162(yo[0], yo[1]);
    xs[q] = *reinterpret_cast<const uint32_t*>(&xp);
    ys[q] = *reinterpret_cast<const uint32_t*>(&yp);
  }
  x = make_uint4(xs[0], xs[1], xs[2], xs[3]);
  y = make_uint4(ys[0], ys[1], ys[2], ys[3]);
}

// ------------------------------------------------------------------ update
// One CTA per sequence. Thread 0 plans the step, all threads copy rows (16-byte vectors). With a
// Past Window (P > 0) the step that makes the usage reach c then compresses it: a block-wide
// scan numbers the past window's separators k = 0, 1, ... (oldest first); the FIFO keeps the
// last s of its current entries followed by them, so separator k lands at ring index
// (sep_head + sep_cnt + k) mod s and is kept when it is among the last s (k >= nnew - s).
constexpr int kUpdateThreads = 128;

__global__ void __launch_bounds__(kUpdateThreads) sepcache_update_kernel(
    int Hkv, int d, int a, int s, int w, int P, int c, int orig, double theta,
    uint4* __restrict__ k_slots,
    uint4* __restrict__ v_slots, int32_t* __restrict__ slot_pos, uint8_t* __restrict__ slot_sep,
    int32_t* __restrict__ meta, const uint4* __restrict__ k_new, const uint4* __restrict__ v_new,
    const uint8_t* __restrict__ sep_new) {
  extern __shared__ int2 s_moves[];  // compression: (past slot, separator slot), min(s, P) at most
  const int seq = blockIdx.x;
  const int ns = a + s + P + w;       // slots per sequence
  const int win_base = a + s + P;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int32_t* m = meta + (size_t)seq * SEPCACHE_META;
  // slot_new, move_from, move_to, t, compress, past_cnt, sep_head, sep_cnt
  __shared__ int plan[8];
  __shared__ int s_warp[kUpdateThreads / 32];
  // the metadata and the flag of the window's oldest slot, loaded in parallel
  __shared__ int s_meta[SEPCACHE_META];
  __shared__ int s_oldsep;
  if (tid < SEPCACHE_META) s_meta[tid] = m[tid];
  if (tid == 32) {
    const int wh = m[SEPCACHE_META_WIN_HEAD];
    s_oldsep = slot_sep[(size_t)seq * ns + win_base + wh];
  }
  __syncthreads();
  if (tid == 0) {
    const int t = s_meta[SEPCACHE_META_T];
    int slot_new, move_from = -1, move_to = -1;
    int ninit = s_meta[SEPCACHE_META_NINIT];
    int sep_head = s_meta[SEPCACHE_META_SEP_HEAD], sep_cnt = s_meta[SEPCACHE_META_SEP_CNT];
    int win_head = s_meta[SEPCACHE_META_WIN_HEAD], win_cnt = s_meta[SEPCACHE_META_WIN_CNT];
    int past_cnt = (P > 0) ? s_meta[SEPCACHE_META_PAST_CNT] : 0;
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
      }
      slot_new = old_slot;
      win_head = (win_head + 1) % w;
    }
    const bool compress = P > 0 && ninit + sep_cnt + past_cnt + win_cnt >= c;
    m[SEPCACHE_META_T] = t + 1;
    m[SEPCACHE_META_NINIT] = ninit;
    m[SEPCACHE_META_SEP_HEAD] = sep_head;
    m[SEPCACHE_META_SEP_CNT] = sep_cnt;
    m[SEPCACHE_META_WIN_HEAD] = win_head;
    m[SEPCACHE_META_WIN_CNT] = win_cnt;
    if (P > 0) m[SEPCACHE_META_PAST_CNT] = past_cnt;
    plan[0] = slot_new;
    plan[1] = move_from;
    plan[2] = move_to;
    plan[3] = t;
    plan[4] = compress ? 1 : 0;
    plan[5] = past_cnt;
    plan[6] = sep_head;
    plan[7] = sep_cnt;
  }
  __syncthreads();
  const int slot_new = plan[0], move_from = plan[1], move_to = plan[2], t = plan[3];
  const int vec = d / 8;  // 16-byte vectors per row
  const size_t seq_rows = (size_t)seq * Hkv * ns;
  auto copy_row = [&](int from, int to) {  // all heads, all threads
    for (int e = tid; e < Hkv * vec; e += kUpdateThreads) {
      const int hh = e / vec, q = e % vec;
      const size_t src = (seq_rows + (size_t)hh * ns + from) * vec + q;
      const size_t dst = (seq_rows + (size_t)hh * ns + to) * vec + q;
      k_slots[dst] = k_slots[src];
      v_slots[dst] = v_slots[src];
    }
  };
  if (move_from >= 0) {
    copy_row(move_from, move_to);
    if (tid == 0) {
      slot_pos[(size_t)seq * ns + move_to] = slot_pos[(size_t)seq * ns + move_from];
      slot_sep[(size_t)seq * ns + move_to] = slot_sep[(size_t)seq * ns + move_from];
    }
    __syncthreads();
  }
  const int hv = vec / 2;  // chunks per RoPE half
  for (int e = tid; e < Hkv * hv; e += kUpdateThreads) {  // K: chunk q and its partner q + hv
    const int hh = e / hv, q = e % hv;
    const size_t dst = (seq_rows + (size_t)hh * ns + slot_new) * vec + q;
    const size_t src = ((size_t)seq * Hkv + hh) * vec + q;
    uint4 x = k_new[src], y = k_new[src + hv];
    if (orig) rope_rotate_chunks(x, y, 8 * q, t, d, theta);
    k_slots[dst] = x;
    k_slots[dst + hv] = y;
  }
  for (int e = tid; e < Hkv * vec; e += kUpdateThreads) {
    const int hh = e / vec, q = e % vec;
    v_slots[(seq_rows + (size_t)hh * ns + slot_new) * vec + q] = v_new[((size_t)seq * Hkv + hh) * vec + q];
  }
  if (tid == 0) {
    slot_pos[(size_t)seq * ns + slot_new] = t;
    slot_sep[(size_t)seq * ns + slot_new] = sep_new[seq] != 0;
  }
  if (!plan[4]) return;

  // ---- compression of the past window [a + s, a + s + past_cnt)
  __syncthreads();
  const int past_cnt = plan[5], sep_head = plan[6], sep_cnt = plan[7];
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
    copy_row(mv.x, mv.y);
    if (tid == 0) {
      slot_pos[(size_t)seq * ns + mv.y] = slot_pos[(size_t)seq * ns + mv.x];
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
  }
}

// ------------------------------------------------------------------ prefill
// State after appending the L prompt tokens of every sequence one at a time to an empty cache,
// in one pass (the same rule as sepcache_update, solved in closed form):
//   initial slots 0..min(a, L)-1 hold tokens 0..min(a, L)-1;
//   the window ring holds the last min(w, L - a) tokens, token u at ring index (u - a) mod w,
//   its head at (L - a) mod w once the ring has wrapped;
//   the tokens u in [a, L - w) have left the window; the k-th separator among them (k = 0,
//   1, ...) went to separator ring index k mod s, so the ring keeps the last min(s, count) of
//   them, its head at count mod s once full (nothing is kept when s = 0).
// One CTA per (sequence, KV head): each scans the flags (block-wide exclusive scan) to place the
// kept separators, copies its head's K/V rows, and the head-0 CTA writes the metadata and the
// slot maps. K/V rows of unused slots are left as they are.
constexpr int kPrefillThreads = 256;
constexpr int kPrefillItems = 16;

__global__ void __launch_bounds__(kPrefillThreads) sepcache_prefill_kernel(
    int L, int Hkv, int d, int a, int s, int w, int orig, double theta,
    const uint4* __restrict__ k_in,
    const uint4* __restrict__ v_in, const uint8_t* __restrict__ sep_in, uint4* __restrict__ k_slots,
    uint4* __restrict__ v_slots, int32_t* __restrict__ slot_pos, uint8_t* __restrict__ slot_sep,
    int32_t* __restrict__ meta) {
  extern __shared__ int s_seppos[];  // [s]: position of the separator at each ring index
  __shared__ int s_warp[kPrefillThreads / 32];
  __shared__ int s_total;
  const int seq = blockIdx.x, head = blockIdx.y;
  const int c = a + s + w;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint8_t* flags = sep_in + (size_t)seq * L;
  const int ninit = min(a, L);
  const int nwin = max(0, min(w, L - a));
  const int left_end = max(a, L - w);  // tokens in [a, left_end) have left the window

  // ---- pass 1: how many separators left the window
  int cnt = 0;
  for (int u = a + tid; u < left_end; u += kPrefillThreads) cnt += flags[u] != 0;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) cnt += __shfl_down_sync(0xffffffffu, cnt, o);
  if (lane == 0) s_warp[warp] = cnt;
  __syncthreads();
  if (tid == 0) {
    int tot = 0;
    for (int x = 0; x < kPrefillThreads / 32; ++x) tot += s_warp[x];
    s_total = tot;
  }
  __syncthreads();
  const int count = (s > 0) ? s_total : 0;
  const int sep_cnt = min(s, count);
  const int first_kept = count - sep_cnt;

  // ---- pass 2: exclusive scan; the kept separators record their positions by ring index
  if (sep_cnt > 0) {
    int carry = 0;
    for (int base = a; base < left_end; base += kPrefillThreads * kPrefillItems) {
      const int u0 = base + tid * kPrefillItems;
      uint32_t bits = 0;
#pragma unroll
      for (int q = 0; q < kPrefillItems; ++q)
        if (u0 + q < left_end && flags[u0 + q] != 0) bits |= 1u << q;
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

  // slot -> original position (-1: unused)
  auto pos_of = [&](int slot) -> int {
    if (slot < a) return slot < ninit ? slot : -1;
    if (slot < a + s) {
      const int r = slot - a;
      return (count >= s || r < count) ? s_seppos[r] : -1;
    }
    const int r = slot - a - s;
    if (nwin == w || r < nwin) {
      const int first = L - nwin;  // oldest token in the window
      const int r0 = (first - a) % w;
      return first + (r - r0 + w) % w;
    }
    return -1;
  };

  // ---- metadata and slot maps (once per sequence)
  if (head == 0) {
    for (int slot = tid; slot < c; slot += kPrefillThreads) {
      const int pos = pos_of(slot);
      slot_pos[(size_t)seq * c + slot] = pos;
      slot_sep[(size_t)seq * c + slot] = (pos >= 0 && flags[pos] != 0) ? 1 : 0;
    }
    if (tid == 0) {
      int32_t* m = meta + (size_t)seq * SEPCACHE_META;
      m[SEPCACHE_META_T] = L;
      m[SEPCACHE_META_NINIT] = ninit;
      m[SEPCACHE_META_SEP_HEAD] = (count >= s && s > 0) ? count % s : 0;
      m[SEPCACHE_META_SEP_CNT] = sep_cnt;
      m[SEPCACHE_META_WIN_HEAD] = (L - a >= w) ? (L - a) % w : 0;
      m[SEPCACHE_META_WIN_CNT] = nwin;
    }
  }
  // ---- this head's K/V rows of the occupied slots (one warp per row, 16-byte vectors)
  const int vec = d / 8;
  const size_t dst_base = ((size_t)seq * Hkv + head) * c;
  for (int slot = warp; slot < c; slot += kPrefillThreads / 32) {
    const int pos = pos_of(slot);
    if (pos < 0) continue;
    const size_t src = (((size_t)seq * L + pos) * Hkv + head) * vec;
    const size_t dst = (dst_base + slot) * vec;
    for (int e = lane; e < vec / 2; e += 32) {  // K: chunk e and its RoPE partner
      uint4 x = __ldg(k_in + src + e), y = __ldg(k_in + src + e + vec / 2);
      if (orig) rope_rotate_chunks(x, y, 8 * e, pos, d, theta);
      k_slots[dst + e] = x;
      k_slots[dst + e + vec / 2] = y;
    }
    for (int e = lane; e < vec; e += 32) v_slots[dst + e] = __ldg(v_in + src + e);
  }
}

cudaError_t launch_sepcache_prefill(const SepCacheState& st, const void* k, const void* v,
                                    const uint8_t* sep, int L, cudaStream_t stream) {
  const size_t smem = (size_t)max(st.s, 1) * sizeof(int);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(sepcache_prefill_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  sepcache_prefill_kernel<<<dim3(st.S, st.Hkv), kPrefillThreads, smem, stream>>>(
      L, st.Hkv, st.d, st.a, st.s, st.w, st.original_positions, (double)st.rope_theta,
      static_cast<const uint4*>(k),
      static_cast<const uint4*>(v), sep, reinterpret_cast<uint4*>(st.k_slots),
      reinterpret_cast<uint4*>(st.v_slots), st.slot_pos, st.slot_sep, st.meta);
  return cudaGetLastError();
}

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

// N consecutive bf16 from shared memory (4- or 8-byte aligned) to fp32.
template <int N>
__device__ __forceinline__ void load_bf16_vec_smem(const __nv_bfloat16* p, float (&out)[N]) {
  if constexpr (N == 4) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    const __nv_bfloat162 x = *reinterpret_cast<const __nv_bfloat162*>(&u.x);
    const __nv_bfloat162 y = *reinterpret_cast<const __nv_bfloat162*>(&u.y);
    out[0] = __low2float(x); out[1] = __high2float(x);
    out[2] = __low2float(y); out[3] = __high2float(y);
  } else {
    static_assert(N == 2, "two or four elements per lane");
    const uint32_t u = *reinterpret_cast<const unsigned int*>(p);
    const __nv_bfloat162 x = *reinterpret_cast<const __nv_bfloat162*>(&u);
    out[0] = __low2float(x); out[1] = __high2float(x);
  }
}

// ------------------------------------------------------------------ decode
// Streaming: bulk copies bring the K and V rows of kChunk consecutive ranks (as few contiguous
// slot segments as the rings allow) into a kStages-deep shared-memory ring. Thread 0 fills the
// first stages; afterwards the last warp to finish reading a stage refills it with the chunk
// kStages further on, so no thread waits to issue. Half-warp hw handles ranks r0 + hw + 16k;
// lane16 owns HP rotation pairs (k, k + d/2), k = lane16 * HP + e, of every row it reads.
// Half-warp reduction of the G per-query partial dot products of one key row: the first
// log2(G) butterfly levels halve what a lane holds (it keeps one half, adding its partner's copy
// of it, and sends the other half), the remaining levels sum a single value. Afterwards lane
// l16 holds the full score of query own_query<G>(l16): 2G + 3 - log2(G) shuffles and adds
// instead of 4G for one reduction per query.
template <int G>
__host__ __device__ constexpr int log2_of() {
  return G >= 16 ? 4 : G >= 8 ? 3 : G >= 4 ? 2 : G >= 2 ? 1 : 0;
}
template <int G>
__device__ __forceinline__ float halfwarp_reduce_own(float (&v)[G], int lane16) {
  constexpr int LG = log2_of<G>();
  static_assert((1 << LG) == G && G <= 16, "G must be a power of two <= 16");
#pragma unroll
  for (int l = 0; l < LG; ++l) {
    const int off = 8 >> l, h = (G >> l) >> 1;
    const bool upper = (lane16 & off) != 0;
#pragma unroll
    for (int i = 0; i < h; ++i) {
      const float send = upper ? v[i] : v[i + h];
      const float keep = upper ? v[i + h] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
    }
  }
  float r = v[0];
#pragma unroll
  for (int l = LG; l < 4; ++l) r += __shfl_xor_sync(0xffffffffu, r, 8 >> l);
  return r;
}
// The query whose score lane l16 holds after halfwarp_reduce_own, and a lane holding query g.
template <int G>
__device__ __forceinline__ int own_query(int lane16) {
  int g = 0;
#pragma unroll
  for (int l = 0; l < log2_of<G>(); ++l)
    if (lane16 & (8 >> l)) g += G >> (l + 1);
  return g;
}
template <int G>
__device__ __forceinline__ int lane_of_query(int g) {
  int src = 0;
#pragma unroll
  for (int l = 0; l < log2_of<G>(); ++l)
    if (g & (G >> (l + 1))) src |= 8 >> l;
  return src;
}

constexpr int kChunk = 16;
constexpr int kStages = 4;
constexpr int kConsumerWarps = kDecThreads / 32;

template <int D>
struct DecSmem {
  alignas(128) __nv_bfloat16 k[kStages][kChunk][D];
  alignas(128) __nv_bfloat16 v[kStages][kChunk][D];
  uint64_t full[kStages];
  int done[kStages];  // warps finished with the stage's current chunk
  int abort_flag;
};

// ORIG: keys were stored rotated at their original positions (no positional shifting): no
// rotation of keys here, and the query is rotated at its own original position T - 1.
template <int D, int G, bool ORIG>
__global__ void __launch_bounds__(kDecThreads, (G >= 8) ? 2 : 4)
    sepcache_decode_kernel(int Hq, int Hkv, int a, int s, int P, int w,
                           const __nv_bfloat16* __restrict__ k_slots,
                           const __nv_bfloat16* __restrict__ v_slots,
                           const int32_t* __restrict__ meta, const float2* __restrict__ rope_cs,
                           const __nv_bfloat16* __restrict__ q, __nv_bfloat16* __restrict__ o,
                           float* __restrict__ lse, float scale_log2, double theta,
                           unsigned* err) {
  constexpr int HP = D / 32;       // rotation pairs per lane
  constexpr int HALF = D / 2;
  const int kvh = blockIdx.x, seq = blockIdx.y;
  const int c = a + s + P + w;  // slots per sequence (and rows of the cos/sin table)
  const int tid = threadIdx.x, lane16 = tid & 15, hw = tid >> 4, warp = tid >> 5;
  extern __shared__ __align__(128) uint8_t dsm_raw[];
  DecSmem<D>& sm = *reinterpret_cast<DecSmem<D>*>(dsm_raw);

  const int32_t* m = meta + (size_t)seq * SEPCACHE_META;
  const int ninit = m[SEPCACHE_META_NINIT];
  const int sep_head = m[SEPCACHE_META_SEP_HEAD], sep_cnt = m[SEPCACHE_META_SEP_CNT];
  const int win_head = m[SEPCACHE_META_WIN_HEAD], win_cnt = m[SEPCACHE_META_WIN_CNT];
  const int past_cnt = (P > 0) ? m[SEPCACHE_META_PAST_CNT] : 0;
  const int occ = ninit + sep_cnt + past_cnt + win_cnt;
  const int mq = occ - 1;  // the query's own rank
  const int r0 = 0, r1 = occ;
  const int nchunks = r1 > r0 ? (r1 - r0 + kChunk - 1) / kChunk : 0;
  const size_t row_base = ((size_t)seq * Hkv + kvh) * c;
  volatile int* abort_flag = &sm.abort_flag;

  auto issue_chunk = [&](int ch) {  // one thread: bulk copies of chunk ch into its stage
    const int st = ch % kStages;
    const int c0 = r0 + ch * kChunk;
    const int rows = min(kChunk, r1 - c0);
    mbar_arrive_expect_tx(&sm.full[st], (uint32_t)(rows * D * 2 * 2));
    // ranks map to slots piecewise contiguously: initial block, then the separator ring, then
    // the past window, then the window ring; a run ends at a block boundary or a ring wrap
    int r = c0;
    const int end = c0 + rows;
    while (r < end) {
      int slot, len;
      if (r < ninit) {
        slot = r;
        len = min(end, ninit) - r;
      } else if (r < ninit + sep_cnt) {
        const int x = (sep_head + (r - ninit)) % s;
        slot = a + x;
        len = min(min(end, ninit + sep_cnt) - r, s - x);
      } else if (r < ninit + sep_cnt + past_cnt) {
        slot = a + s + (r - ninit - sep_cnt);
        len = min(end, ninit + sep_cnt + past_cnt) - r;
      } else {
        const int x = (win_head + (r - ninit - sep_cnt - past_cnt)) % w;
        slot = a + s + P + x;
        len = min(end - r, w - x);
      }
      const size_t src = (row_base + slot) * D;
      bulk_load(&sm.k[st][r - c0][0], k_slots + src, (uint32_t)(len * D * 2), &sm.full[st]);
      bulk_load(&sm.v[st][r - c0][0], v_slots + src, (uint32_t)(len * D * 2), &sm.full[st]);
      r += len;
    }
  };
  if (tid == 0) {
    for (int st = 0; st < kStages; ++st) {
      mbar_init(&sm.full[st], 1);
      sm.done[st] = 0;
    }
    sm.abort_flag = 0;
    fence_barrier_init();
    for (int ch = 0; ch < min(kStages, nchunks); ++ch) issue_chunk(ch);
  }
  __syncthreads();

  // per-head softmax state (consumers)
  // softmax state of this lane's own query (see halfwarp_reduce_own); V sums of every query,
  // as pairs of consecutive elements for the packed fp32x2 arithmetic (lo: elements
  // lane16 * HP + 2i, +1; hi: the same plus d/2)
  static_assert(HP % 2 == 0, "rotation pairs per lane come in twos");
  constexpr int HP2 = HP / 2;
  float m_own = -INFINITY, l_own = 0.f;
  float2 acc_lo[G][HP2], acc_hi[G][HP2];
#pragma unroll
  for (int g = 0; g < G; ++g) {
#pragma unroll
    for (int i = 0; i < HP2; ++i) acc_lo[g][i] = acc_hi[g][i] = make_float2(0.f, 0.f);
  }

  {
    // ---------------------------------------------------------------- consumers
    // query heads of this KV head, rotated by RoPE(mq) (by RoPE(T - 1) without shifting) and
    // scaled by scale*log2(e)
    float2 q_lo[G][HP2], q_hi[G][HP2];
    {
      float2 qcs[HP];
#pragma unroll
      for (int e = 0; e < HP; ++e) {
        const int k = lane16 * HP + e;
        if constexpr (ORIG) {
          double sn, cs;
          sincos((double)(m[SEPCACHE_META_T] - 1) * pow(theta, -2.0 * (double)k / (double)D), &sn,
                 &cs);
          qcs[e] = make_float2((float)cs, (float)sn);
        } else {
          qcs[e] = rope_cs[(size_t)max(mq, 0) * HALF + k];
        }
      }
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const __nv_bfloat16* qh = q + ((size_t)seq * Hq + kvh * G + g) * D;
        float qa[HP], qb[HP];
#pragma unroll
        for (int e = 0; e < HP; ++e) {
          const int k = lane16 * HP + e;
          const float x1 = __bfloat162float(qh[k]), x2 = __bfloat162float(qh[k + HALF]);
          const float2 rr = qcs[e];
          qa[e] = (x1 * rr.x - x2 * rr.y) * scale_log2;
          qb[e] = (x2 * rr.x + x1 * rr.y) * scale_log2;
        }
#pragma unroll
        for (int i = 0; i < HP2; ++i) {
          q_lo[g][i] = make_float2(qa[2 * i], qa[2 * i + 1]);
          q_hi[g][i] = make_float2(qb[2 * i], qb[2 * i + 1]);
        }
      }
    }
    // cos/sin of this half-warp's current rank, advanced by kHalfWarps per step (pairs of
    // consecutive frequencies; nsd = -sin of the step)
    float2 cr[HP2], sr[HP2], cd[HP2], sd[HP2], nsd[HP2];
    {
      const int rf = r0 + hw;
#pragma unroll
      for (int i = 0; i < HP2; ++i) {
        const int k = lane16 * HP + 2 * i;
        const float2 v0 = (rf < r1) ? rope_cs[(size_t)rf * HALF + k] : make_float2(1.f, 0.f);
        const float2 v1 = (rf < r1) ? rope_cs[(size_t)rf * HALF + k + 1] : make_float2(1.f, 0.f);
        cr[i] = make_float2(v0.x, v1.x);
        sr[i] = make_float2(v0.y, v1.y);
        const float2 t0 = rope_cs[(size_t)min(kHalfWarps, c - 1) * HALF + k];
        const float2 t1 = rope_cs[(size_t)min(kHalfWarps, c - 1) * HALF + k + 1];
        cd[i] = make_float2(t0.x, t1.x);
        sd[i] = make_float2(t0.y, t1.y);
        nsd[i] = make_float2(-t0.y, -t1.y);
      }
    }
    bool ok = true;
    for (int ch = 0; ch < nchunks && ok; ++ch) {
      const int st = ch % kStages;
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.full[st], (ch / kStages) & 1, err, abort_flag))) {
        ok = false;
        break;
      }
      const int c0 = r0 + ch * kChunk;
#pragma unroll
      for (int sub = 0; sub < kChunk / kHalfWarps; ++sub) {
        const int row = sub * kHalfWarps + hw;
        const bool valid = c0 + row < r1;
        float k1[HP], k2[HP], v1[HP], v2[HP];
        const __nv_bfloat16* kr = &sm.k[st][row][lane16 * HP];
        const __nv_bfloat16* vr = &sm.v[st][row][lane16 * HP];
        if (valid) {
          load_bf16_vec_smem<HP>(kr, k1);
          load_bf16_vec_smem<HP>(kr + HALF, k2);
          load_bf16_vec_smem<HP>(vr, v1);
          load_bf16_vec_smem<HP>(vr + HALF, v2);
        } else {
#pragma unroll
          for (int e = 0; e < HP; ++e) k1[e] = k2[e] = v1[e] = v2[e] = 0.f;
        }
        // rotate (y1, y2) = RoPE(rank) (k1, k2) and form the G partial dot products, two
        // frequencies per packed instruction
        float2 part2[G];
#pragma unroll
        for (int g = 0; g < G; ++g) part2[g] = make_float2(0.f, 0.f);
#pragma unroll
        for (int i = 0; i < HP2; ++i) {
          const float2 x1 = make_float2(k1[2 * i], k1[2 * i + 1]);
          const float2 x2 = make_float2(k2[2 * i], k2[2 * i + 1]);
          float2 y1 = x1, y2 = x2;
          if constexpr (!ORIG) {
            y1 = f2_sub(f2_mul(x1, cr[i]), f2_mul(x2, sr[i]));
            y2 = f2_fma(x2, cr[i], f2_mul(x1, sr[i]));
          }
#pragma unroll
          for (int g = 0; g < G; ++g) part2[g] = f2_fma(q_lo[g][i], y1, f2_fma(q_hi[g][i], y2, part2[g]));
        }
        float part[G];
#pragma unroll
        for (int g = 0; g < G; ++g) part[g] = part2[g].x + part2[g].y;
        if constexpr (!ORIG) {
#pragma unroll
          for (int i = 0; i < HP2; ++i) {
            const float2 cn = f2_fma(cr[i], cd[i], f2_mul(sr[i], nsd[i]));
            sr[i] = f2_fma(sr[i], cd[i], f2_mul(cr[i], sd[i]));
            cr[i] = cn;
          }
        }
        // this lane's query score; the online softmax of that query only, its probability
        // then broadcast to the lanes of the half-warp for the V accumulation of every query
        const float sc = halfwarp_reduce_own<G>(part, lane16);
        const bool need = valid && sc > m_own + 8.0f;  // lazy rescale (max grew by > 2^8)
        if (__any_sync(0xffffffffu, need)) {
          const float alpha = need ? ex2(m_own - sc) : 1.0f;
          if (need) {
            l_own *= alpha;
            m_own = sc;
          }
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const float ag = __shfl_sync(0xffffffffu, alpha, lane_of_query<G>(g), 16);
            const float2 ag2 = make_float2(ag, ag);
#pragma unroll
            for (int i = 0; i < HP2; ++i) {
              acc_lo[g][i] = f2_mul(acc_lo[g][i], ag2);
              acc_hi[g][i] = f2_mul(acc_hi[g][i], ag2);
            }
          }
        }
        const float p_own = valid ? ex2(sc - m_own) : 0.f;
        l_own += p_own;
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float pg = __shfl_sync(0xffffffffu, p_own, lane_of_query<G>(g), 16);
          const float2 pg2 = make_float2(pg, pg);
#pragma unroll
          for (int i = 0; i < HP2; ++i) {
            acc_lo[g][i] = f2_fma(pg2, make_float2(v1[2 * i], v1[2 * i + 1]), acc_lo[g][i]);
            acc_hi[g][i] = f2_fma(pg2, make_float2(v2[2 * i], v2[2 * i + 1]), acc_hi[g][i]);
          }
        }
      }
      // the last warp done with this stage refills it (its reads all precede the atomic)
      __syncwarp();
      if ((tid & 31) == 0) {
        if (atomicAdd(&sm.done[st], 1) == kConsumerWarps - 1) {
          sm.done[st] = 0;
          if (ch + kStages < nchunks) {
            fence_proxy_async_smem();
            issue_chunk(ch + kStages);
          }
        }
      }
    }
    if (!ok) {
      // a wait ran out: let every copy still in flight land before the CTA leaves
      if (tid == 0)
        for (int ch = 0; ch < nchunks; ++ch)
          mbar_wait(&sm.full[ch % kStages], (ch / kStages) & 1, nullptr, nullptr);
    }
  }

  float acc[G][2 * HP];  // V sums, elements lane16 * HP + e (e < HP) and the same plus d/2
#pragma unroll
  for (int g = 0; g < G; ++g) {
#pragma unroll
    for (int i = 0; i < HP2; ++i) {
      acc[g][2 * i] = acc_lo[g][i].x;
      acc[g][2 * i + 1] = acc_lo[g][i].y;
      acc[g][HP + 2 * i] = acc_hi[g][i].x;
      acc[g][HP + 2 * i + 1] = acc_hi[g][i].y;
    }
  }
  // every query's softmax state from the lanes that own it
  float mrun[G], lrun[G];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    mrun[g] = __shfl_sync(0xffffffffu, m_own, lane_of_query<G>(g), 16);
    lrun[g] = __shfl_sync(0xffffffffu, l_own, lane_of_query<G>(g), 16);
  }
  // ---- combine the two half-warps of each warp (lanes l and l^16 hold the same columns)
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const float mo = __shfl_xor_sync(0xffffffffu, mrun[g], 16);
    const float lo = __shfl_xor_sync(0xffffffffu, lrun[g], 16);
    const float M = fmaxf(mrun[g], mo);
    const float Mu = (M == -INFINITY) ? 0.f : M;
    const float fs = ex2(mrun[g] - Mu), fo = ex2(mo - Mu);
#pragma unroll
    for (int e = 0; e < 2 * HP; ++e) {
      const float ao = __shfl_xor_sync(0xffffffffu, acc[g][e], 16);
      acc[g][e] = acc[g][e] * fs + ao * fo;
    }
    lrun[g] = lrun[g] * fs + lo * fo;
    mrun[g] = M;
  }
  // ---- combine the consumer warps of this CTA through shared memory
  __shared__ float s_m[kConsumerWarps][G], s_l[kConsumerWarps][G];
  __shared__ float s_acc[kConsumerWarps][G][D];
  __shared__ float s_res[G][D + 2];  // this CTA's combined (acc..., m, l) per head
  if ((tid & 31) < 16) {
    if (lane16 == 0) {
#pragma unroll
      for (int g = 0; g < G; ++g) {
        s_m[warp][g] = mrun[g];
        s_l[warp][g] = lrun[g];
      }
    }
#pragma unroll
    for (int g = 0; g < G; ++g) {
#pragma unroll
      for (int e = 0; e < HP; ++e) {
        s_acc[warp][g][lane16 * HP + e] = acc[g][e];
        s_acc[warp][g][HALF + lane16 * HP + e] = acc[g][HP + e];
      }
    }
  }
  __syncthreads();
  for (int e = tid; e < G * D; e += blockDim.x) {
    const int g = e / D, col = e % D;
    float M = -INFINITY;
    for (int x = 0; x < kConsumerWarps; ++x) M = fmaxf(M, s_m[x][g]);
    const float Mu = (M == -INFINITY) ? 0.f : M;
    float sum = 0.f, lsum = 0.f;
    for (int x = 0; x < kConsumerWarps; ++x) {
      const float f = ex2(s_m[x][g] - Mu);
      sum += s_acc[x][g][col] * f;
      lsum += s_l[x][g] * f;
    }
    s_res[g][col] = sum;
    if (col == 0) {
      s_res[g][D] = M;
      s_res[g][D + 1] = lsum;
    }
  }
  __syncthreads();
  for (int e = tid; e < G * D; e += blockDim.x) {
    const int g = e / D, col = e % D;
    const int hq = kvh * G + g;
    o[((size_t)seq * Hq + hq) * D + col] = __float2bfloat16(s_res[g][col] / s_res[g][D + 1]);
    if (col == 0 && lse)
      lse[(size_t)seq * Hq + hq] = (s_res[g][D] + __log2f(s_res[g][D + 1])) * 0.69314718055994531f;
  }
}

// ------------------------------------------------------------------ export order
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

// Past Window slots and slots per sequence of a cache state.
static int past_slots(const SepCacheState& st) { return st.c > 0 ? st.c - st.a - st.w : 0; }
static int cache_slots(const SepCacheState& st) { return st.a + st.s + past_slots(st) + st.w; }

cudaError_t launch_sepcache_init(const SepCacheState& st, cudaStream_t stream) {
  const int c = cache_slots(st);
  sepcache_init_kernel<<<64, 256, 0, stream>>>(st.S, c, st.d, (double)st.rope_theta, st.meta,
                                               st.slot_pos, st.slot_sep, st.rope_cs);
  return cudaGetLastError();
}

cudaError_t launch_sepcache_update(const SepCacheState& st, const void* k_new, const void* v_new,
                                   const uint8_t* sep_new, cudaStream_t stream) {
  const int P = past_slots(st);
  const size_t smem = (size_t)max(1, min(st.s, P)) * sizeof(int2);  // compression moves
  sepcache_update_kernel<<<st.S, kUpdateThreads, smem, stream>>>(
      st.Hkv, st.d, st.a, st.s, st.w, P, st.c, st.original_positions, (double)st.rope_theta,
      reinterpret_cast<uint4*>(st.k_slots),
      reinterpret_cast<uint4*>(st.v_slots), st.slot_pos, st.slot_sep, st.meta,
      static_cast<const uint4*>(k_new), static_cast<const uint4*>(v_new), sep_new);
  return cudaGetLastError();
}

template <int D, int G, bool ORIG>
static cudaError_t launch_decode_t(const SepCacheState& st, const void* q, void* o, float* lse,
                                   float scale, cudaStream_t stream) {
  constexpr size_t smem = sizeof(DecSmem<D>);
  static bool attr_set[64] = {false};  // per device: set once, outside any stream capture
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    e = cudaFuncSetAttribute(sepcache_decode_kernel<D, G, ORIG>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  dim3 grid(st.Hkv, st.S);
  sepcache_decode_kernel<D, G, ORIG><<<grid, kDecThreads, smem, stream>>>(
      st.Hq, st.Hkv, st.a, st.s, past_slots(st), st.w,
      reinterpret_cast<const __nv_bfloat16*>(st.k_slots),
      reinterpret_cast<const __nv_bfloat16*>(st.v_slots), st.meta,
      reinterpret_cast<const float2*>(st.rope_cs), static_cast<const __nv_bfloat16*>(q),
      static_cast<__nv_bfloat16*>(o), lse, scale * 1.4426950408889634f, (double)st.rope_theta,
      device_error_word());
  return cudaGetLastError();
}

cudaError_t launch_sepcache_decode(const SepCacheState& st, const void* q, void* o, float* lse,
                                   float scale, cudaStream_t stream) {
  const int G = st.Hq / st.Hkv;
#define SEP_DEC_CASE(DD, GG) \
  if (st.d == DD && G == GG)                                                             \
    return st.original_positions ? launch_decode_t<DD, GG, true>(st, q, o, lse, scale, stream) \
                                 : launch_decode_t<DD, GG, false>(st, q, o, lse, scale, stream);
  SEP_DEC_CASE(128, 1)
  SEP_DEC_CASE(128, 2)
  SEP_DEC_CASE(128, 4)
  SEP_DEC_CASE(128, 8)
  SEP_DEC_CASE(64, 1)
  SEP_DEC_CASE(64, 2)
  SEP_DEC_CASE(64, 4)
  SEP_DEC_CASE(64, 8)
#undef SEP_DEC_CASE
  return cudaErrorInvalidValue;
}

cudaError_t launch_sepcache_export(const SepCacheState& st, int32_t* pos_out, int32_t* count,
                                   cudaStream_t stream) {
  sepcache_export_kernel<<<st.S, 256, 0, stream>>>(st.a, st.s, past_slots(st), st.w, st.meta,
                                                   st.slot_pos, pos_out, count);
  return cudaGetLastError();
}

}  // namespace sep
