/*
 * sepattn.h - C ABI of the B200 (sm_100a) separator-sparse attention library (libsepattn.so).
 *
 * SepLLM keeps, for every query, only the initial tokens, every preceding separator and the n
 * most recent neighbours ("SepLLM: Accelerate Large Language Models by Compressing One Segment
 * into One Separator", atlas.scime.ai summary, section "Approach"); attention is the sparse
 * product O = M(A, V, M_b) with a binary mask M_b ("How SepLLM reorchestrates the language
 * model for speed and efficiency", beiduofen.top, section "SepLLM's Architecture: Composing
 * Efficiency"). Streaming inference keeps initial, separator and local-window KV blocks with
 * positions taken inside the cache (same section; SepLLM project card on sourcepulse.org,
 * section "Limitations & Caveats").
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All tensor arguments are DEVICE pointers to contiguous row-major memory owned by the
 *    caller. The library never allocates, frees or retains memory; scratch memory is passed
 *    in as `workspace` with its size in bytes.
 *  - bf16 tensors are raw IEEE bfloat16 bit patterns (sep_bf16). Every tensor base address
 *    must be 16-byte aligned (SEP_ERR_MISALIGNED otherwise).
 *  - Token-major layouts: Q, O, dO, dQ are [B, L, Hq, d]; K, V, dK, dV are [B, L, Hkv, d].
 *    Query head h reads KV head h / (Hq / Hkv). Head dimension d is 64 or 128.
 *  - Every call is asynchronous and stream-ordered on `stream` (a cudaStream_t; NULL is the
 *    legacy default stream). Nothing synchronises except sep_last_device_error().
 *  - Return value: SEP_OK, or an error code below; on an argument error nothing is launched.
 *    Device-side failures (a bounded wait that ran out) set a sticky device error word that
 *    sep_last_device_error() reads and clears.
 */
#ifndef SEPATTN_H_
#define SEPATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t sep_bf16;           /* raw bfloat16 bits */
typedef struct CUstream_st* sep_stream_t; /* same type as cudaStream_t */

enum {
  SEP_OK = 0,
  SEP_ERR_INVALID_ARG = 1,   /* null pointer, non-positive size, Hq % Hkv != 0, ... */
  SEP_ERR_UNSUPPORTED = 2,   /* a size this build has no kernel for (e.g. d not 64/128) */
  SEP_ERR_MISALIGNED = 3,    /* a tensor base address not 16-byte aligned */
  SEP_ERR_CUDA = 4,          /* a CUDA runtime/driver call or a launch failed */
  SEP_ERR_TIMEOUT = 5,       /* device: a bounded pipeline wait ran out (reported sticky) */
  SEP_ERR_WORKSPACE = 6,     /* workspace pointer null or smaller than the size query says */
  SEP_ERR_SCRATCH_LIMIT = 7  /* sep_attn_fwd_noalloc: problem larger than its fixed scratch */
};

/* Tile sizes the attention kernels use: query tiles of 128 rows, key tiles of 128 columns. */
#define SEP_TILE_M 128
#define SEP_TILE_N 128

/* Tile map values. */
#define SEP_TILE_SKIP 0
#define SEP_TILE_PARTIAL 1
#define SEP_TILE_FULL 2

/*
 * sep_mask_build - the separator-sparse mask M_b in compressed form (one kernel pair).
 *
 * Defines, per batch element b, the anchor flag f[j] = (j < a) || sep[b][j] (initial tokens and
 * separators, "Approach" section cited above) and the keep rule
 *     keep(i, j) = j <= i && (i - j < n || f[j])
 * (n neighbours counted including the query itself). Outputs:
 *   anchor_idx [B, L] int32  positions j with f[j], ascending; entries past anchor_cnt[b] = -1.
 *   anchor_cnt [B]    int32  number of anchors.
 *   anchor_bits [B, W] uint32 W = ceil(L / 32): bit k of word w is f[32w + k] (0 past L).
 *   gather_end [B, T] int32  T = ceil(L / bm). With lo(t) = max(0, t*bm - n + 1) / bn (integer
 *                            division), gather_end[b][t] = number of anchors at positions
 *                            < lo(t)*bn: the anchors that every row of query tile t keeps and
 *                            that lie left of its window key tiles lo(t)..t.
 *   tile_map [B, T, U] int8  U = ceil(L / bn). SEP_TILE_SKIP if no pair of block (t, u) is
 *                            kept, SEP_TILE_FULL if every in-bounds pair is kept,
 *                            SEP_TILE_PARTIAL otherwise.
 *   kept_pairs [B]   int64   number of kept pairs (nullable: not written when NULL).
 * sep is [B, L] uint8 (non-zero = separator). Requires B >= 1, L >= 1, a >= 0, n >= 1,
 * bm >= 1, bn >= 1. The attention calls need bm = SEP_TILE_M and bn = SEP_TILE_N.
 */
int sep_mask_build(const uint8_t* sep, int B, int L, int a, int n, int bm, int bn,
                   int32_t* anchor_idx, int32_t* anchor_cnt, uint32_t* anchor_bits,
                   int32_t* gather_end, int8_t* tile_map, int64_t* kept_pairs,
                   sep_stream_t stream);

/* The outputs of sep_mask_build (built with bm = SEP_TILE_M, bn = SEP_TILE_N) plus the flags. */
typedef struct SepMask {
  int B, L, a, n;
  const uint8_t* sep;         /* [B, L] the flags the mask was built from */
  const int32_t* anchor_idx;  /* [B, L] */
  const int32_t* anchor_cnt;  /* [B] */
  const uint32_t* anchor_bits; /* [B, ceil(L/32)] */
  const int32_t* gather_end;  /* [B, ceil(L/128)] */
  const int8_t* tile_map;     /* [B, ceil(L/128), ceil(L/128)] */
} SepMask;

/*
 * sep_attn_fwd - O = M(A, V, M_b): softmax attention restricted to kept pairs.
 *
 * For every batch b, query head h and row i: S_ij = scale * q_i . k_j over kept j, P = softmax
 * over those j, O_i = sum_j P_ij v_j, lse[b][h][i] = ln sum_j exp(S_ij) (fp32). bf16 inputs,
 * fp32 accumulation, bf16 O. `mask` must describe the same B, L, a, n. Skipped tiles are never
 * loaded; anchors left of the window are read from a compacted copy built in `workspace`
 * (size: sep_attn_fwd_workspace_size).
 * Arguments: q [B,L,Hq,d], k/v [B,L,Hkv,d], o [B,L,Hq,d], lse [B,Hq,L]. Hq % Hkv == 0,
 * d in {64, 128}.
 */
size_t sep_attn_fwd_workspace_size(int B, int L, int Hkv, int d);
int sep_attn_fwd(const sep_bf16* q, const sep_bf16* k, const sep_bf16* v,
                 int B, int L, int Hq, int Hkv, int d, float scale, int a, int n,
                 const SepMask* mask, sep_bf16* o, float* lse,
                 void* workspace, size_t workspace_bytes, sep_stream_t stream);

/*
 * sep_attn_bwd - gradients of sum(O * dO) for sep_attn_fwd over the same kept pairs.
 *
 * With P_ij = exp(S_ij - lse_i) on kept pairs: dV = P^T dO, dP = dO V^T,
 * Delta_i = sum_c dO_ic O_ic, dS = P * (dP - Delta), dQ = scale dS K, dK = scale dS^T Q;
 * dK and dV of a KV head are summed over the Hq/Hkv query heads that share it. Standard
 * flash-attention backward, which the pages use when training with the mask from scratch
 * ("Key results": training-from-scratch speedup; "The Mechanics of Compression").
 * Arguments: q, k, v, o (from sep_attn_fwd), lse (from sep_attn_fwd), dout [B,L,Hq,d];
 * outputs dq [B,L,Hq,d], dk/dv [B,L,Hkv,d] (bf16, fp32 accumulation). `workspace` holds the
 * compacted anchors, Delta and fp32 partial sums (size: sep_attn_bwd_workspace_size).
 */
size_t sep_attn_bwd_workspace_size(int B, int L, int Hq, int Hkv, int d);
int sep_attn_bwd(const sep_bf16* q, const sep_bf16* k, const sep_bf16* v, const sep_bf16* o,
                 const float* lse, const sep_bf16* dout,
                 int B, int L, int Hq, int Hkv, int d, float scale, int a, int n,
                 const SepMask* mask, sep_bf16* dq, sep_bf16* dk, sep_bf16* dv,
                 void* workspace, size_t workspace_bytes, sep_stream_t stream);

/*
 * Staged forms, for timing one pass at a time: the same arguments as sep_attn_fwd /
 * sep_attn_bwd plus a stage number. Running the stages 0, 1 (, 2) in order on one stream is
 * exactly the one-call form; a stage reads what the earlier stages left in `workspace`.
 *   sep_attn_fwd_stage: 0 = anchor compaction into the workspace, 1 = attention kernel.
 *   sep_attn_bwd_stage: 0 = anchor compaction, zeroed fp32 anchor partials, Delta;
 *                       1 = dQ pass; 2 = dK/dV pass and the anchor combine.
 * Returns SEP_ERR_INVALID_ARG for any other stage number.
 */
int sep_attn_fwd_stage(int stage, const sep_bf16* q, const sep_bf16* k, const sep_bf16* v,
                       int B, int L, int Hq, int Hkv, int d, float scale, int a, int n,
                       const SepMask* mask, sep_bf16* o, float* lse,
                       void* workspace, size_t workspace_bytes, sep_stream_t stream);
int sep_attn_bwd_stage(int stage, const sep_bf16* q, const sep_bf16* k, const sep_bf16* v,
                       const sep_bf16* o, const float* lse, const sep_bf16* dout,
                       int B, int L, int Hq, int Hkv, int d, float scale, int a, int n,
                       const SepMask* mask, sep_bf16* dq, sep_bf16* dk, sep_bf16* dv,
                       void* workspace, size_t workspace_bytes, sep_stream_t stream);

/*
 * SepCache: streaming KV cache of S independent sequences ("SepLLM's Architecture: Composing
 * Efficiency", beiduofen.top): a initial slots, a separator FIFO of s slots, a local-window
 * FIFO of w slots and, when the usage threshold c is non-zero, a Past Window of P = c - a - w
 * slots that holds the tokens leaving the window until the total usage reaches c. With c = 0
 * there is no Past Window and compression is one token at a time. Keys are seen at their
 * positions inside the cache (positional-encoding shifting, SepLLM project card, "Limitations &
 * Caveats"): the key of rank p at RoPE(p), the newest token's query at RoPE(occupied - 1).
 *
 * Storage of the keys: every key is stored rotated once, in bf16, by RoPE(u) where u is a
 * counter that differs from its rank by an offset shared by its whole block: its original
 * position t for initial, past-window and window keys, and its admission index A (the A-th
 * separator admitted to the FIFO since the cache was empty) for separators. A key is rotated by
 * RoPE(t) when it is appended and by RoPE(A - t) more when it enters the separator FIFO;
 * decode rotates the query once per block. Rotation angles are formed in fp64.
 *
 * Slots per sequence: n = a + s + P + w (P = 0 when c = 0), in this order: initial, separator
 * ring, past window, window ring. Every pointer below is caller-owned device memory; the
 * struct itself lives on the host and is read by each call. Sizes in elements:
 *   k_slots, v_slots  S * Hkv * n * d bf16   slot-major per (sequence, KV head)
 *   slot_pos          S * n int32             original position held by each slot (-1 empty)
 *   slot_sep          S * n uint8             separator flag of each slot's token
 *   meta              S * SEPCACHE_META int32 per-sequence counters (see below)
 *   rope_freq         d / 2 double            RoPE inverse frequencies theta^(-2k/d)
 */
#define SEPCACHE_META 8
/* meta[seq * SEPCACHE_META + ...] */
#define SEPCACHE_META_T 0         /* tokens appended so far */
#define SEPCACHE_META_NINIT 1     /* occupied initial slots */
#define SEPCACHE_META_SEP_HEAD 2  /* separator FIFO: ring index of the oldest entry */
#define SEPCACHE_META_SEP_CNT 3   /* separator FIFO: entries */
#define SEPCACHE_META_WIN_HEAD 4  /* window FIFO: ring index of the oldest entry */
#define SEPCACHE_META_WIN_CNT 5   /* window FIFO: entries */
#define SEPCACHE_META_PAST_CNT 6  /* past window: entries (c > 0) */
#define SEPCACHE_META_SEP_ADMIT 7 /* separators admitted to the FIFO so far (the FIFO holds
                                     admission indices SEP_ADMIT - SEP_CNT .. SEP_ADMIT - 1) */

typedef struct SepCacheState {
  int32_t S, Hq, Hkv, d;     /* sequences, query heads, KV heads, head dim (d = 128 or 64);
                                Hq / Hkv query heads share a KV head, 1 to 8 of them */
  int32_t a, s, w;           /* initial / separator / window capacities */
  int32_t c;                 /* usage threshold of the Past Window (0: none; else > a + s + w) */
  int32_t original_positions; /* 0: positional-encoding shifting (ranks inside the cache);
                                 1: no shifting, every key and the query at their original
                                 positions (keys stay at RoPE(t) in every block) */
  float rope_theta;          /* RoPE base: angle of pair k at position p = p * theta^(-2k/d) */
  sep_bf16* k_slots;
  sep_bf16* v_slots;
  int32_t* slot_pos;
  uint8_t* slot_sep;
  int32_t* meta;
  double* rope_freq;
} SepCacheState;

/* Empties every sequence (meta and slot_pos) and fills rope_freq. Call once before use. */
int sepcache_state_init(const SepCacheState* st, sep_stream_t stream);

/*
 * sepcache_update - append one token to every sequence (one kernel).
 * k_new, v_new [S, Hkv, d] without rotary embedding; sep_new [S] uint8. Token t of a sequence goes to
 * initial slot t when t < a; otherwise to the window. If the window then holds more than w
 * tokens its oldest token leaves. With c = 0 it goes into the separator FIFO if it is a
 * separator and is dropped otherwise. With c > 0 it goes to the Past Window, and when the
 * total usage (initial + separators + past + window) then reaches c the Past Window is
 * compressed: its separators enter the separator FIFO oldest first, the rest is dropped.
 * Whenever the separator FIFO holds more than s entries its oldest are dropped.
 * With c > 0, min(s, c - a - w) must be at most 4096 (SEP_ERR_UNSUPPORTED otherwise).
 */
int sepcache_update(const SepCacheState* st, const sep_bf16* k_new, const sep_bf16* v_new,
                    const uint8_t* sep_new, sep_stream_t stream);

/*
 * sepcache_prefill - seed every sequence's cache with an L-token prompt in one call.
 * Sets the state to the one L sepcache_update calls (tokens 0..L-1 in order) would leave on an
 * empty cache, whatever the state was before; K/V rows of slots left unused are not touched.
 * This is how a prompt processed by sep_attn_fwd (the prefill pass) hands its keys and values
 * to streaming decode ("How SepLLM reorchestrates the language model...", "SepLLM's
 * Architecture: Composing Efficiency": initial, separator and local-window blocks).
 * With a Past Window (c > 0) the compressions the updates would have made are replayed run by
 * run: each run of c - a - w - (separators held) tokens that has left the window is one
 * compression, so the call costs one block-wide count per run.
 * k, v [S, L, Hkv, d] without rotary embedding (the layout sep_attn_fwd reads); sep [S, L]
 * uint8. L >= 1; s <= 16384 (SEP_ERR_UNSUPPORTED otherwise).
 */
int sepcache_prefill(const SepCacheState* st, const sep_bf16* k, const sep_bf16* v,
                     const uint8_t* sep, int L, sep_stream_t stream);

/*
 * sepcache_decode - single-query attention of each sequence's newest token over its cache.
 * Logical order = [initial | separators oldest first | past window oldest first | window
 * oldest first]; the key of rank p is seen at RoPE(p) and the query at RoPE(m),
 * m = occupied - 1 (its own rank): the stored keys are read as they are and the query is rotated
 * once per block by RoPE(m - offset of the block). With original_positions = 1 (training-free
 * use without shifting) keys and query are at their original positions (query at T - 1).
 * q [S, Hq, d] un-rotated; o [S, Hq, d] bf16; lse [S, Hq] fp32 natural log (nullable).
 * Call after sepcache_update of the same step.
 */
int sepcache_decode(const SepCacheState* st, const sep_bf16* q, sep_bf16* o, float* lse,
                    float scale, sep_stream_t stream);

/* Original positions of each sequence's retained tokens in logical order: pos_out [S, c]
 * (-1 past count), count [S]. For exact checks of the cache trajectory. */
int sepcache_export_order(const SepCacheState* st, int32_t* pos_out, int32_t* count,
                          sep_stream_t stream);

/* Reads and clears the sticky device error word of the current device (synchronises the
 * device). Returns SEP_OK or the first SEP_ERR_* a kernel recorded. */
int sep_last_device_error(void);

/*
 * sep_set_wait_limit_ns - test hook for the device-side failure path.
 *
 * Every wait of the kernels on a pipeline barrier is bounded; when one runs out the kernel
 * records SEP_ERR_TIMEOUT in the sticky device error word, lets the copies and tensor-core work
 * it issued finish, frees its tensor memory and returns. This call sets the limit of the
 * pipeline waits of the attention forward kernels launched afterwards, process-wide (ns = 0
 * restores the default of 1.5 s); waits that drain issued work always keep 1.5 s. A very short
 * limit makes a normal launch give up part-way, which is how a test exercises that path
 * without any fault. Returns SEP_OK.
 */
int sep_set_wait_limit_ns(unsigned long long ns);

/* Human-readable name of a status code. */
const char* sep_status_string(int status);

/*
 * sep_attn_fwd_noalloc - sep_attn_fwd without a caller workspace and without any allocation.
 *
 * The SepLLM method has no counterpart to this call: it is an engineering variant of
 * sep_attn_fwd (same arguments minus workspace, same kernels, same results). Some callers
 * cannot hand over a workspace: a host whose device memory is all carved out in advance by a
 * pool it owns (a serving engine that reserves HBM for its KV cache at start-up) has no spare
 * buffer to give, and a latency-critical loop cannot call cudaMalloc / cudaFree, which may block
 * on the driver or synchronise the whole device. This call uses instead a fixed array of
 * SEP_NOALLOC_SCRATCH_BYTES that lives in the library's device image, and allocates nothing.
 *
 * Limit: the compacted anchor K and V need 2 * roundup256(B * L * Hkv * d * 2) bytes; a problem
 * above SEP_NOALLOC_SCRATCH_BYTES returns SEP_ERR_SCRATCH_LIMIT before any device work.
 * Setup: the first call on each device (with that device current) looks up the array's device
 * address with cudaGetSymbolAddress, which loads the library's module on that device; make that
 * first call before any stream capture. A failed lookup returns SEP_ERR_CUDA. The address is
 * cached per device for the life of the process: after cudaDeviceReset (or anything else that
 * destroys and recreates the device's primary context) it is stale, so this call must not be
 * used again in that process.
 * Zeroing: none is needed; the compaction writes every row the attention kernel reads (the
 * anchors, then zero rows up to the end of their last 128-row tile).
 * Concurrency: every call on a device shares the one array. Calls that may overlap in time
 * (different streams, or host threads, without ordering between them) race on it and give wrong
 * results; calls in order on one stream are safe.
 */
#define SEP_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)
int sep_attn_fwd_noalloc(const sep_bf16* q, const sep_bf16* k, const sep_bf16* v,
                         int B, int L, int Hq, int Hkv, int d, float scale, int a, int n,
                         const SepMask* mask, sep_bf16* o, float* lse, sep_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* SEPATTN_H_ */
