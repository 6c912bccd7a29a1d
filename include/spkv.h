/*
 * spkv.h -- C ABI of libspkv.so: the hot path of Self-Pruned Key-Value attention
 * (SP-KV) on NVIDIA B200 (sm_100a).
 *
 * Source of the method: "Self-Pruned Key-Value Attention: Learning When to Write
 * by Predicting Future Utility" (arXiv 2605.14037), §2.1:
 *   Eq. (1)  u_s = sigmoid(f(h_s)), f a small two-layer perceptron per layer,
 *            one output per key head;
 *   Eq. (2)  z_s = 1[u_s >= tau];
 *   Eq. (3)  a_{t,s} = softmax(q_t k_s^T / sqrt(d_k) + M_{t,s});
 *   Eq. (4)  M_{t,s} = 0 if 0 <= t-s < w, or z_s = 1 and s <= t; else -inf;
 *   "efficient implementation at deployment": only pairs with z_s = 1 are kept in
 *   a persistent cache; each query attends to that cache plus the local window.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - All tensor pointers are DEVICE pointers owned by the caller.  The library
 *   allocates nothing; the caller provides every buffer (the decode workspace
 *   included) and must keep it alive until the stream work that uses it ends.
 * - Every call enqueues work on `stream` (a cudaStream_t; NULL means the legacy
 *   default stream) and returns without synchronising, except spkv_cache_check.
 * - Return value: SPKV_OK, or an error code.  Arguments are validated on the host
 *   before anything is enqueued; on SPKV_ERR_ARG nothing was enqueued.  Conditions
 *   only the device can see (cache pool exhausted, page table full, a bounded wait
 *   that gave up) set bits of cache->err_flag, read by spkv_cache_check.
 *   No entry point aborts, throws or traps.
 * - Every entry point that enqueues work marks an NVTX range named after itself for
 *   the duration of the host call (visible in Nsight Systems; a no-op call when no
 *   tool is attached).
 * - Element types: `dtype` SPKV_F32 or SPKV_BF16 applies to h, W1, q, k, v, the
 *   cache pool, the ring and the attention output.  b1, W2, b2, u and lse are fp32
 *   in both cases.  Arithmetic is fp32 (bf16 inputs are widened exactly).
 * - Layouts are dense row-major with the shapes given below.  head_dim must be
 *   64 or 128, Hq a multiple of Hkv with Hq/Hkv in {1,2,4,8}, window in [1, 1024],
 *   page_rows 64.  Pointers to tensors must be 16-byte aligned.
 * - Positions are absolute token indices (int32, >= 0; positions given in device
 *   memory, such as t_pos, are not range-checked on the device).  Query head h reads
 *   key head h / (Hq/Hkv) (grouped-query attention).
 * - The decode-step kernels (few-token scoring, retirement, decode attention and its
 *   merge) are launched as programmatic dependents: each may start while the kernel
 *   before it on the stream is finishing, and waits for that kernel to complete before
 *   touching memory it may write.  The perceptron weights (W1, b1, W2, b2) are read
 *   before that wait, so they must not be written by the kernel launched immediately
 *   before a scoring call (weights written earlier on the stream are fine).
 */
#ifndef SPKV_H
#define SPKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef void* spkv_stream_t; /* cudaStream_t */

enum spkv_status {
  SPKV_OK = 0,
  SPKV_ERR_ARG = 1,         /* invalid argument: nothing enqueued */
  SPKV_ERR_CAPACITY = 2,    /* device-detected: pool or page table exhausted */
  SPKV_ERR_CUDA = 3,        /* a CUDA runtime call or a launch failed */
  SPKV_ERR_UNSUPPORTED = 4, /* valid but not built (shape/dtype combination) */
  SPKV_ERR_TIMEOUT = 5,     /* device-detected: a bounded wait gave up */
  SPKV_ERR_INDEX = 6        /* device-detected (debug build): an index check failed */
};

enum spkv_dtype { SPKV_F32 = 0, SPKV_BF16 = 1 };

enum spkv_src_kind {
  SPKV_SRC_CHUNK = 0, /* rows come from a chunk tensor [B][src_batch_rows][Hkv][head_dim] */
  SPKV_SRC_RING = 1   /* rows come from the ring: position p lives in slot p mod window */
};

/* err_flag bits */
#define SPKV_FLAG_POOL_FULL 1u  /* no free page was left for an append */
#define SPKV_FLAG_TABLE_FULL 2u /* a key head reached max_pages_per_head */
#define SPKV_FLAG_TIMEOUT 4u    /* a bounded wait inside a kernel gave up */
#define SPKV_FLAG_INDEX 8u      /* debug build (SPKV_DEBUG): a page number read from a page
                                   table lay outside the pool, or a query position was
                                   negative; the access was skipped or redirected */

/* Shapes of one attention layer. */
typedef struct spkv_params {
  int B;        /* batch rows */
  int Hq;       /* query heads */
  int Hkv;      /* key/value heads */
  int head_dim; /* d_k */
  int d_model;  /* width of h */
  int hid;      /* hidden width of the utility perceptron, <= 128 */
  int window;   /* w of Eq. (4) */
  float tau;    /* threshold of Eq. (2) */
  int dtype;    /* enum spkv_dtype */
} spkv_params;

/* Persistent gated cache of one layer (§2.1, deployment).  Storage is paged:
 * key head kh of batch row b (index bh = b*Hkv + kh) owns the pages listed in
 * page_table[bh][0..], assigned on demand by the device from a bump allocator
 * (pool_top).  Cache row i of head bh is row i % page_rows of page
 * page_table[bh][i / page_rows]; its absolute position is pos_pool at the same
 * place.  Rows are appended in increasing position order. */
typedef struct spkv_cache {
  void* K_pool;        /* [num_pages][page_rows][head_dim] dtype */
  void* V_pool;        /* [num_pages][page_rows][head_dim] dtype */
  int32_t* pos_pool;   /* [num_pages][page_rows] absolute positions */
  int32_t* page_table; /* [B*Hkv][max_pages_per_head], -1 = none */
  int32_t* count;      /* [B*Hkv] rows stored per key head */
  int32_t* count_prev; /* [B*Hkv] value of count before the last chunk append */
  int32_t* pool_top;   /* [1] next free page */
  uint32_t* err_flag;  /* [1] SPKV_FLAG_* bits, sticky until spkv_cache_reset */
  float* u_pool;       /* [num_pages][page_rows] utility u (Eq. (1)) of every stored row, or
                          NULL: utilities are not kept (spkv_cache_rethreshold needs them) */
  int num_pages;
  int page_rows; /* must be 64 */
  int max_pages_per_head;
} spkv_cache;

/* Local window (Eq. (4), 1_win): the last `window` keys/values of every
 * (batch row, key head), position p in slot p % window; z_win holds the gate of
 * the token in each slot (for retirement into the cache).  u_win (optional) holds
 * the utility of a slot's token while its retirement is pending, and NaN (all bits
 * set) when the token is not pending (already cached, or not yet scored). */
typedef struct spkv_ring {
  void* K_win;    /* [B][Hkv][window][head_dim] dtype */
  void* V_win;    /* [B][Hkv][window][head_dim] dtype */
  uint8_t* z_win; /* [B][window][Hkv] */
  float* u_win;   /* [B][window][Hkv] f32, or NULL */
} spkv_ring;

/* Static text for a status code. */
const char* spkv_status_str(int status);

/* Library version (major*10000 + minor*100 + patch). */
int spkv_version(void);

/* Zero the cache (count, count_prev, pool_top, err_flag), set page_table to -1
 * and, if ring is not NULL, zero its z_win and set its u_win (if any) to NaN. */
int spkv_cache_reset(const spkv_params* p, const spkv_cache* cache, const spkv_ring* ring,
                     spkv_stream_t stream);

/* Synchronise `stream`, copy err_flag to *flags_out (if not NULL) and return
 * SPKV_ERR_CAPACITY if a pool/table bit is set, SPKV_ERR_TIMEOUT if the timeout
 * bit is set, SPKV_ERR_INDEX if the index bit is set, else SPKV_OK. */
int spkv_cache_check(const spkv_cache* cache, spkv_stream_t stream, uint32_t* flags_out);

/* a1 -- utility score and gate, Eqs. (1)-(2), fused:
 *   a = h W1^T + b1;  x = GELU(a) (exact erf form);  l = x W2^T + b2;
 *   u = sigmoid(l);   z = 1[u >= tau]   for every token and key head.
 * h [n_tok][d_model] dtype; W1 [hid][d_model] dtype; b1 [hid] f32;
 * W2 [Hkv][hid] f32; b2 [Hkv] f32.  Outputs u_out [n_tok][Hkv] f32 (may be
 * NULL) and z_out [n_tok][Hkv] uint8.  n_tok >= 0 (0 enqueues nothing). */
int spkv_score(const spkv_params* p, const void* h, int n_tok, const void* W1, const float* b1,
               const float* W2, const float* b2, float* u_out, uint8_t* z_out,
               spkv_stream_t stream);

/* a2 -- stream compaction (§2.1 deployment): for every (b, key head), append the
 * rows i in [0, n_rows) with z = 1, in increasing i, to the cache, recording
 * position src_pos[b] + i (and utility u[b][i][kh] when cache->u_pool is set).
 *   src_kind SPKV_SRC_CHUNK: K_src/V_src [B][src_batch_rows][Hkv][head_dim];
 *   src_kind SPKV_SRC_RING: rows are read from ring->K_win/V_win (K_src/V_src
 *     ignored), row i of batch b from slot (src_pos[b] + i) % window; requires
 *     n_rows <= window.
 * z [B][src_batch_rows][Hkv] uint8, u [B][src_batch_rows][Hkv] f32 (required when
 * cache->u_pool is not NULL, else ignored); src_pos [B] int32; all device.
 * Positions must exceed those already stored for that head.  Rows that do not fit
 * are dropped and flagged in err_flag.  Two kernels: plan (page allocation), then
 * scatter. */
int spkv_write_compact(const spkv_params* p, const spkv_cache* cache, const spkv_ring* ring,
                       int src_kind, const void* K_src, const void* V_src, const uint8_t* z,
                       const float* u, const int32_t* src_pos, int n_rows, int src_batch_rows,
                       spkv_stream_t stream);

/* a2 + a3 for one decode step per batch row (per-token retirement): with
 * t = t_pos[b], if retire != 0 and t - window >= 0, the token s = t - window
 * leaves the window; it is appended to the cache if its gate (ring->z_win of its
 * slot) is 1 (with its utility from ring->u_win when cache->u_pool is set).  Then
 * k_new, v_new (and z_new, if not NULL; else 0) are stored in slot t % window, and
 * u_new in ring->u_win if that is set (NaN when z_new is NULL).  k_new, v_new
 * [B][Hkv][head_dim] dtype; z_new [B][Hkv] uint8; u_new [B][Hkv] f32 (required when
 * ring->u_win and z_new are set); t_pos [B] int32, all device.  cache may be NULL for
 * a window-only layer (a local layer of a hybrid local/global stack, §3.3
 * "Hybrids": it keeps no long-range cache); retire must then be 0. */
int spkv_decode_append(const spkv_params* p, const spkv_cache* cache, const spkv_ring* ring,
                       const int32_t* t_pos, const void* k_new, const void* v_new,
                       const uint8_t* z_new, const float* u_new, int retire,
                       spkv_stream_t stream);

/* Flag of spkv_decode_score_append: h was written by work that had completed before
 * the kernel enqueued just before this call on `stream` started (e.g. the step's inputs,
 * copied in ahead of the step).  The perceptron then runs while that kernel finishes;
 * the ring and cache, which it may still read, are touched only after it ends. */
#define SPKV_INPUTS_SETTLED 1u

/* a1 + a2 + a3 fused for one per-token decode step: the same result as spkv_score on
 * the B new tokens (h [B][d_model], one per batch row, at positions t_pos) followed by
 * spkv_decode_append(..., z_new = z_out, u_new = u_out, retire = 1).  The warp that finishes the gate
 * of (batch row b, key head kh) also retires token t-window of (b, kh) and stores the
 * new token, so the step costs one launch.  u_out [B][Hkv] (may be NULL), z_out
 * [B][Hkv] as in spkv_score; k_new, v_new [B][Hkv][head_dim].  flags: 0 or
 * SPKV_INPUTS_SETTLED (other bits: SPKV_ERR_ARG). */
int spkv_decode_score_append(const spkv_params* p, const spkv_cache* cache, const spkv_ring* ring,
                             const int32_t* t_pos, const void* h, const void* W1, const float* b1,
                             const float* W2, const float* b2, const void* k_new,
                             const void* v_new, float* u_out, uint8_t* z_out, unsigned flags,
                             spkv_stream_t stream);

/* a1 for one per-token decode step, kept off the attention's critical path: the
 * utility and gate of the B new tokens (h [B][d_model], the token of batch row b at
 * position t_pos[b]) exactly as spkv_score computes them, each gate (and utility, if
 * ring->u_win is set) stored in its token's window slot t_pos[b] % window.  Use it after
 * spkv_decode_append(..., z_new = NULL, u_new = NULL, retire = 1) of the same step
 * (which retires token t - window and stores the new token with gate 0).  The gate of a
 * token is read only when it leaves the window, so this call may run on another stream
 * while spkv_decode_attn of the step (and later layers) proceed; it must finish before
 * the step that retires the token.  u_out [B][Hkv] f32 (required when ring->u_win is
 * set, else may be NULL), z_out [B][Hkv] uint8. */
int spkv_decode_score(const spkv_params* p, const spkv_ring* ring, const int32_t* t_pos,
                      const void* h, const void* W1, const float* b1, const float* W2,
                      const float* b2, float* u_out, uint8_t* z_out, spkv_stream_t stream);

/* a3 -- store the last min(n_rows, window) rows of a chunk in the ring: row i of
 * batch b (position src_pos[b] + i) goes to slot (src_pos[b] + i) % window.  The
 * slot's gate is 0 for rows i < gated_from (already in the cache, so retiring them
 * appends nothing) and z_src[b][i][kh] for the others (z_src may be NULL when
 * gated_from >= n_rows); ring->u_win, if set, gets NaN for the former and
 * u_src[b][i][kh] for the latter (u_src is then required when gated_from < n_rows).
 * K_src/V_src [B][src_batch_rows][Hkv][head_dim], z_src [B][src_batch_rows][Hkv],
 * u_src [B][src_batch_rows][Hkv] f32. */
int spkv_ring_write(const spkv_params* p, const spkv_ring* ring, const void* K_src,
                    const void* V_src, const uint8_t* z_src, const float* u_src, int gated_from,
                    const int32_t* src_pos, int n_rows, int src_batch_rows, spkv_stream_t stream);

/* Bytes of decode workspace spkv_decode_attn needs for this cache geometry.  The
 * workspace must be zero-filled once before its first use; the library leaves
 * its counters at zero after every call.  Calls that share a workspace must not
 * overlap on the device. */
size_t spkv_decode_workspace_bytes(const spkv_params* p, const spkv_cache* cache);

/* a4 + a5 -- gated decode attention, Eqs. (3)-(4), one query per batch row:
 * query t = t_pos[b] attends to the window slots holding positions
 * max(0, t-window+1)..t and to the cache rows with position <= t - window.
 * Split-K over balanced chunks of rows (a5: the chunk partials of a head are
 * combined by their log-sum-exp weights in a second kernel on the same stream).
 * q [B][Hq][head_dim] dtype; o [B][Hq][head_dim] dtype; lse [B][Hq] f32 natural
 * log (may be NULL).  The token t itself must already be in the ring.  cache may be
 * NULL: a window-only layer (the local layers of a hybrid stack, §3.3 "Hybrids"),
 * whose keys are the window slots alone. */
int spkv_decode_attn(const spkv_params* p, const spkv_cache* cache, const spkv_ring* ring,
                     const void* q, const int32_t* t_pos, void* o, float* lse, void* workspace,
                     size_t ws_bytes, spkv_stream_t stream);

/* a4 + a5 before the step's retirement and ring write -- the same attention as
 * spkv_decode_attn (Eqs. (3)-(4) at query t = t_pos[b]), taken from the state the
 * cache and ring are in BEFORE spkv_decode_append of this step:
 *   - the ring holds positions max(0, t-window) .. t-1; the slot t % window (position
 *     t - window, which leaves the window at query t and belongs to the cache from
 *     now on, Eq. (4)) counts iff its stored gate ring->z_win is 1;
 *   - cache rows count up to position t - window - 1;
 *   - the new token t is k_new / v_new [B][Hkv][head_dim] dtype (the rows the step's
 *     spkv_decode_append will store).
 * This is the state of the per-token schedule: no row still in the window has been
 * compacted into the cache (the cache holds positions <= t - window - 1 only) and every
 * window slot holds its token's gate.  A schedule that compacts window rows early (bulk
 * scoring from the ring, or a prefill that compacts every row of its last chunk) must
 * use spkv_decode_attn instead.
 * The step's spkv_decode_append (and spkv_decode_score) may then run after this call,
 * off the attention's path: they must start after it has finished (they overwrite
 * slot t % window) and finish before the next step's call on the same layer.  Same
 * workspace, q, o and lse as spkv_decode_attn; ring->z_win is required; cache may be
 * NULL (window-only layer).  Returns SPKV_ERR_UNSUPPORTED where
 * spkv_decode_attn_before_append_supported says 0.
 * flags: 0, or SPKV_DECODE_STATE_SETTLED -- the caller vouches that t_pos and every
 * part of this cache and ring (counts, page table, positions, rows, gates) were last
 * written by work that completes before this call's place on the stream without a
 * programmatic launch in between: written on another stream joined to this one by an
 * event, or followed on this stream by an event wait, a copy or a kernel of the
 * caller's own.  The kernel then plans its chunks from them, and reads its first
 * page-table entries, while the kernel before it on the stream is still finishing;
 * q, k_new, v_new and the workspace are still accessed only after that kernel has
 * completed.  Any other flag bit is an argument error. */
#define SPKV_DECODE_STATE_SETTLED 1u
int spkv_decode_attn_before_append(const spkv_params* p, const spkv_cache* cache,
                                   const spkv_ring* ring, const void* q, const int32_t* t_pos,
                                   const void* k_new, const void* v_new, void* o, float* lse,
                                   void* workspace, size_t ws_bytes, unsigned flags,
                                   spkv_stream_t stream);

/* 1 if spkv_decode_attn_before_append runs for these parameters (bf16, head_dim 64 or
 * 128, window a multiple of 64), else 0.  Host only; enqueues nothing. */
int spkv_decode_attn_before_append_supported(const spkv_params* p);

/* Sequence split (decode over slices of one sequence's keys, combined afterwards).
 *
 * A sequence whose gated cache is spread over several caches (for instance over
 * several GPUs: each holds the cache rows of a range of positions, one of them also
 * the window) is decoded slice by slice and the slices' partials are combined.  The
 * combination rests on Eq. (3) ("Self-Pruned Key-Value Attention", §2.1): the softmax
 * over a disjoint union of key sets S_1..S_n factorises, so with o_i the attention
 * output over S_i alone and lse_i the log of its sum of exponentials,
 *   lse = log sum_i e^{lse_i},  o = sum_i e^{lse_i - lse} o_i
 * is the attention over the whole set (the log-sum-exp merge that also combines the
 * split-K chunks of one decode call). */

/* flags of spkv_decode_attn_partial */
#define SPKV_SLICE_WINDOW 1u /* this slice holds the window: the ring is read */

/* a4 over one slice: for query t = t_pos[b] (as in spkv_decode_attn, after the step's
 * update), the keys of this slice are the cache rows with position <= t - window and,
 * with SPKV_SLICE_WINDOW, the window slots holding positions max(0, t-window+1)..t.
 * Outputs (fp32): o_part [B][Hq][head_dim], the attention output over the slice's keys
 * alone, and lse_part [B][Hq], the natural log of the slice's sum of exponentials of
 * the scaled logits; a head with no key in the slice gets o_part = 0, lse_part = -inf.
 * cache may be NULL for a slice that holds only the window; without SPKV_SLICE_WINDOW
 * the cache is required and ring is ignored (may be NULL).  Each cache must hold
 * distinct positions (the slices are disjoint), each in increasing order.  q
 * [B][Hq][head_dim] dtype; workspace as for spkv_decode_attn
 * (spkv_decode_workspace_bytes; calls sharing a workspace must not overlap).  Returns
 * SPKV_ERR_UNSUPPORTED where spkv_decode_attn_partial_supported says 0. */
int spkv_decode_attn_partial(const spkv_params* p, const spkv_cache* cache,
                             const spkv_ring* ring, const void* q, const int32_t* t_pos,
                             unsigned flags, float* o_part, float* lse_part, void* workspace,
                             size_t ws_bytes, spkv_stream_t stream);

/* 1 if spkv_decode_attn_partial runs for these parameters (bf16, head_dim 64 or 128,
 * window a multiple of 64), else 0.  Host only. */
int spkv_decode_attn_partial_supported(const spkv_params* p);

/* a5 across slices: combine n_parts >= 1 slice partials of the same queries.
 * o_parts [n_parts][B][Hq][head_dim] f32 and lse_parts [n_parts][B][Hq] f32 (as
 * spkv_decode_attn_partial writes them; parts in any order) -> o [B][Hq][head_dim]
 * dtype and lse [B][Hq] f32 natural log (may be NULL).  Parts with lse = -inf count
 * for nothing; if every part is empty, o = 0 and lse = -inf. */
int spkv_decode_merge(const spkv_params* p, int n_parts, const float* o_parts,
                      const float* lse_parts, void* o, float* lse, spkv_stream_t stream);

/* Size of the fixed device scratch used by spkv_decode_attn_noalloc (8 MiB).  Every
 * GPU on which the library is loaded keeps this much memory until the process exits. */
#define SPKV_NOALLOC_SCRATCH_BYTES (8u << 20)

/* Gated decode attention without a caller-provided workspace.  The SP-KV paper has
 * no counterpart: this is a deployment convenience of this library.
 *
 * spkv_decode_attn needs scratch memory for its split partials and counters, which
 * the caller must allocate.  Some callers cannot: code running inside a host that
 * owns all device memory through its own pool, a serving path that must not call
 * cudaMalloc after start-up, or a runtime with no allocator to borrow from.  This
 * entry point computes exactly what spkv_decode_attn computes (same arguments minus
 * the workspace, the same argument checks, same kernels; cache may be NULL for a
 * window-only layer) but takes its scratch from a fixed array of
 * SPKV_NOALLOC_SCRATCH_BYTES inside the library.  It allocates and frees nothing.
 *
 * - Shapes whose scratch need (spkv_decode_workspace_bytes) exceeds the fixed size
 *   are rejected with SPKV_ERR_UNSUPPORTED before anything is enqueued.
 * - The first call in a CUDA context (per device; again after a device reset, which
 *   makes a new context) looks up the array's device address with that context
 *   current; make that first call before any stream capture.
 * - Every call shares the one array, whatever its shape: each call clears the counters
 *   of its own shape at the start, on `stream` (one memset before the kernels, which
 *   also keeps the first kernel from overlapping the previous kernel on the stream).
 *   Calls whose work overlaps on the device (other streams, concurrent graph
 *   branches) race on the scratch and must not be issued. */
int spkv_decode_attn_noalloc(const spkv_params* p, const spkv_cache* cache,
                             const spkv_ring* ring, const void* q, const int32_t* t_pos,
                             void* o, float* lse, spkv_stream_t stream);

/* Bytes of the optional workspace of spkv_prefill_attn (a tile counter). */
#define SPKV_PREFILL_WORKSPACE_BYTES 256

/* a6 -- gated prefill attention, Eqs. (3)-(4), for the chunk of queries at
 * positions chunk_start .. chunk_start+chunk_len-1 of every batch row.  Keys:
 * the window, from K_chunk/V_chunk (positions >= chunk_start) and from the ring
 * (earlier positions, which must hold the previous chunk's last rows), and the
 * cache rows with position <= t - window (the cache may already hold rows of
 * this chunk; those are used only by queries they have left the window of).
 * q [B][chunk_len][Hq][head_dim]; K_chunk, V_chunk [B][chunk_len][Hkv][head_dim];
 * o [B][chunk_len][Hq][head_dim]; lse [B][chunk_len][Hq] f32 (may be NULL).  cache
 * may be NULL for a window-only layer.
 * workspace: NULL, or at least SPKV_PREFILL_WORKSPACE_BYTES (ws_bytes) of 16-byte
 * aligned device memory, zero-filled once before its first use; the library leaves it
 * zeroed after every call.  With it, the tensor-core path hands out its 128-query tiles
 * heaviest first to whichever CTA is free (cache densities differ per key head, so no
 * fixed order balances them); without it, a fixed order is used.  Calls sharing a
 * workspace must not overlap. */
int spkv_prefill_attn(const spkv_params* p, const spkv_cache* cache, const spkv_ring* ring,
                      const void* q, const void* K_chunk, const void* V_chunk, int chunk_start,
                      int chunk_len, void* o, float* lse, void* workspace, size_t ws_bytes,
                      spkv_stream_t stream);

/* Bytes of workspace spkv_cache_rethreshold needs for this cache geometry.  The
 * workspace must be zero-filled once before its first use; the library leaves its
 * counters at zero after every call.  Calls sharing a workspace must not overlap. */
size_t spkv_rethreshold_workspace_bytes(const spkv_params* p, const spkv_cache* cache);

/* Post-hoc re-threshold ("Self-Pruned Key-Value Attention", §3.3: at inference the
 * sparsity can be changed after the fact by changing the threshold): every key head
 * keeps exactly its cache rows whose stored utility satisfies u >= tau_new, in their
 * order (an in-place stable compaction inside the head's pages), and count and
 * count_prev become the kept count.  Rows removed earlier are not recovered, so a
 * tau_new below the threshold the rows were gated with removes nothing.  Pages a head
 * no longer fills stay in its page list and are reused by its later appends (they
 * are not returned to the pool).  If ring and ring->u_win are set, every slot's gate
 * becomes z = 1[u_win >= tau_new] (NaN slots: 0), so the tokens still in the window
 * retire under the new threshold; later scoring should be given tau_new in p.
 * Requires cache->u_pool.  Three kernels (plan, move, finish); a bounded wait inside
 * the move kernel that gives up latches SPKV_FLAG_TIMEOUT and skips the writes of its
 * page, and the call's later waits then give up at once (those pages are skipped too). */
int spkv_cache_rethreshold(const spkv_params* p, const spkv_cache* cache, const spkv_ring* ring,
                           float tau_new, void* workspace, size_t ws_bytes,
                           spkv_stream_t stream);

/* Diagnostics, for testing failure reporting: the limit, in nanoseconds, of the bounded
 * waits of spkv_cache_rethreshold's move kernel on the "page read" flags of other CTAs
 * (default 2 s; 0 restores it).  A wait that runs out latches SPKV_FLAG_TIMEOUT and the
 * rows bound for the unread page are not written.  Process-wide; applies to calls
 * enqueued afterwards.  No other wait of the library is affected. */
int spkv_debug_set_flag_wait_ns(unsigned long long ns);

/* Bytes of workspace spkv_soft_attn needs (a per-key bias buffer). */
size_t spkv_soft_attn_workspace_bytes(const spkv_params* p, int seq_len);

/* Soft-gated attention of SP-KV training ("Self-Pruned Key-Value Attention", §2.1,
 * soft relaxation at training time), forward pass over whole sequences:
 *   alpha_s = sigmoid((u_s - tau) / beta)                                  (Eq. (5))
 *   M(t,s)  = 0 if 0 <= t-s < window, c (alpha_s - 1) if s <= t-window,
 *             -inf if s > t                                                 (Eq. (6))
 *   o_t     = softmax_s(q_t . k_s / sqrt(head_dim) + M(t,s)) v_s             (Eq. (3))
 * for every batch row, query head and position t < seq_len (GQA grouping as
 * elsewhere; tau and window from p).  No key is skipped: this is the dense training
 * form; the backward pass is not provided.
 * q [B][seq_len][Hq][head_dim], K, V [B][seq_len][Hkv][head_dim] dtype, u
 * [B][seq_len][Hkv] f32 (e.g. from spkv_score), o like q, lse [B][seq_len][Hq] f32
 * natural log (may be NULL).  workspace: spkv_soft_attn_workspace_bytes, no
 * initialisation needed.  beta > 0, c >= 0.  err_flag (may be NULL) latches
 * SPKV_FLAG_TIMEOUT if a bounded wait inside the kernel gives up. */
int spkv_soft_attn(const spkv_params* p, const void* q, const void* K, const void* V,
                   const float* u, int seq_len, float beta, float c, void* o, float* lse,
                   void* workspace, size_t ws_bytes, uint32_t* err_flag, spkv_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* SPKV_H */
