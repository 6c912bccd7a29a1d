// decode_tc.cu -- a4 + a5 for bf16: gated decode attention, split-K over balanced
// chunks, with tensor-core tiles for the per-group dot products.
//
// "Self-Pruned Key-Value Attention" (arXiv 2605.14037), §2.1, Eqs. (3)-(4): query t
// of every (batch row, key head) attends to the window slots and to the cache rows
// with pos <= t - w; decode reads that whole key set once per step (memory bound,
// §3.4).  On CUDA cores the G-head dot products cost ~90 instructions per 512-byte
// K/V row (widening, FMAs, cross-lane reductions) and leave HBM half idle; here the
// G query heads of a group are the rows of a 16-row MMA tile, so the same bytes cost
// a few instructions and the kernel is left bound by HBM.
//
// Structure (one CTA per SM, 6 warps: 4 consumers, a producer, a finisher):
//  * Plan (every CTA, same result): live cache rows per head, rows rounded to 64-row
//    tiles (cache pages), chunk size so that all heads give about 4 chunks per CTA,
//    chunk prefix.  Each CTA's first chunk is its own index; the producer pulls later
//    chunks from a global atomic counter, so ragged heads balance.
//  * Producer warp: per chunk, its lanes fetch all the chunk's page-table entries at
//    once into shared memory; then one lane streams 64-row tiles (TMA boxes of
//    64 rows x 64 bf16, 128B-swizzled) of K and V from the cache pages or the ring
//    into a 4-stage ring of shared memory, the chunk's G query rows riding along with
//    its first tile (bulk copy).  Four queued tiles cover the next chunk's fetches.
//  * 4 consumer warps, 16 rows of each tile apiece: S = Q K^T with mma.m16n8k16 (Q rows
//    = the G heads, zero-padded to 16), fp32 softmax in the log2 domain (running max
//    raised only when exceeded by > 8), P re-packed in registers as the A operand of
//    O += P V (V via ldmatrix.trans).
//  * Chunk end: the consumer warps hand their partials to the finisher warp through
//    double-buffered shared slots and go on with the next chunk; the finisher combines
//    them: a head with one chunk gets its o and lse written, otherwise the chunk's
//    (o, m, l) partial goes to the workspace.
//  * decode_merge_kernel (one CTA per head, launched next on the same stream as a
//    programmatic dependent; heads with one chunk return at once) combines the
//    partials: o = sum_i 2^{m_i-m} o_i / sum_i 2^{m_i-m} l_i, and resets the work counter
//    for the next call.  A second launch costs less than the decode CTAs waiting on an
//    arrival count at the end of every head.
//  * Before-append mode (k_new given): the step's retirement and ring write have not
//    run yet.  The ring then holds rows t-w .. t-1; slot t mod w (row t - w, which
//    leaves the window at query t) counts only if its stored gate is 1, cache rows
//    count up to pos t - w - 1, and the new row t is folded into the head's last
//    chunk by the finisher as one more (m, l, o) term.  The retirement and ring write
//    can then run after the attention, off its path.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math.h>

#include <mutex>
#include <type_traits>

#include "common.cuh"
#include "host.h"
#include "launch.h"

namespace spkv {
namespace {

constexpr int kTileR = 64;           // rows per tile (one cache page)
constexpr int kCons = 4;             // consumer warps, 16 rows each
constexpr int kThreadsT = (kCons + 2) * 32;   // + producer + finisher
constexpr int kMergeThreads = 512;   // merge CTA when heads average many chunks
constexpr int kMergeThreadsFew = 128;
constexpr int kConsThreads = kCons * 32;
constexpr int kStagesT = 4;
constexpr int kUnitsPerCta = 4;      // target chunks per CTA
constexpr int kMaxHeadsT = 2048;
constexpr int kChunkPages = 256;     // page numbers staged per fetch
constexpr int kPgRegs = kChunkPages / 32;
constexpr int kLookClaim = 4;        // tiles before a chunk's end: claim the next chunk
constexpr int kLookPages = 2;        // ... and fetch its page-table entries
constexpr int kMergeBatch = 16;      // partials a merge thread loads at once
constexpr float kLog2eT = 1.4426950408889634f;
constexpr float kLn2T = 0.6931471805599453f;
constexpr float kSlackT = 8.f;

template <int D>
struct TileBuf {
  static constexpr int kHalves = D / 64;
  static constexpr int kHalfBytes = kTileR * 128;       // 64 rows x 128 B
  static constexpr int kBytes = kHalves * kHalfBytes;   // K (or V) of one tile
  alignas(1024) char k[kHalves][kHalfBytes];
  alignas(1024) char v[kHalves][kHalfBytes];
};

struct TileRef {
  int chunk;  // -1: no more work
  int bh;
  int valid;  // valid rows
  int last;   // last tile of its chunk
  int qslot;  // query staging slot of the chunk
  int hide;   // row of the tile that does not count (-1: none)
};

template <int D, int G>
struct TcDecSmem {
  TileBuf<D> st[kStagesT];
  alignas(16) __nv_bfloat16 qbuf[2][G * D];
  float red_o[2][kCons][G][D];  // per-warp chunk partials, two chunks in flight
  float red_m[2][kCons][G];
  float red_l[2][kCons][G];
  int fin_chunk[2];
  int fin_bh[2];
  uint64_t cdone[2];   // consumers -> finisher: a chunk's partials are in red_*[parity]
  uint64_t cfree[2];   // finisher -> consumers: red_*[parity] may be rewritten
  int pages[kChunkPages];
  uint64_t full[kStagesT];
  uint64_t empty[kStagesT];
  uint64_t q_free[2];
  TileRef info[kStagesT];
  int red[kThreadsT];
  int misc[4];
  // followed (dynamic) by rows[n_heads], live[n_heads], nw[n_heads], hide[n_heads],
  // base[n_heads + 1]
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// D = A(16x16, rows lane/4 and lane/4+8) * B(16x8) + D, bf16 in, fp32 accumulate.
__device__ __forceinline__ void mma16816(float* d, uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Two bf16 (low half first) widened to fp32 (exact: a bf16 is the top half of an fp32).
__device__ __forceinline__ float2 bf2_to_f2(uint32_t x) {
  return make_float2(__uint_as_float(x << 16), __uint_as_float(x & 0xffff0000u));
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

__device__ __forceinline__ void tma2d(void* dst, const CUtensorMap* map, int c0, int c1, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tma4d(void* dst, const CUtensorMap* map, int c0, int c1, int c2,
                                      int c3, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_u32(bar))
      : "memory");
}

// Byte offset of 16-byte chunk `c` (0..7) of row `r` in a 128B-swizzled half tile.
__device__ __forceinline__ uint32_t swz(int r, int c) {
  return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4));
}

// One chunk of one head's key rows, in 64-row tiles: cache tiles k0 .. kc1-1 (page
// list order), then the window slots.
struct ChunkDesc {
  int c;    // chunk id (>= total: no more work)
  int bh;   // head: b * hkv + kh
  int k0, k1, kc1;
  int nl, nlp, nw;  // live cache rows, rounded up to tiles, window rows
  int hide;         // window slot that does not count (-1: none)
};

__device__ __forceinline__ ChunkDesc describe_chunk(int c, int total, int chunk_rows,
                                                    const int* s_base, const int* s_rows,
                                                    const int* s_live, const int* s_nw,
                                                    const int* s_hide, int n_heads, int hkv) {
  ChunkDesc d;
  d.c = c;
  if (c >= total) {
    d.bh = d.k0 = d.k1 = d.kc1 = d.nl = d.nlp = d.nw = 0;
    d.hide = -1;
    return d;
  }
  int lo = 0, hi = n_heads - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s_base[mid] <= c) lo = mid; else hi = mid - 1;
  }
  d.bh = lo;
  const int r0 = (c - s_base[lo]) * chunk_rows;
  const int r1 = min(s_rows[lo], r0 + chunk_rows);
  d.nl = s_live[lo];
  d.nlp = ((d.nl + kTileR - 1) / kTileR) * kTileR;
  d.nw = s_nw[lo];
  d.hide = s_hide[lo];
  d.k0 = r0 / kTileR;
  d.k1 = (r1 + kTileR - 1) / kTileR;
  d.kc1 = min(d.k1, d.nlp / kTileR);
  return d;
}

// Page numbers of a chunk's first kChunkPages cache tiles, lane-strided into registers
// (the loads stay in flight until the registers are stored to shared memory).
__device__ __forceinline__ void fetch_pages(int (&pg)[kPgRegs], const ChunkDesc& d,
                                            const CacheView& cache, int lane) {
#pragma unroll
  for (int j = 0; j < kPgRegs; ++j) {
    const int k = d.k0 + lane + 32 * j;
    pg[j] = k < d.kc1 ? __ldcg(cache.page_table + (size_t)d.bh * cache.max_pages + k) : 0;
  }
}

template <int D, int G, bool F32OUT>
__global__ void __launch_bounds__(kThreadsT, 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tm_kp,
                     const __grid_constant__ CUtensorMap tm_vp,
                     const __grid_constant__ CUtensorMap tm_kr,
                     const __grid_constant__ CUtensorMap tm_vr, CacheView cache,
                     const __nv_bfloat16* __restrict__ q, const int32_t* __restrict__ t_pos,
                     void* __restrict__ out_, float* __restrict__ lse_out,
                     int* __restrict__ ws_ctrl, float* __restrict__ ws_ml,
                     float* __restrict__ ws_o, int n_heads, int hkv, int window,
                     uint32_t* err, const __nv_bfloat16* __restrict__ k_new,
                     const __nv_bfloat16* __restrict__ v_new, const uint8_t* __restrict__ z_win,
                     int early_plan, int win_on) {
  using TB = TileBuf<D>;
  using OutT = typename std::conditional<F32OUT, float, __nv_bfloat16>::type;
  OutT* __restrict__ out = static_cast<OutT*>(out_);
  using S = TcDecSmem<D, G>;
  constexpr int NT_D = D / 8;     // n-tiles of 8 along head_dim
  constexpr int KS_D = D / 16;    // k-steps of 16 along head_dim
  extern __shared__ __align__(1024) char smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  S& sm = *reinterpret_cast<S*>(smem_raw + pad);
  int* s_rows = reinterpret_cast<int*>(smem_raw + pad + sizeof(S));
  int* s_live = s_rows + n_heads;
  int* s_nw = s_live + n_heads;
  int* s_hide = s_nw + n_heads;
  int* s_base = s_hide + n_heads;
  const bool pre = k_new != nullptr;  // before the step's retirement and ring write
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int* next_chunk = ws_ctrl + n_heads;  // reset by the merge kernel

  if (tid == 0) {  // descriptor fetches overlap the wait below
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_kp)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_vp)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_kr)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_vr)) : "memory");
  }
  // the merge kernel may be scheduled now (it waits for this grid to complete).  The
  // cache counts and the ring may be written by the kernel before this one, unless the
  // caller vouched that they are settled: then the plan and the producer's first
  // page-table reads, which touch only them and the positions, run before the wait,
  // while the previous kernel finishes.  The consumer warps read shared memory only.
  grid_dependents_launch();
  if (!early_plan) grid_dependency_wait();

  // ---- plan (identical in every CTA) ---------------------------------------------
  int my_rows = 0;
  for (int bh = tid; bh < n_heads; bh += kThreadsT) {
    const int b = bh / hkv;
    const int t = checked_position(__ldcg(t_pos + b), err);
    int nl, nw, hide = -1;
    if (!pre) {
      nl = cache_live_rows(cache, bh, t - window, window);
      nw = !win_on ? 0 : t + 1 < window ? t + 1 : window;
    } else {  // ring rows t-w .. t-1; row t - w (slot t mod w) counts if its gate is 1
      // before the step's update the per-token schedule's cache holds positions up to
      // t - w - 1 only (the entry point's precondition): every stored row is live
      nl = cache.count ? __ldcg(cache.count + bh) : 0;
      nw = t < window ? t : window;
      if (t >= window && __ldcg(z_win + ((size_t)b * window + t % window) * hkv + bh % hkv) == 0)
        hide = t % window;
    }
    int rows = ((nl + kTileR - 1) / kTileR) * kTileR + nw;
    // a head with no key here (before-append mode at t = 0, or a slice of a split
    // sequence without rows for it) gets one empty tile: nothing is loaded or computed
    // for it, and its chunk carries the new row or writes the empty partial (o = 0,
    // lse = -inf)
    if (rows == 0) rows = 1;
    s_live[bh] = nl;
    s_nw[bh] = nw;
    s_hide[bh] = hide;
    s_rows[bh] = rows;
    my_rows += rows;
  }
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) my_rows += __shfl_xor_sync(0xffffffffu, my_rows, m);
  if (lane == 0) sm.red[warp] = my_rows;
  if (tid == 0) {
    for (int s = 0; s < kStagesT; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], kCons);
    }
    mbar_init(&sm.q_free[0], kCons);
    mbar_init(&sm.q_free[1], kCons);
    mbar_init(&sm.cdone[0], kConsThreads);
    mbar_init(&sm.cdone[1], kConsThreads);
    mbar_init(&sm.cfree[0], 1);
    mbar_init(&sm.cfree[1], 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (tid == 0) {
    long long total = 0;
    for (int w = 0; w < kThreadsT / 32; ++w) total += sm.red[w];
    const long long units = (long long)gridDim.x * kUnitsPerCta;
    long long cr = (total + units - 1) / units;
    cr = ((cr + kTileR - 1) / kTileR) * kTileR;
    sm.misc[0] = (int)(cr < kTileR ? kTileR : cr);
  }
  __syncthreads();
  const int chunk_rows = sm.misc[0];
  {
    // chunks per head, exclusive prefix over heads: thread segments, warp shuffle scan
    const int per = (n_heads + kThreadsT - 1) / kThreadsT;
    const int lo = tid * per, hi = min(n_heads, lo + per);
    int s = 0;
    for (int bh = lo; bh < hi; ++bh) s += (s_rows[bh] + chunk_rows - 1) / chunk_rows;
    int inc = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += v;
    }
    if (lane == 31) sm.red[warp] = inc;
    __syncthreads();
    int before = 0, total = 0;
#pragma unroll
    for (int w = 0; w < kThreadsT / 32; ++w) {
      const int v = sm.red[w];
      before += w < warp ? v : 0;
      total += v;
    }
    int acc = before + inc - s;
    for (int bh = lo; bh < hi; ++bh) {
      s_base[bh] = acc;
      acc += (s_rows[bh] + chunk_rows - 1) / chunk_rows;
    }
    if (tid == 0) s_base[n_heads] = total;
  }
  __syncthreads();
  const int total_chunks = s_base[n_heads];

  if (warp == kCons) {
    // ------------------------------ producer ------------------------------------
    // The whole warp walks the tiles; lane 0 issues the copies.  The next chunk is
    // claimed kLookClaim tiles before the current one ends and its page-table entries
    // are fetched into registers kLookPages tiles before the end, so neither the
    // global atomic nor the page-table read stalls the stage ring between chunks.
    int it = 0;
    const int c = blockIdx.x;  // first chunk: static; later ones from the counter
    ChunkDesc cd = describe_chunk(c, total_chunks, chunk_rows, s_base, s_rows, s_live, s_nw,
                                  s_hide, n_heads, hkv);
    int pg[kPgRegs];
    fetch_pages(pg, cd, cache, lane);
    // with a settled state the plan and the first page-table reads above ran while the
    // previous kernel finished; the queries and the work counter come after the wait
    if (early_plan) grid_dependency_wait();
    for (int seq = 0; cd.c < total_chunks; ++seq) {
      __syncwarp();
#pragma unroll
      for (int j = 0; j < kPgRegs; ++j) sm.pages[lane + 32 * j] = pg[j];
      __syncwarp();
      const int qslot = seq & 1;
      if (lane == 0) mbar_wait(&sm.q_free[qslot], ((seq >> 1) & 1) ^ 1, err);
      int c_next = 0;
      ChunkDesc nd;
      nd.c = total_chunks;
      const int k_claim = max(cd.k0, cd.k1 - kLookClaim);
      const int k_pages = max(cd.k0, cd.k1 - kLookPages);
      for (int k = cd.k0; k < cd.k1; ++k, ++it) {
        if (k != cd.k0 && (k - cd.k0) % kChunkPages == 0) {
          // a chunk longer than the staged page list: next segment, read in place
          __syncwarp();
          for (int i = lane; i < kChunkPages; i += 32) {
            const int kk = k + i;
            sm.pages[i] = kk < cd.kc1 ? __ldcg(cache.page_table + (size_t)cd.bh * cache.max_pages + kk) : 0;
          }
          __syncwarp();
        }
        const int s = it % kStagesT;
        mbar_wait(&sm.empty[s], ((it / kStagesT) & 1) ^ 1, err);
        if (lane == 0) {
          TB& tb = sm.st[s];
          const bool from_cache = k < cd.kc1;
          const int slot = k * kTileR - cd.nlp;
          const int valid = from_cache ? min(kTileR, cd.nl - k * kTileR) : max(0, min(kTileR, cd.nw - slot));
          const int hide = !from_cache && cd.hide >= slot && cd.hide < slot + kTileR ? cd.hide - slot : -1;
          // the tile description must be in place before the phase can complete
          sm.info[s] = TileRef{cd.c, cd.bh, valid, k == cd.k1 - 1, qslot, hide};
          const bool first = k == cd.k0;
          const uint32_t tx = (valid > 0 ? 2 * TB::kBytes : 0) + (first ? G * D * 2 : 0);
          if (tx)
            mbar_arrive_expect_tx(&sm.full[s], tx);
          else
            mbar_arrive(&sm.full[s]);
          if (first)
            bulk_g2s(sm.qbuf[qslot], q + (size_t)cd.bh * G * D, G * D * 2, &sm.full[s]);
          if (valid == 0) {
            // the empty tile of a head without keys: nothing to load
          } else if (from_cache) {
            int page = sm.pages[(k - cd.k0) % kChunkPages];
            if (!page_ok(page, cache.num_pages, err)) page = cache.num_pages;  // zero rows
#pragma unroll
            for (int hf = 0; hf < TB::kHalves; ++hf) {
              tma2d(tb.k[hf], &tm_kp, hf * 64, page * kPageRows, &sm.full[s]);
              tma2d(tb.v[hf], &tm_vp, hf * 64, page * kPageRows, &sm.full[s]);
            }
          } else {
            const int b = cd.bh / hkv, kh = cd.bh % hkv;
#pragma unroll
            for (int hf = 0; hf < TB::kHalves; ++hf) {
              tma4d(tb.k[hf], &tm_kr, hf * 64, slot, kh, b, &sm.full[s]);
              tma4d(tb.v[hf], &tm_vr, hf * 64, slot, kh, b, &sm.full[s]);
            }
          }
          if (k == k_claim) c_next = atomicAdd(next_chunk, 1) + (int)gridDim.x;
        }
        if (k == k_pages) {
          c_next = __shfl_sync(0xffffffffu, c_next, 0);
          nd = describe_chunk(c_next, total_chunks, chunk_rows, s_base, s_rows, s_live, s_nw,
                              s_hide, n_heads, hkv);
          fetch_pages(pg, nd, cache, lane);
        }
      }
      cd = nd;
    }
    if (lane == 0) {
      const int s = it % kStagesT;
      mbar_wait(&sm.empty[s], ((it / kStagesT) & 1) ^ 1, err);
      sm.info[s].chunk = -1;
      mbar_arrive(&sm.full[s]);
    }
  } else if (warp == kCons + 1) {
    // ------------------------------ finisher ------------------------------------
    // Combines the 4 consumer warps' partials of each finished chunk (max-weighted
    // sums) and writes the head's output (single-chunk head) or the chunk partial for
    // the merge kernel, while the consumers already work on the next chunk.
    if (early_plan) grid_dependency_wait();  // new rows, queries, outputs: after the wait
    for (int nf = 0;; ++nf) {
      const int par = nf & 1;
      mbar_wait(&sm.cdone[par], (nf >> 1) & 1, err);
      const int c = sm.fin_chunk[par];
      if (c < 0) break;
      const int bh = sm.fin_bh[par];
      const size_t hrow = (size_t)bh * G;
      const int nch = s_base[bh + 1] - s_base[bh];
      // before-append mode: the head's last chunk also takes the new row t.  Each lane
      // owns columns 4 lane .. 4 lane + 3 (D <= 128); the new key, value and the group's
      // queries are loaded together, one memory round trip.
      static_assert(D <= 128, "one 4-column slice per finisher lane");
      const bool fold = pre && c == s_base[bh + 1] - 1;
      const bool has_cols = 4 * lane < D;
      uint2 kn = make_uint2(0u, 0u), vn = make_uint2(0u, 0u), qn[G];
#pragma unroll
      for (int g = 0; g < G; ++g) qn[g] = make_uint2(0u, 0u);
      if (fold && has_cols) {
        kn = __ldg(reinterpret_cast<const uint2*>(k_new + (size_t)bh * D + 4 * lane));
        vn = __ldg(reinterpret_cast<const uint2*>(v_new + (size_t)bh * D + 4 * lane));
#pragma unroll
        for (int g = 0; g < G; ++g)
          qn[g] = __ldg(reinterpret_cast<const uint2*>(q + (hrow + g) * D + 4 * lane));
      }
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float M = -INFINITY;
        float s_new = -INFINITY;  // q . k_new in the log2 domain
        if (fold) {
          const float2 q0 = bf2_to_f2(qn[g].x), q1 = bf2_to_f2(qn[g].y);
          const float2 k0 = bf2_to_f2(kn.x), k1 = bf2_to_f2(kn.y);
          float part = fmaf(q0.x, k0.x, fmaf(q0.y, k0.y, fmaf(q1.x, k1.x, q1.y * k1.y)));
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
          s_new = part * (kLog2eT * rsqrtf((float)D));
          M = s_new;
        }
#pragma unroll
        for (int w = 0; w < kCons; ++w) M = fmaxf(M, sm.red_m[par][w][g]);
        float wt[kCons], L = 0.f;
#pragma unroll
        for (int w = 0; w < kCons; ++w) {
          const float mw = sm.red_m[par][w][g];
          wt[w] = mw == -INFINITY ? 0.f : exp2f(mw - M);
          L += wt[w] * sm.red_l[par][w][g];
        }
        const float w_new = fold ? exp2f(s_new - M) : 0.f;
        L += w_new;
#pragma unroll
        for (int d = 4 * lane; d < D; d += 128) {
          float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
          if (fold) {
            const float2 v0 = bf2_to_f2(vn.x), v1 = bf2_to_f2(vn.y);
            O = make_float4(w_new * v0.x, w_new * v0.y, w_new * v1.x, w_new * v1.y);
          }
#pragma unroll
          for (int w = 0; w < kCons; ++w) {
            const float4 v = *reinterpret_cast<const float4*>(&sm.red_o[par][w][g][d]);
            O.x = fmaf(wt[w], v.x, O.x);
            O.y = fmaf(wt[w], v.y, O.y);
            O.z = fmaf(wt[w], v.z, O.z);
            O.w = fmaf(wt[w], v.w, O.w);
          }
          if (nch == 1) {
            const float inv = L > 0.f ? 1.f / L : 0.f;
            if constexpr (F32OUT) {
              *reinterpret_cast<float4*>(out + (hrow + g) * D + d) =
                  make_float4(O.x * inv, O.y * inv, O.z * inv, O.w * inv);
            } else {
              uint2 pk;
              pk.x = pack2(O.x * inv, O.y * inv);
              pk.y = pack2(O.z * inv, O.w * inv);
              *reinterpret_cast<uint2*>(out + (hrow + g) * D + d) = pk;
            }
          } else {
            *reinterpret_cast<float4*>(ws_o + ((size_t)c * G + g) * D + d) = O;
          }
        }
        if (lane == 0) {
          if (nch == 1) {
            if (lse_out) lse_out[hrow + g] = L > 0.f ? (M + log2f(L)) * kLn2T : -INFINITY;
          } else {
            ws_ml[((size_t)c * G + g) * 2 + 0] = M;
            ws_ml[((size_t)c * G + g) * 2 + 1] = L;
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.cfree[par]);
    }
  } else {
    // ------------------------------ consumers -----------------------------------
    const float sc = kLog2eT * rsqrtf((float)D);
    const int qrow = lane >> 2;        // MMA row owned (rows >= G are padding)
    const int qcol = (lane & 3) * 2;   // first of the two columns owned
    const int row0 = warp * 16;        // this warp's rows of every tile
    const int mtx = lane >> 3;
    uint32_t qa[KS_D][2];
    float o[NT_D][4];
    float m_run = -INFINITY, l_run = 0.f;
    int cur = -1, cur_bh = 0;
    int nfin = 0;  // chunks handed to the finisher
    for (int it = 0;; ++it) {
      const int s = it % kStagesT;
      mbar_wait(&sm.full[s], (it / kStagesT) & 1, err);
      const TileRef ti = sm.info[s];
      if (ti.chunk < 0) break;
      if (ti.chunk != cur) {  // new chunk: its head's queries (staged), fresh state
        cur = ti.chunk;
        cur_bh = ti.bh;
        const __nv_bfloat16* qh = sm.qbuf[ti.qslot] + qrow * D;
#pragma unroll
        for (int k = 0; k < KS_D; ++k) {
          qa[k][0] = qrow < G ? *reinterpret_cast<const uint32_t*>(qh + 16 * k + qcol) : 0u;
          qa[k][1] = qrow < G ? *reinterpret_cast<const uint32_t*>(qh + 16 * k + 8 + qcol) : 0u;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.q_free[ti.qslot]);
#pragma unroll
        for (int n = 0; n < NT_D; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
        m_run = -INFINITY;
        l_run = 0.f;
      }
      if (ti.valid > 0) {  // (an empty tile holds no data: nothing to compute)
        const TB& tb = sm.st[s];
        const uint32_t kbase = smem_u32(tb.k[0]);
        const uint32_t vbase = smem_u32(tb.v[0]);

        // S = Q K^T for keys row0 .. row0+15 (two n-tiles of 8)
        float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int k = 0; k < KS_D; ++k) {
          const int key = row0 + 8 * (mtx >> 1) + (lane & 7);
          const int c16 = 2 * k + (mtx & 1);  // 16-byte chunk along d
          uint32_t b0, b1, b2, b3;
          ldsm_x4(kbase + (c16 >> 3) * TB::kHalfBytes + swz(key, c16 & 7), b0, b1, b2, b3);
          mma16816(sa, qa[k][0], 0u, qa[k][1], 0u, b0, b1);
          mma16816(sb, qa[k][0], 0u, qa[k][1], 0u, b2, b3);
        }
        float x[4];
        const int r0 = row0 + qcol;
        x[0] = r0 < ti.valid && r0 != ti.hide ? sa[0] * sc : -INFINITY;
        x[1] = r0 + 1 < ti.valid && r0 + 1 != ti.hide ? sa[1] * sc : -INFINITY;
        x[2] = r0 + 8 < ti.valid && r0 + 8 != ti.hide ? sb[0] * sc : -INFINITY;
        x[3] = r0 + 9 < ti.valid && r0 + 9 != ti.hide ? sb[1] * sc : -INFINITY;
        float rmax = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
        rmax = fmaxf(rmax, __shfl_xor_sync(0xffffffffu, rmax, 1));
        rmax = fmaxf(rmax, __shfl_xor_sync(0xffffffffu, rmax, 2));
        const bool need = rmax > m_run + kSlackT;
        if (__any_sync(0xffffffffu, need)) {
          const float mnew = need ? rmax : m_run;
          const float alpha = (m_run == -INFINITY) ? 0.f : exp2f(m_run - mnew);
#pragma unroll
          for (int n = 0; n < NT_D; ++n) {
            o[n][0] *= alpha;
            o[n][1] *= alpha;
          }
          l_run *= alpha;
          m_run = mnew;
        }
        float p[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          p[i] = x[i] == -INFINITY ? 0.f : exp2f(x[i] - m_run);
          l_run += p[i];
        }
        // O += P V over the 16 keys
        const uint32_t a0 = pack2(p[0], p[1]);
        const uint32_t a2 = pack2(p[2], p[3]);
#pragma unroll
        for (int dnp = 0; dnp < NT_D / 2; ++dnp) {
          const int key = row0 + 8 * (mtx & 1) + (lane & 7);
          const int c16 = 2 * dnp + (mtx >> 1);
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(vbase + (c16 >> 3) * TB::kHalfBytes + swz(key, c16 & 7), b0, b1, b2, b3);
          mma16816(o[2 * dnp], a0, 0u, a2, 0u, b0, b1);
          mma16816(o[2 * dnp + 1], a0, 0u, a2, 0u, b2, b3);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.empty[s]);

      if (ti.last) {
        // ---- this warp's chunk partial -> finisher ---------------------------------
        float l = l_run;
        l += __shfl_xor_sync(0xffffffffu, l, 1);
        l += __shfl_xor_sync(0xffffffffu, l, 2);
        const int par = nfin & 1;
        mbar_wait(&sm.cfree[par], ((nfin >> 1) & 1) ^ 1, err);
        if (qrow < G) {
#pragma unroll
          for (int n = 0; n < NT_D; ++n)
            *reinterpret_cast<float2*>(&sm.red_o[par][warp][qrow][8 * n + qcol]) =
                make_float2(o[n][0], o[n][1]);
          if (qcol == 0) {
            sm.red_m[par][warp][qrow] = m_run;
            sm.red_l[par][warp][qrow] = l;
          }
        }
        if (warp == 0 && lane == 0) {
          sm.fin_chunk[par] = cur;
          sm.fin_bh[par] = cur_bh;
        }
        mbar_arrive(&sm.cdone[par]);
        ++nfin;
      }
    }
    // no more chunks: tell the finisher
    const int par = nfin & 1;
    mbar_wait(&sm.cfree[par], ((nfin >> 1) & 1) ^ 1, err);
    if (warp == 0 && lane == 0) sm.fin_chunk[par] = -1;
    mbar_arrive(&sm.cdone[par]);
  }
  // the chunk prefix for the merge kernel (identical in every CTA; CTA 0 publishes it)
  if (blockIdx.x == 0) {
    grid_dependency_wait();  // returns at once where it was already passed
    for (int i = tid; i <= n_heads; i += kThreadsT) ws_ctrl[n_heads + 2 + i] = s_base[i];
  }
}

// Second kernel of a decode step: merges the chunk partials of every head that was
// split (o = sum_i 2^{m_i-m} o_i / sum_i 2^{m_i-m} l_i), one CTA per (batch row, key
// head).  Each thread owns 4 output columns of one query head and walks that head's
// partials kMergeBatch at a time: the batch's loads are issued together, then folded
// in with a running maximum, so a merge costs a few memory round trips.  Launched as
// a programmatic dependent of the decode kernel: it waits for the decode grid to
// complete before reading anything.  It also clears the work counter for the next
// decode launch.
template <int D, int G, bool F32OUT, int MT>
__global__ void __launch_bounds__(MT)
    decode_merge_kernel(int* __restrict__ ws_ctrl, const float* __restrict__ ws_ml,
                        const float* __restrict__ ws_o, void* __restrict__ out_,
                        float* __restrict__ lse_out, int n_heads, int hkv) {
  using OutT = typename std::conditional<F32OUT, float, __nv_bfloat16>::type;
  OutT* __restrict__ out = static_cast<OutT*>(out_);
  // the next kernel may start launching now (its CTAs take SMs as the decode CTAs exit);
  // it waits for this grid before touching anything written here
  grid_dependents_launch();
  grid_dependency_wait();
  const int tid = threadIdx.x;
  const int bh = blockIdx.x;
  if (bh == 0 && tid == 0) ws_ctrl[n_heads] = 0;  // work counter of the next launch
  const int* plan = ws_ctrl + n_heads + 2;
  const int c0 = __ldcg(plan + bh), nch = __ldcg(plan + bh + 1) - c0;
  if (nch <= 1) return;  // a single chunk wrote its output directly
  const size_t hrow = (size_t)bh * G;  // == (b * hkv + kh) * G
  constexpr int kVec = D / 4;
  constexpr int kPairs = G * kVec;  // (query head, 4 columns) pairs of the head's output
  // kSub threads per pair, each over every kSub-th chunk, combined through shared memory
  constexpr int kSub = kPairs >= MT ? 1 : MT / kPairs;
  constexpr int kSlotPairs = kPairs < MT ? kPairs : MT;
  __shared__ float s_m[kSub][kSlotPairs], s_l[kSub][kSlotPairs];
  __shared__ float4 s_o[kSub][kSlotPairs];
  for (int p0 = 0; p0 < kPairs; p0 += kSlotPairs) {
    const int sub = tid / kSlotPairs, pi = p0 + tid % kSlotPairs;
    const int g = pi / kVec, d = (pi % kVec) * 4;
    float M = -INFINITY, L = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (sub < kSub && pi < kPairs) {
      for (int cb = sub; cb < nch; cb += kSub * kMergeBatch) {
        float mv[kMergeBatch], lv[kMergeBatch];
        float4 ov[kMergeBatch];
#pragma unroll
        for (int j = 0; j < kMergeBatch; ++j) {
          const int c = cb + j * kSub;
          if (c < nch) {
            const size_t e = ((size_t)(c0 + c) * G + g);
            mv[j] = __ldcg(ws_ml + e * 2);
            lv[j] = __ldcg(ws_ml + e * 2 + 1);
            ov[j] = __ldcg(reinterpret_cast<const float4*>(ws_o + e * D + d));
          } else {
            mv[j] = -INFINITY;
            lv[j] = 0.f;
            ov[j] = make_float4(0.f, 0.f, 0.f, 0.f);
          }
        }
        float mb = M;
#pragma unroll
        for (int j = 0; j < kMergeBatch; ++j) mb = fmaxf(mb, mv[j]);
        if (mb == -INFINITY) continue;
        const float sc = M == -INFINITY ? 0.f : exp2f(M - mb);
        acc.x *= sc;
        acc.y *= sc;
        acc.z *= sc;
        acc.w *= sc;
        L *= sc;
#pragma unroll
        for (int j = 0; j < kMergeBatch; ++j) {
          const float w = mv[j] == -INFINITY ? 0.f : exp2f(mv[j] - mb);
          acc.x = fmaf(w, ov[j].x, acc.x);
          acc.y = fmaf(w, ov[j].y, acc.y);
          acc.z = fmaf(w, ov[j].z, acc.z);
          acc.w = fmaf(w, ov[j].w, acc.w);
          L = fmaf(w, lv[j], L);
        }
        M = mb;
      }
    }
    if (kSub > 1) {
      if (sub < kSub) {
        s_m[sub][tid % kSlotPairs] = M;
        s_l[sub][tid % kSlotPairs] = L;
        s_o[sub][tid % kSlotPairs] = acc;
      }
      __syncthreads();
      if (sub == 0) {  // the kSub partial sums of this pair
        float mb = -INFINITY;
#pragma unroll
        for (int q = 0; q < kSub; ++q) mb = fmaxf(mb, s_m[q][tid]);
        M = mb;
        L = 0.f;
        acc = make_float4(0.f, 0.f, 0.f, 0.f);
        if (mb != -INFINITY) {
#pragma unroll
          for (int q = 0; q < kSub; ++q) {
            const float w = s_m[q][tid] == -INFINITY ? 0.f : exp2f(s_m[q][tid] - mb);
            const float4 o = s_o[q][tid];
            acc.x = fmaf(w, o.x, acc.x);
            acc.y = fmaf(w, o.y, acc.y);
            acc.z = fmaf(w, o.z, acc.z);
            acc.w = fmaf(w, o.w, acc.w);
            L = fmaf(w, s_l[q][tid], L);
          }
        }
      }
      __syncthreads();  // the slots are reused by the next pairs
    }
    if (sub != 0 || pi >= kPairs) continue;
    const float inv = L > 0.f ? 1.f / L : 0.f;
    if constexpr (F32OUT) {
      *reinterpret_cast<float4*>(out + (hrow + g) * D + d) =
          make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
    } else {
      uint2 pk;
      pk.x = pack2(acc.x * inv, acc.y * inv);
      pk.y = pack2(acc.z * inv, acc.w * inv);
      *reinterpret_cast<uint2*>(out + (hrow + g) * D + d) = pk;
    }
    if (d == 0 && lse_out) lse_out[hrow + g] = L > 0.f ? (M + log2f(L)) * kLn2T : -INFINITY;
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn_t() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) == cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

bool map_bf16(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims,
              const cuuint64_t* strides, const cuuint32_t* box) {
  auto fn = encode_fn_t();
  if (!fn) return false;
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Control words at the front of the workspace: [n_heads] unused, work counter,
// spare, chunk prefix [n_heads + 1] (written by the decode kernel for the merge).
size_t ctrl_bytes_tc(int n_heads) { return ((size_t)(2 * n_heads + 3) * 4 + 255) / 256 * 256; }

size_t max_chunks_tc(const spkv_params& p, int num_sms) {
  return (size_t)num_sms * kUnitsPerCta + (size_t)p.B * p.Hkv;
}

template <int D, int G, bool F32OUT>
cudaError_t run_tc(const spkv_params& p, const spkv_cache& c, const spkv_ring& ring, const void* q,
                   const int32_t* t_pos, const void* k_new, const void* v_new, bool early_plan,
                   bool window_on, void* o, float* lse, void* ws, int num_sms,
                   cudaStream_t stream) {
  using S = TcDecSmem<D, G>;
  const size_t smem = sizeof(S) + 1024 + ((size_t)5 * p.B * p.Hkv + 1) * 4;
  {
    cudaError_t e = ensure_dynamic_smem((const void*)decode_tc_kernel<D, G, F32OUT>, (int)smem);
    if (e != cudaSuccess) return e;
  }
  const cuuint64_t es = 2;
  CUtensorMap tkp, tvp, tkr, tvr;
  if (c.K_pool) {  // else a window-only layer: the cache maps are never used
    const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)c.num_pages * kPageRows};
    const cuuint64_t str[1] = {(cuuint64_t)D * es};
    const cuuint32_t box[2] = {64, kTileR};
    if (!map_bf16(&tkp, c.K_pool, 2, dims, str, box) || !map_bf16(&tvp, c.V_pool, 2, dims, str, box))
      return cudaErrorInvalidValue;
  }
  if (ring.K_win) {  // else a slice of a split sequence without the window: never read
    const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)p.window, (cuuint64_t)p.Hkv, (cuuint64_t)p.B};
    const cuuint64_t str[3] = {(cuuint64_t)D * es, (cuuint64_t)p.window * D * es,
                               (cuuint64_t)p.Hkv * p.window * D * es};
    const cuuint32_t box[4] = {64, kTileR, 1, 1};
    if (!map_bf16(&tkr, ring.K_win, 4, dims, str, box) || !map_bf16(&tvr, ring.V_win, 4, dims, str, box))
      return cudaErrorInvalidValue;
  }
  if (!c.K_pool && !ring.K_win) return cudaErrorInvalidValue;
  if (!c.K_pool) {
    tkp = tkr;
    tvp = tvr;
  } else if (!ring.K_win) {
    tkr = tkp;
    tvr = tvp;
  }
  const int n_heads = p.B * p.Hkv;
  char* w = static_cast<char*>(ws);
  const size_t ctrl_bytes = ctrl_bytes_tc(n_heads);
  const size_t ml_bytes = (max_chunks_tc(p, num_sms) * G * 2 * 4 + 255) / 256 * 256;
  CacheView cv = cache_view(c);
  int* ctrl = reinterpret_cast<int*>(w);
  float* ml = reinterpret_cast<float*>(w + ctrl_bytes);
  float* po = reinterpret_cast<float*>(w + ctrl_bytes + ml_bytes);
  cudaError_t e = launch_pdl(decode_tc_kernel<D, G, F32OUT>, dim3(num_sms), dim3(kThreadsT), smem,
                             stream, tkp, tvp, tkr, tvr, cv, static_cast<const __nv_bfloat16*>(q),
                             t_pos, o, lse, ctrl, ml, po, n_heads, p.Hkv, p.window, c.err_flag,
                             static_cast<const __nv_bfloat16*>(k_new),
                             static_cast<const __nv_bfloat16*>(v_new), ring.z_win,
                             early_plan ? 1 : 0, window_on ? 1 : 0);
  if (e != cudaSuccess) return e;
  // about kUnitsPerCta chunks per SM are spread over the heads: a wide merge CTA (chunks
  // over thread subsets) only when a head averages 16 or more, else a narrow one (its
  // launch and barriers cost the next layer's decode less)
  if (kUnitsPerCta * num_sms >= 16 * n_heads)
    return launch_pdl(decode_merge_kernel<D, G, F32OUT, kMergeThreads>, dim3(n_heads),
                      dim3(kMergeThreads), 0, stream, ctrl, ml, po, o, lse, n_heads, p.Hkv);
  return launch_pdl(decode_merge_kernel<D, G, F32OUT, kMergeThreadsFew>, dim3(n_heads),
                    dim3(kMergeThreadsFew), 0, stream, ctrl, ml, po, o, lse, n_heads, p.Hkv);
}

template <int D, bool F32OUT>
cudaError_t dispatch_tc(const spkv_params& p, const spkv_cache& c, const spkv_ring& ring,
                        const void* q, const int32_t* t_pos, const void* k_new, const void* v_new,
                        bool early_plan, bool window_on, void* o, float* lse, void* ws,
                        int num_sms, cudaStream_t stream) {
  switch (p.Hq / p.Hkv) {
    case 1: return run_tc<D, 1, F32OUT>(p, c, ring, q, t_pos, k_new, v_new, early_plan, window_on, o, lse, ws, num_sms, stream);
    case 2: return run_tc<D, 2, F32OUT>(p, c, ring, q, t_pos, k_new, v_new, early_plan, window_on, o, lse, ws, num_sms, stream);
    case 4: return run_tc<D, 4, F32OUT>(p, c, ring, q, t_pos, k_new, v_new, early_plan, window_on, o, lse, ws, num_sms, stream);
    case 8: return run_tc<D, 8, F32OUT>(p, c, ring, q, t_pos, k_new, v_new, early_plan, window_on, o, lse, ws, num_sms, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

bool decode_tc_supported(const spkv_params& p) {
  return p.dtype == SPKV_BF16 && (p.head_dim == 64 || p.head_dim == 128) &&
         p.window % kTileR == 0 && p.B * p.Hkv <= kMaxHeadsT && encode_fn_t() != nullptr;
}

size_t decode_tc_ctrl_bytes(const spkv_params& p) { return ctrl_bytes_tc(p.B * p.Hkv); }

size_t decode_tc_workspace_bytes(const spkv_params& p, int num_sms) {
  const int n_heads = p.B * p.Hkv;
  const int G = p.Hq / p.Hkv;
  const size_t ctrl_bytes = ctrl_bytes_tc(n_heads);
  const size_t mc = max_chunks_tc(p, num_sms);
  const size_t ml_bytes = (mc * G * 2 * 4 + 255) / 256 * 256;
  return ctrl_bytes + ml_bytes + mc * G * p.head_dim * 4;
}

cudaError_t launch_decode_tc(const spkv_params& p, const spkv_cache& c, const spkv_ring& ring,
                             const void* q, const int32_t* t_pos, void* o, float* lse,
                             void* workspace, int num_sms, cudaStream_t stream,
                             const void* k_new, const void* v_new, bool early_plan) {
  if (p.head_dim == 128)
    return dispatch_tc<128, false>(p, c, ring, q, t_pos, k_new, v_new, early_plan, true, o, lse,
                                   workspace, num_sms, stream);
  return dispatch_tc<64, false>(p, c, ring, q, t_pos, k_new, v_new, early_plan, true, o, lse,
                                workspace, num_sms, stream);
}

cudaError_t launch_decode_partial(const spkv_params& p, const spkv_cache& c, const spkv_ring& ring,
                                  const void* q, const int32_t* t_pos, bool window_on,
                                  float* o_part, float* lse_part, void* workspace, int num_sms,
                                  cudaStream_t stream) {
  if (p.head_dim == 128)
    return dispatch_tc<128, true>(p, c, ring, q, t_pos, nullptr, nullptr, false, window_on, o_part,
                                  lse_part, workspace, num_sms, stream);
  return dispatch_tc<64, true>(p, c, ring, q, t_pos, nullptr, nullptr, false, window_on, o_part,
                               lse_part, workspace, num_sms, stream);
}

}  // namespace spkv
