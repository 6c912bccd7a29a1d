// prefill_tc.cu -- a6 on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// "Self-Pruned Key-Value Attention" (arXiv 2605.14037), §2.1, Eqs. (3)-(4), for a
// chunk of queries.  Persistent CTAs (one per SM) take tiles: 128 consecutive query
// positions t0 .. t0+127 of two query heads of one key head, heaviest tiles first.  A
// tile's key set is, in 128-key blocks:
//   * the causal window band first: the block t0-128 .. t0-1 (from the ring for
//     positions before the chunk, else from the chunk's K/V; visible to query t0+r
//     for keys i > r of the block) and the block t0 .. t0+127 (keys i <= r);
//   * then the compacted cache, two 64-row pages per block, holding the rows with
//     pos <= t0+127-w (gated-in keys of Eq. (4)); blocks whose rows all have
//     pos <= t0-w need no mask, the last one or two are masked per query
//     (pos <= t-w: since rows are stored in position order, a prefix of the block
//     whose length each query finds by bisection), and rows beyond are never
//     touched: the dead key blocks of the causal mask are simply absent.
// The window blocks need no plan, so their loads and MMAs start at once while two
// otherwise idle warps find the cache extent (a few dependent global reads), one tile
// ahead.
//
// Both contractions are dense tensor-core tiles: S = Q K^T (M=128 queries, N=128 keys,
// K=128) and O += P V (M=128, N=128, K=128 keys), bf16 operands, fp32 accumulators in
// TMEM.  TMEM (512 columns): O of head 0, O of head 1, S of head 0, S of head 1; P is
// written back over its S and fed to the second MMA from TMEM.  The single MMA thread
// issues, per head and block, PV(j) and then S(j+1), alternating the heads: while one
// head's softmax runs, the tensor cores do the other head's PV and next S.  The commit
// that signals S(j+1) also covers PV(j) (a commit tracks every earlier MMA of the
// thread), so a softmax that must rescale O (its running maximum grew by more than 8)
// does it in TMEM at once, with no further wait.  A tile's Q is released once its
// last S is issued, so the next tile's Q loads while the last blocks finish, and head
// 0's first S of the next tile is issued right after its last PV when that Q and the
// first K block have landed (the heads stay staggered across tiles); the output is
// written through a shared-memory staging tile per softmax warp, so every store covers
// whole 128-byte pieces of output rows.
//
// Warp roles (384 threads):
//   warp 0      TMA producer: Q per tile; per block K (+ positions) and V, through one
//               ring of four 32 KB slots;
//   warp 1      TMEM allocation and the single MMA-issuing thread;
//   warps 2-3   the tile scheduler (thread 64) and the cache plan (extent and fully
//               visible rows of the tile);
//   warps 4-7   softmax of head 0 (one query row per thread, TMEM lanes 0..127);
//   warps 8-11  softmax of head 1.
// Per-block side data (cache positions, or soft-mask biases) ride in a 2-slot ring of
// their own, released by the softmax warps; tiles and cache plans pass through 2-slot
// rings too, so no barrier can run more than one phase ahead of a waiter.  Softmax runs
// in the log2 domain.  Every mbarrier wait is bounded (a stuck wait raises
// SPKV_FLAG_TIMEOUT).
//
// The same kernel (SOFT = true) computes the soft-gated attention used at training
// time (§2.1, "soft relaxation", Eqs. (5)-(6)): every key s <= t of the sequence,
// read in 128-key blocks from the sequence K/V, with the additive score 0 inside the
// causal window and c (alpha_s - 1) outside it; the per-key bias (already divided by
// the score scale, i.e. in raw q.k units) rides with each block.  No key block is
// skipped.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "host.h"
#include "launch.h"
#include "tc.cuh"

namespace spkv {
namespace {

constexpr int kQT = 128;          // queries per CTA and head
constexpr int kKB = 128;          // keys per block
constexpr int kHD = 128;          // head_dim
constexpr int kWin = 128;         // window of this path
constexpr int kSlots = 4;         // K/V ring: K(j) is item 2j, V(j) item 2j+1, slot = item % kSlots
constexpr int kAux = 2;           // side-data slots
constexpr int kThr = 384;
constexpr int kSoftWarps = 8;
constexpr int kPlanReaders = 1 + 1 + kSoftWarps;  // producer, MMA thread, softmax warps
constexpr int kTileReaders = kPlanReaders;        // the same roles read the tile slots
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kSlack = 8.f;
constexpr int kHalf = kKB * 128;  // one 64-column half of a K or V block (128 rows x 128 B)

constexpr uint32_t kColO0 = 0, kColO1 = 128, kColS = 256;  // S of head h at kColS + 128 h

struct __align__(1024) TcSmem {
  char q[2][2][kQT * 128];   // [head][d half], 128B-swizzled rows
  char kv[kSlots][2][kHalf];  // [slot][d half]: K or V of one block
  char ostage[kSoftWarps][32 * 128];  // per softmax warp: 32 output rows x 64 columns (bf16)
  int aux[kAux][kKB];         // per block: cache positions, or soft-mask biases
  uint64_t q_full, q_empty;
  uint64_t kv_full[kSlots], kv_empty[kSlots];
  uint64_t aux_full[kAux], aux_empty[kAux];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t o_full[2];
  uint64_t plan_ready[2], plan_free[2];  // plan slot of tile n: n % 2
  uint64_t tile_ready[2], tile_free[2];  // tile slot of tile n: n % 2
  int tile[2];                           // tile index, -1: no more tiles
  uint32_t tmem_base;
  int plan[2][4];  // nc (cache blocks), nfull (rows visible to the whole tile), nrows, -
  int red[2][4];
};

// 2^x on the MUFU unit (ex2.approx, flush-to-zero): the scores are <= 8 above the
// running max, so x < 8 and the result is a normal number or 0.
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// Phase `parity` of an mbarrier completed?  (no waiting)
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Kinds of key block, each with its own straight-line softmax code.
enum BlockKind : int {
  kOpen = 0,        // every key visible to every query (a cache block below the tile's limit)
  kKeysAfter = 1,   // window block [t0-128, t0): query r keeps keys i > r
  kKeysUpTo = 2,    // window block [t0, t0+128): query r keeps keys i <= r
  kCacheMask = 3,   // cache block at the tile's limit: its first `vis` rows (pos <= t - w)
  kSoftFar = 4,     // soft mask, block outside every window: every key + its bias
  kSoftBefore = 5   // soft mask, block [t0-128, t0): keys i > r + 0, keys i <= r + bias
};

struct RowStats {
  float ps;    // sum of this block's p
  float mnew;  // running maximum after this block
  bool need;   // the maximum moved (O and l are rescaled)
};

// One query row's softmax over one 128-key block: scores (raw q.k from TMEM) masked as
// KIND says, row maximum, p = 2^(x c - m) packed to bf16 pairs in pk, and their sum.
// The running maximum is raised only when a score exceeds it by more than kSlack.
// r: the query's row in the tile; vis: visible rows of a kCacheMask block; aux: the
// block's soft-mask biases.
template <int KIND>
__device__ __forceinline__ RowStats block_softmax(const uint32_t (&raw)[128], uint32_t (&pk)[64],
                                                  float m, float c, int r, int vis,
                                                  const int* __restrict__ aux) {
  float x[128];
#pragma unroll
  for (int i = 0; i < 128; ++i) {
    const float sc = __uint_as_float(raw[i]);
    if constexpr (KIND == kOpen) {
      x[i] = sc;
    } else if constexpr (KIND == kKeysAfter) {
      x[i] = i > r ? sc : -INFINITY;
    } else if constexpr (KIND == kKeysUpTo) {
      x[i] = i <= r ? sc : -INFINITY;
    } else if constexpr (KIND == kCacheMask) {
      x[i] = i < vis ? sc : -INFINITY;
    } else if constexpr (KIND == kSoftFar) {
      x[i] = sc + __int_as_float(aux[i]);
    } else {
      x[i] = sc + (i > r ? 0.f : __int_as_float(aux[i]));
    }
  }
  // row maximum: three-input max over 8 independent partials (x[0..23], then 16 at a
  // time up to x[119], then x[120..127])
  float mx[8];
#pragma unroll
  for (int a = 0; a < 8; ++a) mx[a] = max3(x[a], x[a + 8], x[a + 16]);
#pragma unroll
  for (int i = 24; i < 120; i += 16)
#pragma unroll
    for (int a = 0; a < 8; ++a) mx[a] = max3(mx[a], x[i + a], x[i + 8 + a]);
#pragma unroll
  for (int a = 0; a < 8; ++a) mx[a] = fmaxf(mx[a], x[120 + a]);
  const float rmax = max3(max3(mx[0], mx[1], mx[2]), max3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7])) * c;
  RowStats st;
  st.need = rmax > m + kSlack;
  st.mnew = st.need ? fmaxf(m, rmax) : m;
  // p = 2^(x c - m): one packed fma per pair, then MUFU; masked keys give 2^-inf = 0
  const float msafe = st.mnew == -INFINITY ? 0.f : st.mnew;
  float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                   make_float2(0.f, 0.f)};
  const float2 c2 = make_float2(c, c), nm2 = make_float2(-msafe, -msafe);
#pragma unroll
  for (int i = 0; i < 64; ++i) {
    const float2 e = fma2(make_float2(x[2 * i], x[2 * i + 1]), c2, nm2);
    const float2 pp = make_float2(fast_exp2(e.x), fast_exp2(e.y));
    acc[i & 3] = add2(acc[i & 3], pp);
    pk[i] = pack_bf16(pp.x, pp.y);
  }
  st.ps = (acc[0].x + acc[0].y) + (acc[1].x + acc[1].y) + (acc[2].x + acc[2].y) +
          (acc[3].x + acc[3].y);
  return st;
}

// Tile i of a launch, heaviest first (later query tiles see more cache rows): query
// tile n_qt - 1 - i / (n_hp n_bh), head pair and (batch row, key head) from the rest.
struct Tile {
  int qt, hp, bh;
};

__device__ __forceinline__ Tile tile_of(int i, int n_qt, int n_hp, int n_bh) {
  Tile t;
  const int per = n_hp * n_bh;
  t.qt = n_qt - 1 - i / per;
  const int rem = i % per;
  t.hp = rem % n_hp;
  t.bh = rem / n_hp;
  return t;
}

// The k-th tile of CTA c among `grid` persistent CTAs (-1: none left): rounds of `grid`
// tiles, taken forwards and backwards in turn, so that heavy and light tiles even out.
__device__ __forceinline__ int tile_index(int k, int c, int grid, int n_tiles) {
  const int i = k * grid + ((k & 1) ? grid - 1 - c : c);
  return i < n_tiles ? i : -1;
}

template <bool SOFT>
__global__ void __launch_bounds__(kThr, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_kc,
                      const __grid_constant__ CUtensorMap tm_vc,
                      const __grid_constant__ CUtensorMap tm_kp,
                      const __grid_constant__ CUtensorMap tm_vp,
                      const __grid_constant__ CUtensorMap tm_kr,
                      const __grid_constant__ CUtensorMap tm_vr, CacheView cache, int num_pages,
                      __nv_bfloat16* __restrict__ out, float* __restrict__ lse_out,
                      int chunk_start, int chunk_len, int hkv, int G, int n_qt, int n_hp,
                      int n_bh, uint32_t* err, const float* __restrict__ soft_bias,
                      int* __restrict__ sched) {
  extern __shared__ __align__(1024) char smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;  // 128B-swizzle atoms
  TcSmem& sm = *reinterpret_cast<TcSmem*>(smem_raw + pad);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int Hq = hkv * G;
  const int n_tiles = n_qt * n_hp * n_bh;
  const int grid = gridDim.x, cta = blockIdx.x;

  // ---- set-up (once per CTA): barriers, TMEM -----------------------------------------
  if (tid == 0) {
    mbar_init(&sm.q_full, 1);
    mbar_init(&sm.q_empty, 1);
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(&sm.kv_full[s], 1);
      mbar_init(&sm.kv_empty[s], 1);
    }
    for (int s = 0; s < kAux; ++s) {
      mbar_init(&sm.aux_full[s], 1);
      mbar_init(&sm.aux_empty[s], kSoftWarps);
    }
    for (int h = 0; h < 2; ++h) {
      mbar_init(&sm.s_full[h], 1);
      mbar_init(&sm.p_full[h], 128);
      mbar_init(&sm.o_full[h], 1);
      mbar_init(&sm.plan_ready[h], 1);
      mbar_init(&sm.plan_free[h], kPlanReaders);
      mbar_init(&sm.tile_ready[h], 1);
      mbar_init(&sm.tile_free[h], kTileReaders);
    }
    fence_mbar_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(
                     smem_u32(&sm.tmem_base))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  // tile n of this CTA from tile slot n % 2 (-1: none left); every reader role reads it
  // once (a warp: all lanes, then lane 0 frees it)
  auto read_tile = [&](int n) -> int {
    mbar_wait(&sm.tile_ready[n & 1], (n >> 1) & 1, err);
    return sm.tile[n & 1];
  };

  // Every role walks the same tiles of this CTA.  Blocks are numbered across tiles (g):
  // the K/V ring, the side-data ring and the S/P barriers run on g; tile n (of this
  // CTA) uses plan slot n % 2 and the n-th phases of q_full, q_empty and o_full.
  if (warp == 0) {
    // ------------------------------ TMA producer --------------------------------
    // Lane l keeps the page numbers of cache blocks 32 i + l (two pages each), fetched
    // 32 blocks at a time; lane 0 issues every copy.
    int g = 0;
    for (int n = 0;; ++n) {
      const int ti = read_tile(n);
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.tile_free[n & 1]);
      if (ti < 0) break;
      const Tile tl = tile_of(ti, n_qt, n_hp, n_bh);
      const int bh = tl.bh, b = bh / hkv, kh = bh % hkv;
      const int t0 = chunk_start + tl.qt * kQT;
      const int h0 = kh * G + 2 * tl.hp;
      const int nw = t0 >= kWin ? 2 : 1;
      const int wfirst = t0 - (nw - 1) * kKB;
      int pg0 = -1, pg1 = -1, pg_base = -1;
      int n_pages = 0;
      int J = SOFT ? nw + (t0 >= kWin ? t0 / kKB - 1 : 0) : -1;
      for (int j = 0;; ++j, ++g) {
        if (j == 1 && lane == 0) {
          // Q of this tile (after its first K/V, whose ring slots may free earlier), once
          // the previous tile's last S has read the old Q
          if (n > 0) mbar_wait(&sm.q_empty, (n - 1) & 1, err);
          mbar_arrive_expect_tx(&sm.q_full, 2 * 2 * kQT * 128);
          for (int hh = 0; hh < 2; ++hh)
            for (int half = 0; half < 2; ++half)
              tma_4d(sm.q[hh][half], &tm_q, half * 64, h0 + hh, t0 - chunk_start, b, &sm.q_full);
        }
        if (J < 0 && j >= nw) {  // the far blocks' count: from the plan
          const int ps = n & 1;
          mbar_wait(&sm.plan_ready[ps], (n >> 1) & 1, err);
          J = nw + sm.plan[ps][0];
          n_pages = (sm.plan[ps][2] + kPageRows - 1) / kPageRows;
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm.plan_free[ps]);
        }
        if (J >= 0 && j >= J) break;
        const int ks = (2 * g) % kSlots, kph = ((2 * g) / kSlots) & 1;          // K(g)
        const int vs = (2 * g + 1) % kSlots, vph = ((2 * g + 1) / kSlots) & 1;  // V(g)
        const int ax = g % kAux, aph = (g / kAux) & 1;
        const bool far = j >= nw;
        const int cj = j - nw;  // far block index
        int p_a = -1, p_b = -1;
        if (!SOFT && far) {
          if ((cj >> 5) != pg_base) {  // next 32 blocks' page numbers, one load per lane
            pg_base = cj >> 5;
            const int blk = pg_base * 32 + lane;
            pg0 = 2 * blk < n_pages ? __ldg(cache.page_table + (size_t)bh * cache.max_pages + 2 * blk) : -1;
            pg1 = 2 * blk + 1 < n_pages
                      ? __ldg(cache.page_table + (size_t)bh * cache.max_pages + 2 * blk + 1)
                      : -1;
          }
          p_a = __shfl_sync(0xffffffffu, pg0, cj & 31);
          p_b = __shfl_sync(0xffffffffu, pg1, cj & 31);
          if (p_a >= 0 && !page_ok(p_a, num_pages, err)) p_a = -1;  // debug build: zero rows
          if (p_b >= 0 && !page_ok(p_b, num_pages, err)) p_b = -1;
        }
        if (lane == 0) {
          // side data of this block (positions of the cache rows, or soft-mask biases)
          mbar_wait(&sm.aux_empty[ax], aph ^ 1, err);
          int aux_bytes = 0;
          if (SOFT) {
            if (far || (nw == 2 && j == 0)) aux_bytes = kKB * 4;
          } else if (far) {
            aux_bytes = (p_a >= 0 ? kPageRows * 4 : 0) + (p_b >= 0 ? kPageRows * 4 : 0);
          }
          if (aux_bytes) {
            mbar_arrive_expect_tx(&sm.aux_full[ax], aux_bytes);
            if (SOFT) {
              const int pb = far ? cj * kKB : wfirst;
              bulk_g2s(sm.aux[ax], soft_bias + (size_t)bh * chunk_len + pb, kKB * 4, &sm.aux_full[ax]);
            } else {
              if (p_a >= 0)
                bulk_g2s(sm.aux[ax], cache.pos + (size_t)p_a * kPageRows, kPageRows * 4, &sm.aux_full[ax]);
              if (p_b >= 0)
                bulk_g2s(sm.aux[ax] + kPageRows, cache.pos + (size_t)p_b * kPageRows, kPageRows * 4,
                         &sm.aux_full[ax]);
            }
          } else {
            mbar_arrive(&sm.aux_full[ax]);
          }
          // K of block j (a missing page: an out-of-range row, which the copy fills with
          // zeros; its rows are masked), then V
          const int oob = num_pages * kPageRows;
          for (int which = 0; which < 2; ++which) {
            const int sl = which ? vs : ks, ph = which ? vph : kph;
            const CUtensorMap* mc = which ? &tm_vc : &tm_kc;
            const CUtensorMap* mr = which ? &tm_vr : &tm_kr;
            const CUtensorMap* mp = which ? &tm_vp : &tm_kp;
            mbar_wait(&sm.kv_empty[sl], ph ^ 1, err);
            mbar_arrive_expect_tx(&sm.kv_full[sl], 2 * kHalf);
            for (int half = 0; half < 2; ++half) {
              if (!far || SOFT) {
                const int pb = far ? cj * kKB : wfirst + j * kKB;
                if (pb >= chunk_start)
                  tma_4d(sm.kv[sl][half], mc, half * 64, kh, pb - chunk_start, b, &sm.kv_full[sl]);
                else
                  tma_4d(sm.kv[sl][half], mr, half * 64, 0, kh, b, &sm.kv_full[sl]);
              } else {
                tma_2d(sm.kv[sl][half], mp, half * 64, p_a >= 0 ? p_a * kPageRows : oob, &sm.kv_full[sl]);
                tma_2d(sm.kv[sl][half] + kPageRows * 128, mp, half * 64,
                       p_b >= 0 ? p_b * kPageRows : oob, &sm.kv_full[sl]);
              }
            }
          }
        }
        __syncwarp();
      }
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer -----------------------------------
    if (lane == 0) {
      constexpr uint32_t idesc_s = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kKB >> 3) << 17) |
                                   ((uint32_t)(kQT >> 4) << 24);
      constexpr uint32_t idesc_pv = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) |
                                    ((uint32_t)(kHD >> 3) << 17) | ((uint32_t)(kQT >> 4) << 24);
      // S_h = Q_h K^T (K in ring slot st)
      auto issue_s = [&](int hh, int st) {
        const uint32_t col = kColS + 128 * hh;
#pragma unroll
        for (int kk = 0; kk < kHD / 16; ++kk) {
          const uint64_t ad = smem_desc(sm.q[hh][kk >> 2] + (kk & 3) * 32, 16, 1024);
          const uint64_t bd = smem_desc(sm.kv[st][kk >> 2] + (kk & 3) * 32, 16, 1024);
          mma_ss(tmem + col, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
        }
        mma_commit(&sm.s_full[hh]);
      };
      // O_h += P_h V (V in ring slot st, P over S_h in TMEM)
      auto issue_pv = [&](int hh, int st, bool acc) {
        const uint32_t colO = hh ? kColO1 : kColO0;
        const uint32_t colP = kColS + 128 * hh;
#pragma unroll
        for (int kk = 0; kk < kKB / 16; ++kk) {
          const uint64_t bd = smem_desc(sm.kv[st][0] + kk * 16 * 128, kHalf, 1024);
          mma_ts(tmem + colO, tmem + colP + kk * 8, bd, idesc_pv, (acc || kk > 0) ? 1u : 0u);
        }
      };
      int g = 0;
      int ti = read_tile(0);
      mbar_arrive(&sm.tile_free[0]);
      bool s0_issued = false;  // this tile's first S went out at the end of the previous one
      for (int n = 0;; ++n) {
        if (ti < 0) break;
        const Tile tl = tile_of(ti, n_qt, n_hp, n_bh);
        const int t0 = chunk_start + tl.qt * kQT;
        const int nw = t0 >= kWin ? 2 : 1;
        int J = SOFT ? nw + (t0 >= kWin ? t0 / kKB - 1 : 0) : -1;
        bool q_released = false;
        int ti_next = -2;  // the next tile, once read (-2: not yet)
        if (!s0_issued) {
          // S(0) of this tile: after its Q has landed (the S region it writes held the
          // previous tile's last P, whose PV was issued before: MMAs run in order)
          mbar_wait(&sm.q_full, n & 1, err);
          mbar_wait(&sm.kv_full[(2 * g) % kSlots], ((2 * g) / kSlots) & 1, err);
          tc_fence_after();
          issue_s(0, (2 * g) % kSlots);
          issue_s(1, (2 * g) % kSlots);
          mma_commit(&sm.kv_empty[(2 * g) % kSlots]);
        }
        s0_issued = false;
        for (int j = 0;; ++j, ++g) {
          if (J < 0 && j + 1 >= nw) {  // the far blocks' count: from the plan
            const int ps = n & 1;
            mbar_wait(&sm.plan_ready[ps], (n >> 1) & 1, err);
            J = nw + sm.plan[ps][0];
            mbar_arrive(&sm.plan_free[ps]);
          }
          const bool more = J < 0 || j + 1 < J;
          const int vs = (2 * g + 1) % kSlots, vph = ((2 * g + 1) / kSlots) & 1;  // V(g)
          const int ks = (2 * g + 2) % kSlots, kph = ((2 * g + 2) / kSlots) & 1;  // K(g+1)
          mbar_wait(&sm.kv_full[vs], vph, err);
          mbar_wait(&sm.p_full[0], g & 1, err);
          tc_fence_after();
          issue_pv(0, vs, j > 0);
          if (more) {
            mbar_wait(&sm.kv_full[ks], kph, err);
            tc_fence_after();
            issue_s(0, ks);
          } else {
            mma_commit(&sm.o_full[0]);  // head 0's epilogue overlaps head 1's last PV
            if (!q_released) {
              mma_commit(&sm.q_empty);
              q_released = true;
            }
            // head 0's first S of the next tile goes out now if that tile, its Q and its
            // first K are already in place (tested without waiting): head 0 then starts
            // the next tile while head 1 finishes this one, and the two heads' softmax
            // stay staggered across the boundary
            const int n1 = n + 1;
            const int ks1 = (2 * (g + 1)) % kSlots, kph1 = ((2 * (g + 1)) / kSlots) & 1;
            if (mbar_test(&sm.tile_ready[n1 & 1], (n1 >> 1) & 1)) {
              ti_next = sm.tile[n1 & 1];
              mbar_arrive(&sm.tile_free[n1 & 1]);
              if (ti_next >= 0 && mbar_test(&sm.q_full, n1 & 1) && mbar_test(&sm.kv_full[ks1], kph1)) {
                tc_fence_after();
                issue_s(0, ks1);
                s0_issued = true;
              }
            }
          }
          mbar_wait(&sm.p_full[1], g & 1, err);
          tc_fence_after();
          issue_pv(1, vs, j > 0);
          mma_commit(&sm.kv_empty[vs]);
          if (!more) {
            mma_commit(&sm.o_full[1]);
            if (s0_issued) {
              const int ks1 = (2 * (g + 1)) % kSlots;
              issue_s(1, ks1);
              mma_commit(&sm.kv_empty[ks1]);
            }
            ++g;
            break;
          }
          issue_s(1, ks);
          mma_commit(&sm.kv_empty[ks]);
          if (!q_released && J >= 0 && j + 2 >= J) {
            // block j + 1 is the tile's last: its S was the last read of this Q, so the
            // next tile's Q can load while these blocks' softmax and PV run
            mma_commit(&sm.q_empty);
            q_released = true;
          }
        }
        if (ti_next == -2) {
          ti = read_tile(n + 1);
          mbar_arrive(&sm.tile_free[(n + 1) & 1]);
        } else {
          ti = ti_next;
        }
      }
    }
  } else if (warp < 4) {
    // --------------------------- tile scheduler, cache plan ------------------------
    // Thread 64 hands out this CTA's tiles through tile slot n % 2, one tile ahead of
    // their readers.  With a schedule counter (sched), the first tile of CTA c is tile
    // c and every later one the next unclaimed tile of the launch (tiles go heaviest
    // first, so the CTAs that finish early take the light ones); without it, the
    // fixed order of tile_index.  The last CTA to run out of tiles zeroes the counter
    // for the next launch.
    // Warps 2-3 then write, for tile n into plan slot n % 2, the number of cache
    // blocks, the rows visible to every query of the tile and the head's row count.
    {
      const int pt = tid - 64;  // 0..63
      for (int n = 0;; ++n) {
        if (pt == 0) {
          if (n >= 2) mbar_wait(&sm.tile_free[n & 1], ((n >> 1) - 1) & 1, err);
          int ti = sched ? (n == 0 ? cta : grid + atomicAdd(sched, 1)) : tile_index(n, cta, grid, n_tiles);
          if (ti >= n_tiles) ti = -1;
          sm.tile[n & 1] = ti;
          mbar_arrive(&sm.tile_ready[n & 1]);
          if (ti < 0 && sched) {
            __threadfence();  // this CTA's claims precede its count
            if (atomicAdd(sched + 1, 1) == grid - 1) {  // every CTA has stopped claiming
              __threadfence();
              sched[0] = 0;
              sched[1] = 0;
            }
          }
        }
        named_bar_sync(1, 64);
        const int ti = sm.tile[n & 1];  // rewritten only after both plan warps pass the next barrier
        if (ti < 0) break;
        if constexpr (SOFT) continue;
        const Tile tl = tile_of(ti, n_qt, n_hp, n_bh);
        const int bh = tl.bh;
        const int t0 = chunk_start + tl.qt * kQT;
        const int ps = n & 1;
        if (n >= 2) mbar_wait(&sm.plan_free[ps], ((n >> 1) - 1) & 1, err);
        const int nrow = cache.count ? __ldcg(cache.count + bh) : 0;  // no cache: window only
        const int npages = (nrow + kPageRows - 1) / kPageRows;
        const int lim_full = t0 - kWin, lim_any = t0 + kQT - 1 - kWin;
        // pages whose first row is visible to the whole tile / to some query of it
        int pf = 0, pa = 0;
        for (int pg = pt; pg < npages; pg += 64) {
          const int p0 = cache_pos(cache, bh, pg * kPageRows);
          pf += p0 <= lim_full;
          pa += p0 <= lim_any;
        }
#pragma unroll
        for (int m = 16; m > 0; m >>= 1) {
          pf += __shfl_xor_sync(0xffffffffu, pf, m);
          pa += __shfl_xor_sync(0xffffffffu, pa, m);
        }
        if (lane == 0) {
          sm.red[warp - 2][0] = pf;
          sm.red[warp - 2][1] = pa;
        }
        named_bar_sync(1, 64);
        const int Pf = sm.red[0][0] + sm.red[1][0], Pa = sm.red[0][1] + sm.red[1][1];
        // rows of the last such page: thread pt checks row pt of page Pf-1 and of Pa-1
        int cf = 0, ca = 0;
        if (Pf > 0) {
          const int row = (Pf - 1) * kPageRows + pt;
          cf = row < nrow && cache_pos(cache, bh, row) <= lim_full;
        }
        if (Pa > 0) {
          const int row = (Pa - 1) * kPageRows + pt;
          ca = row < nrow && cache_pos(cache, bh, row) <= lim_any;
        }
        cf = __popc(__ballot_sync(0xffffffffu, cf));
        ca = __popc(__ballot_sync(0xffffffffu, ca));
        named_bar_sync(1, 64);
        if (lane == 0) {
          sm.red[warp - 2][2] = cf;
          sm.red[warp - 2][3] = ca;
        }
        named_bar_sync(1, 64);
        if (pt == 0) {
          const int nfull = Pf > 0 ? (Pf - 1) * kPageRows + sm.red[0][2] + sm.red[1][2] : 0;
          const int n_any = Pa > 0 ? (Pa - 1) * kPageRows + sm.red[0][3] + sm.red[1][3] : 0;
          sm.plan[ps][0] = (n_any + kKB - 1) / kKB;
          sm.plan[ps][1] = nfull;
          sm.plan[ps][2] = nrow;
          mbar_arrive(&sm.plan_ready[ps]);  // release: the plan words are visible to its waiters
        }
        named_bar_sync(1, 64);  // sm.red is reused by the next tile
      }
    }
  } else {
    // ------------------------------ softmax --------------------------------------
    const int hh = (warp - 4) >> 2;
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const uint32_t lane_addr = tmem + ((uint32_t)(quad * 32) << 16);
    const uint32_t colO = hh ? kColO1 : kColO0;
    const uint32_t colS = kColS + 128 * hh;
    const float c = kLog2e * rsqrtf((float)kHD);
    int g = 0;
    for (int n = 0;; ++n) {
      const int ti = read_tile(n);
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.tile_free[n & 1]);
      if (ti < 0) break;
      const Tile tl = tile_of(ti, n_qt, n_hp, n_bh);
      const int bh = tl.bh, b = bh / hkv, kh = bh % hkv;
      const int t0 = chunk_start + tl.qt * kQT;
      const int t = t0 + r;
      const int nw = t0 >= kWin ? 2 : 1;
      float m = -INFINITY, l = 0.f;
      int J = SOFT ? nw + (t0 >= kWin ? t0 / kKB - 1 : 0) : -1;
      int nfull = 0, nrows = 0;
      for (int j = 0;; ++j, ++g) {
        if (J < 0 && j >= nw) {
          const int ps = n & 1;
          mbar_wait(&sm.plan_ready[ps], (n >> 1) & 1, err);
          J = nw + sm.plan[ps][0];
          nfull = sm.plan[ps][1];
          nrows = sm.plan[ps][2];
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm.plan_free[ps]);
        }
        if (J >= 0 && j >= J) break;
        const int ax = g % kAux;
        mbar_wait(&sm.s_full[hh], g & 1, err);
        tc_fence_after();
        uint32_t raw[128];
        tmem_ld32(lane_addr + colS, raw);
        tmem_ld32(lane_addr + colS + 32, raw + 32);
        tmem_ld32(lane_addr + colS + 64, raw + 64);
        tmem_ld32(lane_addr + colS + 96, raw + 96);
        mbar_wait(&sm.aux_full[ax], (g / kAux) & 1, err);
        tmem_wait_ld();
        // scores in the raw (unscaled) domain, masked keys at -inf; for the soft mask the
        // per-key bias is pre-divided by the scale so that one fma gives the exponent
        const bool far = j >= nw;
        const int row0 = (j - nw) * kKB;
        const int* aux = sm.aux[ax];
        uint32_t pk[64];
        RowStats st;
        if (!far && nw == 2 && j == 0) {
          st = SOFT ? block_softmax<kSoftBefore>(raw, pk, m, c, r, 0, aux)
                    : block_softmax<kKeysAfter>(raw, pk, m, c, r, 0, aux);
        } else if (!far) {
          st = block_softmax<kKeysUpTo>(raw, pk, m, c, r, 0, aux);
        } else if (SOFT) {
          st = block_softmax<kSoftFar>(raw, pk, m, c, r, 0, aux);
        } else if (row0 + kKB <= nfull) {  // every row visible to every query of the tile
          st = block_softmax<kOpen>(raw, pk, m, c, r, 0, aux);
        } else {
          // cache positions ascend (rows are appended in position order), so the rows of
          // this block that query t sees are its first vis, found by bisection
          int vis = 0, hi = min(kKB, nrows - row0);
          while (vis < hi) {
            const int mid = (vis + hi) >> 1;
            if (aux[mid] <= t - kWin) vis = mid + 1; else hi = mid;
          }
          st = block_softmax<kCacheMask>(raw, pk, m, c, r, vis, aux);
        }
        // the side data of this block have been read
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.aux_empty[ax]);
        // O holds P V of this tile's blocks before j (complete: S(j) was issued after
        // PV(j-1) and its commit covers it); rescale it in TMEM when the maximum moved
        if (__any_sync(0xffffffffu, st.need)) {
          const float alpha = (m == -INFINITY) ? 0.f : fast_exp2(m - st.mnew);
          if (j > 0) {
#pragma unroll
            for (int cc = 0; cc < kHD; cc += 32) {
              uint32_t o[32];
              tmem_ld32(lane_addr + colO + cc, o);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
              tmem_st32(lane_addr + colO + cc, o);
            }
          }
          l *= alpha;
          m = st.mnew;
        }
        l += st.ps;
        tmem_st32(lane_addr + colS, pk);
        tmem_st32(lane_addr + colS + 32, pk + 32);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&sm.p_full[hh]);
      }
      // epilogue of the tile: O / l (the next tile's first PV overwrites O only after
      // this warpgroup's next P, i.e. after these reads)
      mbar_wait(&sm.o_full[hh], n & 1, err);
      tc_fence_after();
      const int hg = kh * G + 2 * tl.hp + hh;
      const size_t row_out = ((size_t)b * chunk_len + (t - chunk_start)) * Hq + hg;
      const float inv = l > 0.f ? 1.f / l : 0.f;
      // O / l to bf16: the row's 128 columns come out of TMEM at once (one wait), then go
      // through this warp's staging tile 64 columns at a time: lane r writes its row's
      // eight 16-byte pieces (piece c at slot c ^ (r & 7), so that each group of 8 lanes
      // covers all banks), then every store covers 4 whole 128-byte row pieces of the
      // output (rows are Hq * head_dim apart)
      char* stg = sm.ostage[warp - 4];
      const size_t row_w = row_out - (size_t)lane * Hq;  // the warp's first query row
      uint32_t o[kHD];
#pragma unroll
      for (int cc = 0; cc < kHD; cc += 32) tmem_ld32(lane_addr + colO + cc, o + cc);
      tmem_wait_ld();
#pragma unroll
      for (int pass = 0; pass < 2; ++pass) {
        const uint32_t* oh = o + pass * 64;
#pragma unroll
        for (int pc = 0; pc < 8; ++pc) {
          const uint32_t* v = oh + pc * 8;
          uint4 pkt;
          pkt.x = pack_bf16(__uint_as_float(v[0]) * inv, __uint_as_float(v[1]) * inv);
          pkt.y = pack_bf16(__uint_as_float(v[2]) * inv, __uint_as_float(v[3]) * inv);
          pkt.z = pack_bf16(__uint_as_float(v[4]) * inv, __uint_as_float(v[5]) * inv);
          pkt.w = pack_bf16(__uint_as_float(v[6]) * inv, __uint_as_float(v[7]) * inv);
          *reinterpret_cast<uint4*>(stg + lane * 128 + ((pc ^ (lane & 7)) << 4)) = pkt;
        }
        __syncwarp();
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int rr = k * 4 + (lane >> 3), pc = lane & 7;
          const uint4 v = *reinterpret_cast<const uint4*>(stg + rr * 128 + ((pc ^ (rr & 7)) << 4));
          *reinterpret_cast<uint4*>(out + (row_w + (size_t)rr * Hq) * kHD + pass * 64 + pc * 8) = v;
        }
        __syncwarp();  // the tile is refilled by the next pass
      }
      if (lse_out) lse_out[row_out] = l > 0.f ? (m + log2f(l)) * kLn2 : -INFINITY;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
  }
}

// ---- host: tensor maps -------------------------------------------------------------------

constexpr size_t kSmem = sizeof(TcSmem) + 1024;  // + alignment slack
static_assert(kSmem <= 232448, "shared memory of one CTA (227 KB on sm_100)");

template <bool SOFT>
cudaError_t configure() {
  return ensure_dynamic_smem((const void*)prefill_tc_kernel<SOFT>, (int)kSmem);
}

}  // namespace

bool prefill_tc_supported(const spkv_params& p, const spkv_cache& c, int chunk_start, int chunk_len) {
  (void)c;
  const int G = p.Hq / p.Hkv;
  return p.dtype == SPKV_BF16 && p.head_dim == kHD && p.window == kWin && G % 2 == 0 &&
         chunk_start % kQT == 0 && chunk_len % kQT == 0 && chunk_len > 0 && encode_fn() != nullptr;
}

cudaError_t launch_prefill_tc(const spkv_params& p, const spkv_cache& c, const spkv_ring& ring,
                              const void* q, const void* K_chunk, const void* V_chunk,
                              int chunk_start, int chunk_len, void* o, float* lse, int* sched,
                              cudaStream_t stream) {
  const int G = p.Hq / p.Hkv;
  const cuuint64_t e = 2;  // bytes per element
  CUtensorMap tq, tkc, tvc, tkp, tvp, tkr, tvr;
  {
    const cuuint64_t dims[4] = {(cuuint64_t)kHD, (cuuint64_t)p.Hq, (cuuint64_t)chunk_len, (cuuint64_t)p.B};
    const cuuint64_t str[3] = {kHD * e, (cuuint64_t)p.Hq * kHD * e, (cuuint64_t)chunk_len * p.Hq * kHD * e};
    const cuuint32_t box[4] = {64, 1, kQT, 1};
    if (!make_map(&tq, q, 4, dims, str, box)) return cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[4] = {(cuuint64_t)kHD, (cuuint64_t)p.Hkv, (cuuint64_t)chunk_len, (cuuint64_t)p.B};
    const cuuint64_t str[3] = {kHD * e, (cuuint64_t)p.Hkv * kHD * e, (cuuint64_t)chunk_len * p.Hkv * kHD * e};
    const cuuint32_t box[4] = {64, 1, kKB, 1};
    if (!make_map(&tkc, K_chunk, 4, dims, str, box) || !make_map(&tvc, V_chunk, 4, dims, str, box))
      return cudaErrorInvalidValue;
  }
  if (c.K_pool) {  // one 64-row page per box
    const cuuint64_t dims[2] = {(cuuint64_t)kHD, (cuuint64_t)c.num_pages * kPageRows};
    const cuuint64_t str[1] = {kHD * e};
    const cuuint32_t box[2] = {64, kPageRows};
    if (!make_map(&tkp, c.K_pool, 2, dims, str, box) || !make_map(&tvp, c.V_pool, 2, dims, str, box))
      return cudaErrorInvalidValue;
  } else {  // window-only layer: no cache block is ever loaded
    tkp = tkc;
    tvp = tvc;
  }
  {  // the whole window of one (batch row, key head) per box
    const cuuint64_t dims[4] = {(cuuint64_t)kHD, (cuuint64_t)kWin, (cuuint64_t)p.Hkv, (cuuint64_t)p.B};
    const cuuint64_t str[3] = {kHD * e, (cuuint64_t)kWin * kHD * e, (cuuint64_t)p.Hkv * kWin * kHD * e};
    const cuuint32_t box[4] = {64, kKB, 1, 1};
    if (!make_map(&tkr, ring.K_win, 4, dims, str, box) || !make_map(&tvr, ring.V_win, 4, dims, str, box))
      return cudaErrorInvalidValue;
  }
  cudaError_t e2 = configure<false>();
  if (e2 != cudaSuccess) return e2;
  CacheView cv = cache_view(c);
  const int n_qt = chunk_len / kQT, n_hp = G / 2, n_bh = p.B * p.Hkv;
  const int n_tiles = n_qt * n_hp * n_bh;
  const int sms = sm_count();
  if (sms <= 0) return cudaErrorInvalidValue;
  prefill_tc_kernel<false><<<n_tiles < sms ? n_tiles : sms, kThr, kSmem, stream>>>(
      tq, tkc, tvc, tkp, tvp, tkr, tvr, cv, c.K_pool ? c.num_pages : 0,
      static_cast<__nv_bfloat16*>(o), lse, chunk_start, chunk_len, p.Hkv, G, n_qt, n_hp, n_bh,
      c.err_flag, nullptr, sched);
  return cudaGetLastError();
}

bool soft_tc_supported(const spkv_params& p, int seq_len) {
  const int G = p.Hq / p.Hkv;
  return p.dtype == SPKV_BF16 && p.head_dim == kHD && p.window == kWin && G % 2 == 0 &&
         seq_len % kQT == 0 && seq_len > 0 && encode_fn() != nullptr;
}

cudaError_t launch_soft_tc(const spkv_params& p, const void* q, const void* K, const void* V,
                           const float* bias, int seq_len, void* o, float* lse, uint32_t* err,
                           cudaStream_t stream) {
  const int G = p.Hq / p.Hkv;
  const cuuint64_t e = 2;
  CUtensorMap tq, tk, tv;
  {
    const cuuint64_t dims[4] = {(cuuint64_t)kHD, (cuuint64_t)p.Hq, (cuuint64_t)seq_len, (cuuint64_t)p.B};
    const cuuint64_t str[3] = {kHD * e, (cuuint64_t)p.Hq * kHD * e, (cuuint64_t)seq_len * p.Hq * kHD * e};
    const cuuint32_t box[4] = {64, 1, kQT, 1};
    if (!make_map(&tq, q, 4, dims, str, box)) return cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[4] = {(cuuint64_t)kHD, (cuuint64_t)p.Hkv, (cuuint64_t)seq_len, (cuuint64_t)p.B};
    const cuuint64_t str[3] = {kHD * e, (cuuint64_t)p.Hkv * kHD * e, (cuuint64_t)seq_len * p.Hkv * kHD * e};
    const cuuint32_t box[4] = {64, 1, kKB, 1};
    if (!make_map(&tk, K, 4, dims, str, box) || !make_map(&tv, V, 4, dims, str, box))
      return cudaErrorInvalidValue;
  }
  cudaError_t e2 = configure<true>();
  if (e2 != cudaSuccess) return e2;
  CacheView cv{nullptr, nullptr, nullptr, nullptr, nullptr, 0, 0, nullptr};
  const int n_qt = seq_len / kQT, n_hp = G / 2, n_bh = p.B * p.Hkv;
  const int n_tiles = n_qt * n_hp * n_bh;
  const int sms = sm_count();
  if (sms <= 0) return cudaErrorInvalidValue;
  // the cache and ring maps are not read in this mode: the sequence maps stand in
  prefill_tc_kernel<true><<<n_tiles < sms ? n_tiles : sms, kThr, kSmem, stream>>>(
      tq, tk, tv, tk, tv, tk, tv, cv, 0, static_cast<__nv_bfloat16*>(o), lse, 0, seq_len, p.Hkv,
      G, n_qt, n_hp, n_bh, err, bias, nullptr);
  return cudaGetLastError();
}

}  // namespace spkv
