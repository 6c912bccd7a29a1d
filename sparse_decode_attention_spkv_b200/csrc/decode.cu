// decode.cu -- a4 + a5: gated decode attention with split-K and a log-sum-exp merge.
//
// "Self-Pruned Key-Value Attention" (arXiv 2605.14037), §2.1, Eqs. (3)-(4): the
// query at position t attends to the keys in its causal window (0 <= t-s < w) and
// to the gated-in keys (z_s = 1, s <= t).  At deployment (§2.1) the gated keys
// live in the compacted per-head cache, so the key set of one (batch row, key
// head) is: cache rows with position <= t-w, then the window slots.  Decode reads
// the whole of that set once per step, which is why the paper's kernel is memory
// bound and lower density gives lower latency (§3.4, Fig. 3 right).
//
// Design (CUDA cores; decode is ~2 FMA per byte of K/V):
//  * Virtual rows of head bh: [0, roundup64(n_live)) cache rows (page k = rows
//    64k..64k+63), then [.., + n_win) window slots.  Rows are cut into equal
//    chunks sized so that all heads together give a few chunks per CTA; CTAs
//    (one per SM) pull chunks from an atomic counter, so ragged heads balance.
//  * Per CTA, one producer warp streams 64-row K and V tiles with 1-D bulk
//    async copies (cp.async.bulk, mbarrier completion) into a 4-stage ring in
//    shared memory; 8 consumer warps compute from shared memory.
//  * A row is read by LPR lanes (16 for a 256-byte row), 16 bytes each.  Scores
//    for all G query heads of the group are formed with packed fp32 FMAs and
//    reduced across the lane group by a transposing butterfly (one shuffle per
//    value), softmax runs in the log2 domain with a running max that is raised
//    only when a score exceeds it by more than 8 (so p <= 256), and P*V is
//    accumulated in registers.
//  * End of a chunk: the 8 warps combine through shared memory; a head that
//    spans several chunks writes (o, m, l) partials, and the CTA that finishes
//    its last chunk (atomic arrival count) merges them: o = sum_i e^{m_i-m} o_i /
//    sum_i e^{m_i-m} l_i.
#include <math.h>

#include "common.cuh"
#include "host.h"
#include "launch.h"

namespace spkv {
namespace {

constexpr int kTileRows = 64;
constexpr int kConsumerWarps = 8;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kUnitsPerCta = 8;   // target chunks per CTA
constexpr int kMaxHeads = 2048;   // B * Hkv per launch
constexpr float kRescaleSlack = 8.f;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

template <typename E, int D>
struct Geo {
  static constexpr int kRowBytes = D * E::kSize;
  static constexpr int kLPR = kRowBytes / 16;  // lanes per row
  static constexpr int kEPL = 16 / E::kSize;   // elements per lane
  static constexpr int kRPW = 32 / kLPR;       // rows per warp step
  static constexpr int kSteps = kTileRows / (kConsumerWarps * kRPW);
  static constexpr int kTileBytes = kTileRows * kRowBytes;
  static constexpr int kStages = (2 * kTileBytes <= 32768) ? 4 : 2;  // <= 128 KB of tiles
  static_assert(kLPR >= 2 && kLPR <= 32, "row must be 32..512 bytes");
  static_assert(kSteps >= 1, "tile too small");
};

// Transposing butterfly: N values per lane reduced across the lanes that differ
// in bits M, M/2, .., 1.  While N >= 2 each step halves the vector (one shuffle
// per kept value); afterwards it is a plain butterfly.
template <int N, int M>
__device__ __forceinline__ void xreduce(float* v, int lane) {
  if constexpr (M >= 1) {
    if constexpr (N >= 2) {
      const bool upper = (lane & M) != 0;
#pragma unroll
      for (int i = 0; i < N / 2; ++i) {
        const float send = upper ? v[i] : v[i + N / 2];
        const float keep = upper ? v[i + N / 2] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, M);
      }
      xreduce<N / 2, M / 2>(v, lane);
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], M);
      xreduce<1, M / 2>(v, lane);
    }
  }
}

// Index (into the original N values) of the first value a lane keeps.
template <int N, int M>
__device__ __forceinline__ int xindex(int lane) {
  if constexpr (M >= 1 && N >= 2) {
    return ((lane & M) ? N / 2 : 0) + xindex<N / 2, M / 2>(lane);
  } else {
    return 0;
  }
}

struct TileInfo {
  int chunk;  // -1: no more work
  int bh;
  int tile;   // virtual tile index within the head
  int valid;  // valid rows in the tile
  int last;   // last tile of its chunk
};

struct Plan {
  int* rows;   // [H] virtual rows per head
  int* live;   // [H] live cache rows per head
  int* base;   // [H+1] first chunk of each head
  int chunk_rows;
  int total_chunks;
};

template <typename E, int D, int G>
struct Smem {
  using Gm = Geo<E, D>;
  alignas(128) char K[Gm::kStages][Gm::kTileBytes];
  alignas(128) char V[Gm::kStages][Gm::kTileBytes];
  float red_o[kConsumerWarps][G][D];
  float red_m[kConsumerWarps][G];
  float red_l[kConsumerWarps][G];
  float pbuf[kConsumerWarps][Gm::kRPW][Gm::kSteps * G];
  uint64_t full[Gm::kStages];
  uint64_t empty[Gm::kStages];
  TileInfo info[Gm::kStages];
  int rows[kMaxHeads];
  int live[kMaxHeads];
  int base[kMaxHeads + 1];
  int scan_tmp[kThreads];
  int misc[4];
};

template <typename E, int D, int G>
__global__ void __launch_bounds__(kThreads, 1)
    decode_kernel(CacheView cache, const char* __restrict__ Kwin, const char* __restrict__ Vwin,
                  const typename E::T* __restrict__ q, const int32_t* __restrict__ t_pos,
                  typename E::T* __restrict__ out, float* __restrict__ lse_out,
                  int* __restrict__ ws_ctrl, float* __restrict__ ws_ml, float* __restrict__ ws_o,
                  int n_heads, int hkv, int window, float qscale, uint32_t* err) {
  using Gm = Geo<E, D>;
  using S = Smem<E, D, G>;
  extern __shared__ __align__(128) char smem_raw[];
  S& sm = *reinterpret_cast<S*>(smem_raw);
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  int* counters = ws_ctrl;              // [n_heads] per-head arrival counts
  int* next_chunk = ws_ctrl + n_heads;  // work counter
  int* done_ctas = ws_ctrl + n_heads + 1;

  // ---- plan: rows per head, chunk size, chunk prefix (every CTA, same result) --
  int my_rows = 0;
  for (int bh = tid; bh < n_heads; bh += kThreads) {
    const int b = bh / hkv;
    const int t = __ldg(t_pos + b);
    const int nl = cache_live_rows(cache, bh, t - window, window);
    const int nw = t + 1 < window ? t + 1 : window;
    const int rows = ((nl + kTileRows - 1) / kTileRows) * kTileRows + nw;
    sm.live[bh] = nl;
    sm.rows[bh] = rows;
    my_rows += rows;
  }
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) my_rows += __shfl_xor_sync(0xffffffffu, my_rows, m);
  if (lane == 0) sm.scan_tmp[warp] = my_rows;
  __syncthreads();
  if (tid == 0) {
    long long total = 0;
    for (int w = 0; w < kThreads / 32; ++w) total += sm.scan_tmp[w];
    const long long units = (long long)gridDim.x * kUnitsPerCta;
    long long cr = (total + units - 1) / units;
    cr = ((cr + kTileRows - 1) / kTileRows) * kTileRows;
    if (cr < kTileRows) cr = kTileRows;
    sm.misc[0] = (int)cr;
  }
  __syncthreads();
  const int chunk_rows = sm.misc[0];
  // exclusive scan of chunks per head: each thread owns a contiguous segment
  {
    const int per = (n_heads + kThreads - 1) / kThreads;
    const int lo = tid * per;
    const int hi = lo + per < n_heads ? lo + per : n_heads;
    int s = 0;
    for (int bh = lo; bh < hi; ++bh) s += (sm.rows[bh] + chunk_rows - 1) / chunk_rows;
    sm.scan_tmp[tid] = s;
    __syncthreads();
    if (tid == 0) {
      int acc = 0;
      for (int i = 0; i < kThreads; ++i) {
        const int v = sm.scan_tmp[i];
        sm.scan_tmp[i] = acc;
        acc += v;
      }
      sm.base[n_heads] = acc;
    }
    __syncthreads();
    int acc = sm.scan_tmp[tid];
    for (int bh = lo; bh < hi; ++bh) {
      sm.base[bh] = acc;
      acc += (sm.rows[bh] + chunk_rows - 1) / chunk_rows;
    }
  }
  if (tid == 0) {
    for (int s = 0; s < Gm::kStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], kConsumerWarps);
    }
    fence_mbar_init();
  }
  __syncthreads();
  const int total_chunks = sm.base[n_heads];

  if (warp == kConsumerWarps) {
    // ------------------------------ producer ------------------------------------
    if (lane == 0) {
      int it = 0;
      for (;;) {
        const int c = atomicAdd(next_chunk, 1);
        if (c >= total_chunks) break;
        int lo = 0, hi = n_heads - 1;  // last head with base <= c
        while (lo < hi) {
          const int mid = (lo + hi + 1) >> 1;
          if (sm.base[mid] <= c) lo = mid; else hi = mid - 1;
        }
        const int bh = lo;
        const int lc = c - sm.base[bh];
        const int r0 = lc * chunk_rows;
        const int r1 = min(sm.rows[bh], r0 + chunk_rows);
        const int nl = sm.live[bh];
        const int nlp = ((nl + kTileRows - 1) / kTileRows) * kTileRows;
        const int b = bh / hkv;
        const int t = __ldg(t_pos + b);
        const int nw = t + 1 < window ? t + 1 : window;
        const int k0 = r0 / kTileRows, k1 = (r1 + kTileRows - 1) / kTileRows;
        for (int k = k0; k < k1; ++k, ++it) {
          const int s = it % Gm::kStages;
          const uint32_t ph = (it / Gm::kStages) & 1;
          mbar_wait(&sm.empty[s], ph ^ 1, err);
          const char* srcK;
          const char* srcV;
          int valid;
          if (k * kTileRows < nlp) {
            int page = __ldg(cache.page_table + (size_t)bh * cache.max_pages + k);
            if (!page_ok(page, cache.num_pages, err)) page = 0;  // debug build: flagged
            valid = min(kTileRows, nl - k * kTileRows);
            srcK = cache.K + (size_t)page * Gm::kTileBytes;
            srcV = cache.V + (size_t)page * Gm::kTileBytes;
          } else {
            const int j = k - nlp / kTileRows;
            valid = min(kTileRows, nw - j * kTileRows);
            const size_t row = (size_t)bh * window + (size_t)j * kTileRows;
            srcK = Kwin + row * Gm::kRowBytes;
            srcV = Vwin + row * Gm::kRowBytes;
          }
          sm.info[s] = TileInfo{c, bh, k, valid, k == k1 - 1};
          const uint32_t bytes = (uint32_t)valid * Gm::kRowBytes;
          mbar_arrive_expect_tx(&sm.full[s], 2 * bytes);
          bulk_g2s(sm.K[s], srcK, bytes, &sm.full[s]);
          bulk_g2s(sm.V[s], srcV, bytes, &sm.full[s]);
        }
      }
      const int s = it % Gm::kStages;
      const uint32_t ph = (it / Gm::kStages) & 1;
      mbar_wait(&sm.empty[s], ph ^ 1, err);
      sm.info[s].chunk = -1;
      mbar_arrive(&sm.full[s]);
    }
  } else {
    // ------------------------------ consumers -----------------------------------
    constexpr int LPR = Gm::kLPR, EPL = Gm::kEPL, RPW = Gm::kRPW, STEPS = Gm::kSteps;
    constexpr int N = STEPS * G;                 // partial dots per lane per tile
    constexpr int R = N >= LPR ? N / LPR : 1;    // values a lane keeps after the reduce
    constexpr int REPL = N >= LPR ? 1 : LPR / N; // lanes sharing one value
    const int grp = lane / LPR;                  // row group within the warp
    const int col = lane % LPR;                  // 16-byte column
    const int xbase = xindex<N, LPR / 2>(col);
    const bool owner = (col & (REPL - 1)) == 0;
    int gsel[R];
#pragma unroll
    for (int j = 0; j < R; ++j) gsel[j] = (xbase + j) % G;

    float2 qf[G][EPL / 2];
    float2 acc[G][EPL / 2];
    float m_run[G];
    float m_mine[R], l_mine[R];
    int cur = -1, cur_bh = 0;
    int it = 0;
    for (;;) {
      const int s = it % Gm::kStages;
      const uint32_t ph = (it / Gm::kStages) & 1;
      mbar_wait(&sm.full[s], ph, err);
      const TileInfo ti = sm.info[s];
      if (ti.chunk < 0) break;
      if (ti.chunk != cur) {
        cur = ti.chunk;
        cur_bh = ti.bh;
        const int b = cur_bh / hkv, kh = cur_bh % hkv;
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const uint4 raw = *reinterpret_cast<const uint4*>(
              q + ((size_t)b * hkv * G + (size_t)kh * G + g) * D + col * EPL);
          float f[EPL];
          Vec<E>::widen(raw, f);
#pragma unroll
          for (int e = 0; e < EPL / 2; ++e) {
            qf[g][e] = make_float2(f[2 * e] * qscale, f[2 * e + 1] * qscale);
            acc[g][e] = make_float2(0.f, 0.f);
          }
          m_run[g] = -INFINITY;
        }
#pragma unroll
        for (int j = 0; j < R; ++j) {
          m_mine[j] = -INFINITY;
          l_mine[j] = 0.f;
        }
      }
      const char* Ks = sm.K[s];
      const char* Vs = sm.V[s];

      // scores
      float sc[N];
#pragma unroll
      for (int st = 0; st < STEPS; ++st) {
        const int r = (st * kConsumerWarps + warp) * RPW + grp;
        const uint4 raw = *reinterpret_cast<const uint4*>(Ks + r * Gm::kRowBytes + col * 16);
        float f[EPL];
        Vec<E>::widen(raw, f);
#pragma unroll
        for (int g = 0; g < G; ++g) {
          float2 a = make_float2(0.f, 0.f);
#pragma unroll
          for (int e = 0; e < EPL / 2; ++e) a = fma2(make_float2(f[2 * e], f[2 * e + 1]), qf[g][e], a);
          sc[st * G + g] = a.x + a.y;
        }
      }
      xreduce<N, LPR / 2>(sc, col);
      // mask invalid rows, test whether the running max must rise
      bool raise = false;
#pragma unroll
      for (int j = 0; j < R; ++j) {
        const int st = (xbase + j) / G;
        const int r = (st * kConsumerWarps + warp) * RPW + grp;
        if (r >= ti.valid) sc[j] = -INFINITY;
        raise |= sc[j] > m_mine[j] + kRescaleSlack;
      }
      if (__any_sync(0xffffffffu, raise)) {
        float mx[G];
#pragma unroll
        for (int g = 0; g < G; ++g) mx[g] = -INFINITY;
#pragma unroll
        for (int j = 0; j < R; ++j)
#pragma unroll
          for (int g = 0; g < G; ++g)
            if (gsel[j] == g) mx[g] = fmaxf(mx[g], sc[j]);
#pragma unroll
        for (int g = 0; g < G; ++g) {
#pragma unroll
          for (int m = 16; m > 0; m >>= 1) mx[g] = fmaxf(mx[g], __shfl_xor_sync(0xffffffffu, mx[g], m));
          const float mnew = fmaxf(m_run[g], mx[g]);
          const float alpha = (m_run[g] == -INFINITY) ? 0.f : exp2f(m_run[g] - mnew);
#pragma unroll
          for (int e = 0; e < EPL / 2; ++e) acc[g][e] = mul2(acc[g][e], make_float2(alpha, alpha));
#pragma unroll
          for (int j = 0; j < R; ++j)
            if (gsel[j] == g) l_mine[j] *= alpha;
          m_run[g] = mnew;
        }
#pragma unroll
        for (int j = 0; j < R; ++j)
#pragma unroll
          for (int g = 0; g < G; ++g)
            if (gsel[j] == g) m_mine[j] = m_run[g];
      }
      // probabilities -> shared memory (one value per owner lane)
#pragma unroll
      for (int j = 0; j < R; ++j) {
        const float pj = (sc[j] == -INFINITY) ? 0.f : exp2f(sc[j] - m_mine[j]);
        if (owner) l_mine[j] += pj;
        sm.pbuf[warp][grp][xbase + j] = pj;
      }
      __syncwarp();
      // P * V
#pragma unroll
      for (int st = 0; st < STEPS; ++st) {
        const int r = (st * kConsumerWarps + warp) * RPW + grp;
        float pv[G];
#pragma unroll
        for (int g = 0; g < G; ++g) pv[g] = sm.pbuf[warp][grp][st * G + g];
        uint4 raw = *reinterpret_cast<const uint4*>(Vs + r * Gm::kRowBytes + col * 16);
        if (r >= ti.valid) raw = make_uint4(0u, 0u, 0u, 0u);
        float f[EPL];
        Vec<E>::widen(raw, f);
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
          for (int e = 0; e < EPL / 2; ++e)
            acc[g][e] = fma2(make_float2(f[2 * e], f[2 * e + 1]), make_float2(pv[g], pv[g]), acc[g][e]);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.empty[s]);
      ++it;

      if (ti.last) {
        // ---- finish the chunk: warp -> CTA combine ----------------------------
#pragma unroll
        for (int m = LPR; m < 32; m <<= 1)
#pragma unroll
          for (int g = 0; g < G; ++g)
#pragma unroll
            for (int e = 0; e < EPL / 2; ++e) {
              acc[g][e].x += __shfl_xor_sync(0xffffffffu, acc[g][e].x, m);
              acc[g][e].y += __shfl_xor_sync(0xffffffffu, acc[g][e].y, m);
            }
        float lsum[G];
#pragma unroll
        for (int g = 0; g < G; ++g) {
          lsum[g] = 0.f;
#pragma unroll
          for (int j = 0; j < R; ++j)
            if (gsel[j] == g) lsum[g] += l_mine[j];
#pragma unroll
          for (int m = 16; m > 0; m >>= 1) lsum[g] += __shfl_xor_sync(0xffffffffu, lsum[g], m);
        }
        if (lane < LPR) {
#pragma unroll
          for (int g = 0; g < G; ++g)
#pragma unroll
            for (int e = 0; e < EPL / 2; ++e) {
              sm.red_o[warp][g][col * EPL + 2 * e] = acc[g][e].x;
              sm.red_o[warp][g][col * EPL + 2 * e + 1] = acc[g][e].y;
            }
        }
        if (lane == 0) {
#pragma unroll
          for (int g = 0; g < G; ++g) {
            sm.red_m[warp][g] = m_run[g];
            sm.red_l[warp][g] = lsum[g];
          }
        }
        named_bar_sync(1, kConsumerWarps * 32);
        const int bh = cur_bh;
        const int b = bh / hkv, kh = bh % hkv;
        const int nch = sm.base[bh + 1] - sm.base[bh];
        const int slot = cur;  // global chunk index = partial slot
        constexpr int CT = kConsumerWarps * 32;
        for (int e = tid; e < G * D; e += CT) {
          const int g = e / D, d = e % D;
          float M = -INFINITY;
#pragma unroll
          for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, sm.red_m[w][g]);
          float O = 0.f, L = 0.f;
#pragma unroll
          for (int w = 0; w < kConsumerWarps; ++w) {
            const float mw = sm.red_m[w][g];
            const float sc_w = (mw == -INFINITY) ? 0.f : exp2f(mw - M);
            O += sc_w * sm.red_o[w][g][d];
            L += sc_w * sm.red_l[w][g];
          }
          if (nch == 1) {
            const size_t oi = ((size_t)b * hkv * G + (size_t)kh * G + g) * D + d;
            from_f32(L > 0.f ? O / L : 0.f, out + oi);
            if (d == 0 && lse_out)
              lse_out[(size_t)b * hkv * G + kh * G + g] = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
          } else {
            ws_o[((size_t)slot * G + g) * D + d] = O;
            if (d == 0) {
              ws_ml[((size_t)slot * G + g) * 2 + 0] = M;
              ws_ml[((size_t)slot * G + g) * 2 + 1] = L;
            }
          }
        }
        if (nch > 1) {
          __threadfence();
          named_bar_sync(1, kConsumerWarps * 32);
          if (tid == 0) {
            const int prev = atomicAdd(counters + bh, 1);
            const int last = (prev == nch - 1);
            if (last) counters[bh] = 0;
            sm.misc[1] = last;
          }
          named_bar_sync(1, kConsumerWarps * 32);
          if (sm.misc[1]) {
            __threadfence();
            const int c0 = sm.base[bh];
            for (int e = tid; e < G * D; e += CT) {
              const int g = e / D, d = e % D;
              float M = -INFINITY;
              for (int c = 0; c < nch; ++c) M = fmaxf(M, __ldcg(ws_ml + ((size_t)(c0 + c) * G + g) * 2));
              float O = 0.f, L = 0.f;
              for (int c = 0; c < nch; ++c) {
                const float mc = __ldcg(ws_ml + ((size_t)(c0 + c) * G + g) * 2);
                const float w_c = (mc == -INFINITY) ? 0.f : exp2f(mc - M);
                O += w_c * __ldcg(ws_o + ((size_t)(c0 + c) * G + g) * D + d);
                L += w_c * __ldcg(ws_ml + ((size_t)(c0 + c) * G + g) * 2 + 1);
              }
              const size_t oi = ((size_t)b * hkv * G + (size_t)kh * G + g) * D + d;
              from_f32(L > 0.f ? O / L : 0.f, out + oi);
              if (d == 0 && lse_out)
                lse_out[(size_t)b * hkv * G + kh * G + g] = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
            }
          }
        }
        named_bar_sync(1, kConsumerWarps * 32);  // red_* reused by the next chunk
      }
    }
  }
  __syncthreads();
  if (tid == 0) {
    const int d = atomicAdd(done_ctas, 1);
    if (d == (int)gridDim.x - 1) {  // every CTA has stopped pulling work
      *next_chunk = 0;
      *done_ctas = 0;
    }
  }
}

// Control words at the front of the CUDA-core kernel's workspace: per-head arrival
// counters [n_heads], work counter, finished-CTA counter.
size_t ctrl_bytes_simple(int n_heads) { return ((size_t)(n_heads + 2) * 4 + 255) / 256 * 256; }

template <typename E, int D, int G>
cudaError_t run(const spkv_params& p, const spkv_cache& c, const spkv_ring& ring, const void* q,
                const int32_t* t_pos, void* o, float* lse, void* ws, int num_sms,
                cudaStream_t stream) {
  using S = Smem<E, D, G>;
  const size_t smem = sizeof(S);
  {
    cudaError_t e = ensure_dynamic_smem((const void*)decode_kernel<E, D, G>, (int)smem);
    if (e != cudaSuccess) return e;
  }
  const int n_heads = p.B * p.Hkv;
  char* w = static_cast<char*>(ws);
  int* ctrl = reinterpret_cast<int*>(w);
  const size_t ctrl_bytes = ctrl_bytes_simple(n_heads);
  const int grid = num_sms;
  const size_t max_chunks = (size_t)grid * kUnitsPerCta + n_heads;
  float* ml = reinterpret_cast<float*>(w + ctrl_bytes);
  const size_t ml_bytes = (max_chunks * G * 2 * 4 + 255) / 256 * 256;
  float* po = reinterpret_cast<float*>(w + ctrl_bytes + ml_bytes);
  CacheView cv = cache_view(c);
  const float qscale = kLog2e / sqrtf((float)D);
  decode_kernel<E, D, G><<<grid, kThreads, smem, stream>>>(
      cv, static_cast<const char*>(ring.K_win), static_cast<const char*>(ring.V_win),
      static_cast<const typename E::T*>(q), t_pos, static_cast<typename E::T*>(o), lse, ctrl, ml,
      po, n_heads, p.Hkv, p.window, qscale, c.err_flag);
  return cudaGetLastError();
}

template <typename E, int D>
cudaError_t dispatch_g(const spkv_params& p, const spkv_cache& c, const spkv_ring& ring,
                       const void* q, const int32_t* t_pos, void* o, float* lse, void* ws,
                       int num_sms, cudaStream_t stream) {
  switch (p.Hq / p.Hkv) {
    case 1: return run<E, D, 1>(p, c, ring, q, t_pos, o, lse, ws, num_sms, stream);
    case 2: return run<E, D, 2>(p, c, ring, q, t_pos, o, lse, ws, num_sms, stream);
    case 4: return run<E, D, 4>(p, c, ring, q, t_pos, o, lse, ws, num_sms, stream);
    case 8: return run<E, D, 8>(p, c, ring, q, t_pos, o, lse, ws, num_sms, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

size_t decode_ctrl_bytes(const spkv_params& p) {
  return decode_tc_supported(p) ? decode_tc_ctrl_bytes(p) : ctrl_bytes_simple(p.B * p.Hkv);
}

size_t decode_workspace_bytes(const spkv_params& p, int num_sms) {
  const int n_heads = p.B * p.Hkv;
  const int G = p.Hq / p.Hkv;
  const size_t ctrl_bytes = ctrl_bytes_simple(n_heads);
  const size_t max_chunks = (size_t)num_sms * kUnitsPerCta + n_heads;
  const size_t ml_bytes = (max_chunks * G * 2 * 4 + 255) / 256 * 256;
  const size_t o_bytes = max_chunks * G * p.head_dim * 4;
  const size_t tc = decode_tc_workspace_bytes(p, num_sms);
  return ctrl_bytes + ml_bytes + o_bytes > tc ? ctrl_bytes + ml_bytes + o_bytes : tc;
}

cudaError_t launch_decode(const spkv_params& p, const spkv_cache& c, const spkv_ring& ring,
                          const void* q, const int32_t* t_pos, void* o, float* lse,
                          void* workspace, size_t ws_bytes, int num_sms, cudaStream_t stream) {
  if (p.B * p.Hkv > kMaxHeads) return cudaErrorInvalidValue;
  if (ws_bytes < decode_workspace_bytes(p, num_sms)) return cudaErrorInvalidValue;
  if (decode_tc_supported(p))
    return launch_decode_tc(p, c, ring, q, t_pos, o, lse, workspace, num_sms, stream);
  if (p.dtype == SPKV_BF16) {
    if (p.head_dim == 128) return dispatch_g<BF16, 128>(p, c, ring, q, t_pos, o, lse, workspace, num_sms, stream);
    if (p.head_dim == 64) return dispatch_g<BF16, 64>(p, c, ring, q, t_pos, o, lse, workspace, num_sms, stream);
  } else {
    if (p.head_dim == 128) return dispatch_g<F32, 128>(p, c, ring, q, t_pos, o, lse, workspace, num_sms, stream);
    if (p.head_dim == 64) return dispatch_g<F32, 64>(p, c, ring, q, t_pos, o, lse, workspace, num_sms, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace spkv
