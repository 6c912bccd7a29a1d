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
// Structure (one CTA per SM, 10 warps):
//  * Plan (every CTA, same result): live cache rows per head, rows rounded to
//    128-row tiles (two cache pages), chunk size so that all heads give ~8 chunks per
//    CTA, chunk prefix.  The producer pulls chunks from a global atomic counter, so
//    ragged heads balance.
//  * Producer warp: per tile, TMA boxes (64 rows x 64 bf16, 128B-swizzled) of K and V
//    from two cache pages or the ring into a ring of shared-memory stages; with a
//    chunk's first tile it also copies the chunk's G query rows (bulk copy).
//  * 8 consumer warps, 16 rows of each tile apiece: S = Q K^T with mma.m16n8k16 (Q rows
//    = the G heads, zero-padded to 16), fp32 softmax in the log2 domain (running max
//    raised only when exceeded by > 8), P re-packed in registers as the A operand of
//    O += P V (V via ldmatrix.trans).  When a chunk ends they leave their (o, m, l) in
//    shared memory for the finisher and go straight on with the next chunk.
//  * Finisher warp: combines the 8 warps' states; a head with one chunk gets o and lse
//    written, otherwise the chunk's partial goes to the workspace, and the finisher
//    that completes a head's last chunk (atomic count) merges all of them:
//    o = sum_i 2^{m_i-m} o_i / sum_i 2^{m_i-m} l_i.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math.h>

#include <mutex>

#include "common.cuh"
#include "launch.h"

namespace spkv {
namespace {

constexpr int kTileR = 128;          // rows per tile: two cache pages, or the whole window
constexpr int kCons = 8;             // consumer warps, 16 rows each
constexpr int kProducer = kCons;     // warp index of the producer
constexpr int kFinisher = kCons + 1; // warp index of the finisher
constexpr int kThreadsT = (kCons + 2) * 32;
constexpr int kConsThreads = kCons * 32;
constexpr int kUnitsPerCta = 8;      // target chunks per CTA
constexpr int kMaxHeadsT = 2048;
constexpr int kMergeBatch = 128;     // partials whose weights the finisher stages at once
constexpr int kSegTiles = 64;        // tiles whose page numbers the producer fetches at once
constexpr float kLog2eT = 1.4426950408889634f;
constexpr float kLn2T = 0.6931471805599453f;
constexpr float kSlackT = 8.f;

template <int D>
struct TileBuf {
  static constexpr int kHalves = D / 64;
  static constexpr int kHalfBytes = kTileR * 128;       // 128 rows x 128 B
  static constexpr int kBytes = kHalves * kHalfBytes;   // K (or V) of one tile
  alignas(1024) char k[kHalves][kHalfBytes];
  alignas(1024) char v[kHalves][kHalfBytes];
};

struct TileRef {
  int chunk;  // -1: no more work
  int bh;
  int valid;  // valid rows
  int qslot;  // query staging slot of the chunk
};

template <int D, int G, int NST>
struct TcDecSmem {
  TileBuf<D> st[NST];
  alignas(16) __nv_bfloat16 qbuf[2][G * D];
  float red_o[kCons][G][D];
  float red_m[kCons][G];
  float red_l[kCons][G];
  float fin_w[kMergeBatch * G];   // finisher: weights of a batch of partials
  int pages[2 * kSegTiles];       // producer: page numbers of a stretch of tiles
  uint64_t full[NST];
  uint64_t empty[NST];
  uint64_t q_free[2];
  uint64_t chunk_done;
  uint64_t red_free;
  TileRef info[NST];
  int red_chunk, red_bh;
  int red[kThreadsT];
  int misc[4];
  // followed (dynamic) by rows[n_heads], live[n_heads], base[n_heads + 1]
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

template <int D, int G, int NST>
__global__ void __launch_bounds__(kThreadsT, 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tm_kp,
                     const __grid_constant__ CUtensorMap tm_vp,
                     const __grid_constant__ CUtensorMap tm_kr,
                     const __grid_constant__ CUtensorMap tm_vr, CacheView cache,
                     const __nv_bfloat16* __restrict__ q, const int32_t* __restrict__ t_pos,
                     __nv_bfloat16* __restrict__ out, float* __restrict__ lse_out,
                     int* __restrict__ ws_ctrl, float* __restrict__ ws_ml,
                     float* __restrict__ ws_o, int n_heads, int hkv, int window,
                     uint32_t* err) {
  using TB = TileBuf<D>;
  using S = TcDecSmem<D, G, NST>;
  constexpr int NT_D = D / 8;     // n-tiles of 8 along head_dim
  constexpr int KS_D = D / 16;    // k-steps of 16 along head_dim
  extern __shared__ __align__(1024) char smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  S& sm = *reinterpret_cast<S*>(smem_raw + pad);
  int* s_rows = reinterpret_cast<int*>(smem_raw + pad + sizeof(S));
  int* s_live = s_rows + n_heads;
  int* s_base = s_live + n_heads;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int* counters = ws_ctrl;
  int* next_chunk = ws_ctrl + n_heads;
  int* done_ctas = ws_ctrl + n_heads + 1;

  // ---- plan (identical in every CTA) ---------------------------------------------
  int my_rows = 0;
  for (int bh = tid; bh < n_heads; bh += kThreadsT) {
    const int t = __ldg(t_pos + bh / hkv);
    const int nl = cache_live_rows(cache, bh, t - window, window);
    const int nw = t + 1 < window ? t + 1 : window;
    const int rows = ((nl + kTileR - 1) / kTileR) * kTileR + nw;
    s_live[bh] = nl;
    s_rows[bh] = rows;
    my_rows += rows;
  }
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) my_rows += __shfl_xor_sync(0xffffffffu, my_rows, m);
  if (lane == 0) sm.red[warp] = my_rows;
  if (tid == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], kCons);
    }
    mbar_init(&sm.q_free[0], kConsThreads);
    mbar_init(&sm.q_free[1], kConsThreads);
    mbar_init(&sm.chunk_done, kConsThreads);
    mbar_init(&sm.red_free, 32);
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
    const int per = (n_heads + kThreadsT - 1) / kThreadsT;
    const int lo = tid * per, hi = min(n_heads, lo + per);
    int s = 0;
    for (int bh = lo; bh < hi; ++bh) s += (s_rows[bh] + chunk_rows - 1) / chunk_rows;
    sm.red[tid] = s;
    __syncthreads();
    if (tid == 0) {
      int acc = 0;
      for (int i = 0; i < kThreadsT; ++i) {
        const int v = sm.red[i];
        sm.red[i] = acc;
        acc += v;
      }
      s_base[n_heads] = acc;
    }
    __syncthreads();
    int acc = sm.red[tid];
    for (int bh = lo; bh < hi; ++bh) {
      s_base[bh] = acc;
      acc += (s_rows[bh] + chunk_rows - 1) / chunk_rows;
    }
  }
  __syncthreads();
  const int total_chunks = s_base[n_heads];

  if (warp == kProducer) {
    // ------------------------------ producer ------------------------------------
    // The whole warp fetches a stretch of the chunk's page-table entries at once (one
    // round trip instead of one per tile); lane 0 then issues the copies.
    int it = 0;
    for (int seq = 0;; ++seq) {
      int c = 0;
      if (lane == 0) c = atomicAdd(next_chunk, 1);
      c = __shfl_sync(0xffffffffu, c, 0);
      if (c >= total_chunks) break;
      int lo = 0, hi = n_heads - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_base[mid] <= c) lo = mid; else hi = mid - 1;
      }
      const int bh = lo;
      const int r0 = (c - s_base[bh]) * chunk_rows;
      const int r1 = min(s_rows[bh], r0 + chunk_rows);
      const int nl = s_live[bh];
      const int nlp = ((nl + kTileR - 1) / kTileR) * kTileR;
      const int live_pages = (nl + kPageRows - 1) / kPageRows;
      const int b = bh / hkv, kh = bh % hkv;
      const int t = __ldg(t_pos + b);
      const int nw = t + 1 < window ? t + 1 : window;
      const int k0 = r0 / kTileR, k1 = (r1 + kTileR - 1) / kTileR;
      const int qslot = seq & 1;
      if (lane == 0) mbar_wait(&sm.q_free[qslot], ((seq >> 1) & 1) ^ 1, err);
      for (int ks = k0; ks < k1; ks += kSegTiles) {
        const int ke = min(k1, ks + kSegTiles);
        const int pg_lo = 2 * ks, pg_hi = min(2 * ke, live_pages);
        __syncwarp();
        for (int i = lane; i < pg_hi - pg_lo; i += 32)
          sm.pages[i] = __ldg(cache.page_table + (size_t)bh * cache.max_pages + pg_lo + i);
        __syncwarp();
        if (lane == 0) {
          for (int k = ks; k < ke; ++k, ++it) {
            const int s = it % NST;
            mbar_wait(&sm.empty[s], ((it / NST) & 1) ^ 1, err);
            TB& tb = sm.st[s];
            const bool from_cache = k * kTileR < nlp;
            const int slot = k * kTileR - nlp;
            const int valid = from_cache ? min(kTileR, nl - k * kTileR) : min(kTileR, nw - slot);
            // the tile description must be in place before the phase can complete
            sm.info[s] = TileRef{c, bh, valid, qslot};
            const bool first = k == k0;
            mbar_arrive_expect_tx(&sm.full[s], 2 * TB::kBytes + (first ? G * D * 2 : 0));
            if (first)
              bulk_g2s(sm.qbuf[qslot], q + ((size_t)b * hkv + kh) * G * D, G * D * 2, &sm.full[s]);
            if (from_cache) {
              const int pg0 = 2 * k;
              const int page0 = sm.pages[pg0 - pg_lo];
              // a missing second page is replaced by the first (its rows are masked)
              const int page1 = pg0 + 1 < live_pages ? sm.pages[pg0 + 1 - pg_lo] : page0;
#pragma unroll
              for (int hf = 0; hf < TB::kHalves; ++hf) {
                tma2d(tb.k[hf], &tm_kp, hf * 64, page0 * kPageRows, &sm.full[s]);
                tma2d(tb.k[hf] + 64 * 128, &tm_kp, hf * 64, page1 * kPageRows, &sm.full[s]);
                tma2d(tb.v[hf], &tm_vp, hf * 64, page0 * kPageRows, &sm.full[s]);
                tma2d(tb.v[hf] + 64 * 128, &tm_vp, hf * 64, page1 * kPageRows, &sm.full[s]);
              }
            } else {
#pragma unroll
              for (int hf = 0; hf < TB::kHalves; ++hf) {
                tma4d(tb.k[hf], &tm_kr, hf * 64, slot, kh, b, &sm.full[s]);
                tma4d(tb.v[hf], &tm_vr, hf * 64, slot, kh, b, &sm.full[s]);
              }
            }
          }
        }
        it = __shfl_sync(0xffffffffu, it, 0);
      }
    }
    if (lane == 0) {
      const int s = it % NST;
      mbar_wait(&sm.empty[s], ((it / NST) & 1) ^ 1, err);
      sm.info[s].chunk = -1;
      mbar_arrive(&sm.full[s]);
    }
  } else if (warp == kFinisher) {
    // ------------------------------ finisher ------------------------------------
    for (int n = 0;; ++n) {
      mbar_wait(&sm.chunk_done, n & 1, err);
      const int c = sm.red_chunk, bh = sm.red_bh;
      if (c < 0) break;
      const int b = bh / hkv, kh = bh % hkv;
      const size_t hrow = (size_t)b * hkv * G + (size_t)kh * G;
      const int nch = s_base[bh + 1] - s_base[bh];
      float Mg[G], Lg[G];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kCons; ++w) M = fmaxf(M, sm.red_m[w][g]);
        float L = 0.f;
#pragma unroll
        for (int w = 0; w < kCons; ++w) {
          const float mw = sm.red_m[w][g];
          L += (mw == -INFINITY ? 0.f : exp2f(mw - M)) * sm.red_l[w][g];
        }
        Mg[g] = M;
        Lg[g] = L;
      }
      for (int e = lane; e < G * D / 4; e += 32) {
        const int g = (e * 4) / D, d = (e * 4) % D;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int w = 0; w < kCons; ++w) {
          const float mw = sm.red_m[w][g];
          const float ww = mw == -INFINITY ? 0.f : exp2f(mw - Mg[g]);
          const float4 v = *reinterpret_cast<const float4*>(&sm.red_o[w][g][d]);
          acc.x += ww * v.x;
          acc.y += ww * v.y;
          acc.z += ww * v.z;
          acc.w += ww * v.w;
        }
        if (nch == 1) {
          const float L = Lg[g], inv = L > 0.f ? 1.f / L : 0.f;
          uint2 pk;
          pk.x = pack2(acc.x * inv, acc.y * inv);
          pk.y = pack2(acc.z * inv, acc.w * inv);
          *reinterpret_cast<uint2*>(out + (hrow + g) * D + d) = pk;
        } else {
          *reinterpret_cast<float4*>(ws_o + ((size_t)c * G + g) * D + d) = acc;
        }
      }
      if (nch == 1) {
        if (lane < G && lse_out)
          lse_out[hrow + lane] = Lg[lane] > 0.f ? (Mg[lane] + log2f(Lg[lane])) * kLn2T : -INFINITY;
      } else if (lane < G) {
        ws_ml[((size_t)c * G + lane) * 2 + 0] = Mg[lane];
        ws_ml[((size_t)c * G + lane) * 2 + 1] = Lg[lane];
      }
      mbar_arrive(&sm.red_free);  // the consumers may overwrite red_* now
      if (nch > 1) {
        __syncwarp();
        int last = 0;
        if (lane == 0) {
          __threadfence();
          const int prev = atomicAdd(counters + bh, 1);
          last = prev == nch - 1;
          if (last) counters[bh] = 0;
        }
        last = __shfl_sync(0xffffffffu, last, 0);
        if (last) {
          // ---- merge all partials of the head ----------------------------------------
          // Lane l works on the (chunk, head) pairs e = c*G + g with e = l (mod 32), so its
          // head is g = l % G throughout; the outputs (head g, 4 columns) are spread over
          // the lanes, and the chunk weights are staged in shared memory per batch.
          __threadfence();
          const size_t e0 = (size_t)s_base[bh] * G;
          float Mx = -INFINITY;
          for (int e = lane; e < nch * G; e += 32) Mx = fmaxf(Mx, __ldcg(ws_ml + (e0 + e) * 2));
#pragma unroll
          for (int m = G; m < 32; m <<= 1) Mx = fmaxf(Mx, __shfl_xor_sync(0xffffffffu, Mx, m));
          constexpr int kPairs = G * D / 4;           // (head, 4 columns) outputs
          constexpr int kPerLane = (kPairs + 31) / 32;
          float4 acc[kPerLane];
#pragma unroll
          for (int k = 0; k < kPerLane; ++k) acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
          float Lx = 0.f;
          for (int cb = 0; cb < nch; cb += kMergeBatch) {
            const int nb = min(kMergeBatch, nch - cb);
            for (int e = lane; e < nb * G; e += 32) {
              const size_t idx = (e0 + (size_t)cb * G + e) * 2;
              const float mc = __ldcg(ws_ml + idx);
              const float wc = mc == -INFINITY ? 0.f : exp2f(mc - Mx);
              sm.fin_w[e] = wc;
              Lx += wc * __ldcg(ws_ml + idx + 1);
            }
            __syncwarp();
#pragma unroll
            for (int k = 0; k < kPerLane; ++k) {
              const int pi = lane + 32 * k;
              if (pi < kPairs) {
                const int g = pi / (D / 4), d = (pi % (D / 4)) * 4;
                const float* src = ws_o + (e0 + (size_t)cb * G + g) * D + d;
#pragma unroll 4
                for (int c = 0; c < nb; ++c) {
                  const float wc = sm.fin_w[c * G + g];
                  const float4 v = __ldcg(reinterpret_cast<const float4*>(src + (size_t)c * G * D));
                  acc[k].x += wc * v.x;
                  acc[k].y += wc * v.y;
                  acc[k].z += wc * v.z;
                  acc[k].w += wc * v.w;
                }
              }
            }
            __syncwarp();
          }
#pragma unroll
          for (int m = G; m < 32; m <<= 1) Lx += __shfl_xor_sync(0xffffffffu, Lx, m);
#pragma unroll
          for (int k = 0; k < kPerLane; ++k) {
            const int pi = lane + 32 * k;
            const int g = (pi < kPairs ? pi : 0) / (D / 4);
            const float L = __shfl_sync(0xffffffffu, Lx, g);  // lane g holds head g's sum
            if (pi < kPairs) {
              const int d = (pi % (D / 4)) * 4;
              const float inv = L > 0.f ? 1.f / L : 0.f;
              uint2 pk;
              pk.x = pack2(acc[k].x * inv, acc[k].y * inv);
              pk.y = pack2(acc[k].z * inv, acc[k].w * inv);
              *reinterpret_cast<uint2*>(out + (hrow + g) * D + d) = pk;
            }
          }
          if (lane < G && lse_out)
            lse_out[hrow + lane] = Lx > 0.f ? (Mx + log2f(Lx)) * kLn2T : -INFINITY;
        }
      }
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
    int cur = -1, cur_bh = 0, n_ev = 0;
    // hand this warp's state of the finished chunk to the finisher
    auto dump = [&](int chunk, int bh) {
      mbar_wait(&sm.red_free, (n_ev & 1) ^ 1, err);
      float l = l_run;
      l += __shfl_xor_sync(0xffffffffu, l, 1);
      l += __shfl_xor_sync(0xffffffffu, l, 2);
      if (qrow < G) {
#pragma unroll
        for (int n = 0; n < NT_D; ++n)
          *reinterpret_cast<float2*>(&sm.red_o[warp][qrow][8 * n + qcol]) = make_float2(o[n][0], o[n][1]);
        if (qcol == 0) {
          sm.red_m[warp][qrow] = m_run;
          sm.red_l[warp][qrow] = l;
        }
      }
      if (warp == 0 && lane == 0) {
        sm.red_chunk = chunk;
        sm.red_bh = bh;
      }
      mbar_arrive(&sm.chunk_done);
      ++n_ev;
    };
    for (int it = 0;; ++it) {
      const int s = it % NST;
      mbar_wait(&sm.full[s], (it / NST) & 1, err);
      const TileRef ti = sm.info[s];
      if (ti.chunk < 0) {
        if (cur >= 0) dump(cur, cur_bh);
        break;
      }
      if (ti.chunk != cur) {
        if (cur >= 0) dump(cur, cur_bh);
        cur = ti.chunk;
        cur_bh = ti.bh;
        const __nv_bfloat16* qh = sm.qbuf[ti.qslot] + qrow * D;
#pragma unroll
        for (int k = 0; k < KS_D; ++k) {
          qa[k][0] = qrow < G ? *reinterpret_cast<const uint32_t*>(qh + 16 * k + qcol) : 0u;
          qa[k][1] = qrow < G ? *reinterpret_cast<const uint32_t*>(qh + 16 * k + 8 + qcol) : 0u;
        }
        mbar_arrive(&sm.q_free[ti.qslot]);
#pragma unroll
        for (int n = 0; n < NT_D; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
        m_run = -INFINITY;
        l_run = 0.f;
      }
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
      x[0] = row0 + qcol < ti.valid ? sa[0] * sc : -INFINITY;
      x[1] = row0 + qcol + 1 < ti.valid ? sa[1] * sc : -INFINITY;
      x[2] = row0 + 8 + qcol < ti.valid ? sb[0] * sc : -INFINITY;
      x[3] = row0 + 9 + qcol < ti.valid ? sb[1] * sc : -INFINITY;
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
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.empty[s]);
    }
    // no more chunks: tell the finisher
    mbar_wait(&sm.red_free, (n_ev & 1) ^ 1, err);
    if (warp == 0 && lane == 0) sm.red_chunk = -1;
    mbar_arrive(&sm.chunk_done);
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

size_t max_chunks_tc(const spkv_params& p, int num_sms) {
  return (size_t)num_sms * kUnitsPerCta + (size_t)p.B * p.Hkv;
}

template <int D, int G, int NST>
cudaError_t run_nst(const spkv_params& p, const spkv_cache& c, const spkv_ring& ring, const void* q,
                   const int32_t* t_pos, void* o, float* lse, void* ws, int num_sms,
                   cudaStream_t stream) {
  using S = TcDecSmem<D, G, NST>;
  const int n_heads_ = p.B * p.Hkv;
  const size_t smem = sizeof(S) + 1024 + ((size_t)3 * n_heads_ + 1) * 4;
  static int configured = 0;
  if ((int)smem > configured) {
    cudaError_t e = cudaFuncSetAttribute(decode_tc_kernel<D, G, NST>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    configured = (int)smem;
  }
  const cuuint64_t es = 2;
  CUtensorMap tkp, tvp, tkr, tvr;
  {
    const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)c.num_pages * kPageRows};
    const cuuint64_t str[1] = {(cuuint64_t)D * es};
    const cuuint32_t box[2] = {64, kPageRows};  // one cache page per box; a tile takes two
    if (!map_bf16(&tkp, c.K_pool, 2, dims, str, box) || !map_bf16(&tvp, c.V_pool, 2, dims, str, box))
      return cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)p.window, (cuuint64_t)p.Hkv, (cuuint64_t)p.B};
    const cuuint64_t str[3] = {(cuuint64_t)D * es, (cuuint64_t)p.window * D * es,
                               (cuuint64_t)p.Hkv * p.window * D * es};
    const cuuint32_t box[4] = {64, kTileR, 1, 1};
    if (!map_bf16(&tkr, ring.K_win, 4, dims, str, box) || !map_bf16(&tvr, ring.V_win, 4, dims, str, box))
      return cudaErrorInvalidValue;
  }
  const int n_heads = p.B * p.Hkv;
  char* w = static_cast<char*>(ws);
  const size_t ctrl_bytes = ((size_t)(n_heads + 2) * 4 + 255) / 256 * 256;
  const size_t ml_bytes = (max_chunks_tc(p, num_sms) * G * 2 * 4 + 255) / 256 * 256;
  CacheView cv{static_cast<const char*>(c.K_pool), static_cast<const char*>(c.V_pool), c.pos_pool,
               c.page_table, c.count, c.max_pages_per_head};
  decode_tc_kernel<D, G, NST><<<num_sms, kThreadsT, smem, stream>>>(
      tkp, tvp, tkr, tvr, cv, static_cast<const __nv_bfloat16*>(q), t_pos,
      static_cast<__nv_bfloat16*>(o), lse, reinterpret_cast<int*>(w),
      reinterpret_cast<float*>(w + ctrl_bytes), reinterpret_cast<float*>(w + ctrl_bytes + ml_bytes),
      n_heads, p.Hkv, p.window, c.err_flag);
  return cudaGetLastError();
}

// Three stages when they fit in shared memory with the plan, else two.
template <int D, int G>
cudaError_t run_tc(const spkv_params& p, const spkv_cache& c, const spkv_ring& ring, const void* q,
                   const int32_t* t_pos, void* o, float* lse, void* ws, int num_sms,
                   cudaStream_t stream) {
  const size_t plan = ((size_t)3 * p.B * p.Hkv + 1) * 4 + 1024;
  if (sizeof(TcDecSmem<D, G, 3>) + plan <= 227 * 1024)
    return run_nst<D, G, 3>(p, c, ring, q, t_pos, o, lse, ws, num_sms, stream);
  return run_nst<D, G, 2>(p, c, ring, q, t_pos, o, lse, ws, num_sms, stream);
}

template <int D>
cudaError_t dispatch_tc(const spkv_params& p, const spkv_cache& c, const spkv_ring& ring,
                        const void* q, const int32_t* t_pos, void* o, float* lse, void* ws,
                        int num_sms, cudaStream_t stream) {
  switch (p.Hq / p.Hkv) {
    case 1: return run_tc<D, 1>(p, c, ring, q, t_pos, o, lse, ws, num_sms, stream);
    case 2: return run_tc<D, 2>(p, c, ring, q, t_pos, o, lse, ws, num_sms, stream);
    case 4: return run_tc<D, 4>(p, c, ring, q, t_pos, o, lse, ws, num_sms, stream);
    case 8: return run_tc<D, 8>(p, c, ring, q, t_pos, o, lse, ws, num_sms, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

bool decode_tc_supported(const spkv_params& p) {
  return p.dtype == SPKV_BF16 && (p.head_dim == 64 || p.head_dim == 128) &&
         p.window % kTileR == 0 && p.B * p.Hkv <= kMaxHeadsT && encode_fn_t() != nullptr;
}

size_t decode_tc_workspace_bytes(const spkv_params& p, int num_sms) {
  const int n_heads = p.B * p.Hkv;
  const int G = p.Hq / p.Hkv;
  const size_t ctrl_bytes = ((size_t)(n_heads + 2) * 4 + 255) / 256 * 256;
  const size_t mc = max_chunks_tc(p, num_sms);
  const size_t ml_bytes = (mc * G * 2 * 4 + 255) / 256 * 256;
  return ctrl_bytes + ml_bytes + mc * G * p.head_dim * 4;
}

cudaError_t launch_decode_tc(const spkv_params& p, const spkv_cache& c, const spkv_ring& ring,
                             const void* q, const int32_t* t_pos, void* o, float* lse,
                             void* workspace, int num_sms, cudaStream_t stream) {
  if (p.head_dim == 128) return dispatch_tc<128>(p, c, ring, q, t_pos, o, lse, workspace, num_sms, stream);
  return dispatch_tc<64>(p, c, ring, q, t_pos, o, lse, workspace, num_sms, stream);
}

}  // namespace spkv
