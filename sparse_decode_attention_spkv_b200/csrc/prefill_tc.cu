// prefill_tc.cu -- a6 on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// "Self-Pruned Key-Value Attention" (arXiv 2605.14037), §2.1, Eqs. (3)-(4), for a
// chunk of queries.  One CTA owns 128 consecutive query positions of two query
// heads of one key head.  Its key set is, in 64-key blocks:
//   * the compacted cache pages holding rows with pos <= t_last - w (gated-in keys
//     of Eq. (4)); pages whose rows all have pos <= t_first - w need no mask, the
//     last one or two are masked per query (pos <= t - w), and pages beyond are
//     never touched: the dead key blocks of the causal mask are simply absent;
//   * the causal window band, positions t_first-128 .. t_first+127 (four blocks,
//     from the ring for positions before the chunk, else from the chunk's K/V),
//     masked per query by 0 <= t - s < 128.
// Both contractions are dense tensor-core tiles: S = Q K^T (M=128 queries, N=64
// keys, K=128) and O += P V (M=128, N=128, K=64 keys), bf16 operands, fp32
// accumulators in TMEM.  P is written back into TMEM over S and fed to the second
// MMA as its A operand.  S is double-buffered per head (TMEM: O0, O1, then two S
// buffers per head, 512 columns), and the MMA thread issues S(j+1) before PV(j):
// the softmax of block j+1 runs while the tensor cores do PV(j) and the other
// head's work, so the tensor pipe is not left waiting on one softmax at a time.
//
// Warp roles (384 threads):
//   warp 0      TMA producer: Q once, then K/V (+ positions) per block, 3 stages;
//   warp 1      TMEM allocation and the single MMA-issuing thread;
//   warps 4-7   softmax of head 0 (one query row per thread, TMEM lanes 0..127);
//   warps 8-11  softmax of head 1.
// Softmax runs in the log2 domain; the running max is raised only when a score
// exceeds it by more than 8, and only then is the O row in TMEM rescaled (after the
// previous block's PV has completed: pv_done).
// Every mbarrier wait is bounded (a stuck wait raises SPKV_FLAG_TIMEOUT).
//
// The same kernel (SOFT = true) computes the soft-gated attention used at training
// time (§2.1, "soft relaxation", Eqs. (5)-(6)): every key s <= t of the sequence,
// read in 64-key blocks from the sequence K/V, with the additive score 0 inside the
// causal window and c (alpha_s - 1) outside it; the per-key bias (already divided by
// the score scale, i.e. in raw q.k units) rides with each block.  No key block is
// skipped.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "host.h"
#include "launch.h"
#include "tc.cuh"

namespace spkv {
namespace {

constexpr int kQT = 128;          // queries per CTA and head
constexpr int kKB = 64;           // keys per block
constexpr int kHD = 128;          // head_dim
constexpr int kWin = 128;         // window of this path
constexpr int kStg = 3;
constexpr int kThr = 384;
constexpr int kMaxPages = 4096;   // pages per key head scanned in shared memory
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kSlack = 8.f;

constexpr uint32_t kColO0 = 0, kColO1 = 128, kColS = 256;  // S[h][buf] at kColS + 128 h + 64 buf

struct __align__(1024) TcSmem {
  char q[2][2][kQT * 128];        // [head][d half] 128 rows x 128 B, 128B-swizzled
  char k[kStg][2][kKB * 128];     // [stage][d half] 64 rows x 128 B
  char v[kStg][2][kKB * 128];
  int pos[kStg][kKB];
  int first_pos[kMaxPages];
  uint64_t q_full;
  uint64_t kv_full[kStg];
  uint64_t kv_empty[kStg];
  uint64_t s_ready[2][2];  // [head][buffer]
  uint64_t p_ready[2];
  uint64_t pv_done[2];
  uint64_t o_ready[2];
  uint32_t tmem_base;
  int cnt[4];
};

// 2^x on the MUFU unit (ex2.approx, flush-to-zero): the scores are <= 8 above the
// running max, so x < 8 and the result is a normal number or 0.
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

struct Blocks {
  int nc;      // cache blocks (pages 0..nc-1)
  int nfull;   // rows visible to every query of the tile
  int nrows;   // cache rows (count)
  int wfirst;  // position of the first window block
  int nw;      // window blocks
};

template <bool SOFT>
__global__ void __launch_bounds__(kThr, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_kc,
                      const __grid_constant__ CUtensorMap tm_vc,
                      const __grid_constant__ CUtensorMap tm_kp,
                      const __grid_constant__ CUtensorMap tm_vp,
                      const __grid_constant__ CUtensorMap tm_kr,
                      const __grid_constant__ CUtensorMap tm_vr, CacheView cache,
                      __nv_bfloat16* __restrict__ out, float* __restrict__ lse_out,
                      int chunk_start, int chunk_len, int hkv, int G, uint32_t* err,
                      const float* __restrict__ soft_bias) {
  extern __shared__ __align__(1024) char smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;  // 128B-swizzle atoms
  TcSmem& sm = *reinterpret_cast<TcSmem*>(smem_raw + pad);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_qt = gridDim.x;
  const int qt = n_qt - 1 - (int)blockIdx.x;  // later tiles (more cache) first
  const int hp = blockIdx.y;
  const int bh = blockIdx.z, b = bh / hkv, kh = bh % hkv;
  const int Hq = hkv * G;
  const int t0 = chunk_start + qt * kQT;
  const int h0 = kh * G + 2 * hp;  // first of the two query heads

  // ---- set-up: barriers, TMEM, cache extents -------------------------------------
  if (tid == 0) {
    mbar_init(&sm.q_full, 1);
    for (int s = 0; s < kStg; ++s) {
      mbar_init(&sm.kv_full[s], 1);
      mbar_init(&sm.kv_empty[s], 1);
    }
    for (int h = 0; h < 2; ++h) {
      mbar_init(&sm.s_ready[h][0], 1);
      mbar_init(&sm.s_ready[h][1], 1);
      mbar_init(&sm.p_ready[h], 128);
      mbar_init(&sm.pv_done[h], 1);
      mbar_init(&sm.o_ready[h], 1);
    }
    sm.cnt[0] = sm.cnt[1] = sm.cnt[2] = sm.cnt[3] = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(
                     smem_u32(&sm.tmem_base))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  Blocks bl;
  if constexpr (SOFT) {
    bl.nc = bl.nfull = bl.nrows = 0;
    bl.wfirst = 0;                    // every key block from the start of the sequence
    bl.nw = (t0 + kQT) / kKB;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  } else {
    const int n = cache.count ? __ldg(cache.count + bh) : 0;  // no cache: window only
    const int npages = (n + kPageRows - 1) / kPageRows;
    const int lim_full = t0 - kWin, lim_any = t0 + kQT - 1 - kWin;
    for (int pg = tid; pg < npages; pg += kThr) sm.first_pos[pg] = cache_pos(cache, bh, pg * kPageRows);
    __syncthreads();
    {
      int pf = 0, pa = 0;
      for (int pg = tid; pg < npages; pg += kThr) {
        pf += sm.first_pos[pg] <= lim_full;
        pa += sm.first_pos[pg] <= lim_any;
      }
      if (pf) atomicAdd(&sm.cnt[0], pf);
      if (pa) atomicAdd(&sm.cnt[1], pa);
    }
    __syncthreads();
    {
      const int Pf = sm.cnt[0], Pa = sm.cnt[1];
      if (tid < 64 && Pf > 0) {
        const int row = (Pf - 1) * kPageRows + tid;
        if (row < n && cache_pos(cache, bh, row) <= lim_full) atomicAdd(&sm.cnt[2], 1);
      } else if (tid >= 64 && tid < 128 && Pa > 0) {
        const int row = (Pa - 1) * kPageRows + (tid - 64);
        if (row < n && cache_pos(cache, bh, row) <= lim_any) atomicAdd(&sm.cnt[3], 1);
      }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    {
      const int Pf = sm.cnt[0], Pa = sm.cnt[1];
      bl.nfull = Pf > 0 ? (Pf - 1) * kPageRows + sm.cnt[2] : 0;
      const int n_any = Pa > 0 ? (Pa - 1) * kPageRows + sm.cnt[3] : 0;
      bl.nc = (n_any + kKB - 1) / kKB;
      bl.nrows = n;
      bl.wfirst = t0 >= kWin ? t0 - kWin : t0;
      bl.nw = (t0 + kQT - bl.wfirst) / kKB;
    }
  }
  const int J = bl.nc + bl.nw;
  const uint32_t tmem = sm.tmem_base;

  if (warp == 0) {
    // ------------------------------ TMA producer --------------------------------
    if (lane == 0) {
      mbar_arrive_expect_tx(&sm.q_full, 2 * 2 * kQT * 128);
      for (int hh = 0; hh < 2; ++hh)
        for (int half = 0; half < 2; ++half)
          tma_4d(sm.q[hh][half], &tm_q, half * 64, h0 + hh, t0 - chunk_start, b, &sm.q_full);
      for (int j = 0; j < J; ++j) {
        const int s = j % kStg;
        mbar_wait(&sm.kv_empty[s], ((j / kStg) & 1) ^ 1, err);
        if (j < bl.nc) {
          const int page = __ldg(cache.page_table + (size_t)bh * cache.max_pages + j);
          mbar_arrive_expect_tx(&sm.kv_full[s], 4 * kKB * 128 + kKB * 4);
          for (int half = 0; half < 2; ++half) {
            tma_2d(sm.k[s][half], &tm_kp, half * 64, page * kPageRows, &sm.kv_full[s]);
            tma_2d(sm.v[s][half], &tm_vp, half * 64, page * kPageRows, &sm.kv_full[s]);
          }
          bulk_g2s(sm.pos[s], cache.pos + (size_t)page * kPageRows, kKB * 4, &sm.kv_full[s]);
        } else {
          const int pb = bl.wfirst + (j - bl.nc) * kKB;
          mbar_arrive_expect_tx(&sm.kv_full[s], 4 * kKB * 128 + (SOFT ? kKB * 4 : 0));
          if constexpr (SOFT)  // the block's per-key bias, [B][Hkv][T] layout
            bulk_g2s(sm.pos[s], soft_bias + (size_t)bh * chunk_len + pb, kKB * 4, &sm.kv_full[s]);
          for (int half = 0; half < 2; ++half) {
            if (pb >= chunk_start) {
              tma_4d(sm.k[s][half], &tm_kc, half * 64, kh, pb - chunk_start, b, &sm.kv_full[s]);
              tma_4d(sm.v[s][half], &tm_vc, half * 64, kh, pb - chunk_start, b, &sm.kv_full[s]);
            } else {
              tma_4d(sm.k[s][half], &tm_kr, half * 64, pb & (kWin - 1), kh, b, &sm.kv_full[s]);
              tma_4d(sm.v[s][half], &tm_vr, half * 64, pb & (kWin - 1), kh, b, &sm.kv_full[s]);
            }
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer -----------------------------------
    if (lane == 0) {
      constexpr uint32_t idesc_s = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kKB >> 3) << 17) |
                                   ((uint32_t)(kQT >> 4) << 24);
      constexpr uint32_t idesc_pv = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) |
                                    ((uint32_t)(kHD >> 3) << 17) | ((uint32_t)(kQT >> 4) << 24);
      const uint32_t colO[2] = {kColO0, kColO1};
      mbar_wait(&sm.q_full, 0, err);
      tc_fence_after();
      // S_h(j) = Q_h K(j)^T into buffer j % 2 of head h
      auto issue_s = [&](int j) {
        const int s = j % kStg;
        mbar_wait(&sm.kv_full[s], (j / kStg) & 1, err);
        tc_fence_after();
        for (int hh = 0; hh < 2; ++hh) {
          const uint32_t col = kColS + 128 * hh + 64 * (j & 1);
#pragma unroll
          for (int kk = 0; kk < kHD / 16; ++kk) {
            const uint64_t ad = smem_desc(sm.q[hh][kk >> 2] + (kk & 3) * 32, 16, 1024);
            const uint64_t bd = smem_desc(sm.k[s][kk >> 2] + (kk & 3) * 32, 16, 1024);
            mma_ss(tmem + col, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
          }
          mma_commit(&sm.s_ready[hh][j & 1]);
        }
      };
      if (J > 0) issue_s(0);
      for (int j = 0; j < J; ++j) {
        // the next block's scores go ahead of this block's PV (double-buffered S; the
        // buffer they overwrite held P(j-1), whose PV was issued before)
        if (j + 1 < J) issue_s(j + 1);
        const int s = j % kStg;
        for (int hh = 0; hh < 2; ++hh) {  // O_h += P_h(j) V(j)
          mbar_wait(&sm.p_ready[hh], j & 1, err);
          tc_fence_after();
          const uint32_t col = kColS + 128 * hh + 64 * (j & 1);
#pragma unroll
          for (int kk = 0; kk < kKB / 16; ++kk) {
            const uint64_t bd = smem_desc(sm.v[s][0] + kk * 16 * 128, 8192, 1024);
            mma_ts(tmem + colO[hh], tmem + col + kk * 8, bd, idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&sm.pv_done[hh]);
        }
        mma_commit(&sm.kv_empty[s]);
      }
      for (int hh = 0; hh < 2; ++hh) mma_commit(&sm.o_ready[hh]);
    }
  } else if (warp >= 4) {
    // ------------------------------ softmax --------------------------------------
    const int hh = (warp - 4) >> 2;
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const int t = t0 + r;
    const uint32_t lane_addr = tmem + ((uint32_t)(quad * 32) << 16);
    const uint32_t colO = hh ? kColO1 : kColO0;
    const float c = kLog2e * rsqrtf((float)kHD);
    float m = -INFINITY, l = 0.f;
    for (int j = 0; j < J; ++j) {
      const int s = j % kStg;
      const uint32_t colS = kColS + 128 * hh + 64 * (j & 1);
      mbar_wait(&sm.s_ready[hh][j & 1], (j >> 1) & 1, err);
      mbar_wait(&sm.kv_full[s], (j / kStg) & 1, err);
      tc_fence_after();
      uint32_t raw[64];
      tmem_ld32(lane_addr + colS, raw);
      tmem_ld32(lane_addr + colS + 32, raw + 32);
      tmem_wait_ld();
      // scores in the raw (unscaled) domain, masked keys at -inf; for the soft mask the
      // per-key bias is pre-divided by the scale so that one fma gives the exponent
      float x[64];
      if (j < bl.nc) {
        const bool dense = (j + 1) * kKB <= bl.nfull;
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          const int row = j * kKB + i;
          const bool vis = dense || (row < bl.nrows && sm.pos[s][i] <= t - kWin);
          x[i] = vis ? __uint_as_float(raw[i]) : -INFINITY;
        }
      } else {
        const int pb = bl.wfirst + (j - bl.nc) * kKB;
        if constexpr (SOFT) {
          const float* bias = reinterpret_cast<const float*>(sm.pos[s]);  // raw-score units
          if (pb + kKB - 1 <= t0 - kWin) {  // every key of the block is outside every window
#pragma unroll
            for (int i = 0; i < 64; ++i) x[i] = __uint_as_float(raw[i]) + bias[i];
          } else {
#pragma unroll
            for (int i = 0; i < 64; ++i) {
              const int dlt = t - (pb + i);
              x[i] = dlt < 0 ? -INFINITY : __uint_as_float(raw[i]) + (dlt >= kWin ? bias[i] : 0.f);
            }
          }
        } else {
#pragma unroll
          for (int i = 0; i < 64; ++i) {
            const int dlt = t - (pb + i);
            const bool vis = dlt >= 0 && dlt < kWin;
            x[i] = vis ? __uint_as_float(raw[i]) : -INFINITY;
          }
        }
      }
      // row maximum: 8 independent partial maxima, then a short tree
      float mx[8];
#pragma unroll
      for (int a = 0; a < 8; ++a) mx[a] = x[a];
#pragma unroll
      for (int i = 8; i < 64; ++i) mx[i & 7] = fmaxf(mx[i & 7], x[i]);
      const float rmax = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                               fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7]))) * c;
      const bool need = rmax > m + kSlack;
      const bool any_need = __any_sync(0xffffffffu, need);
      const float mnew = need ? fmaxf(m, rmax) : m;
      // p = 2^(x c - m): one packed fma per pair, then MUFU; masked keys give 2^-inf = 0
      const float msafe = mnew == -INFINITY ? 0.f : mnew;
      uint32_t pk[32];
      float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                       make_float2(0.f, 0.f)};
      const float2 c2 = make_float2(c, c), nm2 = make_float2(-msafe, -msafe);
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float2 e = fma2(make_float2(x[2 * i], x[2 * i + 1]), c2, nm2);
        const float2 pp = make_float2(fast_exp2(e.x), fast_exp2(e.y));
        acc[i & 3] = add2(acc[i & 3], pp);
        pk[i] = pack_bf16(pp.x, pp.y);
      }
      const float ps = (acc[0].x + acc[0].y) + (acc[1].x + acc[1].y) + (acc[2].x + acc[2].y) +
                       (acc[3].x + acc[3].y);
      // O may be touched only once the previous block's PV has landed in it
      if (j > 0) {
        mbar_wait(&sm.pv_done[hh], (j - 1) & 1, err);
        tc_fence_after();
      }
      if (any_need) {
        const float alpha = (m == -INFINITY) ? 0.f : fast_exp2(m - mnew);
        if (j > 0) {  // O holds P V of earlier blocks: rescale it in TMEM
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
        m = mnew;
      }
      l += ps;
      tmem_st32(lane_addr + colS, pk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sm.p_ready[hh]);
    }
    // epilogue: O / l
    mbar_wait(&sm.o_ready[hh], 0, err);
    tc_fence_after();
    const int hg = h0 + hh;
    const size_t row_out = ((size_t)b * chunk_len + (t - chunk_start)) * Hq + hg;
    __nv_bfloat16* dst = out + row_out * kHD;
    const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
    for (int cc = 0; cc < kHD; cc += 32) {
      uint32_t o[32];
      tmem_ld32(lane_addr + colO + cc, o);
      tmem_wait_ld();
#pragma unroll
      for (int v4 = 0; v4 < 4; ++v4) {
        uint4 pkt;
        pkt.x = pack_bf16(__uint_as_float(o[v4 * 8 + 0]) * inv, __uint_as_float(o[v4 * 8 + 1]) * inv);
        pkt.y = pack_bf16(__uint_as_float(o[v4 * 8 + 2]) * inv, __uint_as_float(o[v4 * 8 + 3]) * inv);
        pkt.z = pack_bf16(__uint_as_float(o[v4 * 8 + 4]) * inv, __uint_as_float(o[v4 * 8 + 5]) * inv);
        pkt.w = pack_bf16(__uint_as_float(o[v4 * 8 + 6]) * inv, __uint_as_float(o[v4 * 8 + 7]) * inv);
        *reinterpret_cast<uint4*>(dst + cc + v4 * 8) = pkt;
      }
    }
    if (lse_out) lse_out[row_out] = l > 0.f ? (m + log2f(l)) * kLn2 : -INFINITY;
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

template <bool SOFT>
cudaError_t configure() {
  return ensure_dynamic_smem((const void*)prefill_tc_kernel<SOFT>, (int)kSmem);
}

}  // namespace

bool prefill_tc_supported(const spkv_params& p, const spkv_cache& c, int chunk_start, int chunk_len) {
  const int G = p.Hq / p.Hkv;
  return p.dtype == SPKV_BF16 && p.head_dim == kHD && p.window == kWin && G % 2 == 0 &&
         chunk_start % kQT == 0 && chunk_len % kQT == 0 && chunk_len > 0 &&
         c.max_pages_per_head <= kMaxPages && encode_fn() != nullptr;
}

cudaError_t launch_prefill_tc(const spkv_params& p, const spkv_cache& c, const spkv_ring& ring,
                              const void* q, const void* K_chunk, const void* V_chunk,
                              int chunk_start, int chunk_len, void* o, float* lse,
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
  if (c.K_pool) {
    const cuuint64_t dims[2] = {(cuuint64_t)kHD, (cuuint64_t)c.num_pages * kPageRows};
    const cuuint64_t str[1] = {kHD * e};
    const cuuint32_t box[2] = {64, kKB};
    if (!make_map(&tkp, c.K_pool, 2, dims, str, box) || !make_map(&tvp, c.V_pool, 2, dims, str, box))
      return cudaErrorInvalidValue;
  } else {  // window-only layer: no cache block is ever loaded
    tkp = tkc;
    tvp = tvc;
  }
  {
    const cuuint64_t dims[4] = {(cuuint64_t)kHD, (cuuint64_t)kWin, (cuuint64_t)p.Hkv, (cuuint64_t)p.B};
    const cuuint64_t str[3] = {kHD * e, (cuuint64_t)kWin * kHD * e, (cuuint64_t)p.Hkv * kWin * kHD * e};
    const cuuint32_t box[4] = {64, kKB, 1, 1};
    if (!make_map(&tkr, ring.K_win, 4, dims, str, box) || !make_map(&tvr, ring.V_win, 4, dims, str, box))
      return cudaErrorInvalidValue;
  }
  cudaError_t e2 = configure<false>();
  if (e2 != cudaSuccess) return e2;
  CacheView cv{static_cast<const char*>(c.K_pool), static_cast<const char*>(c.V_pool), c.pos_pool,
               c.page_table, c.count, c.max_pages_per_head};
  dim3 grid(chunk_len / kQT, G / 2, p.B * p.Hkv);
  prefill_tc_kernel<false><<<grid, kThr, kSmem, stream>>>(
      tq, tkc, tvc, tkp, tvp, tkr, tvr, cv, static_cast<__nv_bfloat16*>(o), lse, chunk_start,
      chunk_len, p.Hkv, G, c.err_flag, nullptr);
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
  CacheView cv{nullptr, nullptr, nullptr, nullptr, nullptr, 0};
  dim3 grid(seq_len / kQT, G / 2, p.B * p.Hkv);
  // the cache and ring maps are not read in this mode: the sequence maps stand in
  prefill_tc_kernel<true><<<grid, kThr, kSmem, stream>>>(
      tq, tk, tv, tk, tv, tk, tv, cv, static_cast<__nv_bfloat16*>(o), lse, 0, seq_len, p.Hkv, G,
      err, bias);
  return cudaGetLastError();
}

}  // namespace spkv
