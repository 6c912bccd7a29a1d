// score.cu -- a1: utility score and gate (Eqs. (1)-(2) of "Self-Pruned Key-Value
// Attention", arXiv 2605.14037, §2.1), fused in one kernel:
//   a = h W1^T + b1, x = GELU(a), l = x W2^T + b2, u = sigmoid(l), z = [u >= tau].
//
// Work split: a cluster of 8 CTAs owns a tile of 32 tokens; CTA rank r computes the
// partial first-layer sums over its eighth of d_model (split-K, so that a handful
// of decode tokens still spreads the W1 read over 8 SMs), the partials are summed
// through distributed shared memory, and each rank finishes 4 of the 32 tokens
// (bias, GELU, second layer in fp32, sigmoid, threshold).
#include <cooperative_groups.h>

#include "append.cuh"
#include "common.cuh"
#include "host.h"
#include "launch.h"

namespace cg = cooperative_groups;

namespace spkv {
namespace {

constexpr int kTok = 32;     // tokens per cluster
constexpr int kKS = 8;       // cluster size (split of d_model)
constexpr int kKT = 32;      // K step staged in shared memory
constexpr int kThreads = 256;
constexpr int kMaxHid = 128;

template <typename E>
__global__ void __cluster_dims__(1, kKS, 1) __launch_bounds__(kThreads)
    score_kernel(const typename E::T* __restrict__ h, int n_tok, int d_model,
                 const typename E::T* __restrict__ W1, const float* __restrict__ b1,
                 const float* __restrict__ W2, const float* __restrict__ b2, int hid, int hkv,
                 float tau, float* __restrict__ u_out, uint8_t* __restrict__ z_out) {
  using T = typename E::T;
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int tid = threadIdx.x;
  const int tok0 = blockIdx.x * kTok;

  __shared__ float hs[kTok][kKT + 1];
  __shared__ float ws[kMaxHid][kKT + 1];
  __shared__ float part[kTok][kMaxHid];
  __shared__ float xs[kTok / kKS][kMaxHid];

  const int ty = tid >> 5;  // tokens ty*4 .. ty*4+3
  const int tx = tid & 31;  // hidden units tx + 32*j
  const int nj = (hid + 31) >> 5;
  float acc[4][kMaxHid / 32];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < kMaxHid / 32; ++j) acc[i][j] = 0.f;

  const int steps = d_model / kKT;
  const int s_begin = rank * steps / kKS;
  const int s_end = (rank + 1) * steps / kKS;
  for (int s = s_begin; s < s_end; ++s) {
    const int k0 = s * kKT;
    for (int e = tid; e < kTok * kKT; e += kThreads) {
      const int r = e / kKT, c = e % kKT;
      const int tok = tok0 + r;
      hs[r][c] = tok < n_tok ? to_f32(h[(size_t)tok * d_model + k0 + c]) : 0.f;
    }
    for (int e = tid; e < hid * kKT; e += kThreads) {
      const int r = e / kKT, c = e % kKT;
      ws[r][c] = to_f32(W1[(size_t)r * d_model + k0 + c]);
    }
    __syncthreads();
#pragma unroll 8
    for (int k = 0; k < kKT; ++k) {
      float hv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) hv[i] = hs[ty * 4 + i][k];
#pragma unroll
      for (int j = 0; j < kMaxHid / 32; ++j) {
        if (j < nj) {
          const int unit = tx + 32 * j;
          const float wv = unit < hid ? ws[unit][k] : 0.f;
#pragma unroll
          for (int i = 0; i < 4; ++i) acc[i][j] = fmaf(hv[i], wv, acc[i][j]);
        }
      }
    }
    __syncthreads();
  }

#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < kMaxHid / 32; ++j) {
      const int unit = tx + 32 * j;
      if (j < nj && unit < hid) part[ty * 4 + i][unit] = acc[i][j];
    }
  cluster.sync();

  // Rank r finishes tokens r*4 .. r*4+3 of the tile.
  constexpr int kMine = kTok / kKS;
  for (int e = tid; e < kMine * hid; e += kThreads) {
    const int r = e / hid, unit = e % hid;
    const int row = rank * kMine + r;
    float a = 0.f;
#pragma unroll
    for (int q = 0; q < kKS; ++q) {
      const float* remote = cluster.map_shared_rank(&part[0][0], q);
      a += remote[row * kMaxHid + unit];
    }
    a += b1[unit];
    xs[r][unit] = 0.5f * a * (1.f + erff(a * 0.70710678118654752440f));
  }
  __syncthreads();

  // Second layer: one warp per (token, key head) pair, lanes over hidden units.
  const int warp = tid >> 5, lane = tid & 31;
  for (int pair = warp; pair < kMine * hkv; pair += kThreads / 32) {
    const int r = pair / hkv, kh = pair % hkv;
    const int tok = tok0 + rank * kMine + r;
    float sum = 0.f;
    for (int unit = lane; unit < hid; unit += 32) sum = fmaf(xs[r][unit], W2[kh * hid + unit], sum);
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, m);
    if (lane == 0 && tok < n_tok) {
      const float logit = sum + b2[kh];
      const float u = 1.f / (1.f + expf(-logit));
      if (u_out) u_out[(size_t)tok * hkv + kh] = u;
      z_out[(size_t)tok * hkv + kh] = (u >= tau) ? 1 : 0;
    }
  }
  cluster.sync();  // keep this CTA's partials alive until every rank has read them
}

// ---- few tokens (decode): W1 streamed once, hidden units split over the cluster ----------
//
// With a handful of tokens the first layer is a matrix-vector product bound by the
// W1 read (d_model x hid).  A cluster of 8 CTAs splits the hidden units, one warp per
// unit: the warp's W1 row is loaded into registers all at once while one bulk copy
// brings the tokens' h into shared memory, the dot products use packed fp32 FMAs,
// and the GELU outputs are exchanged through distributed shared memory for the
// second layer.  In kScoreAppend mode the warp that finishes (token b, key head kh) of
// a per-token decode step also does that step's ring/cache update for (b, kh); in
// kScoreGates mode it stores the gate in the token's window slot.
constexpr int kSmallRanks = 8;
constexpr int kSmallThreads = 512;   // one warp per hidden unit of the rank (<= 16 units)
constexpr int kSmallMaxVec = 16;     // 16-byte W1 vectors per lane
constexpr uint32_t kBulkPiece = 32768;

// What the few-token kernels do after the gates: nothing, the per-token decode step's
// ring/cache update (retire t - window, store the new token), or store each new token's
// gate and utility in its window slot (the step's update having been done before).
constexpr int kScoreOnly = 0, kScoreAppend = 1, kScoreGates = 2;

struct SmallAppend {
  CacheMut c;
  RingMut r;
  const int32_t* t_pos;
  const char* k_new;
  const char* v_new;
  int window;
  int row_bytes;
  int settled;  // kScoreAppend: h was written before the preceding kernel started
};

// The gate (and, if the ring keeps them, the utility) of the token of batch row b at
// its window slot t_pos[b] % window.
__device__ __forceinline__ void store_gate(const SmallAppend& ap, int b, int kh, int hkv,
                                           uint8_t z, float u) {
  const int t = ap.t_pos[b];
  if (t < 0) return;
  const size_t zi = ((size_t)b * ap.window + t % ap.window) * hkv + kh;
  ap.r.z[zi] = z;
  if (ap.r.u) ap.r.u[zi] = u;
}

// Gates of a scored batch into their window slots (after the separate score kernel).
__global__ void __launch_bounds__(256)
    store_gates_kernel(SmallAppend ap, const uint8_t* __restrict__ z, const float* __restrict__ u,
                       int B, int hkv) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < B * hkv) store_gate(ap, i / hkv, i % hkv, hkv, z[i], u ? u[i] : no_utility());
}


template <typename E, int NT, int MODE>
__global__ void __cluster_dims__(kSmallRanks, 1, 1) __launch_bounds__(kSmallThreads, 1)
    score_small_kernel(const typename E::T* __restrict__ h, int n_tok, int d_model,
                       const typename E::T* __restrict__ W1, const float* __restrict__ b1,
                       const float* __restrict__ W2, const float* __restrict__ b2, int hid,
                       int hkv, float tau, float* __restrict__ u_out, uint8_t* __restrict__ z_out,
                       SmallAppend ap) {
  using T = typename E::T;
  constexpr int EPL = 16 / E::kSize;
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tok0 = (blockIdx.x / kSmallRanks) * NT;
  const int nt = min(NT, n_tok - tok0);
  extern __shared__ __align__(16) char smem_raw[];
  __shared__ uint64_t hbar;
  T* hs = reinterpret_cast<T*>(smem_raw);                           // [NT][d_model]
  float* xs = reinterpret_cast<float*>(hs + (size_t)NT * d_model);  // [units][NT]
  const int units = (hid + kSmallRanks - 1) / kSmallRanks;
  const int j = rank * units + warp;  // this warp's hidden unit
  const bool active = warp < units && j < hid;
  const int vec_per_row = d_model / EPL;
  const int nv = vec_per_row / 32;    // vectors per lane

  if (tid == 0) {
    mbar_init(&hbar, 1);
    fence_mbar_init();
  }
  // the weights do not depend on the previous kernel: their loads are issued before
  // waiting for it (programmatic dependent launch)
  uint4 wv[kSmallMaxVec];
  if (active) {
    const uint4* wrow = reinterpret_cast<const uint4*>(W1 + (size_t)j * d_model);
#pragma unroll
    for (int i = 0; i < kSmallMaxVec; ++i)
      if (i < nv) wv[i] = __ldg(wrow + lane + 32 * i);
  }
  grid_dependency_wait();
  grid_dependents_launch();
  __syncthreads();
  if (tid == 0) {  // the tokens' hidden states: one contiguous block
    const uint32_t bytes = (uint32_t)nt * d_model * E::kSize;
    mbar_arrive_expect_tx(&hbar, bytes);
    const char* src = reinterpret_cast<const char*>(h + (size_t)tok0 * d_model);
    for (uint32_t off = 0; off < bytes; off += kBulkPiece)
      bulk_g2s(reinterpret_cast<char*>(hs) + off, src + off, min(kBulkPiece, bytes - off), &hbar);
  }
  mbar_wait(&hbar, 0, nullptr);

  if (active) {
    float2 acc[NT];
#pragma unroll
    for (int n = 0; n < NT; ++n) acc[n] = make_float2(0.f, 0.f);
#pragma unroll
    for (int i = 0; i < kSmallMaxVec; ++i) {
      if (i < nv) {
        float wf[EPL];
        Vec<E>::widen(wv[i], wf);
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          if (n < nt) {
            float hf[EPL];
            Vec<E>::widen(reinterpret_cast<const uint4*>(hs)[(size_t)n * vec_per_row + lane + 32 * i], hf);
#pragma unroll
            for (int e = 0; e < EPL / 2; ++e)
              acc[n] = fma2(make_float2(wf[2 * e], wf[2 * e + 1]), make_float2(hf[2 * e], hf[2 * e + 1]), acc[n]);
          }
        }
      }
    }
    float sum[NT];
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      sum[n] = acc[n].x + acc[n].y;
#pragma unroll
      for (int m = 16; m > 0; m >>= 1) sum[n] += __shfl_xor_sync(0xffffffffu, sum[n], m);
    }
    if (lane == 0) {
      const float bias = b1[j];
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        const float a = sum[n] + bias;
        xs[warp * NT + n] = 0.5f * a * (1.f + erff(a * 0.70710678118654752440f));
      }
    }
  }
  cluster.sync();

  // second layer: token n is finished by rank n % 8, one warp per (token, key head)
  for (int pair = warp; pair < NT * hkv; pair += kSmallThreads / 32) {
    const int n = pair / hkv, kh = pair % hkv;
    if (n % kSmallRanks != rank || n >= nt) continue;
    float sum = 0.f;
    for (int jj = lane; jj < hid; jj += 32) {
      const float* remote = cluster.map_shared_rank(xs, jj / units);
      sum = fmaf(remote[(jj % units) * NT + n], W2[kh * hid + jj], sum);
    }
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, m);
    const float logit = sum + b2[kh];
    const float uval = 1.f / (1.f + expf(-logit));
    const uint8_t z = (uval >= tau) ? 1 : 0;
    const size_t o = (size_t)(tok0 + n) * hkv + kh;
    if (lane == 0) {
      if (u_out) u_out[o] = uval;
      z_out[o] = z;
    }
    if constexpr (MODE == kScoreAppend) {
      const int b = tok0 + n;  // one new token per batch row
      const int t = ap.t_pos[b];
      if (t >= 0)
        decode_append_warp(ap.c, ap.r, b * hkv + kh, b, kh, t, ap.k_new, ap.v_new, z, uval, 1, hkv,
                           ap.window, ap.row_bytes, lane);
    } else if constexpr (MODE == kScoreGates) {
      const int b = tok0 + n;
      if (lane == 0) store_gate(ap, b, kh, hkv, z, uval);
    }
  }
  cluster.sync();
}

template <typename E, int NT, int MODE>
cudaError_t launch_small(const spkv_params& p, const void* h, int n_tok, const void* W1,
                         const float* b1, const float* W2, const float* b2, float* u_out,
                         uint8_t* z_out, const SmallAppend& ap, cudaStream_t stream) {
  using T = typename E::T;
  const int units = (p.hid + kSmallRanks - 1) / kSmallRanks;
  const size_t smem = (size_t)NT * p.d_model * E::kSize + (size_t)units * NT * 4;
  {
    cudaError_t e = ensure_dynamic_smem((const void*)score_small_kernel<E, NT, MODE>, (int)smem);
    if (e != cudaSuccess) return e;
  }
  const int groups = (n_tok + NT - 1) / NT;
  return launch_pdl(score_small_kernel<E, NT, MODE>, dim3(groups * kSmallRanks),
                    dim3(kSmallThreads), smem, stream, static_cast<const T*>(h), n_tok, p.d_model,
                    static_cast<const T*>(W1), b1, W2, b2, p.hid, p.Hkv, p.tau, u_out, z_out, ap);
}

template <int MODE>
cudaError_t dispatch_small(const spkv_params& p, const void* h, int n_tok, const void* W1,
                           const float* b1, const float* W2, const float* b2, float* u_out,
                           uint8_t* z_out, const SmallAppend& ap, cudaStream_t stream) {
  if (p.dtype == SPKV_BF16) {
    return n_tok <= 8
               ? launch_small<BF16, 8, MODE>(p, h, n_tok, W1, b1, W2, b2, u_out, z_out, ap, stream)
               : launch_small<BF16, 16, MODE>(p, h, n_tok, W1, b1, W2, b2, u_out, z_out, ap, stream);
  }
  return n_tok <= 8
             ? launch_small<F32, 8, MODE>(p, h, n_tok, W1, b1, W2, b2, u_out, z_out, ap, stream)
             : launch_small<F32, 16, MODE>(p, h, n_tok, W1, b1, W2, b2, u_out, z_out, ap, stream);
}

// ---- few tokens, bf16, hid = 128: the first layer on tensor cores ---------------------
//
// h W1^T for up to 8 tokens is a skinny GEMM: M = 128 hidden units (W1 rows), N = 8
// tokens, K = d_model.  A cluster of 8 CTAs takes 8 tokens; CTA rank r owns hidden
// units 16r .. 16r+15 (one m16n8k16 row tile) and its 16 warps split K.  Inside each
// pair of k-steps the K index is permuted the same way for W1 and h, so that a lane's
// A and B fragments of both k-steps are 16 contiguous bytes of a W1 row or an h row
// (one 16-byte load each, no shared-memory staging).  The K-split partials are summed
// in shared memory, bias + GELU follow, and the 128 x 8 GELU outputs are all-gathered
// into every CTA of the cluster with distributed shared-memory stores; rank n then
// finishes token n (second layer in fp32, sigmoid, threshold).  W1 and W2 loads are
// issued before the kernel waits for the preceding kernel on the stream.  In
// kScoreAppend mode the per-token ring/cache reads of the step are issued while the MLP
// runs and the step is written once the gate is known; in kScoreGates mode the gates
// go to the tokens' window slots.
constexpr int kMmaRanks = 8;
constexpr int kMmaWarps = 16;
constexpr int kMmaThreads = kMmaWarps * 32;
constexpr int kMmaTok = 8;          // tokens per cluster (the MMA's N)
constexpr int kMmaHid = 16 * kMmaRanks;
constexpr int kMmaMaxPairs = 8;     // 32-column k-step pairs per warp (d_model <= 4096)
constexpr int kMmaMaxHkv = 16;
constexpr int kMmaMaxRowBytes = 256;

__device__ __forceinline__ void mma_bf16_16816(float* d, uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

template <int MODE>
__global__ void __cluster_dims__(kMmaRanks, 1, 1) __launch_bounds__(kMmaThreads, 1)
    score_mma_kernel(const __nv_bfloat16* __restrict__ h, int n_tok, int d_model,
                     const __nv_bfloat16* __restrict__ W1, const float* __restrict__ b1,
                     const float* __restrict__ W2, const float* __restrict__ b2, int hkv,
                     float tau, float* __restrict__ u_out, uint8_t* __restrict__ z_out,
                     SmallAppend ap) {
  __shared__ float red[kMmaWarps][16][kMmaTok];
  __shared__ float xs[kMmaHid][kMmaTok];  // GELU outputs of all hidden units (all-gathered)
  __shared__ __align__(16) char stage[MODE == kScoreAppend ? kMmaMaxHkv : 1][4 * kMmaMaxRowBytes];
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int r = lane >> 2, q = lane & 3;
  const int tok0 = (blockIdx.x / kMmaRanks) * kMmaTok;
  const int nt = min(kMmaTok, n_tok - tok0);
  const int pairs = d_model / (32 * kMmaWarps);
  const int kbeg = warp * pairs * 32;

  // weights first: they do not depend on the preceding kernel
  uint4 a_lo[kMmaMaxPairs], a_hi[kMmaMaxPairs];
  {
    const __nv_bfloat16* w0 = W1 + (size_t)(16 * rank + r) * d_model + kbeg + 8 * q;
    const __nv_bfloat16* w1 = w0 + (size_t)8 * d_model;
#pragma unroll
    for (int i = 0; i < kMmaMaxPairs; ++i) {
      if (i < pairs) {
        a_lo[i] = __ldg(reinterpret_cast<const uint4*>(w0 + 32 * i));
        a_hi[i] = __ldg(reinterpret_cast<const uint4*>(w1 + 32 * i));
      }
    }
  }
  const int my_n = rank;  // token finished by this rank
  float w2v[4];
  float b2v = 0.f;
  if (warp < hkv) {
#pragma unroll
    for (int i = 0; i < 4; ++i) w2v[i] = __ldg(W2 + (size_t)warp * kMmaHid + lane + 32 * i);
    b2v = __ldg(b2 + warp);
  }
  const float b1v = tid < 16 * kMmaTok ? __ldg(b1 + 16 * rank + tid / kMmaTok) : 0.f;
  // with settled inputs the perceptron runs before the wait for the preceding kernel:
  // only the ring and cache, which that kernel may still read, wait for it
  const bool early = MODE == kScoreAppend && ap.settled;
  if (!early) {
    grid_dependency_wait();
    grid_dependents_launch();
  }

  AppendPre pre;
  pre.t = -1;
  if constexpr (MODE == kScoreAppend) {
    if (!early && warp < hkv && my_n < nt) {
      const int b = tok0 + my_n, bh = b * hkv + warp;
      pre = append_prefetch(ap.c, ap.r, bh, b, warp, __ldg(ap.t_pos + b), ap.k_new, ap.v_new, hkv,
                            ap.window, ap.row_bytes, lane, stage[warp]);
    }
  }

  // first layer: this warp's K slice, tokens as the MMA's N
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  {
    const bool tok_ok = r < nt;
    const __nv_bfloat16* hp = h + (size_t)(tok0 + (tok_ok ? r : 0)) * d_model + kbeg + 8 * q;
    uint4 bv[kMmaMaxPairs];
#pragma unroll
    for (int i = 0; i < kMmaMaxPairs; ++i)
      if (i < pairs) bv[i] = tok_ok ? __ldg(reinterpret_cast<const uint4*>(hp + 32 * i)) : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int i = 0; i < kMmaMaxPairs; ++i) {
      if (i < pairs) {
        mma_bf16_16816(acc, a_lo[i].x, a_hi[i].x, a_lo[i].y, a_hi[i].y, bv[i].x, bv[i].y);
        mma_bf16_16816(acc, a_lo[i].z, a_hi[i].z, a_lo[i].w, a_hi[i].w, bv[i].z, bv[i].w);
      }
    }
  }
  red[warp][r][2 * q] = acc[0];
  red[warp][r][2 * q + 1] = acc[1];
  red[warp][r + 8][2 * q] = acc[2];
  red[warp][r + 8][2 * q + 1] = acc[3];
  __syncthreads();
  if (tid < 16 * kMmaTok) {
    const int j = tid / kMmaTok, n = tid % kMmaTok;
    float a = b1v;
#pragma unroll
    for (int w = 0; w < kMmaWarps; ++w) a += red[w][j][n];
    const float x = 0.5f * a * (1.f + erff(a * 0.70710678118654752440f));
#pragma unroll
    for (int dst = 0; dst < kMmaRanks; ++dst)
      cluster.map_shared_rank(&xs[0][0], dst)[(16 * rank + j) * kMmaTok + n] = x;
  }
  cluster.sync();  // every rank now holds all 128 x 8 GELU outputs; no remote access follows
  if (early) {
    grid_dependency_wait();
    grid_dependents_launch();
    if constexpr (MODE == kScoreAppend) {
      if (warp < hkv && my_n < nt) {
        const int b = tok0 + my_n, bh = b * hkv + warp;
        pre = append_prefetch(ap.c, ap.r, bh, b, warp, __ldg(ap.t_pos + b), ap.k_new, ap.v_new,
                              hkv, ap.window, ap.row_bytes, lane, stage[warp]);
      }
    }
  }

  // second layer: token my_n, one warp per key head
  if (warp < hkv && my_n < nt) {
    float sum = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) sum = fmaf(xs[lane + 32 * i][my_n], w2v[i], sum);
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, m);
    const float logit = sum + b2v;
    const float uval = 1.f / (1.f + expf(-logit));
    const uint8_t z = (uval >= tau) ? 1 : 0;
    const size_t o = (size_t)(tok0 + my_n) * hkv + warp;
    if (lane == 0) {
      if (u_out) u_out[o] = uval;
      z_out[o] = z;
    }
    if constexpr (MODE == kScoreGates) {
      if (lane == 0) store_gate(ap, tok0 + my_n, warp, hkv, z, uval);
    }
    if constexpr (MODE == kScoreAppend) {
      const int b = tok0 + my_n;
      append_commit(ap.c, ap.r, pre, b * hkv + warp, b, warp, z, uval, hkv, ap.window, ap.row_bytes,
                    lane, stage[warp]);
    }
  }
}

bool mma_ok(const spkv_params& p, int n_tok) {
  return p.dtype == SPKV_BF16 && p.hid == kMmaHid && p.d_model % (32 * kMmaWarps) == 0 &&
         p.d_model / (32 * kMmaWarps) <= kMmaMaxPairs && p.Hkv <= kMmaMaxHkv &&
         p.head_dim * 2 <= kMmaMaxRowBytes && n_tok >= 1 && n_tok <= 64;
}

template <int MODE>
cudaError_t launch_mma(const spkv_params& p, const void* h, int n_tok, const void* W1,
                       const float* b1, const float* W2, const float* b2, float* u_out,
                       uint8_t* z_out, const SmallAppend& ap, cudaStream_t stream) {
  const int groups = (n_tok + kMmaTok - 1) / kMmaTok;
  return launch_pdl(score_mma_kernel<MODE>, dim3(groups * kMmaRanks), dim3(kMmaThreads), 0,
                    stream, static_cast<const __nv_bfloat16*>(h), n_tok, p.d_model,
                    static_cast<const __nv_bfloat16*>(W1), b1, W2, b2, p.Hkv, p.tau, u_out, z_out,
                    ap);
}

// The few-token kernel applies when the tokens fit in shared memory, every lane
// holds whole 16-byte W1 vectors, and one warp per hidden unit covers a rank.
bool small_ok(const spkv_params& p, int n_tok) {
  const int esize = p.dtype == SPKV_BF16 ? 2 : 4;
  const int epl = 16 / esize;
  const int units = (p.hid + kSmallRanks - 1) / kSmallRanks;
  return n_tok <= 16 && p.d_model % (32 * epl) == 0 && p.d_model / (32 * epl) <= kSmallMaxVec &&
         units <= kSmallThreads / 32 &&
         (size_t)16 * p.d_model * esize + (size_t)units * 16 * 4 <= 160 * 1024;
}

}  // namespace

cudaError_t launch_score(const spkv_params& p, const void* h, int n_tok, const void* W1,
                         const float* b1, const float* W2, const float* b2, float* u_out,
                         uint8_t* z_out, cudaStream_t stream) {
  if (mma_ok(p, n_tok))
    return launch_mma<kScoreOnly>(p, h, n_tok, W1, b1, W2, b2, u_out, z_out, SmallAppend{}, stream);
  if (small_ok(p, n_tok))
    return dispatch_small<kScoreOnly>(p, h, n_tok, W1, b1, W2, b2, u_out, z_out, SmallAppend{}, stream);
  if (score_tc_supported(p, n_tok))
    return launch_score_tc(p, h, n_tok, W1, b1, W2, b2, u_out, z_out, stream);
  dim3 grid((n_tok + kTok - 1) / kTok, kKS);
  if (p.dtype == SPKV_BF16) {
    score_kernel<BF16><<<grid, kThreads, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(h), n_tok, p.d_model,
        static_cast<const __nv_bfloat16*>(W1), b1, W2, b2, p.hid, p.Hkv, p.tau, u_out, z_out);
  } else {
    score_kernel<F32><<<grid, kThreads, 0, stream>>>(
        static_cast<const float*>(h), n_tok, p.d_model, static_cast<const float*>(W1), b1, W2,
        b2, p.hid, p.Hkv, p.tau, u_out, z_out);
  }
  return cudaGetLastError();
}

cudaError_t launch_score_append(const spkv_params& p, const spkv_cache& c, const spkv_ring& ring,
                                const int32_t* t_pos, const void* h, const void* W1,
                                const float* b1, const float* W2, const float* b2,
                                const void* k_new, const void* v_new, float* u_out,
                                uint8_t* z_out, bool settled, cudaStream_t stream) {
  const bool mma = mma_ok(p, p.B);
  if (!mma && !small_ok(p, p.B)) {  // many rows: the two steps as separate launches
    cudaError_t e = launch_score(p, h, p.B, W1, b1, W2, b2, u_out, z_out, stream);
    if (e != cudaSuccess) return e;
    return launch_decode_append(p, c, ring, t_pos, k_new, v_new, z_out, u_out, 1, stream);
  }
  const int esize = p.dtype == SPKV_BF16 ? 2 : 4;
  SmallAppend ap{cache_mut(c),
                 ring_mut(ring),
                 t_pos, static_cast<const char*>(k_new), static_cast<const char*>(v_new), p.window,
                 p.head_dim * esize, settled ? 1 : 0};
  if (mma) return launch_mma<kScoreAppend>(p, h, p.B, W1, b1, W2, b2, u_out, z_out, ap, stream);
  return dispatch_small<kScoreAppend>(p, h, p.B, W1, b1, W2, b2, u_out, z_out, ap, stream);
}

cudaError_t launch_score_gates(const spkv_params& p, const spkv_ring& ring, const int32_t* t_pos,
                               const void* h, const void* W1, const float* b1, const float* W2,
                               const float* b2, float* u_out, uint8_t* z_out, cudaStream_t stream) {
  SmallAppend ap{};
  ap.r = ring_mut(ring);
  ap.t_pos = t_pos;
  ap.window = p.window;
  if (mma_ok(p, p.B))
    return launch_mma<kScoreGates>(p, h, p.B, W1, b1, W2, b2, u_out, z_out, ap, stream);
  if (small_ok(p, p.B))
    return dispatch_small<kScoreGates>(p, h, p.B, W1, b1, W2, b2, u_out, z_out, ap, stream);
  cudaError_t e = launch_score(p, h, p.B, W1, b1, W2, b2, u_out, z_out, stream);
  if (e != cudaSuccess) return e;
  store_gates_kernel<<<(p.B * p.Hkv + 255) / 256, 256, 0, stream>>>(ap, z_out, u_out, p.B, p.Hkv);
  return cudaGetLastError();
}

bool score_supported(const spkv_params& p) {
  return p.hid >= 1 && p.hid <= kMaxHid && p.d_model % kKT == 0 && p.Hkv <= 64;
}

}  // namespace spkv
