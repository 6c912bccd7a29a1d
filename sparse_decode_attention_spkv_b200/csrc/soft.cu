// soft.cu -- soft-gated attention of SP-KV training ("Self-Pruned Key-Value
// Attention", arXiv 2605.14037, §2.1 "soft relaxation at training time").
//
// At training time the hard gate z_s = 1[u_s >= tau] is replaced by
// alpha_s = sigmoid((u_s - tau) / beta) (Eq. (5)) and the mask of Eq. (4) by an
// additive score (Eq. (6)): 0 inside the causal window (0 <= t - s < w) and
// c (alpha_s - 1) outside it, so every earlier key takes part with a large negative
// bias instead of being removed.  The forward pass here is
//   o_t = softmax_s(q_t k_s / sqrt(d_k) + M_soft(t, s)) v_s   over all s <= t.
// soft_bias computes the per-key bias c (alpha_s - 1) = -c / (1 + exp((u_s - tau) /
// beta)) (the second form has no cancellation for alpha near 1) into a [B][Hkv][T]
// buffer, in the units the attention kernel adds it in; the attention itself runs on the tensor cores
// (prefill_tc.cu, SOFT mode) or, for other shapes, in soft_simple_kernel below.
#include <math.h>

#include "common.cuh"
#include "launch.h"

namespace spkv {
namespace {

constexpr int kWarps = 4;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// u [B][T][Hkv] -> bias [B][Hkv][T] in units of out_scale (1/(score scale) for the
// tensor-core path, which adds it to raw q.k; log2 e for the CUDA-core path).
__global__ void __launch_bounds__(256)
    soft_bias_kernel(const float* __restrict__ u, float* __restrict__ bias, int B, int T, int hkv,
                     float tau, float inv_beta, float c, float out_scale) {
  const size_t n = (size_t)B * T * hkv;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x) {
    const int kh = (int)(i % hkv);
    const size_t bt = i / hkv;
    const int t = (int)(bt % T), b = (int)(bt / T);
    const float x = (u[i] - tau) * inv_beta;
    const float m = -c / (1.f + expf(x));  // c (alpha - 1)
    bias[((size_t)b * hkv + kh) * T + t] = m * out_scale;
  }
}

// CUDA-core form: one CTA per (query, batch row, key head), the G query heads of the
// group served from each K/V row read; 4 warps split the keys 0..t, each with an
// online softmax, then combine through shared memory.
template <typename E, int D, int G>
__global__ void __launch_bounds__(kWarps * 32)
    soft_simple_kernel(const typename E::T* __restrict__ q, const char* __restrict__ K,
                       const char* __restrict__ V, const float* __restrict__ bias,
                       typename E::T* __restrict__ out, float* __restrict__ lse_out, int T,
                       int hkv, int window, float qscale) {
  constexpr int kRowBytes = D * E::kSize;
  constexpr int LPR = kRowBytes / 16, EPL = 16 / E::kSize, RPW = 32 / LPR;
  __shared__ float red_o[kWarps][G][D];
  __shared__ float red_m[kWarps][G], red_l[kWarps][G];
  const int t = blockIdx.x;
  const int bh = blockIdx.y;
  const int b = bh / hkv, kh = bh % hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int grp = lane / LPR, col = lane % LPR;
  const float* bias_h = bias + (size_t)bh * T;

  float qf[G][EPL];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const uint4 raw = *reinterpret_cast<const uint4*>(
        q + (((size_t)b * T + t) * hkv * G + (size_t)kh * G + g) * D + col * EPL);
    Vec<E>::widen(raw, qf[g]);
#pragma unroll
    for (int e = 0; e < EPL; ++e) qf[g][e] *= qscale;
  }
  float m[G], l[G], acc[G][EPL];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    m[g] = -INFINITY;
    l[g] = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) acc[g][e] = 0.f;
  }
  const int n_keys = t + 1;
  for (int k0 = warp * RPW; k0 < n_keys; k0 += kWarps * RPW) {
    const int s = k0 + grp;
    const bool valid = s < n_keys;
    float kf[EPL], vf[EPL];
    float add = 0.f;
    if (valid) {
      const size_t r = ((size_t)b * T + s) * hkv + kh;
      Vec<E>::widen(*reinterpret_cast<const uint4*>(K + r * kRowBytes + col * 16), kf);
      Vec<E>::widen(*reinterpret_cast<const uint4*>(V + r * kRowBytes + col * 16), vf);
      add = t - s >= window ? bias_h[s] : 0.f;
    } else {
#pragma unroll
      for (int e = 0; e < EPL; ++e) kf[e] = vf[e] = 0.f;
    }
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float sc = 0.f;
#pragma unroll
      for (int e = 0; e < EPL; ++e) sc = fmaf(qf[g][e], kf[e], sc);
#pragma unroll
      for (int msk = LPR / 2; msk > 0; msk >>= 1) sc += __shfl_xor_sync(0xffffffffu, sc, msk);
      sc = valid ? sc + add : -INFINITY;
      float smax = sc;
#pragma unroll
      for (int msk = LPR; msk < 32; msk <<= 1) smax = fmaxf(smax, __shfl_xor_sync(0xffffffffu, smax, msk));
      const float mnew = fmaxf(m[g], smax);
      if (mnew == -INFINITY) continue;
      const float alpha = (m[g] == -INFINITY) ? 0.f : exp2f(m[g] - mnew);
      const float p = valid ? exp2f(sc - mnew) : 0.f;
      float psum = p;
#pragma unroll
      for (int msk = LPR; msk < 32; msk <<= 1) psum += __shfl_xor_sync(0xffffffffu, psum, msk);
      l[g] = l[g] * alpha + psum;
#pragma unroll
      for (int e = 0; e < EPL; ++e) acc[g][e] = acc[g][e] * alpha + p * vf[e];
      m[g] = mnew;
    }
  }
#pragma unroll
  for (int msk = LPR; msk < 32; msk <<= 1)
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int e = 0; e < EPL; ++e) acc[g][e] += __shfl_xor_sync(0xffffffffu, acc[g][e], msk);
  if (lane < LPR) {
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int e = 0; e < EPL; ++e) red_o[warp][g][col * EPL + e] = acc[g][e];
  }
  if (lane == 0) {
#pragma unroll
    for (int g = 0; g < G; ++g) {
      red_m[warp][g] = m[g];
      red_l[warp][g] = l[g];
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < G * D; e += kWarps * 32) {
    const int g = e / D, d = e % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, red_m[w][g]);
    float O = 0.f, L = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float ww = red_m[w][g] == -INFINITY ? 0.f : exp2f(red_m[w][g] - M);
      O += ww * red_o[w][g][d];
      L += ww * red_l[w][g];
    }
    const size_t row = ((size_t)b * T + t) * hkv * G + (size_t)kh * G + g;
    from_f32(L > 0.f ? O / L : 0.f, out + row * D + d);
    if (d == 0 && lse_out) lse_out[row] = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
  }
}

template <typename E, int D, int G>
cudaError_t launch_simple(const spkv_params& p, const void* q, const void* K, const void* V,
                          const float* bias, int T, void* o, float* lse, cudaStream_t stream) {
  using Tt = typename E::T;
  dim3 grid(T, p.B * p.Hkv);
  soft_simple_kernel<E, D, G><<<grid, kWarps * 32, 0, stream>>>(
      static_cast<const Tt*>(q), static_cast<const char*>(K), static_cast<const char*>(V), bias,
      static_cast<Tt*>(o), lse, T, p.Hkv, p.window, kLog2e / sqrtf((float)D));
  return cudaGetLastError();
}

template <typename E, int D>
cudaError_t dispatch_g(const spkv_params& p, const void* q, const void* K, const void* V,
                       const float* bias, int T, void* o, float* lse, cudaStream_t stream) {
  switch (p.Hq / p.Hkv) {
    case 1: return launch_simple<E, D, 1>(p, q, K, V, bias, T, o, lse, stream);
    case 2: return launch_simple<E, D, 2>(p, q, K, V, bias, T, o, lse, stream);
    case 4: return launch_simple<E, D, 4>(p, q, K, V, bias, T, o, lse, stream);
    case 8: return launch_simple<E, D, 8>(p, q, K, V, bias, T, o, lse, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

size_t soft_workspace_bytes(const spkv_params& p, int seq_len) {
  return ((size_t)p.B * p.Hkv * seq_len * 4 + 255) / 256 * 256;
}

cudaError_t launch_soft(const spkv_params& p, const void* q, const void* K, const void* V,
                        const float* u, int seq_len, float beta, float c, void* o, float* lse,
                        void* workspace, uint32_t* err, cudaStream_t stream) {
  float* bias = static_cast<float*>(workspace);
  const size_t n = (size_t)p.B * seq_len * p.Hkv;
  const int blocks = (int)((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
  const bool tc = soft_tc_supported(p, seq_len);
  // the tensor-core path adds the bias to raw q.k (scaled by log2 e / sqrt(d) later);
  // the CUDA-core path adds it to scores already in the log2 domain
  const float out_scale = tc ? sqrtf((float)p.head_dim) : kLog2e;
  soft_bias_kernel<<<blocks, 256, 0, stream>>>(u, bias, p.B, seq_len, p.Hkv, p.tau, 1.f / beta, c,
                                               out_scale);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (tc) return launch_soft_tc(p, q, K, V, bias, seq_len, o, lse, err, stream);
  if (p.dtype == SPKV_BF16)
    return p.head_dim == 128 ? dispatch_g<BF16, 128>(p, q, K, V, bias, seq_len, o, lse, stream)
                             : dispatch_g<BF16, 64>(p, q, K, V, bias, seq_len, o, lse, stream);
  return p.head_dim == 128 ? dispatch_g<F32, 128>(p, q, K, V, bias, seq_len, o, lse, stream)
                           : dispatch_g<F32, 64>(p, q, K, V, bias, seq_len, o, lse, stream);
}

}  // namespace spkv
