// prefill.cu -- a6: gated prefill attention for a chunk of queries.
//
// "Self-Pruned Key-Value Attention" (arXiv 2605.14037), §2.1, Eqs. (3)-(4).  The
// key set of query t is its causal window (t-w, t] plus the gated-in keys with
// position <= t-w, which at deployment are the cache rows with pos <= t-w (the
// cache may already hold rows of this chunk: compact-after-each-chunk).  Window
// keys at positions >= chunk_start come from the chunk's own K/V, earlier ones
// from the ring (the previous chunk's last rows).
//
// This is the direct CUDA-core form: one CTA per (query, batch row, key head),
// serving the G query heads of the group from each K/V row read; 4 warps split
// the key set, each with an online softmax, then combine through shared memory.
#include <math.h>

#include "common.cuh"
#include "launch.h"

namespace spkv {
namespace {

constexpr int kWarps = 4;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

template <typename E, int D, int G>
__global__ void __launch_bounds__(kWarps * 32)
    prefill_simple_kernel(CacheView cache, const char* __restrict__ Kwin,
                          const char* __restrict__ Vwin, const typename E::T* __restrict__ q,
                          const char* __restrict__ Kc, const char* __restrict__ Vc,
                          typename E::T* __restrict__ out, float* __restrict__ lse_out,
                          int chunk_start, int chunk_len, int hkv, int window, float qscale) {
  constexpr int kRowBytes = D * E::kSize;
  constexpr int LPR = kRowBytes / 16, EPL = 16 / E::kSize, RPW = 32 / LPR;
  __shared__ float red_o[kWarps][G][D];
  __shared__ float red_m[kWarps][G], red_l[kWarps][G];
  const int i = blockIdx.x;           // query index within the chunk
  const int bh = blockIdx.y;          // batch row * Hkv + key head
  const int b = bh / hkv, kh = bh % hkv;
  const int t = chunk_start + i;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int grp = lane / LPR, col = lane % LPR;

  float qf[G][EPL];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const uint4 raw = *reinterpret_cast<const uint4*>(
        q + (((size_t)b * chunk_len + i) * hkv * G + (size_t)kh * G + g) * D + col * EPL);
    Vec<E>::widen(raw, qf[g]);
#pragma unroll
    for (int e = 0; e < EPL; ++e) qf[g][e] *= qscale;
  }
  // key set: cache rows [0, n_live) then window positions [lo, t]
  const int n_live = cache_live_rows(cache, bh, t - window, 1 << 30);
  const int lo = t - window + 1 > 0 ? t - window + 1 : 0;
  const int n_keys = n_live + (t - lo + 1);

  float m[G], l[G], acc[G][EPL];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    m[g] = -INFINITY;
    l[g] = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) acc[g][e] = 0.f;
  }
  for (int k0 = warp * RPW; k0 < n_keys; k0 += kWarps * RPW) {
    const int k = k0 + grp;
    const bool valid = k < n_keys;
    const char* krow = nullptr;
    const char* vrow = nullptr;
    if (valid) {
      if (k < n_live) {
        int page = __ldg(cache.page_table + (size_t)bh * cache.max_pages + (k >> 6));
        if (!page_ok(page, cache.num_pages, cache.err)) page = 0;  // debug build: flagged
        const size_t r = (size_t)page * kPageRows + (k & 63);
        krow = cache.K + r * kRowBytes;
        vrow = cache.V + r * kRowBytes;
      } else {
        const int s = lo + (k - n_live);
        size_t r;
        if (s >= chunk_start) {
          r = ((size_t)b * chunk_len + (s - chunk_start)) * hkv + kh;
          krow = Kc + r * kRowBytes;
          vrow = Vc + r * kRowBytes;
        } else {
          r = (size_t)bh * window + (s % window);
          krow = Kwin + r * kRowBytes;
          vrow = Vwin + r * kRowBytes;
        }
      }
    }
    float kf[EPL], vf[EPL];
    if (valid) {
      Vec<E>::widen(*reinterpret_cast<const uint4*>(krow + col * 16), kf);
      Vec<E>::widen(*reinterpret_cast<const uint4*>(vrow + col * 16), vf);
    } else {
#pragma unroll
      for (int e = 0; e < EPL; ++e) kf[e] = vf[e] = 0.f;
    }
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float s = 0.f;
#pragma unroll
      for (int e = 0; e < EPL; ++e) s = fmaf(qf[g][e], kf[e], s);
#pragma unroll
      for (int msk = LPR / 2; msk > 0; msk >>= 1) s += __shfl_xor_sync(0xffffffffu, s, msk);
      if (!valid) s = -INFINITY;
      // rows of the other lane groups of this warp
      float smax = s;
#pragma unroll
      for (int msk = LPR; msk < 32; msk <<= 1) smax = fmaxf(smax, __shfl_xor_sync(0xffffffffu, smax, msk));
      const float mnew = fmaxf(m[g], smax);
      if (mnew == -INFINITY) continue;
      const float alpha = (m[g] == -INFINITY) ? 0.f : exp2f(m[g] - mnew);
      const float p = valid ? exp2f(s - mnew) : 0.f;
      float psum = p;
#pragma unroll
      for (int msk = LPR; msk < 32; msk <<= 1) psum += __shfl_xor_sync(0xffffffffu, psum, msk);
      l[g] = l[g] * alpha + psum;
#pragma unroll
      for (int e = 0; e < EPL; ++e) acc[g][e] = acc[g][e] * alpha + p * vf[e];
      m[g] = mnew;
    }
  }
  // combine the lane groups (same m across the warp), then the warps
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
      const float sw = red_m[w][g] == -INFINITY ? 0.f : exp2f(red_m[w][g] - M);
      O += sw * red_o[w][g][d];
      L += sw * red_l[w][g];
    }
    const size_t row = ((size_t)b * chunk_len + i) * hkv * G + (size_t)kh * G + g;
    from_f32(L > 0.f ? O / L : 0.f, out + row * D + d);
    if (d == 0 && lse_out) lse_out[row] = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
  }
}

template <typename E, int D, int G>
cudaError_t run(const spkv_params& p, const spkv_cache& c, const spkv_ring& ring, const void* q,
                const void* Kc, const void* Vc, int chunk_start, int chunk_len, void* o,
                float* lse, cudaStream_t stream) {
  CacheView cv = cache_view(c);
  dim3 grid(chunk_len, p.B * p.Hkv);
  prefill_simple_kernel<E, D, G><<<grid, kWarps * 32, 0, stream>>>(
      cv, static_cast<const char*>(ring.K_win), static_cast<const char*>(ring.V_win),
      static_cast<const typename E::T*>(q), static_cast<const char*>(Kc),
      static_cast<const char*>(Vc), static_cast<typename E::T*>(o), lse, chunk_start, chunk_len,
      p.Hkv, p.window, kLog2e / sqrtf((float)D));
  return cudaGetLastError();
}

template <typename E, int D>
cudaError_t dispatch_g(const spkv_params& p, const spkv_cache& c, const spkv_ring& ring,
                       const void* q, const void* Kc, const void* Vc, int cs, int cl, void* o,
                       float* lse, cudaStream_t stream) {
  switch (p.Hq / p.Hkv) {
    case 1: return run<E, D, 1>(p, c, ring, q, Kc, Vc, cs, cl, o, lse, stream);
    case 2: return run<E, D, 2>(p, c, ring, q, Kc, Vc, cs, cl, o, lse, stream);
    case 4: return run<E, D, 4>(p, c, ring, q, Kc, Vc, cs, cl, o, lse, stream);
    case 8: return run<E, D, 8>(p, c, ring, q, Kc, Vc, cs, cl, o, lse, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_prefill(const spkv_params& p, const spkv_cache& c, const spkv_ring& ring,
                           const void* q, const void* K_chunk, const void* V_chunk,
                           int chunk_start, int chunk_len, void* o, float* lse, int* sched,
                           cudaStream_t stream) {
  if (prefill_tc_supported(p, c, chunk_start, chunk_len))
    return launch_prefill_tc(p, c, ring, q, K_chunk, V_chunk, chunk_start, chunk_len, o, lse, sched,
                             stream);
  if (p.dtype == SPKV_BF16) {
    if (p.head_dim == 128) return dispatch_g<BF16, 128>(p, c, ring, q, K_chunk, V_chunk, chunk_start, chunk_len, o, lse, stream);
    if (p.head_dim == 64) return dispatch_g<BF16, 64>(p, c, ring, q, K_chunk, V_chunk, chunk_start, chunk_len, o, lse, stream);
  } else {
    if (p.head_dim == 128) return dispatch_g<F32, 128>(p, c, ring, q, K_chunk, V_chunk, chunk_start, chunk_len, o, lse, stream);
    if (p.head_dim == 64) return dispatch_g<F32, 64>(p, c, ring, q, K_chunk, V_chunk, chunk_start, chunk_len, o, lse, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace spkv
