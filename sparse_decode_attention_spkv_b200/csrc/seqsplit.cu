// seqsplit.cu -- one sequence's decode attention split into slices of its key set.
//
// "Self-Pruned Key-Value Attention" (arXiv 2605.14037), §2.1, Eq. (3): the softmax
// over a key set that is the disjoint union of slices S_1 .. S_n factorises.  With
// o_i the softmax-weighted mean of V over S_i and lse_i = log sum_{s in S_i} e^{x_s}
// (x the scaled logits of Eq. (3)),
//   lse = log sum_i e^{lse_i},   o = sum_i e^{lse_i - lse} o_i,
// which is the attention over the whole set.  A slice without keys has lse = -inf and
// drops out.  Each slice's partial comes from the decode kernel in its partial mode
// (decode_tc.cu); this file holds the combination.  The same arithmetic merges the
// split-K chunks inside one decode call; here the parts come from separate calls (on
// one device, or gathered from the devices that hold the slices).
#include <math.h>

#include "common.cuh"
#include "launch.h"

namespace spkv {
namespace {

constexpr int kMergeWarps = 4;

// One warp per (batch row, query head); lane j owns columns j*C .. j*C + C - 1 (C = D/32).
template <typename OutT, int D>
__global__ void __launch_bounds__(kMergeWarps * 32)
    merge_parts_kernel(int n_parts, int n_rows, const float* __restrict__ o_parts,
                       const float* __restrict__ lse_parts, OutT* __restrict__ o,
                       float* __restrict__ lse) {
  constexpr int C = D / 32;
  const int row = blockIdx.x * kMergeWarps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= n_rows) return;
  float m = -INFINITY;
  for (int i = 0; i < n_parts; ++i) m = fmaxf(m, __ldg(lse_parts + (size_t)i * n_rows + row));
  float acc[C];
#pragma unroll
  for (int c = 0; c < C; ++c) acc[c] = 0.f;
  float L = 0.f;
  if (m != -INFINITY) {
    for (int i = 0; i < n_parts; ++i) {
      const float li = __ldg(lse_parts + (size_t)i * n_rows + row);
      if (li == -INFINITY) continue;  // an empty slice
      const float wgt = expf(li - m);
      L += wgt;
      const float* src = o_parts + ((size_t)i * n_rows + row) * D + lane * C;
      if constexpr (C == 4) {
        const float4 v = __ldg(reinterpret_cast<const float4*>(src));
        acc[0] = fmaf(wgt, v.x, acc[0]);
        acc[1] = fmaf(wgt, v.y, acc[1]);
        acc[2] = fmaf(wgt, v.z, acc[2]);
        acc[3] = fmaf(wgt, v.w, acc[3]);
      } else {
        const float2 v = __ldg(reinterpret_cast<const float2*>(src));
        acc[0] = fmaf(wgt, v.x, acc[0]);
        acc[1] = fmaf(wgt, v.y, acc[1]);
      }
    }
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  OutT* dst = o + (size_t)row * D + lane * C;
#pragma unroll
  for (int c = 0; c < C; ++c) from_f32(acc[c] * inv, dst + c);
  if (lse && lane == 0) lse[row] = L > 0.f ? m + logf(L) : -INFINITY;
}

template <typename OutT>
cudaError_t run_merge(const spkv_params& p, int n_parts, const float* o_parts,
                      const float* lse_parts, void* o, float* lse, cudaStream_t stream) {
  const int n_rows = p.B * p.Hq;
  const dim3 grid((n_rows + kMergeWarps - 1) / kMergeWarps);
  if (p.head_dim == 128)
    merge_parts_kernel<OutT, 128><<<grid, kMergeWarps * 32, 0, stream>>>(
        n_parts, n_rows, o_parts, lse_parts, static_cast<OutT*>(o), lse);
  else
    merge_parts_kernel<OutT, 64><<<grid, kMergeWarps * 32, 0, stream>>>(
        n_parts, n_rows, o_parts, lse_parts, static_cast<OutT*>(o), lse);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_merge_parts(const spkv_params& p, int n_parts, const float* o_parts,
                                      const float* lse_parts, void* o, float* lse,
                                      cudaStream_t stream) {
  if (p.dtype == SPKV_BF16)
    return run_merge<__nv_bfloat16>(p, n_parts, o_parts, lse_parts, o, lse, stream);
  return run_merge<float>(p, n_parts, o_parts, lse_parts, o, lse, stream);
}

}  // namespace spkv
