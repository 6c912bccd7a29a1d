// inputs_gen.cu -- device side of the seeded input generator (no SP-KV arithmetic).
// Same definition as gen.py: SplitMix64 output function over a counter stream,
// two 32-bit uniforms per draw, Box-Muller (cosine branch) in fp64, scale in fp64,
// round to fp32 (nearest), then to bf16 (nearest even) for bf16 tensors.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ull;

__device__ __forceinline__ uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__device__ __forceinline__ double normal_at(uint64_t key, uint64_t i) {
  const uint64_t d = mix64(key + (i + 1) * kGamma);
  const double u1 = ((double)(d >> 32) + 0.5) * 2.3283064365386963e-10;
  const double u2 = ((double)(d & 0xffffffffull) + 0.5) * 2.3283064365386963e-10;
  return sqrt(-2.0 * log(u1)) * cos(2.0 * 3.141592653589793 * u2);
}

__device__ __forceinline__ void store(double x, int dtype, void* out, uint64_t j) {
  const float f = __double2float_rn(x);
  if (dtype == 1) static_cast<__nv_bfloat16*>(out)[j] = __float2bfloat16_rn(f);
  else static_cast<float*>(out)[j] = f;
}

// out[j] = scale * N(0,1) draw (offset + j), j < n
__global__ void gen_normal(uint64_t key, uint64_t offset, uint64_t n, double scale, int dtype,
                           void* out) {
  for (uint64_t j = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; j < n;
       j += (uint64_t)gridDim.x * blockDim.x)
    store(normal_at(key, offset + j) * scale, dtype, out, j);
}

// Rows [row0, row0+n_rows) of a [tokens][n_heads][head_dim] tensor with rotary
// embedding: row r (token index) has absolute position pos0 + (r % tokens_per_batch).
__global__ void gen_rope(uint64_t key, uint64_t row0, uint64_t n_rows, int n_heads, int head_dim,
                         int tokens_per_batch, double scale, double base, int dtype, void* out) {
  const uint64_t row_len = (uint64_t)n_heads * head_dim;
  const uint64_t n = n_rows * row_len;
  const int half = head_dim / 2;
  for (uint64_t j = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; j < n;
       j += (uint64_t)gridDim.x * blockDim.x) {
    const uint64_t r = row0 + j / row_len;
    const int within = (int)(j % row_len);
    const int hd = within / head_dim * head_dim;
    const int i = within % head_dim;
    const int ii = i < half ? i : i - half;
    const double pos = (double)(r % (uint64_t)tokens_per_batch);
    const double theta = pow(base, -2.0 * ii / head_dim);
    const double ang = pos * theta;
    const double c = cos(ang), s = sin(ang);
    const uint64_t e1 = r * row_len + hd + ii, e2 = e1 + half;
    const double x1 = normal_at(key, e1) * scale, x2 = normal_at(key, e2) * scale;
    const double y = i < half ? x1 * c - x2 * s : x1 * s + x2 * c;
    store(y, dtype, out, j);
  }
}

}  // namespace

extern "C" {

int spkv_gen_normal(uint64_t key, uint64_t offset, uint64_t n, double scale, int dtype, void* out,
                    void* stream) {
  if (n == 0) return 0;
  gen_normal<<<1184, 256, 0, static_cast<cudaStream_t>(stream)>>>(key, offset, n, scale, dtype, out);
  return cudaGetLastError() == cudaSuccess ? 0 : 3;
}

int spkv_gen_rope(uint64_t key, uint64_t row0, uint64_t n_rows, int n_heads, int head_dim,
                  int tokens_per_batch, double scale, double base, int dtype, void* out,
                  void* stream) {
  if (n_rows == 0) return 0;
  gen_rope<<<1184, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      key, row0, n_rows, n_heads, head_dim, tokens_per_batch, scale, base, dtype, out);
  return cudaGetLastError() == cudaSuccess ? 0 : 3;
}

}  // extern "C"
