// score_tc.cu -- a1 for many tokens at once (chunked prefill, bulk scoring of buffered
// decode tokens) on the 5th-generation tensor cores.
//
// "Self-Pruned Key-Value Attention" (arXiv 2605.14037), §2.1, Eqs. (1)-(2):
//   a = h W1^T + b1, x = GELU(a), l = x W2^T + b2, u = sigmoid(l), z = [u >= tau].
// The first layer is a dense GEMM, M = tokens, N = hid = 128, K = d_model: a chunk of
// 4096 tokens at d_model 4096 is 4.3 GFLOP.  One cluster of 4 CTAs owns 128 tokens;
// CTA rank r runs tcgen05.mma over its quarter of d_model (64-column K blocks of h and
// W1 streamed by TMA, 128-byte swizzled, 4 stages), accumulating the 128 x 128 fp32
// tile in TMEM.  The four partial tiles are summed through distributed shared memory:
// each rank copies its tile from TMEM to shared memory, and rank r then finishes tokens
// 32r .. 32r+31 of the tile (sum of the partials, bias, exact-erf GELU, second layer in
// fp32 on CUDA cores, sigmoid, threshold).
//
// Warp roles (128 threads): warp 0 lane 0 issues the TMA copies, warp 1 allocates TMEM
// and its lane 0 issues the MMAs; all four warps then read the accumulator (warp w owns
// TMEM lanes 32w .. 32w+31, i.e. tokens 32w .. 32w+31) and do the epilogue.  Every
// mbarrier wait is bounded.
#include <cooperative_groups.h>

#include "common.cuh"
#include "host.h"
#include "launch.h"
#include "tc.cuh"

namespace cg = cooperative_groups;

namespace spkv {
namespace {

constexpr int kSTok = 128;     // tokens per cluster (MMA M)
constexpr int kSHid = 128;     // hidden units (MMA N)
constexpr int kSKB = 64;       // K block: 64 bf16 = one 128-byte swizzled row
constexpr int kSRanks = 4;     // cluster size: split of d_model
constexpr int kSStages = 4;
constexpr int kSThreads = 128;
constexpr int kSMine = kSTok / kSRanks;  // tokens finished per rank
constexpr int kSPartLd = kSHid + 1;      // padded row of the partial tile (no bank conflicts)
constexpr int kSMaxHkv = 16;

struct __align__(1024) ScoreTcSmem {
  // stage buffers; after the last MMA they hold this rank's partial tile
  // (128 x kSPartLd fp32 = 66 KB of the 128 KB)
  char a[kSStages][kSTok * 128];   // h: 128 tokens x 64 bf16 per stage
  char b[kSStages][kSHid * 128];   // W1: 128 hidden units x 64 bf16 per stage
  float xs[kSMine][kSHid + 1];     // GELU outputs of this rank's tokens (padded rows)
  float w2[kSMaxHkv][kSHid];       // second-layer weights
  uint64_t full[kSStages];
  uint64_t empty[kSStages];
  uint64_t done;
  uint32_t tmem_base;
};
static_assert(sizeof(float) * kSTok * kSPartLd <= sizeof(ScoreTcSmem::a) + sizeof(ScoreTcSmem::b),
              "the partial tile reuses the stage buffers");

__global__ void __cluster_dims__(kSRanks, 1, 1) __launch_bounds__(kSThreads, 1)
    score_tc_kernel(const __grid_constant__ CUtensorMap tm_h, const __grid_constant__ CUtensorMap tm_w,
                    int n_tok, int d_model, const float* __restrict__ b1,
                    const float* __restrict__ W2, const float* __restrict__ b2, int hkv,
                    float tau, float* __restrict__ u_out, uint8_t* __restrict__ z_out) {
  extern __shared__ __align__(1024) char smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  ScoreTcSmem& sm = *reinterpret_cast<ScoreTcSmem*>(smem_raw + pad);
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tok0 = (blockIdx.x / kSRanks) * kSTok;
  const int n_kb = d_model / kSKB;
  const int kb0 = rank * n_kb / kSRanks, kb1 = (rank + 1) * n_kb / kSRanks;

  if (tid == 0) {
    for (int s = 0; s < kSStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    mbar_init(&sm.done, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 128;" ::"r"(
                     smem_u32(&sm.tmem_base))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp == 0 && lane == 0) {
    // ---- TMA producer: K blocks kb0 .. kb1-1 of h (this tile's tokens) and W1 ----
    for (int i = 0; i < kb1 - kb0; ++i) {
      const int s = i % kSStages;
      mbar_wait(&sm.empty[s], ((i / kSStages) & 1) ^ 1, nullptr);
      mbar_arrive_expect_tx(&sm.full[s], (kSTok + kSHid) * 128);
      tma_2d(sm.a[s], &tm_h, (kb0 + i) * kSKB, tok0, &sm.full[s]);  // rows past n_tok: zeros
      tma_2d(sm.b[s], &tm_w, (kb0 + i) * kSKB, 0, &sm.full[s]);
    }
  } else if (warp == 1 && lane == 0) {
    // ---- MMA issuer: D[128 tokens][128 units] += h_blk W1_blk^T, four k-steps of 16 ----
    constexpr uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kSHid >> 3) << 17) |
                               ((uint32_t)(kSTok >> 4) << 24);
    for (int i = 0; i < kb1 - kb0; ++i) {
      const int s = i % kSStages;
      mbar_wait(&sm.full[s], (i / kSStages) & 1, nullptr);
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < kSKB / 16; ++kk) {
        const uint64_t ad = smem_desc(sm.a[s] + kk * 32, 16, 1024);
        const uint64_t bd = smem_desc(sm.b[s] + kk * 32, 16, 1024);
        mma_ss(tmem, ad, bd, idesc, (i > 0 || kk > 0) ? 1u : 0u);
      }
      mma_commit(&sm.empty[s]);
    }
    mma_commit(&sm.done);
  }

  // ---- this rank's partial tile: TMEM -> shared memory (row = token) ----------------
  float* part = reinterpret_cast<float*>(sm.a[0]);
  const int row = warp * 32 + lane;
  if (kb1 > kb0) {
    mbar_wait(&sm.done, 0, nullptr);
    tc_fence_after();
#pragma unroll
    for (int c0 = 0; c0 < kSHid; c0 += 32) {
      uint32_t r[32];
      tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + c0, r);
      tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < 32; ++i) part[row * kSPartLd + c0 + i] = __uint_as_float(r[i]);
    }
  } else {  // no K block for this rank (d_model < 4 blocks): a zero partial
    for (int c = 0; c < kSHid; ++c) part[row * kSPartLd + c] = 0.f;
  }
  tc_fence_before();
  cluster.sync();  // every rank's partial tile is in place
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 128;" ::"r"(tmem) : "memory");
  }

  // ---- rank r finishes tokens 32r .. 32r+31: sum of partials, bias, GELU ------------
  // thread = hidden unit; its 32 rows x 4 ranks of partial sums are loaded in batches of
  // 8 rows so that the distributed shared-memory reads overlap
  static_assert(kSThreads == kSHid, "one thread per hidden unit");
  {
    const float* parts[kSRanks];
#pragma unroll
    for (int q = 0; q < kSRanks; ++q) parts[q] = cluster.map_shared_rank(part, q);
    const int unit = tid;
    const float bias = b1[unit];
#pragma unroll
    for (int r0 = 0; r0 < kSMine; r0 += 8) {
      float a[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int pr = (rank * kSMine + r0 + i) * kSPartLd + unit;
        a[i] = parts[0][pr];
#pragma unroll
        for (int q = 1; q < kSRanks; ++q) a[i] += parts[q][pr];
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float x = a[i] + bias;
        sm.xs[r0 + i][unit] = 0.5f * x * (1.f + erff(x * 0.70710678118654752440f));
      }
    }
    for (int e = tid; e < hkv * kSHid; e += kSThreads) sm.w2[e / kSHid][e % kSHid] = W2[e];
  }
  __syncthreads();

  // ---- second layer: one thread per (token, key head), warps over key heads ----------
  for (int pair = tid; pair < kSMine * hkv; pair += kSThreads) {
    const int rl = pair % kSMine, kh = pair / kSMine;  // lanes: tokens; w2 row: broadcast
    const int tok = tok0 + rank * kSMine + rl;
    float sum = 0.f;
#pragma unroll 16
    for (int unit = 0; unit < kSHid; ++unit) sum = fmaf(sm.xs[rl][unit], sm.w2[kh][unit], sum);
    if (tok < n_tok) {
      const float logit = sum + b2[kh];
      const float u = 1.f / (1.f + expf(-logit));
      if (u_out) u_out[(size_t)tok * hkv + kh] = u;
      z_out[(size_t)tok * hkv + kh] = (u >= tau) ? 1 : 0;
    }
  }
  cluster.sync();  // keep this rank's partial tile alive until every rank has read it
}

constexpr size_t kScoreTcSmem = sizeof(ScoreTcSmem) + 1024;  // + alignment slack

}  // namespace

// At least one whole 128-token tile (shorter calls go to the other score kernels, so the
// tensor map's box never exceeds the token dimension).
bool score_tc_supported(const spkv_params& p, int n_tok) {
  return p.dtype == SPKV_BF16 && p.hid == kSHid && p.d_model % kSKB == 0 &&
         p.d_model >= kSKB * kSRanks && p.Hkv <= kSMaxHkv && n_tok >= kSTok &&
         encode_fn() != nullptr;
}

cudaError_t launch_score_tc(const spkv_params& p, const void* h, int n_tok, const void* W1,
                            const float* b1, const float* W2, const float* b2, float* u_out,
                            uint8_t* z_out, cudaStream_t stream) {
  {
    cudaError_t e = ensure_dynamic_smem((const void*)score_tc_kernel, (int)kScoreTcSmem);
    if (e != cudaSuccess) return e;
  }
  CUtensorMap th, tw;
  {
    const cuuint64_t dims[2] = {(cuuint64_t)p.d_model, (cuuint64_t)n_tok};
    const cuuint64_t str[1] = {(cuuint64_t)p.d_model * 2};
    const cuuint32_t box[2] = {kSKB, kSTok};
    if (!make_map(&th, h, 2, dims, str, box)) return cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[2] = {(cuuint64_t)p.d_model, (cuuint64_t)kSHid};
    const cuuint64_t str[1] = {(cuuint64_t)p.d_model * 2};
    const cuuint32_t box[2] = {kSKB, kSHid};
    if (!make_map(&tw, W1, 2, dims, str, box)) return cudaErrorInvalidValue;
  }
  const int tiles = (n_tok + kSTok - 1) / kSTok;
  score_tc_kernel<<<tiles * kSRanks, kSThreads, kScoreTcSmem, stream>>>(
      th, tw, n_tok, p.d_model, b1, W2, b2, p.Hkv, p.tau, u_out, z_out);
  return cudaGetLastError();
}

}  // namespace spkv
