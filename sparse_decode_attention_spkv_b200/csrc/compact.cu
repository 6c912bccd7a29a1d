// compact.cu -- a2/a3: writes into the persistent gated cache and the window ring.
//
// "Self-Pruned Key-Value Attention" (arXiv 2605.14037), §2.1, efficient
// implementation at deployment: the persistent cache stores only the KV pairs
// with z_s = 1; the most recent w tokens stay reachable through the local window
// (Eq. (4), 1_win).  These kernels move rows between those two stores:
//   compact_plan / compact_scatter  stable stream compaction of gated rows (a2),
//   decode_append                   per-token retirement t-w -> cache, then the
//                                   new token into its ring slot (a2 + a3),
//   ring_write                      last rows of a prefill chunk into the ring (a3).
// Rows are moved as 16-byte vectors by the lanes of one warp (a 256-byte row is
// 16 lanes), so every copy is coalesced.
#include "append.cuh"
#include "common.cuh"
#include "launch.h"

namespace spkv {
namespace {

CacheMut mut(const spkv_cache& c) { return cache_mut(c); }

// Gates of rows [r0, r1) of one key head (stride hkv bytes), summed by the block: every
// thread keeps 8 loads in flight per round.  The loads go to L2 (ld.global.cg): they may
// run while the kernel that wrote the gates has only just finished.
__device__ __forceinline__ int count_gates(const uint8_t* zb, int r0, int r1, int hkv) {
  int kept = 0;
  const int stride = blockDim.x;
  for (int i0 = r0 + (int)threadIdx.x; i0 < r1; i0 += 8 * stride) {
    int v[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int i = i0 + k * stride;
      v[k] = i < r1 ? __ldcg(zb + (size_t)i * hkv) : 0;
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) kept += v[k];
  }
  return kept;
}

__device__ __forceinline__ int block_sum(int v, int* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) v += __shfl_xor_sync(0xffffffffu, v, m);
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  int total = 0;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) total += red[w];
  return total;
}

// One CTA per (batch row, key head): count this call's gated rows, extend the
// head's page list (pages it still owns past its count, left by a re-threshold, first;
// then new ones from the bump allocator), and publish count_prev / count.  Launched as
// a programmatic dependent: it waits for the kernel before it (which may have written
// the gates or the cache), then lets the scatter start launching at once.
__global__ void __launch_bounds__(256)
    compact_plan(CacheMut c, const uint8_t* __restrict__ z, int n_rows, int src_batch_rows,
                 int hkv) {
  __shared__ int red[8];
  __shared__ int s_have, s_need, s_free, s_first, s_grant;
  grid_dependency_wait();
  grid_dependents_launch();
  const int bh = blockIdx.x, b = bh / hkv, kh = bh % hkv;
  const uint8_t* zb = z + (size_t)b * src_batch_rows * hkv + kh;
  int32_t* table = c.page_table + (size_t)bh * c.max_pages;
  const int total = block_sum(count_gates(zb, 0, n_rows, hkv), red);
  int old = 0, want = 0;
  if (threadIdx.x == 0) {
    old = __ldcg(c.count + bh);
    const int cap = c.max_pages * kPageRows;
    want = old + total;
    if (want > cap) {
      atomicOr(c.err, SPKV_FLAG_TABLE_FULL);
      want = cap;
    }
    s_have = (old + kPageRows - 1) / kPageRows;
    s_need = (want + kPageRows - 1) / kPageRows;
    s_free = s_need;
  }
  __syncthreads();
  // owned pages form a prefix of the table: find the first unowned entry we need
  for (int j = s_have + threadIdx.x; j < s_need; j += blockDim.x)
    if (__ldcg(table + j) < 0) atomicMin(&s_free, j);
  __syncthreads();
  if (threadIdx.x == 0) {
    int need = s_need;
    const int own_end = s_free;
    int first = 0, grant = 0;
    if (need > own_end) {
      first = atomicAdd(c.pool_top, need - own_end);
      grant = need - own_end;
      if (first + grant > c.num_pages) {
        grant = c.num_pages - first > 0 ? c.num_pages - first : 0;
        atomicOr(c.err, SPKV_FLAG_POOL_FULL);
        need = own_end + grant;
        if (want > need * kPageRows) want = need * kPageRows;
      }
    }
    c.count_prev[bh] = old;
    c.count[bh] = want;
    s_first = first;
    s_free = own_end;
    s_grant = grant;
  }
  __syncthreads();
  for (int j = threadIdx.x; j < s_grant; j += blockDim.x) table[s_free + j] = s_first + j;
}

constexpr int kScatterTile = 256;
constexpr int kScatterThreads = 256;

// grid (B*Hkv, tiles of 256 rows).  Each CTA counts the gated rows before its
// tile (z is tiny), so tiles need no inter-CTA ordering; inside a tile, 256-row
// rounds are ranked with a warp-ballot prefix sum and copied by lane groups.
// Launched as a programmatic dependent of compact_plan: the prefix count (gates only,
// which the plan does not write; the plan itself started after the gates' producer had
// completed) runs while the plan works; the counts and page lists are read after the
// wait for the plan.
__global__ void __launch_bounds__(kScatterThreads)
    compact_scatter(CacheMut c, const char* __restrict__ Ksrc, const char* __restrict__ Vsrc,
                    const uint8_t* __restrict__ z, const float* __restrict__ u,
                    const int32_t* __restrict__ src_pos,
                    int n_rows, int src_batch_rows, int hkv, int row_bytes, int from_ring,
                    int window) {
  __shared__ int red[8];
  __shared__ int warp_tot[8];
  __shared__ int list_src[kScatterThreads];
  __shared__ int list_dst[kScatterThreads];
  const int bh = blockIdx.x, b = bh / hkv, kh = bh % hkv;
  const int tile0 = blockIdx.y * kScatterTile;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint8_t* zb = z + (size_t)b * src_batch_rows * hkv + kh;

  const int prefix = block_sum(count_gates(zb, 0, tile0, hkv), red);
  grid_dependency_wait();  // the plan's counts and page lists
  const int base = __ldcg(c.count_prev + bh);
  const int limit = __ldcg(c.count + bh);
  const int p0 = __ldcg(src_pos + b);
  int running = base + prefix;

  const int lpr = row_bytes >> 4;      // lanes per row
  const int rpw = 32 / lpr;            // rows per warp pass
  const int sub = lane / lpr, col = lane % lpr;

  for (int r0 = tile0; r0 < tile0 + kScatterTile && r0 < n_rows; r0 += kScatterThreads) {
    const int i = r0 + threadIdx.x;
    const int flag = (i < n_rows) ? __ldcg(zb + (size_t)i * hkv) : 0;
    const unsigned ball = __ballot_sync(0xffffffffu, flag);
    const int in_warp = __popc(ball & ((1u << lane) - 1u));
    if (lane == 0) warp_tot[warp] = __popc(ball);
    __syncthreads();
    int warp_off = 0, round_total = 0;
    for (int w = 0; w < kScatterThreads / 32; ++w) {
      if (w < warp) warp_off += warp_tot[w];
      round_total += warp_tot[w];
    }
    const int rank = warp_off + in_warp;
    if (flag) {
      list_src[rank] = i;
      list_dst[rank] = running + rank;
    }
    __syncthreads();
    for (int e = warp * rpw + sub; e < round_total; e += (kScatterThreads / 32) * rpw) {
      const int src_i = list_src[e];
      const int dst = list_dst[e];
      if (dst >= limit) continue;  // dropped: capacity (flag already raised by the plan)
      const int page = __ldcg(c.page_table + (size_t)bh * c.max_pages + (dst >> 6));
      if (!page_ok(page, c.num_pages, c.err)) continue;  // debug build: flagged, skipped
      const size_t drow = (size_t)page * kPageRows + (dst & 63);
      size_t srow;
      if (from_ring) {
        const int slot = (p0 + src_i) % window;
        srow = ((size_t)bh * window + slot);
      } else {
        srow = ((size_t)b * src_batch_rows + src_i) * hkv + kh;
      }
      const uint4 kv = *reinterpret_cast<const uint4*>(Ksrc + srow * row_bytes + col * 16);
      const uint4 vv = *reinterpret_cast<const uint4*>(Vsrc + srow * row_bytes + col * 16);
      *reinterpret_cast<uint4*>(c.K + drow * row_bytes + col * 16) = kv;
      *reinterpret_cast<uint4*>(c.V + drow * row_bytes + col * 16) = vv;
      if (col == 0) {
        c.pos[drow] = p0 + src_i;
        if (c.u) c.u[drow] = u[((size_t)b * src_batch_rows + src_i) * hkv + kh];
      }
    }
    running += round_total;
    __syncthreads();
  }
}

// One warp per (batch row, key head).
__global__ void __launch_bounds__(128)
    decode_append_kernel(CacheMut c, RingMut r, const int32_t* __restrict__ t_pos,
                         const char* __restrict__ k_new, const char* __restrict__ v_new,
                         const uint8_t* __restrict__ z_new, const float* __restrict__ u_new,
                         int retire, int n_heads, int hkv, int window, int row_bytes) {
  grid_dependency_wait();    // programmatic dependent launch: inputs may come from the
  grid_dependents_launch();  // kernel before; the attention after may start its launch
  const int lane = threadIdx.x & 31;
  const int bh = blockIdx.x * 4 + (threadIdx.x >> 5);
  if (bh >= n_heads) return;
  const int b = bh / hkv, kh = bh % hkv;
  const int t = t_pos[b];
  if (t < 0) return;  // positions are non-negative by contract
  decode_append_warp(c, r, bh, b, kh, t, k_new, v_new, z_new ? z_new[bh] : (uint8_t)0,
                     (z_new && u_new) ? u_new[bh] : no_utility(), retire, hkv, window, row_bytes,
                     lane);
}

// grid (B*Hkv); the last min(n_rows, window) rows of a chunk go to their slots.
__global__ void __launch_bounds__(256)
    ring_write_kernel(char* __restrict__ Kwin, char* __restrict__ Vwin, uint8_t* __restrict__ zwin,
                      float* __restrict__ uwin, const char* __restrict__ Ksrc,
                      const char* __restrict__ Vsrc, const uint8_t* __restrict__ z_src,
                      const float* __restrict__ u_src, int gated_from,
                      const int32_t* __restrict__ src_pos, int n_rows, int src_batch_rows, int hkv,
                      int window, int row_bytes) {
  const int bh = blockIdx.x, b = bh / hkv, kh = bh % hkv;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int lpr = row_bytes >> 4, rpw = 32 / lpr, sub = lane / lpr, col = lane % lpr;
  const int n_w = n_rows < window ? n_rows : window;
  const int first = n_rows - n_w;
  const int p0 = src_pos[b];
  for (int r = warp * rpw + sub; r < n_w; r += (blockDim.x >> 5) * rpw) {
    const int i = first + r;
    const int slot = (p0 + i) % window;
    const size_t srow = ((size_t)b * src_batch_rows + i) * hkv + kh;
    const size_t drow = (size_t)bh * window + slot;
    const uint4 kv = *reinterpret_cast<const uint4*>(Ksrc + srow * row_bytes + col * 16);
    const uint4 vv = *reinterpret_cast<const uint4*>(Vsrc + srow * row_bytes + col * 16);
    *reinterpret_cast<uint4*>(Kwin + drow * row_bytes + col * 16) = kv;
    *reinterpret_cast<uint4*>(Vwin + drow * row_bytes + col * 16) = vv;
    if (col == 0) {
      const size_t zi = ((size_t)b * window + slot) * hkv + kh;
      zwin[zi] = (i >= gated_from) ? z_src[srow] : 0;
      if (uwin) uwin[zi] = (i >= gated_from) ? u_src[srow] : no_utility();
    }
  }
}

}  // namespace

cudaError_t launch_write_compact(const spkv_params& p, const spkv_cache& c, const spkv_ring* ring,
                                 int src_kind, const void* K_src, const void* V_src,
                                 const uint8_t* z, const float* u, const int32_t* src_pos,
                                 int n_rows, int src_batch_rows, cudaStream_t stream) {
  const int n_heads = p.B * p.Hkv;
  const int esize = p.dtype == SPKV_BF16 ? 2 : 4;
  const int row_bytes = p.head_dim * esize;
  CacheMut m = mut(c);
  cudaError_t e = launch_pdl(compact_plan, dim3(n_heads), dim3(256), 0, stream, m, z, n_rows,
                             src_batch_rows, p.Hkv);
  if (e != cudaSuccess) return e;
  const char* Ks = static_cast<const char*>(src_kind == SPKV_SRC_RING ? ring->K_win : K_src);
  const char* Vs = static_cast<const char*>(src_kind == SPKV_SRC_RING ? ring->V_win : V_src);
  dim3 grid(n_heads, (n_rows + kScatterTile - 1) / kScatterTile);
  return launch_pdl(compact_scatter, grid, dim3(kScatterThreads), 0, stream, m, Ks, Vs, z, u,
                    src_pos, n_rows, src_batch_rows, p.Hkv, row_bytes,
                    (int)(src_kind == SPKV_SRC_RING), p.window);
}

cudaError_t launch_decode_append(const spkv_params& p, const spkv_cache& c, const spkv_ring& ring,
                                 const int32_t* t_pos, const void* k_new, const void* v_new,
                                 const uint8_t* z_new, const float* u_new, int retire,
                                 cudaStream_t stream) {
  const int n_heads = p.B * p.Hkv;
  const int esize = p.dtype == SPKV_BF16 ? 2 : 4;
  return launch_pdl(decode_append_kernel, dim3((n_heads + 3) / 4), dim3(128), 0, stream, mut(c),
                    ring_mut(ring), t_pos, static_cast<const char*>(k_new),
                    static_cast<const char*>(v_new), z_new, u_new, retire, n_heads, p.Hkv, p.window,
                    p.head_dim * esize);
}

cudaError_t launch_ring_write(const spkv_params& p, const spkv_ring& ring, const void* K_src,
                              const void* V_src, const uint8_t* z_src, const float* u_src,
                              int gated_from, const int32_t* src_pos, int n_rows,
                              int src_batch_rows, cudaStream_t stream) {
  const int n_heads = p.B * p.Hkv;
  const int esize = p.dtype == SPKV_BF16 ? 2 : 4;
  ring_write_kernel<<<n_heads, 256, 0, stream>>>(
      static_cast<char*>(ring.K_win), static_cast<char*>(ring.V_win), ring.z_win, ring.u_win,
      static_cast<const char*>(K_src), static_cast<const char*>(V_src), z_src, u_src, gated_from,
      src_pos, n_rows, src_batch_rows, p.Hkv, p.window, p.head_dim * esize);
  return cudaGetLastError();
}

}  // namespace spkv
