// rethreshold.cu -- post-hoc change of the gate threshold on a filled cache.
//
// "Self-Pruned Key-Value Attention" (arXiv 2605.14037), §3.3: at inference the
// sparsity can be adjusted after the fact by changing the threshold tau of Eq. (2).
// With the utility u of every stored row kept in u_pool, raising tau to tau' means
// dropping the rows with u < tau' from every key head's cache, keeping the others in
// order.  This is done in place, inside each head's own pages:
//   plan    one CTA per head: rows kept per page (u >= tau'), exclusive prefix over
//           the head's pages, read flags of its pages cleared;
//   move    persistent CTAs take pages in order from a global counter.  A CTA copies
//           its page (K, V, pos, u) into shared memory, publishes "page read", then
//           writes the page's kept rows to their new places, while its next page is
//           already being read into a second buffer.  A kept row only moves
//           towards the front, so its new place lies in this page or in an earlier
//           page of the same head; before writing into an earlier page the CTA waits
//           (bounded) until that page has been read.  A page's flag is raised before
//           its CTA waits on anything, and pages are taken in increasing order by
//           running CTAs, so every wait ends.
//   finish  counts become the kept counts; the ring's gates are recomputed from the
//           pending utilities; the work counter is cleared.
#include <atomic>

#include "append.cuh"
#include "common.cuh"
#include "host.h"
#include "launch.h"

namespace spkv {
namespace {

// limit of the page-flag waits of the move kernel (ns); 0: the library default
std::atomic<unsigned long long> g_flag_wait_ns{0};

constexpr int kPlanThreads = 256;
constexpr int kMoveThreads = 128;
constexpr int kMaxHeadsR = 2048;

struct RethrWs {
  int* ctr;      // [4]: work counter
  int* pref;     // [heads][max_pages + 1] kept rows before each page
  int* flag;     // [heads][max_pages] page read
};

RethrWs carve(void* ws, int heads, int max_pages) {
  char* w = static_cast<char*>(ws);
  RethrWs r;
  r.ctr = reinterpret_cast<int*>(w);
  r.pref = reinterpret_cast<int*>(w + 256);
  r.flag = r.pref + (size_t)heads * (max_pages + 1);
  return r;
}

__device__ __forceinline__ int block_scan_excl(int v, int* red, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int x = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += x;
  }
  if (lane == 31) red[warp] = inc;
  __syncthreads();
  int before = 0;
  total = 0;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {
    before += w < warp ? red[w] : 0;
    total += red[w];
  }
  __syncthreads();
  return before + inc - v;
}

// One CTA per head.  Pages are counted 256 at a time (one thread per page, 64 rows).
__global__ void __launch_bounds__(kPlanThreads)
    rethr_plan(CacheMut c, RethrWs ws, float tau) {
  __shared__ int red[kPlanThreads / 32];
  const int bh = blockIdx.x;
  const int n = c.count[bh];
  const int np = (n + kPageRows - 1) / kPageRows;
  int* pref = ws.pref + (size_t)bh * (c.max_pages + 1);
  int* flag = ws.flag + (size_t)bh * c.max_pages;
  int carry = 0;
  for (int j0 = 0; j0 < np; j0 += kPlanThreads) {
    const int j = j0 + threadIdx.x;
    int kept = 0;
    if (j < np) {
      int page = c.page_table[(size_t)bh * c.max_pages + j];
      if (!page_ok(page, c.num_pages, c.err)) page = 0;  // debug build: flagged
      const int rows = min(kPageRows, n - j * kPageRows);
      const float4* u4 = reinterpret_cast<const float4*>(c.u + (size_t)page * kPageRows);
#pragma unroll 4
      for (int i = 0; i < kPageRows / 4; ++i) {
        const float4 v = u4[i];
        kept += (4 * i + 0 < rows && v.x >= tau) + (4 * i + 1 < rows && v.y >= tau) +
                (4 * i + 2 < rows && v.z >= tau) + (4 * i + 3 < rows && v.w >= tau);
      }
      flag[j] = 0;
    }
    int total = 0;
    const int ex = block_scan_excl(kept, red, total);
    if (j < np) pref[j] = carry + ex;
    carry += total;
  }
  if (threadIdx.x == 0) pref[np] = carry;
}

// Persistent: pages of all heads in order (head-major), claimed from ws.ctr[0].  Two
// page buffers: while a page's kept rows are written out, the next claimed page is
// already being read.  Progress: pages are claimed in increasing order, a page's flag
// is raised as soon as its read lands (before its CTA waits on anything), and a page only
// waits for earlier pages of its head; every page below the lowest claimed page whose
// flag is still down is flagged, so the CTA holding that page (current, or next after a
// current page whose waits all end) raises its flag.
struct MoveItem {
  int item;  // >= total: none
  int bh, j, page, rows, base;
};

__global__ void __launch_bounds__(kMoveThreads)
    rethr_move(CacheMut c, RethrWs ws, float tau, int n_heads, int row_bytes,
               unsigned long long wait_ns) {
  extern __shared__ __align__(16) char smem[];
  const uint32_t page_bytes = (uint32_t)kPageRows * row_bytes;
  char* buf[2] = {smem, smem + 2 * (size_t)page_bytes};  // [K page][V page] x 2
  int* s_base = reinterpret_cast<int*>(smem + 4 * (size_t)page_bytes);  // [n_heads + 1]
  __shared__ int s_pos[2][kPageRows];
  __shared__ float s_u[2][kPageRows];
  __shared__ int s_dst[kPageRows];  // new row index, or -1
  __shared__ MoveItem s_it[2];
  __shared__ int s_ok, s_wc[2];
  __shared__ __align__(8) uint64_t bar[2];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  if (tid == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    fence_mbar_init();
  }
  // pages per head, prefix over heads
  {
    __shared__ int red[kMoveThreads / 32];
    int carry = 0;
    for (int h0 = 0; h0 < n_heads; h0 += kMoveThreads) {
      const int h = h0 + tid;
      const int np = h < n_heads ? (c.count[h] + kPageRows - 1) / kPageRows : 0;
      int tot = 0;
      const int ex = block_scan_excl(np, red, tot);
      if (h < n_heads) s_base[h] = carry + ex;
      carry += tot;
    }
    if (tid == 0) s_base[n_heads] = carry;
  }
  __syncthreads();
  const int total = s_base[n_heads];

  // thread 0: claim the next page and start reading it into buffer b (K, V by bulk copy;
  // positions and utilities by the first 64 threads after the item is published)
  auto claim = [&](int b) {
    MoveItem it;
    it.item = atomicAdd(ws.ctr, 1);
    it.bh = it.j = it.page = it.rows = it.base = 0;
    if (it.item < total) {
      int lo = 0, hi = n_heads - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_base[mid] <= it.item) lo = mid; else hi = mid - 1;
      }
      it.bh = lo;
      it.j = it.item - s_base[lo];
      it.rows = min(kPageRows, c.count[lo] - it.j * kPageRows);
      it.page = c.page_table[(size_t)lo * c.max_pages + it.j];
      if (!page_ok(it.page, c.num_pages, c.err)) it.page = 0;  // debug build: flagged
      it.base = ws.pref[(size_t)lo * (c.max_pages + 1) + it.j];
      mbar_arrive_expect_tx(&bar[b], 2 * page_bytes);
      bulk_g2s(buf[b], c.K + (size_t)it.page * page_bytes, page_bytes, &bar[b]);
      bulk_g2s(buf[b] + page_bytes, c.V + (size_t)it.page * page_bytes, page_bytes, &bar[b]);
    }
    s_it[b] = it;
  };
  if (tid == 0) claim(0);
  __syncthreads();
  for (int round = 0;; ++round) {
    const int cur = round & 1;
    const MoveItem it = s_it[cur];
    if (it.item >= total) break;
    if (tid < kPageRows) {
      s_pos[cur][tid] = c.pos[(size_t)it.page * kPageRows + tid];
      s_u[cur][tid] = c.u[(size_t)it.page * kPageRows + tid];
    }
    if (tid == 0) claim(cur ^ 1);  // the next page's read overlaps this page's writes
    mbar_wait(&bar[cur], (round >> 1) & 1, c.err);
    __syncthreads();
    int* flag = ws.flag + (size_t)it.bh * c.max_pages;
    if (tid == 0) {
      __threadfence();
      atomicExch(flag + it.j, 1);  // this page has been read
    }
    // new places of the kept rows: rows 0-31 by warp 0, rows 32-63 by warp 1
    bool keep = false;
    unsigned ball = 0;
    if (warp < 2) {
      const int r = warp * 32 + lane;
      keep = r < it.rows && s_u[cur][r] >= tau;
      ball = __ballot_sync(0xffffffffu, keep);
      if (lane == 0) s_wc[warp] = __popc(ball);
    }
    __syncthreads();
    if (warp < 2) {
      const int r = warp * 32 + lane;
      s_dst[r] = keep ? it.base + (warp ? s_wc[0] : 0) + __popc(ball & ((1u << lane) - 1u)) : -1;
    }
    __syncthreads();
    const int kept = s_wc[0] + s_wc[1];
    // wait until every earlier page we write into has been read
    if (tid == 0) {
      int ok = 1;
      if (kept > 0) {
        const int d0 = it.base / kPageRows, d1 = (it.base + kept - 1) / kPageRows;
        for (int d = d0; d <= d1 && ok; ++d) {
          if (d >= it.j) break;
          if (atomicAdd(flag + d, 0) != 0) continue;
          const uint64_t t0 = global_ns();
          while (atomicAdd(flag + d, 0) == 0) {
            if (global_ns() - t0 > wait_ns) {
              atomicOr(c.err, SPKV_FLAG_TIMEOUT);
              ok = 0;
              break;
            }
          }
        }
        __threadfence();
      }
      s_ok = ok;
    }
    __syncthreads();
    const int32_t* table = c.page_table + (size_t)it.bh * c.max_pages;
    if (s_ok && kept > 0) {
      const char* kbuf = buf[cur];
      const char* vbuf = buf[cur] + page_bytes;
      const int lpr = row_bytes >> 4;  // 16-byte pieces per row
      for (int e = tid; e < kPageRows * lpr; e += kMoveThreads) {
        const int r = e / lpr, off = (e % lpr) * 16;
        const int dst = s_dst[r];
        if (dst < 0) continue;
        const int dpage = table[dst / kPageRows];
        if (!page_ok(dpage, c.num_pages, c.err)) continue;  // debug build: flagged, skipped
        const size_t drow = (size_t)dpage * kPageRows + (dst % kPageRows);
        *reinterpret_cast<uint4*>(c.K + drow * row_bytes + off) =
            *reinterpret_cast<const uint4*>(kbuf + (size_t)r * row_bytes + off);
        *reinterpret_cast<uint4*>(c.V + drow * row_bytes + off) =
            *reinterpret_cast<const uint4*>(vbuf + (size_t)r * row_bytes + off);
      }
      if (tid < kPageRows && s_dst[tid] >= 0) {
        const int dst = s_dst[tid];
        const int dpage = table[dst / kPageRows];
        if (page_ok(dpage, c.num_pages, c.err)) {
          const size_t drow = (size_t)dpage * kPageRows + (dst % kPageRows);
          c.pos[drow] = s_pos[cur][tid];
          c.u[drow] = s_u[cur][tid];
        }
      }
    }
    __syncthreads();  // this buffer is refilled two pages from now
  }
  // a page claimed past the end was never read: nothing in flight
}

// Counts, ring gates, work counter.
__global__ void __launch_bounds__(256)
    rethr_finish(CacheMut c, RethrWs ws, RingMut r, float tau, int n_heads, int ring_entries) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n_heads) {
    const int n = c.count[i];
    const int np = (n + kPageRows - 1) / kPageRows;
    const int kept = ws.pref[(size_t)i * (c.max_pages + 1) + np];
    c.count[i] = kept;
    c.count_prev[i] = kept;
  }
  if (r.u && i < ring_entries) r.z[i] = r.u[i] >= tau ? 1 : 0;
  if (i == 0) ws.ctr[0] = 0;
}

}  // namespace

void set_flag_wait_ns(unsigned long long ns) { g_flag_wait_ns.store(ns); }

size_t rethreshold_workspace_bytes(const spkv_params& p, const spkv_cache& c) {
  const size_t heads = (size_t)p.B * p.Hkv;
  return 256 + heads * (c.max_pages_per_head + 1) * 4 + heads * c.max_pages_per_head * 4;
}

cudaError_t launch_rethreshold(const spkv_params& p, const spkv_cache& c, const spkv_ring* ring,
                               float tau_new, void* workspace, int num_sms, cudaStream_t stream) {
  const int n_heads = p.B * p.Hkv;
  if (n_heads > kMaxHeadsR) return cudaErrorInvalidValue;
  const int esize = p.dtype == SPKV_BF16 ? 2 : 4;
  const int row_bytes = p.head_dim * esize;
  CacheMut m = cache_mut(c);
  RethrWs ws = carve(workspace, n_heads, c.max_pages_per_head);
  rethr_plan<<<n_heads, kPlanThreads, 0, stream>>>(m, ws, tau_new);
  const size_t smem = (size_t)4 * kPageRows * row_bytes + (size_t)(n_heads + 1) * 4;
  {
    cudaError_t e = ensure_dynamic_smem((const void*)rethr_move, (int)smem);
    if (e != cudaSuccess) return e;
  }
  // as many CTAs per SM as shared memory allows (each has two pages in flight)
  int per_sm = (int)((216u << 10) / (smem + (2u << 10)));
  per_sm = per_sm < 1 ? 1 : (per_sm > 8 ? 8 : per_sm);
  const unsigned long long w = g_flag_wait_ns.load();
  rethr_move<<<num_sms * per_sm, kMoveThreads, smem, stream>>>(m, ws, tau_new, n_heads, row_bytes,
                                                               w ? w : kWaitLimitNs);
  RingMut r = ring ? ring_mut(*ring) : RingMut{nullptr, nullptr, nullptr, nullptr};
  const int ring_entries = ring ? p.B * p.window * p.Hkv : 0;
  const int n = n_heads > ring_entries ? n_heads : ring_entries;
  rethr_finish<<<(n + 255) / 256, 256, 0, stream>>>(m, ws, r, tau_new, n_heads, ring_entries);
  return cudaGetLastError();
}

}  // namespace spkv
