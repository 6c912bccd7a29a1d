// rethreshold.cu -- post-hoc change of the gate threshold on a filled cache.
//
// "Self-Pruned Key-Value Attention" (arXiv 2605.14037), §3.3: at inference the
// sparsity can be adjusted after the fact by changing the threshold tau of Eq. (2).
// With the utility u of every stored row kept in u_pool, raising tau to tau' means
// dropping the rows with u < tau' from every key head's cache, keeping the others in
// order.  This is done in place, inside each head's own pages:
//   plan    one CTA per head: rows kept per page (u >= tau'), exclusive prefix over
//           the head's pages, read flags of its pages cleared;
//   move    persistent CTAs take pages, page-major, from a global counter; each CTA runs a
//           few independent pipelines (two page buffers, one agent lane that claims,
//           copies, raises the page's "page read" flag and checks those of the pages
//           it writes into, four writer warps), so that one page is read while the
//           previous one is written.  A kept row only moves towards the front, so its
//           new place lies in this page or in an earlier page of the same head; rows
//           are written into an earlier page only once that page has been read
//           (bounded wait).  A page's flag is raised before anything is waited on for
//           it, and pages are taken in increasing order, so every wait ends.
//   finish  counts become the kept counts; the ring's gates are recomputed from the
//           pending utilities; the workspace counters are cleared.
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
constexpr int kMaxHeadsR = 2048;

struct RethrWs {
  int* ctr;      // [4]: work counter, "a wait gave up"
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
  grid_dependents_launch();
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
#pragma unroll
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

// Persistent; pages in page-major order (item i is page i / n_heads of head
// i % n_heads, skipped where the head has fewer pages), claimed from ws.ctr[0] kBatch
// items at a time, so that the earlier pages a page writes into (about page j / 2 of
// its head, for half the rows kept) were claimed long before and have been read.  A CTA
// runs kPipes independent pipelines, each with two page buffers (K, V, positions,
// utilities), one agent lane and kWriters writer warps.  The agent, for its pages in turn
// (page k of the pipeline in buffer k % 2):
//   waits until the writers have emptied the buffer (page k - 2) and starts the copies
//   of page k, claimed earlier with its page-table entry and prefix looked up;
//   looks up the (at most two) pages the page's rows can land in (destinations lie in
//   [base, base + rows)), loads their "read" flags and claims page k + 1 while the
//   copies are in flight;
//   once they land raises page k's "read" flag, then waits (bounded) until the
//   destination pages that are earlier pages of the head have been read.
// The writers take the buffers in turn, place the kept rows and write them out, so
// that page k + 1 is read while page k is written.
// Ordering: a page's copies have completed (its mbarrier phase) before its flag is
// stored, and stores into a page are issued only after its flag has been seen, so no
// store can reach a page before its reads; no fence is needed.
// Progress: pages are claimed in increasing order; a pipeline holds its pages in that
// order and a page waits only on lower pages.  Take the lowest claimed page M whose
// flag is down: the pages its pipeline holds before M are lower, so flagged, their
// waits are on still lower pages (all flagged), and their writes need nothing from
// elsewhere; so the agent reaches M, its buffer frees, its copies start, and its flag
// is raised when they land.
constexpr int kPipes = 3;
constexpr int kBatch = 4;  // items per claim
constexpr int kWriters = 4;  // writer warps per pipeline
// warps: writer wi of pipeline s is warp wi * kPipes + s; the agent of s is warp
// kWriters * kPipes + s
constexpr int kMoveThreads = 32 * (kWriters + 1) * kPipes;

struct MoveItem {
  int item;  // >= total: no more pages for this pipeline
  int bh, j, page, rows, base;
  int dpage[2];  // pool pages of the head's pages base / 64 and base / 64 + 1 (or -1)
};

__device__ __forceinline__ int load_relaxed(const int* p) {
  int v;
  asm volatile("ld.relaxed.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void store_relaxed(int* p, int v) {
  asm volatile("st.relaxed.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__global__ void __launch_bounds__(kMoveThreads)
    rethr_move(CacheMut c, RethrWs ws, float tau, int n_heads, int row_bytes,
               unsigned long long wait_ns) {
  extern __shared__ __align__(128) char smem[];
  const uint32_t page_bytes = (uint32_t)kPageRows * row_bytes;
  const uint32_t buf_bytes = 2 * page_bytes + 2 * kPageRows * 4;  // K, V, pos, u
  int* s_np = reinterpret_cast<int*>(smem + 2 * kPipes * (size_t)buf_bytes);  // [n_heads] pages
  __shared__ MoveItem s_it[kPipes][2];
  __shared__ int s_src[kPipes][2][kPageRows], s_dst[kPipes][2][kPageRows];  // kept rows: from, to
  __shared__ int s_maxp;
  __shared__ int s_ok[kPipes][2];
  __shared__ __align__(8) uint64_t full[kPipes][2], ready[kPipes][2], empty[kPipes][2];
  __shared__ __align__(8) uint64_t lists[kPipes][2];  // writer 0 has written the row lists
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  grid_dependents_launch();
  if (tid == 0) {
    for (int s = 0; s < kPipes; ++s)
      for (int b = 0; b < 2; ++b) {
        mbar_init(&full[s][b], 1);
        mbar_init(&ready[s][b], 1);
        mbar_init(&empty[s][b], kWriters);
        mbar_init(&lists[s][b], 1);
      }
    fence_mbar_init();
  }
  // pages per head and their maximum (counts are not written by the plan kernel)
  if (tid == 0) s_maxp = 0;
  __syncthreads();
  for (int h = tid; h < n_heads; h += kMoveThreads) {
    const int np = (c.count[h] + kPageRows - 1) / kPageRows;
    s_np[h] = np;
    atomicMax(&s_maxp, np);
  }
  __syncthreads();
  grid_dependency_wait();  // prefix sums and cleared flags of the plan kernel
  const int total = n_heads * s_maxp;  // items, holes included
  const int s = warp % kPipes;
  auto buf = [&](int b) { return smem + (size_t)(2 * s + b) * buf_bytes; };

  if (warp >= kWriters * kPipes) {
    // ------------------------------ agent of pipeline s -----------------------------
    if (lane != 0) return;
    // the next page of this pipeline: the next item of its batch that is a page (a new
    // batch when the batch is used up), with its page-table entry and destination base
    int bnext = 0, bend = 0;
    auto claim = [&]() {
      MoveItem it;
      it.bh = it.j = it.page = it.rows = it.base = 0;
      it.dpage[0] = it.dpage[1] = -1;
      while (true) {
        if (bnext == bend) {
          bnext = atomicAdd(ws.ctr, kBatch);
          bend = bnext + kBatch;
        }
        it.item = bnext++;
        if (it.item >= total) return it;
        it.bh = it.item % n_heads;
        it.j = it.item / n_heads;
        if (it.j < s_np[it.bh]) break;
      }
      const int lo = it.bh;
      const int n = c.count[lo];
      it.page = c.page_table[(size_t)lo * c.max_pages + it.j];
      it.base = ws.pref[(size_t)lo * (c.max_pages + 1) + it.j];
      it.rows = min(kPageRows, n - it.j * kPageRows);
      if (!page_ok(it.page, c.num_pages, c.err)) it.page = 0;  // debug build: flagged
      return it;
    };
    MoveItem nxt = claim();
    for (int k = 0;; ++k) {
      const int b = k & 1;
      if (k >= 2 && !mbar_wait(&empty[s][b], ((k >> 1) - 1) & 1, c.err)) return;
      if (nxt.item >= total) {
        s_it[s][b].item = total;  // the end marker
        mbar_arrive(&ready[s][b]);
        return;
      }
      MoveItem it = nxt;
      char* st = buf(b);
      mbar_arrive_expect_tx(&full[s][b], buf_bytes);
      bulk_g2s(st, c.K + (size_t)it.page * page_bytes, page_bytes, &full[s][b]);
      bulk_g2s(st + page_bytes, c.V + (size_t)it.page * page_bytes, page_bytes, &full[s][b]);
      bulk_g2s(st + 2 * page_bytes, c.pos + (size_t)it.page * kPageRows, kPageRows * 4, &full[s][b]);
      bulk_g2s(st + 2 * page_bytes + kPageRows * 4, c.u + (size_t)it.page * kPageRows,
               kPageRows * 4, &full[s][b]);
      // while the copies are in flight: destination pages, their flags, the next claim
      const int32_t* table = c.page_table + (size_t)it.bh * c.max_pages;
      int* flag = ws.flag + (size_t)it.bh * c.max_pages;
      const int d0 = it.base / kPageRows;
      const int dl = (it.base + it.rows - 1) / kPageRows;  // <= it.j
      const int dw = min(dl, it.j - 1);                     // last earlier page written into
      it.dpage[0] = table[d0];
      if (dl > d0) it.dpage[1] = table[d0 + 1];
      int f0 = dw >= d0 ? load_relaxed(flag + d0) : 1;
      int f1 = dw > d0 ? load_relaxed(flag + d0 + 1) : 1;
      nxt = claim();
      if (!mbar_wait(&full[s][b], (k >> 1) & 1, c.err)) return;
      store_relaxed(flag + it.j, 1);  // this page has been read
      int ok = 1;
      if (!(f0 && f1)) {
        const uint64_t t0 = global_ns();
        while (true) {
          if (!f0) f0 = load_relaxed(flag + d0);
          if (!f1) f1 = load_relaxed(flag + d0 + 1);
          if (f0 && f1) break;
          // once any wait of this call has given up, the others give up at once, so
          // that a call with a lost page ends after one wait limit
          if (global_ns() - t0 > wait_ns || load_relaxed(ws.ctr + 1) != 0) {
            atomicOr(c.err, SPKV_FLAG_TIMEOUT);
            atomicExch(ws.ctr + 1, 1);
            ok = 0;
            break;
          }
        }
      }
      s_it[s][b] = it;
      s_ok[s][b] = ok;
      mbar_arrive(&ready[s][b]);  // release: s_it and s_ok are visible to the writer
    }
  }
  // ------------------------------ writers of pipeline s -----------------------------
  const int wi = warp / kPipes;  // 0: also places the rows and writes positions, utilities
  const uint32_t lt = (1u << lane) - 1u;
  for (int k = 0;; ++k) {
    const int b = k & 1;
    const uint32_t ph = (k >> 1) & 1;
    if (!mbar_wait(&ready[s][b], ph, c.err)) return;
    const MoveItem it = s_it[s][b];
    if (it.item >= total) return;
    if (!mbar_wait(&full[s][b], ph, c.err)) return;  // the copies' data, seen by this warp
    const char* st = buf(b);
    const int* s_pos = reinterpret_cast<const int*>(st + 2 * page_bytes);
    const float* s_u = reinterpret_cast<const float*>(st + 2 * page_bytes + kPageRows * 4);
    // rows lane and 32 + lane: kept?  new places in the head's row order
    const bool k0 = lane < it.rows && s_u[lane] >= tau;
    const bool k1 = 32 + lane < it.rows && s_u[32 + lane] >= tau;
    const unsigned b0 = __ballot_sync(0xffffffffu, k0), b1 = __ballot_sync(0xffffffffu, k1);
    const int d0 = it.base / kPageRows;
    auto drow_of = [&](int dst) {
      const int dpage = dst / kPageRows == d0 ? it.dpage[0] : it.dpage[1];
      return page_ok(dpage, c.num_pages, c.err) ? dpage * kPageRows + dst % kPageRows : -1;
    };
    const int dr0 = k0 ? drow_of(it.base + __popc(b0 & lt)) : -1;
    const int dr1 = k1 ? drow_of(it.base + __popc(b0) + __popc(b1 & lt)) : -1;
    // the kept rows in order: where from (row of the page), where to (row of the pool)
    if (wi == 0) {
      if (k0) {
        s_src[s][b][__popc(b0 & lt)] = lane;
        s_dst[s][b][__popc(b0 & lt)] = dr0;
      }
      if (k1) {
        s_src[s][b][__popc(b0) + __popc(b1 & lt)] = 32 + lane;
        s_dst[s][b][__popc(b0) + __popc(b1 & lt)] = dr1;
      }
    }
    if (wi == 0) {
      __syncwarp();
      if (lane == 0) mbar_arrive(&lists[s][b]);
    } else if (!mbar_wait(&lists[s][b], ph, c.err)) {
      return;
    }
    if (s_ok[s][b]) {
      // (kept row, 16-byte piece) pairs over the lanes: K pieces, then V pieces of a row
      const int lpr = row_bytes >> 4;               // pieces per row, a power of two
      const int sh = __ffs(2 * lpr) - 1;             // log2 of the pieces of K and V
      const int n_e = (__popc(b0) + __popc(b1)) << sh;
#pragma unroll 4
      for (int e = wi * 32 + lane; e < n_e; e += 32 * kWriters) {
        const int kr = e >> sh, pc = e & (2 * lpr - 1);
        const int drow = s_dst[s][b][kr];
        if (drow < 0) continue;
        const int kv = pc >= lpr, off = (pc - kv * lpr) * 16;
        char* dbase = kv ? c.V : c.K;
        *reinterpret_cast<uint4*>(dbase + (size_t)drow * row_bytes + off) =
            *reinterpret_cast<const uint4*>(st + kv * page_bytes + (size_t)s_src[s][b][kr] * row_bytes + off);
      }
      if (wi == 0 && dr0 >= 0) {
        c.pos[dr0] = s_pos[lane];
        c.u[dr0] = s_u[lane];
      }
      if (wi == 0 && dr1 >= 0) {
        c.pos[dr1] = s_pos[32 + lane];
        c.u[dr1] = s_u[32 + lane];
      }
    }
    // this warp is done with the buffer (and its row lists, rewritten for page k + 2,
    // which is issued only after both warps have arrived here)
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s][b]);
  }
}

// Counts, ring gates, work counter.
__global__ void __launch_bounds__(256)
    rethr_finish(CacheMut c, RethrWs ws, RingMut r, float tau, int n_heads, int ring_entries) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  grid_dependency_wait();  // every page has been moved
  if (i < n_heads) {
    const int n = c.count[i];
    const int np = (n + kPageRows - 1) / kPageRows;
    const int kept = ws.pref[(size_t)i * (c.max_pages + 1) + np];
    c.count[i] = kept;
    c.count_prev[i] = kept;
  }
  if (r.u && i < ring_entries) r.z[i] = r.u[i] >= tau ? 1 : 0;
  if (i == 0) ws.ctr[0] = ws.ctr[1] = 0;
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
  const size_t smem = (size_t)2 * kPipes * (2 * kPageRows * row_bytes + 2 * kPageRows * 4) +
                      ((size_t)n_heads * 4 + 15) / 16 * 16;
  {
    cudaError_t e = ensure_dynamic_smem((const void*)rethr_move, (int)smem);
    if (e != cudaSuccess) return e;
  }
  int per_sm = 0;
  {
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, rethr_move,
                                                                  kMoveThreads, smem);
    if (e != cudaSuccess) return e;
  }
  per_sm = per_sm < 1 ? 1 : (per_sm > 8 ? 8 : per_sm);
  const unsigned long long w = g_flag_wait_ns.load();
  cudaError_t e = launch_pdl(rethr_move, dim3(num_sms * per_sm), dim3(kMoveThreads), smem, stream,
                             m, ws, tau_new, n_heads, row_bytes, w ? w : kWaitLimitNs);
  if (e != cudaSuccess) return e;
  RingMut r = ring ? ring_mut(*ring) : RingMut{nullptr, nullptr, nullptr, nullptr};
  const int ring_entries = ring ? p.B * p.window * p.Hkv : 0;
  const int n = n_heads > ring_entries ? n_heads : ring_entries;
  e = launch_pdl(rethr_finish, dim3((n + 255) / 256), dim3(256), 0, stream, m, ws, r, tau_new,
                 n_heads, ring_entries);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace spkv
