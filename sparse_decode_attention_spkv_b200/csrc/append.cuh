// append.cuh -- one warp's part of a per-token decode step on the window ring and the
// gated cache ("Self-Pruned Key-Value Attention", arXiv 2605.14037, §2.1: the token
// that leaves the causal window is written to the persistent cache only if its gate
// is 1; the new token takes its ring slot).  Shared by the append kernel and the
// fused score + append kernel.
#pragma once

#include "common.cuh"

namespace spkv {

struct CacheMut {
  char* K;
  char* V;
  int32_t* pos;
  int32_t* page_table;
  int32_t* count;
  int32_t* count_prev;
  int32_t* pool_top;
  uint32_t* err;
  float* u;  // per stored row, or null
  int num_pages;
  int max_pages;
};

inline CacheMut cache_mut(const spkv_cache& c) {
  return CacheMut{static_cast<char*>(c.K_pool), static_cast<char*>(c.V_pool), c.pos_pool,
                  c.page_table, c.count, c.count_prev, c.pool_top, c.err_flag, c.u_pool,
                  c.num_pages, c.max_pages_per_head};
}

struct RingMut {
  char* K;
  char* V;
  uint8_t* z;
  float* u;  // [B][window][hkv] pending utilities, or null
};

inline RingMut ring_mut(const spkv_ring& r) {
  return RingMut{static_cast<char*>(r.K_win), static_cast<char*>(r.V_win), r.z_win, r.u_win};
}

// "no pending utility" in the ring (all bits set: a NaN, never >= a threshold)
__device__ __forceinline__ float no_utility() { return __uint_as_float(0xffffffffu); }

// A head's page for cache row i when i starts a page: the page it already owns there
// (kept from before a re-threshold), else a new one from the pool (-1 if none fits).
__device__ __forceinline__ int page_for_new_row(const CacheMut& c, int bh, int i) {
  if ((i >> 6) >= c.max_pages) {
    atomicOr(c.err, SPKV_FLAG_TABLE_FULL);
    return -1;
  }
  int32_t* slot = c.page_table + (size_t)bh * c.max_pages + (i >> 6);
  const int owned = *slot;
  if (owned >= 0) return page_ok(owned, c.num_pages, c.err) ? owned : -1;
  const int pg = atomicAdd(c.pool_top, 1);
  if (pg >= c.num_pages) {
    atomicOr(c.err, SPKV_FLAG_POOL_FULL);
    return -1;
  }
  *slot = pg;
  return pg;
}

// Whole warp, head bh = b * hkv + kh, query position t >= 0: retire s = t - window
// (appended to the cache when `retire` and its stored gate is 1), then store the
// new token's k/v rows and gate in slot t % window.
__device__ __forceinline__ void decode_append_warp(const CacheMut& c, const RingMut& r, int bh,
                                                   int b, int kh, int t, const char* k_new,
                                                   const char* v_new, uint8_t z_new, float u_new,
                                                   int retire, int hkv, int window, int row_bytes,
                                                   int lane) {
  const int slot = t % window;
  const int s = t - window;
  const int lpr = row_bytes >> 4;
  const size_t ring_row = (size_t)bh * window + slot;
  uint8_t* zslot = r.z + ((size_t)b * window + slot) * hkv + kh;
  if (retire && s >= 0 && *zslot) {
    const int i = c.count[bh];
    int page = -1;
    if ((i & 63) == 0) {
      if (lane == 0) page = page_for_new_row(c, bh, i);
      page = __shfl_sync(0xffffffffu, page, 0);
    } else {
      page = c.page_table[(size_t)bh * c.max_pages + (i >> 6)];
      if (!page_ok(page, c.num_pages, c.err)) page = -1;  // debug build: flagged, skipped
    }
    if (page >= 0) {
      const size_t drow = (size_t)page * kPageRows + (i & 63);
      if (lane < lpr) {
        const uint4 kv = *reinterpret_cast<const uint4*>(r.K + ring_row * row_bytes + lane * 16);
        const uint4 vv = *reinterpret_cast<const uint4*>(r.V + ring_row * row_bytes + lane * 16);
        *reinterpret_cast<uint4*>(c.K + drow * row_bytes + lane * 16) = kv;
        *reinterpret_cast<uint4*>(c.V + drow * row_bytes + lane * 16) = vv;
      }
      if (lane == 0) {
        c.pos[drow] = s;
        if (c.u) c.u[drow] = r.u ? r.u[((size_t)b * window + slot) * hkv + kh] : no_utility();
        c.count[bh] = i + 1;
      }
    }
  }
  __syncwarp();
  if (lane < lpr) {
    const uint4 kv = *reinterpret_cast<const uint4*>(k_new + (size_t)bh * row_bytes + lane * 16);
    const uint4 vv = *reinterpret_cast<const uint4*>(v_new + (size_t)bh * row_bytes + lane * 16);
    *reinterpret_cast<uint4*>(r.K + ring_row * row_bytes + lane * 16) = kv;
    *reinterpret_cast<uint4*>(r.V + ring_row * row_bytes + lane * 16) = vv;
  }
  if (lane == 0) {
    *zslot = z_new;
    if (r.u) r.u[((size_t)b * window + slot) * hkv + kh] = u_new;
  }
}

// ---- the same step split in two, for kernels that know the new gate late -------------
//
// append_prefetch issues every read of the step that does not depend on the new gate
// (the old row in slot t % window and its gate, the head's count and current page, the
// new k/v rows) with the old and new rows copied into `stage` (4 * row_bytes of shared
// memory, 16-byte aligned) by cp.async; append_commit then writes the step once the gate
// is known.  Together they do exactly what decode_append_warp does.
struct AppendPre {
  int t;     // query position (< 0: no step for this row)
  int zs;    // stored gate of the retiring slot
  int cnt;   // head's cache count before the step
  int page;  // page table entry of row cnt (-1: none yet)
  float us;  // stored utility of the retiring slot
};

__device__ __forceinline__ void cp_async16(void* dst_smem, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst_smem)), "l"(src)
               : "memory");
}

__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;" ::: "memory");
}

__device__ __forceinline__ AppendPre append_prefetch(const CacheMut& c, const RingMut& r, int bh,
                                                     int b, int kh, int t, const char* k_new,
                                                     const char* v_new, int hkv, int window,
                                                     int row_bytes, int lane, char* stage) {
  AppendPre a;
  a.t = t;
  a.zs = 0;
  a.cnt = 0;
  a.page = -1;
  a.us = 0.f;
  if (t < 0) return a;
  const int slot = t % window;
  const size_t ring_row = (size_t)bh * window + slot;
  const int lpr = row_bytes >> 4;
  for (int e = lane; e < 4 * lpr; e += 32) {
    const int which = e / lpr, off = (e % lpr) * 16;
    const char* src = which == 0   ? r.K + ring_row * row_bytes
                      : which == 1 ? r.V + ring_row * row_bytes
                      : which == 2 ? k_new + (size_t)bh * row_bytes
                                   : v_new + (size_t)bh * row_bytes;
    cp_async16(stage + which * row_bytes + off, src + off);
  }
  a.zs = r.z[((size_t)b * window + slot) * hkv + kh];
  if (r.u && c.u) a.us = r.u[((size_t)b * window + slot) * hkv + kh];
  a.cnt = c.count[bh];
  if (t - window >= 0 && a.zs && (a.cnt >> 6) < c.max_pages)
    a.page = c.page_table[(size_t)bh * c.max_pages + (a.cnt >> 6)];
  return a;
}

__device__ __forceinline__ void append_commit(const CacheMut& c, const RingMut& r, const AppendPre& a,
                                              int bh, int b, int kh, uint8_t z_new, float u_new,
                                              int hkv, int window, int row_bytes, int lane,
                                              const char* stage) {
  if (a.t < 0) return;
  const int t = a.t;
  const int slot = t % window;
  const int s = t - window;
  const int lpr = row_bytes >> 4;
  const size_t ring_row = (size_t)bh * window + slot;
  cp_async_wait_all();
  __syncwarp();
  if (s >= 0 && a.zs) {
    const int i = a.cnt;
    int page = a.page;
    if ((i & 63) == 0 && page < 0) {  // a page boundary with no page owned there yet
      if (lane == 0) page = page_for_new_row(c, bh, i);
      page = __shfl_sync(0xffffffffu, page, 0);
    } else if (page >= 0 && !page_ok(page, c.num_pages, c.err)) {
      page = -1;  // debug build: flagged, skipped
    }
    if (page >= 0) {
      const size_t drow = (size_t)page * kPageRows + (i & 63);
      for (int e = lane; e < 2 * lpr; e += 32) {
        const int which = e / lpr, off = (e % lpr) * 16;
        const uint4 v = *reinterpret_cast<const uint4*>(stage + which * row_bytes + off);
        *reinterpret_cast<uint4*>((which == 0 ? c.K : c.V) + drow * row_bytes + off) = v;
      }
      if (lane == 0) {
        c.pos[drow] = s;
        if (c.u) c.u[drow] = r.u ? a.us : no_utility();
        c.count[bh] = i + 1;
      }
    }
  }
  for (int e = lane; e < 2 * lpr; e += 32) {
    const int which = e / lpr, off = (e % lpr) * 16;
    const uint4 v = *reinterpret_cast<const uint4*>(stage + (2 + which) * row_bytes + off);
    *reinterpret_cast<uint4*>((which == 0 ? r.K : r.V) + ring_row * row_bytes + off) = v;
  }
  if (lane == 0) {
    r.z[((size_t)b * window + slot) * hkv + kh] = z_new;
    if (r.u) r.u[((size_t)b * window + slot) * hkv + kh] = u_new;
  }
}

}  // namespace spkv
