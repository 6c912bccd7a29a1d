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
  int num_pages;
  int max_pages;
};

inline CacheMut cache_mut(const spkv_cache& c) {
  return CacheMut{static_cast<char*>(c.K_pool), static_cast<char*>(c.V_pool), c.pos_pool,
                  c.page_table, c.count, c.count_prev, c.pool_top, c.err_flag, c.num_pages,
                  c.max_pages_per_head};
}

struct RingMut {
  char* K;
  char* V;
  uint8_t* z;
};

// Whole warp, head bh = b * hkv + kh, query position t >= 0: retire s = t - window
// (appended to the cache when `retire` and its stored gate is 1), then store the
// new token's k/v rows and gate in slot t % window.
__device__ __forceinline__ void decode_append_warp(const CacheMut& c, const RingMut& r, int bh,
                                                   int b, int kh, int t, const char* k_new,
                                                   const char* v_new, uint8_t z_new, int retire,
                                                   int hkv, int window, int row_bytes, int lane) {
  const int slot = t % window;
  const int s = t - window;
  const int lpr = row_bytes >> 4;
  const size_t ring_row = (size_t)bh * window + slot;
  uint8_t* zslot = r.z + ((size_t)b * window + slot) * hkv + kh;
  if (retire && s >= 0 && *zslot) {
    const int i = c.count[bh];
    int page = -1;
    if ((i & 63) == 0) {
      if (lane == 0) {
        if ((i >> 6) >= c.max_pages) {
          atomicOr(c.err, SPKV_FLAG_TABLE_FULL);
        } else {
          const int pg = atomicAdd(c.pool_top, 1);
          if (pg >= c.num_pages) {
            atomicOr(c.err, SPKV_FLAG_POOL_FULL);
          } else {
            page = pg;
            c.page_table[(size_t)bh * c.max_pages + (i >> 6)] = pg;
          }
        }
      }
      page = __shfl_sync(0xffffffffu, page, 0);
    } else {
      page = c.page_table[(size_t)bh * c.max_pages + (i >> 6)];
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
  if (lane == 0) *zslot = z_new;
}

}  // namespace spkv
