// host.h -- host-side helpers shared by the entry points: argument validation (no CUDA
// call, so argument errors are reported without a GPU), the SM count of the current
// device, and per-context kernel set-up.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/spkv.h"

namespace spkv {

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline bool params_ok(const spkv_params* p) {
  if (!p) return false;
  if (p->B < 1 || p->Hkv < 1 || p->Hq < p->Hkv || p->Hq % p->Hkv) return false;
  const int G = p->Hq / p->Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return false;
  if (p->head_dim != 64 && p->head_dim != 128) return false;
  if (p->window < 1 || p->window > 1024) return false;
  if (p->dtype != SPKV_F32 && p->dtype != SPKV_BF16) return false;
  if (!(p->tau == p->tau)) return false;  // NaN threshold
  return true;
}

inline bool cache_ok(const spkv_cache* c) {
  if (!c) return false;
  if (!c->K_pool || !c->V_pool || !c->pos_pool || !c->page_table || !c->count ||
      !c->count_prev || !c->pool_top || !c->err_flag)
    return false;
  if (c->page_rows != 64 || c->num_pages < 1 || c->max_pages_per_head < 1) return false;
  if (!aligned16(c->K_pool) || !aligned16(c->V_pool)) return false;
  return true;
}

inline bool ring_ok(const spkv_ring* r) {
  return r && r->K_win && r->V_win && r->z_win && aligned16(r->K_win) && aligned16(r->V_win);
}

// A layer without a persistent cache (window-only, e.g. the local layers of a hybrid
// local/global stack) passes cache == NULL; the kernels see an all-zero cache.
inline const spkv_cache& cache_or_none(const spkv_cache* c) {
  static const spkv_cache none = {};
  return c ? *c : none;
}

// Multiprocessors of the current device (cached per device), or -1 on error.
int sm_count();

// A 64-bit identifier of the CUDA context current on this thread, unique for the life
// of the process (a context created after a device reset gets a new one); the primary
// context of the current device is initialised if no context is current yet.
cudaError_t current_context_id(unsigned long long* id);

// Raises the dynamic shared-memory limit of kernel `fn` to `bytes` in the current
// context, once per (context, kernel): a kernel attribute belongs to the context it
// was set in, so a second device, or a context rebuilt after a reset, is set up anew.
cudaError_t ensure_dynamic_smem(const void* fn, int bytes);

}  // namespace spkv
