// api.cu -- the C ABI (include/spkv.h): host-side validation, then launches.
// Validation touches no CUDA API, so argument errors are reported without a GPU.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "../../include/spkv.h"
#include "common.cuh"
#include "host.h"
#include "launch.h"
#include "trace.h"

namespace {

using spkv::aligned16;
using spkv::cache_or_none;
using spkv::params_ok;
using spkv::ring_ok;
using spkv::sm_count;

int status_of(cudaError_t e) { return e == cudaSuccess ? SPKV_OK : SPKV_ERR_CUDA; }

bool cache_ok(const spkv_params* p, const spkv_cache* c) {
  (void)p;
  return spkv::cache_ok(c);
}

}  // namespace

extern "C" {

const char* spkv_status_str(int status) {
  switch (status) {
    case SPKV_OK: return "ok";
    case SPKV_ERR_ARG: return "invalid argument";
    case SPKV_ERR_CAPACITY: return "cache capacity exhausted";
    case SPKV_ERR_CUDA: return "CUDA error";
    case SPKV_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case SPKV_ERR_TIMEOUT: return "device wait timed out";
    case SPKV_ERR_INDEX: return "device index check failed";
  }
  return "unknown status";
}

int spkv_version(void) { return 300; }

int spkv_cache_reset(const spkv_params* p, const spkv_cache* c, const spkv_ring* ring,
                     spkv_stream_t stream) {
  SPKV_TRACE("spkv_cache_reset");
  if (!params_ok(p) || !cache_ok(p, c)) return SPKV_ERR_ARG;
  if (ring && !ring_ok(ring)) return SPKV_ERR_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t heads = (size_t)p->B * p->Hkv;
  cudaError_t e = cudaMemsetAsync(c->page_table, 0xff, heads * c->max_pages_per_head * 4, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(c->count, 0, heads * 4, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(c->count_prev, 0, heads * 4, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(c->pool_top, 0, 4, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(c->err_flag, 0, 4, s);
  if (e == cudaSuccess && ring) e = cudaMemsetAsync(ring->z_win, 0, (size_t)p->B * p->window * p->Hkv, s);
  if (e == cudaSuccess && ring && ring->u_win)  // NaN: no pending utility
    e = cudaMemsetAsync(ring->u_win, 0xff, (size_t)p->B * p->window * p->Hkv * 4, s);
  return status_of(e);
}

int spkv_cache_check(const spkv_cache* c, spkv_stream_t stream, uint32_t* flags_out) {
  SPKV_TRACE("spkv_cache_check");
  if (!c || !c->err_flag) return SPKV_ERR_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t flags = 0;
  cudaError_t e = cudaMemcpyAsync(&flags, c->err_flag, 4, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return SPKV_ERR_CUDA;
  if (flags_out) *flags_out = flags;
  if (flags & (SPKV_FLAG_POOL_FULL | SPKV_FLAG_TABLE_FULL)) return SPKV_ERR_CAPACITY;
  if (flags & SPKV_FLAG_TIMEOUT) return SPKV_ERR_TIMEOUT;
  if (flags & SPKV_FLAG_INDEX) return SPKV_ERR_INDEX;
  return SPKV_OK;
}

int spkv_score(const spkv_params* p, const void* h, int n_tok, const void* W1, const float* b1,
               const float* W2, const float* b2, float* u_out, uint8_t* z_out,
               spkv_stream_t stream) {
  SPKV_TRACE("spkv_score");
  if (!params_ok(p) || n_tok < 0) return SPKV_ERR_ARG;
  if (p->d_model < 1 || p->hid < 1) return SPKV_ERR_ARG;
  if (n_tok == 0) return SPKV_OK;
  if (!h || !W1 || !b1 || !W2 || !b2 || !z_out) return SPKV_ERR_ARG;
  if (!aligned16(h) || !aligned16(W1)) return SPKV_ERR_ARG;  // 16-byte vector and TMA loads
  if (!spkv::score_supported(*p)) return SPKV_ERR_UNSUPPORTED;
  return status_of(spkv::launch_score(*p, h, n_tok, W1, b1, W2, b2, u_out, z_out,
                                      static_cast<cudaStream_t>(stream)));
}

int spkv_write_compact(const spkv_params* p, const spkv_cache* c, const spkv_ring* ring,
                       int src_kind, const void* K_src, const void* V_src, const uint8_t* z,
                       const float* u, const int32_t* src_pos, int n_rows, int src_batch_rows,
                       spkv_stream_t stream) {
  SPKV_TRACE("spkv_write_compact");
  if (!params_ok(p) || !cache_ok(p, c) || n_rows < 0 || src_batch_rows < n_rows) return SPKV_ERR_ARG;
  if (n_rows == 0) return SPKV_OK;
  if (!z || !src_pos) return SPKV_ERR_ARG;
  if (c->u_pool && !u) return SPKV_ERR_ARG;
  if (src_kind == SPKV_SRC_CHUNK) {
    if (!K_src || !V_src || !aligned16(K_src) || !aligned16(V_src)) return SPKV_ERR_ARG;
  } else if (src_kind == SPKV_SRC_RING) {
    if (!ring_ok(ring) || n_rows > p->window) return SPKV_ERR_ARG;
  } else {
    return SPKV_ERR_ARG;
  }
  return status_of(spkv::launch_write_compact(*p, *c, ring, src_kind, K_src, V_src, z, u, src_pos,
                                              n_rows, src_batch_rows,
                                              static_cast<cudaStream_t>(stream)));
}

int spkv_decode_append(const spkv_params* p, const spkv_cache* c, const spkv_ring* ring,
                       const int32_t* t_pos, const void* k_new, const void* v_new,
                       const uint8_t* z_new, const float* u_new, int retire,
                       spkv_stream_t stream) {
  SPKV_TRACE("spkv_decode_append");
  if (!params_ok(p) || (c && !cache_ok(p, c)) || !ring_ok(ring)) return SPKV_ERR_ARG;
  if (!c && retire) return SPKV_ERR_ARG;  // nowhere to retire into
  if (!t_pos || !k_new || !v_new || !aligned16(k_new) || !aligned16(v_new)) return SPKV_ERR_ARG;
  if (ring->u_win && z_new && !u_new) return SPKV_ERR_ARG;
  return status_of(spkv::launch_decode_append(*p, cache_or_none(c), *ring, t_pos, k_new, v_new, z_new, u_new, retire,
                                              static_cast<cudaStream_t>(stream)));
}

int spkv_decode_score_append(const spkv_params* p, const spkv_cache* c, const spkv_ring* ring,
                             const int32_t* t_pos, const void* h, const void* W1, const float* b1,
                             const float* W2, const float* b2, const void* k_new,
                             const void* v_new, float* u_out, uint8_t* z_out, unsigned flags,
                             spkv_stream_t stream) {
  SPKV_TRACE("spkv_decode_score_append");
  if (flags & ~SPKV_INPUTS_SETTLED) return SPKV_ERR_ARG;
  if (!params_ok(p) || !cache_ok(p, c) || !ring_ok(ring)) return SPKV_ERR_ARG;
  if (p->d_model < 1 || p->hid < 1) return SPKV_ERR_ARG;
  if (!t_pos || !h || !W1 || !b1 || !W2 || !b2 || !k_new || !v_new || !z_out) return SPKV_ERR_ARG;
  if (!aligned16(h) || !aligned16(W1) || !aligned16(k_new) || !aligned16(v_new)) return SPKV_ERR_ARG;
  if (ring->u_win && !u_out) return SPKV_ERR_ARG;
  if (!spkv::score_supported(*p)) return SPKV_ERR_UNSUPPORTED;
  return status_of(spkv::launch_score_append(*p, *c, *ring, t_pos, h, W1, b1, W2, b2, k_new, v_new,
                                             u_out, z_out, (flags & SPKV_INPUTS_SETTLED) != 0,
                                             static_cast<cudaStream_t>(stream)));
}

int spkv_decode_score(const spkv_params* p, const spkv_ring* ring, const int32_t* t_pos,
                      const void* h, const void* W1, const float* b1, const float* W2,
                      const float* b2, float* u_out, uint8_t* z_out, spkv_stream_t stream) {
  SPKV_TRACE("spkv_decode_score");
  if (!params_ok(p) || !ring_ok(ring)) return SPKV_ERR_ARG;
  if (p->d_model < 1 || p->hid < 1) return SPKV_ERR_ARG;
  if (!t_pos || !h || !W1 || !b1 || !W2 || !b2 || !z_out) return SPKV_ERR_ARG;
  if (!aligned16(h) || !aligned16(W1)) return SPKV_ERR_ARG;
  if (ring->u_win && !u_out) return SPKV_ERR_ARG;
  if (!spkv::score_supported(*p)) return SPKV_ERR_UNSUPPORTED;
  return status_of(spkv::launch_score_gates(*p, *ring, t_pos, h, W1, b1, W2, b2, u_out, z_out,
                                            static_cast<cudaStream_t>(stream)));
}

int spkv_ring_write(const spkv_params* p, const spkv_ring* ring, const void* K_src,
                    const void* V_src, const uint8_t* z_src, const float* u_src, int gated_from,
                    const int32_t* src_pos, int n_rows, int src_batch_rows, spkv_stream_t stream) {
  SPKV_TRACE("spkv_ring_write");
  if (!params_ok(p) || !ring_ok(ring) || n_rows < 0 || src_batch_rows < n_rows) return SPKV_ERR_ARG;
  if (n_rows == 0) return SPKV_OK;
  if (!K_src || !V_src || !src_pos || !aligned16(K_src) || !aligned16(V_src)) return SPKV_ERR_ARG;
  if (gated_from < 0) return SPKV_ERR_ARG;
  if (!z_src && gated_from < n_rows) return SPKV_ERR_ARG;
  if (ring->u_win && !u_src && gated_from < n_rows) return SPKV_ERR_ARG;
  return status_of(spkv::launch_ring_write(*p, *ring, K_src, V_src, z_src, u_src, gated_from, src_pos,
                                           n_rows, src_batch_rows,
                                           static_cast<cudaStream_t>(stream)));
}

size_t spkv_decode_workspace_bytes(const spkv_params* p, const spkv_cache* c) {
  (void)c;
  if (!params_ok(p)) return 0;
  const int sms = sm_count();
  if (sms <= 0) return 0;
  return spkv::decode_workspace_bytes(*p, sms);
}

int spkv_decode_attn(const spkv_params* p, const spkv_cache* c, const spkv_ring* ring,
                     const void* q, const int32_t* t_pos, void* o, float* lse, void* workspace,
                     size_t ws_bytes, spkv_stream_t stream) {
  SPKV_TRACE("spkv_decode_attn");
  if (!params_ok(p) || (c && !cache_ok(p, c)) || !ring_ok(ring)) return SPKV_ERR_ARG;
  if (!q || !t_pos || !o || !workspace || !aligned16(q) || !aligned16(o)) return SPKV_ERR_ARG;
  if ((size_t)p->B * p->Hkv > 2048) return SPKV_ERR_UNSUPPORTED;
  const int sms = sm_count();
  if (sms <= 0) return SPKV_ERR_CUDA;
  if (ws_bytes < spkv::decode_workspace_bytes(*p, sms)) return SPKV_ERR_ARG;
  return status_of(spkv::launch_decode(*p, cache_or_none(c), *ring, q, t_pos, o, lse, workspace, ws_bytes, sms,
                                       static_cast<cudaStream_t>(stream)));
}

int spkv_decode_attn_before_append_supported(const spkv_params* p) {
  return params_ok(p) && spkv::decode_tc_supported(*p) ? 1 : 0;
}

int spkv_decode_attn_before_append(const spkv_params* p, const spkv_cache* c,
                                   const spkv_ring* ring, const void* q, const int32_t* t_pos,
                                   const void* k_new, const void* v_new, void* o, float* lse,
                                   void* workspace, size_t ws_bytes, unsigned flags,
                                   spkv_stream_t stream) {
  SPKV_TRACE("spkv_decode_attn_before_append");
  if (!params_ok(p) || (c && !cache_ok(p, c)) || !ring_ok(ring)) return SPKV_ERR_ARG;
  if (flags & ~SPKV_DECODE_STATE_SETTLED) return SPKV_ERR_ARG;
  if (!q || !t_pos || !o || !workspace || !aligned16(q) || !aligned16(o)) return SPKV_ERR_ARG;
  if (!k_new || !v_new || !aligned16(k_new) || !aligned16(v_new)) return SPKV_ERR_ARG;
  if ((size_t)p->B * p->Hkv > 2048) return SPKV_ERR_UNSUPPORTED;
  if (!spkv::decode_tc_supported(*p)) return SPKV_ERR_UNSUPPORTED;
  const int sms = sm_count();
  if (sms <= 0) return SPKV_ERR_CUDA;
  if (ws_bytes < spkv::decode_workspace_bytes(*p, sms)) return SPKV_ERR_ARG;
  return status_of(spkv::launch_decode_tc(*p, cache_or_none(c), *ring, q, t_pos, o, lse, workspace,
                                          sms, static_cast<cudaStream_t>(stream), k_new, v_new,
                                          (flags & SPKV_DECODE_STATE_SETTLED) != 0));
}

int spkv_decode_attn_partial(const spkv_params* p, const spkv_cache* c, const spkv_ring* ring,
                             const void* q, const int32_t* t_pos, unsigned flags, float* o_part,
                             float* lse_part, void* workspace, size_t ws_bytes,
                             spkv_stream_t stream) {
  SPKV_TRACE("spkv_decode_attn_partial");
  if (!params_ok(p) || (flags & ~SPKV_SLICE_WINDOW)) return SPKV_ERR_ARG;
  const bool window_on = (flags & SPKV_SLICE_WINDOW) != 0;
  if (c && !cache_ok(p, c)) return SPKV_ERR_ARG;
  if (window_on ? !ring_ok(ring) : !c) return SPKV_ERR_ARG;  // a slice holds something
  if (!q || !t_pos || !o_part || !lse_part || !workspace) return SPKV_ERR_ARG;
  if (!aligned16(q) || !aligned16(o_part)) return SPKV_ERR_ARG;
  if ((size_t)p->B * p->Hkv > 2048) return SPKV_ERR_UNSUPPORTED;
  if (!spkv::decode_tc_supported(*p)) return SPKV_ERR_UNSUPPORTED;
  const int sms = sm_count();
  if (sms <= 0) return SPKV_ERR_CUDA;
  if (ws_bytes < spkv::decode_workspace_bytes(*p, sms)) return SPKV_ERR_ARG;
  static const spkv_ring no_ring = {};
  return status_of(spkv::launch_decode_partial(*p, cache_or_none(c), window_on ? *ring : no_ring,
                                               q, t_pos, window_on, o_part, lse_part, workspace,
                                               sms, static_cast<cudaStream_t>(stream)));
}

int spkv_decode_attn_partial_supported(const spkv_params* p) {
  return params_ok(p) && spkv::decode_tc_supported(*p) ? 1 : 0;
}

int spkv_decode_merge(const spkv_params* p, int n_parts, const float* o_parts,
                      const float* lse_parts, void* o, float* lse, spkv_stream_t stream) {
  SPKV_TRACE("spkv_decode_merge");
  if (!params_ok(p) || n_parts < 1) return SPKV_ERR_ARG;
  if (!o_parts || !lse_parts || !o) return SPKV_ERR_ARG;
  if (!aligned16(o_parts) || !aligned16(o)) return SPKV_ERR_ARG;
  return status_of(spkv::launch_decode_merge_parts(*p, n_parts, o_parts, lse_parts, o, lse,
                                                   static_cast<cudaStream_t>(stream)));
}

size_t spkv_rethreshold_workspace_bytes(const spkv_params* p, const spkv_cache* c) {
  if (!params_ok(p) || !cache_ok(p, c)) return 0;
  return spkv::rethreshold_workspace_bytes(*p, *c);
}

int spkv_cache_rethreshold(const spkv_params* p, const spkv_cache* c, const spkv_ring* ring,
                           float tau_new, void* workspace, size_t ws_bytes,
                           spkv_stream_t stream) {
  SPKV_TRACE("spkv_cache_rethreshold");
  if (!params_ok(p) || !cache_ok(p, c) || !c->u_pool) return SPKV_ERR_ARG;
  if (ring && !ring_ok(ring)) return SPKV_ERR_ARG;
  if (!(tau_new == tau_new) || !workspace) return SPKV_ERR_ARG;
  if ((size_t)p->B * p->Hkv > 2048) return SPKV_ERR_UNSUPPORTED;
  if (ws_bytes < spkv::rethreshold_workspace_bytes(*p, *c)) return SPKV_ERR_ARG;
  const int sms = sm_count();
  if (sms <= 0) return SPKV_ERR_CUDA;
  return status_of(spkv::launch_rethreshold(*p, *c, ring, tau_new, workspace, sms,
                                            static_cast<cudaStream_t>(stream)));
}

int spkv_debug_set_flag_wait_ns(unsigned long long ns) {
  spkv::set_flag_wait_ns(ns);
  return SPKV_OK;
}

size_t spkv_soft_attn_workspace_bytes(const spkv_params* p, int seq_len) {
  if (!params_ok(p) || seq_len < 0) return 0;
  return spkv::soft_workspace_bytes(*p, seq_len);
}

int spkv_soft_attn(const spkv_params* p, const void* q, const void* K, const void* V,
                   const float* u, int seq_len, float beta, float c, void* o, float* lse,
                   void* workspace, size_t ws_bytes, uint32_t* err_flag, spkv_stream_t stream) {
  SPKV_TRACE("spkv_soft_attn");
  if (!params_ok(p) || seq_len < 0) return SPKV_ERR_ARG;
  if (!(beta > 0.f) || !(c >= 0.f) || !(c < INFINITY)) return SPKV_ERR_ARG;
  if (seq_len == 0) return SPKV_OK;
  if (!q || !K || !V || !u || !o || !workspace) return SPKV_ERR_ARG;
  if (!aligned16(q) || !aligned16(K) || !aligned16(V) || !aligned16(o) || !aligned16(workspace))
    return SPKV_ERR_ARG;
  if (ws_bytes < spkv::soft_workspace_bytes(*p, seq_len)) return SPKV_ERR_ARG;
  return status_of(spkv::launch_soft(*p, q, K, V, u, seq_len, beta, c, o, lse, workspace, err_flag,
                                     static_cast<cudaStream_t>(stream)));
}

int spkv_prefill_attn(const spkv_params* p, const spkv_cache* c, const spkv_ring* ring,
                      const void* q, const void* K_chunk, const void* V_chunk, int chunk_start,
                      int chunk_len, void* o, float* lse, void* workspace, size_t ws_bytes,
                      spkv_stream_t stream) {
  SPKV_TRACE("spkv_prefill_attn");
  if (!params_ok(p) || (c && !cache_ok(p, c)) || !ring_ok(ring)) return SPKV_ERR_ARG;
  if (chunk_start < 0 || chunk_len < 0) return SPKV_ERR_ARG;
  if (chunk_len == 0) return SPKV_OK;
  if (!q || !K_chunk || !V_chunk || !o) return SPKV_ERR_ARG;
  if (!aligned16(q) || !aligned16(K_chunk) || !aligned16(V_chunk) || !aligned16(o)) return SPKV_ERR_ARG;
  if (workspace && (!aligned16(workspace) || ws_bytes < SPKV_PREFILL_WORKSPACE_BYTES)) return SPKV_ERR_ARG;
  return status_of(spkv::launch_prefill(*p, cache_or_none(c), *ring, q, K_chunk, V_chunk, chunk_start,
                                        chunk_len, o, lse, static_cast<int*>(workspace),
                                        static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
