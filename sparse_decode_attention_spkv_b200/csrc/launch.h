// launch.h -- internal launchers behind the C ABI (host side).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/spkv.h"

namespace spkv {

cudaError_t launch_score(const spkv_params& p, const void* h, int n_tok, const void* W1,
                         const float* b1, const float* W2, const float* b2, float* u_out,
                         uint8_t* z_out, cudaStream_t stream);
bool score_supported(const spkv_params& p);
cudaError_t launch_score_append(const spkv_params& p, const spkv_cache& c, const spkv_ring& ring,
                                const int32_t* t_pos, const void* h, const void* W1,
                                const float* b1, const float* W2, const float* b2,
                                const void* k_new, const void* v_new, float* u_out,
                                uint8_t* z_out, bool settled, cudaStream_t stream);

cudaError_t launch_score_gates(const spkv_params& p, const spkv_ring& ring, const int32_t* t_pos,
                               const void* h, const void* W1, const float* b1, const float* W2,
                               const float* b2, float* u_out, uint8_t* z_out, cudaStream_t stream);

cudaError_t launch_write_compact(const spkv_params& p, const spkv_cache& c, const spkv_ring* ring,
                                 int src_kind, const void* K_src, const void* V_src,
                                 const uint8_t* z, const float* u, const int32_t* src_pos,
                                 int n_rows, int src_batch_rows, cudaStream_t stream);

cudaError_t launch_decode_append(const spkv_params& p, const spkv_cache& c, const spkv_ring& ring,
                                 const int32_t* t_pos, const void* k_new, const void* v_new,
                                 const uint8_t* z_new, const float* u_new, int retire,
                                 cudaStream_t stream);

cudaError_t launch_ring_write(const spkv_params& p, const spkv_ring& ring, const void* K_src,
                              const void* V_src, const uint8_t* z_src, const float* u_src,
                              int gated_from, const int32_t* src_pos, int n_rows,
                              int src_batch_rows, cudaStream_t stream);

// a1 on tcgen05 tensor cores for 128 tokens or more (bf16, hid 128).
bool score_tc_supported(const spkv_params& p, int n_tok);
cudaError_t launch_score_tc(const spkv_params& p, const void* h, int n_tok, const void* W1,
                            const float* b1, const float* W2, const float* b2, float* u_out,
                            uint8_t* z_out, cudaStream_t stream);

size_t decode_workspace_bytes(const spkv_params& p, int num_sms);
// Bytes of counters at the front of the decode workspace, for the kernel launch_decode
// picks for these parameters (the rest of the workspace needs no initialisation).
size_t decode_ctrl_bytes(const spkv_params& p);
size_t decode_tc_ctrl_bytes(const spkv_params& p);
bool decode_tc_supported(const spkv_params& p);
size_t decode_tc_workspace_bytes(const spkv_params& p, int num_sms);
// k_new / v_new given: before-append mode (the ring holds rows t-w .. t-1, the new row
// comes from k_new / v_new, row t - w counts if its gate in the ring is 1).
cudaError_t launch_decode_tc(const spkv_params& p, const spkv_cache& c, const spkv_ring& ring,
                             const void* q, const int32_t* t_pos, void* o, float* lse,
                             void* workspace, int num_sms, cudaStream_t stream,
                             const void* k_new = nullptr, const void* v_new = nullptr,
                             bool early_plan = false);
// Decode attention over one slice of a sequence's keys: the cache's rows with pos <=
// t - w and, with window_on, the window; fp32 o_part normalised over the slice and its
// lse (natural log), o = 0 and lse = -inf for a head without keys in the slice.
// ring.K_win may be NULL when window_on is false.
cudaError_t launch_decode_partial(const spkv_params& p, const spkv_cache& c, const spkv_ring& ring,
                                  const void* q, const int32_t* t_pos, bool window_on,
                                  float* o_part, float* lse_part, void* workspace, int num_sms,
                                  cudaStream_t stream);
// Log-sum-exp combination of n_parts slice partials into one output per query head.
cudaError_t launch_decode_merge_parts(const spkv_params& p, int n_parts, const float* o_parts,
                                      const float* lse_parts, void* o, float* lse,
                                      cudaStream_t stream);
cudaError_t launch_decode(const spkv_params& p, const spkv_cache& c, const spkv_ring& ring,
                          const void* q, const int32_t* t_pos, void* o, float* lse,
                          void* workspace, size_t ws_bytes, int num_sms, cudaStream_t stream);

bool prefill_tc_supported(const spkv_params& p, const spkv_cache& c, int chunk_start, int chunk_len);
cudaError_t launch_prefill_tc(const spkv_params& p, const spkv_cache& c, const spkv_ring& ring,
                              const void* q, const void* K_chunk, const void* V_chunk,
                              int chunk_start, int chunk_len, void* o, float* lse, int* sched,
                              cudaStream_t stream);
size_t rethreshold_workspace_bytes(const spkv_params& p, const spkv_cache& c);
// Limit of the re-threshold move kernel's waits on page-read flags (0: default).
void set_flag_wait_ns(unsigned long long ns);
cudaError_t launch_rethreshold(const spkv_params& p, const spkv_cache& c, const spkv_ring* ring,
                               float tau_new, void* workspace, int num_sms, cudaStream_t stream);

cudaError_t launch_prefill(const spkv_params& p, const spkv_cache& c, const spkv_ring& ring,
                           const void* q, const void* K_chunk, const void* V_chunk,
                           int chunk_start, int chunk_len, void* o, float* lse, int* sched,
                           cudaStream_t stream);

bool soft_tc_supported(const spkv_params& p, int seq_len);
cudaError_t launch_soft_tc(const spkv_params& p, const void* q, const void* K, const void* V,
                           const float* bias, int seq_len, void* o, float* lse, uint32_t* err,
                           cudaStream_t stream);
size_t soft_workspace_bytes(const spkv_params& p, int seq_len);
cudaError_t launch_soft(const spkv_params& p, const void* q, const void* K, const void* V,
                        const float* u, int seq_len, float beta, float c, void* o, float* lse,
                        void* workspace, uint32_t* err, cudaStream_t stream);

}  // namespace spkv
