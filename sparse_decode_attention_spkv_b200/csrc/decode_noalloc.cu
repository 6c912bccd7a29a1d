// decode_noalloc.cu -- gated decode attention for callers that cannot allocate.
//
// spkv_decode_attn needs a caller-provided workspace for its split-K partials and
// arrival counters.  Some callers cannot make that allocation: code that runs where
// cudaMalloc is unavailable or forbidden (a plugin inside a host that owns all device
// memory through its own pool, a path that must not allocate after start-up, a
// runtime that has no allocator hook to lend).  This entry point runs the same
// kernels with the scratch taken from a fixed array that lives in the library's
// device image instead.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "../../include/spkv.h"
#include "common.cuh"
#include "launch.h"
#include "trace.h"

namespace {

// Fixed scratch of the no-allocation decode.  Every GPU that loads the library keeps
// this much device memory until the process exits.
constexpr size_t kNoAllocScratchBytes = (size_t)SPKV_NOALLOC_SCRATCH_BYTES;
__device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};
int g_sms[kMaxDevices] = {};

// Device address of the scratch on the current device; looked up once per device
// (the array's host-side name is not a device address).
cudaError_t scratch_for_current_device(void** ptr, int* sms) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess) return e;
    int n = 0;
    e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
    g_sms[dev] = n;
  }
  *ptr = g_scratch_ptr[dev];
  *sms = g_sms[dev];
  return cudaSuccess;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" int spkv_decode_attn_noalloc(const spkv_params* p, const spkv_cache* c,
                                        const spkv_ring* ring, const void* q,
                                        const int32_t* t_pos, void* o, float* lse,
                                        spkv_stream_t stream) {
  SPKV_TRACE("spkv_decode_attn_noalloc");
  if (!p || !c || !ring || !q || !t_pos || !o) return SPKV_ERR_ARG;
  if (!c->K_pool || !c->V_pool || !c->pos_pool || !c->page_table || !c->count || !c->err_flag ||
      c->page_rows != spkv::kPageRows || !ring->K_win || !ring->V_win || !ring->z_win)
    return SPKV_ERR_ARG;
  if (!aligned16(q) || !aligned16(o) || !aligned16(c->K_pool) || !aligned16(c->V_pool) ||
      !aligned16(ring->K_win) || !aligned16(ring->V_win))
    return SPKV_ERR_ARG;
  if (p->B < 1 || p->Hkv < 1 || p->Hq % p->Hkv || p->window < 1 || p->window > 1024 ||
      (p->head_dim != 64 && p->head_dim != 128) || (p->dtype != SPKV_F32 && p->dtype != SPKV_BF16))
    return SPKV_ERR_ARG;
  const int G = p->Hq / p->Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return SPKV_ERR_ARG;
  if ((size_t)p->B * p->Hkv > 2048) return SPKV_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  int sms = 0;
  if (scratch_for_current_device(&scratch, &sms) != cudaSuccess) return SPKV_ERR_CUDA;
  const size_t need = spkv::decode_workspace_bytes(*p, sms);
  if (need > kNoAllocScratchBytes) return SPKV_ERR_UNSUPPORTED;  // beyond the fixed scratch
  // the arrival and work counters at the front of the scratch must start at zero
  const size_t ctrl = (((size_t)p->B * p->Hkv + 2) * 4 + 255) / 256 * 256;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(scratch, 0, ctrl, s) != cudaSuccess) return SPKV_ERR_CUDA;
  const cudaError_t e =
      spkv::launch_decode(*p, *c, *ring, q, t_pos, o, lse, scratch, kNoAllocScratchBytes, sms, s);
  return e == cudaSuccess ? SPKV_OK : SPKV_ERR_CUDA;
}
