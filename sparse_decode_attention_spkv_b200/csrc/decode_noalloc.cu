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
#include "host.h"
#include "launch.h"
#include "trace.h"

namespace {

// Fixed scratch of the no-allocation decode.  Every GPU that loads the library keeps
// this much device memory until the process exits.
constexpr size_t kNoAllocScratchBytes = (size_t)SPKV_NOALLOC_SCRATCH_BYTES;
__device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

constexpr int kMaxContexts = 64;
std::mutex g_mu;
struct ScratchRef {
  unsigned long long ctx;  // context the address belongs to (0: slot unused)
  void* ptr;
};
ScratchRef g_scratch[kMaxContexts] = {};

// Device address of the scratch in the current context.  The array's host-side name is
// not a device address; its address is looked up once per context (set-up of the first
// call in that context) and kept with the context's identifier, so a context created
// after a device reset (where the module is loaded anew) looks it up again.
cudaError_t scratch_for_current_context(void** ptr) {
  unsigned long long ctx = 0;
  cudaError_t e = spkv::current_context_id(&ctx);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_mu);
  for (const ScratchRef& r : g_scratch)
    if (r.ctx == ctx) {
      *ptr = r.ptr;
      return cudaSuccess;
    }
  void* p = nullptr;
  e = cudaGetSymbolAddress(&p, g_decode_scratch);
  if (e != cudaSuccess) return e;
  // remember it (a full table is reused from the front: a stale entry only costs a lookup)
  static int next = 0;
  g_scratch[next] = ScratchRef{ctx, p};
  next = (next + 1) % kMaxContexts;
  *ptr = p;
  return cudaSuccess;
}

}  // namespace

extern "C" int spkv_decode_attn_noalloc(const spkv_params* p, const spkv_cache* c,
                                        const spkv_ring* ring, const void* q,
                                        const int32_t* t_pos, void* o, float* lse,
                                        spkv_stream_t stream) {
  SPKV_TRACE("spkv_decode_attn_noalloc");
  // the same argument rules as spkv_decode_attn (cache NULL: a window-only layer)
  if (!spkv::params_ok(p) || (c && !spkv::cache_ok(c)) || !spkv::ring_ok(ring)) return SPKV_ERR_ARG;
  if (!q || !t_pos || !o || !spkv::aligned16(q) || !spkv::aligned16(o)) return SPKV_ERR_ARG;
  if ((size_t)p->B * p->Hkv > 2048) return SPKV_ERR_UNSUPPORTED;
  const int sms = spkv::sm_count();
  if (sms <= 0) return SPKV_ERR_CUDA;
  const size_t need = spkv::decode_workspace_bytes(*p, sms);
  if (need > kNoAllocScratchBytes) return SPKV_ERR_UNSUPPORTED;  // beyond the fixed scratch
  void* scratch = nullptr;
  if (scratch_for_current_context(&scratch) != cudaSuccess) return SPKV_ERR_CUDA;
  // The array is shared by calls of every shape, and the counters a call needs at zero
  // sit at shape-dependent offsets that another shape's call may have filled with plan
  // words (or that an aborted call left set): clear the control region of the kernel
  // that will run, on the stream, before it.
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(scratch, 0, spkv::decode_ctrl_bytes(*p), s) != cudaSuccess) return SPKV_ERR_CUDA;
  const cudaError_t e = spkv::launch_decode(*p, spkv::cache_or_none(c), *ring, q, t_pos, o, lse,
                                            scratch, kNoAllocScratchBytes, sms, s);
  return e == cudaSuccess ? SPKV_OK : SPKV_ERR_CUDA;
}
