// common.cuh -- small device helpers shared by the SP-KV kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/spkv.h"

namespace spkv {

constexpr int kPageRows = 64;

// ---- element types -----------------------------------------------------------

struct F32 {
  using T = float;
  static constexpr int kSize = 4;
};
struct BF16 {
  using T = __nv_bfloat16;
  static constexpr int kSize = 2;
};

// bf16 -> fp32 is exact: the bf16 bits are the high half of the fp32 bits.
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Widen one 16-byte vector to fp32: 8 elements for bf16, 4 for fp32.
template <typename E>
struct Vec;

template <>
struct Vec<BF16> {
  static constexpr int kElems = 8;
  __device__ __forceinline__ static void widen(const uint4& v, float* out) {
    out[0] = bf16lo(v.x); out[1] = bf16hi(v.x);
    out[2] = bf16lo(v.y); out[3] = bf16hi(v.y);
    out[4] = bf16lo(v.z); out[5] = bf16hi(v.z);
    out[6] = bf16lo(v.w); out[7] = bf16hi(v.w);
  }
};

template <>
struct Vec<F32> {
  static constexpr int kElems = 4;
  __device__ __forceinline__ static void widen(const uint4& v, float* out) {
    out[0] = __uint_as_float(v.x); out[1] = __uint_as_float(v.y);
    out[2] = __uint_as_float(v.z); out[3] = __uint_as_float(v.w);
  }
};

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ void from_f32(float x, float* dst) { *dst = x; }
__device__ __forceinline__ void from_f32(float x, __nv_bfloat16* dst) { *dst = __float2bfloat16_rn(x); }

// ---- packed fp32 arithmetic (sm_100 f32x2 pipe) -----------------------------------

__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  unsigned long long ra, rb, rc, rd;
  ra = *reinterpret_cast<unsigned long long*>(&a);
  rb = *reinterpret_cast<unsigned long long*>(&b);
  rc = *reinterpret_cast<unsigned long long*>(&c);
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(rd) : "l"(ra), "l"(rb), "l"(rc));
  return *reinterpret_cast<float2*>(&rd);
}

__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  unsigned long long ra, rb, rd;
  ra = *reinterpret_cast<unsigned long long*>(&a);
  rb = *reinterpret_cast<unsigned long long*>(&b);
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(rd) : "l"(ra), "l"(rb));
  return *reinterpret_cast<float2*>(&rd);
}

__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  unsigned long long ra, rb, rd;
  ra = *reinterpret_cast<unsigned long long*>(&a);
  rb = *reinterpret_cast<unsigned long long*>(&b);
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(rd) : "l"(ra), "l"(rb));
  return *reinterpret_cast<float2*>(&rd);
}

// ---- programmatic dependent launch ---------------------------------------------------
// Kernels launched with launch_pdl may start while the previous kernel on the stream
// is still running; each of them calls grid_dependency_wait() before it touches memory
// that the previous kernel writes (the wait returns once that grid has completed and
// its writes are visible).  grid_dependents_launch() lets the next such kernel start
// its own launch early.  Both are no-ops for a kernel launched the ordinary way.

__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

__device__ __forceinline__ void grid_dependents_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// ---- time and bounded waits ------------------------------------------------------------

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Every wait in these kernels gives up after this many nanoseconds, sets
// SPKV_FLAG_TIMEOUT and lets the kernel run to its end.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\t"
      "mbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\t"
      "mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(smem_u32(bar)),
      "r"(bytes)
      : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for phase `parity` of an mbarrier; returns false (and raises the flag)
// if the wait gave up.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint32_t* err_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_ns() - t0 > kWaitLimitNs) {
      if (err_flag) atomicOr(err_flag, SPKV_FLAG_TIMEOUT);
      return false;
    }
  }
  return true;
}

// 1-D bulk copy global -> shared, completion counted on an mbarrier (bytes and
// both addresses multiples of 16).
__device__ __forceinline__ void bulk_g2s(void* dst_smem, const void* src_gmem, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst_smem)),
      "l"(src_gmem), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ---- index checks of the debug build -----------------------------------------------------
// Built with SPKV_DEBUG, every page number read from a page table is checked against the
// pool (and query positions against 0) before it is used as an address: a failed check
// latches SPKV_FLAG_INDEX in err_flag and the access is skipped or redirected to page 0
// (the results are then wrong, and flagged).  Nothing traps.  Without SPKV_DEBUG the
// checks compile away.
#ifdef SPKV_DEBUG
constexpr bool kDebugChecks = true;
#else
constexpr bool kDebugChecks = false;
#endif

__device__ __forceinline__ bool page_ok(int page, int num_pages, uint32_t* err) {
  if constexpr (kDebugChecks) {
    if ((unsigned)page >= (unsigned)num_pages) {
      if (err) atomicOr(err, SPKV_FLAG_INDEX);
      return false;
    }
  }
  return true;
}

__device__ __forceinline__ int checked_position(int t, uint32_t* err) {
  if constexpr (kDebugChecks) {
    if (t < 0) {
      if (err) atomicOr(err, SPKV_FLAG_INDEX);
      return 0;
    }
  }
  return t;
}

// ---- cache addressing ------------------------------------------------------------------

struct CacheView {
  const char* K;
  const char* V;
  const int32_t* pos;
  const int32_t* page_table;
  const int32_t* count;
  int max_pages;
  int num_pages;
  uint32_t* err;
};

inline CacheView cache_view(const spkv_cache& c) {
  return CacheView{static_cast<const char*>(c.K_pool), static_cast<const char*>(c.V_pool),
                   c.pos_pool, c.page_table, c.count, c.max_pages_per_head, c.num_pages,
                   c.err_flag};
}

// Position of cache row i of head bh (debug build: a bad page reads as "beyond every
// limit").
__device__ __forceinline__ int cache_pos(const CacheView& c, int bh, int i) {
  const int page = __ldcg(c.page_table + (size_t)bh * c.max_pages + (i >> 6));
  if (!page_ok(page, c.num_pages, c.err)) return 0x7fffffff;
  return __ldcg(c.pos + (size_t)page * kPageRows + (i & 63));
}

// Number of cache rows of head bh whose position is <= limit (positions are
// increasing, so this is a binary search).  `tail` bounds how many rows can
// exceed the limit: in decode the cache holds no position beyond the query t, so
// at most `window` rows lie in (t - window, t]; prefill passes the row count.
__device__ __forceinline__ int cache_live_rows(const CacheView& c, int bh, int limit, int tail) {
  if (!c.count) return 0;  // no cache: a local (window-only) layer
  const int n = __ldcg(c.count + bh);
  if (n == 0) return 0;
  if (cache_pos(c, bh, n - 1) <= limit) return n;
  int lo = n - tail > 0 ? n - tail : 0;  // rows before lo are <= limit
  int hi = n - 1;                         // row hi is > limit
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (cache_pos(c, bh, mid) <= limit) lo = mid + 1; else hi = mid;
  }
  return lo;
}

}  // namespace spkv
