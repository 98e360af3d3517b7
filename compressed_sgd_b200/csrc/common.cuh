// Internal helpers shared by the gsparse kernels (not part of the C ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "gsparse.h"

namespace gs {

constexpr int kWarp = 32;
constexpr uint32_t kFull = 0xffffffffu;

// Device error word: kernels OR bits in; a null pointer drops them.
__device__ __forceinline__ void raise(int32_t* st, int32_t bit) {
  if (st) atomicOr(st, bit);
}

__host__ __device__ __forceinline__ int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }
__host__ __device__ __forceinline__ int64_t round_up(int64_t a, int64_t b) { return cdiv(a, b) * b; }

// Magnitude order key: fp32 bits with the sign cleared (larger key = larger |x| for finite x).
__device__ __forceinline__ uint32_t mag_key(float x) { return __float_as_uint(x) & 0x7fffffffu; }

// ceil(n_s * num / den) clamped to [0, n_s], exact.
__host__ __device__ __forceinline__ int64_t kept_count(int64_t n_s, int64_t num, int64_t den) {
  if (n_s <= 0 || num <= 0) return 0;
  unsigned __int128 p = (unsigned __int128)n_s * (unsigned __int128)num;
  unsigned __int128 k = (p + (unsigned __int128)(den - 1)) / (unsigned __int128)den;
  return k > (unsigned __int128)n_s ? n_s : (int64_t)k;
}

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Exclusive warp prefix sum of small non-negative counts (< 8) via bit-plane ballots.
// Returns the prefix; *total receives the warp total.
__device__ __forceinline__ uint32_t warp_prefix_small(uint32_t c, uint32_t* total) {
  const uint32_t b0 = __ballot_sync(kFull, c & 1u);
  const uint32_t b1 = __ballot_sync(kFull, c & 2u);
  const uint32_t b2 = __ballot_sync(kFull, c & 4u);
  const uint32_t lt = lanemask_lt();
  *total = __popc(b0) + 2u * __popc(b1) + 4u * __popc(b2);
  return __popc(b0 & lt) + 2u * __popc(b1 & lt) + 4u * __popc(b2 & lt);
}

// Inclusive warp scan (any values).
template <class T>
__device__ __forceinline__ T warp_inclusive_scan(T v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    T o = __shfl_up_sync(kFull, v, d);
    if (lane >= d) v += o;
  }
  return v;
}

template <class T>
__device__ __forceinline__ T warp_sum(T v) {
#pragma unroll
  for (int d = 16; d > 0; d >>= 1) v += __shfl_xor_sync(kFull, v, d);
  return v;
}

// Block-wide exclusive scan of one int64 per thread (blockDim.x multiple of 32, <= 1024).
// `sh` must hold 33 int64. Returns the exclusive prefix; *total gets the block total.
__device__ __forceinline__ int64_t block_exclusive_scan(int64_t v, int64_t* sh, int64_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int64_t inc = warp_inclusive_scan(v);
  if (lane == 31) sh[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    int64_t w = lane < nw ? sh[lane] : 0;
    int64_t wi = warp_inclusive_scan(w);
    if (lane < nw) sh[lane] = wi - w;
    if (lane == nw - 1) sh[32] = wi;
  }
  __syncthreads();
  int64_t ex = inc - v + sh[warp];
  *total = sh[32];
  __syncthreads();
  return ex;
}

// Streaming 128-bit accesses: the data is touched once, so keep it out of L1 and mark it
// evict-first in L2.
__device__ __forceinline__ float4 ld_stream(const float* p) {
  return __ldcs(reinterpret_cast<const float4*>(p));
}
__device__ __forceinline__ void st_stream(float* p, float4 v) {
  __stcs(reinterpret_cast<float4*>(p), v);
}

// Brings the 128-byte line holding p into L2 (a hint: nothing waits for it).
__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(__cvta_generic_to_global(p)));
}

// Upper bound search: number of entries of a[0..len) that are <= x (a ascending).
__device__ __forceinline__ int64_t upper_bound_i64(const int64_t* a, int64_t len, int64_t x) {
  int64_t lo = 0, hi = len;
  while (lo < hi) {
    int64_t mid = (lo + hi) >> 1;
    if (a[mid] <= x) lo = mid + 1; else hi = mid;
  }
  return lo;
}

// Lower bound over int32: first position with a[pos] >= x.
__device__ __forceinline__ int64_t lower_bound_i32(const int32_t* a, int64_t len, int64_t x) {
  int64_t lo = 0, hi = len;
  while (lo < hi) {
    int64_t mid = (lo + hi) >> 1;
    if ((int64_t)a[mid] < x) lo = mid + 1; else hi = mid;
  }
  return lo;
}

// Workspace carving: 256-byte aligned bump allocator over the caller's buffer. With base == null
// it only measures.
struct Carver {
  char* base;
  size_t off = 0;
  explicit Carver(void* b) : base(static_cast<char*>(b)) {}
  template <class T>
  T* take(int64_t count) {
    off = (size_t)round_up((int64_t)off, 256);
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off += (size_t)(count > 0 ? count : 0) * sizeof(T);
    return p;
  }
};

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline int launch_status() {
  return cudaGetLastError() == cudaSuccess ? GSPARSE_OK : GSPARSE_ERR_CUDA;
}

// SM count of the current device, cached per device.
int sm_count();

// Bulk asynchronous copies into shared memory with mbarrier completion (no multicast: every copy
// reads this GPU's own memory into the issuing CTA's shared memory). Every wait is bounded.
constexpr long long kWaitCycles = 1ll << 31;   // about a second of SM clock

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits until the barrier's phase with this parity has completed; false after `limit` SM cycles.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  long long limit = kWaitCycles) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity))
    if (clock64() - t0 > limit) return false;
  return true;
}

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void fence_mbarrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Programmatic dependent launch (sm_90 and later). Every kernel of the library is launched with
// launch(), which lets it start while the kernel before it in the stream is finishing, and begins
// with pdl_begin(): griddepcontrol.wait blocks until every earlier grid it depends on has completed
// and its memory is visible, so nothing is read or written before that; the kernel then allows
// the next kernel to launch at once. Only the launch latency overlaps. A kernel whose
// predecessor was launched without this attribute (a memset, another library's kernel) simply
// starts after it.
__device__ __forceinline__ void pdl_begin() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... P, typename... A>
inline void launch(void (*kernel)(P...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, A&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaLaunchKernelEx(&cfg, kernel, static_cast<A&&>(args)...);
}

}  // namespace gs
