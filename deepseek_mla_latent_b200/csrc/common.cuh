// common.cuh -- shared device helpers: the device error word, bounded waits,
// bf16 conversion and reductions.  No attention arithmetic lives here.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace mla {

// Error codes a kernel may raise in the device error word (bit flags).
enum : uint32_t {
  kErrTimeoutTmaFull = 1u << 0,    // consumer waited too long for a TMA tile
  kErrTimeoutStageFree = 1u << 1,  // producer waited too long for a free stage
  kErrTimeoutMma = 1u << 2,        // waited too long for a tensor-core commit
  kErrTimeoutSoftmax = 1u << 3,    // MMA issuer waited too long for P
  kErrTimeoutPeer = 1u << 4,       // waited too long for the partner CTA's scores
  kErrTimeoutDrain = 1u << 5,      // exit path waited too long for copies in flight
  kErrBadSchedule = 1u << 6,       // a work item pointed outside its buffers
  kErrBadPage = 1u << 7,           // a block-table entry of a page holding keys lies outside the cache
};

// One word per device; set with atomicOr, read and cleared by mla_device_status.
__device__ uint32_t g_mla_error_word;

__device__ __forceinline__ void raise_error(uint32_t code) { atomicOr(&g_mla_error_word, code); }

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

#ifndef MLA_FAULT_INJECT
// A wait gives up after this long (device time).  Legitimate waits in these
// kernels last microseconds; a second means a peer will never arrive.
constexpr uint64_t kWaitLimitNs = 1000000000ull;

__device__ __forceinline__ bool fault_plan(uint32_t) { return false; }
#else
// Fault-injection build (a separate library used only by the tests of the bounded waits):
// waits give up after 2 ms, and the host sets a plan word that makes one copy go missing.
constexpr uint64_t kWaitLimitNs = 2000000ull;

// Plan bits: 1 = the score CTA of work unit 0 skips the rotary copy of its first score tile.
__device__ uint32_t g_mla_fault_plan;
__device__ __forceinline__ bool fault_plan(uint32_t bit) { return (*(volatile uint32_t*)&g_mla_fault_plan & bit) != 0; }
#endif

template <typename T> struct Elem;
template <> struct Elem<float> {
  __device__ __forceinline__ static float load(const float* p) { return *p; }
  __device__ __forceinline__ static void store(float* p, float v) { *p = v; }
};
template <> struct Elem<__nv_bfloat16> {
  __device__ __forceinline__ static float load(const __nv_bfloat16* p) { return __bfloat162float(*p); }
  __device__ __forceinline__ static void store(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }
};

__host__ __device__ __forceinline__ int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }
__host__ __device__ __forceinline__ int64_t max64(int64_t a, int64_t b) { return a > b ? a : b; }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Sequence of packed row n: largest b with cu[b] <= n (cu has batch+1 entries).
__device__ __forceinline__ int find_sequence(const int* cu, int batch, int64_t n) {
  int lo = 0, hi = batch - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if ((int64_t)__ldg(cu + mid) <= n) lo = mid; else hi = mid - 1;
  }
  return lo;
}

}  // namespace mla
