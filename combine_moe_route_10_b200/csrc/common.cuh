// Shared device-side helpers of libmoe: status bits, vector types and small PTX wrappers.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace moe {

// Status word bits written by kernels into the first 4 bytes of a workspace.
constexpr int kStatusInvalidTopk = 1;  // an expert id outside [0, E) was seen
constexpr int kStatusTimeout = 2;      // a bounded pipeline wait ran out

// Bound on any single device-side wait (ns of %globaltimer).  A healthy wait in these kernels is
// microseconds; one second means something upstream is broken, and the kernel gives up cleanly.
constexpr unsigned long long kWaitLimitNs = 1000000000ull;

constexpr int kWarp = 32;

__device__ __forceinline__ unsigned long long global_timer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void record_status(int* status, int bit) {
  if (status != nullptr) atomicOr(status, bit);
}

// Programmatic dependent launch: every kernel of the path is launched with programmatic stream
// serialisation, so its launch and pre-wait prologue overlap the previous kernel's tail.  Each
// kernel calls griddep_wait() before its first global-memory access (read or write), which returns
// once the previous grid has completed and its memory is visible: stream-order semantics are kept.
__device__ __forceinline__ void griddep_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ void st_v4(void* p, uint4 v) {
  asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}

__device__ __forceinline__ void st_cs_v4(void* p, uint4 v) {
  asm volatile("st.global.cs.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);  // round to nearest even, each half
  return *reinterpret_cast<uint32_t*>(&v);
}

}  // namespace moe
