// common.cuh -- device helpers shared by the route / layout / dispatch /
// combine kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "moe_route07.h"

namespace moe {

constexpr unsigned kFull = 0xffffffffu;

// Workspace header (first 256 bytes of every workspace).
struct WsHeader {
  int32_t err;             // first device-side error code (moe_status_t), 0 = none
  int32_t detail;          // index that caused it
  uint32_t reserved[2];
  uint32_t epoch;          // layout: which of the two tile tables the next call fills
  uint32_t done;           // layout: place CTAs finished (the last one bumps epoch)
  uint32_t words_used[2];  // layout: words of each table filled since it was last cleared
  uint32_t pad[56];        // (epoch..words_used form one 16-byte word at offset 16)
};
static_assert(sizeof(WsHeader) == 256, "workspace header is 256 bytes");

// Record the first device-side problem; later ones are dropped.
__device__ __forceinline__ void report(WsHeader* h, int code, int detail) {
  if (atomicCAS(&h->err, 0, code) == 0) atomicExch(&h->detail, detail);
}

// Relaxed, GPU-scope 32-bit load/store (one word carries flag and value, so
// no extra ordering is needed between them).
__device__ __forceinline__ uint32_t ld_relaxed(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.relaxed.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_relaxed(uint32_t* p, uint32_t v) {
  asm volatile("st.relaxed.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release(uint32_t* p, uint32_t v) {
  asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// L2-coherent 32-bit load (bypasses L1), for data another CTA published.
__device__ __forceinline__ int32_t ld_cg(const int32_t* p) { return __ldcg(p); }

// Programmatic dependent launch.  pdl_wait(): block until the kernel this one
// was launched behind has finished and its writes are visible (returns at once
// when launched without the attribute).  pdl_trigger(): allow the kernel
// launched behind this one to start placing its CTAs.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// 16-byte global accesses.
__device__ __forceinline__ uint4 ldg16(const void* p) {
  return __ldg(reinterpret_cast<const uint4*>(p));
}
// Streaming load: data read once, keep it out of L1.
__device__ __forceinline__ uint4 ld16_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}
__device__ __forceinline__ void st16(void* p, const uint4& v) {
  *reinterpret_cast<uint4*>(p) = v;
}

// bf16 pair <-> fp32 (exact widening; nearest-even narrowing).
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

}  // namespace moe
