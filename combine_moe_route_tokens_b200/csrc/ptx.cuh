// ptx.cuh — thin inline-PTX wrappers for sm_100a: programmatic dependent
// launch, cache-hinted vector loads, bf16 packing and the global timer used to
// bound every device-side wait.
#pragma once

#include <cstdint>

namespace moert {

__device__ __forceinline__ uint64_t global_timer_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// --------------------------------------------- programmatic dependent launch --
// A kernel launched with programmatic stream serialization may start before
// the previous kernel in the stream has finished. pdl_wait() blocks until that
// kernel has completed and its memory is visible; every kernel here calls it
// before its first read of data a predecessor may have written (without the
// launch attribute it returns at once). pdl_trigger() lets the next kernel in
// the stream be launched once every CTA of this one has started.

__device__ __forceinline__ void pdl_wait()
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

__device__ __forceinline__ void pdl_trigger()
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ------------------------------------------------------------ vector I/O ----

// 16-byte read-only load that does not allocate in L1 (streamed once).
__device__ __forceinline__ uint4 ld_stream_u4(const void *p)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ void st_u4(void *p, uint4 v)
{
    asm volatile("st.global.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

// ------------------------------------------------------------------ bf16 ----
// bf16 is the upper half of an fp32: widening is a shift; narrowing uses the
// hardware round-to-nearest-even conversion (cvt.rn.bf16x2.f32).

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t pack_bf16x2_rn(float lo, float hi)
{
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

} // namespace moert
