// cf_common.cuh -- small device helpers shared by the libcf kernels.
//
// Memory access wrappers pick cache behaviour explicitly: every activation
// and state element is touched exactly once per step, so reads bypass L1
// allocation and write-only outputs use the streaming (evict-first) hint.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace cf {

constexpr unsigned kFullMask = 0xffffffffu;

// bf16 bit pattern -> fp32, exact (bf16 is the upper half of binary32).
__device__ __forceinline__ float bf16_bits_to_f32(uint32_t h) {
    return __uint_as_float(h << 16);
}

// 16-byte read-only load of data not written by this kernel, no L1 allocate.
__device__ __forceinline__ uint4 ld_ro_v4(const void *p) {
    uint4 r;
    asm("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
        : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
        : "l"(p));
    return r;
}

// 16-byte load of state this thread later overwrites (coherent path).
__device__ __forceinline__ float4 ld_state_v4(const float *p) {
    float4 r;
    asm volatile("ld.global.L1::no_allocate.v4.f32 {%0,%1,%2,%3}, [%4];"
                 : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ void st_state_v4(float *p, float4 v) {
    asm volatile("st.global.v4.f32 [%0], {%1,%2,%3,%4};" ::"l"(p), "f"(v.x),
                 "f"(v.y), "f"(v.z), "f"(v.w)
                 : "memory");
}

// Streaming store for write-only outputs (error buffer).
__device__ __forceinline__ void st_stream_v4(float *p, float4 v) {
    asm volatile("st.global.cs.v4.f32 [%0], {%1,%2,%3,%4};" ::"l"(p), "f"(v.x),
                 "f"(v.y), "f"(v.z), "f"(v.w)
                 : "memory");
}

__device__ __forceinline__ bool misaligned16(const void *p) {
    return (reinterpret_cast<uintptr_t>(p) & 15u) != 0;
}

}  // namespace cf
