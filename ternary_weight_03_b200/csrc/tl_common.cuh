// tl_common.cuh -- small device helpers shared by the libternary kernels
// (inline PTX wrappers for sm_100a).
#pragma once
#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_fp16.h>

namespace tlk {

// Per-device error word.  Kernels OR a code in when a bounded wait gives up;
// tl_device_status() reads and clears it.  (All kernels live in the single
// CUDA translation unit tl_device.cu, which is the only includer.)
__device__ unsigned int g_error_word = 0;
constexpr unsigned int kErrTimeout = 1u;

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// 128-bit streaming load of data read exactly once (weights): not kept in L1.
__device__ __forceinline__ uint4 ld_stream(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// 128-bit read-only load of data shared by many CTAs (activations): L1-cached.
__device__ __forceinline__ uint4 ld_shared_ro(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// D = A (16x16 fp16, row) * B (16x8 fp16, col) + D, fp32 accumulate.
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Programmatic dependent launch.  wait: block until the preceding grid on the
// stream has completed and its memory is visible (a no-op when the kernel was
// launched without the programmatic-serialization attribute).  launch:
// allow the next grid on the stream to begin its own pre-wait prologue.
__device__ __forceinline__ void pdl_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ uint16_t f32_to_f16_bits(float v) {
    return __half_as_ushort(__float2half_rn(v));
}

}  // namespace tlk
