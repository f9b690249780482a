// Shared device helpers and host-side status plumbing of libi4rt (sm_100a only).
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "i4rt.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "libi4rt is built for sm_100a only"
#endif

namespace i4 {

// ------------------------------------------------------------------ host side

// Record a failure message for i4_last_error() and return `status`.
int fail(int status, const char *fmt, ...);
// Map a CUDA error to I4_ECUDA with its text; I4_OK when err == cudaSuccess.
int cuda_check(cudaError_t err, const char *what);
// Launch error of the last kernel (cudaGetLastError) as a status.
int launch_check(const char *what);

inline bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Launch with the programmatic-dependent-launch attribute when `pdl` is set
// (the kernel may start while its predecessor on the stream finishes; every
// kernel here calls griddepcontrol.wait before touching its predecessor's output).
template <typename... KArgs, typename... Args>
cudaError_t launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream, bool pdl,
                   Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

constexpr int kNumSMs = 148;

// When set, launch helpers only configure their kernels (attributes, occupancy)
// and return without launching; used before a stream capture.
extern bool g_dry_run;

// ------------------------------------------------------------------ device side

// Wait until the grids this one depends on (programmatic launch) have completed
// and their writes are visible; a no-op for ordinary launches.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// Allow the next kernel on the stream to begin launching.
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ uint32_t lop3_and_xor(uint32_t a, uint32_t mask, uint32_t flip) {
    // (a ^ flip) & mask
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0x48;" : "=r"(d) : "r"(a), "r"(mask), "r"(flip));
    return d;
}

__device__ __forceinline__ uint32_t lop3_select(uint32_t a, uint32_t mask, uint32_t c) {
    // bits under mask: a ^ c; bits outside mask: c   i.e. (mask & (a ^ c)) | (~mask & c)
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(d) : "r"(a), "r"(mask), "r"(c));
    return d;
}

// Streaming 16-byte load of read-once data: bypass L1, evict first from L2.
__device__ __forceinline__ uint4 ldg_stream(const uint4 *p, uint64_t policy) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p), "l"(policy));
    return v;
}

__device__ __forceinline__ uint64_t evict_first_policy() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

__device__ __forceinline__ uint16_t ldg_u16(const uint16_t *p) {
    uint16_t v;
    asm volatile("ld.global.nc.u16 %0, [%1];" : "=h"(v) : "l"(p));
    return v;
}

// acc + a.lo * b.lo + a.hi * b.hi with fp16 inputs, fp32 products and sums.
__device__ __forceinline__ float fma2_f16_f32(uint32_t a, uint32_t b, float acc) {
    float d;
    asm("{\n\t.reg .f16 al, ah, bl, bh;\n\t.reg .f32 t;\n\t"
        "mov.b32 {al, ah}, %1;\n\tmov.b32 {bl, bh}, %2;\n\t"
        "fma.rn.f32.f16 t, al, bl, %3;\n\t"
        "fma.rn.f32.f16 %0, ah, bh, t;\n\t}"
        : "=f"(d)
        : "r"(a), "r"(b), "f"(acc));
    return d;
}

__device__ __forceinline__ uint32_t hsub2_bits(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

__device__ __forceinline__ uint32_t hfma2_bits(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// Packed fp32 pair arithmetic of sm_100 (one instruction for two lanes of math).
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
    unsigned long long d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;"
        : "=l"(d)
        : "l"(*reinterpret_cast<unsigned long long *>(&a)), "l"(*reinterpret_cast<unsigned long long *>(&b)),
          "l"(*reinterpret_cast<unsigned long long *>(&c)));
    return *reinterpret_cast<float2 *>(&d);
}

__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
    unsigned long long d;
    asm("add.rn.f32x2 %0, %1, %2;"
        : "=l"(d)
        : "l"(*reinterpret_cast<unsigned long long *>(&a)), "l"(*reinterpret_cast<unsigned long long *>(&b)));
    return *reinterpret_cast<float2 *>(&d);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float half_bits_to_float(uint16_t h) { return __half2float(__ushort_as_half(h)); }
__device__ __forceinline__ uint16_t float_to_half_bits(float f) { return __half_as_ushort(__float2half_rn(f)); }

}  // namespace i4
