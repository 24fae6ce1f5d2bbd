// Shared device/host helpers for the ds4moe CUDA library (sm_100a).
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "ds4moe.h"

namespace ds4 {

constexpr int QK = 256;  // weights per quantization block

// ---------------------------------------------------------------------------
// Per-device error word.  Kernels record the first data error they meet
// (bad expert id, fp16 overflow, timed-out wait) here instead of trapping.
// ---------------------------------------------------------------------------
__device__ int32_t g_device_error;

__device__ __forceinline__ void set_device_error(int32_t code) { atomicCAS(&g_device_error, 0, code); }

// ---------------------------------------------------------------------------
// Prepared-layout plane offsets (see include/ds4moe.h, "PREPARED layout").
// ---------------------------------------------------------------------------
__host__ __device__ __forceinline__ uint64_t align256(uint64_t x) { return (x + 255) & ~uint64_t(255); }

struct Planes {
    uint64_t off[4];
    uint64_t total;
};

__host__ __device__ __forceinline__ Planes plane_layout(int fmt, uint64_t nblk) {
    Planes p{};
    uint64_t sz[4] = {0, 0, 0, 0};
    int n = 0;
    if (fmt == DS4MOE_FMT_IQ2X) {
        sz[0] = 32 * nblk; sz[1] = 32 * nblk; sz[2] = 4 * nblk; sz[3] = 2 * nblk; n = 4;
    } else if (fmt == DS4MOE_FMT_Q2K) {
        sz[0] = 64 * nblk; sz[1] = 16 * nblk; sz[2] = 4 * nblk; n = 3;
    } else if (fmt == DS4MOE_FMT_Q4K) {
        sz[0] = 128 * nblk; sz[1] = 12 * nblk; sz[2] = 4 * nblk; n = 3;
    }
    uint64_t o = 0;
    for (int i = 0; i < 4; i++) {
        p.off[i] = o;
        if (i < n) o += align256(sz[i]);
    }
    p.total = o;
    return p;
}

__host__ __device__ __forceinline__ int canonical_block_bytes(int fmt) {
    return fmt == DS4MOE_FMT_IQ2X ? 66 : fmt == DS4MOE_FMT_Q2K ? 84 : fmt == DS4MOE_FMT_Q4K ? 144 : 0;
}

// ---------------------------------------------------------------------------
// Small device helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ float half_bits_to_float(uint16_t h) { return __half2float(__ushort_as_half(h)); }

__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }

__device__ __forceinline__ __half2 u32_as_half2(uint32_t u) {
    __half2 h;
    *reinterpret_cast<uint32_t *>(&h) = u;
    return h;
}
__device__ __forceinline__ uint32_t half2_as_u32(__half2 h) { return *reinterpret_cast<uint32_t *>(&h); }

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

// Power-of-two exponent e such that amax * 2^e lies in [2^(top-1), 2^top);
// 0 when amax is zero or not finite.  Scaling by 2^e is exact.
__device__ __forceinline__ int pow2_exponent_for(float amax, int top) {
    if (!(amax > 0.f) || !isfinite(amax)) return 0;
    int q;
    frexpf(amax, &q);  // amax = m * 2^q, m in [0.5, 1)
    int e = top - q;
    return max(-100, min(100, e));
}

// silu(g) = g * sigmoid(g), with the fast hardware exponential and divide (relative error ~1e-6, far inside the
// layer's tolerance).  For g below about -88 the denominator overflows to +inf and the result is -0; the exact
// value is smaller than 1e-36 in magnitude.
__device__ __forceinline__ float silu(float g) { return __fdividef(g, 1.f + __expf(-g)); }

// Programmatic dependent launch: wait for the preceding grid's results.
// A no-op when the kernel was launched without the PDL attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" :::); }

__device__ __forceinline__ uint4 ldg_nc_v4(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}
__device__ __forceinline__ uint32_t ldg_nc_u32(const void *p) {
    uint32_t r;
    asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(r) : "l"(p));
    return r;
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

}  // namespace ds4
