// Shared device helpers for the tiered MoE kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "moe_tiered.h"

namespace moe {

constexpr int kWarp = 32;

__device__ __forceinline__ float bf16_to_f32(uint16_t b) {
    return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

__device__ __forceinline__ uint16_t f32_to_bf16_rne(float v) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(v));
}

__device__ __forceinline__ float f16_bits_to_f32(uint16_t b) {
    return __half2float(__ushort_as_half(b));
}

// Low and high bf16 halves of a 32-bit word, widened exactly to fp32.
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Streaming 16-byte load that bypasses L1 allocation (weights are read once).
__device__ __forceinline__ uint4 ld_stream_v4(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ uint2 ld_stream_v2(const void *p) {
    uint2 r;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];"
                 : "=r"(r.x), "=r"(r.y)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ uint32_t ld_stream_u32(const void *p) {
    uint32_t r;
    asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(r) : "l"(p));
    return r;
}

// Programmatic dependent launch: a kernel launched with programmatic stream
// serialization may start while its predecessor on the stream still runs;
// pdl_wait() returns once the predecessor has completed and its writes are
// visible (immediately when there is no such predecessor), and pdl_trigger()
// lets the successor start its own prologue.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Sum over groups of `width` consecutive lanes (width a power of two <= 32).
__device__ __forceinline__ float group_sum(float v, int width) {
    for (int o = width >> 1; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ void status_or(int32_t *status, int32_t bits) {
    if (status) atomicOr(status, bits);
}

// ---------------------------------------------------------------------------
// Code -> float conversion.  Exact, by building the float's bit pattern:
// 2^23 + c has the integer c in its low mantissa bits, so subtracting the
// bias constant (2^23 + offset) leaves c - offset exactly (the "magic number"
// int->float conversion).
// ---------------------------------------------------------------------------
constexpr float kMagic = 8388608.0f;  // 2^23

// Four signed 8-bit codes in a word -> four floats (q values).
__device__ __forceinline__ void s8x4_to_f32(uint32_t w, float *f) {
    const uint32_t u = w ^ 0x80808080u;  // q + 128 in each byte, 0..255
    f[0] = __uint_as_float(__byte_perm(u, 0x4b000000u, 0x7650)) - (kMagic + 128.0f);
    f[1] = __uint_as_float(__byte_perm(u, 0x4b000000u, 0x7651)) - (kMagic + 128.0f);
    f[2] = __uint_as_float(__byte_perm(u, 0x4b000000u, 0x7652)) - (kMagic + 128.0f);
    f[3] = __uint_as_float(__byte_perm(u, 0x4b000000u, 0x7653)) - (kMagic + 128.0f);
}

// Eight 4-bit codes (c = q + 8) in a word -> eight floats (q values), in order.
__device__ __forceinline__ void u4x8_to_f32(uint32_t w, float *f) {
#pragma unroll
    for (int i = 0; i < 8; ++i)
        f[i] = __uint_as_float(0x4b000000u | ((w >> (4 * i)) & 0xfu)) - (kMagic + 8.0f);
}

// 3-bit codes (c = q + 4): 4 low-plane bits pairs from `lo` byte positions and
// the matching high bits.  Produces 16 floats from 32 low bits and 16 high bits.
__device__ __forceinline__ void u3x16_to_f32(uint32_t lo, uint32_t hi16, float *f) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const uint32_t c = ((lo >> (2 * i)) & 3u) | (((hi16 >> i) & 1u) << 2);
        f[i] = __uint_as_float(0x4b000000u | c) - (kMagic + 4.0f);
    }
}

// Launch attribute list for a kernel that may overlap its predecessor
// (programmatic dependent launch); `extra` (e.g. cooperative) is appended.
struct PdlAttrs {
    cudaLaunchAttribute a[2];
    int n;
    explicit PdlAttrs(bool cooperative = false) : n(0) {
        a[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        a[n].val.programmaticStreamSerializationAllowed = 1;
        ++n;
        if (cooperative) {
            a[n].id = cudaLaunchAttributeCooperative;
            a[n].val.cooperative = 1;
            ++n;
        }
    }
};

}  // namespace moe
