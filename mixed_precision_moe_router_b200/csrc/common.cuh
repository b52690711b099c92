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

// ---------------------------------------------------------------------------
// FP4 (E2M1) codes of an FP4 shelf ([P1] "step 4": MXFP4 for the rarest
// down projections).  A code is sign * 8 + m, the magnitude index m of
// 0, 0.5, 1, 1.5, 2, 3, 4, 6; the shelf stores d = X / 2 for the block scale X,
// so a weight is d * q with the integer q = 2 * value in {0, +-1, +-2, +-3,
// +-4, +-6, +-8, +-12}, exact in fp16 like the integer shelves' codes.
// Plans and kernels carry an FP4 shelf as bits = kBitsFp4 (4-bit storage).
// ---------------------------------------------------------------------------
constexpr int kBitsFp4 = MOE_FP4;
__host__ __device__ __forceinline__ int storage_bits(int bits) { return bits == kBitsFp4 ? 4 : bits; }

// A shelf's two formats as one int (plans and per-slot tables): the gate_up
// format in the low byte, the down format in the next.
__host__ __device__ __forceinline__ int tier_dn_bits(const moe_tier &t) { return t.dn_bits ? t.dn_bits : t.bits; }
__host__ __device__ __forceinline__ int tier_formats(const moe_tier &t) { return t.bits | (tier_dn_bits(t) << 8); }
__host__ __device__ __forceinline__ int phase_bits(int formats, int phase) {
    return phase == 0 ? (formats & 0xff) : (formats >> 8);
}

// The 8 codes of one 32-bit word (nibble i = weight i) as four half2 of the
// integers q: P[j] = (q_j, q_{j+4}), the pairing the 4-bit decoders use.  The
// fp16 encodings of 0, 1, 2, 3, 4, 6, 8 and 12 all have a zero low byte, so a
// byte table of their high bytes, indexed by each nibble's magnitude bits
// through prmt, builds the halves directly; the sign bit is then or-ed in.
__device__ __forceinline__ void fp4_pairs(uint32_t v, uint32_t (&P)[4]) {
    constexpr uint32_t kLo = 0x42403C00u, kHi = 0x4A484644u;  // 0 1 2 3 | 4 6 8 12 (high bytes)
    uint32_t m0, m1;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(m0) : "r"(kLo), "r"(kHi), "r"(v & 0x7777u));          // q0..q3
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(m1) : "r"(kLo), "r"(kHi), "r"((v >> 16) & 0x7777u));  // q4..q7
    // bytes (0, hb(q_j), 0, hb(q_{j+4})): a selector nibble with bit 3 set
    // copies the sign of a table byte, which is 0
    const uint32_t sel[4] = {0x4808u, 0x5818u, 0x6828u, 0x7838u};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        uint32_t y;
        asm("prmt.b32 %0, %1, %2, %3;" : "=r"(y) : "r"(m0), "r"(m1), "r"(sel[j]));
        P[j] = y | ((v << (12 - 4 * j)) & 0x80008000u);  // sign bits 4j+3 and 4j+19
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
