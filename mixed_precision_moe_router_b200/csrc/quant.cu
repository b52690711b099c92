// Block quantisation and dequantisation of the shelf format.
//
// [P1] "step 4: three shelves, all on the GPU": popular experts keep more bits,
// rare ones are squeezed harder.  [P3] "Why the model fits at all": a code per
// weight plus one 16-bit scale per 32 weights (4.5 bits/weight at 4 bits).
// The exact rules (absmax, fp16 scale, fp32 division, half-away rounding; for
// an FP4 shelf the MX power-of-two scale and E2M1 rounding) and the byte
// layout are stated in moe_tiered.h.  Internally an FP4 shelf is bits = 5.
#include "common.cuh"

namespace moe {

__device__ __forceinline__ int qmax_of(int bits) { return bits == 8 ? 127 : (bits == 4 ? 7 : 3); }

// FP4 (E2M1) code of w in a block whose largest magnitude is amax, the
// OCP MX conversion: X = 2^(floor(log2 amax) - 2), the E2M1 value nearest to
// w / X (a tie goes to the even magnitude index; beyond 6 it saturates);
// *d receives X / 2 as fp16 bits (0 for an all-zero block).
__device__ __forceinline__ uint32_t fp4_code(float w, float amax, uint16_t *d) {
    if (amax == 0.0f) {
        *d = 0;
        return 0;
    }
    int e = 0;
    frexpf(amax, &e);  // amax = f * 2^e, f in [0.5, 1): floor(log2 amax) = e - 1
    const int shared = min(max(e - 3, -23), 16);
    *d = __half_as_ushort(__float2half_rn(ldexpf(1.0f, shared - 1)));
    const float a = fabsf(ldexpf(w, -shared));  // |w| / X, exact
    // magnitude index: midpoints between 0, 0.5, 1, 1.5, 2, 3, 4, 6; a value
    // on a midpoint after an odd index moves up to the even one
    int m = (a > 0.25f) + (a > 0.75f) + (a > 1.25f) + (a > 1.75f) + (a > 2.5f) + (a > 3.5f) + (a > 5.0f);
    m += (a == 0.75f) + (a == 1.75f) + (a == 3.5f);
    return static_cast<uint32_t>(m | ((w < 0.0f && m > 0) ? 8 : 0));
}

// One warp per block of 32 weights; lane i owns weight i of the block.
__global__ void quantize_kernel(const float *__restrict__ src, int64_t rows, int K, int bits,
                                uint8_t *__restrict__ qs, uint16_t *__restrict__ scale) {
    const int lane = threadIdx.x & 31;
    const int64_t nblk_row = K / 32;
    const int64_t total = rows * nblk_row;
    const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    const size_t row_bytes = static_cast<size_t>(K) * storage_bits(bits) / 8;
    const float qmax = static_cast<float>(qmax_of(bits));
    for (int64_t b = warp0; b < total; b += nwarps) {
        const int64_t row = b / nblk_row;
        const int blk = static_cast<int>(b - row * nblk_row);
        const float w = src[row * K + blk * 32 + lane];
        float amax = fabsf(w);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        uint8_t *rowp = qs + row * row_bytes;
        if (bits == kBitsFp4) {
            uint16_t d4;
            const uint32_t c = fp4_code(w, amax, &d4);
            if (lane == 0) scale[row * nblk_row + blk] = d4;
            const uint32_t nb = __shfl_down_sync(0xffffffffu, c, 1);
            if ((lane & 1) == 0) rowp[blk * 16 + (lane >> 1)] = static_cast<uint8_t>(c | (nb << 4));
            continue;
        }
        const __half d = __float2half_rn(__fdiv_rn(amax, qmax));
        const float df = __half2float(d);
        int q = 0;
        if (df != 0.0f) {
            float r = roundf(__fdiv_rn(w, df));  // round half away from zero
            r = fminf(fmaxf(r, -qmax), qmax);
            q = static_cast<int>(r);
        }
        if (lane == 0) scale[row * nblk_row + blk] = __half_as_ushort(d);
        if (bits == 8) {
            rowp[blk * 32 + lane] = static_cast<uint8_t>(static_cast<int8_t>(q));
        } else if (bits == 4) {
            const uint32_t c = static_cast<uint32_t>(q + 8);
            const uint32_t nb = __shfl_down_sync(0xffffffffu, c, 1);
            if ((lane & 1) == 0) rowp[blk * 16 + (lane >> 1)] = static_cast<uint8_t>(c | (nb << 4));
        } else {  // 3 bits, two planes
            const uint32_t c = static_cast<uint32_t>(q + 4);
            const uint32_t lo = (c & 3u) << (2 * (lane & 3));
            const uint32_t hi = ((c >> 2) & 1u) << (lane & 7);
            uint32_t lob = lo, hib = hi;
#pragma unroll
            for (int o = 1; o < 8; o <<= 1) {
                const uint32_t l2 = __shfl_xor_sync(0xffffffffu, lob, o);
                const uint32_t h2 = __shfl_xor_sync(0xffffffffu, hib, o);
                if (o < 4) lob |= l2;
                hib |= h2;
            }
            const int i = blk * 32 + lane;
            if ((lane & 3) == 0) rowp[i >> 2] = static_cast<uint8_t>(lob);
            if ((lane & 7) == 0) rowp[K / 4 + (i >> 3)] = static_cast<uint8_t>(hib);
        }
    }
}

// One thread per weight.
__global__ void dequantize_kernel(const uint8_t *__restrict__ qs, const uint16_t *__restrict__ scale,
                                  int64_t rows, int K, int bits, float *__restrict__ out_f32,
                                  uint16_t *__restrict__ out_f16) {
    const int64_t n = rows * K;
    const size_t row_bytes = static_cast<size_t>(K) * storage_bits(bits) / 8;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t row = i / K;
        const int k = static_cast<int>(i - row * K);
        const uint8_t *rowp = qs + row * row_bytes;
        int q;
        if (bits == kBitsFp4) {
            const int c = (rowp[k >> 1] >> (4 * (k & 1))) & 0xf;
            const int mag = static_cast<int>((0x0C08060403020100ull >> (8 * (c & 7))) & 0xff);  // 2|value|
            q = (c & 8) ? -mag : mag;
        } else if (bits == 8) {
            q = static_cast<int8_t>(rowp[k]);
        } else if (bits == 4) {
            q = static_cast<int>((rowp[k >> 1] >> (4 * (k & 1))) & 0xf) - 8;
        } else {
            const int lo = (rowp[k >> 2] >> (2 * (k & 3))) & 3;
            const int hi = (rowp[K / 4 + (k >> 3)] >> (k & 7)) & 1;
            q = (lo | (hi << 2)) - 4;
        }
        const float w = f16_bits_to_f32(scale[row * (K / 32) + k / 32]) * static_cast<float>(q);
        if (out_f32) out_f32[i] = w;
        if (out_f16) out_f16[i] = __half_as_ushort(__float2half_rn(w));
    }
}

}  // namespace moe

// host launchers (called from api.cu after validation)
cudaError_t moe_launch_quantize(const float *src, int64_t rows, int K, int bits, uint8_t *qs,
                                uint16_t *scale, cudaStream_t s) {
    const int64_t blocks = rows * (K / 32);
    const int threads = 256;
    int64_t grid = (blocks * 32 + threads - 1) / threads;
    if (grid > 148 * 64) grid = 148 * 64;
    if (grid < 1) grid = 1;
    moe::quantize_kernel<<<static_cast<unsigned>(grid), threads, 0, s>>>(src, rows, K, bits, qs, scale);
    return cudaGetLastError();
}

cudaError_t moe_launch_dequantize(const uint8_t *qs, const uint16_t *scale, int64_t rows, int K,
                                  int bits, float *out_f32, uint16_t *out_f16, cudaStream_t s) {
    const int64_t n = rows * K;
    const int threads = 256;
    int64_t grid = (n + threads - 1) / threads;
    if (grid > 148 * 64) grid = 148 * 64;
    if (grid < 1) grid = 1;
    moe::dequantize_kernel<<<static_cast<unsigned>(grid), threads, 0, s>>>(qs, scale, rows, K, bits,
                                                                          out_f32, out_f16);
    return cudaGetLastError();
}
