// Router: logits GEMV over the expert table, then a warp-level softmax/top-k.
//
// [P1] "a small dictionary before we start": each layer has 512 experts and a
// router picks the best 10 for each word.  [P5] "What the model actually is":
// 10 routed plus 1 shared expert per token.  Selection order is (logit desc,
// id asc); weights are the softmax restricted to the chosen k, renormalised.
#include <float.h>

#include "common.cuh"

namespace moe {

constexpr int kRouterTokTile = 16;   // tokens staged in shared memory per CTA
constexpr int kRouterWarps = 4;      // one expert per warp

// logits[t, e] = x[t] . w_router[e] + bias[e], fp32 accumulation.
// grid = (ceil(E / 4), ceil(T / 16)); x tile of 16 tokens staged as bf16.
__global__ void __launch_bounds__(kRouterWarps * 32)
router_logits_kernel(const uint16_t *__restrict__ x, const uint16_t *__restrict__ wr,
                     const float *__restrict__ bias, int T, int H, int E,
                     float *__restrict__ logits) {
    extern __shared__ __align__(16) uint16_t xs[];  // [kRouterTokTile][H]
    const int t0 = blockIdx.y * kRouterTokTile;
    const int nt = min(kRouterTokTile, T - t0);
    const int vec_per_row = H / 8;
    for (int i = threadIdx.x; i < nt * vec_per_row; i += blockDim.x) {
        const int t = i / vec_per_row, c = i - t * vec_per_row;
        reinterpret_cast<uint4 *>(xs)[t * vec_per_row + c] =
            reinterpret_cast<const uint4 *>(x + static_cast<size_t>(t0 + t) * H)[c];
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int e = blockIdx.x * kRouterWarps + warp;
    if (e >= E) return;
    float acc[kRouterTokTile];
#pragma unroll
    for (int t = 0; t < kRouterTokTile; ++t) acc[t] = 0.f;
    const uint16_t *wrow = wr + static_cast<size_t>(e) * H;
#pragma unroll 4
    for (int c = lane; c < vec_per_row; c += 32) {
        const uint4 wv = ld_stream_v4(wrow + c * 8);
        const float w[8] = {bf16lo(wv.x), bf16hi(wv.x), bf16lo(wv.y), bf16hi(wv.y),
                            bf16lo(wv.z), bf16hi(wv.z), bf16lo(wv.w), bf16hi(wv.w)};
#pragma unroll
        for (int t = 0; t < kRouterTokTile; ++t) {
            if (t < nt) {
                const uint4 xv = reinterpret_cast<const uint4 *>(xs)[t * vec_per_row + c];
                float a = acc[t];
                a = fmaf(w[0], bf16lo(xv.x), a);
                a = fmaf(w[1], bf16hi(xv.x), a);
                a = fmaf(w[2], bf16lo(xv.y), a);
                a = fmaf(w[3], bf16hi(xv.y), a);
                a = fmaf(w[4], bf16lo(xv.z), a);
                a = fmaf(w[5], bf16hi(xv.z), a);
                a = fmaf(w[6], bf16lo(xv.w), a);
                a = fmaf(w[7], bf16hi(xv.w), a);
                acc[t] = a;
            }
        }
    }
    const float b = bias ? bias[e] : 0.f;
#pragma unroll
    for (int t = 0; t < kRouterTokTile; ++t) {
        if (t < nt) {
            const float s = warp_sum(acc[t]);
            if (lane == 0) logits[static_cast<size_t>(t0 + t) * E + e] = s + b;
        }
    }
}

// Is (va, ia) ranked before (vb, ib)?  Larger logit first, then lower id.
__device__ __forceinline__ bool ranks_before(float va, int ia, float vb, int ib) {
    return va > vb || (va == vb && ia < ib);
}

// One warp per token: k rounds of a warp-wide arg-max over the E logits held
// in registers (NJ per lane), then the renormalised softmax over the winners.
template <int NJ>
__global__ void __launch_bounds__(256)
topk_softmax_kernel(const float *__restrict__ logits, int T, int E, int k,
                    int32_t *__restrict__ topk_idx, float *__restrict__ topk_w) {
    const int lane = threadIdx.x & 31;
    const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (t >= T) return;
    const float *row = logits + static_cast<size_t>(t) * E;
    float v[NJ];
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
        const int e = lane + 32 * j;
        v[j] = e < E ? row[e] : -FLT_MAX;
    }
    uint32_t taken = 0;
#pragma unroll
    for (int j = 0; j < NJ; ++j)
        if (lane + 32 * j >= E) taken |= 1u << j;
    float my_v = 0.f;
    int my_i = 0;
    for (int r = 0; r < k; ++r) {
        float bv = -FLT_MAX;
        int bi = 0x7fffffff;
#pragma unroll
        for (int j = 0; j < NJ; ++j) {
            const int e = lane + 32 * j;
            if (!((taken >> j) & 1u) && ranks_before(v[j], e, bv, bi)) { bv = v[j]; bi = e; }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
            if (ranks_before(ov, oi, bv, bi)) { bv = ov; bi = oi; }
        }
        if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
        if (lane == r) { my_v = bv; my_i = bi; }
    }
    const float l0 = __shfl_sync(0xffffffffu, my_v, 0);
    const float z = lane < k ? expf(my_v - l0) : 0.f;
    const float sum = warp_sum(z);
    if (lane < k) {
        topk_idx[static_cast<size_t>(t) * k + lane] = my_i;
        topk_w[static_cast<size_t>(t) * k + lane] = z / sum;
    }
}

}  // namespace moe

cudaError_t moe_launch_router_logits(const uint16_t *x, const uint16_t *wr, const float *bias, int T,
                                     int H, int E, float *logits, cudaStream_t s) {
    const size_t smem = static_cast<size_t>(moe::kRouterTokTile) * H * sizeof(uint16_t);
    dim3 grid((E + moe::kRouterWarps - 1) / moe::kRouterWarps,
              (T + moe::kRouterTokTile - 1) / moe::kRouterTokTile);
    moe::router_logits_kernel<<<grid, moe::kRouterWarps * 32, smem, s>>>(x, wr, bias, T, H, E, logits);
    return cudaGetLastError();
}

cudaError_t moe_configure_router() {
    return cudaFuncSetAttribute(moe::router_logits_kernel,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
}

cudaError_t moe_launch_topk(const float *logits, int T, int E, int k, int32_t *idx, float *w,
                            cudaStream_t s) {
    const int threads = 256;
    const int grid = (T * 32 + threads - 1) / threads;
    const int nj = (E + 31) / 32;
    if (nj <= 4) moe::topk_softmax_kernel<4><<<grid, threads, 0, s>>>(logits, T, E, k, idx, w);
    else if (nj <= 8) moe::topk_softmax_kernel<8><<<grid, threads, 0, s>>>(logits, T, E, k, idx, w);
    else if (nj <= 16) moe::topk_softmax_kernel<16><<<grid, threads, 0, s>>>(logits, T, E, k, idx, w);
    else moe::topk_softmax_kernel<32><<<grid, threads, 0, s>>>(logits, T, E, k, idx, w);
    return cudaGetLastError();
}
