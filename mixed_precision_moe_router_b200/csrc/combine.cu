// Combine: out[t] = bf16(sum_j w[t,j] * y[t*k+j] + y_shared[t]), fixed order;
// optional residual stream x_next = bf16(residual + out).
//
// [P1] "step 4: three shelves, all on the GPU": the per-shelf results simply
// add up; with one shared expert always on ([P5] "What the model actually is").
#include "common.cuh"

namespace moe {

// One thread per 4 consecutive hidden elements of one token.
__global__ void __launch_bounds__(256)
combine_kernel(const float *__restrict__ y, const float *__restrict__ ysh, const float *__restrict__ w,
               int T, int k, int H, const uint16_t *__restrict__ res, uint16_t *__restrict__ out,
               uint16_t *__restrict__ xnext) {
    const int per_tok = H / 4;
    const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (idx >= static_cast<int64_t>(T) * per_tok) return;
    const int t = static_cast<int>(idx / per_tok);
    const int c = static_cast<int>(idx - static_cast<int64_t>(t) * per_tok);
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < k; ++j) {
        const float wj = w[static_cast<size_t>(t) * k + j];
        const float4 v = reinterpret_cast<const float4 *>(y + (static_cast<size_t>(t) * k + j) * H)[c];
        a.x = fmaf(wj, v.x, a.x);
        a.y = fmaf(wj, v.y, a.y);
        a.z = fmaf(wj, v.z, a.z);
        a.w = fmaf(wj, v.w, a.w);
    }
    if (ysh) {
        const float4 v = reinterpret_cast<const float4 *>(ysh + static_cast<size_t>(t) * H)[c];
        a.x += v.x; a.y += v.y; a.z += v.z; a.w += v.w;
    }
    const uint16_t o0 = f32_to_bf16_rne(a.x), o1 = f32_to_bf16_rne(a.y);
    const uint16_t o2 = f32_to_bf16_rne(a.z), o3 = f32_to_bf16_rne(a.w);
    const size_t base = static_cast<size_t>(t) * H + 4 * c;
    if (out) {
        uint2 pk;
        pk.x = static_cast<uint32_t>(o0) | (static_cast<uint32_t>(o1) << 16);
        pk.y = static_cast<uint32_t>(o2) | (static_cast<uint32_t>(o3) << 16);
        *reinterpret_cast<uint2 *>(out + base) = pk;
    }
    if (res) {
        const uint2 r = *reinterpret_cast<const uint2 *>(res + base);
        const uint16_t n0 = f32_to_bf16_rne(bf16lo(r.x) + bf16_to_f32(o0));
        const uint16_t n1 = f32_to_bf16_rne(bf16hi(r.x) + bf16_to_f32(o1));
        const uint16_t n2 = f32_to_bf16_rne(bf16lo(r.y) + bf16_to_f32(o2));
        const uint16_t n3 = f32_to_bf16_rne(bf16hi(r.y) + bf16_to_f32(o3));
        uint2 pk;
        pk.x = static_cast<uint32_t>(n0) | (static_cast<uint32_t>(n1) << 16);
        pk.y = static_cast<uint32_t>(n2) | (static_cast<uint32_t>(n3) << 16);
        *reinterpret_cast<uint2 *>(xnext + base) = pk;
    }
}

}  // namespace moe

cudaError_t moe_launch_combine(const float *y, const float *ysh, const float *w, int T, int k, int H,
                               const uint16_t *res, uint16_t *out, uint16_t *xnext, cudaStream_t s) {
    const int64_t n = static_cast<int64_t>(T) * (H / 4);
    const int threads = 256;
    const int64_t grid = (n + threads - 1) / threads;
    moe::combine_kernel<<<static_cast<unsigned>(grid), threads, 0, s>>>(y, ysh, w, T, k, H, res, out, xnext);
    return cudaGetLastError();
}
