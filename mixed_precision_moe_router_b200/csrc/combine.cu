// Combine: out[t] = bf16(sum_j w[t,j] * y[t*k+j] + y_shared[t]), fixed order;
// optional residual stream x_next = bf16(residual + out) and its RMS-normalised
// copy n_next = bf16(x_next / sqrt(mean(x_next^2) + eps)), the next layer's input.
//
// [P1] "step 4: three shelves, all on the GPU": the per-shelf results simply
// add up; with one shared expert always on ([P5] "What the model actually is").
#include "common.cuh"

namespace moe {

constexpr int kCombineThreads = 512;

__device__ __forceinline__ float block_sum(float v, float *red) {
    v = warp_sum(v);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float s = 0.f;
    if (threadIdx.x < 32) {
        s = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
        s = warp_sum(s);
        if (threadIdx.x == 0) red[0] = s;
    }
    __syncthreads();
    return red[0];
}

__device__ __forceinline__ uint2 pack4(uint16_t a, uint16_t b, uint16_t c, uint16_t d) {
    return make_uint2(static_cast<uint32_t>(a) | (static_cast<uint32_t>(b) << 16),
                      static_cast<uint32_t>(c) | (static_cast<uint32_t>(d) << 16));
}

__device__ __forceinline__ void fma4(float4 &a, float w, const float4 &v) {
    a.x = fmaf(w, v.x, a.x);
    a.y = fmaf(w, v.y, a.y);
    a.z = fmaf(w, v.z, a.z);
    a.w = fmaf(w, v.w, a.w);
}

// One CTA per token; each thread owns 4-element chunks c = threadIdx.x + i*blockDim.
// The k slot rows of a chunk are loaded eight at a time (independent loads in
// flight) and added in slot order j = 0 .. k-1; the new residual values stay
// in registers for the RMS norm (up to kKeep chunks per thread).
constexpr int kKeep = 4;

// out / x_next of one 4-element chunk; returns the x_next values (fp32).
__device__ __forceinline__ float4 combine_chunk(const float4 *yt, const float *ysh, const float *ws, int k, int chunks,
                                                int c, size_t row, const uint16_t *res, uint16_t *out,
                                                uint16_t *xnext) {
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j0 = 0; j0 < k; j0 += 8) {
        float4 v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
            if (j0 + u < k) v[u] = __ldcg(yt + static_cast<size_t>(j0 + u) * chunks + c);
#pragma unroll
        for (int u = 0; u < 8; ++u)
            if (j0 + u < k) fma4(a, ws[j0 + u], v[u]);
    }
    if (ysh) {
        const float4 v = __ldcg(reinterpret_cast<const float4 *>(ysh + row) + c);
        a.x += v.x; a.y += v.y; a.z += v.z; a.w += v.w;
    }
    const uint16_t o0 = f32_to_bf16_rne(a.x), o1 = f32_to_bf16_rne(a.y);
    const uint16_t o2 = f32_to_bf16_rne(a.z), o3 = f32_to_bf16_rne(a.w);
    if (out) *reinterpret_cast<uint2 *>(out + row + 4 * c) = pack4(o0, o1, o2, o3);
    if (!res) return make_float4(0.f, 0.f, 0.f, 0.f);
    const uint2 r = *reinterpret_cast<const uint2 *>(res + row + 4 * c);
    const uint16_t n0 = f32_to_bf16_rne(bf16lo(r.x) + bf16_to_f32(o0));
    const uint16_t n1 = f32_to_bf16_rne(bf16hi(r.x) + bf16_to_f32(o1));
    const uint16_t n2 = f32_to_bf16_rne(bf16lo(r.y) + bf16_to_f32(o2));
    const uint16_t n3 = f32_to_bf16_rne(bf16hi(r.y) + bf16_to_f32(o3));
    *reinterpret_cast<uint2 *>(xnext + row + 4 * c) = pack4(n0, n1, n2, n3);
    return make_float4(bf16_to_f32(n0), bf16_to_f32(n1), bf16_to_f32(n2), bf16_to_f32(n3));
}

__device__ __forceinline__ void ss4(float &ss, const float4 &f) {
    ss = fmaf(f.x, f.x, fmaf(f.y, f.y, fmaf(f.z, f.z, fmaf(f.w, f.w, ss))));
}

__device__ __forceinline__ void norm_chunk(uint16_t *nnext, size_t row, int c, const float4 &f, float rinv) {
    *reinterpret_cast<uint2 *>(nnext + row + 4 * c) =
        pack4(f32_to_bf16_rne(f.x * rinv), f32_to_bf16_rne(f.y * rinv), f32_to_bf16_rne(f.z * rinv),
              f32_to_bf16_rne(f.w * rinv));
}

__global__ void __launch_bounds__(kCombineThreads)
combine_kernel(const float *__restrict__ y, const float *__restrict__ ysh, const float *__restrict__ w,
               int T, int k, int H, const uint16_t *__restrict__ res, uint16_t *__restrict__ out,
               uint16_t *__restrict__ xnext, uint16_t *__restrict__ nnext, float eps) {
    __shared__ float red[32];
    __shared__ float ws[MOE_MAX_TOPK];
    pdl_wait();
    pdl_trigger();
    const int t = blockIdx.x;
    const int chunks = H / 4;
    const size_t row = static_cast<size_t>(t) * H;
    if (threadIdx.x < k) ws[threadIdx.x] = w[static_cast<size_t>(t) * k + threadIdx.x];
    __syncthreads();
    const float4 *yt = reinterpret_cast<const float4 *>(y + static_cast<size_t>(t) * k * H);
    const int stride = blockDim.x;
    float ss = 0.f;
    float4 keep[kKeep];
#pragma unroll
    for (int q = 0; q < kKeep; ++q) {
        const int c = threadIdx.x + q * stride;
        keep[q] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (c < chunks) {
            keep[q] = combine_chunk(yt, ysh, ws, k, chunks, c, row, res, out, xnext);
            ss4(ss, keep[q]);
        }
    }
    for (int c = threadIdx.x + kKeep * stride; c < chunks; c += stride)
        ss4(ss, combine_chunk(yt, ysh, ws, k, chunks, c, row, res, out, xnext));
    if (!res || !nnext) return;  // uniform across the CTA
    const float tot = block_sum(ss, red);
    const float rinv = 1.0f / sqrtf(tot / static_cast<float>(H) + eps);
#pragma unroll
    for (int q = 0; q < kKeep; ++q) {
        const int c = threadIdx.x + q * stride;
        if (c < chunks) norm_chunk(nnext, row, c, keep[q], rinv);
    }
    for (int c = threadIdx.x + kKeep * stride; c < chunks; c += stride) {
        const uint2 v = *reinterpret_cast<const uint2 *>(xnext + row + 4 * c);
        norm_chunk(nnext, row, c, make_float4(bf16lo(v.x), bf16hi(v.x), bf16lo(v.y), bf16hi(v.y)), rinv);
    }
}

// n = bf16(x / sqrt(mean(x^2) + eps)), one CTA per token.
__global__ void __launch_bounds__(kCombineThreads)
rmsnorm_kernel(const uint16_t *__restrict__ x, int H, float eps, uint16_t *__restrict__ n) {
    __shared__ float red[32];
    pdl_wait();
    pdl_trigger();
    const size_t row = static_cast<size_t>(blockIdx.x) * H;
    const int chunks = H / 4;
    float ss = 0.f;
    for (int c = threadIdx.x; c < chunks; c += blockDim.x) {
        const uint2 v = *reinterpret_cast<const uint2 *>(x + row + 4 * c);
        const float f0 = bf16lo(v.x), f1 = bf16hi(v.x), f2 = bf16lo(v.y), f3 = bf16hi(v.y);
        ss = fmaf(f0, f0, fmaf(f1, f1, fmaf(f2, f2, fmaf(f3, f3, ss))));
    }
    const float tot = block_sum(ss, red);
    const float rinv = 1.0f / sqrtf(tot / static_cast<float>(H) + eps);
    for (int c = threadIdx.x; c < chunks; c += blockDim.x) {
        const uint2 v = *reinterpret_cast<const uint2 *>(x + row + 4 * c);
        *reinterpret_cast<uint2 *>(n + row + 4 * c) =
            pack4(f32_to_bf16_rne(bf16lo(v.x) * rinv), f32_to_bf16_rne(bf16hi(v.x) * rinv),
                  f32_to_bf16_rne(bf16lo(v.y) * rinv), f32_to_bf16_rne(bf16hi(v.y) * rinv));
    }
}

}  // namespace moe

cudaError_t moe_launch_combine(const float *y, const float *ysh, const float *w, int T, int k, int H,
                               const uint16_t *res, uint16_t *out, uint16_t *xnext, uint16_t *nnext,
                               cudaStream_t s) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(T);
    cfg.blockDim = dim3(moe::kCombineThreads);
    cfg.stream = s;
    moe::PdlAttrs at;
    cfg.attrs = at.a;
    cfg.numAttrs = at.n;
    return cudaLaunchKernelEx(&cfg, moe::combine_kernel, y, ysh, w, T, k, H, res, out, xnext, nnext, MOE_NORM_EPS);
}

cudaError_t moe_launch_rmsnorm(const uint16_t *x, int T, int H, uint16_t *n, cudaStream_t s) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(T);
    cfg.blockDim = dim3(moe::kCombineThreads);
    cfg.stream = s;
    moe::PdlAttrs at;
    cfg.attrs = at.a;
    cfg.numAttrs = at.n;
    return cudaLaunchKernelEx(&cfg, moe::rmsnorm_kernel, x, H, MOE_NORM_EPS, n);
}
