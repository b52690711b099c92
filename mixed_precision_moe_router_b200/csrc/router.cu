// Router: logits GEMV over the expert table, then a warp-level softmax/top-k.
//
// [P1] "a small dictionary before we start": each layer has 512 experts and a
// router picks the best 10 for each word.  [P5] "What the model actually is":
// 10 routed plus 1 shared expert per token.  Selection order is (logit desc,
// id asc); weights are the softmax restricted to the chosen k, renormalised.
#include <float.h>

#include "common.cuh"
#include "route_cta.cuh"

namespace moe {

// Stage nt tokens of x (bf16 rows of H) into shared memory, 16 bytes a thread.
__device__ __forceinline__ void stage_tokens(const uint16_t *x, int nt, int vec_per_row, uint16_t *xs) {
    for (int i = threadIdx.x; i < nt * vec_per_row; i += blockDim.x) {
        const int t = i / vec_per_row, c = i - t * vec_per_row;
        reinterpret_cast<uint4 *>(xs)[t * vec_per_row + c] = reinterpret_cast<const uint4 *>(x)[t * vec_per_row + c];
    }
}

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
    stage_tokens(x + static_cast<size_t>(t0) * H, nt, vec_per_row, xs);
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int e = blockIdx.x * kRouterWarps + warp;
    if (e >= E) return;
    float acc[kRouterTokTile];
    const float b = bias ? bias[e] : 0.f;
    expert_dots(xs, wr + static_cast<size_t>(e) * H, nt, vec_per_row, acc);
#pragma unroll
    for (int t = 0; t < kRouterTokTile; ++t) {
        if (t < nt) {
            const float v = warp_sum(acc[t]);
            if (lane == 0) logits[static_cast<size_t>(t0 + t) * E + e] = v + b;
        }
    }
}

// Top-k of one logit row by one warp: k rounds of a warp-wide arg-max over
// the E logits held in registers (NJ per lane), then the renormalised softmax
// over the winners.  Lane j < k returns the j-th choice (id, weight).
template <int NJ>
__device__ __forceinline__ void topk_row(const float *row, int E, int k, int &out_i, float &out_w) {
    const int lane = threadIdx.x & 31;
    float v[NJ];
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
        const int e = lane + 32 * j;
        v[j] = e < E ? __ldcg(row + e) : -FLT_MAX;
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
    out_i = my_i;
    out_w = z / sum;
}

// One warp per token.
template <int NJ>
__global__ void __launch_bounds__(256)
topk_softmax_kernel(const float *__restrict__ logits, int T, int E, int k,
                    int32_t *__restrict__ topk_idx, float *__restrict__ topk_w) {
    const int lane = threadIdx.x & 31;
    const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (t >= T) return;
    int i;
    float w;
    topk_row<NJ>(logits + static_cast<size_t>(t) * E, E, k, i, w);
    if (lane < k) {
        topk_idx[static_cast<size_t>(t) * k + lane] = i;
        topk_w[static_cast<size_t>(t) * k + lane] = w;
    }
}

// ---------------------------------------------------------------------------
// Fused routing for small batches (T <= kRouterTokTile): the logits of every
// expert, computed by all CTAs (one expert per warp), and then, in the CTA
// that finishes last (a ticket counter), the top-k of every token and the
// stable token -> expert grouping of its T*k slots, with the outputs and
// conventions of the top-k and bucketize kernels.  One launch replaces three
// for decode-sized batches.
// ---------------------------------------------------------------------------
constexpr int kRouteWarps = 8;

// Block-wide exclusive scan of one int per thread (kRouteWarps warps).
__device__ __forceinline__ int route_scan(int v, int *warp_tot, int *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    __syncthreads();  // earlier readers of warp_tot are done
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int w = lane < kRouteWarps ? warp_tot[lane] : 0;
        int wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += n;
        }
        if (lane < kRouteWarps) warp_tot[lane] = wi - w;
        if (lane == 31) *total = wi;
    }
    __syncthreads();
    return warp_tot[warp] + incl - v;
}

// Shared memory of the fused kernel: the staged tokens, reused by the
// last CTA for the slot ids [S] and per-expert counts/offsets [E].
__host__ __device__ __forceinline__ size_t route_small_smem(int T, int H, int E, int k) {
    const size_t stage = static_cast<size_t>(T) * H * sizeof(uint16_t);
    const size_t tail = (static_cast<size_t>(T) * k + 2 * static_cast<size_t>(E)) * sizeof(int);
    return stage > tail ? stage : tail;
}

template <int NJ>
__global__ void __launch_bounds__(kRouteWarps * 32)
route_small_kernel(const uint16_t *__restrict__ x, const uint16_t *__restrict__ wr, const float *__restrict__ bias,
                   int T, int H, int E, int k, float *__restrict__ logits, int32_t *__restrict__ topk_idx,
                   float *__restrict__ topk_w, int32_t *__restrict__ offsets, int32_t *__restrict__ sorted_slot,
                   int32_t *__restrict__ slot_pos, int32_t *__restrict__ active, int32_t *status, int *ticket,
                   int *clear, int n_clear) {
    extern __shared__ __align__(16) uint16_t xs[];
    __shared__ int warp_tot[32];
    __shared__ int total_slots, total_active, is_last;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int vec_per_row = H / 8;
    pdl_wait();  // x is the previous kernel's output
    pdl_trigger();
    stage_tokens(x, T, vec_per_row, xs);
    __syncthreads();
    const int e = blockIdx.x * kRouteWarps + warp;
    if (e < E) {
        float acc[kRouterTokTile];
        expert_dots(xs, wr + static_cast<size_t>(e) * H, T, vec_per_row, acc);
        const float b = bias ? bias[e] : 0.f;
#pragma unroll
        for (int t = 0; t < kRouterTokTile; ++t) {
            if (t < T) {
                const float v = warp_sum(acc[t]);
                if (lane == 0) logits[static_cast<size_t>(t) * E + e] = v + b;
            }
        }
    }
    // publish this CTA's logits: every thread's writes, a barrier, then one
    // fence and the ticket
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        is_last = atomicAdd(ticket, 1) == static_cast<int>(gridDim.x) - 1;
    }
    __syncthreads();
    if (!is_last) return;
    __threadfence();
    // top-k of every token (the logit rows are read from L2)
    const int S = T * k;
    int *sid = reinterpret_cast<int *>(xs);  // [S]
    int *cnt = sid + S;                      // [E]
    int *off = cnt + E;                      // [E]
    for (int t = warp; t < T; t += kRouteWarps) {
        int i;
        float w;
        topk_row<NJ>(logits + static_cast<size_t>(t) * E, E, k, i, w);
        if (lane < k) {
            topk_idx[static_cast<size_t>(t) * k + lane] = i;
            topk_w[static_cast<size_t>(t) * k + lane] = w;
            sid[t * k + lane] = i;
        }
    }
    for (int i = threadIdx.x; i < E; i += blockDim.x) cnt[i] = 0;
    for (int i = threadIdx.x; i < n_clear; i += blockDim.x) clear[i] = 0;
    __syncthreads();
    bool bad = false;
    for (int s = threadIdx.x; s < S; s += blockDim.x) {
        const int id = sid[s];
        if (id >= 0 && id < E) atomicAdd(&cnt[id], 1);
        else bad = true;
    }
    if (__syncthreads_or(bad) && threadIdx.x == 0) status_or(status, MOE_STATUS_BAD_EXPERT_ID);
    // offsets and the active list: each thread scans a run of consecutive experts
    const int per = (E + blockDim.x - 1) / blockDim.x;
    const int e0 = min(E, static_cast<int>(threadIdx.x) * per), e1 = min(E, e0 + per);
    int run = 0, nact = 0;
    for (int i = e0; i < e1; ++i) {
        run += cnt[i];
        nact += cnt[i] > 0;
    }
    int base = route_scan(run, warp_tot, &total_slots);
    int abase = route_scan(nact, warp_tot, &total_active);
    for (int i = e0; i < e1; ++i) {
        off[i] = base;
        offsets[i] = base;
        base += cnt[i];
        if (cnt[i] > 0) active[1 + abase++] = i;
    }
    if (threadIdx.x == 0) {
        offsets[E] = total_slots;
        active[0] = total_active;
        *ticket = 0;  // ready for the next launch on this workspace
    }
    __syncthreads();
    // placement: a slot's rank among the earlier slots of its expert
    for (int s = threadIdx.x; s < S; s += blockDim.x) {
        const int id = sid[s];
        int p = -1;
        if (id >= 0 && id < E) {
            int rank = 0;
            for (int u = 0; u < s; ++u) rank += sid[u] == id;
            p = off[id] + rank;
            sorted_slot[p] = s;
        }
        slot_pos[s] = p;
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

// The fused kernel serves batches of up to 16 tokens whose staged rows fit in
// the configured shared memory.
bool moe_route_small_supported(int T, int H, int E, int k) {
    return T >= 1 && T <= moe::kRouterTokTile && moe::route_small_smem(T, H, E, k) <= 200 * 1024;
}

cudaError_t moe_configure_route_small() {
    cudaError_t e = cudaSuccess;
    const int lim = 200 * 1024;
    if (e == cudaSuccess) e = cudaFuncSetAttribute(moe::route_small_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, lim);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(moe::route_small_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, lim);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(moe::route_small_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize, lim);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(moe::route_small_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize, lim);
    return e;
}

// ticket: one int, zero on entry (left zero on exit).  clear[0, n_clear) is
// zeroed before the kernel ends (the caller's next kernel may rely on it).
cudaError_t moe_launch_route_small(const uint16_t *x, const uint16_t *wr, const float *bias, int T, int H, int E,
                                   int k, float *logits, int32_t *idx, float *w, int32_t *offsets, int32_t *sorted,
                                   int32_t *pos, int32_t *active, int32_t *status, int *ticket, int *clear,
                                   int n_clear, cudaStream_t s) {
    const size_t smem = moe::route_small_smem(T, H, E, k);
    const int grid = (E + moe::kRouteWarps - 1) / moe::kRouteWarps;
    const int threads = moe::kRouteWarps * 32;
    const int nj = (E + 31) / 32;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    moe::PdlAttrs at;
    cfg.attrs = at.a;
    cfg.numAttrs = at.n;
#define MOE_ROUTE_ARGS x, wr, bias, T, H, E, k, logits, idx, w, offsets, sorted, pos, active, status, ticket, clear, n_clear
    cudaError_t e;
    if (nj <= 4) e = cudaLaunchKernelEx(&cfg, moe::route_small_kernel<4>, MOE_ROUTE_ARGS);
    else if (nj <= 8) e = cudaLaunchKernelEx(&cfg, moe::route_small_kernel<8>, MOE_ROUTE_ARGS);
    else if (nj <= 16) e = cudaLaunchKernelEx(&cfg, moe::route_small_kernel<16>, MOE_ROUTE_ARGS);
    else e = cudaLaunchKernelEx(&cfg, moe::route_small_kernel<32>, MOE_ROUTE_ARGS);
#undef MOE_ROUTE_ARGS
    return e;
}
