// Routing building blocks shared by the routing kernels and by the expert
// FFN kernel when it routes a small batch itself.
//
// [P1] "a small dictionary before we start": each layer has 512 experts and a
// router picks the best 10 for each word; selection order is (logit desc,
// id asc) and the weights are the softmax restricted to the chosen k,
// renormalised.
#pragma once
#include <float.h>

#include "common.cuh"

namespace moe {

constexpr int kRouterTokTile = 16;   // tokens staged in shared memory per CTA
constexpr int kRouterWarps = 4;      // one expert per warp

// Dot products of one expert row with the nt (<= kRouterTokTile) tokens staged
// in xs, by one warp: lane-strided 8-element chunks and an fma chain per token
// (per-lane partial sums; the caller adds them with warp_sum).  Every routing
// kernel below uses this one function, so a logit has the same bits whichever
// kernel computed it.
__device__ __forceinline__ void expert_dots(const uint16_t *xs, const uint16_t *wrow, int nt, int vec_per_row,
                                            float (&acc)[kRouterTokTile]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int t = 0; t < kRouterTokTile; ++t) acc[t] = 0.f;
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
}

// Is (va, ia) ranked before (vb, ib)?  Larger logit first, then lower id.
__device__ __forceinline__ bool ranks_before(float va, int ia, float vb, int ib) {
    return va > vb || (va == vb && ia < ib);
}

// ---------------------------------------------------------------------------
// Top-k of T logit rows by a whole CTA.  Each row is cut into quarters of
// 128 logits (4 per lane); a warp finds a quarter's top-k by k rounds of a
// warp arg-max, then one warp per row merges the quarters' candidates the
// same way.  Ties go to the lower id at every stage, so the result is the
// top-k of the whole row in (logit desc, id asc) order.
// ---------------------------------------------------------------------------
constexpr int kTopkQuarter = 128;

// Shared memory for cta_topk: candidates [T][quarters][k] as (value, id).
__host__ __device__ __forceinline__ size_t cta_topk_smem(int T, int E, int k) {
    const int nq = (E + kTopkQuarter - 1) / kTopkQuarter;
    return static_cast<size_t>(T) * nq * k * (sizeof(float) + sizeof(int));
}

// k rounds of a warp arg-max over NJ values per lane (v, id), skipping the
// ones already taken; lane r < k returns choice r.
template <int NJ>
__device__ __forceinline__ void warp_topk(const float (&v)[NJ], const int (&id)[NJ], int k, float &out_v,
                                          int &out_i) {
    const int lane = threadIdx.x & 31;
    uint32_t taken = 0;
    out_v = -FLT_MAX;
    out_i = 0x7fffffff;
    for (int r = 0; r < k; ++r) {
        float bv = -FLT_MAX;
        int bi = 0x7fffffff, bj = -1;
#pragma unroll
        for (int j = 0; j < NJ; ++j)
            if (!((taken >> j) & 1u) && id[j] != 0x7fffffff && ranks_before(v[j], id[j], bv, bi)) {
                bv = v[j];
                bi = id[j];
                bj = j;
            }
        float wv = bv;
        int wi = bi;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, wv, o);
            const int oi = __shfl_xor_sync(0xffffffffu, wi, o);
            if (ranks_before(ov, oi, wv, wi)) {
                wv = ov;
                wi = oi;
            }
        }
        if (bj >= 0 && bi == wi) taken |= 1u << bj;  // ids are unique: only the owner matches
        if (lane == r) {
            out_v = wv;
            out_i = wi;
        }
    }
}

// Every thread of the CTA calls it.  logits fp32 [T][E] (read through L2);
// on return (after a barrier) idx_s / w_s [T][k] hold each row's choices and
// their renormalised softmax weights, bit-identical to the top-k kernels.
__device__ __forceinline__ void cta_topk(const float *logits, int T, int E, int k, void *scratch, int *idx_s,
                                         float *w_s) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
    const int nq = (E + kTopkQuarter - 1) / kTopkQuarter;
    float *cv = static_cast<float *>(scratch);
    int *ci = reinterpret_cast<int *>(cv + T * nq * k);
    for (int task = warp; task < T * nq; task += nwarps) {
        const int t = task / nq, q = task - t * nq;
        float v[4];
        int id[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int e = q * kTopkQuarter + lane + 32 * j;
            v[j] = e < E ? __ldcg(logits + static_cast<size_t>(t) * E + e) : -FLT_MAX;
            id[j] = e < E ? e : 0x7fffffff;
        }
        float ov;
        int oi;
        warp_topk<4>(v, id, k, ov, oi);
        if (lane < k) {
            cv[(t * nq + q) * k + lane] = ov;
            ci[(t * nq + q) * k + lane] = oi;
        }
    }
    __syncthreads();
    for (int t = warp; t < T; t += nwarps) {
        // at most 8 quarters (E <= 1024) x k <= 32 candidates: 8 per lane
        float v[8];
        int id[8];
        const int nc = nq * k;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int c = lane + 32 * j;
            v[j] = c < nc ? cv[t * nc + c] : -FLT_MAX;
            id[j] = c < nc ? ci[t * nc + c] : 0x7fffffff;
        }
        float my_v;
        int my_i;
        warp_topk<8>(v, id, k, my_v, my_i);
        const float l0 = __shfl_sync(0xffffffffu, my_v, 0);
        const float z = lane < k ? expf(my_v - l0) : 0.f;
        const float sum = warp_sum(z);
        if (lane < k) {
            idx_s[t * k + lane] = my_i;
            w_s[t * k + lane] = z / sum;
        }
    }
    __syncthreads();
}

// ---------------------------------------------------------------------------
// Stable token -> expert grouping of the S = T*k slots by a whole CTA
// (S <= blockDim; every id in [0, E), as the top-k produces them):
//   srt[p]  the slot at sorted position p (expert ascending, then slot)
//   pos[s]  the inverse: srt[pos[s]] == s
//   act[0]  the number of active experts, act[1 + a] their ids ascending
//   off[e]  the first sorted position of expert e (E + 1 entries)
// tmp: 32 ints of scratch.  Every thread calls it; ends with a barrier.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void cta_group(const int *idx_s, int S, int E, int *srt, int *pos, int *act, int *off,
                                          int *tmp) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
    if (tid < S) {
        const int e = idx_s[tid];
        int rank = 0;
        for (int u = 0; u < S; ++u) {
            const int eu = idx_s[u];
            rank += eu < e || (eu == e && u < tid);
        }
        srt[rank] = tid;
        pos[tid] = rank;
    }
    __syncthreads();
    // runs of one expert in sorted order: their starts, counted in order
    const int ep = tid < S ? idx_s[srt[tid]] : -1;
    const bool start = tid < S && (tid == 0 || ep != idx_s[srt[tid - 1]]);
    const unsigned m = __ballot_sync(0xffffffffu, start);
    if (lane == 0) tmp[warp] = __popc(m);
    __syncthreads();
    if (warp == 0) {
        const int v = lane < nwarps ? tmp[lane] : 0;
        int incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += n;
        }
        if (lane < nwarps) tmp[lane] = incl - v;
        if (lane == 31) act[0] = incl;
    }
    __syncthreads();
    if (start) act[1 + tmp[warp] + __popc(m & ((1u << lane) - 1u))] = ep;
    // off[e]: the first sorted position whose expert is >= e
    for (int e = tid; e <= E; e += blockDim.x) {
        int lo = 0, hi = S;
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (idx_s[srt[mid]] < e) lo = mid + 1;
            else hi = mid;
        }
        off[e] = lo;
    }
    __syncthreads();
}

}  // namespace moe
