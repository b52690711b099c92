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
// Top-k of one logit row by one warp with warp-wide reductions: lane l holds
// logits l, l+32, ... (16 for E <= 512, 32 for E <= 1024); each of the k
// rounds takes every lane's best untaken value, the warp maximum of an
// order-preserving 32-bit key of the logit (redux.sync) and, among the lanes
// holding that maximum, the lowest id.  Lane r < k returns choice r and its
// renormalised softmax weight, with the same arithmetic as topk_row.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t order_key(float v) {
    const uint32_t u = __float_as_uint(v);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// The float whose order_key is `key`.
__device__ __forceinline__ float key_value(uint32_t key) {
    return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}

// The k rounds on keys already held by the lanes (entry lane + 32 j in
// key[j], 0 for none); the position of choice r is returned in lane r.
template <int NJ>
__device__ __forceinline__ void warp_topk_rounds(uint32_t (&key)[NJ], int k, int &out_i, float &out_w) {
    const int lane = threadIdx.x & 31;
    float my_v = 0.f;
    int my_i = 0;
    for (int r = 0; r < k; ++r) {
        // this lane's best untaken entry, the largest key then the lowest id:
        // up to 16 keys by a tree over adjacent pairs (a left subtree holds
        // the lower ids), more by one pass (fewer registers)
        uint32_t bk = 0u;
        int bj = 0;
        if constexpr (NJ <= 16) {
            uint32_t kk[NJ];
            int jj[NJ];
#pragma unroll
            for (int j = 0; j < NJ; ++j) {
                kk[j] = key[j];
                jj[j] = j;
            }
#pragma unroll
            for (int s = 1; s < NJ; s *= 2)
#pragma unroll
                for (int m = 0; m + s < NJ; m += 2 * s)
                    if (kk[m + s] > kk[m]) {
                        kk[m] = kk[m + s];
                        jj[m] = jj[m + s];
                    }
            bk = kk[0];
            bj = jj[0];
        } else {
#pragma unroll
            for (int j = 0; j < NJ; ++j)
                if (key[j] > bk) {
                    bk = key[j];
                    bj = j;
                }
        }
        const uint32_t wk = __reduce_max_sync(0xffffffffu, bk);
        const uint32_t id = (bk != 0u && bk == wk) ? static_cast<uint32_t>(lane + 32 * bj) : 0xffffffffu;
        const uint32_t wi = __reduce_min_sync(0xffffffffu, id);
        // the winner's lane marks it taken (a select per key: a conditional
        // store would send the array to local memory)
        const int wj = static_cast<int>(wi & 31u) == lane ? static_cast<int>(wi >> 5) : -1;
#pragma unroll
        for (int j = 0; j < NJ; ++j) key[j] = j == wj ? 0u : key[j];
        if (lane == r) {  // the value from its key: no load in the loop
            my_i = static_cast<int>(wi);
            my_v = key_value(wk);
        }
    }
    const float l0 = __shfl_sync(0xffffffffu, my_v, 0);
    const float z = lane < k ? expf(my_v - l0) : 0.f;
    const float sum = warp_sum(z);
    out_i = my_i;
    out_w = z / sum;
}

template <int NJ>
__device__ __forceinline__ void warp_topk_redux(const float *row, int E, int k, int &out_i, float &out_w) {
    const int lane = threadIdx.x & 31;
    // key 0 marks an entry out of range or already taken (no float maps to 0
    // but a NaN with every bit set)
    uint32_t key[NJ];
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
        const int e = lane + 32 * j;
        key[j] = e < E ? order_key(__ldcg(row + e) + 0.0f) : 0u;  // -0 keys as +0
    }
    warp_topk_rounds<NJ>(key, k, out_i, out_w);
}

// Top-k of one row, first stage, by every warp of the CTA: warp w ranks the
// 32 logits of each chunk c = w, w + warps, ... (ids 32c .. 32c + 31, one per
// lane) and keeps its k best as candidates c * k .. c * k + k - 1, in rank
// order (equal keys lowest id first; key 0 and id -1 past the chunk's
// entries).  A row's top k are among its chunks' candidates, and because the
// chunks follow the ids, a lower candidate position among equal keys is a
// lower id: warp_topk_rounds over the candidate keys, with positions for ids,
// then makes exactly the choices warp_topk_redux makes over the whole row.
// k <= 31.
__device__ __forceinline__ void cta_topk_candidates(const float *row, int E, int k, uint32_t *ckey, int *cid) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    const int nc = (E + 31) / 32;
    for (int c = warp; c < nc; c += nw) {
        const int e = 32 * c + lane;
        uint32_t key = e < E ? order_key(__ldcg(row + e) + 0.0f) : 0u;  // -0 keys as +0
        for (int r = 0; r < k; ++r) {
            const uint32_t wk = __reduce_max_sync(0xffffffffu, key);
            // the ids rise with the lane: the lowest lane holding the maximum
            // has the lowest id (-1 when no entry is left)
            const unsigned m = __ballot_sync(0xffffffffu, key != 0u && key == wk);
            const int wl = m ? __ffs(m) - 1 : -1;
            if (lane == r) {
                ckey[c * k + r] = wk;
                cid[c * k + r] = wl >= 0 ? 32 * c + wl : -1;
            }
            if (lane == wl) key = 0u;
        }
    }
}

// Top-k of T rows by a whole CTA: one warp per row (E <= 1024, k <= 32).
// idx_s / w_s [T][k]; ends with a barrier.
__device__ __forceinline__ void cta_topk_rows(const float *logits, int T, int E, int k, int *idx_s, float *w_s) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
    for (int t = warp; t < T; t += nwarps) {
        int i;
        float w;
        if (E <= 512) warp_topk_redux<16>(logits + static_cast<size_t>(t) * E, E, k, i, w);
        else warp_topk_redux<32>(logits + static_cast<size_t>(t) * E, E, k, i, w);
        if (lane < k) {
            idx_s[t * k + lane] = i;
            w_s[t * k + lane] = w;
        }
    }
    __syncthreads();
}

// ---------------------------------------------------------------------------
// Router logits of experts [e0, e1) for T <= NT tokens by a whole CTA: each
// warp takes (expert, quarter of the row) tasks, so one round of row loads
// covers the CTA's share; the quarters are added in order afterwards.
//   x_s bf16 [T][H] in shared memory; part: 4 * (e1 - e0) * NT floats of
//   shared scratch; logits fp32 [T][E] (global).  Ends with a barrier.
// ---------------------------------------------------------------------------
// rows: the router rows e0 .. e1 - 1 (row e0 at rows[0]), in global memory or,
// with SMEM, staged in shared memory; the values and their order of use are
// the same either way.
template <int NT, bool SMEM>
__device__ __forceinline__ void cta_logits_nt(const uint16_t *x_s, int T, int H, int E, const uint16_t *rows,
                                              const float *bias, int e0, int e1, float *part, float *logits) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
    const int vec = H / 8, qv = vec / 4;  // 16-byte chunks per row and per quarter
    const int ntask = 4 * (e1 - e0);
    for (int task = warp; task < ntask; task += nwarps) {
        const int el = task >> 2, q = task & 3;
        const uint16_t *row = rows + static_cast<size_t>(el) * H;
        float acc[NT];
#pragma unroll
        for (int t = 0; t < NT; ++t) acc[t] = 0.f;
        for (int c0 = q * qv; c0 < (q + 1) * qv; c0 += 32 * 4) {
            uint4 wv[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int c = c0 + lane + 32 * u;
                wv[u] = c < (q + 1) * qv ? (SMEM ? *reinterpret_cast<const uint4 *>(row + 8 * c) : ld_stream_v4(row + 8 * c))
                                         : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int c = c0 + lane + 32 * u;
                if (c >= (q + 1) * qv) continue;
                const float w[8] = {bf16lo(wv[u].x), bf16hi(wv[u].x), bf16lo(wv[u].y), bf16hi(wv[u].y),
                                    bf16lo(wv[u].z), bf16hi(wv[u].z), bf16lo(wv[u].w), bf16hi(wv[u].w)};
#pragma unroll
                for (int t = 0; t < NT; ++t) {
                    if (t < T) {
                        const uint4 xv = reinterpret_cast<const uint4 *>(x_s)[t * vec + c];
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
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            const float v = warp_sum(acc[t]);
            if (lane == 0) part[(el * 4 + q) * NT + t] = v;
        }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < (e1 - e0) * T; i += blockDim.x) {
        const int el = i / T, t = i - el * T;
        const float *pp = part + el * 4 * NT + t;
        const float v = ((pp[0] + pp[NT]) + pp[2 * NT]) + pp[3 * NT];
        logits[static_cast<size_t>(t) * E + e0 + el] = v + (bias ? bias[e0 + el] : 0.f);
    }
}

__host__ __device__ __forceinline__ int cta_logits_nt_for(int T) { return T <= 1 ? 1 : (T <= 2 ? 2 : (T <= 4 ? 4 : (T <= 8 ? 8 : 16))); }

// wr_s: this CTA's rows staged in shared memory, or null to read wr.
__device__ __forceinline__ void cta_logits(const uint16_t *x_s, int T, int H, int E, const uint16_t *wr,
                                           const uint16_t *wr_s, const float *bias, int e0, int e1, float *part,
                                           float *logits) {
    const uint16_t *rows = wr + static_cast<size_t>(e0) * H;
    if (wr_s) {
        switch (cta_logits_nt_for(T)) {
            case 1: cta_logits_nt<1, true>(x_s, T, H, E, wr_s, bias, e0, e1, part, logits); break;
            case 2: cta_logits_nt<2, true>(x_s, T, H, E, wr_s, bias, e0, e1, part, logits); break;
            case 4: cta_logits_nt<4, true>(x_s, T, H, E, wr_s, bias, e0, e1, part, logits); break;
            case 8: cta_logits_nt<8, true>(x_s, T, H, E, wr_s, bias, e0, e1, part, logits); break;
            default: cta_logits_nt<16, true>(x_s, T, H, E, wr_s, bias, e0, e1, part, logits); break;
        }
        return;
    }
    switch (cta_logits_nt_for(T)) {
        case 1: cta_logits_nt<1, false>(x_s, T, H, E, rows, bias, e0, e1, part, logits); break;
        case 2: cta_logits_nt<2, false>(x_s, T, H, E, rows, bias, e0, e1, part, logits); break;
        case 4: cta_logits_nt<4, false>(x_s, T, H, E, rows, bias, e0, e1, part, logits); break;
        case 8: cta_logits_nt<8, false>(x_s, T, H, E, rows, bias, e0, e1, part, logits); break;
        default: cta_logits_nt<16, false>(x_s, T, H, E, rows, bias, e0, e1, part, logits); break;
    }
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
