// Tiered expert FFN, GEMV path (decode-sized token groups).
//
// [P1] "step 4: three shelves, all on the GPU": mul_mat_id runs each word
// through its chosen experts; each shelf computes only the ids on it and the
// shelf results add up; the decode kernel fuses gate, up and the activation.
// Here one launch walks every shelf: a CTA takes one active expert (whatever
// its shelf) and a slice of its rows, streams those rows once, dequantises
// the 8/4/3-bit blocks in registers (w = d*q exact in fp32) and applies them
// to all of that expert's tokens with fp32 accumulation.
//
//   gate_up kernel: h[s, i] = silu(W_gate[e][i] . x[t]) * (W_up[e][i] . x[t])
//   down kernel:    y[s, n] = W_down[e][n] . h[s]
//
// Row s of h is slot s = t*k + j for routed experts and T*k + t for the
// shared expert.
#include "common.cuh"
#include "ffn.cuh"

namespace moe {

constexpr int kGemvWarps = 8;
constexpr int kGemvThreads = kGemvWarps * 32;
constexpr int kGuPairsPerWarp = 2;   // gate/up row pairs per warp (gate_up)
constexpr int kDnRowsPerCta = 64;    // output rows per CTA (down)

// ---------------------------------------------------------------------------
// One 16-byte unit of packed codes (plus, for 3 bits, its 8-byte high plane):
//   8 bits: 16 weights, 4 bits: 32 weights, 3 bits: 64 weights.
// ---------------------------------------------------------------------------
template <int BITS> struct UnitTraits;
template <> struct UnitTraits<8> { static constexpr int W = 16; };
template <> struct UnitTraits<4> { static constexpr int W = 32; };
template <> struct UnitTraits<3> { static constexpr int W = 64; };

struct UnitRaw {
    uint4 lo;
    uint2 hi;   // 3 bits only
    uint32_t sc; // one (8/4 bits) or two (3 bits) fp16 scales
};

template <int BITS>
__device__ __forceinline__ UnitRaw load_unit(const uint8_t *qs_row, const uint16_t *sc_row, int K, int u) {
    UnitRaw r;
    r.lo = ld_stream_v4(qs_row + 16 * u);
    if constexpr (BITS == 3) {
        r.hi = ld_stream_v2(qs_row + K / 4 + 8 * u);
        r.sc = ld_stream_u32(sc_row + 2 * u);
    } else if constexpr (BITS == 4) {
        r.hi = make_uint2(0, 0);
        r.sc = sc_row[u];
    } else {
        r.hi = make_uint2(0, 0);
        r.sc = sc_row[u >> 1];
    }
    return r;
}

// dot of one unit with one activation vector xs (fp32, in shared memory),
// returning sum_i d*q_i*x_i with the scale applied per block.
template <int BITS, int NT>
__device__ __forceinline__ void unit_dot(const UnitRaw &r, const float *xs, int nt, int stride,
                                         int k0, float (&acc)[NT]) {
    if constexpr (BITS == 8) {
        float w[16];
        s8x4_to_f32(r.lo.x, w);
        s8x4_to_f32(r.lo.y, w + 4);
        s8x4_to_f32(r.lo.z, w + 8);
        s8x4_to_f32(r.lo.w, w + 12);
        const float d = f16_bits_to_f32(static_cast<uint16_t>(r.sc));
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            if (t >= nt) break;
            const float4 *xv = reinterpret_cast<const float4 *>(xs + t * stride + k0);
            float p = 0.f;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float4 v = xv[i];
                p = fmaf(w[4 * i + 0], v.x, p);
                p = fmaf(w[4 * i + 1], v.y, p);
                p = fmaf(w[4 * i + 2], v.z, p);
                p = fmaf(w[4 * i + 3], v.w, p);
            }
            acc[t] = fmaf(d, p, acc[t]);
        }
    } else if constexpr (BITS == 4) {
        float w[32];
        u4x8_to_f32(r.lo.x, w);
        u4x8_to_f32(r.lo.y, w + 8);
        u4x8_to_f32(r.lo.z, w + 16);
        u4x8_to_f32(r.lo.w, w + 24);
        const float d = f16_bits_to_f32(static_cast<uint16_t>(r.sc));
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            if (t >= nt) break;
            const float4 *xv = reinterpret_cast<const float4 *>(xs + t * stride + k0);
            float p = 0.f;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float4 v = xv[i];
                p = fmaf(w[4 * i + 0], v.x, p);
                p = fmaf(w[4 * i + 1], v.y, p);
                p = fmaf(w[4 * i + 2], v.z, p);
                p = fmaf(w[4 * i + 3], v.w, p);
            }
            acc[t] = fmaf(d, p, acc[t]);
        }
    } else {
        float w[64];
        u3x16_to_f32(r.lo.x, r.hi.x & 0xffffu, w);
        u3x16_to_f32(r.lo.y, r.hi.x >> 16, w + 16);
        u3x16_to_f32(r.lo.z, r.hi.y & 0xffffu, w + 32);
        u3x16_to_f32(r.lo.w, r.hi.y >> 16, w + 48);
        const float d0 = f16_bits_to_f32(static_cast<uint16_t>(r.sc & 0xffffu));
        const float d1 = f16_bits_to_f32(static_cast<uint16_t>(r.sc >> 16));
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            if (t >= nt) break;
            const float4 *xv = reinterpret_cast<const float4 *>(xs + t * stride + k0);
            float p0 = 0.f, p1 = 0.f;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float4 v = xv[i];
                p0 = fmaf(w[4 * i + 0], v.x, p0);
                p0 = fmaf(w[4 * i + 1], v.y, p0);
                p0 = fmaf(w[4 * i + 2], v.z, p0);
                p0 = fmaf(w[4 * i + 3], v.w, p0);
            }
#pragma unroll
            for (int i = 8; i < 16; ++i) {
                const float4 v = xv[i];
                p1 = fmaf(w[4 * i + 0], v.x, p1);
                p1 = fmaf(w[4 * i + 1], v.y, p1);
                p1 = fmaf(w[4 * i + 2], v.z, p1);
                p1 = fmaf(w[4 * i + 3], v.w, p1);
            }
            acc[t] = fmaf(d1, p1, fmaf(d0, p0, acc[t]));
        }
    }
}

// Units per row and the lane-group width for a row of K weights.
template <int BITS> __host__ __device__ __forceinline__ int units_per_row(int K) {
    return K / UnitTraits<BITS>::W;
}
__device__ __forceinline__ int group_width(int U) {
    if (U >= 32) return 32;
    int L = 1;
    while (L < U) L <<= 1;
    return L;
}

// Expert id -> the shelf rows it owns.
struct ExpertRef {
    int bits;
    const uint8_t *gu_qs;
    const uint16_t *gu_sc;
    const uint8_t *dn_qs;
    const uint16_t *dn_sc;
};

__device__ __forceinline__ bool find_expert(const FfnParams &p, int e, ExpertRef &ref) {
    const moe_tier *t = nullptr;
    int j = 0;
    if (e == p.E) {
        t = &p.w.shared;
        j = 0;
    } else {
        for (int i = 0; i < p.w.n_tiers; ++i) {
            const moe_tier &ti = p.w.tiers[i];
            if (e >= ti.first_expert && e < ti.first_expert + ti.n_experts) {
                t = &ti;
                j = e - ti.first_expert;
            }
        }
    }
    if (!t) return false;
    const int H = p.w.H, I = p.w.I, b = t->bits;
    ref.bits = b;
    ref.gu_qs = t->gu_qs + static_cast<size_t>(j) * 2 * I * (H * b / 8);
    ref.gu_sc = t->gu_scale + static_cast<size_t>(j) * 2 * I * (H / 32);
    ref.dn_qs = t->dn_qs + static_cast<size_t>(j) * H * (I * b / 8);
    ref.dn_sc = t->dn_scale + static_cast<size_t>(j) * H * (I / 32);
    return true;
}

// Which expert and which tokens a CTA row (blockIdx.y) serves.
struct Assignment {
    int expert;   // routed id, or E for the shared expert
    int count;    // tokens
    int first;    // offset into sorted_slot (routed)
};

__device__ __forceinline__ bool assignment_of(const FfnParams &p, int a, Assignment &as) {
    const int n_active = p.active[0];
    if (a < n_active) {
        const int e = p.active[1 + a];
        if (e < 0 || e >= p.E) return false;
        as.expert = e;
        as.first = p.offsets[e];
        as.count = p.offsets[e + 1] - as.first;
        return as.count > 0;
    }
    if (p.has_shared && a == p.max_active) {
        as.expert = p.E;
        as.first = 0;
        as.count = p.T;
        return p.T > 0;
    }
    return false;
}

// token of the n-th entry and the h/y row it writes
__device__ __forceinline__ void entry(const FfnParams &p, const Assignment &as, int n, int &tok, int &row) {
    if (as.expert == p.E) {
        tok = n;
        row = p.T * p.k + n;
    } else {
        const int s = p.sorted[as.first + n];
        tok = s / p.k;
        row = s;
    }
}

// ---------------------------------------------------------------------------
// gate_up + SwiGLU
// ---------------------------------------------------------------------------
constexpr int kUnitBatch = 4;  // units per lane whose loads are issued together

template <int BITS, int NT>
__device__ __forceinline__ void gate_up_pass(const FfnParams &p, const ExpertRef &ref, const float *xs,
                                             int nt, const int *rows_out, int pair0) {
    const int H = p.w.H, I = p.w.I;
    const int lane = threadIdx.x & 31;
    const int U = units_per_row<BITS>(H);
    const int L = group_width(U);
    const int g = lane / L, sub = lane % L;
    const int per_step = 32 / L;
    const size_t rb = static_cast<size_t>(H) * BITS / 8;
    const int nsc = H / 32;
#pragma unroll 1
    for (int rp = 0; rp < kGuPairsPerWarp; ++rp) {
        const int i = pair0 + rp * per_step + g;
        const bool live = i < I;
        const uint8_t *gq = ref.gu_qs + static_cast<size_t>(i) * rb;
        const uint8_t *uq = ref.gu_qs + static_cast<size_t>(I + i) * rb;
        const uint16_t *gs = ref.gu_sc + static_cast<size_t>(i) * nsc;
        const uint16_t *us = ref.gu_sc + static_cast<size_t>(I + i) * nsc;
        float ag[NT], au[NT];
#pragma unroll
        for (int t = 0; t < NT; ++t) { ag[t] = 0.f; au[t] = 0.f; }
#pragma unroll 1
        for (int u0 = sub; u0 < U; u0 += kUnitBatch * L) {
            UnitRaw rg[kUnitBatch], ru[kUnitBatch];
#pragma unroll
            for (int c = 0; c < kUnitBatch; ++c) {
                const int u = u0 + c * L;
                if (live && u < U) {
                    rg[c] = load_unit<BITS>(gq, gs, H, u);
                    ru[c] = load_unit<BITS>(uq, us, H, u);
                }
            }
#pragma unroll
            for (int c = 0; c < kUnitBatch; ++c) {
                const int u = u0 + c * L;
                if (live && u < U) {
                    unit_dot<BITS, NT>(rg[c], xs, nt, H, u * UnitTraits<BITS>::W, ag);
                    unit_dot<BITS, NT>(ru[c], xs, nt, H, u * UnitTraits<BITS>::W, au);
                }
            }
        }
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            ag[t] = group_sum(ag[t], L);
            au[t] = group_sum(au[t], L);
        }
        if (live && sub == 0) {
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                if (t < nt) {
                    const float gg = ag[t];
                    const float hv = gg / (1.0f + expf(-gg)) * au[t];
                    p.h[static_cast<size_t>(rows_out[t]) * I + i] = hv;
                }
            }
        }
    }
}

template <int NT>
__device__ __forceinline__ void gate_up_dispatch(const FfnParams &p, const ExpertRef &ref,
                                                 const float *xs, int nt, const int *rows_out,
                                                 int pair0) {
    if (ref.bits == 8) gate_up_pass<8, NT>(p, ref, xs, nt, rows_out, pair0);
    else if (ref.bits == 4) gate_up_pass<4, NT>(p, ref, xs, nt, rows_out, pair0);
    else gate_up_pass<3, NT>(p, ref, xs, nt, rows_out, pair0);
}

__device__ __forceinline__ int row_units(int bits, int K) {
    return bits == 8 ? K / 16 : (bits == 4 ? K / 32 : K / 64);
}

// Fill shared memory with the next group of up to NT tokens of the expert.
__device__ __forceinline__ int stage_rows(const FfnParams &p, const Assignment &as, int n0, int ntmax,
                                          int *rows_out, int *toks) {
    const int nt = min(ntmax, as.count - n0);
    __syncthreads();
    if (threadIdx.x < nt) {
        int tok, row;
        entry(p, as, n0 + threadIdx.x, tok, row);
        toks[threadIdx.x] = tok;
        rows_out[threadIdx.x] = row;
    }
    __syncthreads();
    return nt;
}

// grid = (ceil(I / (kGemvWarps * kGuPairsPerWarp)), max_active + has_shared)
template <int NT>
__global__ void __launch_bounds__(kGemvThreads)
ffn_gate_up_gemv_kernel(const FfnParams p) {
    extern __shared__ __align__(16) float xs[];  // [NT][H]
    __shared__ int rows_out[NT];
    __shared__ int toks[NT];
    Assignment as;
    if (!assignment_of(p, blockIdx.y, as)) return;
    ExpertRef ref;
    if (!find_expert(p, as.expert, ref)) {
        if (threadIdx.x == 0) status_or(p.status, MOE_STATUS_BAD_EXPERT_ID);
        return;
    }
    const int H = p.w.H;
    const int warp = threadIdx.x >> 5;
    const int L = group_width(row_units(ref.bits, H));
    const int per_step = 32 / L;
    // narrower rows (small H) let one warp cover several pairs per step
    const int cta_pair0 = blockIdx.x * kGemvWarps * kGuPairsPerWarp * per_step;
    const int pair0 = cta_pair0 + warp * kGuPairsPerWarp * per_step;
    if (cta_pair0 >= p.w.I) return;
    for (int n0 = 0; n0 < as.count; n0 += NT) {
        const int nt = stage_rows(p, as, n0, NT, rows_out, toks);
        const int vec = H / 8;
        for (int q = threadIdx.x; q < nt * vec; q += kGemvThreads) {
            const int t = q / vec, c = q - t * vec;
            const uint4 v = reinterpret_cast<const uint4 *>(p.x + static_cast<size_t>(toks[t]) * H)[c];
            float4 *dst = reinterpret_cast<float4 *>(xs + t * H + c * 8);
            dst[0] = make_float4(bf16lo(v.x), bf16hi(v.x), bf16lo(v.y), bf16hi(v.y));
            dst[1] = make_float4(bf16lo(v.z), bf16hi(v.z), bf16lo(v.w), bf16hi(v.w));
        }
        __syncthreads();
        int rows_local[NT];
#pragma unroll
        for (int t = 0; t < NT; ++t) rows_local[t] = rows_out[t];
        gate_up_dispatch<NT>(p, ref, xs, nt, rows_local, pair0);
    }
}

// ---------------------------------------------------------------------------
// down projection
// ---------------------------------------------------------------------------
template <int BITS, int NT>
__device__ __forceinline__ void down_pass(const FfnParams &p, const ExpertRef &ref, const float *hs,
                                          int nt, const int *rows_out, int row_begin, int row_end) {
    const int H = p.w.H, I = p.w.I;
    const int lane = threadIdx.x & 31;
    const int U = units_per_row<BITS>(I);
    const int L = group_width(U);
    const int g = lane / L, sub = lane % L;
    const int per_step = 32 / L;
    const size_t rb = static_cast<size_t>(I) * BITS / 8;
    const int nsc = I / 32;
    constexpr int RW = 4;  // row-steps whose first units are loaded together
#pragma unroll 1
    for (int r0 = row_begin; r0 < row_end; r0 += RW * per_step) {
        float acc[RW][NT];
#pragma unroll
        for (int rs = 0; rs < RW; ++rs)
#pragma unroll
            for (int t = 0; t < NT; ++t) acc[rs][t] = 0.f;
#pragma unroll 1
        for (int u = sub; u < U; u += L) {
            UnitRaw ur[RW];
#pragma unroll
            for (int rs = 0; rs < RW; ++rs) {
                const int n = r0 + rs * per_step + g;
                if (n < row_end)
                    ur[rs] = load_unit<BITS>(ref.dn_qs + static_cast<size_t>(n) * rb,
                                             ref.dn_sc + static_cast<size_t>(n) * nsc, I, u);
            }
#pragma unroll
            for (int rs = 0; rs < RW; ++rs) {
                const int n = r0 + rs * per_step + g;
                if (n < row_end) unit_dot<BITS, NT>(ur[rs], hs, nt, I, u * UnitTraits<BITS>::W, acc[rs]);
            }
        }
#pragma unroll
        for (int rs = 0; rs < RW; ++rs) {
            const int n = r0 + rs * per_step + g;
#pragma unroll
            for (int t = 0; t < NT; ++t) acc[rs][t] = group_sum(acc[rs][t], L);
            if (n < row_end && sub == 0) {
#pragma unroll
                for (int t = 0; t < NT; ++t) {
                    if (t < nt) {
                        const int row = rows_out[t];
                        float *dst = row >= p.T * p.k ? p.y_shared + static_cast<size_t>(row - p.T * p.k) * H
                                                      : p.y_slots + static_cast<size_t>(row) * H;
                        dst[n] = acc[rs][t];
                    }
                }
            }
        }
    }
}

template <int NT>
__device__ __forceinline__ void down_dispatch(const FfnParams &p, const ExpertRef &ref, const float *hs,
                                              int nt, const int *rows_out, int rb, int re) {
    if (ref.bits == 8) down_pass<8, NT>(p, ref, hs, nt, rows_out, rb, re);
    else if (ref.bits == 4) down_pass<4, NT>(p, ref, hs, nt, rows_out, rb, re);
    else down_pass<3, NT>(p, ref, hs, nt, rows_out, rb, re);
}

// grid = (ceil(H / kDnRowsPerCta), max_active + has_shared)
template <int NT>
__global__ void __launch_bounds__(kGemvThreads)
ffn_down_gemv_kernel(const FfnParams p) {
    extern __shared__ __align__(16) float hs[];  // [NT][I]
    __shared__ int rows_out[NT];
    __shared__ int toks[NT];
    Assignment as;
    if (!assignment_of(p, blockIdx.y, as)) return;
    ExpertRef ref;
    if (!find_expert(p, as.expert, ref)) return;
    const int I = p.w.I, H = p.w.H;
    const int warp = threadIdx.x >> 5;
    const int rows_per_warp = kDnRowsPerCta / kGemvWarps;
    const int rb = blockIdx.x * kDnRowsPerCta + warp * rows_per_warp;
    const int re = min(H, rb + rows_per_warp);
    for (int n0 = 0; n0 < as.count; n0 += NT) {
        const int nt = stage_rows(p, as, n0, NT, rows_out, toks);
        const int vec = I / 4;
        for (int q = threadIdx.x; q < nt * vec; q += kGemvThreads) {
            const int t = q / vec, c = q - t * vec;
            reinterpret_cast<float4 *>(hs + t * I)[c] =
                reinterpret_cast<const float4 *>(p.h + static_cast<size_t>(rows_out[t]) * I)[c];
        }
        __syncthreads();
        int rows_local[NT];
#pragma unroll
        for (int t = 0; t < NT; ++t) rows_local[t] = rows_out[t];
        if (rb < re) down_dispatch<NT>(p, ref, hs, nt, rows_local, rb, re);
    }
}

}  // namespace moe

template <typename F>
static cudaError_t set_smem(F f) {
    return cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, 160 * 1024);
}

cudaError_t moe_configure_ffn_gemv() {
    cudaError_t e = set_smem(moe::ffn_gate_up_gemv_kernel<1>);
    if (e == cudaSuccess) e = set_smem(moe::ffn_gate_up_gemv_kernel<4>);
    if (e == cudaSuccess) e = set_smem(moe::ffn_down_gemv_kernel<1>);
    if (e == cudaSuccess) e = set_smem(moe::ffn_down_gemv_kernel<4>);
    return e;
}

// NT = 1 when every expert has one token (T == 1), else groups of 4 tokens.
cudaError_t moe_launch_ffn_gemv(const moe::FfnParams &p, cudaStream_t s) {
    const int ctas_y = p.max_active + (p.has_shared ? 1 : 0);
    if (ctas_y == 0) return cudaSuccess;
    const int pairs_per_cta = moe::kGemvWarps * moe::kGuPairsPerWarp;
    dim3 g1((p.w.I + pairs_per_cta - 1) / pairs_per_cta, ctas_y);
    dim3 g2((p.w.H + moe::kDnRowsPerCta - 1) / moe::kDnRowsPerCta, ctas_y);
    const int nt = p.T == 1 ? 1 : 4;
    const size_t smem1 = static_cast<size_t>(nt) * p.w.H * sizeof(float);
    const size_t smem2 = static_cast<size_t>(nt) * p.w.I * sizeof(float);
    if (nt == 1) moe::ffn_gate_up_gemv_kernel<1><<<g1, moe::kGemvThreads, smem1, s>>>(p);
    else moe::ffn_gate_up_gemv_kernel<4><<<g1, moe::kGemvThreads, smem1, s>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (nt == 1) moe::ffn_down_gemv_kernel<1><<<g2, moe::kGemvThreads, smem2, s>>>(p);
    else moe::ffn_down_gemv_kernel<4><<<g2, moe::kGemvThreads, smem2, s>>>(p);
    return cudaGetLastError();
}
