// Tiered expert FFN, GEMV path: one persistent launch that streams every
// touched expert's packed rows once through a shared-memory ring.
//
// [P1] "step 4: three shelves, all on the GPU": mul_mat_id runs each word
// through its chosen experts, each shelf computes only the ids on it and the
// shelf results add up; the decode kernel fuses gate, up and the activation.
//
// Design (B200):
//  * Work is a list of tiles: for every active expert (any shelf) and the
//    shared expert, I/8 gate_up tiles (8 gate rows + the 8 matching up rows)
//    and H/64 down tiles (64 rows).  Each CTA takes a contiguous, byte-balanced
//    share of the gate_up tiles and then of the down tiles, so 8-, 4- and
//    3-bit experts spread evenly over the SMs.
//  * One producer thread per CTA moves each tile's codes and scales into a
//    4-6 stage shared-memory ring with 1-D bulk copies (cp.async.bulk) that
//    complete on an mbarrier; 8 consumer warps dequantise from shared memory
//    (w = d*q exact in fp32) and accumulate in fp32 against activations held
//    in registers.
//  * gate_up tiles write h = silu(g)*u (fp32) and count themselves done per
//    expert; a down tile waits (bounded) for its expert's count before reading
//    h, while its weights may already be in flight.  The grid is launched
//    cooperatively so every CTA is resident and the waits always resolve.
#include "common.cuh"
#include "ffn.cuh"
#include "sync.cuh"

namespace moe {

constexpr int kConsumerWarps = 8;
constexpr int kStreamThreads = (kConsumerWarps + 1) * 32;  // + one producer warp
constexpr int kGuPairs = 16;                                 // gate/up row pairs per tile (2 per warp)
constexpr int kDnRows = 64;                                  // down rows per tile
constexpr int kMaxStages = 6;
constexpr int kMaxRegK = 2048;  // activations held in registers: K <= 2048
constexpr int kMaxSmemEntries = 2048;  // token-entry tables kept in shared memory up to this size

__host__ __device__ __forceinline__ int row_bytes(int K, int bits) { return K * bits / 8; }
__host__ __device__ __forceinline__ int gu_tile_bytes(int H, int bits) {
    return 2 * kGuPairs * (row_bytes(H, bits) + H / 16);
}
__host__ __device__ __forceinline__ int dn_tile_bytes(int I, int bits) {
    return kDnRows * (row_bytes(I, bits) + I / 16);
}
// Work estimate used to balance tiles over CTAs: bytes moved plus a share for
// the per-weight dequant/FMA work, which is the same for every precision.
__host__ __device__ __forceinline__ long long gu_tile_cost(int H, int bits) {
    return gu_tile_bytes(H, bits) + static_cast<long long>(2 * kGuPairs) * H / 2;
}
__host__ __device__ __forceinline__ long long dn_tile_cost(int I, int bits) {
    return dn_tile_bytes(I, bits) + static_cast<long long>(kDnRows) * I / 2;
}

struct SlotTabs {  // per expert slot, in shared memory
    int *expert, *bits, *count, *first;
    int *tok, *row;  // entries [first, first + count) of every slot: token and h/y row
};

// Shelf pointers of expert e, read from the kernel parameters with constant
// indices only (no address of the parameter block is taken).
struct ExpertPtrs {
    const uint8_t *gq;
    const uint16_t *gs;
    const uint8_t *dq;
    const uint16_t *ds;
};

__device__ __forceinline__ int expert_bits(const FfnParams &p, int e) {
    if (e == p.E) return p.w.shared.bits;
    int b = 0;
#pragma unroll
    for (int i = 0; i < MOE_MAX_TIERS; ++i)
        if (i < p.w.n_tiers && e >= p.w.tiers[i].first_expert &&
            e < p.w.tiers[i].first_expert + p.w.tiers[i].n_experts)
            b = p.w.tiers[i].bits;
    return b;
}

__device__ __forceinline__ ExpertPtrs expert_ptrs(const FfnParams &p, int e) {
    const int H = p.w.H, I = p.w.I;
    ExpertPtrs r{nullptr, nullptr, nullptr, nullptr};
    if (e == p.E) {
        r.gq = p.w.shared.gu_qs;
        r.gs = p.w.shared.gu_scale;
        r.dq = p.w.shared.dn_qs;
        r.ds = p.w.shared.dn_scale;
        return r;
    }
#pragma unroll
    for (int i = 0; i < MOE_MAX_TIERS; ++i) {
        if (i < p.w.n_tiers && e >= p.w.tiers[i].first_expert &&
            e < p.w.tiers[i].first_expert + p.w.tiers[i].n_experts) {
            const size_t j = static_cast<size_t>(e - p.w.tiers[i].first_expert);
            const int b = p.w.tiers[i].bits;
            r.gq = p.w.tiers[i].gu_qs + j * 2 * I * row_bytes(H, b);
            r.gs = p.w.tiers[i].gu_scale + j * 2 * I * (H / 32);
            r.dq = p.w.tiers[i].dn_qs + j * H * row_bytes(I, b);
            r.ds = p.w.tiers[i].dn_scale + j * H * (I / 32);
        }
    }
    return r;
}

// Calls f(phase, slot, tile) for this CTA's tiles, in order: its byte-balanced
// share of all gate_up tiles (phase 0), then of all down tiles (phase 1).
template <class F>
__device__ __forceinline__ void for_each_tile(const FfnParams &p, const SlotTabs &st, int n_slots, F &&f) {
    const int G = gridDim.x, c = blockIdx.x;
    for (int phase = 0; phase < 2; ++phase) {
        const int nt = phase == 0 ? p.w.I / kGuPairs : p.w.H / kDnRows;
        long long total = 0;
        for (int a = 0; a < n_slots; ++a)
            total += static_cast<long long>(nt) *
                     (phase == 0 ? gu_tile_cost(p.w.H, st.bits[a]) : dn_tile_cost(p.w.I, st.bits[a]));
        const long long lo = total * c / G, hi = total * (c + 1) / G;
        long long off = 0;
        for (int a = 0; a < n_slots && off < hi; ++a) {
            const long long tb = phase == 0 ? gu_tile_cost(p.w.H, st.bits[a]) : dn_tile_cost(p.w.I, st.bits[a]);
            const long long end = off + nt * tb;
            if (end > lo) {
                const long long b0 = lo > off ? (lo - off + tb - 1) / tb : 0;
                long long b1 = (hi - off + tb - 1) / tb;
                if (b1 > nt) b1 = nt;
                for (long long b = b0; b < b1; ++b) f(phase, a, static_cast<int>(b));
            }
            off = end;
        }
    }
}

// ---------------------------------------------------------------------------
// dot products of one 16-byte unit (shared memory) with activations in registers
// ---------------------------------------------------------------------------
template <int BITS> struct UnitW;
template <> struct UnitW<8> { static constexpr int W = 16; };
template <> struct UnitW<4> { static constexpr int W = 32; };
template <> struct UnitW<3> { static constexpr int W = 64; };

template <int BITS>
__device__ __forceinline__ float unit_dot(const uint8_t *qrow, const uint16_t *srow, int K, int u,
                                          const float *a) {
    if constexpr (BITS == 8) {
        const uint4 q = *reinterpret_cast<const uint4 *>(qrow + 16 * u);
        const uint32_t wd[4] = {q.x, q.y, q.z, q.w};
        float p0 = 0.f, p1 = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float w[4];
            s8x4_to_f32(wd[i], w);
            p0 = fmaf(w[0], a[4 * i + 0], p0);
            p1 = fmaf(w[1], a[4 * i + 1], p1);
            p0 = fmaf(w[2], a[4 * i + 2], p0);
            p1 = fmaf(w[3], a[4 * i + 3], p1);
        }
        return f16_bits_to_f32(srow[u >> 1]) * (p0 + p1);
    } else if constexpr (BITS == 4) {
        const uint4 q = *reinterpret_cast<const uint4 *>(qrow + 16 * u);
        const uint32_t wd[4] = {q.x, q.y, q.z, q.w};
        float p0 = 0.f, p1 = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float w[8];
            u4x8_to_f32(wd[i], w);
#pragma unroll
            for (int m = 0; m < 8; m += 2) {
                p0 = fmaf(w[m], a[8 * i + m], p0);
                p1 = fmaf(w[m + 1], a[8 * i + m + 1], p1);
            }
        }
        return f16_bits_to_f32(srow[u]) * (p0 + p1);
    } else {
        const uint4 lo = *reinterpret_cast<const uint4 *>(qrow + 16 * u);
        const uint2 hi = *reinterpret_cast<const uint2 *>(qrow + K / 4 + 8 * u);
        const uint32_t lw[4] = {lo.x, lo.y, lo.z, lo.w};
        const uint32_t hw[4] = {hi.x & 0xffffu, hi.x >> 16, hi.y & 0xffffu, hi.y >> 16};
        float p[2] = {0.f, 0.f};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float w[16];
            u3x16_to_f32(lw[i], hw[i], w);
            float q0 = 0.f, q1 = 0.f;
#pragma unroll
            for (int m = 0; m < 16; m += 2) {
                q0 = fmaf(w[m], a[16 * i + m], q0);
                q1 = fmaf(w[m + 1], a[16 * i + m + 1], q1);
            }
            p[i >> 1] += q0 + q1;
        }
        return f16_bits_to_f32(srow[2 * u]) * p[0] + f16_bits_to_f32(srow[2 * u + 1]) * p[1];
    }
}

// Load the activations lane `lane` needs for a row of K weights at BITS:
// unit u = lane + 32*j covers weights [W*u, W*u + W).  Source is bf16 (x) or
// fp32 (h, read through L2 since other SMs wrote it).
template <int BITS, int UPL>
__device__ __forceinline__ void load_act_bf16(const uint16_t *row, int K, int lane, float *a) {
    constexpr int W = UnitW<BITS>::W;
    const int U = K / W;
#pragma unroll
    for (int j = 0; j < UPL; ++j) {
        const int u = lane + 32 * j;
        if (u < U) {
#pragma unroll
            for (int v = 0; v < W / 8; ++v) {
                const uint4 q = *reinterpret_cast<const uint4 *>(row + W * u + 8 * v);
                float *d = a + W * j + 8 * v;
                d[0] = bf16lo(q.x); d[1] = bf16hi(q.x); d[2] = bf16lo(q.y); d[3] = bf16hi(q.y);
                d[4] = bf16lo(q.z); d[5] = bf16hi(q.z); d[6] = bf16lo(q.w); d[7] = bf16hi(q.w);
            }
        }
    }
}

template <int BITS, int UPL>
__device__ __forceinline__ void load_act_f32(const float *row, int K, int lane, float *a) {
    constexpr int W = UnitW<BITS>::W;
    const int U = K / W;
#pragma unroll
    for (int j = 0; j < UPL; ++j) {
        const int u = lane + 32 * j;
        if (u < U) {
#pragma unroll
            for (int v = 0; v < W / 4; ++v) {
                const float4 q = __ldcg(reinterpret_cast<const float4 *>(row + W * u + 4 * v));
                float *d = a + W * j + 4 * v;
                d[0] = q.x; d[1] = q.y; d[2] = q.z; d[3] = q.w;
            }
        }
    }
}

// token and output row of the n-th entry of slot a (tables built in the prologue)
__device__ __forceinline__ void slot_entry(const FfnParams &p, const SlotTabs &st, int a, int n, int &tok,
                                           int &row) {
    const int j = st.first[a] + n;
    if (st.tok) {
        tok = st.tok[j];
        row = st.row[j];
    } else if (j >= p.T * p.k) {  // shared expert
        tok = j - p.T * p.k;
        row = j;
    } else {
        row = p.sorted[j];
        tok = row / p.k;
    }
}

// Sum each of N values over the 32 lanes with N-1 + log2(32/N) shuffles instead
// of 5N: at every step each lane keeps half of its values and swaps the other
// half.  On return lane l holds the full sum of value (l / (32 / N)) % N.
template <int N>
__device__ __forceinline__ float transpose_reduce(float (&v)[N]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int n = N, o = 16; n > 1; n >>= 1, o >>= 1) {
        const bool upper = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < n / 2; ++i) {
            const float send = upper ? v[i] : v[i + n / 2];
            const float keep = upper ? v[i + n / 2] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
    }
    float r = v[0];
    constexpr int rest = 32 / N;  // lanes still holding partial sums of the same value
#pragma unroll
    for (int o = rest / 2; o > 0; o >>= 1) r += __shfl_xor_sync(0xffffffffu, r, o);
    return r;
}

// gate_up tile: warp w computes pairs i = 16*tile + 2*w + {0, 1} for every
// token of the slot.  h is written with plain stores; the caller publishes it.
template <int BITS, int UPL>
__device__ __forceinline__ void consume_gu(const FfnParams &p, const SlotTabs &st, int a, int tile,
                                           const uint8_t *stage, float *act, int &act_key) {
    const int H = p.w.H, I = p.w.I;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int W = UnitW<BITS>::W;
    const int U = H / W;
    const int rb = row_bytes(H, BITS);
    const int nsc = H / 32;
    const uint8_t *q0 = stage + (2 * warp) * rb;                 // gate rows 2w, 2w+1
    const uint8_t *q1 = stage + (kGuPairs + 2 * warp) * rb;      // up rows
    const uint16_t *s0 = reinterpret_cast<const uint16_t *>(stage + 2 * kGuPairs * rb) + (2 * warp) * nsc;
    const uint16_t *s1 = s0 + kGuPairs * nsc;
    const int i0 = tile * kGuPairs + 2 * warp;
    for (int n = 0; n < st.count[a]; ++n) {
        int tok, row;
        slot_entry(p, st, a, n, tok, row);
        const int key = tok * 16 + BITS;
        if (key != act_key) {
            load_act_bf16<BITS, UPL>(p.x + static_cast<size_t>(tok) * H, H, lane, act);
            act_key = key;
        }
        float v[4] = {0.f, 0.f, 0.f, 0.f};  // g(i0), g(i0+1), u(i0), u(i0+1)
#pragma unroll
        for (int j = 0; j < UPL; ++j) {
            const int un = lane + 32 * j;
            if (un < U) {
                v[0] += unit_dot<BITS>(q0, s0, H, un, act + W * j);
                v[1] += unit_dot<BITS>(q0 + rb, s0 + nsc, H, un, act + W * j);
                v[2] += unit_dot<BITS>(q1, s1, H, un, act + W * j);
                v[3] += unit_dot<BITS>(q1 + rb, s1 + nsc, H, un, act + W * j);
            }
        }
        // lane l ends with value (l / 8) % 4: lanes 0 and 8 hold the two gates,
        // 16 and 24 the two ups
        const float r = transpose_reduce<4>(v);
        const float up = __shfl_down_sync(0xffffffffu, r, 16);
        if (lane == 0 || lane == 8) {
            const int i = i0 + (lane >> 3);
            p.h[static_cast<size_t>(row) * I + i] = r / (1.0f + expf(-r)) * up;
        }
    }
}

// down tile: warp w computes rows 64*tile + 8*w + r (r < 8) for every token.
template <int BITS, int UPL>
__device__ __forceinline__ void consume_dn(const FfnParams &p, const SlotTabs &st, int a, int tile,
                                           const uint8_t *stage, float *act, int &act_key) {
    const int H = p.w.H, I = p.w.I;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int W = UnitW<BITS>::W;
    const int U = I / W;
    const int rb = row_bytes(I, BITS);
    const uint16_t *sc = reinterpret_cast<const uint16_t *>(stage + kDnRows * rb);
    constexpr int R = kDnRows / kConsumerWarps;
    for (int n = 0; n < st.count[a]; ++n) {
        int tok, row;
        slot_entry(p, st, a, n, tok, row);
        const int key = -(row * 16 + BITS) - 2;
        if (key != act_key) {
            load_act_f32<BITS, UPL>(p.h + static_cast<size_t>(row) * I, I, lane, act);
            act_key = key;
        }
        float acc[R];
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int lr = warp * R + r;
            float v = 0.f;
#pragma unroll
            for (int j = 0; j < UPL; ++j) {
                const int un = lane + 32 * j;
                if (un < U) v += unit_dot<BITS>(stage + lr * rb, sc + lr * (I / 32), I, un, act + W * j);
            }
            acc[r] = v;
        }
        // lane l ends with the full sum of row (l / 4) % 8
        const float res = transpose_reduce<R>(acc);
        float *dst = row >= p.T * p.k ? p.y_shared + static_cast<size_t>(row - p.T * p.k) * H
                                      : p.y_slots + static_cast<size_t>(row) * H;
        if ((lane & 3) == 0) dst[tile * kDnRows + warp * R + (lane >> 2)] = res;
    }
}

__device__ __forceinline__ int upl_of(int K, int bits) {
    const int W = bits == 8 ? 16 : (bits == 4 ? 32 : 64);
    const int U = K / W;
    return (U + 31) / 32;
}

__device__ __forceinline__ void consume_tile(const FfnParams &p, const SlotTabs &st, int phase, int a, int tile,
                             const uint8_t *stage, float *act, int &act_key) {
    const int bits = st.bits[a];
    if (phase == 0) {
        const int upl = upl_of(p.w.H, bits);
        if (bits == 8) {
            if (upl <= 1) consume_gu<8, 1>(p, st, a, tile, stage, act, act_key);
            else if (upl <= 2) consume_gu<8, 2>(p, st, a, tile, stage, act, act_key);
            else consume_gu<8, 4>(p, st, a, tile, stage, act, act_key);
        } else if (bits == 4) {
            if (upl <= 1) consume_gu<4, 1>(p, st, a, tile, stage, act, act_key);
            else consume_gu<4, 2>(p, st, a, tile, stage, act, act_key);
        } else {
            consume_gu<3, 1>(p, st, a, tile, stage, act, act_key);
        }
    } else {
        const int upl = upl_of(p.w.I, bits);
        if (bits == 8) {
            if (upl <= 1) consume_dn<8, 1>(p, st, a, tile, stage, act, act_key);
            else if (upl <= 2) consume_dn<8, 2>(p, st, a, tile, stage, act, act_key);
            else consume_dn<8, 4>(p, st, a, tile, stage, act, act_key);
        } else if (bits == 4) {
            if (upl <= 1) consume_dn<4, 1>(p, st, a, tile, stage, act, act_key);
            else consume_dn<4, 2>(p, st, a, tile, stage, act, act_key);
        } else {
            consume_dn<3, 1>(p, st, a, tile, stage, act, act_key);
        }
    }
}

struct StreamSmem {
    uint8_t *stages;
    uint64_t *full, *empty;
    SlotTabs st;
    int *abort;
};

// The persistent FFN kernel body; `n_slots` slots are described in st.
__device__ __forceinline__ void ffn_stream_body(const FfnParams &p, StreamSmem &S, int n_slots, int nstages,
                                int stage_bytes) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int H = p.w.H, I = p.w.I;
    if (warp == kConsumerWarps) {
        // producer: one elected lane issues the bulk copies
        if (lane != 0) return;
        int i = 0;
        for_each_tile(p, S.st, n_slots, [&](int phase, int a, int tile) {
            if (*static_cast<volatile int *>(S.abort)) return;
            const int s = i % nstages;
            const uint32_t par = ((i / nstages) & 1) ^ 1;
            if (!mbar_wait(&S.empty[s], par)) {
                status_or(p.status, MOE_STATUS_TIMEOUT);
                *static_cast<volatile int *>(S.abort) = 1;
                return;
            }
            uint8_t *dst = S.stages + static_cast<size_t>(s) * stage_bytes;
            const ExpertPtrs e = expert_ptrs(p, S.st.expert[a]);
            const int bits = S.st.bits[a];
            if (phase == 0) {
                const int rb = row_bytes(H, bits);
                const size_t r0 = static_cast<size_t>(tile) * kGuPairs;
                const uint32_t qb = kGuPairs * rb, sb = kGuPairs * (H / 16);
                mbar_expect_tx(&S.full[s], 2 * qb + 2 * sb);
                bulk_g2s(dst, e.gq + r0 * rb, qb, &S.full[s]);
                bulk_g2s(dst + qb, e.gq + (I + r0) * rb, qb, &S.full[s]);
                bulk_g2s(dst + 2 * qb, e.gs + r0 * (H / 32), sb, &S.full[s]);
                bulk_g2s(dst + 2 * qb + sb, e.gs + (I + r0) * (H / 32), sb, &S.full[s]);
            } else {
                const int rb = row_bytes(I, bits);
                const size_t r0 = static_cast<size_t>(tile) * kDnRows;
                const uint32_t qb = kDnRows * rb, sb = kDnRows * (I / 16);
                mbar_expect_tx(&S.full[s], qb + sb);
                bulk_g2s(dst, e.dq + r0 * rb, qb, &S.full[s]);
                bulk_g2s(dst + qb, e.ds + r0 * (I / 32), sb, &S.full[s]);
            }
            ++i;
        });
        // drain: the last stages this thread filled must have landed before exit
        for (int j = i - nstages < 0 ? 0 : i - nstages; j < i; ++j)
            if (!mbar_wait(&S.full[j % nstages], (j / nstages) & 1)) status_or(p.status, MOE_STATUS_TIMEOUT);
        return;
    }
    // consumers
    float act[64];
    int act_key = -1;
    int i = 0;
    // h of a slot is published (fence + count) once per warp when the warp
    // leaves that slot: the count target is (gate_up tiles) x (consumer warps)
    // contributions, each contribution counting its tiles.
    int pend_slot = -1, pend_tiles = 0;
    const int gu_done = (I / kGuPairs) * kConsumerWarps;
    auto publish = [&]() {
        if (pend_slot >= 0) {
            __syncwarp();
            if (lane == 0 || lane == 8) __threadfence();  // the two lanes that wrote h
            __syncwarp();
            if (lane == 0) atomicAdd(p.ctr + pend_slot, pend_tiles);
        }
        pend_slot = -1;
        pend_tiles = 0;
    };
    for_each_tile(p, S.st, n_slots, [&](int phase, int a, int tile) {
        if (*static_cast<volatile int *>(S.abort)) return;
        if (phase == 0 && a != pend_slot) publish();
        if (phase == 1 && pend_slot >= 0) publish();
        const int s = i % nstages;
        const uint32_t par = (i / nstages) & 1;
        bool ok = mbar_wait(&S.full[s], par);
        if (phase == 1) {
            int dep = 1;
            if (lane == 0) dep = wait_geq(p.ctr + a, gu_done) ? 1 : 0;  // this expert's h is complete
            ok = ok && __shfl_sync(0xffffffffu, dep, 0);
        }
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) {
            if (lane == 0) status_or(p.status, MOE_STATUS_TIMEOUT);
            *static_cast<volatile int *>(S.abort) = 1;
            return;
        }
        consume_tile(p, S.st, phase, a, tile, S.stages + static_cast<size_t>(s) * stage_bytes, act, act_key);
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.empty[s]);
        if (phase == 0) {
            pend_slot = a;
            ++pend_tiles;
        }
        ++i;
    });
    publish();
}

__global__ void __launch_bounds__(kStreamThreads, 1)
ffn_stream_kernel(const FfnParams p, int nstages, int stage_bytes) {
    extern __shared__ __align__(1024) uint8_t smem[];
    StreamSmem S;
    S.stages = smem;
    uint8_t *tail = smem + static_cast<size_t>(nstages) * stage_bytes;
    S.full = reinterpret_cast<uint64_t *>(tail);
    S.empty = S.full + kMaxStages;
    S.abort = reinterpret_cast<int *>(S.empty + kMaxStages);
    int *tabs = S.abort + 4;
    const int max_slots = p.max_active + 1;
    S.st.expert = tabs;
    S.st.bits = tabs + max_slots;
    S.st.count = tabs + 2 * max_slots;
    S.st.first = tabs + 3 * max_slots;
    // entry tables in shared memory when they fit, else read from global
    const int n_ent = p.T * p.k + p.T;
    const bool ent_smem = n_ent <= kMaxSmemEntries;
    S.st.tok = ent_smem ? tabs + 4 * max_slots : nullptr;
    S.st.row = ent_smem ? S.st.tok + n_ent : nullptr;
    // slot table: active routed experts with work for this path (compacted),
    // then the shared expert
    __shared__ int n_keep;
    if (threadIdx.x == 0) n_keep = 0;
    __syncthreads();
    const int n_active_all = min(p.active[0], p.max_active);
    for (int a0 = 0; a0 < n_active_all; a0 += blockDim.x) {
        const int a = a0 + threadIdx.x;
        int e = -1, f = 0, cnt = 0;
        if (a < n_active_all) {
            e = p.active[1 + a];
            if (e >= 0 && e < p.E) {
                f = p.offsets[e];
                cnt = p.offsets[e + 1] - f;
            }
        }
        const bool keep = a < n_active_all && e >= 0 && e < p.E && cnt > 0 && cnt <= p.max_count;
        // order-preserving compaction within this block-wide step
        const unsigned m = __ballot_sync(0xffffffffu, keep);
        __shared__ int warp_base[kStreamThreads / 32];
        if ((threadIdx.x & 31) == 0) warp_base[threadIdx.x >> 5] = __popc(m);
        __syncthreads();
        if (threadIdx.x == 0) {
            int run = n_keep;
            for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) {
                const int c = warp_base[w];
                warp_base[w] = run;
                run += c;
            }
            n_keep = run;
        }
        __syncthreads();
        if (keep) {
            const int pos = warp_base[threadIdx.x >> 5] + __popc(m & ((1u << (threadIdx.x & 31)) - 1u));
            S.st.expert[pos] = e;
            S.st.bits[pos] = expert_bits(p, e);
            S.st.first[pos] = f;
            S.st.count[pos] = cnt;
        }
        __syncthreads();
    }
    const int n_active = n_keep;
    // entries: routed slots in sorted order (first = expert offset), then the
    // shared expert's T tokens at [T*k, T*k + T)
    const int S_ = p.T * p.k;
    const int n_routed = min(p.offsets[p.E], S_);
    if (ent_smem) {
        for (int j = threadIdx.x; j < n_routed; j += blockDim.x) {
            const int sl = p.sorted[j];
            const bool okj = sl >= 0 && sl < S_;
            S.st.tok[j] = okj ? sl / p.k : 0;
            S.st.row[j] = okj ? sl : 0;
        }
        for (int t = threadIdx.x; t < p.T; t += blockDim.x) {
            S.st.tok[S_ + t] = t;
            S.st.row[S_ + t] = S_ + t;
        }
    }
    if (threadIdx.x == 0) {
        if (p.has_shared && p.T <= p.max_count) {
            S.st.expert[n_active] = p.E;
            S.st.bits[n_active] = p.w.shared.bits;
            S.st.first[n_active] = S_;
            S.st.count[n_active] = p.T;
        }
        for (int s = 0; s < nstages; ++s) {
            mbar_init(&S.full[s], 1);
            mbar_init(&S.empty[s], kConsumerWarps);
        }
        *S.abort = 0;
        mbar_fence_init();
    }
    __syncthreads();
    const int n_slots = n_active + (p.has_shared && p.T <= p.max_count ? 1 : 0);
    ffn_stream_body(p, S, n_slots, nstages, stage_bytes);
}

}  // namespace moe

size_t moe_ffn_stream_smem(int H, int I, int max_slots, int n_ent, int *nstages, int *stage_bytes) {
    int sb = moe::gu_tile_bytes(H, 8);
    const int d = moe::dn_tile_bytes(I, 8);
    if (d > sb) sb = d;
    sb = (sb + 1023) & ~1023;
    const size_t ent = n_ent <= moe::kMaxSmemEntries ? 2 * sizeof(int) * static_cast<size_t>(n_ent) : 0;
    const size_t tail =
        2 * moe::kMaxStages * sizeof(uint64_t) + 16 + 4 * sizeof(int) * static_cast<size_t>(max_slots) + ent;
    const size_t budget = 220 * 1024;
    int ns = static_cast<int>((budget - tail) / sb);
    if (ns > moe::kMaxStages) ns = moe::kMaxStages;
    *nstages = ns;
    *stage_bytes = sb;
    return static_cast<size_t>(ns) * sb + tail;
}

cudaError_t moe_configure_ffn_stream() {
    // the opt-in limit is 227 KB per CTA including static shared memory
    return cudaFuncSetAttribute(moe::ffn_stream_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                227 * 1024 - 1024);
}

bool moe_ffn_stream_supported(int H, int I) {
    return H <= moe::kMaxRegK && I <= moe::kMaxRegK && H % 128 == 0 && I % 128 == 0;
}

// counters (int[max_active + 1]) must be zero on entry; the caller clears them.
cudaError_t moe_launch_ffn_stream(const moe::FfnParams &p, cudaStream_t s) {
    int nstages = 0, stage_bytes = 0;
    const size_t smem =
        moe_ffn_stream_smem(p.w.H, p.w.I, p.max_active + 1, p.T * p.k + p.T, &nstages, &stage_bytes);
    if (nstages < 2) return cudaErrorInvalidConfiguration;
    int dev = 0;
    cudaGetDevice(&dev);
    int sms = 0;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(sms);
    cfg.blockDim = dim3(moe::kStreamThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, moe::ffn_stream_kernel, p, nstages, stage_bytes);
}
