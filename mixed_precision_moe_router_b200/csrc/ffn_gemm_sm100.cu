// Tiered expert FFN, tensor-core path for prefill-sized token groups.
//
// [P1] "step 4: three shelves, all on the GPU": the patched mul_mat_id runs
// each shelf's experts over the routed tokens and the shelf results add up;
// for large token groups this is a dense contraction per expert, so here it is
// a grouped GEMM on the 5th-generation tensor cores (tcgen05, sm_100a).
//
// Orientation: the expert's weight rows are the MMA M side (128 rows per
// tile) and the expert's tokens the N side (padded to a multiple of 16, at most
// 128 per accumulator), so an expert with few tokens wastes at most 15 columns.
//   gate_up:  D[row, tok] = W_gu[row] . x[tok],  rows interleaved gate/up so a
//             thread and its neighbour lane hold g and u of the same pair;
//             epilogue h = silu(g) * u written as fp16 in expert-grouped order.
//   down:     D[n, tok] = W_dn[n] . h[tok],  epilogue writes fp32 y.
// Operands are staged in fp16 (w = fp16_rne(d*q); x and h in fp16, whose range
// is checked), accumulation is fp32 in tensor memory.
//
// Warp roles (480 threads, one CTA per SM, persistent over tiles):
//   warps 0-7  dequant: thread (warp w, lane l) owns tile row 32*(w%4)+l, which
//              is the tensor-memory lane its warp may access, and one 64-wide
//              half (w/4) of each 128-wide K chunk (BK); its packed codes and
//              scales stream through a RAW-deep (4) cp.async ring in shared
//              memory, are converted with packed half2 arithmetic and stored
//              straight into tensor memory (tcgen05.st), where the MMA reads
//              its A operand (STAGES = 4 stages of BK/2 columns).
//   warps 8-11 epilogue: tcgen05.ld of their 32 accumulator lanes.
//   warps 12-13 token rows: cp.async gather of fp16 rows into 128B-swizzled
//              K-major shared memory, BK wide per stage (zero-filled past the
//              expert's last token).
//   warp  14   allocates 512 TMEM columns (two MAXN = 128-column accumulators,
//              then the A stages); lane 0 issues tcgen05.mma and tcgen05.commit.
#include "common.cuh"
#include "ffn.cuh"
#include "sync.cuh"

namespace moe {
namespace gemm {

constexpr int BM = 128;        // weight rows per tile (MMA M)
constexpr int BK = 128;        // K elements per stage (two 128-byte swizzle atoms of fp16 per token row)
constexpr int MAXN = 128;      // tokens per accumulator (MMA N)
constexpr int STAGES = 4;
constexpr int RAW = 4;         // cp.async depth of the dequant producers
constexpr int B_HALF = MAXN * 128;             // one 64-wide K half of the token tile (128 B rows)
constexpr int B_BYTES = 2 * B_HALF;
constexpr int STAGE_BYTES = B_BYTES;           // shared memory holds the token tile only
constexpr int ACC_COLS = 2 * MAXN;             // two fp32 accumulators
constexpr int A_COLS = BK / 2;                 // one fp16 A stage in TMEM: 2 values per column
constexpr int DQ_THREADS = 2 * BM;  // two dequant warps per TMEM lane quarter, 64 weights per thread
constexpr int RAW_ROW = 80;         // per dequant thread and raw stage: 64 code bytes + 4 scale bytes (+pad)
constexpr int RAW_BYTES = DQ_THREADS * RAW_ROW;
constexpr int WARPS = 15;
constexpr int THREADS = WARPS * 32;
constexpr int EPI_WARP0 = 8, BPROD_WARP0 = 12, MMA_WARP = 14;
constexpr int BPROD_THREADS = 64;
constexpr int TMEM_COLS = 512;

struct Params {
    FfnParams f;
    int phase;              // 0: gate_up, 1: down, 2: router logits
    // router mode: logits[t][e] = x[t] . w_router[e] + bias[e], bf16 operands
    const uint16_t *wr;     // bf16 [E][H]
    const float *bias;      // [E] or null
    float *logits;          // fp32 [T][E]
    const uint16_t *x16;    // fp16 [T][H]
    uint16_t *h16;          // fp16 [T*k + T][I], expert-grouped rows
    int min_count;          // experts with fewer tokens are left to the GEMV path
};

// ---------------------------------------------------------------------------
// PTX wrappers
// ---------------------------------------------------------------------------
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, int src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async8(uint32_t dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_alloc(uint32_t *dst_smem, int ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, int ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                        uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// A from tensor memory (row m in lane m, two fp16 per column), B from shared memory
__device__ __forceinline__ void mma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                           uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Issue a 16-column store into tensor memory; completion is awaited later with
// tmem_st_wait() so that it overlaps the next chunk's conversion.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
        "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
        "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]),
        "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]),
        "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
        : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void mma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
          "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
          "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor: K-major operand in the 128-byte swizzled
// canonical layout (8-row groups of 1024 bytes, 16-byte leading offset),
// descriptor version 1 (sm_100).
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr) {
    return static_cast<uint64_t>((saddr >> 4) & 0x3fff) | (static_cast<uint64_t>(1) << 16) |
           (static_cast<uint64_t>(1024 >> 4) << 32) | (static_cast<uint64_t>(1) << 46) |
           (static_cast<uint64_t>(2) << 61);
}

// Instruction descriptor: kind::f16, A = B = fp16, D = fp32, both K-major,
// M = 128, N = n.
__device__ __forceinline__ uint32_t idesc_f16(int n, bool bf16 = false) {
    const uint32_t ab = bf16 ? ((1u << 7) | (1u << 10)) : 0u;  // A and B format: 0 = fp16, 1 = bf16
    return (1u << 4) | ab | (static_cast<uint32_t>(n >> 3) << 17) | (static_cast<uint32_t>(BM >> 4) << 24);
}

// byte offset of 16-byte chunk c of row r in a 128B-swizzled K-major tile
__device__ __forceinline__ uint32_t sw128(int r, int c) {
    return static_cast<uint32_t>(r * 128 + ((c ^ (r & 7)) << 4));
}

__device__ __forceinline__ uint32_t h2(uint16_t lo, uint16_t hi) { return lo | (static_cast<uint32_t>(hi) << 16); }

__device__ __forceinline__ uint32_t hsub2_u(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}
__device__ __forceinline__ uint32_t hmul2_u(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// ---------------------------------------------------------------------------
// Dequantisation of one 64-weight chunk of a row to 32 fp16 pairs
// w = fp16_rne(d * q): q is built exactly as fp16 from the code bits with the
// 1024-offset exponent trick, then one fp16 multiply rounds the exact product.
// ---------------------------------------------------------------------------
// 32-weight variants (one quantisation block, one scale pair d2)
__device__ __forceinline__ void dequant8_32(const uint8_t *raw, uint32_t d2, uint32_t (&o)[16]) {
    const uint4 *q = reinterpret_cast<const uint4 *>(raw);
    const uint32_t bias = 0x64806480u;
#pragma unroll
    for (int v = 0; v < 2; ++v) {
        const uint4 w = q[v];
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const uint32_t u = ws[m] ^ 0x80808080u;
            o[v * 8 + 2 * m] = hmul2_u(hsub2_u(__byte_perm(u, 0x64646464u, 0x4140), bias), d2);
            o[v * 8 + 2 * m + 1] = hmul2_u(hsub2_u(__byte_perm(u, 0x64646464u, 0x4342), bias), d2);
        }
    }
}

__device__ __forceinline__ void dequant4_32(const uint8_t *raw, uint32_t d2, uint32_t (&o)[16]) {
    const uint4 w = *reinterpret_cast<const uint4 *>(raw);
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
    const uint32_t bias = 0x64086408u;
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        uint32_t P[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) P[j] = hsub2_u(((ws[m] >> (4 * j)) & 0x000f000fu) | 0x64006400u, bias);
        o[4 * m] = hmul2_u(__byte_perm(P[0], P[1], 0x5410), d2);
        o[4 * m + 1] = hmul2_u(__byte_perm(P[2], P[3], 0x5410), d2);
        o[4 * m + 2] = hmul2_u(__byte_perm(P[0], P[1], 0x7632), d2);
        o[4 * m + 3] = hmul2_u(__byte_perm(P[2], P[3], 0x7632), d2);
    }
}

// FP4 codes: the nibble layout of 4-bit codes, the integers q = 2 * value
// from the E2M1 table (exact fp16), so d * q is exact as well.
__device__ __forceinline__ void dequant_fp4_32(const uint8_t *raw, uint32_t d2, uint32_t (&o)[16]) {
    const uint4 w = *reinterpret_cast<const uint4 *>(raw);
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        uint32_t P[4];
        fp4_pairs(ws[m], P);
        o[4 * m] = hmul2_u(__byte_perm(P[0], P[1], 0x5410), d2);
        o[4 * m + 1] = hmul2_u(__byte_perm(P[2], P[3], 0x5410), d2);
        o[4 * m + 2] = hmul2_u(__byte_perm(P[0], P[1], 0x7632), d2);
        o[4 * m + 3] = hmul2_u(__byte_perm(P[2], P[3], 0x7632), d2);
    }
}

__device__ __forceinline__ void dequant3_32(const uint8_t *raw, uint32_t d2, uint32_t (&o)[16]) {
    const uint2 lo = *reinterpret_cast<const uint2 *>(raw);
    const uint32_t hi = *reinterpret_cast<const uint32_t *>(raw + 8);
    const uint32_t lw[2] = {lo.x, lo.y};
    const uint32_t bias = 0x64046404u;
#pragma unroll
    for (int p = 0; p < 2; ++p) {
        const uint32_t hw = hi >> (16 * p);
        const uint32_t Y = ((hw & 0xffu) | ((hw & 0xff00u) << 8)) << 2;
        uint32_t P[8];
#pragma unroll
        for (int j = 0; j < 8; ++j)
            P[j] = hsub2_u(((lw[p] >> (2 * j)) & 0x00030003u) | ((Y >> j) & 0x00040004u) | 0x64006400u, bias);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            o[p * 8 + j] = hmul2_u(__byte_perm(P[2 * j], P[2 * j + 1], 0x5410), d2);
            o[p * 8 + 4 + j] = hmul2_u(__byte_perm(P[2 * j], P[2 * j + 1], 0x7632), d2);
        }
    }
}

// ---------------------------------------------------------------------------
// slots and tiles
// ---------------------------------------------------------------------------
struct Slots {
    int *expert, *bits, *count, *first, *tile0;  // tile0[n_slots + 1]: prefix of tiles
    int n;
};

__device__ __forceinline__ int n_mtiles(const Params &P) {
    return P.phase == 0 ? (2 * P.f.w.I) / BM : (P.phase == 1 ? P.f.w.H / BM : P.f.E / BM);
}
__device__ __forceinline__ int n_kchunks(const Params &P) {
    return (P.phase == 1 ? P.f.w.I : P.f.w.H) / BK;
}

struct Tile {
    int slot, nc, mt;
};

__device__ __forceinline__ Tile tile_of(const Slots &S, int nmt, int t) {
    int lo = 0, hi = S.n;  // last slot with tile0 <= t
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (S.tile0[mid] <= t) lo = mid; else hi = mid;
    }
    const int r = t - S.tile0[lo];
    return Tile{lo, r / nmt, r % nmt};
}

// shelf pointers of an expert (constant-index reads of the parameters)
__device__ __forceinline__ void expert_rows(const Params &P, int e, int &bits, const uint8_t *&qs,
                                            const uint16_t *&sc) {
    const int H = P.f.w.H, I = P.f.w.I;
    if (e == P.f.E) {
        bits = P.phase == 0 ? P.f.w.shared.bits : tier_dn_bits(P.f.w.shared);
        qs = P.phase == 0 ? P.f.w.shared.gu_qs : P.f.w.shared.dn_qs;
        sc = P.phase == 0 ? P.f.w.shared.gu_scale : P.f.w.shared.dn_scale;
        return;
    }
#pragma unroll
    for (int i = 0; i < MOE_MAX_TIERS; ++i) {
        if (i < P.f.w.n_tiers && e >= P.f.w.tiers[i].first_expert &&
            e < P.f.w.tiers[i].first_expert + P.f.w.tiers[i].n_experts) {
            const size_t j = static_cast<size_t>(e - P.f.w.tiers[i].first_expert);
            const int b = P.phase == 0 ? P.f.w.tiers[i].bits : tier_dn_bits(P.f.w.tiers[i]);
            bits = b;
            if (P.phase == 0) {
                qs = P.f.w.tiers[i].gu_qs + j * 2 * I * (H * storage_bits(b) / 8);
                sc = P.f.w.tiers[i].gu_scale + j * 2 * I * (H / 32);
            } else {
                qs = P.f.w.tiers[i].dn_qs + j * H * (I * storage_bits(b) / 8);
                sc = P.f.w.tiers[i].dn_scale + j * H * (I / 32);
            }
        }
    }
}

struct Shared {
    uint8_t *stages;   // STAGES x [A | B], 1024-aligned
    uint8_t *raw;      // RAW x [BM][RAW_ROW]
    uint64_t *full_a, *full_b, *empty, *acc_full, *acc_empty, *fin;
    uint32_t *tmem_slot;
    int *abort;
    Slots slots;
};

__device__ __forceinline__ bool aborted(const Shared &S) { return *static_cast<volatile int *>(S.abort) != 0; }

__device__ __forceinline__ void fail(const Params &P, const Shared &S) {
    status_or(P.f.status, MOE_STATUS_TIMEOUT);
    *static_cast<volatile int *>(S.abort) = 1;
}

// ---------------------------------------------------------------------------
// roles
// ---------------------------------------------------------------------------
// Dequant producer: lane l of warps w and w + 4 (w < 4) owns tile row
// 32*w + l, each streaming one 64-weight half (two 32-weight blocks) of every
// tile's 128-wide K chunk.
__device__ __forceinline__ void role_dequant(const Params &P, const Shared &S, int total_tiles, uint32_t tmem) {
    const int tid = threadIdx.x;  // 0..255
    const int warp = tid >> 5, lane = tid & 31;
    const int r = 32 * (warp & 3) + lane;  // tile row = TMEM lane this warp may access
    const int half = warp >> 2;            // which 32 of the chunk's 64 weights
    const int nmt = n_mtiles(P), NK = n_kchunks(P);
    const int K = P.phase == 0 ? P.f.w.H : P.f.w.I;
    const int G = gridDim.x;
    const int my_tiles = total_tiles > static_cast<int>(blockIdx.x)
                             ? (total_tiles - static_cast<int>(blockIdx.x) + G - 1) / G : 0;
    const int nchunks = my_tiles * NK;
    uint8_t *raw_me = S.raw + tid * RAW_ROW;
    const uint32_t raw_me_s = smem_u32(raw_me);

    // Row source of this thread for the tile holding linear chunk L; recomputed
    // only when a cursor crosses into the next tile.
    struct RowCtx {
        int tile_local = -1, bits = 8;
        const uint8_t *qrow = nullptr;
        const uint16_t *srow = nullptr;
    };
    auto locate = [&](RowCtx &c, int L) {
        const int tl_local = L / NK;
        if (tl_local == c.tile_local) return;
        c.tile_local = tl_local;
        const Tile tl = tile_of(S.slots, nmt, blockIdx.x + tl_local * G);
        const uint8_t *qs;
        const uint16_t *sc;
        expert_rows(P, S.slots.expert[tl.slot], c.bits, qs, sc);
        const int row = P.phase == 0 ? ((r & 1) ? P.f.w.I : 0) + tl.mt * (BM / 2) + (r >> 1) : tl.mt * BM + r;
        c.qrow = qs + static_cast<size_t>(row) * (K * storage_bits(c.bits) / 8);
        c.srow = sc + static_cast<size_t>(row) * (K / 32);
    };
    if (P.phase == 2) {  // router: bf16 weight rows go to tensor memory unchanged
        int pend = -1;
#pragma unroll 1
        for (int L = 0; L < nchunks; ++L) {
            const Tile tl = tile_of(S.slots, nmt, blockIdx.x + (L / NK) * G);
            const int kc = L % NK;
            const uint16_t *src = P.wr + static_cast<size_t>(tl.mt * BM + r) * P.f.w.H + kc * BK + 64 * half;
            uint32_t o[32];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint4 q = *reinterpret_cast<const uint4 *>(src + 8 * c);
                o[4 * c] = q.x; o[4 * c + 1] = q.y; o[4 * c + 2] = q.z; o[4 * c + 3] = q.w;
            }
            if (pend >= 0) {
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&S.full_a[pend]);
                pend = -1;
            }
            const int s = L % STAGES;
            if (!__all_sync(0xffffffffu, mbar_wait_limit(&S.empty[s], ((L / STAGES) & 1) ^ 1, P.f.wait_limit))) { fail(P, S); break; }
            tc_fence_after();
            tmem_st32(tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16) + ACC_COLS + s * A_COLS + 32 * half, o);
            pend = s;
        }
        if (pend >= 0) {
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&S.full_a[pend]);
        }
        return;
    }
    RowCtx ci, cp;  // issue-ahead and processing cursors
    auto issue = [&](int L) {
        if (L < nchunks) {
            locate(ci, L);
            const int kc = L % NK;
            const uint8_t *qrow = ci.qrow;
            const uint32_t dst = raw_me_s + (L % RAW) * RAW_BYTES;
            const int blk = 4 * kc + 2 * half;  // first of this thread's two 32-weight blocks
            if (ci.bits == 8) {
#pragma unroll
                for (int c = 0; c < 4; ++c) cp_async16(dst + 16 * c, qrow + 32 * blk + 16 * c, 16);
            } else if (ci.bits == 4 || ci.bits == kBitsFp4) {
                cp_async16(dst, qrow + 16 * blk, 16);
                cp_async16(dst + 16, qrow + 16 * blk + 16, 16);
            } else {
                cp_async16(dst, qrow + 8 * blk, 16);
                cp_async8(dst + 16, qrow + K / 4 + 4 * blk);
            }
            cp_async4(dst + 64, ci.srow + blk);  // the scales of its two blocks
        }
        cp_async_commit();
    };
#pragma unroll 1
    for (int L = 0; L < RAW - 1; ++L) issue(L);
    int pend = -1;  // stage whose TMEM store is in flight and not yet signalled
#pragma unroll 1
    for (int L = 0; L < nchunks; ++L) {
        issue(L + RAW - 1);
        cp_async_wait<RAW - 1>();
        if (__any_sync(0xffffffffu, aborted(S))) break;  // warp-uniform exit (tcgen05.st is warp-wide)
        locate(cp, L);
        const int bits = cp.bits;
        const uint8_t *raw = raw_me + (L % RAW) * RAW_BYTES;
        const uint32_t sc2 = *reinterpret_cast<const uint32_t *>(raw + 64);
        const uint32_t d2a = (sc2 & 0xffffu) | (sc2 << 16);       // (d0, d0)
        const uint32_t d2b = (sc2 >> 16) | (sc2 & 0xffff0000u);   // (d1, d1)
        uint32_t o[32];
        uint32_t(&o0)[16] = *reinterpret_cast<uint32_t(*)[16]>(o);
        uint32_t(&o1)[16] = *reinterpret_cast<uint32_t(*)[16]>(o + 16);
        if (bits == 8) {
            dequant8_32(raw, d2a, o0);
            dequant8_32(raw + 32, d2b, o1);
        } else if (bits == 4) {
            dequant4_32(raw, d2a, o0);
            dequant4_32(raw + 16, d2b, o1);
        } else if (bits == kBitsFp4) {
            dequant_fp4_32(raw, d2a, o0);
            dequant_fp4_32(raw + 16, d2b, o1);
        } else {
            // lo plane: 8 bytes per block; hi plane: 4 bytes per block
            uint8_t tmp[16];
            *reinterpret_cast<uint2 *>(tmp) = *reinterpret_cast<const uint2 *>(raw);
            *reinterpret_cast<uint32_t *>(tmp + 8) = *reinterpret_cast<const uint32_t *>(raw + 16);
            dequant3_32(tmp, d2a, o0);
            *reinterpret_cast<uint2 *>(tmp) = *reinterpret_cast<const uint2 *>(raw + 8);
            *reinterpret_cast<uint32_t *>(tmp + 8) = *reinterpret_cast<const uint32_t *>(raw + 20);
            dequant3_32(tmp, d2b, o1);
        }
        if (pend >= 0) {  // the previous chunk's store has had a whole conversion to land
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&S.full_a[pend]);  // one arrival per warp
            pend = -1;
        }
        const int s = L % STAGES;
        const bool ok = __all_sync(0xffffffffu, mbar_wait_limit(&S.empty[s], ((L / STAGES) & 1) ^ 1, P.f.wait_limit));
        if (!ok) { fail(P, S); break; }
        tc_fence_after();
        // lanes 32*(warp%4).. of the stage's A columns; this thread's row and half
        tmem_st32(tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16) + ACC_COLS + s * A_COLS + 32 * half, o);
        pend = s;
    }
    if (pend >= 0) {
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.full_a[pend]);
    }
    cp_async_wait<0>();
}

__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t *bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Token-row producer: 64 threads gather the fp16 rows of the tile's tokens.
__device__ __forceinline__ void role_tokens(const Params &P, const Shared &S, int total_tiles) {
    const int b = threadIdx.x - BPROD_WARP0 * 32;  // 0..63
    const int nmt = n_mtiles(P), NK = n_kchunks(P);
    const int K = P.phase == 1 ? P.f.w.I : P.f.w.H;
    const int G = gridDim.x;
    const int S_ = P.f.T * P.f.k;
    int q = 0;  // linear chunk counter
#pragma unroll 1
    for (int t = blockIdx.x; t < total_tiles; t += G) {
        const Tile tl = tile_of(S.slots, nmt, t);
        const int cnt = S.slots.count[tl.slot];
        const int first = S.slots.first[tl.slot];
        const int nvalid = min(MAXN, cnt - tl.nc * MAXN);
        const int Nt = (nvalid + 15) & ~15;
        // source rows of this thread's token rows j = b + 64 m
        const uint16_t *src[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const int j = b + 64 * m;
            src[m] = nullptr;
            if (j < nvalid) {
                const int ent = first + tl.nc * MAXN + j;
                if (P.phase == 2) {
                    src[m] = P.f.x + static_cast<size_t>(ent) * K;  // token rows in order, bf16
                } else if (P.phase == 0) {
                    const int tok = ent >= S_ ? ent - S_ : P.f.sorted[ent] / P.f.k;
                    src[m] = P.x16 + static_cast<size_t>(tok) * K;
                } else {
                    src[m] = P.h16 + static_cast<size_t>(ent) * K;
                }
            }
        }
#pragma unroll 1
        for (int kc = 0; kc < NK; ++kc, ++q) {
            const int s = q % STAGES;
            if (!mbar_wait_limit(&S.empty[s], ((q / STAGES) & 1) ^ 1, P.f.wait_limit)) { fail(P, S); break; }
            const uint32_t B = smem_u32(S.stages + s * STAGE_BYTES);
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const int j = b + 64 * m;
                if (j < Nt) {
                    const uint16_t *row = src[m] ? src[m] + kc * BK : P.x16;
                    const int n = src[m] ? 16 : 0;  // zero-fill rows past the last token
#pragma unroll
                    for (int h = 0; h < 2; ++h)
#pragma unroll
                        for (int c = 0; c < 8; ++c) cp_async16(B + h * B_HALF + sw128(j, c), row + 64 * h + 8 * c, n);
                }
            }
            // the stage's arrival fires when this thread's copies have landed
            cp_async_arrive_noinc(&S.full_b[s]);
        }
        if (aborted(S)) break;
    }
    cp_async_wait<0>();
}

// MMA issuer (one thread).
__device__ __forceinline__ void role_mma(const Params &P, const Shared &S, int total_tiles, uint32_t tmem) {
    const int nmt = n_mtiles(P), NK = n_kchunks(P);
    const int G = gridDim.x;
    int q = 0, acc = 0;
#pragma unroll 1
    for (int t = blockIdx.x; t < total_tiles; t += G, ++acc) {
        const Tile tl = tile_of(S.slots, nmt, t);
        const int nvalid = min(MAXN, S.slots.count[tl.slot] - tl.nc * MAXN);
        const int Nt = (nvalid + 15) & ~15;
        const uint32_t idesc = idesc_f16(Nt, P.phase == 2);
        const int buf = acc & 1;
        if (!mbar_wait_limit(&S.acc_empty[buf], ((acc >> 1) & 1) ^ 1, P.f.wait_limit)) { fail(P, S); break; }
        tc_fence_after();
        const uint32_t d = tmem + buf * MAXN;
        bool ok = true;
#pragma unroll 1
        for (int kc = 0; kc < NK; ++kc, ++q) {
            const int s = q % STAGES;
            const uint32_t par = (q / STAGES) & 1;
            if (!mbar_wait_limit(&S.full_a[s], par, P.f.wait_limit) || !mbar_wait_limit(&S.full_b[s], par, P.f.wait_limit)) { ok = false; break; }
            tc_fence_after();
            const uint32_t b0 = smem_u32(S.stages + s * STAGE_BYTES);
            const uint32_t a = tmem + ACC_COLS + s * A_COLS;
#pragma unroll
            for (int k = 0; k < BK / 16; ++k) {  // K step of 16: 8 TMEM columns of A, 32 bytes of a B half
                const uint64_t bd = smem_desc_sw128(b0 + (k >> 2) * B_HALF) + 2 * (k & 3);
                mma_f16_ts(d, a + 8 * k, bd, idesc, (kc | k) != 0);
            }
            mma_commit(&S.empty[s]);
        }
        if (!ok) { fail(P, S); break; }
        mma_commit(&S.acc_full[buf]);
    }
    // all MMAs issued by this thread are complete before the CTA tears down
    mma_commit(S.fin);
    if (!mbar_wait_limit(S.fin, 0, P.f.wait_limit)) status_or(P.f.status, MOE_STATUS_TIMEOUT);
}

// Epilogue: warp q of the epilogue group owns accumulator lanes 32q..32q+31.
__device__ __forceinline__ void role_epilogue(const Params &P, const Shared &S, int total_tiles, uint32_t tmem) {
    const int q = (threadIdx.x >> 5) - EPI_WARP0, lane = threadIdx.x & 31;
    const int nmt = n_mtiles(P);
    const int G = gridDim.x;
    const int H = P.f.w.H, I = P.f.w.I;
    const int S_ = P.f.T * P.f.k;
    bool range_bad = false;
    int acc = 0;
#pragma unroll 1
    for (int t = blockIdx.x; t < total_tiles; t += G, ++acc) {
        const Tile tl = tile_of(S.slots, nmt, t);
        const int first = S.slots.first[tl.slot];
        const int nvalid = min(MAXN, S.slots.count[tl.slot] - tl.nc * MAXN);
        const int buf = acc & 1;
        if (!__all_sync(0xffffffffu, mbar_wait_limit(&S.acc_full[buf], (acc >> 1) & 1, P.f.wait_limit))) { fail(P, S); break; }
        tc_fence_after();
        const int row = 32 * q + lane;  // accumulator lane = tile row
#pragma unroll 1
        for (int c0 = 0; c0 < nvalid; c0 += 32) {
            uint32_t v[32];
            tmem_ld32(tmem + (static_cast<uint32_t>(32 * q) << 16) + buf * MAXN + c0, v);
            if (P.phase == 2) {
                const int e = tl.mt * BM + row;
                const float b = P.bias ? P.bias[e] : 0.f;
                float *lg = P.logits + static_cast<size_t>(tl.nc * MAXN + c0) * P.f.E + e;
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    if (c0 + j < nvalid) lg[static_cast<size_t>(j) * P.f.E] = __uint_as_float(v[j]) + b;
            } else if (P.phase == 0) {
                // lanes 2p and 2p+1 hold gate and up of pair p; each lane finishes
                // every other column so both lanes of a pair do the SwiGLU work
                const int i = tl.mt * (BM / 2) + (row >> 1);  // pair index
                const bool odd = lane & 1;
                uint16_t *hbase = P.h16 + static_cast<size_t>(first + tl.nc * MAXN + c0) * I + i;
#pragma unroll
                for (int j = 0; j < 32; j += 2) {
                    const float a0 = __uint_as_float(v[j]), a1 = __uint_as_float(v[j + 1]);
                    const float recv = __shfl_xor_sync(0xffffffffu, odd ? a0 : a1, 1);
                    const float g = odd ? recv : a0;  // even: g_j      odd: g_{j+1}
                    const float u = odd ? a1 : recv;  // even: u_j      odd: u_{j+1}
                    const int col = j + (odd ? 1 : 0);
                    if (c0 + col < nvalid) {
                        const float hv = __fdividef(g, 1.0f + __expf(-g)) * u;
                        range_bad |= !(fabsf(hv) <= 65504.0f);
                        hbase[static_cast<size_t>(col) * I] = __half_as_ushort(__float2half_rn(hv));
                    }
                }
            } else {
                const int n = tl.mt * BM + row;
                // one coalesced load of the 32 destination rows, then broadcast per column
                const int my_ent = first + tl.nc * MAXN + c0 + lane;
                int my_row = -1;
                if (c0 + lane < nvalid) my_row = my_ent >= S_ ? -(my_ent - S_) - 2 : P.f.sorted[my_ent];
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int dr = __shfl_sync(0xffffffffu, my_row, j);
                    if (dr != -1) {
                        float *dst = dr <= -2 ? P.f.y_shared + static_cast<size_t>(-dr - 2) * H
                                              : P.f.y_slots + static_cast<size_t>(dr) * H;
                        dst[n] = __uint_as_float(v[j]);
                    }
                }
            }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.acc_empty[buf]);  // one arrival per epilogue warp
    }
    if (range_bad) status_or(P.f.status, MOE_STATUS_FP16_RANGE);
}

__global__ void __launch_bounds__(THREADS, 1) ffn_gemm_kernel(const Params P) {
    extern __shared__ uint8_t smem_raw[];
    Shared S;
    const uint32_t base = smem_u32(smem_raw);
    const uint32_t pad = ((base + 1023u) & ~1023u) - base;
    uint8_t *p = smem_raw + pad;
    S.stages = p;
    p += STAGES * STAGE_BYTES;
    S.raw = p;
    p += RAW * RAW_BYTES;
    uint64_t *bars = reinterpret_cast<uint64_t *>(p);
    S.full_a = bars;
    S.full_b = bars + STAGES;
    S.empty = bars + 2 * STAGES;
    S.acc_full = bars + 3 * STAGES;
    S.acc_empty = S.acc_full + 2;
    S.fin = S.acc_empty + 2;
    p += (3 * STAGES + 5) * sizeof(uint64_t);
    S.tmem_slot = reinterpret_cast<uint32_t *>(p);
    S.abort = reinterpret_cast<int *>(p + 4);
    int *tab = reinterpret_cast<int *>(p + 16);
    const int max_slots = P.f.max_active + 1;
    S.slots.expert = tab;
    S.slots.bits = tab + max_slots;
    S.slots.count = tab + 2 * max_slots;
    S.slots.first = tab + 3 * max_slots;
    S.slots.tile0 = tab + 4 * max_slots;  // max_slots + 1 entries

    const int warp = threadIdx.x >> 5;
    // slot table: routed experts with at least min_count tokens, then the shared expert
    // (router mode: one slot holding every token)
    if (warp == 0 && P.phase == 2) {
        if (threadIdx.x == 0) {
            S.slots.expert[0] = -1;
            S.slots.count[0] = P.f.T;
            S.slots.first[0] = 0;
            S.slots.n = 1;
            S.slots.tile0[0] = 0;
            S.slots.tile0[1] = ((P.f.T + MAXN - 1) / MAXN) * n_mtiles(P);
        }
    } else if (warp == 0) {
        const int n_active = min(P.f.active[0], P.f.max_active);
        int n = 0;
        for (int a0 = 0; a0 < n_active; a0 += 32) {
            const int a = a0 + threadIdx.x;
            int e = -1, cnt = 0, f = 0;
            if (a < n_active) {
                e = P.f.active[1 + a];
                if (e >= 0 && e < P.f.E) {
                    f = P.f.offsets[e];
                    cnt = P.f.offsets[e + 1] - f;
                }
            }
            const bool take = a < n_active && e >= 0 && e < P.f.E && cnt >= P.min_count && cnt > 0;
            const unsigned m = __ballot_sync(0xffffffffu, take);
            if (take) {
                const int pos = n + __popc(m & ((1u << threadIdx.x) - 1u));
                S.slots.expert[pos] = e;
                S.slots.count[pos] = cnt;
                S.slots.first[pos] = f;
            }
            n += __popc(m);
        }
        if (threadIdx.x == 0) {
            if (P.f.has_shared && P.f.T >= P.min_count) {
                S.slots.expert[n] = P.f.E;
                S.slots.count[n] = P.f.T;
                S.slots.first[n] = P.f.T * P.f.k;
                ++n;
            }
            S.slots.n = n;
            // tile prefix (tiles per slot = n-chunks x m-tiles)
            const int nmt = n_mtiles(P);
            int acc = 0;
            for (int a = 0; a < n; ++a) {
                S.slots.tile0[a] = acc;
                acc += ((S.slots.count[a] + MAXN - 1) / MAXN) * nmt;
            }
            S.slots.tile0[n] = acc;
        }
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&S.full_a[s], DQ_THREADS / 32);  // one arrival per dequant warp
            mbar_init(&S.full_b[s], BPROD_THREADS);
            mbar_init(&S.empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&S.acc_full[b], 1);
            mbar_init(&S.acc_empty[b], 4);
        }
        mbar_init(S.fin, 1);
        *S.abort = 0;
        mbar_fence_init();
    }
    if (warp == MMA_WARP) {
        tmem_alloc(S.tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // broadcast the slot count (written by warp 0) through shared memory
    __shared__ int n_slots_sh;
    if (threadIdx.x == 0) n_slots_sh = S.slots.n;
    __syncthreads();
    S.slots.n = n_slots_sh;
    const uint32_t tmem = *S.tmem_slot;
    const int total_tiles = S.slots.tile0[S.slots.n];

    if (warp < EPI_WARP0) role_dequant(P, S, total_tiles, tmem);
    else if (warp < BPROD_WARP0) role_epilogue(P, S, total_tiles, tmem);
    else if (warp < MMA_WARP) role_tokens(P, S, total_tiles);
    else if (threadIdx.x == MMA_WARP * 32) role_mma(P, S, total_tiles, tmem);

    tc_fence_before();
    __syncthreads();
    if (warp == MMA_WARP) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

// x (bf16) -> fp16 with a range check; the tensor-core path stages x in fp16.
__global__ void x_to_f16_kernel(const uint16_t *__restrict__ x, size_t n, uint16_t *__restrict__ x16,
                                int32_t *status) {
    bool bad = false;
    for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n / 8;
         i += static_cast<size_t>(gridDim.x) * blockDim.x) {
        const uint4 v = reinterpret_cast<const uint4 *>(x)[i];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float a = bf16lo(w[j]), b = bf16hi(w[j]);
            bad |= !(fabsf(a) <= 65504.0f) || !(fabsf(b) <= 65504.0f);
            o[j] = h2(__half_as_ushort(__float2half_rn(a)), __half_as_ushort(__float2half_rn(b)));
        }
        reinterpret_cast<uint4 *>(x16)[i] = make_uint4(o[0], o[1], o[2], o[3]);
    }
    if (__any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0) status_or(status, MOE_STATUS_FP16_RANGE);
}

}  // namespace gemm
}  // namespace moe

namespace {
size_t align256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

size_t gemm_smem_bytes(int max_slots) {
    return 1024 + moe::gemm::STAGES * moe::gemm::STAGE_BYTES + moe::gemm::RAW * moe::gemm::RAW_BYTES +
           (3 * moe::gemm::STAGES + 5) * 8 + 16 + sizeof(int) * (5 * static_cast<size_t>(max_slots) + 1);
}
}  // namespace

size_t moe_ffn_gemm_workspace(const moe_layer_weights *w, int T, int k) {
    const size_t x16 = align256(static_cast<size_t>(T) * w->H * 2);
    const size_t h16 = align256((static_cast<size_t>(T) * k + T) * w->I * 2);
    return x16 + h16;
}

constexpr size_t kMaxDynSmem = 232448 - 1024;  // 227 KB opt-in limit per CTA on sm_100, less static smem

cudaError_t moe_configure_ffn_gemm() {
    return cudaFuncSetAttribute(moe::gemm::ffn_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(kMaxDynSmem));
}

bool moe_ffn_gemm_supported(int H, int I) {
    return H % moe::gemm::BM == 0 && I % (moe::gemm::BM / 2) == 0 && H % moe::gemm::BK == 0 &&
           I % moe::gemm::BK == 0;
}

bool moe_router_gemm_supported(int T, int H, int E) {
    return T >= 64 && E % moe::gemm::BM == 0 && H % moe::gemm::BK == 0;
}

// Router logits on the tensor cores: logits[t][e] = x[t] . w_router[e] + bias[e].
cudaError_t moe_launch_router_gemm(const uint16_t *x, const uint16_t *wr, const float *bias, int T, int H, int E,
                                   float *logits, cudaStream_t s) {
    moe::gemm::Params P{};
    P.f.wait_limit = moe::kWaitLimitCycles;
    P.f.w.H = H;
    P.f.w.I = 128;
    P.f.E = E;
    P.f.T = T;
    P.f.k = 1;
    P.f.max_active = 1;
    P.f.x = x;
    P.phase = 2;
    P.wr = wr;
    P.bias = bias;
    P.logits = logits;
    P.min_count = 1;
    int dev = 0, sms = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int tiles = ((T + moe::gemm::MAXN - 1) / moe::gemm::MAXN) * (E / moe::gemm::BM);
    const int grid = tiles < sms ? tiles : sms;
    moe::gemm::ffn_gemm_kernel<<<grid, moe::gemm::THREADS, gemm_smem_bytes(2), s>>>(P);
    return cudaGetLastError();
}

// Runs the experts with at least `min_count` tokens (and the shared expert when
// T >= min_count) through the two tensor-core GEMMs.
cudaError_t moe_launch_ffn_gemm(const moe::FfnParams &f, void *ws, size_t, cudaStream_t s, int min_count) {
    moe::gemm::Params P;
    P.f = f;
    P.min_count = min_count;
    char *base = static_cast<char *>(ws);
    P.x16 = reinterpret_cast<uint16_t *>(base);
    P.h16 = reinterpret_cast<uint16_t *>(base + align256(static_cast<size_t>(f.T) * f.w.H * 2));
    const size_t nx = static_cast<size_t>(f.T) * f.w.H;
    moe::gemm::x_to_f16_kernel<<<148 * 4, 256, 0, s>>>(f.x, nx, const_cast<uint16_t *>(P.x16), f.status);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const size_t smem = gemm_smem_bytes(f.max_active + 1);
    if (smem > kMaxDynSmem) return cudaErrorInvalidConfiguration;  // too many experts for the slot tables
    for (int phase = 0; phase < 2; ++phase) {
        P.phase = phase;
        moe::gemm::ffn_gemm_kernel<<<sms, moe::gemm::THREADS, smem, s>>>(P);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}
