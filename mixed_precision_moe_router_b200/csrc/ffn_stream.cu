// Tiered expert FFN, GEMV path: one persistent launch that streams every
// touched expert's packed rows once through a shared-memory ring and runs the
// dot products on the tensor cores against up to 8 token columns at a time.
//
// [P1] "step 4: three shelves, all on the GPU": mul_mat_id runs each word
// through its chosen experts, each shelf computes only the ids on it and the
// shelf results add up; the decode kernel fuses gate, up and the activation.
//
// Design (B200):
//  * Work is a list of tiles.  For every slot (an active expert whose token
//    count is in (0, max_count], and the shared expert) there are gate_up
//    tiles of 8R gate rows plus the 8R matching up rows, and down tiles of
//    16R rows, with R the largest power of two <= 8 such that a tile holds at
//    most 32K codes.  Each CTA takes a contiguous, cost-balanced share of the
//    gate_up tiles and then of the down tiles, so 8-, 4- and 3-bit experts
//    spread evenly over the SMs.  The prologue turns that share into a tile
//    range per slot, so walking the list is integer increments.
//  * Two consumer groups of 8 warps take alternate tiles of the CTA's list,
//    so one group's barriers, epilogue and waits overlap the other's
//    arithmetic.  Each group stages its own tiles into a shared-memory ring
//    with TMA tensor copies (cp.async.bulk.tensor) that complete on the
//    stage's mbarrier.  A gate_up tile is one 5-D copy when its rows are
//    whole 128-byte lines: [gate|up][8R rows][lines, padded to an odd count
//    with zero-filled out-of-range lines][128 bytes]; otherwise, and for down
//    tiles, one copy per 128-byte column chunk.  Either way the copies store
//    the tile with the TMA swizzle, which makes the fragment reads below
//    bank-conflict free, and one more copy brings the scales.
//  * 8 compute warps split a tile into R row subtiles x 8/R K slices.  For
//    each 32-weight block a warp turns its codes into exact fp16 integers
//    (|q| <= 127), multiplies them with fp16 activation fragments on the
//    tensor cores (mma.sync m16n8k16: exact products, fp32 accumulation) and
//    adds d * partial into fp32 accumulators.  The only roundings besides fp32
//    accumulation are bf16 x -> fp16 (exact for |x| in [2^-14, 65504]) and the
//    split of the fp32 intermediate h into two fp16 columns hi + lo (relative
//    error <= 2^-22).  Dequantisation is paid once per tile for up to 8 tokens;
//    more tokens take further passes over the resident tile.
//  * K slices are summed in shared memory in a fixed order.  gate_up tiles
//    write h = silu(g) * u and count themselves done per slot; a down tile
//    waits (bounded) for its slot's count before reading h, while its weights
//    may already be in flight.  The grid is launched cooperatively so every
//    CTA is resident and the waits resolve.
#include <cuda.h>

#include <cstring>
#include <map>
#include <mutex>

#include "common.cuh"
#include "ffn.cuh"
#include "sync.cuh"

namespace moe {

constexpr int kWarps = 8;                          // compute warps of a group (they split a tile)
constexpr int kThreads = kWarps * 32;              // threads of a group
constexpr int kGroups = 2;                         // consumer groups, taking alternate tiles
constexpr int kBlockThreads = kGroups * kThreads;
constexpr int kBarGroup0 = 1;                      // named barrier of group g: kBarGroup0 + g
constexpr int kStager = 32;  // the thread of a group that stages its tiles: lane 0 of its second
                             // warp, so the staging overlaps the epilogue (low threads first)
constexpr int kMaxStages = 6;
constexpr int kStageBytes = 40 * 1024;
constexpr int kMaxK = 2048;
constexpr int kMaxSmemEntries = 2048;  // token-entry tables kept in shared memory up to this size
constexpr int kTokPerPass = 8;         // gate_up token columns per pass over a resident tile
constexpr int kRedBytes = kWarps * 32 * 4 * 4;

// ---------------------------------------------------------------------------
// tile geometry
// ---------------------------------------------------------------------------
__host__ __device__ __forceinline__ int rows_pow2(int K) {
    int R = 1;
    while (R < 8 && 2 * R * K <= 2048) R *= 2;
    return R;
}

// Swizzle width of a row of `bytes` bytes: the largest of 128, 64 and 32 that
// divides it (its 16-byte chunks are permuted within that span), else 16 (no
// swizzle).
__host__ __device__ __forceinline__ int swizzle_width(int bytes) {
    return bytes % 128 == 0 ? 128 : (bytes % 64 == 0 ? 64 : (bytes % 32 == 0 ? 32 : 16));
}

struct Geo {
    int K, R, rows;  // row subtiles and rows per tile
    int rb, sb;      // code and scale bytes per row
    int W, lw;       // code swizzle width (and log2): the tile is stored as column chunks of W bytes
    int Ws;          // scale swizzle width, 0 when the scales come as plain bulk copies
    int nb, bps;     // 32-weight blocks per row, blocks per K slice
    int pad, nc1;    // padded row-major layout (one 5-D copy per tile): 128-byte lines per row
    int cb;          // code bytes of a staged tile (the scales follow)
};

__host__ __device__ __forceinline__ Geo geo(int K, int bits) {
    Geo g;
    g.K = K;
    g.R = rows_pow2(K);
    g.rows = 16 * g.R;
    g.rb = K * bits / 8;
    g.sb = K / 16;
    g.W = swizzle_width(g.rb);
    g.lw = g.W == 128 ? 7 : (g.W == 64 ? 6 : (g.W == 32 ? 5 : 4));
    // the scale box is a whole row: swizzled only when the row is 32, 64 or 128 bytes
    g.Ws = g.sb % 16 != 0 ? 0 : ((g.sb == 32 || g.sb == 64 || g.sb == 128) ? g.sb : 16);
    g.nb = K / 32;
    const int S = kWarps / g.R;
    g.bps = ((g.nb + S - 1) / S + 1) & ~1;  // even, so blocks go in pairs
    g.pad = 0;
    g.nc1 = 0;
    g.cb = g.rows * g.rb;
    return g;
}

// gate_up tiles: when the rows are whole 128-byte lines and the padded tile
// fits a stage, one 5-D copy stages the whole tile.  Each row then takes nc1
// lines: its rb / 128 lines plus one or two out-of-range lines (zero-filled,
// no memory traffic) so that nc1 is odd; the 128-byte swizzle then puts the 8
// rows an mma reads at one offset into 8 different 16-byte bank groups.
__host__ __device__ __forceinline__ Geo geo_gu(int K, int bits) {
    Geo g = geo(K, bits);
    if (g.W == 128) {
        const int n = g.rb / 128;
        const int nc1 = n + 1 + (n & 1);
        if (nc1 <= 256 && g.rows * (nc1 * 128 + g.sb) <= kStageBytes) {
            g.pad = 1;
            g.nc1 = nc1;
            g.cb = g.rows * nc1 * 128;
        }
    }
    return g;
}

__host__ __device__ __forceinline__ int stage_bytes(const Geo &g) { return g.cb + g.rows * g.sb; }

// XOR that the TMA swizzle of width W applies to the 16-byte chunk index of
// row r of a box (boxes start on a swizzle-atom boundary and hold a multiple
// of 8 rows)
__device__ __forceinline__ int swz(int r, int W) {
    return W == 128 ? (r & 7) << 4 : (W == 64 ? ((r >> 1) & 3) << 4 : (W == 32 ? ((r >> 2) & 1) << 4 : 0));
}

// Byte offset of byte o of row r in a staged tile.  Column-chunk layout: the
// tile is stored as column chunks of W bytes with the TMA swizzle (xr =
// swz(r, W)).  Padded layout: row r starts at 128-byte line xr = r * nc1 and
// the swizzle permutes the 16-byte units of line L by L mod 8.
template <bool PAD>
__device__ __forceinline__ int tile_off(int o, int r, const Geo &G, int xr) {
    if constexpr (PAD) {
        const int line = xr + (o >> 7);
        return (line << 7) + ((o & 127) ^ ((line & 7) << 4));
    } else {
        return (o >> G.lw) * (G.rows << G.lw) + (r << G.lw) + ((o & (G.W - 1)) ^ xr);
    }
}

// xr of row r for tile_off
template <bool PAD>
__device__ __forceinline__ int row_x(int r, const Geo &G) {
    if constexpr (PAD) return r * G.nc1;
    else return swz(r, G.W);
}


// x fragments in shared memory: [column][block][thread t][8 halves], with a
// column stride that keeps the 16-byte reads of two columns in different banks.
__host__ __device__ __forceinline__ int xf_col_stride(int K) { return (K / 32) * 64 + 64; }

__host__ __device__ __forceinline__ int down_ntiles(int I) { return I <= 1024 ? 2 : 1; }

// Fragment columns a pass can use with at most T tokens: gate_up one per
// token (up to 8), down hi + lo per token in n-tiles of 8 (column 8*(n/4) +
// 2*(n%4) + 1 is the last one written for token n).
__host__ __device__ __forceinline__ int xf_bytes(int H, int I, int T) {
    const int cg = T < kTokPerPass ? T : kTokPerPass;
    const int nd = T < 4 * down_ntiles(I) ? T : 4 * down_ntiles(I);
    const int cd = nd <= 4 ? 2 * nd : 8 + 2 * (nd - 4);
    const int a = cg * xf_col_stride(H);
    const int b = cd * xf_col_stride(I);
    const int m = a > b ? a : b;
    return (m + 127) & ~127;
}

// Thread index within its consumer group, and the group.
__device__ __forceinline__ int gtid() { return threadIdx.x & (kThreads - 1); }
__device__ __forceinline__ int group_of_thread() { return threadIdx.x / kThreads; }

// tokens of one pass: gate_up tiles use one column per token, down tiles two
// (h = hi + lo) in n-tiles of 8 columns
__host__ __device__ __forceinline__ int tokens_per_pass(int phase, int I) {
    return phase == 0 ? kTokPerPass : 4 * down_ntiles(I);
}

struct SlotTabs {  // per expert slot, in shared memory
    int *expert, *bits, *count, *first;
    int *tok, *row;  // entries [first, first + count) of every slot: token and h/y row
};

// Table base pointers of the shelves (index < n_tiers) and of the shared
// expert (index n_tiers), copied from the parameters into shared memory so
// that they can be indexed at run time.
struct TierPtrs {
    const uint8_t *gq, *gs, *dq, *ds;
    int bits, first, n, pad;
};

// Balancing weight of a tile: a fixed share for the per-tile work (waits,
// barriers, epilogue), its bytes, and a per-weight share for the
// dequantise-and-multiply work of each pass (3-bit codes take the most).
constexpr long long kTileFixedCost = 65536;
__device__ __forceinline__ long long tile_cost(const FfnParams &p, int phase, int bits, int count) {
    const int K = phase == 0 ? p.w.H : p.w.I;
    const long long rows = 16 * rows_pow2(K);
    const int tp = tokens_per_pass(phase, p.w.I);
    const long long passes = (count + tp - 1) / tp;
    return kTileFixedCost + rows * (K * bits / 8 + K / 16) + passes * (rows * K / 3) * (bits == 3 ? 3 : 2);
}

__device__ __forceinline__ int tiles_per_slot(const FfnParams &p, int phase) {
    return phase == 0 ? p.w.I / (8 * rows_pow2(p.w.H)) : p.w.H / (16 * rows_pow2(p.w.I));
}

// Per-slot tile costs and inclusive prefix sums of the slots' total costs,
// per phase, built once in the prologue (shared memory).
struct Sched {
    long long *tc0, *tc1;    // cost of one tile of each slot
    long long *pre0, *pre1;  // inclusive prefix sums of the slots' total costs
    int2 *rng0, *rng1;       // per slot: this CTA's tiles of it, [b0, b1)
    int *fl;                 // per phase: first and last slot with tiles in this CTA (last < first: none)
};

// floor(x / y) for 0 <= x < 2^52, 0 < y: a double quotient corrected to the
// exact integer result (the 64-bit integer divide is a long routine).
__device__ __forceinline__ long long div_floor(long long x, long long y) {
    long long q = static_cast<long long>(static_cast<double>(x) / static_cast<double>(y));
    while (q * y > x) --q;
    while ((q + 1) * y <= x) ++q;
    return q;
}

// This CTA's tiles, in order: its cost-balanced contiguous share of all
// gate_up tiles (phase 0), then of all down tiles (phase 1).  phase == 2 once
// the list is exhausted.  The per-slot tile ranges are computed once in the
// prologue, so stepping is a few integer operations.
struct TileIt {
    int phase, a, b, b1;  // current tile: slot a, tile b; b1 ends this slot's range
};

// Tiles of a slot (nt tiles of cost tb) that start before cost offset x from
// the slot's start: ceil(x / tb) clamped to [0, nt].  A float quotient
// corrected to the exact integer (the quotient is below nt <= 256 here).
__device__ __forceinline__ int tiles_before(long long x, long long tb, int nt) {
    if (x <= 0) return 0;
    if (x >= nt * tb) return nt;
    long long q = static_cast<long long>(__fdividef(static_cast<float>(x), static_cast<float>(tb)));
    while (q * tb < x) ++q;
    while (q > 0 && (q - 1) * tb >= x) --q;
    return static_cast<int>(q);
}

__device__ __forceinline__ bool it_enter(const Sched &sc, TileIt &it, int phase) {
    const int f = sc.fl[2 * phase], l = sc.fl[2 * phase + 1];
    if (f > l) return false;
    const int2 r = (phase == 0 ? sc.rng0 : sc.rng1)[f];
    it.phase = phase;
    it.a = f;
    it.b = r.x;
    it.b1 = r.y;
    return true;
}

__device__ __forceinline__ void it_begin(const FfnParams &p, const Sched &sc, int n_slots, TileIt &it) {
    (void)p;
    it.phase = 2;
    if (n_slots == 0) return;
    if (!it_enter(sc, it, 0) && !it_enter(sc, it, 1)) it.phase = 2;
}

// Slots strictly between a phase's first and last slot lie wholly inside the
// CTA's contiguous cost range, so each of them has tiles here.
__device__ __forceinline__ void it_next(const FfnParams &p, const Sched &sc, int n_slots, TileIt &it) {
    (void)p;
    (void)n_slots;
    if (it.phase == 2) return;
    if (++it.b < it.b1) return;
    if (it.a < sc.fl[2 * it.phase + 1]) {
        ++it.a;
        const int2 r = (it.phase == 0 ? sc.rng0 : sc.rng1)[it.a];
        it.b = r.x;
        it.b1 = r.y;
        return;
    }
    if (it.phase == 0 && it_enter(sc, it, 1)) return;
    it.phase = 2;
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

// ---------------------------------------------------------------------------
// Codes -> exact fp16 integers: four half2 pairs per row, block and thread.
// A code c placed at mantissa bit s under the exponent of 2^(10-s) reads as
// the half 2^(10-s) + c; subtracting 2^(10-s) + offset leaves q exactly.
// Thread t owns weights 8t .. 8t+7 of each 32-weight block, paired as
// (2p, 2p+1) for 8-bit codes and (p, p+4) for 4- and 3-bit codes, p = 0..3.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

__device__ __forceinline__ uint32_t hsub2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

template <int BITS, bool PAD>
__device__ __forceinline__ void dequant8(const uint8_t *tile, const Geo &G, int r, int xr, int b, int t,
                                         uint32_t (&P)[4]) {
    if constexpr (BITS == 8) {
        const uint2 w = *reinterpret_cast<const uint2 *>(tile + tile_off<PAD>(32 * b + 8 * t, r, G, xr));
        const uint32_t u0 = w.x ^ 0x80808080u, u1 = w.y ^ 0x80808080u;  // c = q + 128
        constexpr uint32_t kBias = 0x64806480u;                         // 1024 + 128
        P[0] = hsub2(prmt(u0, 0x64646464u, 0x4140u), kBias);
        P[1] = hsub2(prmt(u0, 0x64646464u, 0x4342u), kBias);
        P[2] = hsub2(prmt(u1, 0x64646464u, 0x4140u), kBias);
        P[3] = hsub2(prmt(u1, 0x64646464u, 0x4342u), kBias);
    } else if constexpr (BITS == 4) {
        // nibble i of the word at byte 16b + 4t is weight 8t + i (c = q + 8)
        const uint32_t v = *reinterpret_cast<const uint32_t *>(tile + tile_off<PAD>(16 * b + 4 * t, r, G, xr));
        const uint32_t v8 = v >> 8;
        P[0] = hsub2((v & 0x000F000Fu) | 0x64006400u, 0x64086408u);   // 1024 + c - 1032
        P[1] = hsub2((v & 0x00F000F0u) | 0x54005400u, 0x54805480u);   // 64 + c - 72
        P[2] = hsub2((v8 & 0x000F000Fu) | 0x64006400u, 0x64086408u);
        P[3] = hsub2((v8 & 0x00F000F0u) | 0x54005400u, 0x54805480u);
    } else {
        // low plane: bits 0-1 of weight 8t+i at bit 2i of the u16 at byte 8b+2t;
        // high plane: bit 2 at bit i of byte K/4 + 4b + t (c = q + 4)
        const uint32_t lo16 = *reinterpret_cast<const uint16_t *>(tile + tile_off<PAD>(8 * b + 2 * t, r, G, xr));
        const uint32_t hb = tile[tile_off<PAD>(G.K / 4 + 4 * b + t, r, G, xr)];
        const uint32_t X = prmt(lo16, 0u, 0x4140u);  // weights i and i+4 16 bits apart
        const uint32_t Y = hb * 0x4004u;             // hb << 2 | hb << 14
        P[0] = hsub2((X & 0x00030003u) | (Y & 0x00040004u) | 0x64006400u, 0x64046404u);           // 1024 + c - 1028
        P[1] = hsub2((X & 0x000C000Cu) | ((Y << 1) & 0x00100010u) | 0x5C005C00u, 0x5C105C10u);  // 256 + c - 260
        P[2] = hsub2((X & 0x00300030u) | ((Y << 2) & 0x00400040u) | 0x54005400u, 0x54405440u);  // 64 + c - 68
        P[3] = hsub2((X & 0x00C000C0u) | ((Y << 3) & 0x01000100u) | 0x4C004C00u, 0x4D004D00u);  // 16 + c - 20
    }
}

// D = A B + D on one m16n8k16 tile (fp16 inputs, fp32 accumulation).
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float2 half2_to_float2(uint32_t v) {
    return __half22float2(*reinterpret_cast<const __half2 *>(&v));
}

// One warp's share of a tile: stage rows rA (accumulator rows g) and rB (rows
// g + 8), blocks [b0, b1), NT n-tiles of 8 columns.  acc[nt] follows the m16n8
// accumulator layout: (row g, col 2t), (g, 2t+1), (g+8, 2t), (g+8, 2t+1).
struct TileAcc {
    float acc[2][4];
};

template <int BITS, int NT, bool PAD>
__device__ __forceinline__ TileAcc warp_tile(const uint8_t *stage, const Geo G, int rA, int rB, int b0, int b1,
                                          const uint8_t *xf, int cs, int ncol0, int ncol1) {
    TileAcc out;
    float (&acc)[2][4] = out.acc;
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const int xa = row_x<PAD>(rA, G), xb = row_x<PAD>(rB, G);
    // scales: [row][sb] after the codes, swizzled at width Ws (or plain)
    const uint8_t *scl = stage + G.cb;
    const int sxa = G.Ws ? swz(rA, G.Ws) : 0, sxb = G.Ws ? swz(rB, G.Ws) : 0;
    const uint8_t *xg = xf + g * cs + t * 16;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[nt][i] = 0.f;
#pragma unroll 2
    for (int b = b0; b < b1; b += 2) {
        const float2 da = half2_to_float2(*reinterpret_cast<const uint32_t *>(scl + rA * G.sb + ((2 * b) ^ sxa)));
        const float2 db = half2_to_float2(*reinterpret_cast<const uint32_t *>(scl + rB * G.sb + ((2 * b) ^ sxb)));
        uint32_t PA[2][4], PB[2][4];
#pragma unroll
        for (int bb = 0; bb < 2; ++bb) {
            dequant8<BITS, PAD>(stage, G, rA, xa, b + bb, t, PA[bb]);
            dequant8<BITS, PAD>(stage, G, rB, xb, b + bb, t, PB[bb]);
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            uint4 X[2];
#pragma unroll
            for (int bb = 0; bb < 2; ++bb) {
                X[bb] = make_uint4(0u, 0u, 0u, 0u);
                if (g < (nt == 0 ? ncol0 : ncol1))
                    X[bb] = *reinterpret_cast<const uint4 *>(xg + nt * 8 * cs + (b + bb) * 64);
            }
            // four independent products: two k16 halves of two blocks
            float c[4][4] = {};
#pragma unroll
            for (int bb = 0; bb < 2; ++bb) {
                mma16816(c[2 * bb], PA[bb][0], PB[bb][0], PA[bb][1], PB[bb][1], X[bb].x, X[bb].y);
                mma16816(c[2 * bb + 1], PA[bb][2], PB[bb][2], PA[bb][3], PB[bb][3], X[bb].z, X[bb].w);
            }
#pragma unroll
            for (int bb = 0; bb < 2; ++bb) {
                const float dA = bb ? da.y : da.x, dB = bb ? db.y : db.x;
                acc[nt][0] = fmaf(dA, c[2 * bb][0] + c[2 * bb + 1][0], acc[nt][0]);
                acc[nt][1] = fmaf(dA, c[2 * bb][1] + c[2 * bb + 1][1], acc[nt][1]);
                acc[nt][2] = fmaf(dB, c[2 * bb][2] + c[2 * bb + 1][2], acc[nt][2]);
                acc[nt][3] = fmaf(dB, c[2 * bb][3] + c[2 * bb + 1][3], acc[nt][3]);
            }
        }
    }
    return out;
}

// fp32 -> fp16 bits, noting values outside the fp16 range (or NaN)
__device__ __forceinline__ uint16_t to_f16(float v, bool &bad) {
    bad |= !(fabsf(v) <= 65504.f);
    return __half_as_ushort(__float2half_rn(v));
}

__device__ __forceinline__ uint32_t pack_h2(uint16_t lo, uint16_t hi) {
    return static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
}

// 8 consecutive values of a block (weights 8t .. 8t+7) in the pair order of
// the codes, as 4 half2.
__device__ __forceinline__ uint4 pack_frag(const uint16_t (&v)[8], int bits) {
    uint4 r;
    if (bits == 8) {
        r.x = pack_h2(v[0], v[1]);
        r.y = pack_h2(v[2], v[3]);
        r.z = pack_h2(v[4], v[5]);
        r.w = pack_h2(v[6], v[7]);
    } else {
        r.x = pack_h2(v[0], v[4]);
        r.y = pack_h2(v[1], v[5]);
        r.z = pack_h2(v[2], v[6]);
        r.w = pack_h2(v[3], v[7]);
    }
    return r;
}

struct StreamSmem {
    uint8_t *stages;
    uint8_t *xf;             // [kGroups][xf_size]
    int xf_size;
    float4 *red;             // [kGroups][kWarps * 32]
    uint64_t *full;          // per stage: copies landed
    int *abort;
    // per group: how many of its tiles (g, g + 2, ...) are staged, and the
    // iterator at the next one to stage
    struct Ahead { TileIt it; int n; } *ahead;
    SlotTabs st;
    Sched sc;
    int *tier, *jloc;   // per slot: shelf index (n_tiers = shared) and index within the shelf
    TierPtrs *tp;       // [MOE_MAX_TIERS + 1]
    Geo *geo;           // [phase][8-, 4-, 3-bit]
};

__device__ __forceinline__ int bits_idx(int bits) { return bits == 8 ? 0 : (bits == 4 ? 1 : 2); }

// Tensor maps of the shelf tables (index < n_tiers) and of the shared expert
// (index n_tiers), built on the host:
//   gq: 4-D [expert][gate|up][I][rb_H] bytes, box {W_H, 8R, 2, 1}
//   gs: 4-D [expert][gate|up][I][sb_H] bytes, box {sb_H, 8R, 2, 1}
//   dq: 3-D [expert][H][rb_I], box {W_I, 16R, 1};  ds: 3-D [expert][H][sb_I]
// each stored with the swizzle of its inner box width.
struct StreamMaps {
    CUtensorMap gq[MOE_MAX_TIERS + 1], gs[MOE_MAX_TIERS + 1];
    CUtensorMap dq[MOE_MAX_TIERS + 1], ds[MOE_MAX_TIERS + 1];
};

__device__ __forceinline__ void tma_3d(void *dst, const CUtensorMap *map, int x, int y, int z, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
        "[%5];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tma_4d(void *dst, const CUtensorMap *map, int x, int y, int z, int w,
                                       uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, "
        "%5}], [%6];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(w), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tma_5d(void *dst, const CUtensorMap *map, int x, int y, int z, int w, int v,
                                       uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, "
        "%5, %6}], [%7];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(w), "r"(v), "r"(smem_u32(bar))
        : "memory");
}

// Stage the codes and scales of tile (phase, a, tile) into `dst`, completing
// on `bar`: a gate_up tile is its 8R gate rows and the matching 8R up rows, a
// down tile 16R consecutive rows; codes as column chunks of W bytes.
__device__ __forceinline__ void issue_tile(const FfnParams &p, const StreamMaps &M, const StreamSmem &S, int phase,
                                           int a, int tile, uint8_t *dst, uint64_t *bar) {
    const int I = p.w.I;
    const Geo &G = S.geo[phase * 3 + bits_idx(S.st.bits[a])];
    const int ti = S.tier[a], j = S.jloc[a];
    const TierPtrs &T = S.tp[ti];
    uint8_t *dsc = dst + G.cb;
    const int chunk = G.rows << G.lw;  // bytes of one column chunk of the tile
    mbar_expect_tx(bar, static_cast<uint32_t>(stage_bytes(G)));
    if (phase == 0) {
        const int half = 8 * G.R, P = tile * half;
        if (G.pad)  // one box: [gate|up][8R rows][nc1 lines][128 bytes]
            tma_5d(dst, &M.gq[ti], 0, 0, P, 0, j, bar);
        else
            for (int c = 0; c * G.W < G.rb; ++c) tma_4d(dst + c * chunk, &M.gq[ti], c * G.W, P, 0, j, bar);
        if (G.Ws) {
            tma_4d(dsc, &M.gs[ti], 0, P, 0, j, bar);
        } else {
            const uint8_t *sc = T.gs + static_cast<size_t>(j) * 2 * I * G.sb;
            bulk_g2s(dsc, sc + static_cast<size_t>(P) * G.sb, half * G.sb, bar);
            bulk_g2s(dsc + half * G.sb, sc + static_cast<size_t>(I + P) * G.sb, half * G.sb, bar);
        }
    } else {
        const int Q = tile * G.rows;
        for (int c = 0; c * G.W < G.rb; ++c) tma_3d(dst + c * chunk, &M.dq[ti], c * G.W, Q, j, bar);
        if (G.Ws) {
            tma_3d(dsc, &M.ds[ti], 0, Q, j, bar);
        } else {
            const uint8_t *sc = T.ds + static_cast<size_t>(j) * p.w.H * G.sb;
            bulk_g2s(dsc, sc + static_cast<size_t>(Q) * G.sb, G.rows * G.sb, bar);
        }
    }
}

// Barrier of one consumer group that also ANDs a flag over it.
__device__ __forceinline__ bool bar_and(bool ok) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(ok ? 1u : 0u), "r"(kBarGroup0 + group_of_thread()), "n"(kThreads)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ void bar_compute() { named_bar_sync(kBarGroup0 + group_of_thread(), kThreads); }


// gate_up fragments of one pass: column n holds the token of entry pass*8 + n.
__device__ __forceinline__ bool build_xf_gu(const FfnParams &p, const SlotTabs &st, int a, int pass, int ntok,
                                         int bits, uint8_t *xf) {
    bool bad = false;
    const int H = p.w.H, nb = H / 32, cs = xf_col_stride(H);
    const int n_chunks = ntok * nb * 4;
    for (int i = gtid(); i < n_chunks; i += kThreads) {
        const int n = i / (nb * 4), rem = i % (nb * 4);  // rem = 4 * block + t
        int tok, row;
        slot_entry(p, st, a, pass * kTokPerPass + n, tok, row);
        const uint4 q = *reinterpret_cast<const uint4 *>(p.x + static_cast<size_t>(tok) * H + 8 * rem);
        const uint32_t w[4] = {q.x, q.y, q.z, q.w};
        uint16_t v[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            v[2 * j] = to_f16(bf16lo(w[j]), bad);
            v[2 * j + 1] = to_f16(bf16hi(w[j]), bad);
        }
        *reinterpret_cast<uint4 *>(xf + n * cs + rem * 16) = pack_frag(v, bits);
    }
    return bad;
}

// down fragments of one pass: in n-tile nt, column 2m holds hi and column
// 2m + 1 lo of h for the token of entry pass*tp + 4nt + m.
__device__ __forceinline__ bool build_xf_dn(const FfnParams &p, const SlotTabs &st, int a, int pass, int ntok,
                                         int bits, uint8_t *xf) {
    bool bad = false;
    const int I = p.w.I, nb = I / 32, cs = xf_col_stride(I);
    const int tp = tokens_per_pass(1, I);
    const int n_chunks = ntok * nb * 4;
    for (int i = gtid(); i < n_chunks; i += kThreads) {
        const int n = i / (nb * 4), rem = i % (nb * 4);
        int tok, row;
        slot_entry(p, st, a, pass * tp + n, tok, row);
        const float *src = p.h + static_cast<size_t>(row) * I + 8 * rem;
        const float4 f0 = __ldcg(reinterpret_cast<const float4 *>(src));
        const float4 f1 = __ldcg(reinterpret_cast<const float4 *>(src + 4));
        const float f[8] = {f0.x, f0.y, f0.z, f0.w, f1.x, f1.y, f1.z, f1.w};
        uint16_t hi[8], lo[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            hi[j] = to_f16(f[j], bad);
            lo[j] = __half_as_ushort(__float2half_rn(f[j] - __half2float(__ushort_as_half(hi[j]))));
        }
        const int col = (n >> 2) * 8 + 2 * (n & 3);
        *reinterpret_cast<uint4 *>(xf + col * cs + rem * 16) = pack_frag(hi, bits);
        *reinterpret_cast<uint4 *>(xf + (col + 1) * cs + rem * 16) = pack_frag(lo, bits);
    }
    return bad;
}

// This warp's partial sums of the resident tile, to red[warp][lane].
template <int BITS>
__device__ __forceinline__ void compute_tile(const FfnParams &p, const Geo &G, int phase, const uint8_t *stage,
                                             const uint8_t *xf, int ntok, float4 *red) {
    const int warp = gtid() >> 5, lane = threadIdx.x & 31;
    const int r = warp % G.R, s = warp / G.R;
    const int b0 = min(G.nb, s * G.bps), b1 = min(G.nb, (s + 1) * G.bps);
    const int cs = xf_col_stride(G.K);
    const int g = lane >> 2;
    if (phase == 0) {
        const TileAcc t = G.pad ? warp_tile<BITS, 1, true>(stage, G, 8 * r + g, 8 * G.R + 8 * r + g, b0, b1, xf, cs, ntok, 0)
                                : warp_tile<BITS, 1, false>(stage, G, 8 * r + g, 8 * G.R + 8 * r + g, b0, b1, xf, cs, ntok, 0);
        const float(&acc)[2][4] = t.acc;
        red[warp * 32 + lane] = make_float4(acc[0][0], acc[0][1], acc[0][2], acc[0][3]);
    } else {
        const int nc0 = 2 * max(0, min(4, ntok)), nc1 = 2 * max(0, min(4, ntok - 4));
        const TileAcc t = down_ntiles(p.w.I) == 2
                              ? warp_tile<BITS, 2, false>(stage, G, 16 * r + g, 16 * r + g + 8, b0, b1, xf, cs, nc0, nc1)
                              : warp_tile<BITS, 1, false>(stage, G, 16 * r + g, 16 * r + g + 8, b0, b1, xf, cs, nc0, nc1);
        const float(&acc)[2][4] = t.acc;
        // hi + lo columns of each token
        red[warp * 32 + lane] =
            make_float4(acc[0][0] + acc[0][1], acc[0][2] + acc[0][3], acc[1][0] + acc[1][1], acc[1][2] + acc[1][3]);
    }
}

// K slices summed in a fixed order; gate_up -> h = silu(g) * u, down -> y.
__device__ __forceinline__ void epilogue(const FfnParams &p, const SlotTabs &st, int phase, int a, int tile,
                                         int pass, int ntok, const float4 *red) {
    const int K = phase == 0 ? p.w.H : p.w.I;
    const int R = rows_pow2(K), S = kWarps / R;
    const float *rf = reinterpret_cast<const float *>(red);
    if (phase == 0) {
        const int I = p.w.I;
        const int n_out = R * 8 * ntok;
        for (int o = gtid(); o < n_out; o += kThreads) {
            const int n = o % ntok, rg = o / ntok, g = rg % 8, r = rg / 8;
            const int lane = 4 * g + (n >> 1), sub = n & 1;
            float gate = 0.f, up = 0.f;
            for (int s = 0; s < S; ++s) {
                const float *v = rf + ((r + R * s) * 32 + lane) * 4;
                gate += v[sub];
                up += v[2 + sub];
            }
            int tok, row;
            slot_entry(p, st, a, pass * kTokPerPass + n, tok, row);
            p.h[static_cast<size_t>(row) * I + tile * 8 * R + 8 * r + g] = gate / (1.0f + expf(-gate)) * up;
        }
    } else {
        const int H = p.w.H, tp = tokens_per_pass(1, p.w.I);
        const int n_out = R * 16 * ntok;
        for (int o = gtid(); o < n_out; o += kThreads) {
            const int rr = o % (R * 16), n = o / (R * 16);
            const int r = rr / 16, row16 = rr % 16;
            const int lane = 4 * (row16 % 8) + (n & 3), idx = 2 * (n >> 2) + row16 / 8;
            float v = 0.f;
            for (int s = 0; s < S; ++s) v += rf[((r + R * s) * 32 + lane) * 4 + idx];
            int tok, row;
            slot_entry(p, st, a, pass * tp + n, tok, row);
            float *dst = row >= p.T * p.k ? p.y_shared + static_cast<size_t>(row - p.T * p.k) * H
                                          : p.y_slots + static_cast<size_t>(row) * H;
            dst[tile * 16 * R + rr] = v;
        }
    }
}

// Advance an iterator by `n` tiles.
__device__ __forceinline__ void it_skip(const FfnParams &p, const Sched &sc, int n_slots, TileIt &it, int n) {
    for (int k = 0; k < n; ++k) it_next(p, sc, n_slots, it);
}

// The persistent FFN kernel body; `n_slots` slots are described in S.
//
// Two consumer groups of 8 warps take alternate tiles of the CTA's list
// (group g: tiles g, g + 2, ...), so one group's barriers, epilogue and
// dependency waits overlap the other's dequantise-and-multiply.  Tile i lives
// in stage i % nstages; nstages is even, so a stage always serves the same
// group.  The first nstages tiles are staged in the prologue; afterwards a
// group stages its tile i + nstages as soon as its barrier after the last
// pass over tile i shows the stage drained.  A group therefore never waits
// on copies the other group issues, and a group waiting on another slot's
// gate_up count cannot hold back the tiles that produce that count.
__device__ __forceinline__ void ffn_stream_body(const FfnParams &p, const StreamMaps &M, StreamSmem &S, int n_slots,
                                                int nstages) {
    const int grp = group_of_thread(), gt = gtid(), lane = threadIdx.x & 31;
    const int I = p.w.I;
    uint8_t *xf = S.xf + grp * S.xf_size;
    float4 *red = S.red + grp * kWarps * 32;
    const int gu_tiles = tiles_per_slot(p, 0);
    TileIt it;
    it_begin(p, S.sc, n_slots, it);
    it_skip(p, S.sc, n_slots, it, grp);
    if (gt == kStager) {
        // the group's stager stages its first nstages / 2 tiles
        StreamSmem::Ahead &ah = S.ahead[grp];
        ah.it = it;
        ah.n = 0;
        while (ah.n < nstages / kGroups && ah.it.phase < 2) {
            const int k = grp + kGroups * ah.n;
            issue_tile(p, M, S, ah.it.phase, ah.it.a, ah.it.b, S.stages + static_cast<size_t>(k) * kStageBytes,
                       &S.full[k]);
            it_skip(p, S.sc, n_slots, ah.it, kGroups);
            ++ah.n;
        }
    }
    int xf_key = -1;      // (slot, phase, pass) whose fragments xf holds
    int ready_slot = -1;  // a slot whose h is known to be complete
    int pend_tiles = 0;   // gate_up tiles of the current slot not yet counted
    int consumed = 0;     // this group's tiles whose copies have landed
    bool bad = false;
    int i = grp;
    for (; it.phase < 2; i += kGroups) {
        const int phase = it.phase, a = it.a, tile = it.b;
        const int s = i % nstages;
        if (phase == 0) {
            // gate_up fragments of the first pass do not depend on the tile:
            // build them while its copies are in flight (every reader of the
            // old fragments is past the previous tile's barriers, and the
            // barrier below orders these writes before the reads)
            const int key0 = (a * 2) * 65536;
            if (key0 != xf_key) {
                bad |= build_xf_gu(p, S.st, a, 0, min(kTokPerPass, S.st.count[a]), S.st.bits[a], xf);
                xf_key = key0;
            }
        }
        bool ok = mbar_wait(&S.full[s], (i / nstages) & 1);
        // one thread polls the slot's gate_up count (with backoff, so that
        // pollers do not crowd the counters' L2 slice); the barrier passes
        // the result on and orders every thread's reads of h after it
        if (phase == 1 && a != ready_slot && gt == 0) ok = ok && wait_geq_backoff(p.ctr + a, gu_tiles);
        if (!bar_and(ok && !*static_cast<volatile int *>(S.abort))) {
            if (gt == 0) {
                status_or(p.status, MOE_STATUS_TIMEOUT);
                *static_cast<volatile int *>(S.abort) = 1;
            }
            break;
        }
        ++consumed;
        if (phase == 1) ready_slot = a;
        const uint8_t *stage = S.stages + static_cast<size_t>(s) * kStageBytes;
        const int bits = S.st.bits[a], cnt = S.st.count[a];
        const Geo &G = S.geo[phase * 3 + bits_idx(bits)];
        const int tp = tokens_per_pass(phase, I);
        const int np = (cnt + tp - 1) / tp;
        for (int pass = 0; pass < np; ++pass) {
            const int ntok = min(tp, cnt - pass * tp);
            const int key = (a * 2 + phase) * 65536 + pass;
            if (key != xf_key) {  // the last readers of xf passed a barrier since
                bad |= phase == 0 ? build_xf_gu(p, S.st, a, pass, ntok, bits, xf)
                                  : build_xf_dn(p, S.st, a, pass, ntok, bits, xf);
                xf_key = key;
                bar_compute();
            }
            if (bits == 8)
                compute_tile<8>(p, G, phase, stage, xf, ntok, red);
            else if (bits == 4)
                compute_tile<4>(p, G, phase, stage, xf, ntok, red);
            else
                compute_tile<3>(p, G, phase, stage, xf, ntok, red);
            bar_compute();
            if (pass == np - 1 && gt == kStager) {
                // every warp of the group is past its reads of the stage:
                // stage this group's tile i + nstages into it
                StreamSmem::Ahead &ah = S.ahead[grp];
                if (ah.it.phase < 2) {
                    const int k = grp + kGroups * ah.n;  // == i + nstages
                    issue_tile(p, M, S, ah.it.phase, ah.it.a, ah.it.b,
                               S.stages + static_cast<size_t>(k % nstages) * kStageBytes, &S.full[k % nstages]);
                    it_skip(p, S.sc, n_slots, ah.it, kGroups);
                    ++ah.n;
                }
            }
            epilogue(p, S.st, phase, a, tile, pass, ntok, red);
            if (pass + 1 < np) bar_compute();  // red is written again by the next pass
        }
        it_skip(p, S.sc, n_slots, it, kGroups);
        if (phase == 0) {
            // when this group leaves the slot, count its gate_up tiles of it:
            // after every thread's h writes (barrier) and a fence, and before
            // this group waits on any other slot's count
            ++pend_tiles;
            if (it.phase != 0 || it.a != a) {
                bar_compute();
                if (gt == 0) {
                    __threadfence();
                    atomicAdd(p.ctr + a, pend_tiles);
                }
                pend_tiles = 0;
            }
        }
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) status_or(p.status, MOE_STATUS_FP16_RANGE);
    // after an abort, copies this group staged but never consumed must land
    // before the CTA exits (on a normal exit there are none)
    if (gt == kStager) {
        for (int m = consumed; m < S.ahead[grp].n; ++m) {
            const int k = grp + kGroups * m;
            if (!mbar_wait(&S.full[k % nstages], (k / nstages) & 1)) status_or(p.status, MOE_STATUS_TIMEOUT);
        }
    }
}

__global__ void __launch_bounds__(kBlockThreads, 1)
ffn_stream_kernel(const __grid_constant__ FfnParams p, const __grid_constant__ StreamMaps M, int nstages) {
    extern __shared__ __align__(1024) uint8_t smem[];
    StreamSmem S;
    S.stages = smem;
    S.xf_size = xf_bytes(p.w.H, p.w.I, p.T);
    S.xf = smem + static_cast<size_t>(nstages) * kStageBytes;
    S.red = reinterpret_cast<float4 *>(S.xf + kGroups * S.xf_size);
    S.full = reinterpret_cast<uint64_t *>(reinterpret_cast<uint8_t *>(S.red) + kGroups * kRedBytes);
    S.ahead = reinterpret_cast<StreamSmem::Ahead *>(S.full + kMaxStages);
    S.tp = reinterpret_cast<TierPtrs *>(S.ahead + kGroups);
    S.geo = reinterpret_cast<Geo *>(S.tp + MOE_MAX_TIERS + 1);
    S.abort = reinterpret_cast<int *>(S.geo + 6);
    int *tabs = S.abort + 2;
    const int max_slots = p.max_active + 1;
    S.st.expert = tabs;
    S.st.bits = tabs + max_slots;
    S.st.count = tabs + 2 * max_slots;
    S.st.first = tabs + 3 * max_slots;
    S.tier = tabs + 4 * max_slots;
    S.jloc = tabs + 5 * max_slots;
    // entry tables in shared memory when they fit, else read from global
    const int n_ent = p.T * p.k + p.T;
    const bool ent_smem = n_ent <= kMaxSmemEntries;
    S.st.tok = ent_smem ? tabs + 6 * max_slots : nullptr;
    S.st.row = ent_smem ? S.st.tok + n_ent : nullptr;
    // 8-byte aligned: every table before it has an even number of ints
    S.sc.rng0 = reinterpret_cast<int2 *>(tabs + 6 * max_slots + (ent_smem ? 2 * n_ent : 0));
    S.sc.rng1 = S.sc.rng0 + max_slots;
    S.sc.fl = reinterpret_cast<int *>(S.sc.rng1 + max_slots);
    // Tables the prologue alone uses live in the stage ring, which no copy
    // touches before the prologue's last barrier (the ring holds at least two
    // 40 KB stages; these take at most 36 * 1025 + 4 * 1025 bytes): the tile
    // costs and prefix sums, and copies of the active list and the expert
    // offsets.
    long long *sched = reinterpret_cast<long long *>(S.stages);
    S.sc.tc0 = sched;
    S.sc.tc1 = sched + max_slots;
    S.sc.pre0 = sched + 2 * max_slots;
    S.sc.pre1 = sched + 3 * max_slots;
    int *act_s = reinterpret_cast<int *>(sched + 4 * max_slots);
    int *off_s = act_s + max_slots;
    // one round of independent global loads fills every table below
    const int S_ = p.T * p.k;
    for (int i = threadIdx.x; i < max_slots; i += blockDim.x) act_s[i] = p.active[i];
    for (int e = threadIdx.x; e <= p.E; e += blockDim.x) off_s[e] = p.offsets[e];
    if (ent_smem) {
        for (int j = threadIdx.x; j < S_; j += blockDim.x) {
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
    // shelf table pointers (constant-index reads of the parameters), tile
    // geometry of each phase and precision, and the stage barriers
    if (threadIdx.x == 0) {
#pragma unroll
        for (int t = 0; t < MOE_MAX_TIERS; ++t) {
            if (t < p.w.n_tiers) {
                S.tp[t].gq = p.w.tiers[t].gu_qs;
                S.tp[t].gs = reinterpret_cast<const uint8_t *>(p.w.tiers[t].gu_scale);
                S.tp[t].dq = p.w.tiers[t].dn_qs;
                S.tp[t].ds = reinterpret_cast<const uint8_t *>(p.w.tiers[t].dn_scale);
                S.tp[t].bits = p.w.tiers[t].bits;
                S.tp[t].first = p.w.tiers[t].first_expert;
                S.tp[t].n = p.w.tiers[t].n_experts;
            }
        }
        const int t = p.w.n_tiers;
        S.tp[t].gq = p.w.shared.gu_qs;
        S.tp[t].gs = reinterpret_cast<const uint8_t *>(p.w.shared.gu_scale);
        S.tp[t].dq = p.w.shared.dn_qs;
        S.tp[t].ds = reinterpret_cast<const uint8_t *>(p.w.shared.dn_scale);
        S.tp[t].bits = p.w.shared.bits;
        S.tp[t].first = p.E;
        S.tp[t].n = 1;
        for (int st = 0; st < nstages; ++st) mbar_init(&S.full[st], 1);  // the stager's expect_tx arrival
        *S.abort = 0;
        mbar_fence_init();
    }
    if (threadIdx.x < 6) {
        const int phase = threadIdx.x / 3, bi = threadIdx.x % 3;
        const int bits = bi == 0 ? 8 : (bi == 1 ? 4 : 3);
        S.geo[threadIdx.x] = phase == 0 ? geo_gu(p.w.H, bits) : geo(p.w.I, bits);
    }
    __syncthreads();
    // slot table: active routed experts with work for this path, compacted in
    // order by warp 0 (no block-wide barrier per step), then the shared
    // expert; then the schedule (unit costs and their prefix sums)
    __shared__ int n_keep;
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        const int n_active_all = min(act_s[0], p.max_active);
        int run = 0;
        for (int a0 = 0; a0 < n_active_all; a0 += 32) {
            const int a = a0 + lane;
            int e = -1, f = 0, cnt = 0;
            if (a < n_active_all) {
                e = act_s[1 + a];
                if (e >= 0 && e < p.E) {
                    f = off_s[e];
                    cnt = off_s[e + 1] - f;
                }
            }
            const bool keep = a < n_active_all && e >= 0 && e < p.E && cnt > 0 && cnt <= p.max_count;
            const unsigned m = __ballot_sync(0xffffffffu, keep);
            if (keep) {
                const int pos = run + __popc(m & ((1u << lane) - 1u));
                int ti = 0;  // the shelf holding e (shelves cover [0, E) without overlap)
                for (int t = 0; t < p.w.n_tiers; ++t)
                    if (e >= S.tp[t].first && e - S.tp[t].first < S.tp[t].n) ti = t;
                S.st.expert[pos] = e;
                S.st.bits[pos] = S.tp[ti].bits;
                S.st.first[pos] = f;
                S.st.count[pos] = cnt;
                S.tier[pos] = ti;
                S.jloc[pos] = e - S.tp[ti].first;
            }
            run += __popc(m);
        }
        const bool shared_here = p.has_shared && p.T <= p.max_count;
        if (lane == 0 && shared_here) {
            S.st.expert[run] = p.E;
            S.st.bits[run] = p.w.shared.bits;
            S.st.first[run] = S_;
            S.st.count[run] = p.T;
            S.tier[run] = p.w.n_tiers;
            S.jloc[run] = 0;
        }
        const int ns = run + (shared_here ? 1 : 0);
        if (lane == 0) n_keep = ns;
    }
    __syncthreads();
    // the schedule: warp 0 for the gate_up tiles, warp 1 for the down tiles
    if (threadIdx.x < 64) {
        const int lane = threadIdx.x & 31, phase = threadIdx.x >> 5;
        const int ns = n_keep;
        {
            const long long nt = tiles_per_slot(p, phase);
            long long *tc = phase == 0 ? S.sc.tc0 : S.sc.tc1;
            long long *pre = phase == 0 ? S.sc.pre0 : S.sc.pre1;
            long long base = 0;
            for (int a0 = 0; a0 < ns; a0 += 32) {
                const int a = a0 + lane;
                long long v = 0;
                if (a < ns) {
                    const long long c = tile_cost(p, phase, S.st.bits[a], S.st.count[a]);
                    tc[a] = c;
                    v = nt * c;
                }
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const long long u = __shfl_up_sync(0xffffffffu, v, o);
                    if (lane >= o) v += u;
                }
                if (a < ns) pre[a] = base + v;
                base += __shfl_sync(0xffffffffu, v, 31);
            }
            // this CTA's contiguous share [lo, hi) of the phase's total cost,
            // and each slot's tiles whose start falls in it
            const long long lo = div_floor(base * blockIdx.x, gridDim.x);
            const long long hi = div_floor(base * (blockIdx.x + 1), gridDim.x);
            int2 *rng = phase == 0 ? S.sc.rng0 : S.sc.rng1;
            int first = 0x7fffffff, last = -1;
            for (int a0 = 0; a0 < ns; a0 += 32) {
                const int a = a0 + lane;
                bool has = false;
                if (a < ns) {
                    const long long tb = tc[a], off = pre[a] - nt * tb;
                    const int b0 = tiles_before(lo - off, tb, static_cast<int>(nt));
                    const int b1 = tiles_before(hi - off, tb, static_cast<int>(nt));
                    rng[a] = make_int2(b0, b1);
                    has = b0 < b1;
                }
                const unsigned m = __ballot_sync(0xffffffffu, has);
                if (m) {
                    first = min(first, a0 + __ffs(m) - 1);
                    last = max(last, a0 + 31 - __clz(m));
                }
            }
            if (lane == 0) {
                S.sc.fl[2 * phase] = first;
                S.sc.fl[2 * phase + 1] = last;
            }
        }
    }
    // the prologue's tables in the stage ring are overwritten by TMA copies
    // from here on: order this thread's generic accesses before them
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncthreads();
    const int n_slots = n_keep;
    ffn_stream_body(p, M, S, n_slots, nstages);
}

}  // namespace moe

// Shared memory of one CTA: the stage ring, each group's x fragments and
// K-slice partials, shelf and geometry tables, and the slot/entry/schedule
// tables.  Returns the byte count and the number of stages that fit in the
// budget (even: each stage serves one group).
size_t moe_ffn_stream_smem(int H, int I, int T, int max_slots, int n_ent, int *nstages) {
    const size_t ent = n_ent <= moe::kMaxSmemEntries ? 2 * sizeof(int) * static_cast<size_t>(n_ent) : 0;
    const size_t fixed = moe::kGroups * (static_cast<size_t>(moe::xf_bytes(H, I, T)) + moe::kRedBytes) +
                         moe::kMaxStages * sizeof(uint64_t) + moe::kGroups * sizeof(moe::StreamSmem::Ahead) +
                         (MOE_MAX_TIERS + 1) * sizeof(moe::TierPtrs) +
                         6 * sizeof(moe::Geo) + 8 + 6 * sizeof(int) * static_cast<size_t>(max_slots) + ent +
                         2 * sizeof(int2) * static_cast<size_t>(max_slots) + 4 * sizeof(int) + 16;
    const size_t budget = 220 * 1024;
    int ns = fixed < budget ? static_cast<int>((budget - fixed) / moe::kStageBytes) : 0;
    if (ns > moe::kMaxStages) ns = moe::kMaxStages;
    ns &= ~(moe::kGroups - 1);
    *nstages = ns;
    return static_cast<size_t>(ns) * moe::kStageBytes + fixed;
}

cudaError_t moe_configure_ffn_stream() {
    // the opt-in limit is 227 KB per CTA including static shared memory
    return cudaFuncSetAttribute(moe::ffn_stream_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                227 * 1024 - 1024);
}

bool moe_ffn_stream_supported(int H, int I) {
    return H <= moe::kMaxK && I <= moe::kMaxK && H % 128 == 0 && I % 128 == 0;
}

// Whether a launch for this batch gets the two stages the consumer groups need.
bool moe_ffn_stream_fits(int H, int I, int T, int max_slots, int n_ent) {
    int ns = 0;
    moe_ffn_stream_smem(H, I, T, max_slots, n_ent, &ns);
    return ns >= moe::kGroups;
}

namespace {

using EncodeTiled = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                 const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled encode_tiled() {
    static EncodeTiled fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiled>(ptr);
    });
    return fn;
}

CUtensorMapSwizzle swizzle_mode(int w) {
    return w == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                    : (w == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : (w == 32 ? CU_TENSOR_MAP_SWIZZLE_32B : CU_TENSOR_MAP_SWIZZLE_NONE));
}

// A byte tensor map: dims[0] contiguous bytes, dims[i] at strides[i-1] bytes.
// Maps depend only on these arguments, so they are cached by them (a table
// freed and reallocated at the same address with the same shape maps the
// same way).
struct MapKey {
    const void *ptr;
    int rank, sw;
    uint64_t dims[5], strides[4];
    uint32_t box[5];
    bool operator<(const MapKey &o) const { return std::memcmp(this, &o, sizeof(MapKey)) < 0; }
};

std::mutex g_map_mu;
std::map<MapKey, CUtensorMap> g_maps;

bool byte_map(CUtensorMap *out, const void *ptr, int rank, const uint64_t *dims, const uint64_t *strides,
              const uint32_t *box, int sw) {
    MapKey key;
    std::memset(&key, 0, sizeof(key));
    key.ptr = ptr;
    key.rank = rank;
    key.sw = sw;
    for (int i = 0; i < rank; ++i) key.dims[i] = dims[i], key.box[i] = box[i];
    for (int i = 0; i + 1 < rank; ++i) key.strides[i] = strides[i];
    std::lock_guard<std::mutex> lock(g_map_mu);
    auto it = g_maps.find(key);
    if (it != g_maps.end()) {
        *out = it->second;
        return true;
    }
    const EncodeTiled fn = encode_tiled();
    if (!fn) return false;
    const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    if (fn(out, CU_TENSOR_MAP_DATA_TYPE_UINT8, rank, const_cast<void *>(ptr), dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle_mode(sw), CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return false;
    if (g_maps.size() > 4096) g_maps.clear();
    g_maps.emplace(key, *out);
    return true;
}

// Maps of one shelf (or of the shared expert) at table index t.
bool shelf_maps(moe::StreamMaps &M, int t, const moe_tier &tier, int H, int I) {
    const uint64_t n = static_cast<uint64_t>(tier.n_experts);
    const moe::Geo g0 = moe::geo_gu(H, tier.bits), g1 = moe::geo(I, tier.bits);
    if (g0.pad) {
        // [expert][gate|up][row][line][128 bytes], box {128, nc1, 8R, 2, 1}
        const uint64_t dims[5] = {128, static_cast<uint64_t>(g0.rb / 128), static_cast<uint64_t>(I), 2, n};
        const uint64_t str[4] = {128, static_cast<uint64_t>(g0.rb), static_cast<uint64_t>(I) * g0.rb,
                                 2ull * I * g0.rb};
        const uint32_t box[5] = {128, static_cast<uint32_t>(g0.nc1), static_cast<uint32_t>(8 * g0.R), 2, 1};
        if (!byte_map(&M.gq[t], tier.gu_qs, 5, dims, str, box, 128)) return false;
    } else {
        const uint64_t dims[4] = {static_cast<uint64_t>(g0.rb), static_cast<uint64_t>(I), 2, n};
        const uint64_t str[3] = {static_cast<uint64_t>(g0.rb), static_cast<uint64_t>(I) * g0.rb,
                                 2ull * I * g0.rb};
        const uint32_t box[4] = {static_cast<uint32_t>(g0.W), static_cast<uint32_t>(8 * g0.R), 2, 1};
        if (!byte_map(&M.gq[t], tier.gu_qs, 4, dims, str, box, g0.W)) return false;
    }
    if (g0.Ws) {
        const uint64_t dims[4] = {static_cast<uint64_t>(g0.sb), static_cast<uint64_t>(I), 2, n};
        const uint64_t str[3] = {static_cast<uint64_t>(g0.sb), static_cast<uint64_t>(I) * g0.sb,
                                 2ull * I * g0.sb};
        const uint32_t box[4] = {static_cast<uint32_t>(g0.sb), static_cast<uint32_t>(8 * g0.R), 2, 1};
        if (!byte_map(&M.gs[t], tier.gu_scale, 4, dims, str, box, g0.Ws)) return false;
    }
    {
        const uint64_t dims[3] = {static_cast<uint64_t>(g1.rb), static_cast<uint64_t>(H), n};
        const uint64_t str[2] = {static_cast<uint64_t>(g1.rb), static_cast<uint64_t>(H) * g1.rb};
        const uint32_t box[3] = {static_cast<uint32_t>(g1.W), static_cast<uint32_t>(g1.rows), 1};
        if (!byte_map(&M.dq[t], tier.dn_qs, 3, dims, str, box, g1.W)) return false;
    }
    if (g1.Ws) {
        const uint64_t dims[3] = {static_cast<uint64_t>(g1.sb), static_cast<uint64_t>(H), n};
        const uint64_t str[2] = {static_cast<uint64_t>(g1.sb), static_cast<uint64_t>(H) * g1.sb};
        const uint32_t box[3] = {static_cast<uint32_t>(g1.sb), static_cast<uint32_t>(g1.rows), 1};
        if (!byte_map(&M.ds[t], tier.dn_scale, 3, dims, str, box, g1.Ws)) return false;
    }
    return true;
}

}  // namespace

// counters (int[max_active + 1]) must be zero on entry; the caller clears them.
cudaError_t moe_launch_ffn_stream(const moe::FfnParams &p, cudaStream_t s) {
    int nstages = 0;
    const size_t smem = moe_ffn_stream_smem(p.w.H, p.w.I, p.T, p.max_active + 1, p.T * p.k + p.T, &nstages);
    if (nstages < moe::kGroups) return cudaErrorInvalidConfiguration;
    int dev = 0;
    cudaGetDevice(&dev);
    int sms = 0;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(sms);
    cfg.blockDim = dim3(moe::kBlockThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    moe::StreamMaps M;
    std::memset(&M, 0, sizeof(M));
    for (int t = 0; t < p.w.n_tiers; ++t)
        if (!shelf_maps(M, t, p.w.tiers[t], p.w.H, p.w.I)) return cudaErrorInvalidValue;
    if (p.has_shared && !shelf_maps(M, p.w.n_tiers, p.w.shared, p.w.H, p.w.I)) return cudaErrorInvalidValue;
    return cudaLaunchKernelEx(&cfg, moe::ffn_stream_kernel, p, M, nstages);
}
