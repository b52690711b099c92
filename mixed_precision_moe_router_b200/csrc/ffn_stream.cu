// Tiered expert FFN, GEMV path: one persistent launch that streams every
// touched expert's packed rows once through a shared-memory ring and runs the
// dot products on the tensor cores against up to 8 token columns at a time.
//
// [P1] "step 4: three shelves, all on the GPU": mul_mat_id runs each word
// through its chosen experts, each shelf computes only the ids on it and the
// shelf results add up; the decode kernel fuses gate, up and the activation.
//
// Design (B200):
//  * Work is a list of tiles (plan.cuh): for every slot (an active expert
//    whose token count is in (0, max_count], and the shared expert) gate_up
//    tiles of 8R gate rows plus the 8R matching up rows, and down tiles of
//    16R rows.  Each CTA takes a contiguous, cost-balanced run of the gate_up
//    tiles and then of the down tiles, so 8-, 4- and 3-bit experts spread
//    evenly over the SMs.
//  * Warp-specialised pipeline, every hand-off an mbarrier (no block-wide
//    barrier after the prologue):
//      - a producer warp stages tile after tile with TMA tensor copies into a
//        byte ring (tiles of different precisions take different sizes, so
//        the ring holds as many bytes in flight as shared memory allows);
//      - a loader warp builds the B operand of each (slot, pass): fp16
//        fragments of x for gate_up, of h split into hi + lo for down, after
//        waiting (bounded) for the slot's gate_up tiles to be counted done;
//      - 8 compute warps split every tile into R row subtiles x 8/R K
//        slices.  For each 32-weight block a warp turns its codes into exact
//        fp16 integers (|q| <= 127), multiplies them with the B fragments on
//        the tensor cores (mma.sync m16n8k16: exact products, fp32
//        accumulation) and adds d * partial into fp32 accumulators, then
//        hands its partial sums to the epilogue through a small ring;
//      - an epilogue warp sums the K slices in a fixed order and writes
//        h = silu(g) * u or y, and publishes per slot how many gate_up tiles
//        this CTA finished (fence, then an atomic add).
//    The only roundings besides fp32 accumulation are bf16 x -> fp16 (exact
//    for |x| in [2^-14, 65504]) and the split of the fp32 intermediate h into
//    two fp16 columns hi + lo (relative error <= 2^-22).
//  * A down tile's weights are in flight while its slot's h is still being
//    produced elsewhere; the grid is launched cooperatively so every CTA is
//    resident and the waits on other CTAs' counts resolve.  Every wait is
//    bounded; a warp that gives up sets MOE_STATUS_TIMEOUT and a CTA-wide
//    abort flag that releases the others, and the producer waits for its
//    copies in flight before the CTA exits.
#include <cuda.h>

#include <cstring>
#include <map>
#include <mutex>

#include "common.cuh"
#include "ffn.cuh"
#include "route_cta.cuh"
#include "sync.cuh"

namespace moe {

constexpr int kWarps = 8;          // compute warps of a group: they split each tile
constexpr int kGroups = 2;         // compute groups, taking alternate tiles
constexpr int kComputeWarps = kGroups * kWarps;
constexpr int kWarpProducer = kComputeWarps;      // lane 0 stages the tiles
constexpr int kWarpLoader = kComputeWarps + 1;    // builds the B operand of each (slot, pass)
constexpr int kWarpEpilogue0 = kComputeWarps + 2;  // one per group: sums partials, writes h / y
constexpr int kBlockWarps = kComputeWarps + 2 + kGroups;
constexpr int kBlockThreads = kBlockWarps * 32;
constexpr int kND = 8;             // tiles in flight at most (full/empty barrier pairs)
constexpr int kNR = 3;             // partial-sum buffers per group (compute warps -> epilogue)
constexpr int kNBMax = 4;          // B-operand buffers (loader -> compute warps) at most
constexpr int kMaxTileBytes = 40 * 1024;  // a staged tile (codes, padding, scales) at most
constexpr int kTileAlign = 1024;   // ring allocations start on a 128-byte-swizzle atom
constexpr int kMaxK = 2048;
constexpr int kRedBytes = kWarps * 32 * 16;  // one item's partials: a float4 per compute lane
constexpr int kMaxSmemEntries = 2048;        // sorted slot ids kept in shared memory up to this many
constexpr int kMaxExpertShare = 16;          // router rows a CTA computes when it routes the batch itself
constexpr int kDealtMaxTokens = 2;          // tiles dealt out in turn up to this many tokens (plan_in_cta)
constexpr long long kFirstTileHeadStart = 8000;  // cycles the producer gives a layer's first tiles (run_producer)

// B-operand buffers: with dealt tiles every down tile has an operand of its
// own, so the loader gets room to build several ahead (they are small then).
__host__ __device__ __forceinline__ int n_bbufs(int T) { return T <= kDealtMaxTokens ? kNBMax : 2; }

// ---------------------------------------------------------------------------
// tile geometry
// ---------------------------------------------------------------------------
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
    g.rb = K * storage_bits(bits) / 8;
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
        if (nc1 <= 256 && g.rows * (nc1 * 128 + g.sb) <= kMaxTileBytes) {
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

// ---------------------------------------------------------------------------
// Codes -> exact fp16 integers: four half2 pairs per row, block and thread.
// A code c placed at mantissa bit s under the exponent of 2^(10-s) reads as
// the half 2^(10-s) + c; subtracting 2^(10-s) + offset leaves q exactly.
// Thread t owns weights 8t .. 8t+7 of each 32-weight block, paired as
// (2p, 2p+1) for 8-bit codes and (p, p+4) for 4-bit, FP4 and 3-bit codes,
// p = 0..3.
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

// Byte offsets in a staged tile of thread t's codes of block b in row r: the
// code word (8 bytes for 8-bit codes, 4 for 4-bit and FP4, the low-plane u16
// for 3-bit) and, for 3-bit codes, the high-plane byte.
template <int BITS, bool PAD>
__device__ __forceinline__ void code_offsets(const Geo &G, int r, int xr, int b, int t, int &o0, int &o1) {
    if constexpr (BITS == 8) {
        o0 = tile_off<PAD>(32 * b + 8 * t, r, G, xr);
    } else if constexpr (BITS == 4 || BITS == kBitsFp4) {
        o0 = tile_off<PAD>(16 * b + 4 * t, r, G, xr);
    } else {
        o0 = tile_off<PAD>(8 * b + 2 * t, r, G, xr);
        o1 = tile_off<PAD>(G.K / 4 + 4 * b + t, r, G, xr);
    }
}

// The codes at those offsets as four half2 of exact integers q.
template <int BITS>
__device__ __forceinline__ void dequant8(const uint8_t *tile, int o0, int o1, uint32_t (&P)[4]) {
    if constexpr (BITS == 8) {
        const uint2 w = *reinterpret_cast<const uint2 *>(tile + o0);
        const uint32_t u0 = w.x ^ 0x80808080u, u1 = w.y ^ 0x80808080u;  // c = q + 128
        constexpr uint32_t kBias = 0x64806480u;                         // 1024 + 128
        P[0] = hsub2(prmt(u0, 0x64646464u, 0x4140u), kBias);
        P[1] = hsub2(prmt(u0, 0x64646464u, 0x4342u), kBias);
        P[2] = hsub2(prmt(u1, 0x64646464u, 0x4140u), kBias);
        P[3] = hsub2(prmt(u1, 0x64646464u, 0x4342u), kBias);
    } else if constexpr (BITS == 4) {
        // nibble i of the word at byte 16b + 4t is weight 8t + i (c = q + 8)
        const uint32_t v = *reinterpret_cast<const uint32_t *>(tile + o0);
        const uint32_t v8 = v >> 8;
        P[0] = hsub2((v & 0x000F000Fu) | 0x64006400u, 0x64086408u);   // 1024 + c - 1032
        P[1] = hsub2((v & 0x00F000F0u) | 0x54005400u, 0x54805480u);   // 64 + c - 72
        P[2] = hsub2((v8 & 0x000F000Fu) | 0x64006400u, 0x64086408u);
        P[3] = hsub2((v8 & 0x00F000F0u) | 0x54005400u, 0x54805480u);
    } else if constexpr (BITS == kBitsFp4) {
        // FP4 codes in the 4-bit layout: nibble i of the word at byte 16b + 4t
        // is weight 8t + i
        fp4_pairs(*reinterpret_cast<const uint32_t *>(tile + o0), P);
    } else {
        // low plane: bits 0-1 of weight 8t+i at bit 2i of the u16 at byte 8b+2t;
        // high plane: bit 2 at bit i of byte K/4 + 4b + t (c = q + 4)
        const uint32_t lo16 = *reinterpret_cast<const uint16_t *>(tile + o0);
        const uint32_t hb = tile[o1];
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
    const int xa = row_x<PAD>(rA, G);
    // Rows rA and rB are a multiple of 8 rows apart, and every layout's
    // swizzle of a row depends on the row mod 8: row rB's codes and scales
    // sit a fixed distance after row rA's.
    const int dcode = tile_off<PAD>(0, rB, G, row_x<PAD>(rB, G)) - tile_off<PAD>(0, rA, G, xa);
    const uint8_t *stageB = stage + dcode;
    // scales: [row][sb] after the codes, swizzled at width Ws (or plain)
    const uint8_t *sclA = stage + G.cb + rA * G.sb, *sclB = sclA + (rB - rA) * G.sb;
    const int sxa = G.Ws ? swz(rA, G.Ws) : 0;
    const uint8_t *xg = xf + g * cs + t * 16;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[nt][i] = 0.f;
    // one block per iteration: the smallest loop body (a larger unroll
    // measured slower, its code competing with the other roles' for the
    // instruction cache)
#pragma unroll 1
    for (int b = b0; b < b1; ++b) {
        const int so = (2 * b) ^ sxa;
        const float dA = __half2float(*reinterpret_cast<const __half *>(sclA + so));
        const float dB = __half2float(*reinterpret_cast<const __half *>(sclB + so));
        int o0, o1 = 0;
        code_offsets<BITS, PAD>(G, rA, xa, b, t, o0, o1);
        uint32_t PA[4], PB[4];
        dequant8<BITS>(stage, o0, o1, PA);
        dequant8<BITS>(stageB, o0, o1, PB);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            uint4 X = make_uint4(0u, 0u, 0u, 0u);
            if (g < (nt == 0 ? ncol0 : ncol1)) X = *reinterpret_cast<const uint4 *>(xg + nt * 8 * cs + b * 64);
            // the block's two k16 halves chained through the accumulator (the
            // products are exact)
            float c[4] = {0.f, 0.f, 0.f, 0.f};
            mma16816(c, PA[0], PB[0], PA[1], PB[1], X.x, X.y);
            mma16816(c, PA[2], PB[2], PA[3], PB[3], X.z, X.w);
            acc[nt][0] = fmaf(dA, c[0], acc[nt][0]);
            acc[nt][1] = fmaf(dA, c[1], acc[nt][1]);
            acc[nt][2] = fmaf(dB, c[2], acc[nt][2]);
            acc[nt][3] = fmaf(dB, c[3], acc[nt][3]);
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

// geometry index of a shelf: 8-bit, 4-bit storage (integer or FP4), 3-bit
__device__ __forceinline__ int bits_idx(int bits) { return bits == 8 ? 0 : (bits == 3 ? 2 : 1); }

// Table base pointers of the shelves (index < n_tiers) and of the shared
// expert (index n_tiers), copied from the parameters into shared memory so
// that they can be indexed at run time.
struct TierPtrs {
    const uint8_t *gq, *gs, *dq, *ds;
};

// Ring bytes a staged tile takes (its start stays on a swizzle atom).
__host__ __device__ __forceinline__ int stage_alloc_bytes(const Geo &g) {
    return (stage_bytes(g) + kTileAlign - 1) & ~(kTileAlign - 1);
}

// Bytes of the all-token x fragments (batches of at most kTokPerPass tokens):
// column t holds token t, once in the pair order of 8-bit codes and once in
// that of 4- and 3-bit codes.
__host__ __device__ __forceinline__ int xall_bytes(int H, int T) {
    return T <= kTokPerPass ? 2 * T * xf_col_stride(H) : 0;
}

// Bytes of one B-operand buffer: the down fragments of one pass, plus the
// gate_up fragments of one pass when gate_up does not use the all-token copy.
__host__ __device__ __forceinline__ int bbuf_bytes(int H, int I, int T) {
    const int nd = T < 4 * down_ntiles(I) ? T : 4 * down_ntiles(I);
    const int cd = nd <= 4 ? 2 * nd : 8 + 2 * (nd - 4);
    int b = cd * xf_col_stride(I);
    if (T > kTokPerPass) {
        const int a = kTokPerPass * xf_col_stride(H);
        b = a > b ? a : b;
    }
    return (b + 127) & ~127;
}

struct StreamSmem {
    uint8_t *ring;
    int ring_bytes;
    uint8_t *xall;           // all-token gate_up fragments (T <= kTokPerPass), else null
    uint8_t *bbuf;           // [nb][b_bytes]
    int b_bytes;
    float4 *red;             // [kGroups][kNR][kWarps * 32]
    uint64_t *full, *empty;  // [kND]: a tile's copies landed / every compute warp is done with it
    uint64_t *rfull, *rempty;  // [kGroups][kNR]: partials written / partials summed
    uint64_t *bfull, *bempty;  // [nb]: B operand built / every compute warp has moved past it
    int nb, nb_log2;           // B-operand buffers (a power of two)
    int *abort;              // [0] set by a warp that gave up (every wait checks it); [1] grid barriers passed
    int *range;              // this CTA's tiles: [gs0, ge0), [gs1, ge1); then the slot count
    int *pst;                // producer: ring byte range [pst[d], pst[kND + d]) of the tile in descriptor d
    int *srt;                // copy of sorted_slot when it has at most kMaxSmemEntries entries, else null
    PlanTabs pt;
    TierPtrs *tp;            // [MOE_MAX_TIERS + 1]
    Geo *geo;                // [phase][8-, 4-, 3-bit]
    int nt0, nt1;            // tiles per slot of each phase
};

__device__ __forceinline__ const Geo &tile_geo(const StreamSmem &S, int phase, int a) {
    return S.geo[phase * 3 + bits_idx(phase_bits(S.pt.bits[a], phase))];
}

__device__ __forceinline__ void abort_cta(const FfnParams &p, const StreamSmem &S) {
    status_or(p.status, MOE_STATUS_TIMEOUT);
    *static_cast<volatile int *>(S.abort) = 1;
}

// This CTA's tiles in order: its run of gate_up tiles (phase 0), then its run
// of down tiles (phase 1); phase 2 once exhausted.  Tile g of a phase is tile
// b = g % nt of slot a = g / nt.  Every warp role walks the same sequence.
// A CTA's tiles of a phase are the global indices g = range[2 phase] +
// n * range[5] below range[2 phase + 1]: a contiguous run (stride 1) or every
// grid-th tile (stride = grid).
struct Walk {
    int phase, g, ge, a, b;
};

__device__ __forceinline__ void walk_enter(const StreamSmem &S, Walk &w, int phase) {
    const int nt = phase == 0 ? S.nt0 : S.nt1;
    w.phase = phase;
    w.g = S.range[2 * phase];
    w.ge = S.range[2 * phase + 1];
    w.a = w.g / nt;
    w.b = w.g - w.a * nt;
}

// tiles of `phase` in this CTA's list
__device__ __forceinline__ int phase_tiles(const StreamSmem &S, int phase) {
    const int g = S.range[2 * phase], ge = S.range[2 * phase + 1], s = S.range[5];
    return g < ge ? (ge - g + s - 1) / s : 0;
}

__device__ __forceinline__ void walk_begin(const StreamSmem &S, Walk &w) {
    if (S.range[0] < S.range[1]) walk_enter(S, w, 0);
    else if (S.range[2] < S.range[3]) walk_enter(S, w, 1);
    else w.phase = 2;
}

__device__ __forceinline__ void walk_next(const StreamSmem &S, Walk &w) {
    const int stride = S.range[5];
    w.g += stride;
    if (w.g < w.ge) {
        const int nt = w.phase == 0 ? S.nt0 : S.nt1;
        if (stride == 1) {
            if (++w.b == nt) {
                w.b = 0;
                ++w.a;
            }
        } else {
            w.a = w.g / nt;
            w.b = w.g - w.a * nt;
        }
        return;
    }
    if (w.phase == 0 && S.range[2] < S.range[3]) walk_enter(S, w, 1);
    else w.phase = 2;
}

// Passes over a resident tile of slot a, and whether phase `phase` takes its
// B operand from the loader (true) or from the all-token fragments.
__device__ __forceinline__ int n_passes(const FfnParams &p, const StreamSmem &S, int phase, int a) {
    const int tp = tokens_per_pass(phase, p.w.I);
    return (S.pt.count[a] + tp - 1) / tp;
}
__device__ __forceinline__ bool loads_b(const StreamSmem &S, int phase) { return phase == 1 || S.xall == nullptr; }

// Key of the B operand of (phase, slot, pass); consecutive tiles of one slot
// with a single pass share it.
__device__ __forceinline__ long long b_key(int phase, int a, int pass) {
    return (static_cast<long long>(2 * a + phase) << 32) | static_cast<unsigned>(pass);
}

// The ring offset of each tile, in order: every role that needs it takes the
// same allocations (wrapping to 0 when a tile does not fit before the end).
__device__ __forceinline__ int ring_take(int &head, int sz, int ring_bytes) {
    if (head + sz > ring_bytes) head = 0;
    const int s = head;
    head += sz;
    return s;
}

// h / y row of entry n of slot a: the slot's sorted slot ids, or for the
// shared expert (entries from T*k on) the row T*k + t of token t.
__device__ __forceinline__ int entry_row(const FfnParams &p, const StreamSmem &S, int a, int n) {
    const int j = S.pt.first[a] + n;
    const int Sk = p.T * p.k;
    if (j >= Sk) return j;
    const int r = S.srt ? S.srt[j] : __ldg(p.sorted + j);
    return (r >= 0 && r < Sk) ? r : 0;
}

__device__ __forceinline__ int row_token(const FfnParams &p, int row) {
    const int Sk = p.T * p.k;
    return row >= Sk ? row - Sk : row / p.k;
}

// Stage the codes and scales of tile (phase, a, tile) into `dst`, completing
// on `bar`: a gate_up tile is its 8R gate rows and the matching 8R up rows, a
// down tile 16R consecutive rows; codes as column chunks of W bytes.
__device__ __forceinline__ void issue_tile(const FfnParams &p, const StreamMaps &M, const StreamSmem &S, int phase,
                                           int a, int tile, uint8_t *dst, uint64_t *bar) {
    const int I = p.w.I;
    const Geo &G = tile_geo(S, phase, a);
    const int ti = S.pt.tier[a], j = S.pt.jloc[a];
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

// ---------------------------------------------------------------------------
// B operands
// ---------------------------------------------------------------------------

// 8 consecutive bf16 values -> fp16 fragment words in both pair orders.
__device__ __forceinline__ void x_frags(const uint4 q, bool &bad, uint4 &f8, uint4 &f43) {
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
    uint16_t v[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        v[2 * j] = to_f16(bf16lo(w[j]), bad);
        v[2 * j + 1] = to_f16(bf16hi(w[j]), bad);
    }
    f8 = pack_frag(v, 8);
    f43 = pack_frag(v, 4);
}

// All-token gate_up fragments (T <= kTokPerPass) from the bf16 rows of x
// staged in shared memory: column t of copy 0 (8-bit order) and of copy 1
// (4- and 3-bit order) is token t.  Every thread of the CTA takes a share.
__device__ __forceinline__ bool build_xall(const FfnParams &p, const uint8_t *x_s, uint8_t *xall) {
    bool bad = false;
    const int H = p.w.H, nchunk = H / 8, cs = xf_col_stride(H);
    const int n = p.T * nchunk;
    uint8_t *x43 = xall + p.T * cs;
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const int t = i / nchunk, rem = i - t * nchunk;
        const uint4 q = reinterpret_cast<const uint4 *>(x_s)[i];
        uint4 f8, f43;
        x_frags(q, bad, f8, f43);
        *reinterpret_cast<uint4 *>(xall + t * cs + rem * 16) = f8;
        *reinterpret_cast<uint4 *>(x43 + t * cs + rem * 16) = f43;
    }
    return bad;
}

// gate_up fragments of one pass (loader warp): column n holds the token of
// entry pass * 8 + n of slot a, in the pair order of the slot's codes.
__device__ __forceinline__ bool load_b_gu(const FfnParams &p, const StreamSmem &S, int a, int pass, int ntok,
                                          uint8_t *xf) {
    bool bad = false;
    const int lane = threadIdx.x & 31;
    const int H = p.w.H, nchunk = H / 8, cs = xf_col_stride(H), bits = phase_bits(S.pt.bits[a], 0);
    const int my_row = lane < ntok ? entry_row(p, S, a, pass * kTokPerPass + lane) : 0;
    for (int n = 0; n < ntok; ++n) {
        const int tok = row_token(p, __shfl_sync(0xffffffffu, my_row, n));
        const uint16_t *xr = p.x + static_cast<size_t>(tok) * H;
#pragma unroll 4
        for (int rem = lane; rem < nchunk; rem += 32) {
            const uint4 q = *reinterpret_cast<const uint4 *>(xr + 8 * rem);
            uint4 f8, f43;
            x_frags(q, bad, f8, f43);
            *reinterpret_cast<uint4 *>(xf + n * cs + rem * 16) = bits == 8 ? f8 : f43;
        }
    }
    return bad;
}

// down fragments of one pass (loader warp): in n-tile nt, column 2m holds hi
// and column 2m + 1 lo of h for the entry pass * tp + 4nt + m of slot a.
__device__ __forceinline__ bool load_b_dn(const FfnParams &p, const StreamSmem &S, int a, int pass, int ntok,
                                          uint8_t *xf) {
    bool bad = false;
    const int lane = threadIdx.x & 31;
    const int I = p.w.I, nchunk = I / 8, cs = xf_col_stride(I), bits = phase_bits(S.pt.bits[a], 1);
    const int tp = tokens_per_pass(1, I);
    const int my_row = lane < ntok ? entry_row(p, S, a, pass * tp + lane) : 0;
    for (int n = 0; n < ntok; ++n) {
        const int row = __shfl_sync(0xffffffffu, my_row, n);
        const float *hr = p.h + static_cast<size_t>(row) * I;
        const int col = (n >> 2) * 8 + 2 * (n & 3);
#pragma unroll 2
        for (int rem = lane; rem < nchunk; rem += 32) {
            const float4 f0 = __ldcg(reinterpret_cast<const float4 *>(hr + 8 * rem));
            const float4 f1 = __ldcg(reinterpret_cast<const float4 *>(hr + 8 * rem + 4));
            const float f[8] = {f0.x, f0.y, f0.z, f0.w, f1.x, f1.y, f1.z, f1.w};
            uint16_t hi[8], lo[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                hi[j] = to_f16(f[j], bad);
                lo[j] = __half_as_ushort(__float2half_rn(f[j] - __half2float(__ushort_as_half(hi[j]))));
            }
            *reinterpret_cast<uint4 *>(xf + col * cs + rem * 16) = pack_frag(hi, bits);
            *reinterpret_cast<uint4 *>(xf + (col + 1) * cs + rem * 16) = pack_frag(lo, bits);
        }
    }
    return bad;
}

// ---------------------------------------------------------------------------
// warp roles
// ---------------------------------------------------------------------------

// One compute warp's partial sums of a resident tile for one pass.
template <int BITS>
__device__ __forceinline__ float4 compute_part(const Geo &G, int phase, const uint8_t *stage, const uint8_t *xf,
                                               int ncol, int warp) {
    const int r = warp & (G.R - 1), s = warp / G.R;
    const int b0 = min(G.nb, s * G.bps), b1 = min(G.nb, (s + 1) * G.bps);
    const int cs = xf_col_stride(G.K);
    const int g = (threadIdx.x & 31) >> 2;
    if (phase == 0) {
        const TileAcc t = G.pad ? warp_tile<BITS, 1, true>(stage, G, 8 * r + g, 8 * G.R + 8 * r + g, b0, b1, xf, cs,
                                                           ncol, 0)
                                : warp_tile<BITS, 1, false>(stage, G, 8 * r + g, 8 * G.R + 8 * r + g, b0, b1, xf, cs,
                                                            ncol, 0);
        return make_float4(t.acc[0][0], t.acc[0][1], t.acc[0][2], t.acc[0][3]);
    }
    const int nc0 = 2 * max(0, min(4, ncol)), nc1 = 2 * max(0, min(4, ncol - 4));
    const TileAcc t = nc1 > 0 ? warp_tile<BITS, 2, false>(stage, G, 16 * r + g, 16 * r + g + 8, b0, b1, xf, cs,
                                                          nc0, nc1)
                              : warp_tile<BITS, 1, false>(stage, G, 16 * r + g, 16 * r + g + 8, b0, b1, xf, cs,
                                                          nc0, 0);
    // hi + lo columns of each token
    return make_float4(t.acc[0][0] + t.acc[0][1], t.acc[0][2] + t.acc[0][3], t.acc[1][0] + t.acc[1][1],
                       t.acc[1][2] + t.acc[1][3]);
}

// Producer (lane 0 of its warp): allocate each tile in the byte ring, wait
// until no tile still being read overlaps it (tiles are released oldest
// first), and stage it.  Before returning it waits for every copy it issued.
// State a role keeps from one layer to the next in a persistent launch (tile
// and item counts fix the barrier phases and ring offsets).
struct ProducerState {
    int i;  // tiles issued so far
};
struct ComputeState {
    int i, m, kb;
};
struct LoaderState {
    int kb;
};
struct EpilogueState {
    int m, i;
};

// Producer warp for the current tile list; `drain`: wait for every copy in
// flight before returning (the last list of a launch).  Every tile issued
// before the call has been consumed (the previous list's roles have ended),
// so the ring starts empty: the first tiles that fit it, up to kND, take
// consecutive ranges from offset 0 (a warp prefix sum of their sizes) and are
// issued at once, one per lane.  Lane 0 then issues the rest in order, each
// once the ranges it overlaps have been released.  The ring range of the tile
// in descriptor d is [pst[d], pst[kND + d]) (in shared memory: a dynamically
// indexed array of a thread lives in local memory, which has almost no L1
// behind a full shared-memory carve-out); the compute warps read the stage
// offset from there.
__device__ __forceinline__ void run_producer(const FfnParams &p, const StreamMaps &M, StreamSmem &S,
                                             ProducerState &ps, bool drain) {
    const int lane = threadIdx.x & 31;
    int *st = S.pst, *en = S.pst + kND;
    const int i0 = ps.i;
    const int gs0 = S.range[0], n0 = phase_tiles(S, 0);
    const int gs1 = S.range[2], n1 = phase_tiles(S, 1), stride = S.range[5];
    int nfit, head;
    {
        const int j = lane;
        const bool real = j < n0 + n1 && j < kND;
        int phase = 0, a = 0, b = 0, sz = 0;
        if (real) {
            phase = j < n0 ? 0 : 1;
            const int g = phase == 0 ? gs0 + j * stride : gs1 + (j - n0) * stride;
            const int nt = phase == 0 ? S.nt0 : S.nt1;
            a = g / nt;
            b = g - a * nt;
            sz = stage_alloc_bytes(tile_geo(S, phase, a));
        }
        int end = sz;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, end, o);
            if (lane >= o) end += v;
        }
        const bool fits = real && end <= S.ring_bytes;  // a prefix of the lanes
        nfit = __popc(__ballot_sync(0xffffffffu, fits));
        head = nfit > 0 ? __shfl_sync(0xffffffffu, end, nfit - 1) : 0;
        if (fits) {
            const int d = (i0 + j) % kND;
            st[d] = end - sz;
            en[d] = end;
            // the first tile of each compute group goes first; the rest follow
            // once the first has landed (at most about 2 us later), so that
            // compute starts before the whole burst of every CTA has arrived
            if (j >= kGroups) mbar_wait_limit(&S.full[i0 % kND], (i0 / kND) & 1, kFirstTileHeadStart);
            issue_tile(p, M, S, phase, a, b, S.ring + (end - sz), &S.full[d]);
        }
    }
    __syncwarp();  // lane 0 reads the other lanes' ring ranges below
    // every lane keeps the count: the next list's descriptors follow from it
    ps.i = i0 + n0 + n1;
    if (lane == 0) {
        int rel = i0, i = i0 + nfit;
        bool ok = true;
        Walk w;
        walk_begin(S, w);
        for (int n = 0; n < nfit; ++n) walk_next(S, w);
        for (; w.phase < 2; walk_next(S, w), ++i) {
            const int sz = stage_alloc_bytes(tile_geo(S, w.phase, w.a));
            const int s0 = ring_take(head, sz, S.ring_bytes);
            while (rel < i) {
                bool clash = i - rel >= kND;
                for (int j = rel; j < i && !clash; ++j) clash = st[j % kND] < s0 + sz && s0 < en[j % kND];
                if (!clash) break;
                if (!mbar_wait_abortable(&S.empty[rel % kND], (rel / kND) & 1, S.abort, p.wait_limit)) {
                    ok = false;
                    break;
                }
                ++rel;
            }
            if (!ok) break;
            st[i % kND] = s0;
            en[i % kND] = s0 + sz;
            issue_tile(p, M, S, w.phase, w.a, w.b, S.ring + s0, &S.full[i % kND]);
        }
        if (!ok) abort_cta(p, S);
        ps.i = i;  // short of i0 + n0 + n1 only after giving up
        // tiles before i were issued and those before rel consumed: the rest must land
        if (drain || !ok)
            for (int j = max(rel, i - kND); j < i; ++j)
                if (!mbar_wait_limit(&S.full[j % kND], (j / kND) & 1, p.wait_limit))
                    status_or(p.status, MOE_STATUS_TIMEOUT);
    }
    __syncwarp();
}

// Compute warp `cw` (0..kComputeWarps-1): group cw / kWarps computes the
// tiles i with i % kGroups == group, its K slice cw % kWarps of each.  Every
// compute warp follows the whole tile sequence so that it keeps the ring
// offsets and, for the B operands, releases every buffer in order: on each
// change of operand it waits until the next one is built (even when its group
// has no tile that uses it) and releases the previous one, so no release can
// run ahead of the loader.
__device__ __forceinline__ void run_compute(const FfnParams &p, StreamSmem &S, int cw, ComputeState &cs) {
    const int lane = threadIdx.x & 31, grp = cw / kWarps, warp = cw % kWarps;
    int i = cs.i, m = cs.m, kb = cs.kb;
    long long key = -1;
    bool ok = true;
    float4 *red = S.red + grp * kNR * (kWarps * 32);
    uint64_t *rfull = S.rfull + grp * kNR, *rempty = S.rempty + grp * kNR;
    Walk w;
    walk_begin(S, w);
    for (; ok && w.phase < 2; walk_next(S, w), ++i) {
        const int phase = w.phase, a = w.a;
        const int bits = phase_bits(S.pt.bits[a], phase), cnt = S.pt.count[a];
        const Geo &G = tile_geo(S, phase, a);
        const bool mine = i % kGroups == grp;
        if (mine && !mbar_wait_warp(&S.full[i % kND], (i / kND) & 1, S.abort, p.wait_limit)) {
            ok = false;
            break;
        }
        // the stage's offset, written by the producer before the copy it waited for
        const uint8_t *stage = S.ring + (mine ? S.pst[i % kND] : 0);
        const int tp = tokens_per_pass(phase, p.w.I), np = n_passes(p, S, phase, a);
        for (int pass = 0; pass < np; ++pass) {
            const uint8_t *xf;
            int ncol;
            if (loads_b(S, phase)) {
                const long long nk = b_key(phase, a, pass);
                if (nk != key) {
                    ++kb;
                    key = nk;
                    if (!mbar_wait_warp(&S.bfull[kb & (S.nb - 1)], (kb >> S.nb_log2) & 1, S.abort, p.wait_limit)) {
                        ok = false;
                        break;
                    }
                    if (kb > 0) {
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&S.bempty[(kb - 1) & (S.nb - 1)]);
                    }
                }
                xf = S.bbuf + static_cast<size_t>(kb & (S.nb - 1)) * S.b_bytes;
                ncol = min(tp, cnt - pass * tp);
            } else {  // every token is a column; the epilogue keeps the slot's
                xf = S.xall + (bits == 8 ? 0 : p.T * xf_col_stride(p.w.H));
                ncol = p.T;
            }
            if (!mine) continue;
            float4 part;
            if (bits == 8) part = compute_part<8>(G, phase, stage, xf, ncol, warp);
            else if (bits == 4) part = compute_part<4>(G, phase, stage, xf, ncol, warp);
            else if (bits == 3) part = compute_part<3>(G, phase, stage, xf, ncol, warp);
            else part = compute_part<kBitsFp4>(G, phase, stage, xf, ncol, warp);
            if (pass == np - 1) {  // every read of the stage is done
                __syncwarp();
                if (lane == 0) mbar_arrive(&S.empty[i % kND]);
            }
            const int r = m % kNR;
            if (!mbar_wait_warp(&rempty[r], ((m / kNR) & 1) ^ 1, S.abort, p.wait_limit)) {
                ok = false;
                break;
            }
            red[r * (kWarps * 32) + warp * 32 + lane] = part;
            __syncwarp();
            if (lane == 0) mbar_arrive(&rfull[r]);
            ++m;
        }
    }
    cs.i = i;
    cs.m = m;
    cs.kb = kb;
    if (!ok && lane == 0) abort_cta(p, S);
}

// Loader warp: the B operand of every (phase, slot, pass) that takes one, in
// the order the compute warps use them; before a slot's first down operand it
// waits (bounded) until every gate_up tile of the slot has been counted done.
__device__ __forceinline__ void run_loader(const FfnParams &p, StreamSmem &S, LoaderState &ls) {
    const int lane = threadIdx.x & 31;
    int kb = ls.kb, ready = -1;
    long long key = -1;
    bool ok = true, bad = false;
    Walk w;
    walk_begin(S, w);
    for (; ok && w.phase < 2; walk_next(S, w)) {
        const int phase = w.phase, a = w.a;
        if (!loads_b(S, phase)) continue;
        const int tp = tokens_per_pass(phase, p.w.I), np = n_passes(p, S, phase, a), cnt = S.pt.count[a];
        for (int pass = 0; pass < np; ++pass) {
            const long long nk = b_key(phase, a, pass);
            if (nk == key) continue;
            key = nk;
            ++kb;
            if (!mbar_wait_warp(&S.bempty[kb & (S.nb - 1)], ((kb >> S.nb_log2) & 1) ^ 1, S.abort, p.wait_limit)) {
                ok = false;
                break;
            }
            if (phase == 1 && a != ready) {
                bool got = true;
                if (lane == 0) got = wait_geq_abortable(p.ctr + a, S.nt0, S.abort, p.wait_limit);
                got = __shfl_sync(0xffffffffu, got, 0);
                __syncwarp();
                if (!got) {
                    ok = false;
                    break;
                }
                ready = a;
            }
            uint8_t *xf = S.bbuf + static_cast<size_t>(kb & (S.nb - 1)) * S.b_bytes;
            const int ntok = min(tp, cnt - pass * tp);
            bad |= phase == 0 ? load_b_gu(p, S, a, pass, ntok, xf) : load_b_dn(p, S, a, pass, ntok, xf);
            __syncwarp();
            if (lane == 0) mbar_arrive(&S.bfull[kb & (S.nb - 1)]);
        }
    }
    ls.kb = kb;
    if (__any_sync(0xffffffffu, bad) && lane == 0) status_or(p.status, MOE_STATUS_FP16_RANGE);
    if (!ok && lane == 0) abort_cta(p, S);
}

// Epilogue of one (tile, pass): the K slices of every output summed in a
// fixed order; gate_up -> h = silu(g) * u, down -> y.
__device__ __forceinline__ void epilogue_item(const FfnParams &p, const StreamSmem &S, int phase, int a, int tile,
                                              int pass, const float4 *red) {
    const int lane = threadIdx.x & 31;
    const float *rf = reinterpret_cast<const float *>(red);
    const int cnt = S.pt.count[a];
    if (phase == 0) {
        const int I = p.w.I, R = S.geo[0].R, S_ = kWarps / R, lr = __ffs(8 * R) - 1;
        // with the all-token fragments the column of entry n is its token;
        // otherwise entry pass*8 + n sits in column n
        const int ntok = S.xall ? cnt : min(kTokPerPass, cnt - pass * kTokPerPass);
        const int base = S.xall ? 0 : pass * kTokPerPass;
        const int my_row = lane < ntok ? entry_row(p, S, a, base + lane) : 0;
        const int n_out = ntok << lr;
        for (int o0 = 0; o0 < n_out; o0 += 32) {
            const int o = o0 + lane;
            const int n = min(o >> lr, ntok - 1);
            const int row = __shfl_sync(0xffffffffu, my_row, n);
            if (o < n_out) {
                const int rg = o & (8 * R - 1), g = rg & 7, r = rg >> 3;
                const int col = S.xall ? row_token(p, row) : n;
                const int ln = 4 * g + (col >> 1), sub = col & 1;
                float gate = 0.f, up = 0.f;
                for (int s = 0; s < S_; ++s) {
                    const float *v = rf + ((r + R * s) * 32 + ln) * 4;
                    gate += v[sub];
                    up += v[2 + sub];
                }
                p.h[static_cast<size_t>(row) * I + tile * 8 * R + 8 * r + g] = gate / (1.0f + expf(-gate)) * up;
            }
        }
    } else {
        const int H = p.w.H, R = S.geo[3].R, S_ = kWarps / R, tp = tokens_per_pass(1, p.w.I);
        const int lr = __ffs(16 * R) - 1;
        const int ntok = min(tp, cnt - pass * tp);
        const int my_row = lane < ntok ? entry_row(p, S, a, pass * tp + lane) : 0;
        const int n_out = ntok << lr;
        const int Sk = p.T * p.k;
        for (int o0 = 0; o0 < n_out; o0 += 32) {
            const int o = o0 + lane;
            const int n = min(o >> lr, ntok - 1);
            const int row = __shfl_sync(0xffffffffu, my_row, n);
            if (o < n_out) {
                const int rr = o & (16 * R - 1), r = rr >> 4, row16 = rr & 15;
                const int ln = 4 * (row16 & 7) + (n & 3), idx = 2 * (n >> 2) + (row16 >> 3);
                float v = 0.f;
                for (int s = 0; s < S_; ++s) v += rf[((r + R * s) * 32 + ln) * 4 + idx];
                float *dst = row >= Sk ? p.y_shared + static_cast<size_t>(row - Sk) * H
                                       : p.y_slots + static_cast<size_t>(row) * H;
                dst[tile * 16 * R + rr] = v;
            }
        }
    }
}

// Epilogue warp of group `grp`: the group's items in order; when the tile
// sequence leaves a slot's gate_up tiles it publishes how many of them the
// group finished (after a fence, so that another CTA that sees the count also
// sees the h values).
__device__ __forceinline__ void run_epilogue(const FfnParams &p, StreamSmem &S, int grp, EpilogueState &es) {
    const int lane = threadIdx.x & 31;
    int m = es.m, pend = 0, i = es.i;
    bool ok = true;
    float4 *red = S.red + grp * kNR * (kWarps * 32);
    uint64_t *rfull = S.rfull + grp * kNR, *rempty = S.rempty + grp * kNR;
    Walk w;
    walk_begin(S, w);
    for (; ok && w.phase < 2; ++i) {
        const int phase = w.phase, a = w.a, tile = w.b;
        if (i % kGroups == grp) {
            const int np = n_passes(p, S, phase, a);
            for (int pass = 0; pass < np; ++pass) {
                const int r = m % kNR;
                if (!mbar_wait_warp(&rfull[r], (m / kNR) & 1, S.abort, p.wait_limit)) {
                    ok = false;
                    break;
                }
                epilogue_item(p, S, phase, a, tile, pass, red + r * (kWarps * 32));
                __syncwarp();
                if (lane == 0) mbar_arrive(&rempty[r]);
                ++m;
            }
            if (!ok) break;
            if (phase == 0) ++pend;
        }
        walk_next(S, w);
        if (phase == 0 && pend > 0 && (w.phase != 0 || w.a != a)) {
            __syncwarp();
            if (lane == 0 && a != p.skip_publish) {
                __threadfence();
                atomicAdd(p.ctr + a, pend);
            }
            pend = 0;
        }
    }
    es.m = m;
    es.i = i;
    if (!ok && lane == 0) abort_cta(p, S);
}

// Layout of the prologue's scratch inside the ring (byte offsets): the
// routing lists, the bf16 rows of x, and for a
// batch routed in the kernel the top-k candidates, choices, weights, slot
// positions and a few ints of scan space.
struct PrologueScratch {
    size_t lists, x, cand, idx, w, pos, tmp, topk, end;
};

__host__ __device__ __forceinline__ size_t align16(size_t v) { return (v + 15) & ~static_cast<size_t>(15); }

__host__ __device__ __forceinline__ PrologueScratch prologue_scratch(int H, int T, int k, int E, int max_slots,
                                                                     bool fused) {
    PrologueScratch ps;
    const size_t lists = static_cast<size_t>(max_slots) + E + 1;
    const size_t S_ = static_cast<size_t>(T) * k;
    ps.lists = 0;
    ps.x = align16(lists * sizeof(int));
    const bool need_x = fused || T <= kTokPerPass;
    ps.cand = align16(ps.x + (need_x ? static_cast<size_t>(T) * H * 2 : 0));
    // the logits partials: 4 quarters x kMaxExpertShare experts x 16 tokens
    ps.idx = align16(ps.cand + (fused ? 4 * static_cast<size_t>(kMaxExpertShare) * 16 * sizeof(float) : 0));
    ps.w = align16(ps.idx + (fused ? S_ * sizeof(int) : 0));
    ps.pos = align16(ps.w + (fused ? S_ * sizeof(float) : 0));
    ps.tmp = align16(ps.pos + (fused ? S_ * sizeof(int) : 0));
    // one token's top-k candidates: a key and an id per chunk of 32 logits and choice
    ps.topk = align16(ps.tmp + (fused ? 32 * sizeof(int) : 0));
    ps.end = ps.topk + (fused && T == 1 ? static_cast<size_t>((E + 31) / 32) * k * 8 : 0);
    return ps;
}

// The top k of n candidate keys (at most 32 * NJ) held in shared memory.
template <int NJ>
__device__ __forceinline__ void warp_topk_candidates(const uint32_t *ckey, int n, int k, int &pos, float &w) {
    const int lane = threadIdx.x & 31;
    uint32_t key[NJ];
#pragma unroll
    for (int j = 0; j < NJ; ++j) key[j] = lane + 32 * j < n ? ckey[lane + 32 * j] : 0u;
    warp_topk_rounds<NJ>(key, k, pos, w);
}

// One token (T == 1, k <= 31): warp 0 alone ends the routing from the top-k
// candidates of the grid's logits and builds this CTA's schedule.  It writes what cta_topk_rows,
// cta_group and plan_in_cta write (the choices and weights, the sorted slots,
// their positions, the active list, the slot tables and the tile runs), with
// the chosen experts held one per lane: the k choices of one token are
// distinct, so each is one slot and its sorted position is its rank.  The
// offsets are written only when fill_offsets.  The caller synchronises.
__device__ __forceinline__ void route_plan_one(const FfnParams &p, StreamSmem &S, int *act_s, int *off_s, int *idx_s,
                                               float *w_s, int *pos_s, const uint32_t *ckey, const int *cid,
                                               bool fill_offsets) {
    const int lane = threadIdx.x & 31;
    const int E = p.E, k = p.k;
    // the second stage of the top-k, over the candidates of cta_topk_candidates
    const int n = (E + 31) / 32 * k;
    int pos_r;
    float w_r;
    // the fewest keys per lane that hold them (a smaller tree per round)
    if (n <= 256) warp_topk_candidates<8>(ckey, n, k, pos_r, w_r);
    else if (n <= 512) warp_topk_candidates<16>(ckey, n, k, pos_r, w_r);
    else warp_topk_candidates<32>(ckey, n, k, pos_r, w_r);
    // (position -1, as id -1 before, only when fewer than k keys are valid)
    const int e_r = lane < k ? (pos_r >= 0 && pos_r < n ? cid[pos_r] : -1) : 0;
    int rank = 0;
    for (int j = 0; j < k; ++j) rank += __shfl_sync(0xffffffffu, e_r, j) < e_r;
    if (lane < k) {
        idx_s[lane] = e_r;
        w_s[lane] = w_r;
        pos_s[lane] = rank;
        S.srt[rank] = lane;
        act_s[1 + rank] = e_r;
    }
    if (lane == 0) act_s[0] = k;
    __syncwarp();
    // slot a = lane: the a-th chosen expert in id order, then the shared expert
    const PlanIn &pi = p.pi;
    const bool shared = pi.has_shared && pi.T <= pi.max_count;
    const int ns = k + (shared ? 1 : 0);
    int e = -1, bits = 0, ti = 0, jl = 0, first = 0;
    if (lane < k) {
        e = act_s[1 + lane];
        for (int t = 0; t < pi.n_tiers; ++t)
            if (e >= pi.first[t] && e - pi.first[t] < pi.n[t]) ti = t;
        bits = pi.bits[ti];
        jl = e - pi.first[ti];
        first = lane;
    } else if (lane == k && shared) {
        e = pi.E;
        bits = pi.shared_bits;
        ti = pi.n_tiers;
        first = k;
    }
    if (fill_offsets)  // offsets[x] = chosen experts below x
        for (int x0 = 0; x0 <= E; x0 += 32) {
            int c = 0;
            for (int a = 0; a < k; ++a) c += __shfl_sync(0xffffffffu, e, a) < x0 + lane;
            if (x0 + lane <= E) off_s[x0 + lane] = c;
        }
    // the tiles are dealt out in turn (below), so no tile costs are needed
    const int nt0 = S.nt0, nt1 = S.nt1;
    if (lane < ns) {
        const PlanTabs &t = S.pt;
        t.expert[lane] = e;
        t.bits[lane] = bits;
        t.tier[lane] = ti;
        t.jloc[lane] = jl;
        t.first[lane] = first;
        t.count[lane] = 1;
    }
    // one token: every tile is a single pass, so the tiles are dealt out in
    // turn (tile g to CTA g mod grid; see plan_in_cta)
    if (lane == 0) {
        S.range[0] = blockIdx.x;
        S.range[1] = ns * nt0;
        S.range[2] = blockIdx.x;
        S.range[3] = ns * nt1;
        S.range[4] = ns;
        S.range[5] = gridDim.x;
    }
}

// The batch routed by the FFN kernel itself (every thread of every CTA): the
// logits of this CTA's share of the experts, a grid barrier, then the top-k
// of every token and the stable grouping of the T*k slots, into the same
// shared-memory lists the prologue otherwise copies from global memory.  CTA 0
// also writes the routing outputs.  Returns 0 when the grid barrier gave up,
// 2 when the schedule is built too (one token), else 1.
__device__ __forceinline__ int route_in_cta(const FfnParams &p, StreamSmem &S, const uint16_t *x_s, int *act_s,
                                          int *off_s, const PrologueScratch &ps, const uint16_t *wr_s = nullptr) {
    const int T = p.T, E = p.E, k = p.k, H = p.w.H, S_ = T * k;
    // logits of experts [E * c / G, E * (c + 1) / G), all warps
    const int e0 = static_cast<int>(static_cast<long long>(E) * blockIdx.x / gridDim.x);
    const int e1 = static_cast<int>(static_cast<long long>(E) * (blockIdx.x + 1) / gridDim.x);
    cta_logits(x_s, T, H, E, p.route.wr, wr_s, p.route.bias, e0, e1,
               reinterpret_cast<float *>(S.ring + ps.cand), p.route.logits);
    int *barrier_ok = S.range + 7;
    __syncthreads();  // every thread's logits are written before thread 0 arrives
    if (threadIdx.x == 0) {
        const bool ok = grid_barrier(p.route.gbar, S.abort[1]++, S.abort, p.wait_limit);
        if (!ok) {
            status_or(p.status, MOE_STATUS_TIMEOUT);
            *static_cast<volatile int *>(S.abort) = 1;
        }
        *barrier_ok = ok;
    }
    __syncthreads();
    if (!*barrier_ok) return 0;
    int *idx_s = reinterpret_cast<int *>(S.ring + ps.idx);
    float *w_s = reinterpret_cast<float *>(S.ring + ps.w);
    int *pos_s = reinterpret_cast<int *>(S.ring + ps.pos);
    const bool one = T == 1 && k <= 31 && E <= 1024 && p.pi.max_count >= 1 && S.srt != nullptr;
    if (one) {
        uint32_t *ckey = reinterpret_cast<uint32_t *>(S.ring + ps.topk);
        int *cid = reinterpret_cast<int *>(ckey + (E + 31) / 32 * k);
        cta_topk_candidates(p.route.logits, E, k, ckey, cid);
        __syncthreads();
        if (threadIdx.x < 32)
            route_plan_one(p, S, act_s, off_s, idx_s, w_s, pos_s, ckey, cid,
                           blockIdx.x == 0 && p.route.topk_idx != nullptr);
        __syncthreads();
    } else {
        cta_topk_rows(p.route.logits, T, E, k, idx_s, w_s);
        cta_group(idx_s, S_, E, S.srt, pos_s, act_s, off_s, reinterpret_cast<int *>(S.ring + ps.tmp));
    }
    if (blockIdx.x == 0 && p.route.topk_idx) {
        for (int i = threadIdx.x; i < S_; i += blockDim.x) {
            p.route.topk_idx[i] = idx_s[i];
            p.route.topk_w[i] = w_s[i];
            p.route.sorted[i] = S.srt[i];
            p.route.slot_pos[i] = pos_s[i];
        }
        for (int e = threadIdx.x; e <= E; e += blockDim.x) p.route.offsets[e] = off_s[e];
        for (int a = threadIdx.x; a <= act_s[0]; a += blockDim.x) p.route.active[a] = act_s[a];
    }
    return one ? 2 : 1;
}

// Shared memory of a CTA (same layout for every launch shape): the ring,
// the all-token x fragments, B-operand and partial-sum buffers, barriers,
// flags, shelf pointers, geometry, slot tables and the sorted slot ids.
// Returns the first byte past it.
__device__ __forceinline__ uint8_t *carve_stream_smem(uint8_t *smem, int ring_bytes, int H, int I, int T, int k,
                                                      int max_slots, StreamSmem &S) {
    uint8_t *q = smem;
    S.ring = q;
    S.ring_bytes = ring_bytes;
    q += ring_bytes;
    const int xb = xall_bytes(H, T);
    S.xall = xb ? q : nullptr;
    q += xb;
    S.b_bytes = bbuf_bytes(H, I, T);
    S.bbuf = q;
    S.nb = n_bbufs(T);
    S.nb_log2 = S.nb == 4 ? 2 : 1;
    q += S.nb * S.b_bytes;
    S.red = reinterpret_cast<float4 *>(q);
    q += kGroups * kNR * kRedBytes;
    uint64_t *bars = reinterpret_cast<uint64_t *>(q);
    S.full = bars;
    S.empty = bars + kND;
    S.rfull = bars + 2 * kND;
    S.rempty = S.rfull + kGroups * kNR;
    S.bfull = S.rempty + kGroups * kNR;
    S.bempty = S.bfull + kNBMax;
    q = reinterpret_cast<uint8_t *>(S.bempty + kNBMax);
    S.abort = reinterpret_cast<int *>(q);
    S.range = S.abort + 4;  // gs0, ge0, gs1, ge1, n_slots, stride, flag, routing flag (16-byte aligned)
    S.pst = S.abort + 12;
    q += (12 + 2 * kND) * sizeof(int);
    S.tp = reinterpret_cast<TierPtrs *>(q);
    q += (MOE_MAX_TIERS + 1) * sizeof(TierPtrs);
    S.geo = reinterpret_cast<Geo *>(q);
    q += 6 * sizeof(Geo);
    q = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(q) + 15) & ~static_cast<uintptr_t>(15));
    S.pt = plan_tabs(q, max_slots);
    q += plan_tab_bytes(max_slots);
    const int n_srt = T * k;
    S.srt = n_srt <= kMaxSmemEntries ? reinterpret_cast<int *>(q) : nullptr;
    if (S.srt) q += ((n_srt * sizeof(int) + 15) / 16) * 16;
    S.nt0 = tiles_per_slot(H, I, 0);
    S.nt1 = tiles_per_slot(H, I, 1);
    return q;
}

// Host mirror of carve_stream_smem: bytes past the ring.
__host__ __forceinline__ size_t stream_smem_fixed(int H, int I, int T, int k, int max_slots) {
    const size_t n_srt = static_cast<size_t>(T) * k;
    return static_cast<size_t>(xall_bytes(H, T)) + n_bbufs(T) * static_cast<size_t>(bbuf_bytes(H, I, T)) +
           kGroups * kNR * static_cast<size_t>(kRedBytes) +
           (2 * kND + 2 * kGroups * kNR + 2 * kNBMax) * sizeof(uint64_t) + (12 + 2 * kND) * sizeof(int) +
           (MOE_MAX_TIERS + 1) * sizeof(TierPtrs) + 6 * sizeof(Geo) + 16 + plan_tab_bytes(max_slots) +
           (n_srt <= static_cast<size_t>(kMaxSmemEntries) ? (n_srt * sizeof(int) + 15) / 16 * 16 : 0);
}

// The pipeline's barriers, the abort flag and the tile geometry (thread 0
// and threads < 6; the caller synchronises).
__device__ __forceinline__ void init_stream_smem(StreamSmem &S, int H, int I) {
    if (threadIdx.x == 0) {
        for (int i = 0; i < kND; ++i) {
            mbar_init(&S.full[i], 1);  // the producer's expect_tx arrival
            mbar_init(&S.empty[i], kWarps);
        }
        for (int i = 0; i < kGroups * kNR; ++i) {
            mbar_init(&S.rfull[i], kWarps);
            mbar_init(&S.rempty[i], 1);
        }
        for (int i = 0; i < kNBMax; ++i) {
            mbar_init(&S.bfull[i], 1);
            mbar_init(&S.bempty[i], kComputeWarps);
        }
        S.abort[0] = 0;
        S.abort[1] = 0;  // grid barriers this CTA has passed
        mbar_fence_init();
    }
    if (threadIdx.x < 6) {
        const int phase = threadIdx.x / 3, bi = threadIdx.x % 3;
        const int bits = bi == 0 ? 8 : (bi == 1 ? 4 : 3);
        S.geo[threadIdx.x] = phase == 0 ? geo_gu(H, bits) : geo(I, bits);
    }
}

// Table pointers of the layer's shelves and shared expert (thread 0).
__device__ __forceinline__ void fill_tier_ptrs(const moe_layer_weights &w, StreamSmem &S) {
    if (threadIdx.x != 0) return;
#pragma unroll
    for (int t = 0; t < MOE_MAX_TIERS; ++t) {
        if (t < w.n_tiers) {
            S.tp[t].gq = w.tiers[t].gu_qs;
            S.tp[t].gs = reinterpret_cast<const uint8_t *>(w.tiers[t].gu_scale);
            S.tp[t].dq = w.tiers[t].dn_qs;
            S.tp[t].ds = reinterpret_cast<const uint8_t *>(w.tiers[t].dn_scale);
        }
    }
    const int t = w.n_tiers;
    S.tp[t].gq = w.shared.gu_qs;
    S.tp[t].gs = reinterpret_cast<const uint8_t *>(w.shared.gu_scale);
    S.tp[t].dq = w.shared.dn_qs;
    S.tp[t].ds = reinterpret_cast<const uint8_t *>(w.shared.dn_scale);
}

// The slot table and this CTA's tile runs from the active list and the expert
// offsets in shared memory (every thread; ends before a barrier).
__device__ __forceinline__ void plan_in_cta(const FfnParams &p, StreamSmem &S, const int *act_s, const int *off_s) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (warp == 0) {
        const int ns = plan_compact(p.pi, act_s, off_s, S.pt);
        if (lane == 0) S.range[4] = ns;
    }
    __syncthreads();
    // With one or two tokens (every tile a single pass), the tiles of a
    // phase are dealt out in turn: CTA c takes the global tiles c, c + grid,
    // ...  Each CTA then works through the slots in order, so the slots'
    // gate_up results complete one after another and the down tiles of early
    // slots find their operand ready, where contiguous runs finish every slot
    // only near the end of the phase (decode layer at one token: 44.9 ->
    // 42.6 us).  Dealt tiles change slot at every tile, so the loader builds
    // a down operand per tile; from about five tokens on that costs more than
    // it saves, and each CTA takes the contiguous run of an equal share of
    // the phase's cost instead.
    const bool dealt = p.T <= kDealtMaxTokens && p.T <= tokens_per_pass(1, p.w.I);
    if (warp < 2) {
        const int ns = S.range[4];
        const long long total = plan_costs(p.pi, ns, warp, S.pt);
        if (lane == 0) {
            const int nt = warp == 0 ? S.nt0 : S.nt1;
            const int2 r = dealt ? make_int2(static_cast<int>(blockIdx.x), ns * nt)
                                 : plan_cta_range(S.pt, ns, nt, warp, total, blockIdx.x, gridDim.x);
            S.range[2 * warp] = r.x;
            S.range[2 * warp + 1] = r.y;
            if (warp == 0) S.range[5] = dealt ? gridDim.x : 1;
        }
    }
}

__global__ void __launch_bounds__(kBlockThreads, 1)
ffn_stream_kernel(const __grid_constant__ FfnParams p, const __grid_constant__ StreamMaps M, int ring_bytes) {
    extern __shared__ __align__(1024) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int max_slots = p.max_active + 1;
    StreamSmem S;
    carve_stream_smem(smem, ring_bytes, p.w.H, p.w.I, p.T, p.k, max_slots, S);
    const int n_srt = p.T * p.k;

    // Prologue.  One round of asynchronous copies brings into shared memory
    // either the plan the routing kernel wrote (the slot rows and this CTA's
    // tile runs) or the active list and the expert offsets to build it from,
    // and the sorted slot ids and (T <= kTokPerPass) the bf16 rows of x.  The
    // scratch copies sit in the ring, which no TMA copy touches before the
    // prologue's last barrier.
    init_stream_smem(S, p.w.H, p.w.I);
    fill_tier_ptrs(p.w, S);
    if (threadIdx.x == 0) {
        // the tensor maps of the shelves in use
        for (int t = 0; t <= p.w.n_tiers; ++t) {
            if (t == p.w.n_tiers && !p.has_shared) break;
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&M.gq[t])) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&M.dq[t])) : "memory");
        }
    }
    // everything above reads only the parameters; what follows reads the
    // routing kernel's outputs
    pdl_wait();
    pdl_trigger();
    const bool fused = p.route.on != 0;
    const PrologueScratch ps = prologue_scratch(p.w.H, p.T, p.k, p.E, max_slots, fused);
    int *act_s = reinterpret_cast<int *>(S.ring + ps.lists);  // active list + offsets
    int *off_s = act_s + max_slots;
    const uint8_t *x_s = S.ring + ps.x;
    if (!fused) {
        for (int i = threadIdx.x; i <= p.max_active; i += blockDim.x) cp_async_4b(act_s + i, p.active + i);
        for (int e = threadIdx.x; e <= p.E; e += blockDim.x) cp_async_4b(off_s + e, p.offsets + e);
    }
    if (S.srt && !fused)
        for (int j = threadIdx.x; j < n_srt; j += blockDim.x) cp_async_4b(S.srt + j, p.sorted + j);
    if (S.xall || fused)
        for (int c = threadIdx.x; c < p.T * p.w.H / 8; c += blockDim.x)
            cp_async_16b(const_cast<uint8_t *>(x_s) + 16 * c, p.x + 8 * static_cast<size_t>(c));
    cp_async_wait_all();
    __syncthreads();
    if (S.xall) {
        const bool xbad = build_xall(p, x_s, S.xall);
        if (__any_sync(0xffffffffu, xbad) && lane == 0) status_or(p.status, MOE_STATUS_FP16_RANGE);
    }
    int routed = 1;
    if (fused) routed = route_in_cta(p, S, reinterpret_cast<const uint16_t *>(x_s), act_s, off_s, ps);
    if (!routed) {  // the grid barrier gave up: stream nothing
        if (threadIdx.x < 6) S.range[threadIdx.x] = threadIdx.x == 5;  // empty runs, stride 1
    } else if (routed == 1) {
        plan_in_cta(p, S, act_s, off_s);
    }
    // the ring's scratch is overwritten by TMA copies from here on: order
    // this thread's generic accesses before them
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncthreads();

    if (warp == kWarpProducer) {
        ProducerState ps0 = {};
        run_producer(p, M, S, ps0, true);
        return;
    }
    if (warp < kComputeWarps) {
        ComputeState cs = {0, 0, -1};
        run_compute(p, S, warp, cs);
    } else if (warp == kWarpLoader) {
        LoaderState ls = {-1};
        run_loader(p, S, ls);
    } else if (warp >= kWarpEpilogue0) {
        EpilogueState es = {0, 0};
        run_epilogue(p, S, warp - kWarpEpilogue0, es);
    }
}

}  // namespace moe

// Shared memory of one CTA: the byte ring for staged tiles, the all-token x
// fragments, the B-operand and partial-sum buffers, barriers, and the slot
// tables.  Returns the byte count and the ring size in *ring_bytes (0 when
// the ring cannot hold the largest tile and the prologue's scratch).
size_t moe_ffn_stream_smem(int H, int I, int T, int k, int E, int max_slots, bool fused, int *ring_bytes) {
    const size_t fixed = moe::stream_smem_fixed(H, I, T, k, max_slots);
    const size_t budget = 227 * 1024;
    size_t ring = fixed < budget ? ((budget - fixed) & ~static_cast<size_t>(moe::kTileAlign - 1)) : 0;
    const size_t scratch = moe::prologue_scratch(H, T, k, E, max_slots, fused).end;
    if (ring < static_cast<size_t>(moe::kMaxTileBytes) || ring < scratch) ring = 0;
    *ring_bytes = static_cast<int>(ring);
    return ring + fixed;
}

cudaError_t moe_configure_ffn_stream() {
    return cudaFuncSetAttribute(moe::ffn_stream_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
}

bool moe_ffn_stream_supported(int H, int I) {
    return H <= moe::kMaxK && I <= moe::kMaxK && H % 128 == 0 && I % 128 == 0;
}

// Whether a launch for this batch gets a ring that holds the largest tile.
bool moe_ffn_stream_fits(int H, int I, int T, int k, int E, int max_slots) {
    int ring = 0, ring2 = 0;
    moe_ffn_stream_smem(H, I, T, k, E, max_slots, false, &ring);
    moe_ffn_stream_smem(H, I, T, k, E, max_slots, T <= moe::kRouterTokTile, &ring2);
    return ring > 0 && ring2 > 0;
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
    const moe::Geo g0 = moe::geo_gu(H, tier.bits), g1 = moe::geo(I, moe::tier_dn_bits(tier));
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
    int ring = 0;
    const size_t smem = moe_ffn_stream_smem(p.w.H, p.w.I, p.T, p.k, p.E, p.max_active + 1, p.route.on != 0, &ring);
    if (ring == 0) return cudaErrorInvalidConfiguration;
    int dev = 0;
    cudaGetDevice(&dev);
    int sms = 0;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (p.route.on && (p.E + sms - 1) / sms > moe::kMaxExpertShare) return cudaErrorInvalidConfiguration;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(sms);
    cfg.blockDim = dim3(moe::kBlockThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    moe::PdlAttrs at(true);
    cfg.attrs = at.a;
    cfg.numAttrs = at.n;
    moe::StreamMaps M;
    std::memset(&M, 0, sizeof(M));
    for (int t = 0; t < p.w.n_tiers; ++t)
        if (!shelf_maps(M, t, p.w.tiers[t], p.w.H, p.w.I)) return cudaErrorInvalidValue;
    if (p.has_shared && !shelf_maps(M, p.w.n_tiers, p.w.shared, p.w.H, p.w.I)) return cudaErrorInvalidValue;
    cudaError_t e = cudaLaunchKernelEx(&cfg, moe::ffn_stream_kernel, p, M, ring);
    if (e != cudaSuccess) {  // without overlapping the predecessor
        cudaGetLastError();
        cfg.attrs = at.a + 1;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, moe::ffn_stream_kernel, p, M, ring);
    }
    return e;
}

// ---------------------------------------------------------------------------
// A stack of decode layers in one persistent launch ([P5] "What the model
// actually is": 48 layers, a residual design; [P1] "step 3": the per-token
// profile is dominated by launches and syncs, not by expert bytes).
//
// Every CTA loops over the layers.  Per layer: the RMS norm of the residual
// stream (each CTA recomputes it, in one fixed order), the router logits of
// its share of the experts, a grid barrier, then every CTA ranks and groups
// the tokens and plans its tiles; the warp-role pipeline streams the layer's
// experts; a grid barrier; each CTA adds its slice of the combined output
// into the next residual buffer; a grid barrier.  The pipeline's barriers,
// ring offsets and operand buffers carry over from layer to layer, and the
// code stays resident in the instruction caches.
// ---------------------------------------------------------------------------
namespace moe {

struct __align__(64) StackLayer {
    StreamMaps maps;
    moe_layer_weights w;
    const uint16_t *wr;
    const float *bias;
    PlanShelves shelves;                // the schedule's view of w, prepared on the host
    TierPtrs tp[MOE_MAX_TIERS + 1];     // the shelves' table pointers, shared expert last
};

// Copy n 4-byte words from global to shared memory, one word per thread.
__device__ __forceinline__ void copy_words(void *dst, const void *src, int n) {
    for (int i = threadIdx.x; i < n; i += blockDim.x)
        static_cast<int *>(dst)[i] = __ldg(static_cast<const int *>(src) + i);
}

struct StackParams {
    const StackLayer *layers;
    int n_layers, T, k, H, I, E;
    const uint16_t *x_in;  // bf16 [T][H] residual stream entering the first layer
    uint16_t *x_out;       // bf16 [T][H] residual stream leaving the last layer
    uint16_t *x_out_norm;  // its RMS-normalised copy, or null
    uint16_t *x_layers;    // [n_layers + 1][T][H] the stream at every layer boundary, or null
    uint16_t *xbuf;        // [2][T][H] residual stream between layers
    float *logits, *h, *y_slots, *y_shared;
    int *ctr;              // [min(T*k, E) + 1] per-slot gate_up counts (zero on entry)
    int *gbar;             // [2] grid barrier words (zero on entry)
    int32_t *status;
    long long wait_limit;
    int skip_publish;  // test hook, as in FfnParams (-1: none)
    int ring_bytes;
    int wr_stage;      // ring offset of this CTA's router rows staged for the logits, or -1
};

// Bytes past the shared stream layout: this layer's parameters, its top-k
// weights and the norm's scratch.
__host__ __device__ __forceinline__ size_t stack_smem_extra(int T, int k) {
    return (sizeof(FfnParams) + 15) / 16 * 16 + (static_cast<size_t>(T) * k * sizeof(float) + 15) / 16 * 16 +
           (static_cast<size_t>(T) + 32) * sizeof(float);
}

// n = bf16(x / sqrt(mean(x^2) + eps)) of every row of the bf16 tile x_s
// [T][H], in place (whole CTA; red: 32 + T floats of scratch).
__device__ __forceinline__ void cta_rms_norm_rows(uint16_t *x_s, int T, int H, float *red) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
    float *rinv = red + 32;
    for (int t = 0; t < T; ++t) {
        const uint16_t *xr = x_s + static_cast<size_t>(t) * H;
        float ss = 0.f;
        for (int c = threadIdx.x; c < H / 4; c += blockDim.x) {
            const uint2 v = *reinterpret_cast<const uint2 *>(xr + 4 * c);
            const float f0 = bf16lo(v.x), f1 = bf16hi(v.x), f2 = bf16lo(v.y), f3 = bf16hi(v.y);
            ss = fmaf(f0, f0, fmaf(f1, f1, fmaf(f2, f2, fmaf(f3, f3, ss))));
        }
        ss = warp_sum(ss);
        if (lane == 0) red[warp] = ss;
        __syncthreads();
        if (warp == 0) {
            float tot = lane < nwarps ? red[lane] : 0.f;
            tot = warp_sum(tot);
            if (lane == 0) rinv[t] = 1.0f / sqrtf(tot / static_cast<float>(H) + MOE_NORM_EPS);
        }
        __syncthreads();
    }
    for (int i = threadIdx.x; i < T * H / 2; i += blockDim.x) {
        const int t = (2 * i) / H;
        uint32_t v = reinterpret_cast<uint32_t *>(x_s)[i];
        const float r = rinv[t];
        v = static_cast<uint32_t>(f32_to_bf16_rne(bf16lo(v) * r)) |
            (static_cast<uint32_t>(f32_to_bf16_rne(bf16hi(v) * r)) << 16);
        reinterpret_cast<uint32_t *>(x_s)[i] = v;
    }
    __syncthreads();
}

// thread 0 of every CTA at a grid barrier; the result in every thread
__device__ __forceinline__ bool stack_barrier(const StackParams &P, StreamSmem &S) {
    __syncthreads();  // the CTA's writes before the barrier precede thread 0's arrival
    if (threadIdx.x == 0) {
        const bool ok =
            !*static_cast<volatile int *>(S.abort) && grid_barrier(P.gbar, S.abort[1]++, S.abort, P.wait_limit);
        if (!ok) {
            status_or(P.status, MOE_STATUS_TIMEOUT);
            *static_cast<volatile int *>(S.abort) = 1;
        }
        S.range[6] = ok;
    }
    __syncthreads();
    return S.range[6] != 0;
}

__global__ void __launch_bounds__(kBlockThreads, 1) stack_kernel(const __grid_constant__ StackParams P) {
    extern __shared__ __align__(1024) uint8_t smem[];
    const int warp = threadIdx.x >> 5;
    const int T = P.T, k = P.k, H = P.H, E = P.E, S_ = T * k;
    const int max_active = min(S_, E), max_slots = max_active + 1;
    StreamSmem S;
    uint8_t *q = carve_stream_smem(smem, P.ring_bytes, H, P.I, T, k, max_slots, S);
    FfnParams &p = *reinterpret_cast<FfnParams *>(q);
    q += (sizeof(FfnParams) + 15) / 16 * 16;
    float *wkeep = reinterpret_cast<float *>(q);
    q += (static_cast<size_t>(S_) * sizeof(float) + 15) / 16 * 16;
    float *red = reinterpret_cast<float *>(q);
    init_stream_smem(S, H, P.I);
    ProducerState prs = {};
    ComputeState cst = {0, 0, -1};
    LoaderState lds = {-1};
    EpilogueState eps = {0, 0};
    const PrologueScratch ps = prologue_scratch(H, T, k, E, max_slots, true);
    int *act_s = reinterpret_cast<int *>(S.ring + ps.lists);
    int *off_s = act_s + max_slots;
    uint16_t *x_s = reinterpret_cast<uint16_t *>(S.ring + ps.x);
    pdl_wait();
    pdl_trigger();
    if (P.x_layers && blockIdx.x == 0)
        for (int i = threadIdx.x; i < T * H / 8; i += blockDim.x)
            reinterpret_cast<uint4 *>(P.x_layers)[i] = reinterpret_cast<const uint4 *>(P.x_in)[i];
    if (threadIdx.x == 0) {
        p.E = E;
        p.T = T;
        p.k = k;
        p.max_active = max_active;
        p.x = nullptr;
        p.offsets = p.sorted = p.active = nullptr;
        p.h = P.h;
        p.ctr = P.ctr;
        p.max_count = 0x7fffffff;
        p.y_slots = P.y_slots;
        p.y_shared = P.y_shared;
        p.status = P.status;
        PlanIn &pi = p.pi;
        pi.E = E;
        pi.T = T;
        pi.k = k;
        pi.H = H;
        pi.I = P.I;
        pi.max_count = 0x7fffffff;
        pi.max_active = max_active;
        p.route.on = 1;
        p.route.logits = P.logits;
        p.route.topk_idx = nullptr;
        p.route.topk_w = nullptr;
        p.route.offsets = p.route.sorted = p.route.slot_pos = p.route.active = nullptr;
        p.route.gbar = P.gbar;
        p.wait_limit = P.wait_limit;
        p.skip_publish = P.skip_publish;
    }
    bool alive = true;
    for (int l = 0; l < P.n_layers && alive; ++l) {
        const StackLayer &Ld = P.layers[l];
        const uint16_t *xl = l == 0 ? P.x_in : P.xbuf + static_cast<size_t>((l - 1) & 1) * T * H;
        uint16_t *xn = l + 1 == P.n_layers ? P.x_out : P.xbuf + static_cast<size_t>(l & 1) * T * H;
        // the residual stream entering the layer (in flight while the
        // descriptor below is read)
        for (int c = threadIdx.x; c < T * H / 8; c += blockDim.x)
            cp_async_16b(x_s + 8 * c, xl + 8 * static_cast<size_t>(c));
        // and this CTA's router rows (they do not depend on x), so that the
        // logits read them from shared memory after the norm
        const int re0 = static_cast<int>(static_cast<long long>(E) * blockIdx.x / gridDim.x);
        const int re1 = static_cast<int>(static_cast<long long>(E) * (blockIdx.x + 1) / gridDim.x);
        uint16_t *wr_s = P.wr_stage >= 0 ? reinterpret_cast<uint16_t *>(S.ring + P.wr_stage) : nullptr;
        if (wr_s) {
            const uint16_t *rows = Ld.wr + static_cast<size_t>(re0) * H;
            for (int c = threadIdx.x; c < (re1 - re0) * H / 8; c += blockDim.x)
                cp_async_16b(wr_s + 8 * c, rows + 8 * static_cast<size_t>(c));
        }
        // this layer's weights descriptor, the schedule's view of its shelves and
        // their table pointers into shared memory (a word per thread, one round)
        {
            copy_words(&p.w, &Ld.w, sizeof(moe_layer_weights) / sizeof(int));
            copy_words(p.pi.shelves(), &Ld.shelves, sizeof(PlanShelves) / sizeof(int));
            copy_words(S.tp, Ld.tp, sizeof(Ld.tp) / sizeof(int));
            if (threadIdx.x == 0) {
                p.has_shared = __ldg(&Ld.shelves.has_shared);
                p.route.wr = Ld.wr;
                p.route.bias = Ld.bias;
                for (int t = 0; t <= MOE_MAX_TIERS; ++t) {
                    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&Ld.maps.gq[t])) : "memory");
                    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&Ld.maps.dq[t])) : "memory");
                }
            }
        }
        cp_async_wait_all();
        __syncthreads();
        // normalised in place (its barriers also publish the parameters above)
        cta_rms_norm_rows(x_s, T, H, red);
        {
            const bool xbad = build_xall(p, reinterpret_cast<const uint8_t *>(x_s), S.xall);
            if (__any_sync(0xffffffffu, xbad) && (threadIdx.x & 31) == 0) status_or(P.status, MOE_STATUS_FP16_RANGE);
        }
        const int routed = route_in_cta(p, S, x_s, act_s, off_s, ps, wr_s);
        if (!routed) {
            alive = false;
            break;
        }
        for (int i = threadIdx.x; i < S_; i += blockDim.x) wkeep[i] = reinterpret_cast<const float *>(S.ring + ps.w)[i];
        if (routed == 1) plan_in_cta(p, S, act_s, off_s);
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncthreads();
        const bool last = l + 1 == P.n_layers;
        if (!last && threadIdx.x == 32 * kWarpLoader) {
            // the next layer's router rows of this CTA and a slice of its shared
            // expert (needed whatever the routing) into L2 while this layer streams
            const StackLayer &Nx = P.layers[l + 1];
            const int e0 = static_cast<int>(static_cast<long long>(E) * blockIdx.x / gridDim.x);
            const int e1 = static_cast<int>(static_cast<long long>(E) * (blockIdx.x + 1) / gridDim.x);
            prefetch_l2(Nx.wr + static_cast<size_t>(e0) * H, static_cast<uint32_t>((e1 - e0) * H * 2));
            if (Nx.w.shared.n_experts == 1) {
                const moe_tier &sh = Nx.w.shared;
                const int gbits = storage_bits(sh.bits), dbits = storage_bits(tier_dn_bits(sh));
                const size_t gq = static_cast<size_t>(2) * P.I * H * gbits / 8, gs = static_cast<size_t>(2) * P.I * (H / 32) * 2;
                const size_t dq = static_cast<size_t>(H) * P.I * dbits / 8, ds = static_cast<size_t>(H) * (P.I / 32) * 2;
                const void *base[4] = {sh.gu_qs, sh.gu_scale, sh.dn_qs, sh.dn_scale};
                const size_t len[4] = {gq, gs, dq, ds};
                for (int a = 0; a < 4; ++a) {
                    const size_t c0 = (len[a] * blockIdx.x / gridDim.x) & ~static_cast<size_t>(15);
                    const size_t c1 = blockIdx.x + 1 == gridDim.x ? len[a] : ((len[a] * (blockIdx.x + 1) / gridDim.x) & ~static_cast<size_t>(15));
                    prefetch_l2(static_cast<const uint8_t *>(base[a]) + c0, static_cast<uint32_t>(c1 - c0));
                }
            }
        }
        if (warp == kWarpProducer) run_producer(p, Ld.maps, S, prs, last);
        else if (warp < kComputeWarps) run_compute(p, S, warp, cst);
        else if (warp == kWarpLoader) run_loader(p, S, lds);
        else if (warp >= kWarpEpilogue0) run_epilogue(p, S, warp - kWarpEpilogue0, eps);
        __syncthreads();
        if (!stack_barrier(P, S)) {
            alive = false;
            break;
        }
        // this CTA's slice of out = bf16(sum_j w_j y_j + y_shared), x' = bf16(x + out)
        const int nch = T * H / 4;
        const int c0 = static_cast<int>(static_cast<long long>(nch) * blockIdx.x / gridDim.x);
        const int c1 = static_cast<int>(static_cast<long long>(nch) * (blockIdx.x + 1) / gridDim.x);
        for (int c = c0 + static_cast<int>(threadIdx.x); c < c1; c += blockDim.x) {
            const int t = c / (H / 4), col = c - t * (H / 4);
            float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int j = 0; j < k; ++j) {
                const float4 v = __ldcg(reinterpret_cast<const float4 *>(P.y_slots + (static_cast<size_t>(t) * k + j) * H) + col);
                const float wj = wkeep[t * k + j];
                a.x = fmaf(wj, v.x, a.x);
                a.y = fmaf(wj, v.y, a.y);
                a.z = fmaf(wj, v.z, a.z);
                a.w = fmaf(wj, v.w, a.w);
            }
            if (p.has_shared) {
                const float4 v = __ldcg(reinterpret_cast<const float4 *>(P.y_shared + static_cast<size_t>(t) * H) + col);
                a.x += v.x; a.y += v.y; a.z += v.z; a.w += v.w;
            }
            const uint2 r = __ldcg(reinterpret_cast<const uint2 *>(xl + static_cast<size_t>(t) * H) + col);
            const uint16_t n0 = f32_to_bf16_rne(bf16lo(r.x) + bf16_to_f32(f32_to_bf16_rne(a.x)));
            const uint16_t n1 = f32_to_bf16_rne(bf16hi(r.x) + bf16_to_f32(f32_to_bf16_rne(a.y)));
            const uint16_t n2 = f32_to_bf16_rne(bf16lo(r.y) + bf16_to_f32(f32_to_bf16_rne(a.z)));
            const uint16_t n3 = f32_to_bf16_rne(bf16hi(r.y) + bf16_to_f32(f32_to_bf16_rne(a.w)));
            const uint2 o = make_uint2(static_cast<uint32_t>(n0) | (static_cast<uint32_t>(n1) << 16),
                                       static_cast<uint32_t>(n2) | (static_cast<uint32_t>(n3) << 16));
            reinterpret_cast<uint2 *>(xn + static_cast<size_t>(t) * H)[col] = o;
            if (P.x_layers)
                reinterpret_cast<uint2 *>(P.x_layers + (static_cast<size_t>(l + 1) * T + t) * H)[col] = o;
        }
        // the per-slot counts start from zero in the next layer (nobody reads them now)
        if (blockIdx.x == 0)
            for (int i = threadIdx.x; i < max_slots; i += blockDim.x) P.ctr[i] = 0;
        if (!stack_barrier(P, S)) {
            alive = false;
            break;
        }
    }
    // after a failed barrier: wait for any copy this CTA still has in flight
    // (the last kND tiles issued: each was the last use of its descriptor)
    if (!alive && warp == kWarpProducer && (threadIdx.x & 31) == 0)
        for (int j = max(0, prs.i - kND); j < prs.i; ++j)
            if (!mbar_wait_limit(&S.full[j % kND], (j / kND) & 1, P.wait_limit)) status_or(P.status, MOE_STATUS_TIMEOUT);
    if (alive && P.x_out_norm && blockIdx.x == 0) {
        for (int c = threadIdx.x; c < T * H / 8; c += blockDim.x)
            reinterpret_cast<uint4 *>(x_s)[c] = __ldcg(reinterpret_cast<const uint4 *>(P.x_out) + c);
        __syncthreads();
        cta_rms_norm_rows(x_s, T, H, red);
        for (int c = threadIdx.x; c < T * H / 8; c += blockDim.x)
            reinterpret_cast<uint4 *>(P.x_out_norm)[c] = reinterpret_cast<const uint4 *>(x_s)[c];
    }
}

}  // namespace moe

size_t moe_stack_layer_bytes() { return sizeof(moe::StackLayer); }

// One layer of a stack descriptor, encoded on the host into `dst`
// (sizeof(StackLayer) bytes): the tensor maps of its shelves, the weights
// descriptor and the router.
cudaError_t moe_stack_encode_layer(const moe_layer_weights *w, const uint16_t *wr, const float *bias, void *dst) {
    moe::StackLayer L;
    std::memset(&L, 0, sizeof(L));
    for (int t = 0; t < w->n_tiers; ++t)
        if (!shelf_maps(L.maps, t, w->tiers[t], w->H, w->I)) return cudaErrorInvalidValue;
    if (w->shared.n_experts == 1 && !shelf_maps(L.maps, w->n_tiers, w->shared, w->H, w->I)) return cudaErrorInvalidValue;
    L.w = *w;
    L.wr = wr;
    L.bias = bias;
    L.shelves.n_tiers = w->n_tiers;
    L.shelves.has_shared = w->shared.n_experts == 1;
    L.shelves.shared_bits = moe::tier_formats(w->shared);
    for (int t = 0; t < MOE_MAX_TIERS; ++t) {
        const bool on = t < w->n_tiers;
        L.shelves.first[t] = on ? w->tiers[t].first_expert : 0;
        L.shelves.n[t] = on ? w->tiers[t].n_experts : 0;
        L.shelves.bits[t] = on ? moe::tier_formats(w->tiers[t]) : 8 | (8 << 8);
        if (on)
            L.tp[t] = {w->tiers[t].gu_qs, reinterpret_cast<const uint8_t *>(w->tiers[t].gu_scale), w->tiers[t].dn_qs,
                       reinterpret_cast<const uint8_t *>(w->tiers[t].dn_scale)};
    }
    L.tp[w->n_tiers] = {w->shared.gu_qs, reinterpret_cast<const uint8_t *>(w->shared.gu_scale), w->shared.dn_qs,
                        reinterpret_cast<const uint8_t *>(w->shared.dn_scale)};
    std::memcpy(dst, &L, sizeof(L));
    return cudaSuccess;
}

// Shared memory of the stack kernel; *ring_bytes = 0 when the ring cannot
// hold the largest tile and the per-layer scratch.
size_t moe_stack_smem(int H, int I, int T, int k, int E, int *ring_bytes) {
    const int max_slots = (T * k < E ? T * k : E) + 1;
    const size_t fixed = moe::stream_smem_fixed(H, I, T, k, max_slots) + moe::stack_smem_extra(T, k);
    const size_t budget = 227 * 1024;
    size_t ring = fixed < budget ? ((budget - fixed) & ~static_cast<size_t>(moe::kTileAlign - 1)) : 0;
    const size_t scratch = moe::prologue_scratch(H, T, k, E, max_slots, true).end;
    if (ring < static_cast<size_t>(moe::kMaxTileBytes) || ring < scratch) ring = 0;
    *ring_bytes = static_cast<int>(ring);
    return ring + fixed;
}

cudaError_t moe_configure_stack() {
    return cudaFuncSetAttribute(moe::stack_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
}

// ctr and gbar must be zero on entry; the caller clears them.
cudaError_t moe_launch_stack(const void *layers, int n_layers, int T, int k, int H, int I, int E, const uint16_t *x_in,
                             uint16_t *x_out, uint16_t *x_out_norm, uint16_t *x_layers, uint16_t *xbuf, float *logits,
                             float *h, float *y_slots, float *y_shared, int *ctr, int *gbar, int32_t *status,
                             long long wait_limit, int skip_publish, cudaStream_t s) {
    moe::StackParams P;
    std::memset(&P, 0, sizeof(P));
    P.layers = static_cast<const moe::StackLayer *>(layers);
    P.n_layers = n_layers;
    P.T = T;
    P.k = k;
    P.H = H;
    P.I = I;
    P.E = E;
    P.x_in = x_in;
    P.x_out = x_out;
    P.x_out_norm = x_out_norm;
    P.x_layers = x_layers;
    P.xbuf = xbuf;
    P.logits = logits;
    P.h = h;
    P.y_slots = y_slots;
    P.y_shared = y_shared;
    P.ctr = ctr;
    P.gbar = gbar;
    P.status = status;
    P.wait_limit = wait_limit;
    P.skip_publish = skip_publish;
    int ring = 0;
    const size_t smem = moe_stack_smem(H, I, T, k, E, &ring);
    if (ring == 0) return cudaErrorInvalidConfiguration;
    P.ring_bytes = ring;
    int dev = 0, sms = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if ((E + sms - 1) / sms > moe::kMaxExpertShare) return cudaErrorInvalidConfiguration;
    // the router rows of a CTA (at most ceil(E / grid)) staged in the ring's
    // scratch after the routing lists, when they fit, for one or two tokens
    // (with more, the norm already covers their latency and the extra copies
    // measured slower)
    if (T > 2) {
        P.wr_stage = -1;
    } else {
        const int max_slots = (T * k < E ? T * k : E) + 1;
        const size_t at = moe::align16(moe::prologue_scratch(H, T, k, E, max_slots, true).end);
        const size_t need = at + static_cast<size_t>((E + sms - 1) / sms) * H * sizeof(uint16_t);
        P.wr_stage = need <= static_cast<size_t>(ring) ? static_cast<int>(at) : -1;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(sms);
    cfg.blockDim = dim3(moe::kBlockThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    moe::PdlAttrs at(true);
    cfg.attrs = at.a;
    cfg.numAttrs = at.n;
    cudaError_t e = cudaLaunchKernelEx(&cfg, moe::stack_kernel, P);
    if (e != cudaSuccess) {
        cudaGetLastError();
        cfg.attrs = at.a + 1;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, moe::stack_kernel, P);
    }
    return e;
}
