// Tile schedule of the streaming expert FFN: which slots (active experts and
// the shared expert) it serves, and which tiles of them each CTA streams.
//
// [P1] "step 4: three shelves, all on the GPU": every chosen expert is read
// from whichever shelf holds it, so one schedule spans all shelves; tiles of
// 8-, 4- and 3-bit experts differ in bytes and dequantisation work, and the
// schedule balances both across the CTAs.
//
// A slot's gate_up is cut into nt0 tiles (8R gate rows + the matching 8R up
// rows), its down projection into nt1 tiles of 16R rows, R = rows_pow2(K).
// Numbering the tiles of a phase globally as g = slot * nt + tile, each CTA
// takes the contiguous run of tiles whose start falls in its equal share of
// the phase's total cost, first of gate_up (phase 0), then of down (phase 1).
// (For one or two tokens the streaming kernel deals the tiles out in turn
// instead, CTA c taking g = c, c + grid, ...; see plan_in_cta.)
#pragma once
#include "common.cuh"

namespace moe {

constexpr int kTokPerPass = 8;               // gate_up token columns per pass over a resident tile
constexpr long long kTileFixedCost = 4000;  // per-tile waits and hand-offs (tenths of a ns, as tile_cost)

// Rows per tile are 16R: the largest power of two R <= 8 with 2RK <= 2048, so
// a tile holds at most 32K weights.
__host__ __device__ __forceinline__ int rows_pow2(int K) {
    int R = 1;
    while (R < 8 && 2 * R * K <= 2048) R *= 2;
    return R;
}

// n-tiles of 8 columns in a down pass (two fp16 columns, hi and lo, per token)
__host__ __device__ __forceinline__ int down_ntiles(int I) { return I <= 1024 ? 2 : 1; }

__host__ __device__ __forceinline__ int tokens_per_pass(int phase, int I) {
    return phase == 0 ? kTokPerPass : 4 * down_ntiles(I);
}

__host__ __device__ __forceinline__ int tiles_per_slot(int H, int I, int phase) {
    return phase == 0 ? I / (8 * rows_pow2(H)) : H / (16 * rows_pow2(I));
}

// Balancing weight of one tile, in tenths of a nanosecond of its CTA's time:
// a fixed share for waits and hand-offs, then the larger of the time to copy
// its bytes at an even share of HBM (about 44 GB/s per SM) and its dequantise-
// and-multiply time for every pass.  The two compute groups work side by
// side, so a tile occupies the CTA for half of one group's time, which was
// measured on B200 per 32K-weight tile and pass as 1.42 / 1.50 / 2.30 us for
// gate_up and 1.36 / 1.38 / 1.72 us for down with 8- / 4- / 3-bit codes;
// FP4 codes (4-bit storage, a longer decode) measured 5 % above 4-bit ones.
__host__ __device__ __forceinline__ long long tile_cost(int H, int I, int phase, int bits, int count) {
    const int K = phase == 0 ? H : I;
    const long long rows = 16 * rows_pow2(K);
    const int tp = tokens_per_pass(phase, I);
    const long long passes = (count + tp - 1) / tp;
    const long long bytes = rows * (K * storage_bits(bits) / 8 + K / 16);
    const long long copy = bytes * 227 / 1000;
    const long long per_tile = phase == 0 ? (bits == 8 ? 14200 : (bits == 4 ? 15000 : (bits == 3 ? 23000 : 15750)))
                                          : (bits == 8 ? 13600 : (bits == 4 ? 13800 : (bits == 3 ? 17200 : 14500)));
    const long long compute = passes * per_tile * rows * K / (2 * 32768);
    return kTileFixedCost + (copy > compute ? copy : compute);
}

// What the schedule needs to know about a layer and a call (no device pointers).
struct PlanShelves {  // the shelves of a layer; formats as tier_formats packs them
    int n_tiers, has_shared, shared_bits;
    int first[MOE_MAX_TIERS], n[MOE_MAX_TIERS], bits[MOE_MAX_TIERS];
};
struct PlanIn {
    int E, T, k, H, I;
    int max_count;   // slots with more tokens are left to the tensor-core path
    int max_active;  // routed slots at most: min(E, T*k)
    int n_tiers, has_shared, shared_bits;
    int first[MOE_MAX_TIERS], n[MOE_MAX_TIERS], bits[MOE_MAX_TIERS];
    // the fields from n_tiers on, as one block
    __host__ __device__ __forceinline__ PlanShelves *shelves() { return reinterpret_cast<PlanShelves *>(&n_tiers); }
};
static_assert(sizeof(PlanIn) == 7 * sizeof(int) + sizeof(PlanShelves), "PlanIn ends with its shelves block");

// Per-slot tables in shared memory.  tc/pre: per phase, the cost of one tile
// of the slot and the inclusive prefix sum of the slots' total costs.
struct PlanTabs {
    int *expert, *bits, *tier, *jloc, *first, *count;
    long long *tc0, *tc1, *pre0, *pre1;
    __device__ __forceinline__ long long *tc(int phase) const { return phase == 0 ? tc0 : tc1; }
    __device__ __forceinline__ long long *pre(int phase) const { return phase == 0 ? pre0 : pre1; }
};

__host__ __device__ __forceinline__ size_t plan_tab_bytes(int max_slots) {
    return static_cast<size_t>(max_slots) * (6 * sizeof(int) + 4 * sizeof(long long));
}

// Carve the tables from `base` (8-byte aligned, plan_tab_bytes bytes).
__device__ __forceinline__ PlanTabs plan_tabs(void *base, int max_slots) {
    PlanTabs t;
    long long *ll = static_cast<long long *>(base);
    t.tc0 = ll;
    t.tc1 = ll + max_slots;
    t.pre0 = ll + 2 * max_slots;
    t.pre1 = ll + 3 * max_slots;
    int *in = reinterpret_cast<int *>(ll + 4 * max_slots);
    t.expert = in;
    t.bits = in + max_slots;
    t.tier = in + 2 * max_slots;
    t.jloc = in + 3 * max_slots;
    t.first = in + 4 * max_slots;
    t.count = in + 5 * max_slots;
    return t;
}

// Slot table, compacted in order by one warp: the active routed experts whose
// token count is in (0, max_count], then the shared expert (when it has
// work on this path).  active[0] is the number of active experts, active[1..]
// their ids; offsets[e] .. offsets[e+1] are expert e's entries.  Ids outside
// [0, E) and entry ranges outside [0, T*k) are left out.  Returns the slot
// count (in every lane).
__device__ __forceinline__ int plan_compact(const PlanIn &pi, const int32_t *active, const int32_t *offsets,
                                            const PlanTabs &t) {
    const int lane = threadIdx.x & 31;
    const int S = pi.T * pi.k;
    int n_active = active[0];
    n_active = n_active < 0 ? 0 : (n_active > pi.max_active ? pi.max_active : n_active);
    int run = 0;
    for (int a0 = 0; a0 < n_active; a0 += 32) {
        const int a = a0 + lane;
        int e = -1, f = 0, cnt = 0;
        if (a < n_active) {
            e = active[1 + a];
            if (e >= 0 && e < pi.E) {
                f = offsets[e];
                cnt = offsets[e + 1] - f;
            }
        }
        const bool keep = a < n_active && e >= 0 && e < pi.E && cnt > 0 && cnt <= pi.max_count && f >= 0 &&
                          f + cnt <= S;
        const unsigned m = __ballot_sync(0xffffffffu, keep);
        if (keep) {
            const int pos = run + __popc(m & ((1u << lane) - 1u));
            int ti = 0;  // the shelf holding e (shelves cover [0, E) without overlap)
            for (int s = 0; s < pi.n_tiers; ++s)
                if (e >= pi.first[s] && e - pi.first[s] < pi.n[s]) ti = s;
            t.expert[pos] = e;
            t.bits[pos] = pi.bits[ti];
            t.tier[pos] = ti;
            t.jloc[pos] = e - pi.first[ti];
            t.first[pos] = f;
            t.count[pos] = cnt;
        }
        run += __popc(m);
    }
    if (pi.has_shared && pi.T <= pi.max_count) {
        if (lane == 0) {
            t.expert[run] = pi.E;
            t.bits[run] = pi.shared_bits;
            t.tier[run] = pi.n_tiers;
            t.jloc[run] = 0;
            t.first[run] = S;
            t.count[run] = pi.T;
        }
        ++run;
    }
    return run;
}

// One warp: per-slot tile cost and inclusive prefix sums for `phase`;
// returns the phase's total cost (in every lane).
__device__ __forceinline__ long long plan_costs(const PlanIn &pi, int ns, int phase, const PlanTabs &t) {
    const int lane = threadIdx.x & 31;
    const long long nt = tiles_per_slot(pi.H, pi.I, phase);
    long long base = 0;
    for (int a0 = 0; a0 < ns; a0 += 32) {
        const int a = a0 + lane;
        long long v = 0;
        if (a < ns) {
            const long long c = tile_cost(pi.H, pi.I, phase, phase_bits(t.bits[a], phase), t.count[a]);
            t.tc(phase)[a] = c;
            v = nt * c;
        }
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const long long u = __shfl_up_sync(0xffffffffu, v, o);
            if (lane >= o) v += u;
        }
        if (a < ns) t.pre(phase)[a] = base + v;
        base += __shfl_sync(0xffffffffu, v, 31);
    }
    return base;
}

// Global index (slot * nt + tile) of the first tile of `phase` whose start
// cost is >= x; ns * nt when there is none.
__device__ __forceinline__ int plan_first_tile(const PlanTabs &t, int ns, int nt, int phase, long long x) {
    const long long *pre = t.pre(phase);
    // the first slot whose tiles do not all start before x: the first with pre[a] > x
    int lo = 0, hi = ns;
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (pre[mid] > x) hi = mid;
        else lo = mid + 1;
    }
    if (lo == ns) return ns * nt;
    const long long tc = t.tc(phase)[lo];
    const long long off = pre[lo] - nt * tc;  // start cost of the slot's first tile
    // ceil((x - off) / tc) clamped to [0, nt], as a double quotient: every CTA
    // evaluates the same monotone function of x, so neighbouring CTAs agree on
    // the tile where one run ends and the next begins
    if (x <= off) return lo * nt;
    long long b = static_cast<long long>(ceil(static_cast<double>(x - off) / static_cast<double>(tc)));
    if (b > nt) b = nt;
    return lo * nt + static_cast<int>(b);
}

// floor(a * c / g) as a double quotient (deterministic and monotone in c).
__device__ __forceinline__ long long share_floor(long long a, int c, int g) {
    return static_cast<long long>(static_cast<double>(a) * c / static_cast<double>(g));
}

// CTA c's run of phase-`phase` tiles: [gs, ge) in global tile indices.
__device__ __forceinline__ int2 plan_cta_range(const PlanTabs &t, int ns, int nt, int phase, long long total, int c,
                                               int grid) {
    const long long lo = share_floor(total, c, grid), hi = share_floor(total, c + 1, grid);
    const int gs = plan_first_tile(t, ns, nt, phase, lo);
    const int ge = c + 1 == grid ? ns * nt : plan_first_tile(t, ns, nt, phase, hi);
    return make_int2(gs, ge);
}

}  // namespace moe

