// Bucketize: token -> expert scatter with warp ballots, match and prefix sums.
//
// [P1] "the four bugs, briefly": the expert-grouping helper assumes each
// expert appears at most once per word, and a duplicated "skip" silently
// dropped a slot.  Here every slot s = t*k + j with a valid id is listed once,
// under its expert, in ascending s (a stable counting sort); an id outside
// [0,E) is reported and left out, and never used as an address.
#include "common.cuh"

namespace moe {

constexpr int kBucketThreads = 1024;
constexpr int kBucketWarps = kBucketThreads / 32;

// Block-wide exclusive scan of one int per thread (1024 threads).
__device__ __forceinline__ int block_exclusive_scan(int v, int *warp_tot, int *total) {
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
        int w = warp_tot[lane];
        int wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += n;
        }
        warp_tot[lane] = wi - w;  // exclusive prefix of warp totals
        if (lane == 31) *total = wi;
    }
    __syncthreads();
    return warp_tot[warp] + incl - v;
}

// Single CTA.  Warp w owns the contiguous slot range [w*chunk, (w+1)*chunk) and
// cnt[w][e] counts its slots of expert e; an exclusive scan over (warp, expert)
// then gives each warp the first output position of each of its experts, and
// the second pass places slots in order, so the result is stable.
__global__ void __launch_bounds__(kBucketThreads)
bucketize_kernel(const int32_t *__restrict__ ids, int S, int E, int32_t *__restrict__ offsets,
                 int32_t *__restrict__ sorted_slot, int32_t *__restrict__ slot_pos,
                 int32_t *__restrict__ active, int32_t *__restrict__ status) {
    extern __shared__ int smem[];
    int *cnt = smem;                       // [kBucketWarps][E]
    __shared__ int warp_tot[32];
    __shared__ int total_slots, total_active;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int i = threadIdx.x; i < kBucketWarps * E; i += kBucketThreads) cnt[i] = 0;
    __syncthreads();

    const int chunk = (S + kBucketWarps - 1) / kBucketWarps;
    const int begin = min(S, warp * chunk), end = min(S, begin + chunk);
    int *my_cnt = cnt + warp * E;
    bool bad = false;
    for (int base = begin; base < end; base += 32) {
        const int s = base + lane;
        const bool valid = s < end;
        const int id = valid ? ids[s] : -1;
        const bool ok = valid && id >= 0 && id < E;
        bad |= valid && !ok;
        const unsigned okmask = __ballot_sync(0xffffffffu, ok);
        if (ok) {
            const unsigned peers = __match_any_sync(okmask, id);
            if (lane == __ffs(peers) - 1) my_cnt[id] += __popc(peers);
        }
        __syncwarp();
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) status_or(status, MOE_STATUS_BAD_EXPERT_ID);
    __syncthreads();

    // per expert: exclusive prefix over warps, and the expert's total
    int tot = 0;
    const int e = threadIdx.x;  // E <= 1024 == threads
    if (e < E) {
        for (int w = 0; w < kBucketWarps; ++w) {
            const int c = cnt[w * E + e];
            cnt[w * E + e] = tot;
            tot += c;
        }
    }
    const int excl = block_exclusive_scan(e < E ? tot : 0, warp_tot, &total_slots);
    if (e < E) {
        offsets[e] = excl;
        for (int w = 0; w < kBucketWarps; ++w) cnt[w * E + e] += excl;
    }
    const int aflag = (e < E && tot > 0) ? 1 : 0;
    const int apos = block_exclusive_scan(aflag, warp_tot, &total_active);
    if (aflag) active[1 + apos] = e;
    if (threadIdx.x == 0) {
        offsets[E] = total_slots;
        active[0] = total_active;
    }
    __syncthreads();

    // placement, in ascending slot order within each warp's range
    const unsigned lt = (1u << lane) - 1u;
    for (int base = begin; base < end; base += 32) {
        const int s = base + lane;
        const bool valid = s < end;
        const int id = valid ? ids[s] : -1;
        const bool ok = valid && id >= 0 && id < E;
        const unsigned okmask = __ballot_sync(0xffffffffu, ok);
        unsigned peers = 0;
        int p = -1;
        if (ok) {
            peers = __match_any_sync(okmask, id);
            p = my_cnt[id] + __popc(peers & lt);
            sorted_slot[p] = s;
        }
        if (valid) slot_pos[s] = p;
        __syncwarp();
        if (ok && lane == __ffs(peers) - 1) my_cnt[id] += __popc(peers);
        __syncwarp();
    }
}

}  // namespace moe

size_t moe_bucketize_smem(int E) { return static_cast<size_t>(moe::kBucketWarps) * E * sizeof(int); }

cudaError_t moe_configure_bucketize() {
    return cudaFuncSetAttribute(moe::bucketize_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(moe_bucketize_smem(MOE_MAX_EXPERTS)));
}

cudaError_t moe_launch_bucketize(const int32_t *ids, int S, int E, int32_t *offsets, int32_t *sorted,
                                 int32_t *pos, int32_t *active, int32_t *status, cudaStream_t s) {
    moe::bucketize_kernel<<<1, moe::kBucketThreads, moe_bucketize_smem(E), s>>>(
        ids, S, E, offsets, sorted, pos, active, status);
    return cudaGetLastError();
}
