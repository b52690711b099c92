// Parameters shared by the FFN kernels (GEMV and tcgen05 GEMM paths).
#pragma once
#include "common.cuh"
#include "plan.cuh"

namespace moe {

struct FfnParams {
    moe_layer_weights w;  // shelves and the shared expert (device pointers inside)
    int E, T, k;
    int has_shared;
    int max_active;       // CTA rows launched for routed experts: min(E, T*k)
    const uint16_t *x;    // bf16 [T][H]
    const int32_t *offsets, *sorted, *active;
    float *h;             // fp32 [T*k + T][I] (GEMV path)
    int *ctr;             // [max_active + 1] gate_up tiles done per slot (zeroed per call)
    int max_count;        // GEMV path: experts with more tokens are left to the GEMM path
    float *y_slots;       // fp32 [T*k][H]
    float *y_shared;      // fp32 [T][H]
    int32_t *status;
    PlanIn pi;            // the GEMV path's schedule inputs
    // Small batches of a whole layer: the FFN kernel routes the batch itself
    // (logits of its share of the experts, a grid barrier, then every CTA
    // ranks and groups the tokens); CTA 0 writes the routing outputs.
    struct Route {
        int on;
        const uint16_t *wr;  // bf16 [E][H]
        const float *bias;   // [E] or null
        float *logits;       // fp32 [T][E]
        int32_t *topk_idx;   // [T][k]
        float *topk_w;       // [T][k]
        int32_t *offsets, *sorted, *slot_pos, *active;  // the grouping, as moe_bucketize writes it
        int *gbar;           // grid barrier words (2 ints, zero on entry)
    } route;
    long long wait_limit;  // SM clock cycles after which a device-side wait gives up
    int skip_publish;      // test hook: slot whose gate_up completions are never published (-1: none)
};

}  // namespace moe
