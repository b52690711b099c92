// Parameters shared by the FFN kernels (GEMV and tcgen05 GEMM paths).
#pragma once
#include "common.cuh"

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
};

}  // namespace moe
