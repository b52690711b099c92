// Tiered expert FFN, tensor-core path (placeholder until the tcgen05 kernel lands).
#include "common.cuh"
#include "ffn.cuh"

cudaError_t moe_configure_ffn_gemm() { return cudaSuccess; }

size_t moe_ffn_gemm_workspace(const moe_layer_weights *, int, int) { return 0; }

cudaError_t moe_launch_ffn_gemm(const moe::FfnParams &, void *, size_t, cudaStream_t) {
    return cudaErrorNotSupported;
}
