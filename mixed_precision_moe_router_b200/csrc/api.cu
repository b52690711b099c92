// C ABI entry points: argument validation, workspace carving and launches.
// Every check here runs on the host before anything is enqueued; nothing here
// allocates, frees or synchronises.
#include <atomic>
#include <cstdarg>
#include <cstring>
#include <cstdio>
#include <mutex>
#include <string>

#include "common.cuh"
#include "ffn.cuh"

// launchers defined next to their kernels
cudaError_t moe_launch_quantize(const float *, int64_t, int, int, uint8_t *, uint16_t *, cudaStream_t);
cudaError_t moe_launch_dequantize(const uint8_t *, const uint16_t *, int64_t, int, int, float *, uint16_t *,
                                  cudaStream_t);
cudaError_t moe_configure_router();
cudaError_t moe_launch_router_logits(const uint16_t *, const uint16_t *, const float *, int, int, int, float *,
                                     cudaStream_t);
cudaError_t moe_launch_topk(const float *, int, int, int, int32_t *, float *, cudaStream_t);
cudaError_t moe_configure_route_small();
bool moe_route_small_supported(int T, int H, int E, int k);
cudaError_t moe_launch_route_small(const uint16_t *, const uint16_t *, const float *, int, int, int, int, float *,
                                   int32_t *, float *, int32_t *, int32_t *, int32_t *, int32_t *, int32_t *, int *,
                                   int *, int, cudaStream_t);
bool moe_router_gemm_supported(int T, int H, int E);
cudaError_t moe_launch_router_gemm(const uint16_t *, const uint16_t *, const float *, int, int, int, float *,
                                   cudaStream_t);
cudaError_t moe_configure_bucketize();
cudaError_t moe_launch_bucketize(const int32_t *, int, int, int32_t *, int32_t *, int32_t *, int32_t *, int32_t *,
                                 cudaStream_t);
cudaError_t moe_configure_ffn_stream();
cudaError_t moe_launch_ffn_stream(const moe::FfnParams &, cudaStream_t);
bool moe_ffn_stream_supported(int H, int I);
bool moe_ffn_stream_fits(int H, int I, int T, int k, int E, int max_slots);
cudaError_t moe_configure_ffn_gemm();
cudaError_t moe_launch_ffn_gemm(const moe::FfnParams &, void *ws, size_t ws_bytes, cudaStream_t, int min_count);
bool moe_ffn_gemm_supported(int H, int I);
size_t moe_ffn_gemm_workspace(const moe_layer_weights *, int T, int k);
cudaError_t moe_launch_combine(const float *, const float *, const float *, int, int, int, const uint16_t *,
                               uint16_t *, uint16_t *, uint16_t *, cudaStream_t);
cudaError_t moe_launch_rmsnorm(const uint16_t *, int, int, uint16_t *, cudaStream_t);
size_t moe_stack_layer_bytes();
cudaError_t moe_stack_encode_layer(const moe_layer_weights *, const uint16_t *, const float *, void *);
size_t moe_stack_smem(int H, int I, int T, int k, int E, int *ring_bytes);
cudaError_t moe_configure_stack();
cudaError_t moe_launch_stack(const void *, int, int, int, int, int, int, const uint16_t *, uint16_t *, uint16_t *,
                             uint16_t *, uint16_t *, float *, float *, float *, float *, int *, int *, int32_t *,
                             long long, int, cudaStream_t);

namespace {

thread_local std::string g_err;

// Knobs for tests of the failure paths (moe_debug_set); process-wide.
constexpr long long kDefaultWaitLimit = 2000000000LL;  // ~1 s of SM clock
std::atomic<long long> g_wait_limit{kDefaultWaitLimit};
std::atomic<int> g_skip_publish{-1};

int fail(int code, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_err = buf;
    return code;
}

int ok() {
    g_err.clear();
    return MOE_OK;
}

int cuda_fail(cudaError_t e, const char *what) {
    return fail(MOE_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Kernel attributes (dynamic shared memory limits) are set once per device.
constexpr int kMaxDevices = 64;
std::once_flag g_dev_once[kMaxDevices];
cudaError_t g_dev_err[kMaxDevices];

int ensure_configured() {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return fail(MOE_ERR_UNSUPPORTED, "device ordinal %d", dev);
    std::call_once(g_dev_once[dev], [dev]() {
        cudaError_t r = moe_configure_router();
        if (r == cudaSuccess) r = moe_configure_route_small();
        if (r == cudaSuccess) r = moe_configure_bucketize();
        if (r == cudaSuccess) r = moe_configure_ffn_stream();
        if (r == cudaSuccess) r = moe_configure_ffn_gemm();
        if (r == cudaSuccess) r = moe_configure_stack();
        g_dev_err[dev] = r;
    });
    if (g_dev_err[dev] != cudaSuccess) return cuda_fail(g_dev_err[dev], "kernel configuration");
    return MOE_OK;
}

bool valid_bits(int b) { return b == 8 || b == 4 || b == 3 || b == MOE_FP4; }

size_t align_up(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

int check_tier(const moe_tier &t, const char *name, int idx) {
    if (!valid_bits(t.bits)) return fail(MOE_ERR_INVALID_ARG, "%s[%d].bits = %d (want 8, 4, 3 or MOE_FP4)", name, idx, t.bits);
    if (t.dn_bits != 0 && !valid_bits(t.dn_bits))
        return fail(MOE_ERR_INVALID_ARG, "%s[%d].dn_bits = %d (want 0, 8, 4, 3 or MOE_FP4)", name, idx, t.dn_bits);
    if (!t.gu_qs || !t.gu_scale || !t.dn_qs || !t.dn_scale)
        return fail(MOE_ERR_INVALID_ARG, "%s[%d] has a NULL table pointer", name, idx);
    if (!aligned16(t.gu_qs) || !aligned16(t.gu_scale) || !aligned16(t.dn_qs) || !aligned16(t.dn_scale))
        return fail(MOE_ERR_INVALID_ARG, "%s[%d] table pointer not 16-byte aligned", name, idx);
    return MOE_OK;
}

int check_weights(const moe_layer_weights *w) {
    if (!w) return fail(MOE_ERR_INVALID_ARG, "weights descriptor is NULL");
    if (w->H <= 0 || w->H % 128 != 0) return fail(MOE_ERR_INVALID_ARG, "H = %d must be a positive multiple of 128", w->H);
    if (w->I <= 0 || w->I % 128 != 0) return fail(MOE_ERR_INVALID_ARG, "I = %d must be a positive multiple of 128", w->I);
    if (w->H > 16384 || w->I > 16384) return fail(MOE_ERR_UNSUPPORTED, "H and I are limited to 16384");
    if (w->E < 1 || w->E > MOE_MAX_EXPERTS) return fail(MOE_ERR_INVALID_ARG, "E = %d outside [1, %d]", w->E, MOE_MAX_EXPERTS);
    if (w->n_tiers < 1 || w->n_tiers > MOE_MAX_TIERS)
        return fail(MOE_ERR_INVALID_ARG, "n_tiers = %d outside [1, %d]", w->n_tiers, MOE_MAX_TIERS);
    long covered = 0;
    for (int i = 0; i < w->n_tiers; ++i) {
        const moe_tier &t = w->tiers[i];
        if (t.n_experts < 1) return fail(MOE_ERR_INVALID_ARG, "tiers[%d].n_experts = %d", i, t.n_experts);
        if (t.first_expert < 0 || t.first_expert + t.n_experts > w->E)
            return fail(MOE_ERR_INVALID_ARG, "tiers[%d] id range [%d, %d) outside [0, %d)", i, t.first_expert,
                        t.first_expert + t.n_experts, w->E);
        for (int j = 0; j < i; ++j) {
            const moe_tier &o = w->tiers[j];
            if (t.first_expert < o.first_expert + o.n_experts && o.first_expert < t.first_expert + t.n_experts)
                return fail(MOE_ERR_INVALID_ARG, "tiers[%d] and tiers[%d] overlap", j, i);
        }
        covered += t.n_experts;
        int r = check_tier(t, "tiers", i);
        if (r) return r;
    }
    if (covered != w->E) return fail(MOE_ERR_INVALID_ARG, "tiers cover %ld of %d expert ids", covered, w->E);
    if (w->shared.n_experts != 0 && w->shared.n_experts != 1)
        return fail(MOE_ERR_INVALID_ARG, "shared.n_experts = %d (want 0 or 1)", w->shared.n_experts);
    if (w->shared.n_experts == 1) {
        int r = check_tier(w->shared, "shared", 0);
        if (r) return r;
    }
    return MOE_OK;
}

int check_k(int T, int E, int k) {
    if (T < 0) return fail(MOE_ERR_INVALID_ARG, "T = %d", T);
    if (E < 1 || E > MOE_MAX_EXPERTS) return fail(MOE_ERR_INVALID_ARG, "E = %d outside [1, %d]", E, MOE_MAX_EXPERTS);
    if (k < 1 || k > E || k > MOE_MAX_TOPK) return fail(MOE_ERR_INVALID_ARG, "k = %d outside [1, min(E, %d)]", k, MOE_MAX_TOPK);
    if (static_cast<int64_t>(T) * k > (1 << 24)) return fail(MOE_ERR_UNSUPPORTED, "T*k = %lld exceeds 2^24", (long long)T * k);
    return MOE_OK;
}

moe::FfnParams make_params(const moe_layer_weights *w, const uint16_t *x, int T, int k, const int32_t *offsets,
                           const int32_t *sorted, const int32_t *active, float *y_slots, float *y_shared,
                           float *h, int32_t *status) {
    moe::FfnParams p;
    p.w = *w;
    p.E = w->E;
    p.T = T;
    p.k = k;
    p.has_shared = w->shared.n_experts == 1;
    const long ma = static_cast<long>(T) * k;
    p.max_active = static_cast<int>(ma < w->E ? ma : w->E);
    p.x = x;
    p.offsets = offsets;
    p.sorted = sorted;
    p.active = active;
    p.h = h;
    p.ctr = nullptr;
    p.max_count = 0x7fffffff;
    p.y_slots = y_slots;
    p.y_shared = y_shared;
    p.status = status;
    moe::PlanIn &pi = p.pi;
    std::memset(&pi, 0, sizeof(pi));
    pi.E = w->E;
    pi.T = T;
    pi.k = k;
    pi.H = w->H;
    pi.I = w->I;
    pi.n_tiers = w->n_tiers;
    pi.has_shared = p.has_shared;
    pi.shared_bits = moe::tier_formats(w->shared);
    pi.max_count = p.max_count;
    pi.max_active = p.max_active;
    for (int t = 0; t < w->n_tiers; ++t) {
        pi.first[t] = w->tiers[t].first_expert;
        pi.n[t] = w->tiers[t].n_experts;
        pi.bits[t] = moe::tier_formats(w->tiers[t]);
    }
    std::memset(&p.route, 0, sizeof(p.route));
    p.wait_limit = g_wait_limit.load();
    p.skip_publish = g_skip_publish.load();
    return p;
}

// The streaming path's token limit for AUTO mode also enters its schedule.
void set_max_count(moe::FfnParams &p, int max_count) {
    p.max_count = max_count;
    p.pi.max_count = max_count;
}

// The streaming path's per-slot counters, followed by the two grid barrier
// words of a batch that the FFN kernel routes itself.
size_t ffn_ctr_bytes(const moe_layer_weights *w, int T, int k) {
    const long ma = static_cast<long>(T) * k;
    return align_up((static_cast<size_t>(ma < w->E ? ma : w->E) + 1 + 2) * sizeof(int));
}

// Token count from which an expert goes through the tensor-core GEMM in
// MOE_FFN_AUTO mode (below it the streaming GEMV reads the weights once anyway
// and wastes no tensor-core columns).
constexpr int kGemmMinTokens = 8;

// Batches the FFN kernel routes itself inside moe_layer_forward: at most as
// many tokens as its logits pass stages, and one grouping slot per thread.
constexpr int kFusedRouteMaxTokens = 16;
constexpr int kFusedRouteMaxSlots = 512;

bool uses_gemv(int mode) { return mode != MOE_FFN_GEMM; }
bool uses_gemm(int mode, int T) { return mode == MOE_FFN_GEMM || (mode == MOE_FFN_AUTO && T >= kGemmMinTokens); }

size_t gemv_ws_bytes(const moe_layer_weights *w, int T, int k) {
    const size_t rows = static_cast<size_t>(T) * k + static_cast<size_t>(T);
    return align_up(rows * w->I * sizeof(float)) + ffn_ctr_bytes(w, T, k);
}

size_t ffn_ws_bytes(const moe_layer_weights *w, int T, int k, int mode) {
    const size_t gemv = uses_gemv(mode) ? gemv_ws_bytes(w, T, k) : 0;
    const size_t gemm = uses_gemm(mode, T) ? align_up(moe_ffn_gemm_workspace(w, T, k)) : 0;
    return gemv + gemm + 256;
}

}  // namespace

extern "C" {

const char *moe_last_error(void) { return g_err.c_str(); }

const char *moe_version(void) { return "moe_tiered 0.1 (sm_100a)"; }

size_t moe_packed_row_bytes(int32_t K, int32_t bits) {
    if (K <= 0 || K % 64 != 0 || !valid_bits(bits)) return 0;
    return static_cast<size_t>(K) * moe::storage_bits(bits) / 8;
}

int moe_quantize(const float *src, int64_t rows, int32_t K, int32_t bits, uint8_t *qs, uint16_t *scale,
                 moe_stream_t stream) {
    if (!valid_bits(bits)) return fail(MOE_ERR_INVALID_ARG, "bits = %d (want 8, 4, 3 or MOE_FP4)", bits);
    if (K <= 0 || K % 64 != 0) return fail(MOE_ERR_INVALID_ARG, "K = %d must be a positive multiple of 64", K);
    if (rows < 0) return fail(MOE_ERR_INVALID_ARG, "rows = %lld", (long long)rows);
    if (rows == 0) return ok();
    if (!src || !qs || !scale) return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
    if (!aligned16(src) || !aligned16(qs) || !aligned16(scale)) return fail(MOE_ERR_INVALID_ARG, "pointer not 16-byte aligned");
    int r = ensure_configured();
    if (r) return r;
    cudaError_t e = moe_launch_quantize(src, rows, K, bits, qs, scale, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? ok() : cuda_fail(e, "quantize launch");
}

int moe_dequantize(const uint8_t *qs, const uint16_t *scale, int64_t rows, int32_t K, int32_t bits, float *out_f32,
                   uint16_t *out_f16, moe_stream_t stream) {
    if (!valid_bits(bits)) return fail(MOE_ERR_INVALID_ARG, "bits = %d (want 8, 4, 3 or MOE_FP4)", bits);
    if (K <= 0 || K % 64 != 0) return fail(MOE_ERR_INVALID_ARG, "K = %d must be a positive multiple of 64", K);
    if (rows < 0) return fail(MOE_ERR_INVALID_ARG, "rows = %lld", (long long)rows);
    if (!out_f32 && !out_f16) return fail(MOE_ERR_INVALID_ARG, "both outputs are NULL");
    if (rows == 0) return ok();
    if (!qs || !scale) return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
    int r = ensure_configured();
    if (r) return r;
    cudaError_t e = moe_launch_dequantize(qs, scale, rows, K, bits, out_f32, out_f16,
                                          reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? ok() : cuda_fail(e, "dequantize launch");
}

size_t moe_router_workspace_size(int32_t T, int32_t H, int32_t E, int32_t k) {
    (void)H;
    (void)k;
    if (T <= 0 || E <= 0) return 0;
    return align_up(static_cast<size_t>(T) * E * sizeof(float));
}

int moe_router_topk(const uint16_t *x, const uint16_t *w_router, const float *bias, int32_t T, int32_t H, int32_t E,
                    int32_t k, float *logits, int32_t *topk_idx, float *topk_w, void *workspace,
                    size_t workspace_bytes, moe_stream_t stream) {
    int r = check_k(T, E, k);
    if (r) return r;
    if (H <= 0 || H % 64 != 0 || H > 16384) return fail(MOE_ERR_INVALID_ARG, "H = %d must be a multiple of 64 in (0, 16384]", H);
    if (T == 0) return ok();
    if (!x || !w_router || !topk_idx || !topk_w) return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
    if (!aligned16(x) || !aligned16(w_router)) return fail(MOE_ERR_INVALID_ARG, "x / w_router not 16-byte aligned");
    float *lg = logits;
    if (!lg) {
        if (!workspace || workspace_bytes < moe_router_workspace_size(T, H, E, k))
            return fail(MOE_ERR_WORKSPACE, "router workspace needs %zu bytes", moe_router_workspace_size(T, H, E, k));
        lg = static_cast<float *>(workspace);
    }
    r = ensure_configured();
    if (r) return r;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // prefill-sized batches: the logits are a dense bf16 GEMM on the tensor cores
    cudaError_t e = moe_router_gemm_supported(T, H, E) ? moe_launch_router_gemm(x, w_router, bias, T, H, E, lg, s)
                                                       : moe_launch_router_logits(x, w_router, bias, T, H, E, lg, s);
    if (e == cudaSuccess) e = moe_launch_topk(lg, T, E, k, topk_idx, topk_w, s);
    return e == cudaSuccess ? ok() : cuda_fail(e, "router launch");
}

int moe_topk_softmax(const float *logits, int32_t T, int32_t E, int32_t k, int32_t *topk_idx, float *topk_w,
                     moe_stream_t stream) {
    int r = check_k(T, E, k);
    if (r) return r;
    if (T == 0) return ok();
    if (!logits || !topk_idx || !topk_w) return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
    r = ensure_configured();
    if (r) return r;
    cudaError_t e = moe_launch_topk(logits, T, E, k, topk_idx, topk_w, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? ok() : cuda_fail(e, "top-k launch");
}

int moe_bucketize(const int32_t *topk_idx, int32_t T, int32_t k, int32_t E, int32_t *expert_offsets,
                  int32_t *sorted_slot, int32_t *slot_pos, int32_t *active, int32_t *status, moe_stream_t stream) {
    int r = check_k(T, E, k);
    if (r) return r;
    if (!expert_offsets || !active) return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
    if (T > 0 && (!topk_idx || !sorted_slot || !slot_pos)) return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
    r = ensure_configured();
    if (r) return r;
    cudaError_t e = moe_launch_bucketize(topk_idx, T * k, E, expert_offsets, sorted_slot, slot_pos, active, status,
                                         reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? ok() : cuda_fail(e, "bucketize launch");
}

size_t moe_ffn_workspace_size(const moe_layer_weights *w, int32_t T, int32_t k, int32_t mode) {
    if (!w || T < 0 || k < 1) return 0;
    return ffn_ws_bytes(w, T, k, mode);
}

}  // extern "C"

namespace {

// The GEMV path's per-slot counters inside an FFN workspace (NULL when the
// mode does not use that path); *n = how many ints the kernel reads.
int *gemv_counters(const moe_layer_weights *w, int T, int k, int mode, void *workspace, int *n) {
    *n = 0;
    if (!uses_gemv(mode) || !workspace) return nullptr;
    const size_t hb = align_up((static_cast<size_t>(T) * k + T) * w->I * sizeof(float));
    const long ma = static_cast<long>(T) * k;
    *n = static_cast<int>(ma < w->E ? ma : w->E) + 1;
    return reinterpret_cast<int *>(static_cast<char *>(workspace) + hb);
}

// moe_expert_ffn_tiered; counters_clear: the GEMV counters are known to be
// zero already (cleared by an earlier kernel on the stream), so no memset.
int expert_ffn(const moe_layer_weights *w, const uint16_t *x, int32_t T, int32_t k, const int32_t *expert_offsets,
               const int32_t *sorted_slot, const int32_t *active, float *y_slots, float *y_shared, void *workspace,
               size_t workspace_bytes, int32_t mode, int32_t *status, moe_stream_t stream, bool counters_clear,
               const moe::FfnParams::Route *route = nullptr) {
    int r = check_weights(w);
    if (r) return r;
    r = check_k(T, w->E, k);
    if (r) return r;
    if (mode != MOE_FFN_AUTO && mode != MOE_FFN_GEMV && mode != MOE_FFN_GEMM)
        return fail(MOE_ERR_INVALID_ARG, "mode = %d", mode);
    if (T == 0) return ok();
    if (!x || !expert_offsets || !sorted_slot || !active || !y_slots)
        return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
    const bool has_shared = w->shared.n_experts == 1;
    if (has_shared != (y_shared != nullptr))
        return fail(MOE_ERR_INVALID_ARG, "y_shared must be given iff the layer has a shared expert");
    if (!aligned16(x) || !aligned16(y_slots) || (y_shared && !aligned16(y_shared)))
        return fail(MOE_ERR_INVALID_ARG, "x / y pointers not 16-byte aligned");
    const size_t need = ffn_ws_bytes(w, T, k, mode);
    if (!workspace || workspace_bytes < need) return fail(MOE_ERR_WORKSPACE, "ffn workspace needs %zu bytes", need);
    r = ensure_configured();
    if (r) return r;
    if (uses_gemv(mode) && !moe_ffn_stream_supported(w->H, w->I))
        return fail(MOE_ERR_UNSUPPORTED, "GEMV path supports H, I <= 2048");
    if (uses_gemv(mode)) {
        const long ma = static_cast<long>(T) * k;
        const int max_slots = static_cast<int>(ma < w->E ? ma : w->E) + 1;
        if (!moe_ffn_stream_fits(w->H, w->I, T, k, w->E, max_slots))
            return fail(MOE_ERR_UNSUPPORTED, "GEMV path: shared memory for T = %d, k = %d leaves no room for a tile",
                        T, k);
    }
    if (uses_gemm(mode, T) && !moe_ffn_gemm_supported(w->H, w->I))
        return fail(MOE_ERR_UNSUPPORTED, "GEMM path needs H %% 128 == 0 and I %% 64 == 0");
    char *ws = static_cast<char *>(workspace);
    float *h = reinterpret_cast<float *>(ws);
    moe::FfnParams p = make_params(w, x, T, k, expert_offsets, sorted_slot, active, y_slots, y_shared, h, status);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaSuccess;
    const bool gemm = uses_gemm(mode, T);
    const int split = mode == MOE_FFN_GEMM ? 1 : kGemmMinTokens;  // GEMM takes experts with >= split tokens
    if (uses_gemv(mode)) {
        int n_ctr = 0;
        p.ctr = gemv_counters(w, T, k, mode, workspace, &n_ctr);
        set_max_count(p, gemm ? split - 1 : 0x7fffffff);
        if (route) {
            p.route = *route;
            p.route.gbar = p.ctr + n_ctr;
        }
        if (!counters_clear) e = cudaMemsetAsync(p.ctr, 0, ffn_ctr_bytes(w, T, k), s);
        if (e == cudaSuccess) e = moe_launch_ffn_stream(p, s);
    }
    if (e == cudaSuccess && gemm) {
        char *gws = ws + (uses_gemv(mode) ? gemv_ws_bytes(w, T, k) : 0);
        e = moe_launch_ffn_gemm(p, gws, 0, s, split);
    }
    return e == cudaSuccess ? ok() : cuda_fail(e, "ffn launch");
}

size_t route_ws_bytes(int T, int E) { return align_up(static_cast<size_t>(T) * E * sizeof(float)) + 256; }

// moe_route; clear/n_clear: ints the fused kernel zeroes on its way out (the
// next kernel's counters), or a memset when the batch takes the separate
// kernels.
int route(const uint16_t *x, const uint16_t *w_router, const float *bias, int32_t T, int32_t H, int32_t E, int32_t k,
          int32_t *topk_idx, float *topk_w, int32_t *expert_offsets, int32_t *sorted_slot, int32_t *slot_pos,
          int32_t *active, int32_t *status, void *workspace, size_t workspace_bytes, moe_stream_t stream, int *clear,
          int n_clear) {
    int r = check_k(T, E, k);
    if (r) return r;
    if (H <= 0 || H % 64 != 0 || H > 16384) return fail(MOE_ERR_INVALID_ARG, "H = %d must be a multiple of 64 in (0, 16384]", H);
    if (!expert_offsets || !active) return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
    if (T > 0 && (!x || !w_router || !topk_idx || !topk_w || !sorted_slot || !slot_pos))
        return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
    if (T > 0 && (!aligned16(x) || !aligned16(w_router))) return fail(MOE_ERR_INVALID_ARG, "x / w_router not 16-byte aligned");
    const size_t need = route_ws_bytes(T, E);
    if (!workspace || workspace_bytes < need) return fail(MOE_ERR_WORKSPACE, "route workspace needs %zu bytes", need);
    if (!aligned16(workspace)) return fail(MOE_ERR_INVALID_ARG, "workspace not 16-byte aligned");
    r = ensure_configured();
    if (r) return r;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    float *logits = static_cast<float *>(workspace);
    int *ticket = reinterpret_cast<int *>(static_cast<char *>(workspace) + need - 256);
    cudaError_t e = cudaSuccess;
    if (moe_route_small_supported(T, H, E, k)) {
        e = cudaMemsetAsync(ticket, 0, sizeof(int), s);
        if (e == cudaSuccess)
            e = moe_launch_route_small(x, w_router, bias, T, H, E, k, logits, topk_idx, topk_w, expert_offsets,
                                       sorted_slot, slot_pos, active, status, ticket, clear, n_clear, s);
        return e == cudaSuccess ? ok() : cuda_fail(e, "route launch");
    }
    r = moe_router_topk(x, w_router, bias, T, H, E, k, logits, topk_idx, topk_w, nullptr, 0, stream);
    if (r) return r;
    r = moe_bucketize(topk_idx, T, k, E, expert_offsets, sorted_slot, slot_pos, active, status, stream);
    if (r) return r;
    if (n_clear > 0) {
        e = cudaMemsetAsync(clear, 0, static_cast<size_t>(n_clear) * sizeof(int), s);
        if (e != cudaSuccess) return cuda_fail(e, "memset");
    }
    return ok();
}

}  // namespace

extern "C" {

int moe_expert_ffn_tiered(const moe_layer_weights *w, const uint16_t *x, int32_t T, int32_t k,
                          const int32_t *expert_offsets, const int32_t *sorted_slot, const int32_t *active,
                          float *y_slots, float *y_shared, void *workspace, size_t workspace_bytes, int32_t mode,
                          int32_t *status, moe_stream_t stream) {
    return expert_ffn(w, x, T, k, expert_offsets, sorted_slot, active, y_slots, y_shared, workspace, workspace_bytes,
                      mode, status, stream, false);
}

size_t moe_route_workspace_size(int32_t T, int32_t H, int32_t E, int32_t k) {
    (void)H;
    (void)k;
    if (T < 0 || E <= 0) return 0;
    return route_ws_bytes(T, E);
}

int moe_route(const uint16_t *x, const uint16_t *w_router, const float *bias, int32_t T, int32_t H, int32_t E,
              int32_t k, int32_t *topk_idx, float *topk_w, int32_t *expert_offsets, int32_t *sorted_slot,
              int32_t *slot_pos, int32_t *active, int32_t *status, void *workspace, size_t workspace_bytes,
              moe_stream_t stream) {
    return route(x, w_router, bias, T, H, E, k, topk_idx, topk_w, expert_offsets, sorted_slot, slot_pos, active,
                 status, workspace, workspace_bytes, stream, nullptr, 0);
}

int moe_combine(const float *y_slots, const float *y_shared, const float *topk_w, int32_t T, int32_t k, int32_t H,
                const uint16_t *residual, uint16_t *out, uint16_t *x_next, uint16_t *x_next_norm,
                moe_stream_t stream) {
    if (T < 0 || k < 1 || k > MOE_MAX_TOPK) return fail(MOE_ERR_INVALID_ARG, "T = %d, k = %d", T, k);
    if (H <= 0 || H % 4 != 0) return fail(MOE_ERR_INVALID_ARG, "H = %d must be a positive multiple of 4", H);
    if (T == 0) return ok();
    if (!y_slots || !topk_w) return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
    if (!out && !residual) return fail(MOE_ERR_INVALID_ARG, "out is NULL and there is no residual");
    if (residual && !x_next) return fail(MOE_ERR_INVALID_ARG, "x_next is required with a residual");
    if (!aligned16(y_slots) || (y_shared && !aligned16(y_shared)))
        return fail(MOE_ERR_INVALID_ARG, "y pointers not 16-byte aligned");
    if (x_next_norm && !residual) return fail(MOE_ERR_INVALID_ARG, "x_next_norm needs a residual");
    cudaError_t e = moe_launch_combine(y_slots, y_shared, topk_w, T, k, H, residual, out, x_next, x_next_norm,
                                       reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? ok() : cuda_fail(e, "combine launch");
}

int moe_rmsnorm(const uint16_t *x, int32_t T, int32_t H, uint16_t *n, moe_stream_t stream) {
    if (T < 0) return fail(MOE_ERR_INVALID_ARG, "T = %d", T);
    if (H <= 0 || H % 4 != 0) return fail(MOE_ERR_INVALID_ARG, "H = %d must be a positive multiple of 4", H);
    if (T == 0) return ok();
    if (!x || !n) return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
    if ((reinterpret_cast<uintptr_t>(x) & 7u) || (reinterpret_cast<uintptr_t>(n) & 7u))
        return fail(MOE_ERR_INVALID_ARG, "x / n not 8-byte aligned");
    cudaError_t e = moe_launch_rmsnorm(x, T, H, n, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? ok() : cuda_fail(e, "rmsnorm launch");
}

namespace {
struct LayerWs {
    void *route_ws;  // logits and the fused router's ticket
    size_t route_bytes;
    int32_t *idx;
    float *tw;
    int32_t *offsets, *sorted, *pos, *active;
    float *y_slots, *y_shared;
    void *ffn_ws;
    size_t ffn_bytes;
    size_t total;
};

LayerWs carve(const moe_layer_weights *w, int T, int k, int mode, char *base) {
    LayerWs L{};
    size_t off = 0;
    auto take = [&](size_t bytes) {
        char *p = base ? base + off : nullptr;
        off += align_up(bytes);
        return p;
    };
    const size_t S = static_cast<size_t>(T) * k;
    L.route_bytes = route_ws_bytes(T, w->E);
    L.route_ws = take(L.route_bytes);
    L.idx = reinterpret_cast<int32_t *>(take(S * sizeof(int32_t)));
    L.tw = reinterpret_cast<float *>(take(S * sizeof(float)));
    L.offsets = reinterpret_cast<int32_t *>(take((w->E + 1) * sizeof(int32_t)));
    L.sorted = reinterpret_cast<int32_t *>(take(S * sizeof(int32_t)));
    L.pos = reinterpret_cast<int32_t *>(take(S * sizeof(int32_t)));
    L.active = reinterpret_cast<int32_t *>(take((w->E + 1) * sizeof(int32_t)));
    L.y_slots = reinterpret_cast<float *>(take(S * w->H * sizeof(float)));
    L.y_shared = reinterpret_cast<float *>(take(static_cast<size_t>(T) * w->H * sizeof(float)));
    L.ffn_bytes = ffn_ws_bytes(w, T, k, mode);
    L.ffn_ws = take(L.ffn_bytes);
    L.total = off;
    return L;
}
}  // namespace

size_t moe_layer_workspace_size(const moe_layer_weights *w, int32_t T, int32_t k, int32_t mode) {
    if (!w || T < 0 || k < 1 || w->E < 1) return 0;
    return carve(w, T, k, mode, nullptr).total;
}

int moe_layer_forward(const moe_layer_weights *w, const uint16_t *w_router, const float *bias, const uint16_t *x,
                      int32_t T, int32_t k, const uint16_t *residual, uint16_t *out, uint16_t *x_next,
                      uint16_t *x_next_norm, void *workspace, size_t workspace_bytes, int32_t mode, int32_t *status,
                      moe_stream_t stream) {
    int r = check_weights(w);
    if (r) return r;
    r = check_k(T, w->E, k);
    if (r) return r;
    if (T == 0) return ok();
    const size_t need = moe_layer_workspace_size(w, T, k, mode);
    if (!workspace || workspace_bytes < need) return fail(MOE_ERR_WORKSPACE, "layer workspace needs %zu bytes", need);
    if (!aligned16(workspace)) return fail(MOE_ERR_INVALID_ARG, "workspace not 16-byte aligned");
    LayerWs L = carve(w, T, k, mode, static_cast<char *>(workspace));
    // A small batch on the streaming path: the FFN kernel routes it itself
    // (no routing kernel), after one memset of its counters.
    if (uses_gemv(mode) && T <= kFusedRouteMaxTokens && static_cast<long>(T) * k <= kFusedRouteMaxSlots &&
        moe_ffn_stream_supported(w->H, w->I)) {
        if (!w_router || !x) return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
        if (!aligned16(x) || !aligned16(w_router)) return fail(MOE_ERR_INVALID_ARG, "x / w_router not 16-byte aligned");
        moe::FfnParams::Route rt;
        std::memset(&rt, 0, sizeof(rt));
        rt.on = 1;
        rt.wr = w_router;
        rt.bias = bias;
        rt.logits = static_cast<float *>(L.route_ws);
        rt.topk_idx = L.idx;
        rt.topk_w = L.tw;
        rt.offsets = L.offsets;
        rt.sorted = L.sorted;
        rt.slot_pos = L.pos;
        rt.active = L.active;
        r = expert_ffn(w, x, T, k, L.offsets, L.sorted, L.active, L.y_slots,
                       w->shared.n_experts == 1 ? L.y_shared : nullptr, L.ffn_ws, L.ffn_bytes, mode, status, stream,
                       false, &rt);
        if (r) return r;
        return moe_combine(L.y_slots, w->shared.n_experts == 1 ? L.y_shared : nullptr, L.tw, T, k, w->H, residual,
                           out, x_next, x_next_norm, stream);
    }
    // the routing kernel also zeroes the FFN's GEMV counters on its way out
    int n_ctr = 0;
    int *ctr = gemv_counters(w, T, k, mode, L.ffn_ws, &n_ctr);
    r = route(x, w_router, bias, T, w->H, w->E, k, L.idx, L.tw, L.offsets, L.sorted, L.pos, L.active, status,
              L.route_ws, L.route_bytes, stream, ctr, n_ctr);
    if (r) return r;
    r = expert_ffn(w, x, T, k, L.offsets, L.sorted, L.active, L.y_slots, w->shared.n_experts == 1 ? L.y_shared : nullptr,
                   L.ffn_ws, L.ffn_bytes, mode, status, stream, true);
    if (r) return r;
    return moe_combine(L.y_slots, w->shared.n_experts == 1 ? L.y_shared : nullptr, L.tw, T, k, w->H, residual, out,
                       x_next, x_next_norm, stream);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// moe_expert_ffn_tiered_static: the streaming FFN without a caller workspace,
// for hosts that cannot allocate device memory in their decode loop (no
// allocator of their own, or HBM fully reserved up front; cudaFree would also
// wait for the whole device).  Its scratch is the array below, which each GPU
// that loads the library holds until exit; all calls on a device share it.
// ---------------------------------------------------------------------------

static __device__ __align__(256) unsigned char moe_static_scratch[MOE_STATIC_SCRATCH_BYTES];

namespace {

std::atomic<void *> g_scratch_ptr[kMaxDevices];
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device.  Only a
// successful lookup is kept: a failed one (say under stream capture, or with
// an error pending) is reported and tried again by the next call.
int static_scratch(char **ptr) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return fail(MOE_ERR_UNSUPPORTED, "device ordinal %d", dev);
    void *p = g_scratch_ptr[dev].load(std::memory_order_acquire);
    if (!p) {
        std::lock_guard<std::mutex> lock(g_scratch_mu);
        p = g_scratch_ptr[dev].load(std::memory_order_relaxed);
        if (!p) {
            const cudaError_t r = cudaGetSymbolAddress(&p, moe_static_scratch);
            if (r != cudaSuccess || !p) {
                cudaGetLastError();
                return cuda_fail(r != cudaSuccess ? r : cudaErrorInvalidSymbol, "cudaGetSymbolAddress(scratch)");
            }
            g_scratch_ptr[dev].store(p, std::memory_order_release);
        }
    }
    *ptr = static_cast<char *>(p);
    return MOE_OK;
}

}  // namespace

extern "C" int moe_expert_ffn_tiered_static(const moe_layer_weights *w, const uint16_t *x, int32_t T, int32_t k,
                                            const int32_t *expert_offsets, const int32_t *sorted_slot,
                                            const int32_t *active, float *y_slots, float *y_shared,
                                            int32_t *status, moe_stream_t stream) {
    int r = check_weights(w);
    if (r) return r;
    r = check_k(T, w->E, k);
    if (r) return r;
    if (T == 0) return ok();
    if (!x || !expert_offsets || !sorted_slot || !active || !y_slots)
        return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
    const bool has_shared = w->shared.n_experts == 1;
    if (has_shared != (y_shared != nullptr))
        return fail(MOE_ERR_INVALID_ARG, "y_shared must be given iff the layer has a shared expert");
    if (!aligned16(x) || !aligned16(y_slots) || (y_shared && !aligned16(y_shared)))
        return fail(MOE_ERR_INVALID_ARG, "x / y pointers not 16-byte aligned");
    const size_t need = gemv_ws_bytes(w, T, k);
    if (need > static_cast<size_t>(MOE_STATIC_SCRATCH_BYTES))
        return fail(MOE_ERR_UNSUPPORTED,
                    "T = %d, k = %d, I = %d needs %zu bytes of scratch; the static array holds %d "
                    "(use moe_expert_ffn_tiered with a workspace)",
                    T, k, w->I, need, MOE_STATIC_SCRATCH_BYTES);
    r = ensure_configured();
    if (r) return r;
    if (!moe_ffn_stream_supported(w->H, w->I)) return fail(MOE_ERR_UNSUPPORTED, "GEMV path supports H, I <= 2048");
    {
        const long ma = static_cast<long>(T) * k;
        const int max_slots = static_cast<int>(ma < w->E ? ma : w->E) + 1;
        if (!moe_ffn_stream_fits(w->H, w->I, T, k, w->E, max_slots))
            return fail(MOE_ERR_UNSUPPORTED, "GEMV path: shared memory for T = %d, k = %d leaves no room for a tile",
                        T, k);
    }
    char *ws = nullptr;
    r = static_scratch(&ws);
    if (r) return r;
    moe::FfnParams p = make_params(w, x, T, k, expert_offsets, sorted_slot, active, y_slots, y_shared,
                                   reinterpret_cast<float *>(ws), status);
    // counters follow the intermediates, as in the workspace layout; they must
    // start at zero and the previous call left its final counts there
    const size_t hb = align_up((static_cast<size_t>(T) * k + T) * w->I * sizeof(float));
    p.ctr = reinterpret_cast<int *>(ws + hb);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemsetAsync(p.ctr, 0, ffn_ctr_bytes(w, T, k), s);
    if (e == cudaSuccess) e = moe_launch_ffn_stream(p, s);
    return e == cudaSuccess ? ok() : cuda_fail(e, "ffn launch");
}

// ---------------------------------------------------------------------------
// A stack of decode layers in one persistent launch
// ---------------------------------------------------------------------------

namespace {

constexpr int kStackMaxTokens = 8;

struct StackWs {
    float *logits, *h, *y_slots, *y_shared;
    uint16_t *xbuf;
    int *ctr;  // per-slot counts, then the two grid barrier words
    size_t ctr_bytes;
    size_t total;
};

StackWs carve_stack(int H, int I, int E, int T, int k, char *base) {
    StackWs L{};
    size_t off = 0;
    auto take = [&](size_t bytes) {
        char *p = base ? base + off : nullptr;
        off += align_up(bytes);
        return p;
    };
    const size_t S = static_cast<size_t>(T) * k;
    const long ma = static_cast<long>(S) < E ? static_cast<long>(S) : E;
    L.logits = reinterpret_cast<float *>(take(static_cast<size_t>(T) * E * sizeof(float)));
    L.h = reinterpret_cast<float *>(take((S + T) * I * sizeof(float)));
    L.y_slots = reinterpret_cast<float *>(take(S * H * sizeof(float)));
    L.y_shared = reinterpret_cast<float *>(take(static_cast<size_t>(T) * H * sizeof(float)));
    L.xbuf = reinterpret_cast<uint16_t *>(take(2 * static_cast<size_t>(T) * H * sizeof(uint16_t)));
    L.ctr_bytes = align_up((static_cast<size_t>(ma) + 1 + 2) * sizeof(int));
    L.ctr = reinterpret_cast<int *>(take(L.ctr_bytes));
    L.total = off;
    return L;
}

}  // namespace

extern "C" {

size_t moe_stack_desc_bytes(int32_t n_layers) {
    if (n_layers < 1) return 0;
    return static_cast<size_t>(n_layers) * moe_stack_layer_bytes();
}

int moe_stack_prepare(const moe_layer_weights *layers, const uint16_t *const *w_router, const float *const *bias,
                      int32_t n_layers, void *desc, size_t desc_bytes) {
    if (n_layers < 1) return fail(MOE_ERR_INVALID_ARG, "n_layers = %d", n_layers);
    if (!layers || !w_router) return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
    const size_t need = moe_stack_desc_bytes(n_layers);
    if (!desc || desc_bytes < need) return fail(MOE_ERR_WORKSPACE, "stack descriptor needs %zu bytes", need);
    if ((reinterpret_cast<uintptr_t>(desc) & 63u) != 0) return fail(MOE_ERR_INVALID_ARG, "descriptor not 64-byte aligned");
    for (int l = 0; l < n_layers; ++l) {
        int r = check_weights(&layers[l]);
        if (r) return fail(r, "layer %d: %s", l, g_err.c_str());
        if (layers[l].H != layers[0].H || layers[l].I != layers[0].I || layers[l].E != layers[0].E)
            return fail(MOE_ERR_INVALID_ARG, "layer %d: H, I and E must match layer 0", l);
        if (!w_router[l] || !aligned16(w_router[l])) return fail(MOE_ERR_INVALID_ARG, "layer %d: router NULL or misaligned", l);
    }
    if (!moe_ffn_stream_supported(layers[0].H, layers[0].I))
        return fail(MOE_ERR_UNSUPPORTED, "the streaming path supports H, I <= 2048");
    int r = ensure_configured();
    if (r) return r;
    const size_t lb = moe_stack_layer_bytes();
    std::string host(need, '\0');
    for (int l = 0; l < n_layers; ++l) {
        cudaError_t e = moe_stack_encode_layer(&layers[l], w_router[l], bias ? bias[l] : nullptr, &host[l * lb]);
        if (e != cudaSuccess) return cuda_fail(e, "tensor map encoding");
    }
    cudaError_t e = cudaMemcpy(desc, host.data(), need, cudaMemcpyHostToDevice);
    return e == cudaSuccess ? ok() : cuda_fail(e, "descriptor copy");
}

size_t moe_stack_workspace_size(int32_t H, int32_t I, int32_t E, int32_t T, int32_t k) {
    if (H <= 0 || I <= 0 || E <= 0 || T <= 0 || k <= 0) return 0;
    return carve_stack(H, I, E, T, k, nullptr).total;
}

int moe_stack_forward(const void *desc, int32_t n_layers, int32_t H, int32_t I, int32_t E, int32_t T, int32_t k,
                      const uint16_t *x_in, uint16_t *x_out, uint16_t *x_out_norm, uint16_t *x_layers,
                      void *workspace, size_t workspace_bytes, int32_t *status, moe_stream_t stream) {
    if (n_layers < 1) return fail(MOE_ERR_INVALID_ARG, "n_layers = %d", n_layers);
    int r = check_k(T, E, k);
    if (r) return r;
    if (T < 1 || T > kStackMaxTokens) return fail(MOE_ERR_UNSUPPORTED, "T = %d (the stack kernel takes 1..%d tokens)", T, kStackMaxTokens);
    if (H <= 0 || H % 128 != 0 || I <= 0 || I % 128 != 0) return fail(MOE_ERR_INVALID_ARG, "H = %d, I = %d", H, I);
    if (!moe_ffn_stream_supported(H, I)) return fail(MOE_ERR_UNSUPPORTED, "the streaming path supports H, I <= 2048");
    if (!desc || !x_in || !x_out) return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
    if (!aligned16(x_in) || !aligned16(x_out) || (x_out_norm && !aligned16(x_out_norm)) || (x_layers && !aligned16(x_layers)))
        return fail(MOE_ERR_INVALID_ARG, "stream pointers not 16-byte aligned");
    const size_t need = moe_stack_workspace_size(H, I, E, T, k);
    if (!workspace || workspace_bytes < need) return fail(MOE_ERR_WORKSPACE, "stack workspace needs %zu bytes", need);
    if (!aligned16(workspace)) return fail(MOE_ERR_INVALID_ARG, "workspace not 16-byte aligned");
    int ring = 0;
    moe_stack_smem(H, I, T, k, E, &ring);
    if (ring == 0) return fail(MOE_ERR_UNSUPPORTED, "shared memory for T = %d, k = %d leaves no room for a tile", T, k);
    r = ensure_configured();
    if (r) return r;
    StackWs L = carve_stack(H, I, E, T, k, static_cast<char *>(workspace));
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemsetAsync(L.ctr, 0, L.ctr_bytes, s);
    const long ma = static_cast<long>(T) * k < E ? static_cast<long>(T) * k : E;
    if (e == cudaSuccess)
        e = moe_launch_stack(desc, n_layers, T, k, H, I, E, x_in, x_out, x_out_norm, x_layers, L.xbuf, L.logits, L.h,
                             L.y_slots, L.y_shared, L.ctr, L.ctr + ma + 1, status, g_wait_limit.load(),
                             g_skip_publish.load(), s);
    return e == cudaSuccess ? ok() : cuda_fail(e, "stack launch");
}

int moe_debug_set_waits(int64_t wait_limit_cycles, int32_t skip_publish_slot) {
    g_wait_limit.store(wait_limit_cycles > 0 ? wait_limit_cycles : kDefaultWaitLimit);
    g_skip_publish.store(skip_publish_slot < 0 ? -1 : skip_publish_slot);
    return ok();
}

}  // extern "C"
