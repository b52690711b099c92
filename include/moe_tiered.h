/*
 * moe_tiered.h -- C ABI of the tiered mixed-precision MoE layer (B200, sm_100a).
 *
 * One routed mixture-of-experts FFN layer in which a single routing decision
 * drives several expert tables ("shelves") stored at different precisions:
 * popular experts in 8-bit blocks, rarer ones in 4-bit and 3-bit blocks.
 *
 * Sources, cited by page title and section:
 *   [P1] "I ran a 125B model on three RTX 3090s at 80 tokens/s by teaching
 *        llama.cpp which experts matter" (dev.to)
 *   [P2] "Running Qwen3.8-Flash-Next 125B on Three RTX 3090s at 80 Tokens per
 *        Second" (n1n.ai)
 *   [P3] "flashnext-2x3090" README (gitlite mirror)
 *   [P5] "Qwen3.8-Flash-Next hits 39 tok/s on a 24GB GPU, provided you bring
 *        96GB of system RAM" (deniz.in)
 *
 * Conventions shared by every call
 *   - Every pointer argument is a DEVICE pointer unless stated otherwise; the
 *     caller allocates and owns all of them.  The library never allocates,
 *     frees or synchronises: each call only enqueues kernels on `stream`
 *     (a cudaStream_t; NULL is the legacy default stream).
 *   - Tensors are dense, row-major, with the last index contiguous.  bf16 and
 *     fp16 values are passed as their uint16_t bit patterns.
 *   - Device pointers must be 16-byte aligned.
 *   - Expert ids are signed int32.  No call ever writes a "skip" sentinel as an
 *     expert id, and no id reaches an address computation before it has been
 *     range-checked ([P1] "the four bugs, briefly": a -1 "skip" promoted to
 *     unsigned read four billion rows past a buffer).
 *   - Return value: MOE_OK, or an error code after which nothing was enqueued;
 *     moe_last_error() then describes it (per host thread).  Errors found by a
 *     kernel (data-dependent) are OR-ed into an optional device status word as
 *     MOE_STATUS_* bits; the caller clears it and reads it when it wants.
 *   - Calls are asynchronous and contain no host synchronisation, so a
 *     sequence of them can be captured into a CUDA graph.
 */
#ifndef MOE_TIERED_H
#define MOE_TIERED_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *moe_stream_t; /* same type as cudaStream_t */

/* return codes */
#define MOE_OK 0
#define MOE_ERR_INVALID_ARG 1 /* a size, pointer, alignment or layout is invalid */
#define MOE_ERR_UNSUPPORTED 2 /* valid, but outside what the kernels implement */
#define MOE_ERR_WORKSPACE 3   /* workspace missing or smaller than required */
#define MOE_ERR_CUDA 4        /* a CUDA launch failed */

/* device status bits (OR-ed into the optional int32 status word) */
#define MOE_STATUS_BAD_EXPERT_ID 0x1 /* an id outside [0,E) was seen and skipped;
                                        outputs of that token are undefined */
#define MOE_STATUS_FP16_RANGE 0x2    /* the tensor-core path met an activation
                                        beyond the fp16 range (|v| > 65504) */
#define MOE_STATUS_TIMEOUT 0x4       /* a bounded device-side wait gave up */

#define MOE_BLOCK 32     /* weights per quantisation block (one fp16 scale) */
#define MOE_MAX_TIERS 4  /* shelves per layer */
#define MOE_MAX_TOPK 32
#define MOE_MAX_EXPERTS 1024
#define MOE_NORM_EPS 1e-6f /* epsilon of the residual-stream RMS norm */
#define MOE_FP4 5 /* `bits` of an FP4 (E2M1) shelf: 4-bit storage, see below */

/*
 * Packed shelf format ([P1] "step 4: three shelves, all on the GPU": each
 * shelf is one expert table at one precision; [P3] "Why the model fits at
 * all": a 4-bit code plus a 16-bit scale per 32 weights is 4.5 bits/weight).
 *
 * A weight matrix [rows][K] (K % 64 == 0) is stored as two arrays:
 *   qs    uint8  [rows][K*bits/8]   codes, row by row
 *   scale uint16 [rows][K/32]       fp16 scale d of each block of 32 weights
 * and dequantises to w = d * q (exact in fp32).  Per block of 32:
 *   d = fp16_rne(fp32(amax) / fp32(qmax)), qmax = 2^(bits-1) - 1,
 *   q = clamp(round_half_away(fp32(w) / fp32(d)), -qmax, qmax); d == 0 -> q = 0.
 * Codes within a row:
 *   bits 8: the int8 value q.
 *   bits 4: c = q + 8; weight 2m in the low nibble of byte m, 2m+1 in the high.
 *   bits 3: c = q + 4; a low plane of K/4 bytes (bits 0-1 of weight i at bit
 *           2*(i%4) of byte i/4) followed by a high plane of K/8 bytes (bit 2
 *           of weight i at bit i%8 of byte K/4 + i/8).
 *
 * FP4 shelf (bits = MOE_FP4; [P1] "step 4": MXFP4 for the rarest experts'
 * weights).  The OCP MX conversion with E2M1 elements and a power-of-two
 * block scale, stored in the layout above with 4-bit storage (K/2 code bytes
 * per row):
 *   X = 2^(floor(log2 amax) - 2), clamped to [2^-23, 2^16]; amax == 0 -> d = 0,
 *       every code 0;
 *   v = the E2M1 value (0, 0.5, 1, 1.5, 2, 3, 4, 6, signed) nearest to w / X,
 *       a tie to the one of even magnitude index, saturating at 6;
 *   c = 8 * sign + m, m the magnitude index 0..7 (a zero is stored as +0);
 *       weight 2m in the low nibble of byte m, 2m+1 in the high;
 *   d = X / 2 (exact in fp16), q = 2 * v in {0, +-1, +-2, +-3, +-4, +-6, +-8,
 *       +-12}, so that w = d * q as for the integer shelves.
 */
size_t moe_packed_row_bytes(int32_t K, int32_t bits); /* K*bits/8, K/2 for MOE_FP4;
                                                         0 for an invalid K or bits */

/*
 * One shelf: experts [first_expert, first_expert + n_experts), gate_up at
 * `bits` and down at `dn_bits` ([P1] "step 4": the down projections take a
 * ladder of their own, MXFP4 on the rarest shelf).  Per expert (expert j of
 * the shelf at index j), hidden H, intermediate I, b = bits, c = dn_bits:
 *   gu_qs    [n_experts][2*I][H*b/8]   gate rows 0..I-1, up rows I..2I-1
 *   gu_scale [n_experts][2*I][H/32]
 *   dn_qs    [n_experts][H][I*c/8]
 *   dn_scale [n_experts][H][I/32]
 * (in these sizes and in moe_quantize's, MOE_FP4 counts as 4 bits).
 */
typedef struct moe_tier {
    int32_t bits;          /* gate_up format: 8, 4, 3 or MOE_FP4 */
    int32_t first_expert;  /* first id of this shelf's contiguous id range */
    int32_t n_experts;     /* experts on the shelf (0 for an unused shared slot) */
    int32_t dn_bits;       /* down format: 8, 4, 3 or MOE_FP4; 0 = same as bits */
    const uint8_t *gu_qs;
    const uint16_t *gu_scale;
    const uint8_t *dn_qs;
    const uint16_t *dn_scale;
} moe_tier;

/*
 * A layer's expert weights ([P1] "step 4": experts are reordered hottest-first
 * into one table per precision).  The shelves must cover the ids [0, E)
 * exactly, without overlap.  `shared` is the always-on shared expert
 * ([P5] "What the model actually is": 10 routed plus 1 shared expert);
 * shared.n_experts is 1, or 0 for a layer without one; shared.first_expert
 * is ignored.  The descriptor itself is a HOST struct, read during the call.
 */
typedef struct moe_layer_weights {
    int32_t H;        /* hidden size, % 64 == 0 */
    int32_t I;        /* expert intermediate size, % 64 == 0 */
    int32_t E;        /* routed experts, 1..MOE_MAX_EXPERTS */
    int32_t n_tiers;  /* 1..MOE_MAX_TIERS */
    moe_tier tiers[MOE_MAX_TIERS];
    moe_tier shared;
} moe_layer_weights;

/* FFN execution path */
#define MOE_FFN_AUTO 0 /* per expert: GEMV below the token threshold, GEMM above */
#define MOE_FFN_GEMV 1 /* every expert through the streaming GEMV (mma.sync tiles) */
#define MOE_FFN_GEMM 2 /* every expert through the tcgen05 GEMM */

/* Description of the most recent error on the calling host thread. */
const char *moe_last_error(void);
const char *moe_version(void);

/*
 * moe_quantize: source fp32 rows -> packed shelf rows (format above).
 *   src   float  [rows][K]  (device)
 *   qs    uint8  [rows][K*bits/8], scale uint16 [rows][K/32]  (device, written)
 * The codes and scales are bit-identical to the definition above.
 */
int moe_quantize(const float *src, int64_t rows, int32_t K, int32_t bits,
                 uint8_t *qs, uint16_t *scale, moe_stream_t stream);

/*
 * moe_dequantize: packed rows -> w = d*q as fp32 (exact) and/or as the fp16
 * value fp16_rne(d*q) that the tensor-core path stages.  Either output may be
 * NULL, not both.  Sizes [rows][K].
 */
int moe_dequantize(const uint8_t *qs, const uint16_t *scale, int64_t rows,
                   int32_t K, int32_t bits, float *out_f32, uint16_t *out_f16,
                   moe_stream_t stream);

/*
 * moe_router_topk: the router ([P1] "a small dictionary": a router picks the
 * best 10 of 512 experts for each word).
 *   logit[t,e] = sum_h x[t,h] * w_router[e,h] + bias[e]    (fp32 accumulate)
 *   topk_idx[t,j] = the k largest logits, ordered by (logit desc, id asc)
 *   topk_w[t,j]   = exp(l_j - l_0) / sum_{i<k} exp(l_i - l_0)
 *                   (the softmax over all E restricted to the k, renormalised)
 *   x        bf16 [T][H];  w_router bf16 [E][H];  bias fp32 [E] or NULL
 *   logits   fp32 [T][E] or NULL (written when given)
 *   topk_idx int32 [T][k];  topk_w fp32 [T][k]
 *   workspace: moe_router_workspace_size() bytes (may be 0 -> NULL allowed)
 * Limits: 1 <= k <= min(E, MOE_MAX_TOPK), E <= MOE_MAX_EXPERTS, H % 64 == 0.
 * T == 0 enqueues nothing.
 */
size_t moe_router_workspace_size(int32_t T, int32_t H, int32_t E, int32_t k);
int moe_router_topk(const uint16_t *x, const uint16_t *w_router, const float *bias,
                    int32_t T, int32_t H, int32_t E, int32_t k, float *logits,
                    int32_t *topk_idx, float *topk_w, void *workspace,
                    size_t workspace_bytes, moe_stream_t stream);

/* moe_topk_softmax: the selection and weights of moe_router_topk, applied to
 * given fp32 logits [T][E].  Same outputs, same limits. */
int moe_topk_softmax(const float *logits, int32_t T, int32_t E, int32_t k,
                     int32_t *topk_idx, float *topk_w, moe_stream_t stream);

/*
 * moe_bucketize: token -> expert grouping ([P1] "the four bugs, briefly": the
 * grouping helper must see each expert at most once per token and must never
 * drop a slot).  Slot s = t*k + j.
 *   expert_offsets int32 [E+1]: exclusive prefix sum of per-expert counts
 *   sorted_slot    int32 [T*k]: the slots of expert e, ascending, at
 *                               [expert_offsets[e], expert_offsets[e+1])
 *   slot_pos       int32 [T*k]: inverse map, sorted_slot[slot_pos[s]] == s
 *   active         int32 [E+1]: active[0] = number of experts with at least
 *                               one slot, then their ids ascending
 *   status         int32 [1] or NULL: MOE_STATUS_BAD_EXPERT_ID if an id is
 *                               outside [0,E); that slot is left out
 *                               (slot_pos[s] = -1).
 * Limits: T*k <= 2^24.
 */
int moe_bucketize(const int32_t *topk_idx, int32_t T, int32_t k, int32_t E,
                  int32_t *expert_offsets, int32_t *sorted_slot, int32_t *slot_pos,
                  int32_t *active, int32_t *status, moe_stream_t stream);

/*
 * moe_route: moe_router_topk followed by moe_bucketize ([P1] "a small
 * dictionary", "the four bugs, briefly"), with the same outputs bit for bit.
 * A batch of at most 16 tokens (whose bf16 rows fit in 200 KB of shared
 * memory) takes one fused kernel: every CTA computes the logits of 8 experts
 * and the CTA that finishes last ranks every token and groups the T*k slots;
 * larger batches run the two calls' kernels.
 *   outputs: topk_idx, topk_w as in moe_router_topk; expert_offsets,
 *            sorted_slot, slot_pos, active, status as in moe_bucketize
 *   workspace: moe_route_workspace_size() bytes, 16-byte aligned: the logits
 *            and a counter that the call clears with a memset and the fused
 *            kernel leaves at zero.  Calls sharing a workspace must not
 *            overlap on the GPU (issue them on one stream).
 * Limits: those of moe_router_topk and moe_bucketize.  T == 0 writes the
 * empty grouping (expert_offsets all 0, active[0] = 0).
 */
size_t moe_route_workspace_size(int32_t T, int32_t H, int32_t E, int32_t k);
int moe_route(const uint16_t *x, const uint16_t *w_router, const float *bias,
              int32_t T, int32_t H, int32_t E, int32_t k, int32_t *topk_idx,
              float *topk_w, int32_t *expert_offsets, int32_t *sorted_slot,
              int32_t *slot_pos, int32_t *active, int32_t *status, void *workspace,
              size_t workspace_bytes, moe_stream_t stream);

/*
 * moe_expert_ffn_tiered: the tiered SwiGLU expert FFN ([P1] "step 4":
 * mul_mat_id takes an id range, each shelf computes only the ids on it, and
 * the shelf results add up; the decode path fuses gate, up and activation).
 * Every (expert e, slot s) pair with expert_offsets/sorted_slot/active from
 * moe_bucketize, plus the shared expert for every token:
 *   g = W_gate[e] x[t], u = W_up[e] x[t], h = silu(g) * u, y = W_down[e] h
 *   y_slots  fp32 [T*k][H]  (row s = t*k+j)
 *   y_shared fp32 [T][H]    (NULL iff the layer has no shared expert)
 * `mode` is MOE_FFN_AUTO / _GEMV / _GEMM.  The GEMV path multiplies exact
 * integer codes with fp16 x (exact for bf16 magnitudes in [2^-14, 65504]) and
 * with h split into fp16 hi + lo, accumulates in fp32 and applies each block's
 * scale in fp32; the GEMM path stages d*q, x and h in fp16 and accumulates in
 * fp32 (tcgen05).  Both report MOE_STATUS_FP16_RANGE if x or h leaves the fp16
 * range.  AUTO sends experts with at least 8 tokens to the GEMM path.
 * workspace: moe_ffn_workspace_size() bytes.
 */
size_t moe_ffn_workspace_size(const moe_layer_weights *w, int32_t T, int32_t k,
                              int32_t mode);
int moe_expert_ffn_tiered(const moe_layer_weights *w, const uint16_t *x, int32_t T,
                          int32_t k, const int32_t *expert_offsets,
                          const int32_t *sorted_slot, const int32_t *active,
                          float *y_slots, float *y_shared, void *workspace,
                          size_t workspace_bytes, int32_t mode, int32_t *status,
                          moe_stream_t stream);

/*
 * moe_expert_ffn_tiered_static: the streaming (MOE_FFN_GEMV) path of
 * moe_expert_ffn_tiered with no workspace argument.  The pages have no
 * counterpart of this call; it exists for callers that cannot hand the
 * library a device buffer: a C or C++ host with no device allocator of its
 * own, whose decode loop must not call cudaMalloc/cudaFree because cudaFree
 * waits for the whole device and so stalls every other stream on it, and a
 * serving process that reserved its HBM for weights and KV cache up front
 * and has nothing spare to carve a workspace from.
 *
 * Its scratch (the SwiGLU intermediates of every slot and the completion
 * counters) is one array of MOE_STATIC_SCRATCH_BYTES bytes compiled into the
 * library: every GPU that loads the library holds it until the process
 * exits.  The call needs
 *   align256((T*k + T) * I * 4) + align256((min(T*k, E) + 1 + 2) * 4)
 * bytes of it (the intermediates, then the per-slot counters and two words a
 * grid barrier may use; at I = 512, k = 10: up to 46 tokens) and returns
 * MOE_ERR_UNSUPPORTED, enqueueing nothing, when that exceeds the array or
 * when the batch's shared-memory layout leaves the streaming kernel no room
 * for a tile (the same check as moe_expert_ffn_tiered in MOE_FFN_GEMV mode).
 * Arguments, outputs and results are those of moe_expert_ffn_tiered in
 * MOE_FFN_GEMV mode.  It allocates nothing: it clears the counters with an
 * asynchronous memset on `stream` and launches the streaming kernel.
 *
 * All calls on a device share the one array and each overwrites what the
 * previous one left there, so two calls whose work overlaps on the GPU (on
 * different streams, or from several host threads) race and give undefined
 * results: order them on one stream or with events.  The first call on each
 * device looks up the array's device address (with that device current),
 * so make that first call before any stream capture on that device.
 */
#define MOE_STATIC_SCRATCH_BYTES (1 << 20)
int moe_expert_ffn_tiered_static(const moe_layer_weights *w, const uint16_t *x,
                                 int32_t T, int32_t k, const int32_t *expert_offsets,
                                 const int32_t *sorted_slot, const int32_t *active,
                                 float *y_slots, float *y_shared, int32_t *status,
                                 moe_stream_t stream);

/*
 * moe_combine: out[t] = bf16_rne( sum_{j<k} topk_w[t,j] * y_slots[t*k+j]
 *                                 + y_shared[t] )
 * summed in that fixed order ([P1] "step 4": the results simply add up).
 * With residual != NULL it also advances the bf16 residual stream of a stack
 * of layers ([P5] "What the model actually is": 48 layers, residual design):
 *   x_next[t] = bf16_rne(residual[t] + out[t])
 *   x_next_norm[t] = bf16_rne(x_next[t] / sqrt(mean_h(x_next[t]^2) + MOE_NORM_EPS))
 * (the RMS-normalised stream that the next layer reads; NULL to skip).
 *   y_slots fp32 [T*k][H]; y_shared fp32 [T][H] or NULL; topk_w fp32 [T][k]
 *   residual bf16 [T][H] or NULL; out bf16 [T][H] (may be NULL when a residual
 *   is given); x_next, x_next_norm bf16 [T][H] (x_next needed iff residual).
 */
int moe_combine(const float *y_slots, const float *y_shared, const float *topk_w,
                int32_t T, int32_t k, int32_t H, const uint16_t *residual,
                uint16_t *out, uint16_t *x_next, uint16_t *x_next_norm,
                moe_stream_t stream);

/* moe_rmsnorm: n[t] = bf16_rne(x[t] / sqrt(mean_h(x[t]^2) + MOE_NORM_EPS)),
 * the input of the first layer of a stack.  x, n bf16 [T][H], H % 4 == 0. */
int moe_rmsnorm(const uint16_t *x, int32_t T, int32_t H, uint16_t *n, moe_stream_t stream);

/*
 * moe_layer_forward: moe_route -> tiered FFN -> combine, with every
 * intermediate in `workspace` (moe_layer_workspace_size() bytes).  The routing
 * kernel also clears the FFN's counters, so the FFN needs no memset of its own.
 *   x bf16 [T][H] (the layer input); w_router bf16 [E][H]; bias fp32 [E] or NULL
 *   out bf16 [T][H]; with residual != NULL also x_next and x_next_norm as in
 *   moe_combine (in a stack: x = the normalised stream, residual = the stream).
 * Same limits as the calls it chains.  Capturable into a CUDA graph.
 */
size_t moe_layer_workspace_size(const moe_layer_weights *w, int32_t T, int32_t k,
                                int32_t mode);
int moe_layer_forward(const moe_layer_weights *w, const uint16_t *w_router,
                      const float *bias, const uint16_t *x, int32_t T, int32_t k,
                      const uint16_t *residual, uint16_t *out, uint16_t *x_next,
                      uint16_t *x_next_norm, void *workspace, size_t workspace_bytes, int32_t mode,
                      int32_t *status, moe_stream_t stream);

/*
 * A stack of decode layers in one persistent launch ([P5] "What the model
 * actually is": 48 layers with a residual design; [P1] "step 3: split every
 * layer into hot and cold": the per-token time goes to thousands of launches
 * and syncs rather than to expert bytes, so the whole stack runs as one).
 * For each layer l, with x_0 = x_in:
 *   n_l     = bf16_rne(x_l / sqrt(mean_h(x_l^2) + MOE_NORM_EPS))
 *   out_l   = the layer on n_l: router top-k, the tiered expert FFN (every
 *             expert on the streaming path, MOE_FFN_GEMV numerics) and combine
 *   x_{l+1} = bf16_rne(x_l + out_l)
 * x_out = x_L; x_out_norm = n_L when given.  x_layers, when given, receives
 * x_0 .. x_L ([n_layers + 1][T][H]) for inspection.
 *
 * moe_stack_prepare writes a device descriptor of the layers (their weights
 * descriptors, routers and the tensor maps of their shelves):
 *   layers    host array [n_layers]; all share H, I and E
 *   w_router  host array [n_layers] of device pointers, bf16 [E][H]
 *   bias      host array [n_layers] of device pointers fp32 [E] (entries may
 *             be NULL), or NULL for no bias at all
 *   desc      device buffer of moe_stack_desc_bytes(n_layers) bytes, 64-byte
 *             aligned, owned by the caller
 * Unlike every other call it copies synchronously (a set-up step, run once
 * per set of weights; run it again whenever a weight pointer changes).
 *
 * moe_stack_forward enqueues one memset and one cooperative launch:
 *   x_in, x_out bf16 [T][H]; x_out_norm bf16 [T][H] or NULL; x_layers or NULL
 *   workspace  moe_stack_workspace_size() bytes, 16-byte aligned
 *   status     as for the other calls (MOE_STATUS_TIMEOUT if a grid-wide or
 *              pipeline wait gave up; outputs are then undefined)
 * Limits: 1 <= T <= 8; k, E, H and I as for moe_layer_forward on the
 * streaming path.  Calls sharing a workspace must not overlap on the GPU.
 */
size_t moe_stack_desc_bytes(int32_t n_layers);
int moe_stack_prepare(const moe_layer_weights *layers, const uint16_t *const *w_router,
                      const float *const *bias, int32_t n_layers, void *desc, size_t desc_bytes);
size_t moe_stack_workspace_size(int32_t H, int32_t I, int32_t E, int32_t T, int32_t k);
int moe_stack_forward(const void *desc, int32_t n_layers, int32_t H, int32_t I, int32_t E,
                      int32_t T, int32_t k, const uint16_t *x_in, uint16_t *x_out,
                      uint16_t *x_out_norm, uint16_t *x_layers, void *workspace,
                      size_t workspace_bytes, int32_t *status, moe_stream_t stream);

/* ------------------------------------------------------------------------ *
 * Test hook for the failure-detection paths (not for production use).
 *
 * Every device-side wait (mbarrier phases, the per-slot gate_up counters, the
 * grid barriers) gives up after a number of SM clock cycles, about 1 s by
 * default, and the call then reports MOE_STATUS_TIMEOUT in its status word.
 * moe_debug_set_waits sets that limit for the calls enqueued after it
 * (wait_limit_cycles <= 0 restores the default), and with skip_publish_slot
 * >= 0 makes the streaming FFN kernels never publish the gate_up completions
 * of that slot (the slot's position in the kernel's plan order; -1: none), so
 * that a wait on them runs out without any fault.  The setting is
 * process-wide and applies to moe_expert_ffn_tiered, moe_layer_forward and
 * moe_stack_forward; calls already enqueued keep the values they were
 * launched with.  Always returns MOE_OK.
 * ------------------------------------------------------------------------ */
int moe_debug_set_waits(int64_t wait_limit_cycles, int32_t skip_publish_slot);

#ifdef __cplusplus
}
#endif

#endif /* MOE_TIERED_H */
