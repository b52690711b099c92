"""Plain CPU oracle for the tiered mixed-precision MoE layer.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  The product path (the
CUDA library and its Python binding) never calls it and shares no code with it.

Everything here is written to be read against the pages, not to be fast:
floating point is fp64 unless a step is defined in another precision, every
step is the textbook definition, and library primitives (``@`` matmul, stable
sorts, ``exp``) are used only as whole steps.

Sources (cited by page title and section):

* [P1] "I ran a 125B model on three RTX 3090s at 80 tokens/s by teaching
  llama.cpp which experts matter" (dev.to).
* [P2] "Running Qwen3.8-Flash-Next 125B on Three RTX 3090s at 80 Tokens per
  Second" (n1n.ai).
* [P3] "flashnext-2x3090" README (gitlite mirror).
* [P5] "Qwen3.8-Flash-Next hits 39 tok/s on a 24GB GPU, provided you bring 96GB
  of system RAM" (deniz.in).

Readings of points the pages leave open are marked READING and listed in the
design notes; they are the plainest interpretation that the rest supports.

Parity pins: every function below is pinned by ``tests/test_oracle_pins.py``
(closed forms, special cases, brute force on tiny inputs).  Nothing in this
module is "parity unpinned".
"""
from __future__ import annotations

import numpy as np

# ---------------------------------------------------------------------------
# Block quantisation at three precisions
# [P1] "step 4: three shelves, all on the GPU": popular experts keep more bits,
# rare ones are squeezed harder; each shelf is one expert table.
# [P3] "Why the model fits at all": a 4-bit code per weight plus one 16-bit
# scale per 32 weights is 4.5 bits per weight (51.2B x 4.5 / 8 = 28.80 GB).
# READING: symmetric absmax blocks of 32 weights, one fp16 scale per block,
# qmax = 2**(bits-1) - 1, round half away from zero, division (not a
# reciprocal multiply) in IEEE fp32.
# ---------------------------------------------------------------------------

BLOCK = 32
QMAX = {8: 127, 4: 7, 3: 3}


def packed_row_bytes(K: int, bits: int) -> int:
    """Bytes of packed codes for one row of K weights (scales not included)."""
    assert K % BLOCK == 0 and bits in QMAX
    return K * bits // 8


def bits_per_weight(bits: int) -> float:
    """Storage cost per weight including the fp16 block scale ([P3])."""
    return bits + 16.0 / BLOCK


def quantize_rows(w, bits: int):
    """Quantise fp32 rows into (codes q int8 [R,K], scales d fp16 [R,K/32]).

    Per block of 32 consecutive weights along K:
      amax = max |w_i|                      (exact)
      d    = fp16_RNE( fp32(amax) / fp32(qmax) )   fp32 IEEE division
      q_i  = clamp( round_half_away( fp32(w_i) / fp32(d) ), -qmax, qmax )
      d == 0  ->  every q_i = 0
    """
    w = np.ascontiguousarray(w, dtype=np.float32)
    R, K = w.shape
    assert K % BLOCK == 0
    qmax = QMAX[bits]
    blocks = w.reshape(R, K // BLOCK, BLOCK)
    amax = np.abs(blocks).max(axis=2)
    d16 = (amax / np.float32(qmax)).astype(np.float16)  # fp32 divide, RNE to fp16
    d32 = d16.astype(np.float32)[..., None]
    safe = np.where(d32 == 0, np.float32(1), d32)
    ratio = (blocks / safe).astype(np.float32)  # IEEE fp32 division
    r = ratio.astype(np.float64)  # exact widening; the rounding below is exact in fp64
    q = np.trunc(r + np.copysign(0.5, r))  # round half away from zero
    q = np.clip(q, -qmax, qmax)
    q = np.where(d32 == 0, 0.0, q)
    return q.reshape(R, K).astype(np.int8), d16


def pack_rows(q, bits: int):
    """Pack integer codes into the library's byte format (one row at a time).

    8-bit: the int8 code itself, one byte per weight.
    4-bit: c = q + 8 (1..15); weight 2m in the low nibble of byte m, weight 2m+1
           in the high nibble.
    3-bit: c = q + 4 (1..7), stored as two planes per row: a low plane of K/4
           bytes holding bits 0-1 of weight i at bit 2*(i%4) of byte i//4, then a
           high plane of K/8 bytes holding bit 2 of weight i at bit i%8 of byte
           K/4 + i//8.
    """
    q = np.asarray(q, dtype=np.int64)
    R, K = q.shape
    if bits == 8:
        return q.astype(np.int8).view(np.uint8).copy()
    if bits == 4:
        c = (q + 8).astype(np.uint8)
        return (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)
    if bits == 3:
        c = (q + 4).astype(np.uint8)
        lo = c & 3
        hi = (c >> 2) & 1
        lo_plane = np.zeros((R, K // 4), np.uint8)
        for i in range(4):
            lo_plane |= (lo[:, i::4] << (2 * i)).astype(np.uint8)
        hi_plane = np.zeros((R, K // 8), np.uint8)
        for i in range(8):
            hi_plane |= (hi[:, i::8] << i).astype(np.uint8)
        return np.concatenate([lo_plane, hi_plane], axis=1)
    raise ValueError(bits)


def unpack_rows(packed, bits: int, K: int):
    """Inverse of :func:`pack_rows`: bytes -> integer codes q (int64 [R,K])."""
    p = np.asarray(packed, dtype=np.uint8)
    R = p.shape[0]
    if bits == 8:
        return p.view(np.int8).astype(np.int64)
    if bits == 4:
        q = np.empty((R, K), np.int64)
        q[:, 0::2] = (p & 0xF).astype(np.int64) - 8
        q[:, 1::2] = (p >> 4).astype(np.int64) - 8
        return q
    if bits == 3:
        lo_plane, hi_plane = p[:, : K // 4], p[:, K // 4 :]
        c = np.zeros((R, K), np.int64)
        for i in range(4):
            c[:, i::4] |= ((lo_plane >> (2 * i)) & 3).astype(np.int64)
        for i in range(8):
            c[:, i::8] |= (((hi_plane >> i) & 1).astype(np.int64) << 2)
        return c - 4
    raise ValueError(bits)


def dequantize_f32(packed, scale, bits: int, K: int):
    """w = float(d) * float(q); exact in fp32 (11-bit scale x 7-bit code)."""
    q = unpack_rows(packed, bits, K).astype(np.float32)
    d = np.repeat(np.asarray(scale, np.float16).astype(np.float32), BLOCK, axis=1)
    return d * q


def dequantize_f16(packed, scale, bits: int, K: int):
    """The fp16 value the tensor-core path stages: fp16_RNE(fp32(d*q))."""
    return dequantize_f32(packed, scale, bits, K).astype(np.float16)


def quantize_pack(w, bits: int):
    """Source fp32 rows -> (packed bytes, fp16 scales): the stored shelf format."""
    q, d = quantize_rows(w, bits)
    return pack_rows(q, bits), d


# ---------------------------------------------------------------------------
# FP4 (E2M1) shelf.  [P1] "step 4" stores the rarest down projections as
# MXFP4: a 4-bit floating-point code per weight and a power-of-two scale per
# block of 32 weights.
# READING (the pages name the format only): the OCP MX conversion.  The block's
# shared scale is X = 2^(floor(log2 amax) - 2) (2 = the largest exponent of
# E2M1, so amax / X lies in [4, 8)); each weight becomes w / X rounded to the
# nearest E2M1 value (magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6), ties to the even
# code, saturating at 6; a weight that rounds to 0 keeps code 0.  In the shelf
# format the nibbles are packed as the 4-bit codes are (code = sign * 8 +
# magnitude index) and the fp16 scale array holds d = X / 2, so that
# w = d * q with the integer q = 2 * value(code) in {0, +-1, +-2, +-3, +-4, +-6,
# +-8, +-12}; d is a power of two kept within fp16's exact range [2^-24, 2^15]
# (the block exponent is raised or lowered to it), and d = 0 for a zero block.
# ---------------------------------------------------------------------------

FP4_VALUES = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)  # E2M1 magnitude of index 0..7


def quantize_rows_fp4(w):
    """fp32 rows -> (codes uint8 [R,K] in 0..15, scales d fp16 [R,K/32])."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    R, K = w.shape
    assert K % BLOCK == 0
    blocks = w.reshape(R, K // BLOCK, BLOCK).astype(np.float64)
    amax = np.abs(blocks).max(axis=2)
    _, e = np.frexp(amax)                    # amax = f * 2^e, f in [0.5, 1): floor(log2 amax) = e - 1
    shared = np.clip(e - 1 - 2, -23, 16)     # d = 2^(shared - 1) within [2^-24, 2^15]
    X = np.ldexp(1.0, shared)[..., None]
    v = blocks / X                           # exact: a power-of-two divisor
    a = np.abs(v)
    vals = np.asarray(FP4_VALUES)
    dist = np.abs(a[..., None] - vals)       # exact differences of short binary fractions
    m = np.argmin(dist, axis=-1)             # the first (lower) index on a tie ...
    nxt = np.minimum(m + 1, 7)
    tie = (np.take_along_axis(dist, nxt[..., None], -1)[..., 0] == np.take_along_axis(dist, m[..., None], -1)[..., 0]) & (nxt != m)
    m = np.where(tie & (m % 2 == 1), nxt, m)  # ... moved to the even index
    code = m + np.where((v < 0) & (m > 0), 8, 0)
    code = np.where(amax[..., None] == 0, 0, code)
    d = np.where(amax == 0, 0.0, np.ldexp(1.0, shared - 1)).astype(np.float16)
    return code.reshape(R, K).astype(np.uint8), d


def fp4_integers(codes):
    """Codes 0..15 -> the integers q = 2 * value (sign from bit 3)."""
    c = np.asarray(codes, np.int64)
    mag = (2 * np.asarray(FP4_VALUES))[c & 7]
    return np.where(c & 8, -mag, mag).astype(np.int64)


def pack_rows_fp4(codes):
    """Nibbles as in the 4-bit shelf: weight 2m low, 2m+1 high in byte m."""
    c = np.asarray(codes, np.uint8)
    return (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)


def unpack_rows_fp4(packed, K: int):
    p = np.asarray(packed, np.uint8)
    c = np.empty((p.shape[0], K), np.uint8)
    c[:, 0::2] = p & 0xF
    c[:, 1::2] = p >> 4
    return c


def dequantize_fp4_f32(packed, scale, K: int):
    """w = float(d) * float(q); exact in fp32 (a power of two times |q| <= 12)."""
    q = fp4_integers(unpack_rows_fp4(packed, K)).astype(np.float32)
    d = np.repeat(np.asarray(scale, np.float16).astype(np.float32), BLOCK, axis=1)
    return d * q


def quantize_pack_fp4(w):
    c, d = quantize_rows_fp4(w)
    return pack_rows_fp4(c), d


# ---------------------------------------------------------------------------
# Router: logits, top-k, weights
# [P1] "a small dictionary before we start": each layer has 512 experts and a
# router picks the best 10 for each word.  [P5] "What the model actually is":
# 10 routed plus 1 shared expert active per token.
# READING: weights are the softmax over all E restricted to the chosen k and
# renormalised to sum to 1; ties go to the lower expert id; the bias (when
# present) enters both the choice and the weights.
# ---------------------------------------------------------------------------

def router_logits(x, w_router, bias=None):
    """l[t,e] = sum_h x[t,h] * W_r[e,h] + b[e], in fp64.

    x and W_r hold bf16 values (passed as float32 arrays), so every product is
    exact in fp64.
    """
    L = np.asarray(x, np.float64) @ np.asarray(w_router, np.float64).T
    if bias is not None:
        L = L + np.asarray(bias, np.float64)[None, :]
    return L


def select_topk(logits, k: int):
    """Top-k per token ordered by (logit descending, expert id ascending).

    Returns (idx int32 [T,k], w float64 [T,k]) with
    w_j = exp(l_j - l_0) / sum_{i<k} exp(l_i - l_0).
    """
    L = np.asarray(logits, np.float64)
    T, E = L.shape
    assert 1 <= k <= E
    ids = np.arange(E)
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    for t in range(T):
        order = np.lexsort((ids, -L[t]))  # last key is primary: -logit, then id
        sel = order[:k]
        idx[t] = sel
        z = np.exp(L[t, sel] - L[t, sel[0]])
        w[t] = z / z.sum()
    return idx, w


def topk_margin(logits, k: int):
    """Smallest gap between consecutive logits in the sorted top-(k+1) list.

    A selection (and its order) is certified exact when this gap exceeds twice
    the error bound of whatever computed the logits.  Returns float64 [T].
    """
    L = np.asarray(logits, np.float64)
    s = -np.sort(-L, axis=1)[:, : min(k + 1, L.shape[1])]
    if s.shape[1] < 2:
        return np.full(L.shape[0], np.inf)
    return np.min(s[:, :-1] - s[:, 1:], axis=1)


# ---------------------------------------------------------------------------
# Bucketize: token -> expert grouping
# [P1] "the four bugs, briefly": the expert-grouping helper assumes each expert
# appears at most once per word, and a duplicated "skip" id silently dropped a
# slot.  Here every slot s = t*k + j is listed exactly once, under its expert,
# in ascending s.
# ---------------------------------------------------------------------------

def bucketize(topk_idx, E: int):
    """Return (expert_offsets int32 [E+1], sorted_slot int32 [T*k], slot_pos int32 [T*k])."""
    ids = np.asarray(topk_idx, np.int64).reshape(-1)
    assert ids.size == 0 or (ids.min() >= 0 and ids.max() < E)
    counts = np.bincount(ids, minlength=E)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    sorted_slot = np.argsort(ids, kind="stable").astype(np.int32)
    slot_pos = np.empty_like(sorted_slot)
    slot_pos[sorted_slot] = np.arange(sorted_slot.size, dtype=np.int32)
    return offsets, sorted_slot, slot_pos


# ---------------------------------------------------------------------------
# Expert FFN (SwiGLU) on dequantised weights
# [P1] "step 4": mul_mat_id runs each word through its chosen experts; each
# shelf computes only the ids in its range and the three results add up; the
# decode path fuses gate, up and the activation.
# Weight layout per expert: gate_up [2I, H] (rows 0..I-1 gate, I..2I-1 up),
# down [H, I]; K is the contiguous axis.
# ---------------------------------------------------------------------------

def silu(g):
    g = np.asarray(g, np.float64)
    return g / (1.0 + np.exp(-g))


def expert_ffn(x, w_gate_up, w_down):
    """y = W_down @ (silu(W_gate @ x) * (W_up @ x)) for each row of x, in fp64."""
    x = np.asarray(x, np.float64)
    wgu = np.asarray(w_gate_up, np.float64)
    I = wgu.shape[0] // 2
    g = x @ wgu[:I].T
    u = x @ wgu[I:].T
    h = silu(g) * u
    return h @ np.asarray(w_down, np.float64).T


def round_f16(v):
    """Round to the nearest fp16 value, ties to even (one rounding from fp64)."""
    v = np.asarray(v, np.float64)
    out = np.zeros_like(v)
    nz = (v != 0) & np.isfinite(v)
    m, e = np.frexp(v[nz])
    step_exp = np.maximum(e - 11, -24)  # 11 significant bits; subnormal grid 2**-24
    r = np.ldexp(np.rint(np.ldexp(v[nz], -step_exp)), step_exp)
    r = np.where(np.abs(r) > 65504.0, np.copysign(np.inf, r), r)
    out[nz] = r
    out[~np.isfinite(v)] = v[~np.isfinite(v)]
    return out


def expert_ffn_f16_staged(x, w_gate_up_f16, w_down_f16):
    """The tensor-core path's arithmetic: x, the dequantised weights and h are
    each rounded to fp16; products and sums are exact (fp64 here, fp32 on the
    tensor cores).  ``w_*_f16`` are the fp16 staging values fp16(d*q)."""
    x16 = round_f16(x)
    wgu = np.asarray(w_gate_up_f16, np.float64)
    I = wgu.shape[0] // 2
    g = x16 @ wgu[:I].T
    u = x16 @ wgu[I:].T
    h16 = round_f16(silu(g) * u)
    return h16 @ np.asarray(w_down_f16, np.float64).T


# ---------------------------------------------------------------------------
# Rounding to bf16 (outputs and the residual stream are bf16)
# ---------------------------------------------------------------------------

def round_bf16(v):
    """Round fp64 values to the nearest bf16 value, ties to even, in one step."""
    v = np.asarray(v, np.float64)
    out = np.zeros_like(v)
    nz = (v != 0) & np.isfinite(v)
    m, e = np.frexp(v[nz])  # v = m * 2**e, 0.5 <= |m| < 1
    # bf16 keeps 8 significant bits; below 2**-126 the grid is fixed at 2**-133
    step_exp = np.maximum(e - 8, -133)
    scaled = np.ldexp(v[nz], -step_exp)  # exact power-of-two scaling
    r = np.ldexp(np.rint(scaled), step_exp)  # rint: half to even
    r = np.where(np.abs(r) > 3.3895313892515355e38, np.copysign(np.inf, r), r)
    out[nz] = r
    out[~np.isfinite(v)] = v[~np.isfinite(v)]
    return out


# ---------------------------------------------------------------------------
# Combine and the residual stream
# [P1] "step 4": the three shelf results simply add up.
# [P5] "What the model actually is": 48 layers, a residual design.
# READING: out[t] = bf16( sum_j w[t,j] * y[t*k+j] + y_shared[t] ) summed in the
# fixed order j = 0..k-1, then the shared expert.  In a stack the residual
# stream is bf16, x_next = bf16( x + out ), and each MoE layer reads the RMS-
# normalised stream n = bf16( x / sqrt(mean(x^2) + eps) ) (pre-norm, no learned
# gain, eps = 1e-6): without a norm the SwiGLU blocks, which grow like |x|^2,
# drive the stack to overflow within about 14 layers.
# ---------------------------------------------------------------------------

NORM_EPS = 1e-6


def rms_norm(x, eps=NORM_EPS):
    """bf16( x / sqrt(mean(x^2) + eps) ) per row, in fp64."""
    x = np.asarray(x, np.float64)
    r = np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    return round_bf16(x / r)


def combine(y_slots, y_shared, topk_w, residual=None):
    """Returns out, or (out, x_next, n_next) when a residual is given."""
    y = np.asarray(y_slots, np.float64)
    w = np.asarray(topk_w, np.float64)
    T, k = w.shape
    s = np.einsum("tj,tjh->th", w, y.reshape(T, k, -1))
    if y_shared is not None:
        s = s + np.asarray(y_shared, np.float64)
    out = round_bf16(s)
    if residual is None:
        return out
    x_next = round_bf16(np.asarray(residual, np.float64) + out)
    return out, x_next, rms_norm(x_next)


# ---------------------------------------------------------------------------
# Tier tables and the full layer
# ---------------------------------------------------------------------------

class Shelf:
    """One expert table at one precision covering ids [first, first + n)."""

    def __init__(self, bits, first, gu_qs, gu_scale, dn_qs, dn_scale):
        self.bits, self.first = int(bits), int(first)
        self.gu_qs, self.gu_scale = gu_qs, gu_scale
        self.dn_qs, self.dn_scale = dn_qs, dn_scale
        self.n = len(gu_qs)

    def owns(self, e):
        return self.first <= e < self.first + self.n

    def weights(self, e, H, I):
        """Dequantised fp32 (gate_up [2I,H], down [H,I]) of expert e."""
        j = e - self.first
        wgu = dequantize_f32(self.gu_qs[j], self.gu_scale[j], self.bits, H)
        wdn = dequantize_f32(self.dn_qs[j], self.dn_scale[j], self.bits, I)
        return wgu, wdn


def build_shelf(bits, first, sources):
    """Quantise a list of source expert weights [(w_gate_up f32, w_down f32)]."""
    gq, gs, dq, ds = [], [], [], []
    for wgu, wdn in sources:
        a, b = quantize_pack(wgu, bits)
        c, d = quantize_pack(wdn, bits)
        gq.append(a); gs.append(b); dq.append(c); ds.append(d)
    return Shelf(bits, first, gq, gs, dq, ds)


def shelf_of(shelves, e):
    hits = [s for s in shelves if s.owns(e)]
    assert len(hits) == 1, f"expert {e} must lie on exactly one shelf"
    return hits[0]


def shelves_lookup(shelves, H, I):
    """Expert id -> dequantised fp32 (gate_up, down) from a list of shelves."""
    def get(e):
        return shelf_of(shelves, e).weights(e, H, I)
    return get


def moe_layer(x, w_router, bias, k, expert_weights, shared_weights, H, I, residual=None):
    """One routed MoE layer: router -> top-k -> bucketize -> tiered FFN -> combine.

    ``expert_weights(e)`` returns expert e's dequantised fp32 (gate_up [2I,H],
    down [H,I]) from whichever shelf owns it (see :func:`shelves_lookup`);
    ``shared_weights`` is the shared expert's pair, or None.

    Returns a dict with every intermediate the library exposes.
    """
    x = np.asarray(x, np.float32)
    T = x.shape[0]
    E = np.asarray(w_router).shape[0]
    logits = router_logits(x, w_router, bias)
    idx, w = select_topk(logits, k)
    offsets, sorted_slot, slot_pos = bucketize(idx, E)
    y_slots = np.zeros((T * k, H), np.float64)
    for e in range(E):
        lo, hi = offsets[e], offsets[e + 1]
        if lo == hi:
            continue  # an expert nobody chose costs nothing
        slots = sorted_slot[lo:hi]
        wgu, wdn = expert_weights(e)
        y_slots[slots] = expert_ffn(x[slots // k], wgu, wdn)
    y_shared = None
    if shared_weights is not None:
        y_shared = expert_ffn(x, *shared_weights)
    res = combine(y_slots, y_shared, w, residual)
    out, x_next, n_next = (res if residual is not None else (res, None, None))
    return dict(logits=logits, topk_idx=idx, topk_w=w, expert_offsets=offsets,
                sorted_slot=sorted_slot, slot_pos=slot_pos, y_slots=y_slots,
                y_shared=y_shared, out=out, x_next=x_next, n_next=n_next)


def moe_stack(x0, layers, k, H, I):
    """Free-running stack: n_0 = rms_norm(x_0); per layer out = MoE(n_l),
    x_{l+1} = bf16(x_l + out), n_{l+1} = rms_norm(x_{l+1}).

    ``layers`` is a list of (w_router, bias, expert_weights, shared_weights).
    Returns the per-layer results (each holding its input n under key "n")."""
    x = np.asarray(x0, np.float64)
    n = rms_norm(x)
    results = []
    for (wr, bias, ew, sw) in layers:
        r = moe_layer(n.astype(np.float32), wr, bias, k, ew, sw, H, I, residual=x)
        r["n"], r["x"] = n, x
        results.append(r)
        x, n = r["x_next"], r["n_next"]
    return results
