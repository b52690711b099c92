"""ctypes binding of libmoe_tiered.so (argument marshalling only).

Every function here checks shapes and dtypes, passes raw device pointers and the
current CUDA stream to the C ABI declared in include/moe_tiered.h, and raises
if the call reports an error.  All arithmetic runs in the library's kernels;
there is no fallback: if the library is missing, :func:`lib` raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_tiered.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_UNSUPPORTED = 2
MOE_ERR_WORKSPACE = 3
MOE_ERR_CUDA = 4
STATUS_BAD_EXPERT_ID = 0x1
STATUS_FP16_RANGE = 0x2
STATUS_TIMEOUT = 0x4
FFN_AUTO, FFN_GEMV, FFN_GEMM = 0, 1, 2
MAX_TIERS = 4
STATIC_SCRATCH_BYTES = 1 << 20  # size of the scratch array behind moe_expert_ffn_tiered_static

c_i32, c_i64, c_size, c_vp = ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t, ctypes.c_void_p


class Tier(ctypes.Structure):
    _fields_ = [("bits", c_i32), ("first_expert", c_i32), ("n_experts", c_i32), ("dn_bits", c_i32),
                ("gu_qs", c_vp), ("gu_scale", c_vp), ("dn_qs", c_vp), ("dn_scale", c_vp)]


class LayerWeights(ctypes.Structure):
    _fields_ = [("H", c_i32), ("I", c_i32), ("E", c_i32), ("n_tiers", c_i32),
                ("tiers", Tier * MAX_TIERS), ("shared", Tier)]


# (name, restype, argtypes) of every exported symbol
SIGNATURES = [
    ("moe_last_error", ctypes.c_char_p, []),
    ("moe_version", ctypes.c_char_p, []),
    ("moe_packed_row_bytes", c_size, [c_i32, c_i32]),
    ("moe_quantize", c_i32, [c_vp, c_i64, c_i32, c_i32, c_vp, c_vp, c_vp]),
    ("moe_dequantize", c_i32, [c_vp, c_vp, c_i64, c_i32, c_i32, c_vp, c_vp, c_vp]),
    ("moe_router_workspace_size", c_size, [c_i32, c_i32, c_i32, c_i32]),
    ("moe_router_topk", c_i32, [c_vp, c_vp, c_vp, c_i32, c_i32, c_i32, c_i32, c_vp, c_vp, c_vp, c_vp,
                                c_size, c_vp]),
    ("moe_topk_softmax", c_i32, [c_vp, c_i32, c_i32, c_i32, c_vp, c_vp, c_vp]),
    ("moe_bucketize", c_i32, [c_vp, c_i32, c_i32, c_i32, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp]),
    ("moe_route_workspace_size", c_size, [c_i32, c_i32, c_i32, c_i32]),
    ("moe_route", c_i32, [c_vp, c_vp, c_vp, c_i32, c_i32, c_i32, c_i32, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp,
                          c_vp, c_vp, c_size, c_vp]),
    ("moe_ffn_workspace_size", c_size, [ctypes.POINTER(LayerWeights), c_i32, c_i32, c_i32]),
    ("moe_expert_ffn_tiered", c_i32, [ctypes.POINTER(LayerWeights), c_vp, c_i32, c_i32, c_vp, c_vp, c_vp,
                                      c_vp, c_vp, c_vp, c_size, c_i32, c_vp, c_vp]),
    ("moe_expert_ffn_tiered_static", c_i32, [ctypes.POINTER(LayerWeights), c_vp, c_i32, c_i32, c_vp, c_vp,
                                             c_vp, c_vp, c_vp, c_vp, c_vp]),
    ("moe_combine", c_i32, [c_vp, c_vp, c_vp, c_i32, c_i32, c_i32, c_vp, c_vp, c_vp, c_vp, c_vp]),
    ("moe_rmsnorm", c_i32, [c_vp, c_i32, c_i32, c_vp, c_vp]),
    ("moe_layer_workspace_size", c_size, [ctypes.POINTER(LayerWeights), c_i32, c_i32, c_i32]),
    ("moe_layer_forward", c_i32, [ctypes.POINTER(LayerWeights), c_vp, c_vp, c_vp, c_i32, c_i32, c_vp, c_vp,
                                  c_vp, c_vp, c_vp, c_size, c_i32, c_vp, c_vp]),
    ("moe_stack_desc_bytes", c_size, [c_i32]),
    ("moe_stack_prepare", c_i32, [ctypes.POINTER(LayerWeights), ctypes.POINTER(c_vp), ctypes.POINTER(c_vp), c_i32,
                                  c_vp, c_size]),
    ("moe_stack_workspace_size", c_size, [c_i32, c_i32, c_i32, c_i32, c_i32]),
    ("moe_stack_forward", c_i32, [c_vp, c_i32, c_i32, c_i32, c_i32, c_i32, c_i32, c_vp, c_vp, c_vp, c_vp, c_vp,
                                  c_size, c_vp, c_vp]),
    ("moe_debug_set_waits", c_i32, [ctypes.c_int64, c_i32]),
]

_lib = None


def lib():
    """Load the library (once); raise if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m mixed_precision_moe_router_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, res, args in SIGNATURES:
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


class MoeError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__(f"moe error {code}: {msg}")
        self.code = code


def _check(rc):
    if rc != MOE_OK:
        raise MoeError(rc, lib().moe_last_error().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _need(t, dtype, shape=None, name="tensor"):
    if t.dtype != dtype:
        raise TypeError(f"{name}: dtype {t.dtype}, want {dtype}")
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name}: must be a contiguous CUDA tensor")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, want {tuple(shape)}")


# `bits` of an FP4 (E2M1, power-of-two block scale) shelf; stored as 4-bit codes
FP4 = 5


def storage_bits(bits):
    """Code bits per weight in memory (4 for an FP4 shelf)."""
    return 4 if bits == FP4 else bits


def formats(bits):
    """(gate_up format, down format) of a shelf given as one format or a pair."""
    return (bits, bits) if isinstance(bits, int) else (int(bits[0]), int(bits[1]))


def packed_row_bytes(K, bits):
    return int(lib().moe_packed_row_bytes(K, bits))


# ---------------------------------------------------------------------------
# quantisation
# ---------------------------------------------------------------------------

def quantize(src, bits, out_qs=None, out_scale=None):
    """fp32 [rows, K] -> (codes uint8 [rows, K*bits/8], fp16 scale bits int16 [rows, K/32]);
    bits 8, 4, 3 or FP4."""
    _need(src, torch.float32, name="src")
    rows, K = src.shape
    qs = out_qs if out_qs is not None else torch.empty(rows, K * storage_bits(bits) // 8, dtype=torch.uint8,
                                                       device=src.device)
    sc = out_scale if out_scale is not None else torch.empty(rows, K // 32, dtype=torch.int16, device=src.device)
    _check(lib().moe_quantize(_ptr(src), rows, K, bits, _ptr(qs), _ptr(sc), _stream()))
    return qs, sc


def dequantize(qs, scale, K, bits, f32=True, f16=False):
    rows = qs.shape[0]
    o32 = torch.empty(rows, K, dtype=torch.float32, device=qs.device) if f32 else None
    o16 = torch.empty(rows, K, dtype=torch.int16, device=qs.device) if f16 else None
    _check(lib().moe_dequantize(_ptr(qs), _ptr(scale), rows, K, bits, _ptr(o32), _ptr(o16), _stream()))
    return o32, (o16.view(torch.float16) if o16 is not None else None)


# ---------------------------------------------------------------------------
# packed layer
# ---------------------------------------------------------------------------

class TieredLayer:
    """A layer's shelves (one packed table per precision) plus the shared expert.

    ``tiers`` is a list of dicts with keys bits, first, n, gu_qs, gu_scale,
    dn_qs, dn_scale (CUDA tensors laid out as moe_tiered.h states); ``shared``
    is such a dict with n == 1, or None.
    """

    def __init__(self, H, I, E, tiers, shared):
        self.H, self.I, self.E = H, I, E
        self.tiers, self.shared = tiers, shared
        self._desc = None

    @staticmethod
    def allocate(H, I, E, tier_ranges, shared_bits, device):
        def shelf(bits, first, n):
            gu, dn = formats(bits)
            return dict(bits=gu, dn_bits=dn, first=first, n=n,
                        gu_qs=torch.empty(n, 2 * I, H * storage_bits(gu) // 8, dtype=torch.uint8, device=device),
                        gu_scale=torch.empty(n, 2 * I, H // 32, dtype=torch.int16, device=device),
                        dn_qs=torch.empty(n, H, I * storage_bits(dn) // 8, dtype=torch.uint8, device=device),
                        dn_scale=torch.empty(n, H, I // 32, dtype=torch.int16, device=device))
        tiers = [shelf(b, f, n) for b, f, n in tier_ranges]
        shared = shelf(shared_bits, E, 1) if shared_bits else None
        return TieredLayer(H, I, E, tiers, shared)

    def shelf_of(self, e):
        if e == self.E:
            return self.shared, 0
        for t in self.tiers:
            if t["first"] <= e < t["first"] + t["n"]:
                return t, e - t["first"]
        raise KeyError(e)

    def set_expert(self, e, w_gate_up, w_down):
        """Quantise one expert's fp32 source weights into its shelf (on the GPU)."""
        t, j = self.shelf_of(e)
        quantize(w_gate_up.contiguous(), t["bits"], t["gu_qs"][j], t["gu_scale"][j])
        quantize(w_down.contiguous(), t["dn_bits"], t["dn_qs"][j], t["dn_scale"][j])
        self._desc = None

    def nbytes_expert(self, e):
        t, _ = self.shelf_of(e)
        gu, dn = storage_bits(t["bits"]), storage_bits(t["dn_bits"])
        rows_k = 2 * self.I * self.H + self.H * self.I
        return (2 * self.I * self.H * gu + self.H * self.I * dn) // 8 + rows_k // 32 * 2

    def descriptor(self):
        if self._desc is None:
            d = LayerWeights()
            d.H, d.I, d.E, d.n_tiers = self.H, self.I, self.E, len(self.tiers)

            def fill(dst, t):
                dst.bits, dst.first_expert, dst.n_experts = t["bits"], t["first"], t["n"]
                dst.dn_bits = 0 if t["dn_bits"] == t["bits"] else t["dn_bits"]
                dst.gu_qs, dst.gu_scale = t["gu_qs"].data_ptr(), t["gu_scale"].data_ptr()
                dst.dn_qs, dst.dn_scale = t["dn_qs"].data_ptr(), t["dn_scale"].data_ptr()
            for i, t in enumerate(self.tiers):
                fill(d.tiers[i], t)
            if self.shared is not None:
                fill(d.shared, self.shared)
            else:
                d.shared.n_experts = 0
            self._desc = d
        return self._desc


def build_layer(cfg, seed, device, source=None, tier_ranges=None):
    """Allocate a layer for ``cfg`` and quantise every expert from its source weights.

    ``source(cfg, seed, e, device)`` returns (gate_up fp32 [2I,H], down fp32 [H,I]);
    by default the seeded generator in :mod:`.inputs`.
    """
    from . import inputs
    source = source or inputs.expert_source
    ranges = tier_ranges or cfg.tier_ranges()
    layer = TieredLayer.allocate(cfg.H, cfg.I, cfg.E, ranges, cfg.shared_bits if cfg.shared else 0, device)
    for e in range(cfg.E + (1 if cfg.shared else 0)):
        wgu, wdn = source(cfg, seed, e, device)
        layer.set_expert(e, wgu, wdn)
    return layer


# ---------------------------------------------------------------------------
# the four hot-path calls and the fused layer
# ---------------------------------------------------------------------------

def router_topk(x, w_router, bias, k, want_logits=False):
    _need(x, torch.bfloat16, name="x")
    _need(w_router, torch.bfloat16, name="w_router")
    T, H = x.shape
    E = w_router.shape[0]
    dev = x.device
    idx = torch.empty(T, k, dtype=torch.int32, device=dev)
    w = torch.empty(T, k, dtype=torch.float32, device=dev)
    logits = torch.empty(T, E, dtype=torch.float32, device=dev) if want_logits else None
    ws = None
    nws = 0
    if not want_logits:
        nws = int(lib().moe_router_workspace_size(T, H, E, k))
        ws = torch.empty(max(nws, 1), dtype=torch.uint8, device=dev)
    if bias is not None:
        _need(bias, torch.float32, (E,), "bias")
    _check(lib().moe_router_topk(_ptr(x), _ptr(w_router), _ptr(bias), T, H, E, k, _ptr(logits), _ptr(idx),
                                 _ptr(w), _ptr(ws), nws, _stream()))
    return idx, w, logits


def topk_softmax(logits, k):
    _need(logits, torch.float32, name="logits")
    T, E = logits.shape
    idx = torch.empty(T, k, dtype=torch.int32, device=logits.device)
    w = torch.empty(T, k, dtype=torch.float32, device=logits.device)
    _check(lib().moe_topk_softmax(_ptr(logits), T, E, k, _ptr(idx), _ptr(w), _stream()))
    return idx, w


def bucketize(topk_idx, E, status=None):
    _need(topk_idx, torch.int32, name="topk_idx")
    T, k = topk_idx.shape
    dev = topk_idx.device
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    sorted_slot = torch.empty(max(T * k, 1), dtype=torch.int32, device=dev)
    slot_pos = torch.empty(max(T * k, 1), dtype=torch.int32, device=dev)
    active = torch.empty(E + 1, dtype=torch.int32, device=dev)
    _check(lib().moe_bucketize(_ptr(topk_idx), T, k, E, _ptr(offsets), _ptr(sorted_slot), _ptr(slot_pos),
                               _ptr(active), _ptr(status), _stream()))
    return offsets, sorted_slot[: T * k], slot_pos[: T * k], active


def route(x, w_router, bias, k, status=None, workspace=None):
    """moe_route: the router's top-k and the token -> expert grouping in one
    call.  Returns (topk_idx, topk_w, offsets, sorted_slot, slot_pos, active).
    A caller-owned `workspace` (uint8, moe_route_workspace_size bytes) may be
    reused across calls on one stream."""
    _need(x, torch.bfloat16, name="x")
    _need(w_router, torch.bfloat16, name="w_router")
    T, H = x.shape
    E = w_router.shape[0]
    dev = x.device
    if bias is not None:
        _need(bias, torch.float32, (E,), "bias")
    idx = torch.empty(max(T, 1), k, dtype=torch.int32, device=dev)
    w = torch.empty(max(T, 1), k, dtype=torch.float32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    sorted_slot = torch.empty(max(T * k, 1), dtype=torch.int32, device=dev)
    slot_pos = torch.empty(max(T * k, 1), dtype=torch.int32, device=dev)
    active = torch.empty(E + 1, dtype=torch.int32, device=dev)
    nws = int(lib().moe_route_workspace_size(T, H, E, k))
    if workspace is None:
        workspace = torch.empty(max(nws, 1), dtype=torch.uint8, device=dev)
    _check(lib().moe_route(_ptr(x), _ptr(w_router), _ptr(bias), T, H, E, k, _ptr(idx), _ptr(w), _ptr(offsets),
                           _ptr(sorted_slot), _ptr(slot_pos), _ptr(active), _ptr(status), _ptr(workspace),
                           workspace.numel(), _stream()))
    return idx[:T], w[:T], offsets, sorted_slot[: T * k], slot_pos[: T * k], active


def expert_ffn(layer, x, k, offsets, sorted_slot, active, mode=FFN_AUTO, status=None):
    _need(x, torch.bfloat16, name="x")
    T = x.shape[0]
    dev = x.device
    d = layer.descriptor()
    y_slots = torch.empty(T * k, layer.H, dtype=torch.float32, device=dev)
    y_shared = torch.empty(T, layer.H, dtype=torch.float32, device=dev) if layer.shared is not None else None
    nws = int(lib().moe_ffn_workspace_size(ctypes.byref(d), T, k, mode))
    ws = torch.empty(max(nws, 1), dtype=torch.uint8, device=dev)
    _check(lib().moe_expert_ffn_tiered(ctypes.byref(d), _ptr(x), T, k, _ptr(offsets), _ptr(sorted_slot),
                                       _ptr(active), _ptr(y_slots), _ptr(y_shared), _ptr(ws), nws, mode,
                                       _ptr(status), _stream()))
    return y_slots, y_shared


def expert_ffn_static(layer, x, k, offsets, sorted_slot, active, status=None):
    """The streaming expert FFN through the call that takes no workspace: its
    scratch is an array inside the library, for hosts that cannot allocate
    device memory while they decode.  Calls on one device share that array, so
    they must not overlap on the GPU (issue them on one stream)."""
    _need(x, torch.bfloat16, name="x")
    T = x.shape[0]
    dev = x.device
    d = layer.descriptor()
    y_slots = torch.empty(T * k, layer.H, dtype=torch.float32, device=dev)
    y_shared = torch.empty(T, layer.H, dtype=torch.float32, device=dev) if layer.shared is not None else None
    _check(lib().moe_expert_ffn_tiered_static(ctypes.byref(d), _ptr(x), T, k, _ptr(offsets), _ptr(sorted_slot),
                                              _ptr(active), _ptr(y_slots), _ptr(y_shared), _ptr(status),
                                              _stream()))
    return y_slots, y_shared


def combine(y_slots, y_shared, topk_w, residual=None, want_out=True, want_norm=True):
    """Returns out, or (out, x_next, x_next_norm) when a residual is given."""
    T, k = topk_w.shape
    H = y_slots.shape[1]
    dev = y_slots.device
    out = torch.empty(T, H, dtype=torch.bfloat16, device=dev) if want_out else None
    x_next = torch.empty(T, H, dtype=torch.bfloat16, device=dev) if residual is not None else None
    n_next = torch.empty(T, H, dtype=torch.bfloat16, device=dev) if residual is not None and want_norm else None
    _check(lib().moe_combine(_ptr(y_slots), _ptr(y_shared), _ptr(topk_w), T, k, H, _ptr(residual), _ptr(out),
                             _ptr(x_next), _ptr(n_next), _stream()))
    return out if residual is None else (out, x_next, n_next)


def rmsnorm(x, out=None):
    _need(x, torch.bfloat16, name="x")
    T, H = x.shape
    n = out if out is not None else torch.empty_like(x)
    _check(lib().moe_rmsnorm(_ptr(x), T, H, _ptr(n), _stream()))
    return n


def layer_workspace_size(layer, T, k, mode=FFN_AUTO):
    return int(lib().moe_layer_workspace_size(ctypes.byref(layer.descriptor()), T, k, mode))


def layer_forward(layer, w_router, bias, x, k, residual=None, mode=FFN_AUTO, workspace=None, out=None,
                  x_next=None, x_next_norm=None, status=None):
    """One MoE layer through the library's fused entry point.  Returns out, or
    (out, x_next, x_next_norm) when a residual is given."""
    _need(x, torch.bfloat16, name="x")
    T = x.shape[0]
    dev = x.device
    d = layer.descriptor()
    nws = int(lib().moe_layer_workspace_size(ctypes.byref(d), T, k, mode))
    if workspace is None:
        workspace = torch.empty(max(nws, 1), dtype=torch.uint8, device=dev)
    if out is None:
        out = torch.empty(T, layer.H, dtype=torch.bfloat16, device=dev)
    if residual is not None:
        if x_next is None:
            x_next = torch.empty(T, layer.H, dtype=torch.bfloat16, device=dev)
        if x_next_norm is None:
            x_next_norm = torch.empty(T, layer.H, dtype=torch.bfloat16, device=dev)
    _check(lib().moe_layer_forward(ctypes.byref(d), _ptr(w_router), _ptr(bias), _ptr(x), T, k, _ptr(residual),
                                   _ptr(out), _ptr(x_next), _ptr(x_next_norm), _ptr(workspace), workspace.numel(),
                                   mode, _ptr(status), _stream()))
    return out if residual is None else (out, x_next, x_next_norm)


# ---------------------------------------------------------------------------
# a stack of decode layers in one persistent launch
# ---------------------------------------------------------------------------

class Stack:
    """Device descriptor of a stack of layers for :func:`stack_forward`
    (moe_stack_prepare; the layers and routers must outlive it)."""

    def __init__(self, layers, routers):
        n = len(layers)
        self.layers, self.routers = layers, routers
        self.H, self.I, self.E = layers[0].H, layers[0].I, layers[0].E
        self.n = n
        descs = (LayerWeights * n)(*[l.descriptor() for l in layers])
        wr = (c_vp * n)(*[r[0].data_ptr() for r in routers])
        bias = (c_vp * n)(*[(r[1].data_ptr() if r[1] is not None else None) for r in routers])
        nbytes = int(lib().moe_stack_desc_bytes(n))
        dev = routers[0][0].device
        self._buf = torch.empty(nbytes + 64, dtype=torch.uint8, device=dev)
        off = (-self._buf.data_ptr()) % 64
        self.desc = self._buf[off:off + nbytes]
        _check(lib().moe_stack_prepare(descs, wr, bias, n, _ptr(self.desc), nbytes))

    def workspace_size(self, T, k):
        return int(lib().moe_stack_workspace_size(self.H, self.I, self.E, T, k))


def stack_forward(stack, x_in, k, out=None, out_norm=None, x_layers=None, workspace=None, status=None):
    """x_in (bf16 [T, H], the residual stream) through every layer of `stack`
    in one launch; returns x_out (and fills out_norm / x_layers when given)."""
    _need(x_in, torch.bfloat16, name="x_in")
    T, H = x_in.shape
    if out is None:
        out = torch.empty_like(x_in)
    nws = stack.workspace_size(T, k)
    if workspace is None:
        workspace = torch.empty(max(nws, 1), dtype=torch.uint8, device=x_in.device)
    _check(lib().moe_stack_forward(_ptr(stack.desc), stack.n, stack.H, stack.I, stack.E, T, k, _ptr(x_in), _ptr(out),
                                   _ptr(out_norm), _ptr(x_layers), _ptr(workspace), workspace.numel(), _ptr(status),
                                   _stream()))
    return out


def debug_set_waits(wait_limit_cycles=0, skip_publish_slot=-1):
    """Test hook (moe_debug_set_waits): the device-side wait limit in SM clock
    cycles (<= 0: the default, about 1 s) and a slot whose gate_up completions
    the streaming FFN kernels never publish (-1: none)."""
    _check(lib().moe_debug_set_waits(int(wait_limit_cycles), int(skip_publish_slot)))
