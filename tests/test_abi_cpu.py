"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every symbol include/moe_tiered.h declares, and rejects invalid arguments
before it touches the device."""
import ctypes
import os
import re

import pytest

from mixed_precision_moe_router_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", src))
    return names


def test_library_exports_every_declared_symbol():
    L = B.lib()
    declared = header_functions()
    assert len(declared) >= 15
    for name in declared:
        assert hasattr(L, name), name
    assert declared == {n for n, _, _ in B.SIGNATURES}


def test_packed_row_bytes():
    assert B.packed_row_bytes(2048, 8) == 2048
    assert B.packed_row_bytes(2048, 4) == 1024
    assert B.packed_row_bytes(2048, 3) == 768
    assert B.packed_row_bytes(100, 4) == 0
    assert B.packed_row_bytes(128, B.FP4) == 64  # FP4: 4-bit storage
    assert B.packed_row_bytes(128, 6) == 0
    assert B.packed_row_bytes(128, 2) == 0


def test_fp4_format_number_agrees_with_the_header():
    from mixed_precision_moe_router_b200 import inputs
    from tests import helpers
    src = open(os.path.join(ROOT, "include", "moe_tiered.h")).read()
    assert int(re.search(r"#define MOE_FP4 (\d+)", src).group(1)) == B.FP4 == inputs.FP4 == helpers.FP4


def _fake_layer(tiers=((8, 0, 4), (4, 4, 6), (3, 10, 6)), H=256, I=128, E=16, shared=True, ptr=0x10000):
    d = B.LayerWeights()
    d.H, d.I, d.E, d.n_tiers = H, I, E, len(tiers)
    for i, (bits, first, n) in enumerate(tiers):
        t = d.tiers[i]
        t.bits, t.first_expert, t.n_experts = bits, first, n
        t.gu_qs = t.gu_scale = t.dn_qs = t.dn_scale = ptr
    if shared:
        d.shared.bits, d.shared.n_experts = 8, 1
        d.shared.gu_qs = d.shared.gu_scale = d.shared.dn_qs = d.shared.dn_scale = ptr
    return d


def _ffn(d, T=8, k=2, ws=1 << 30, mode=0):
    L = B.lib()
    p = ctypes.c_void_p(0x20000)
    return L.moe_expert_ffn_tiered(ctypes.byref(d), p, T, k, p, p, p, p, p if d.shared.n_experts else None,
                                   p, ws, mode, None, None)


@pytest.mark.parametrize("mutate,code", [
    (lambda d: setattr(d, "H", 192), B.MOE_ERR_INVALID_ARG),            # H % 128
    (lambda d: setattr(d, "I", 100), B.MOE_ERR_INVALID_ARG),
    (lambda d: setattr(d, "E", 0), B.MOE_ERR_INVALID_ARG),
    (lambda d: setattr(d, "n_tiers", 5), B.MOE_ERR_INVALID_ARG),
    (lambda d: setattr(d.tiers[1], "bits", 2), B.MOE_ERR_INVALID_ARG),
    (lambda d: setattr(d.tiers[1], "bits", 6), B.MOE_ERR_INVALID_ARG),
    (lambda d: setattr(d.tiers[2], "dn_bits", 2), B.MOE_ERR_INVALID_ARG),     # down format
    (lambda d: setattr(d.shared, "dn_bits", 7), B.MOE_ERR_INVALID_ARG),
    (lambda d: setattr(d.tiers[1], "first_expert", 3), B.MOE_ERR_INVALID_ARG),  # overlap
    (lambda d: setattr(d.tiers[2], "n_experts", 5), B.MOE_ERR_INVALID_ARG),     # gap
    (lambda d: setattr(d.tiers[2], "first_expert", -1), B.MOE_ERR_INVALID_ARG),  # negative id
    (lambda d: setattr(d.tiers[0], "gu_qs", 0x10008), B.MOE_ERR_INVALID_ARG),    # misaligned
    (lambda d: setattr(d.tiers[0], "dn_scale", None), B.MOE_ERR_INVALID_ARG),
    (lambda d: setattr(d.shared, "n_experts", 2), B.MOE_ERR_INVALID_ARG),
])
def test_ffn_rejects_bad_descriptor(mutate, code):
    d = _fake_layer()
    mutate(d)
    assert _ffn(d) == code
    assert B.lib().moe_last_error()


def test_ffn_rejects_bad_sizes_and_workspace():
    d = _fake_layer()
    assert _ffn(d, k=0) == B.MOE_ERR_INVALID_ARG
    assert _ffn(d, k=17) == B.MOE_ERR_INVALID_ARG       # k > E
    assert _ffn(d, T=-1) == B.MOE_ERR_INVALID_ARG
    assert _ffn(d, mode=7) == B.MOE_ERR_INVALID_ARG
    assert _ffn(d, ws=16) == B.MOE_ERR_WORKSPACE
    assert _ffn(d, T=0) == B.MOE_OK                      # nothing to do
    need = B.lib().moe_ffn_workspace_size(ctypes.byref(d), 8, 2, 0)
    assert need >= (8 * 2 + 8) * 128 * 4


def test_router_and_quantize_reject_bad_args():
    L = B.lib()
    p = ctypes.c_void_p(0x20000)
    assert L.moe_quantize(p, 4, 128, 6, p, p, None) == B.MOE_ERR_INVALID_ARG  # no such format
    assert L.moe_quantize(p, 4, 100, 8, p, p, None) == B.MOE_ERR_INVALID_ARG
    assert L.moe_quantize(ctypes.c_void_p(0x20004), 4, 128, 8, p, p, None) == B.MOE_ERR_INVALID_ARG
    assert L.moe_router_topk(p, p, None, 4, 256, 16, 17, None, p, p, None, 0, None) == B.MOE_ERR_INVALID_ARG
    assert L.moe_router_topk(p, p, None, 4, 256, 2000, 8, None, p, p, None, 0, None) == B.MOE_ERR_INVALID_ARG
    assert L.moe_router_topk(p, p, None, 4, 256, 16, 2, None, p, p, None, 0, None) == B.MOE_ERR_WORKSPACE
    assert L.moe_topk_softmax(p, 4, 16, 0, p, p, None) == B.MOE_ERR_INVALID_ARG
    assert L.moe_bucketize(p, 4, 2, 16, None, p, p, p, None, None) == B.MOE_ERR_INVALID_ARG
    assert L.moe_combine(p, None, p, 4, 2, 6, None, p, None, None, None) == B.MOE_ERR_INVALID_ARG
    assert L.moe_combine(p, None, p, 4, 2, 256, p, p, None, None, None) == B.MOE_ERR_INVALID_ARG  # no x_next
    assert L.moe_combine(p, None, p, 4, 2, 256, None, p, None, p, None) == B.MOE_ERR_INVALID_ARG  # norm w/o res
    assert L.moe_rmsnorm(p, 4, 6, p, None) == B.MOE_ERR_INVALID_ARG
    assert L.moe_dequantize(p, p, 4, 128, 8, None, None, None) == B.MOE_ERR_INVALID_ARG


def test_layer_workspace_sizes_grow_with_tokens():
    d = _fake_layer(H=2048, I=512, E=512, tiers=((8, 0, 128), (4, 128, 192), (3, 320, 192)))
    L = B.lib()
    a = L.moe_layer_workspace_size(ctypes.byref(d), 1, 10, 0)
    b = L.moe_layer_workspace_size(ctypes.byref(d), 4096, 10, 0)
    assert 0 < a < b
    assert b >= 4096 * 10 * 2048 * 4


def _route(T=1, H=2048, E=512, k=10, ws=1 << 20, x=0x20000, wsp=0x40000):
    L = B.lib()
    p = ctypes.c_void_p(0x30000)
    return L.moe_route(ctypes.c_void_p(x), p, None, T, H, E, k, p, p, p, p, p, p, None,
                       ctypes.c_void_p(wsp) if wsp else None, ws, None)


@pytest.mark.parametrize("kw,code", [
    (dict(k=0), B.MOE_ERR_INVALID_ARG),
    (dict(k=33, E=64), B.MOE_ERR_INVALID_ARG),          # k > MOE_MAX_TOPK
    (dict(E=1025), B.MOE_ERR_INVALID_ARG),
    (dict(H=100), B.MOE_ERR_INVALID_ARG),               # H % 64
    (dict(x=0x20008), B.MOE_ERR_INVALID_ARG),           # misaligned x
    (dict(ws=16), B.MOE_ERR_WORKSPACE),                 # smaller than logits + counter
    (dict(wsp=0), B.MOE_ERR_WORKSPACE),
    (dict(wsp=0x40008), B.MOE_ERR_INVALID_ARG),         # misaligned workspace
])
def test_route_rejects_bad_arguments(kw, code):
    assert _route(**kw) == code
    assert B.lib().moe_last_error()


def test_route_workspace_size():
    L = B.lib()
    # fp32 logits [T][E] (256-byte aligned) plus 256 bytes for the counter
    assert L.moe_route_workspace_size(1, 2048, 512, 10) == 2048 + 256
    assert L.moe_route_workspace_size(3, 2048, 100, 10) == 1280 + 256
    assert L.moe_route_workspace_size(0, 2048, 512, 10) == 256


def _layer_fwd(d, T=1, k=2, ws=None, wsp=0x40000, x=0x20000):
    L = B.lib()
    p = ctypes.c_void_p(0x30000)
    if ws is None:
        ws = int(L.moe_layer_workspace_size(ctypes.byref(d), T, k, 0))
    return L.moe_layer_forward(ctypes.byref(d), p, None, ctypes.c_void_p(x), T, k, None, p, None, None,
                               ctypes.c_void_p(wsp) if wsp else None, ws, 0, None, None)


def test_layer_forward_rejects_bad_arguments_before_enqueueing():
    """moe_layer_forward validates everything it can on the host first (fake
    device pointers: nothing here reaches the GPU)."""
    d = _fake_layer()
    assert _layer_fwd(d, T=0) == B.MOE_OK                                # empty batch: nothing to do
    assert _layer_fwd(d, k=0) == B.MOE_ERR_INVALID_ARG
    assert _layer_fwd(d, k=17) == B.MOE_ERR_INVALID_ARG                  # k > E
    assert _layer_fwd(d, ws=64) == B.MOE_ERR_WORKSPACE
    assert _layer_fwd(d, wsp=0) == B.MOE_ERR_WORKSPACE
    assert _layer_fwd(d, wsp=0x40008) == B.MOE_ERR_INVALID_ARG           # misaligned workspace
    assert _layer_fwd(d, x=0x20008) == B.MOE_ERR_INVALID_ARG             # misaligned x (checked by the router)
    bad = _fake_layer()
    bad.tiers[1].bits = 2
    assert _layer_fwd(bad) == B.MOE_ERR_INVALID_ARG
    assert B.lib().moe_last_error()


def test_layer_workspace_holds_the_route_workspace():
    """The layer workspace covers the routing call's logits and counter, the
    routing plan, the FFN intermediates and the slot outputs."""
    L = B.lib()
    d = _fake_layer(H=2048, I=512, E=512, tiers=((8, 0, 128), (4, 128, 192), (3, 320, 192)))
    for T in (1, 16, 17, 300):
        lay = int(L.moe_layer_workspace_size(ctypes.byref(d), T, 10, 0))
        route = int(L.moe_route_workspace_size(T, 2048, 512, 10))
        ffn = int(L.moe_ffn_workspace_size(ctypes.byref(d), T, 10, 0))
        slots = T * 10 * 2048 * 4 + T * 2048 * 4
        assert lay >= route + ffn + slots
