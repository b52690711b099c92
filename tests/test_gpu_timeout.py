"""Failure detection without a fault: a bounded device-side wait runs out.

moe_debug_set_waits shortens the device-side wait limit and makes the
streaming FFN kernels withhold the gate_up completions of one slot.  The wait
for that slot's count (and, across CTAs, the waits and grid barriers behind
it) then gives up: the call returns, reports MOE_STATUS_TIMEOUT, and the next
call, with the defaults restored, gives exactly the result of a call made
before the hook was set.
"""
import pytest
import torch

from mixed_precision_moe_router_b200 import binding as B
from mixed_precision_moe_router_b200 import inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"
STATUS_TIMEOUT = 0x4
SHORT_WAIT = 200_000  # SM clock cycles, about 0.1 ms


@pytest.fixture
def hook():
    yield B.debug_set_waits
    B.debug_set_waits(0, -1)
    torch.cuda.synchronize()


def _status():
    return torch.zeros(1, dtype=torch.int32, device=DEV)


@pytest.fixture(scope="module")
def tiny():
    cfg = inputs.TINY
    seed = inputs.layer_seed(cfg)
    layer = B.build_layer(cfg, seed, DEV)
    router = inputs.router(cfg, seed, DEV)
    torch.cuda.synchronize()
    return cfg, layer, router


def test_expert_ffn_withheld_slot_times_out(tiny, hook):
    cfg, layer, (wr, bias) = tiny
    x = inputs.activations(8, cfg.H, seed=inputs.X_SEED + 21, device=DEV)
    idx, _, _ = B.router_topk(x, wr, bias, cfg.k)
    off, srt, _, act = B.bucketize(idx, cfg.E)
    ref = B.expert_ffn(layer, x, cfg.k, off, srt, act, mode=B.FFN_GEMV)
    hook(SHORT_WAIT, 0)
    st = _status()
    B.expert_ffn(layer, x, cfg.k, off, srt, act, mode=B.FFN_GEMV, status=st)
    torch.cuda.synchronize()  # the call ended: no wait was left hanging
    assert st.item() & STATUS_TIMEOUT, hex(st.item())
    hook(0, -1)
    st = _status()
    again = B.expert_ffn(layer, x, cfg.k, off, srt, act, mode=B.FFN_GEMV, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    assert torch.equal(again[0], ref[0]) and torch.equal(again[1], ref[1])


def test_layer_forward_routed_in_kernel_times_out(tiny, hook):
    """One token: the FFN kernel routes the token itself (grid barrier), then
    the withheld slot stalls its down projection."""
    cfg, layer, (wr, bias) = tiny
    x = inputs.activations(1, cfg.H, seed=inputs.X_SEED + 22, device=DEV)
    ref = B.layer_forward(layer, wr, bias, x, cfg.k, mode=B.FFN_GEMV).clone()
    hook(SHORT_WAIT, 0)
    st = _status()
    B.layer_forward(layer, wr, bias, x, cfg.k, mode=B.FFN_GEMV, status=st)
    torch.cuda.synchronize()
    assert st.item() & STATUS_TIMEOUT, hex(st.item())
    hook(0, -1)
    st = _status()
    again = B.layer_forward(layer, wr, bias, x, cfg.k, mode=B.FFN_GEMV, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    assert torch.equal(again, ref)


@pytest.mark.parametrize("n_layers", [1, 3])
def test_stack_withheld_slot_times_out(tiny, hook, n_layers):
    """The persistent stack: the stalled CTAs give up, the others give up at
    the next grid barrier, and the launch ends with MOE_STATUS_TIMEOUT."""
    cfg, layer, router = tiny
    st_desc = B.Stack([layer] * n_layers, [router] * n_layers)
    x = inputs.activations(2, cfg.H, seed=inputs.X_SEED + 23, device=DEV)
    ref = B.stack_forward(st_desc, x, cfg.k).clone()
    hook(SHORT_WAIT, 0)
    st = _status()
    B.stack_forward(st_desc, x, cfg.k, status=st)
    torch.cuda.synchronize()
    assert st.item() & STATUS_TIMEOUT, hex(st.item())
    hook(0, -1)
    st = _status()
    again = B.stack_forward(st_desc, x, cfg.k, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    assert torch.equal(again, ref)


def test_short_limit_alone_does_not_fail_a_call(tiny, hook):
    """The limit bounds waits that never end; with nothing withheld a call
    under a short limit completes normally."""
    cfg, layer, (wr, bias) = tiny
    x = inputs.activations(8, cfg.H, seed=inputs.X_SEED + 24, device=DEV)
    idx, _, _ = B.router_topk(x, wr, bias, cfg.k)
    off, srt, _, act = B.bucketize(idx, cfg.E)
    ref = B.expert_ffn(layer, x, cfg.k, off, srt, act, mode=B.FFN_GEMV)
    hook(50_000_000, -1)
    st = _status()
    got = B.expert_ffn(layer, x, cfg.k, off, srt, act, mode=B.FFN_GEMV, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    assert torch.equal(got[0], ref[0]) and torch.equal(got[1], ref[1])
