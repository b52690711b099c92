"""The allocation-free expert FFN call against the one that takes a workspace.

moe_expert_ffn_tiered_static serves hosts that cannot allocate device memory
while they decode (a plain C host without an allocator of its own, where
cudaFree would wait for the whole device, or a server whose HBM is reserved up
front): its scratch is one array inside the library, shared by every call on a
device, so each call finds the previous call's intermediates and counters
there and must clear what has to start at zero.  The GPU test makes two calls
in a row with different tokens and routing on one stream and checks both
against moe_expert_ffn_tiered in GEMV mode, bit for bit, up to the largest
decode batch the array holds (46 tokens at I = 512, k = 10).

The file name sorts last, so pytest collects it after the other tests; it
passes alone in a fresh process (where its first call does the per-device
set-up) and after them.
"""
import ctypes

import pytest
import torch

from mixed_precision_moe_router_b200 import binding as B
from mixed_precision_moe_router_b200 import inputs

DEV = "cuda"


def _routing(cfg, T, seed):
    g = torch.Generator().manual_seed(seed)
    ids = torch.stack([torch.randperm(cfg.E, generator=g)[: cfg.k] for _ in range(T)]).to(torch.int32)
    return B.bucketize(ids.to(DEV), cfg.E)


@pytest.mark.gpu
@pytest.mark.parametrize("name,T", [("tiny", 8), ("decode", 1), ("decode", 8), ("decode", 46)])
def test_static_call_matches_workspace_call_twice_in_a_row(name, T):
    cfg = {"tiny": inputs.TINY, "decode": inputs.DECODE}[name]
    seed = inputs.layer_seed(cfg)
    layer = B.build_layer(cfg, seed, DEV)
    batches = []
    for call in range(2):
        x = inputs.activations(T, cfg.H, seed=seed + 50 + call, device=DEV)
        batches.append((x, _routing(cfg, T, 1000 * call + T)))
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    # two calls back to back on one stream: the second reuses the scratch the
    # first left behind
    got = [B.expert_ffn_static(layer, x, cfg.k, off, srt, act, status=status)
           for x, (off, srt, pos, act) in batches]
    want = [B.expert_ffn(layer, x, cfg.k, off, srt, act, mode=B.FFN_GEMV)
            for x, (off, srt, pos, act) in batches]
    torch.cuda.synchronize()
    assert status.item() == 0
    # the same kernel on the same inputs sums in the same order: any stale
    # intermediate or counter left by the first call would show as a difference
    for (ys, yshs), (yw, yshw) in zip(got, want):
        assert torch.isfinite(ys).all()
        assert torch.equal(ys, yw)
        assert torch.equal(yshs, yshw)


def test_static_call_rejects_batches_beyond_its_scratch():
    """Host-side size check: nothing is dereferenced or launched, so fake
    device pointers suffice and no GPU is needed."""
    d = B.LayerWeights()
    d.H, d.I, d.E, d.n_tiers = 2048, 512, 512, 1
    t = d.tiers[0]
    t.bits, t.first_expert, t.n_experts = 4, 0, 512
    t.gu_qs = t.gu_scale = t.dn_qs = t.dn_scale = 0x10000
    p = ctypes.c_void_p(0x20000)
    L = B.lib()
    # (T*k + T) * I * 4 bytes of intermediates: 47 tokens at k = 10 need more
    # than the array's 1 MiB, 46 tokens fit
    rc = L.moe_expert_ffn_tiered_static(ctypes.byref(d), p, 47, 10, p, p, p, p, None, None, None)
    assert rc == B.MOE_ERR_UNSUPPORTED
    msg = L.moe_last_error().decode()
    assert "static array" in msg and str(B.STATIC_SCRATCH_BYTES) in msg
    # invalid arguments are still reported as such
    assert L.moe_expert_ffn_tiered_static(ctypes.byref(d), p, 1, 10, p, p, p, p, p, None, None) \
        == B.MOE_ERR_INVALID_ARG  # y_shared given for a layer without a shared expert
