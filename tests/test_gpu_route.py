"""moe_route (the router's top-k and the token -> expert grouping in one call)
against the two calls it replaces, bit for bit, and against the oracle.

Batches of at most 16 tokens take the fused kernel (logits in every CTA, top-k
and grouping in the CTA that finishes last); larger ones chain the separate
kernels.  Both sides of that boundary are covered, with and without a router
bias, for E a multiple of 8 and not, up to E = 1000 and k = 32.
"""
import numpy as np
import pytest
import torch

import oracle
from mixed_precision_moe_router_b200 import binding as B
from mixed_precision_moe_router_b200 import inputs
from mixed_precision_moe_router_b200.inputs import LayerConfig
from tests import helpers as Hh

DEV = "cuda"

WIDE = LayerConfig("wide", H=256, I=128, E=1000, k=32, tiers=((8, 200), (4, 400), (3, 400)), zipf_alpha=0.0)
ODD = LayerConfig("odd", H=192, I=128, E=37, k=5, tiers=((8, 7), (4, 15), (3, 15)))
CFGS = {"decode": inputs.DECODE, "tiny": inputs.TINY, "wide": WIDE, "odd": ODD}


def _separate(x, wr, bias, k, E):
    idx, w, _ = B.router_topk(x, wr, bias, k)
    return (idx, w) + tuple(B.bucketize(idx, E))


@pytest.mark.gpu
@pytest.mark.parametrize("name,T", [("decode", 1), ("decode", 2), ("decode", 5), ("decode", 8), ("decode", 16),
                                    ("decode", 17), ("decode", 40), ("tiny", 1), ("tiny", 16), ("wide", 3),
                                    ("wide", 16), ("odd", 1), ("odd", 11)])
def test_route_matches_separate_calls(name, T):
    cfg = CFGS[name]
    seed = inputs.layer_seed(cfg)
    wr, bias = inputs.router(cfg, seed, DEV)
    x = inputs.activations(T, cfg.H, seed=seed + 7, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    ws = torch.empty(int(B.lib().moe_route_workspace_size(T, cfg.H, cfg.E, cfg.k)), dtype=torch.uint8, device=DEV)
    want = _separate(x, wr, bias, cfg.k, cfg.E)
    for _ in range(3):  # the workspace is reused: its counter must be left at zero
        got = B.route(x, wr, bias, cfg.k, status=status, workspace=ws)
        for g, e, what in zip(got[:5], want[:5], ("idx", "w", "offsets", "sorted", "pos")):
            assert torch.equal(g, e), what
        # active: the count, then that many ids (the rest is not written)
        n = int(want[5][0])
        assert torch.equal(got[5][: 1 + n], want[5][: 1 + n]), "active"
    assert status.item() == 0


@pytest.mark.gpu
@pytest.mark.parametrize("T", [1, 9, 16])
def test_route_against_oracle(T):
    """The fused kernel's routing: logits within the fp32 bound of the oracle,
    selections certified where the margin allows, and the grouping equal to
    the oracle's grouping of the selected ids."""
    cfg = inputs.DECODE
    seed = inputs.layer_seed(cfg)
    wr, bias = inputs.router(cfg, seed, DEV)
    x = inputs.activations(T, cfg.H, seed=seed + 29, device=DEV)
    idx, w, off, srt, pos, act = B.route(x, wr, bias, cfg.k)
    xn, wn = x.float().cpu().numpy(), wr.float().cpu().numpy()
    bn = None if bias is None else bias.cpu().numpy()
    L = oracle.router_logits(xn, wn, bn)
    bound = Hh.logit_error_bound(xn, wn, bn)
    cert, near = Hh.check_routing(idx.cpu().numpy(), w.cpu().numpy(), L, cfg.k, bound)
    assert cert + near == T
    Hh.assert_few_near_ties(near, T, 0.1, f"fused route T={T}")
    o_off, o_srt, o_pos = oracle.bucketize(idx.cpu().numpy(), cfg.E)
    assert np.array_equal(off.cpu().numpy(), o_off)
    assert np.array_equal(srt.cpu().numpy(), o_srt)
    assert np.array_equal(pos.cpu().numpy(), o_pos)
    counts = np.diff(o_off)
    a = act.cpu().numpy()
    assert a[0] == np.count_nonzero(counts) and np.array_equal(a[1: 1 + a[0]], np.nonzero(counts)[0])


@pytest.mark.gpu
def test_route_empty_batch():
    cfg = inputs.DECODE
    wr, bias = inputs.router(cfg, inputs.layer_seed(cfg), DEV)
    x = torch.empty(0, cfg.H, dtype=torch.bfloat16, device=DEV)
    idx, w, off, srt, pos, act = B.route(x, wr, bias, cfg.k)
    assert idx.shape == (0, cfg.k) and int(act[0]) == 0 and not off.any()
