"""The streaming expert FFN (GEMV mode) against the oracle on layer shapes
that select each tile layout and schedule the kernel has.

- gate_up tiles staged as one padded 5-D copy (rows of whole 128-byte lines:
  H = 2048 and H = 1024 at every precision) and as one copy per column chunk
  (H = 256);
- down tiles of 16R rows with R = 8 (I = 128), R = 4 (I = 512) and R = 2
  (I = 1024);
- few tiles per CTA (16 experts) and many (512 experts at T = 8), so that the
  stage ring wraps around and both consumer groups take several tiles of
  several slots.
The per-slot outputs must match the oracle's expert FFN to 1e-5 relative L2
(the GEMV path's products are exact and its only roundings are x -> fp16 and
the hi + lo split of h).
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

SHAPES = {
    "H256_I1024_many_tiles": (LayerConfig("s1", H=256, I=1024, E=64, k=10, tiers=((8, 16), (4, 24), (3, 24))), 8),
    "H2048_I128_few_tiles": (LayerConfig("s2", H=2048, I=128, E=16, k=2, tiers=((8, 4), (4, 6), (3, 6))), 1),
    "H2048_I128_E512": (LayerConfig("s3", H=2048, I=128, E=512, k=10, tiers=((8, 128), (4, 192), (3, 192))), 1),
    "H1024_I512_E512": (LayerConfig("s4", H=1024, I=512, E=512, k=10, tiers=((8, 128), (4, 192), (3, 192))), 1),
    "H2048_I512_T8": (inputs.DECODE, 8),
}


@pytest.mark.gpu
@pytest.mark.parametrize("name", list(SHAPES))
def test_streaming_ffn_shapes_match_oracle(name):
    cfg, T = SHAPES[name]
    seed = 1234
    layer = B.build_layer(cfg, seed, DEV)
    x = inputs.activations(T, cfg.H, seed=seed, device=DEV)
    ids = torch.stack([torch.randperm(cfg.E, generator=torch.Generator().manual_seed(t))[: cfg.k]
                       for t in range(T)]).to(torch.int32).to(DEV)
    off, srt, pos, act = B.bucketize(ids, cfg.E)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    y, ysh = B.expert_ffn(layer, x, cfg.k, off, srt, act, mode=B.FFN_GEMV, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    ox = Hh.OracleExperts(cfg, seed, DEV)
    xn = x.float().cpu().numpy()
    idn = ids.cpu().numpy().reshape(-1)
    exp = np.stack([oracle.expert_ffn(xn[s // cfg.k: s // cfg.k + 1], *ox(int(idn[s])))[0]
                    for s in range(T * cfg.k)])
    assert Hh.rel_l2(y.cpu().numpy(), exp) < 1e-5
    esh = oracle.expert_ffn(xn, *ox.shared())
    assert Hh.rel_l2(ysh.cpu().numpy(), esh) < 1e-5


@pytest.mark.gpu
def test_streaming_ffn_largest_tables_sampled():
    """E = 1024 experts and 150 tokens through the GEMV path: the largest slot
    and entry tables next to full fragment buffers for both consumer groups
    (the prologue's own tables then share the stage ring).  Every slot is
    finite and 24 sampled slots and the shared expert match the oracle."""
    cfg = LayerConfig("big", H=2048, I=512, E=1024, k=10, tiers=((8, 256), (4, 384), (3, 384)))
    T, seed = 150, 99
    layer = B.build_layer(cfg, seed, DEV)
    x = inputs.activations(T, cfg.H, seed=seed, device=DEV)
    ids = torch.stack([torch.randperm(cfg.E, generator=torch.Generator().manual_seed(7 + t))[: cfg.k]
                       for t in range(T)]).to(torch.int32).to(DEV)
    off, srt, pos, act = B.bucketize(ids, cfg.E)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    y, ysh = B.expert_ffn(layer, x, cfg.k, off, srt, act, mode=B.FFN_GEMV, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    y = y.cpu().numpy()
    assert np.isfinite(y).all()
    ox = Hh.OracleExperts(cfg, seed, DEV)
    xn = x.float().cpu().numpy()
    idn = ids.cpu().numpy().reshape(-1)
    for s in np.random.default_rng(3).choice(T * cfg.k, size=24, replace=False):
        exp = oracle.expert_ffn(xn[s // cfg.k: s // cfg.k + 1], *ox(int(idn[s])))[0]
        assert Hh.rel_l2(y[s], exp) < 1e-5, s
    esh = oracle.expert_ffn(xn, *ox.shared())
    assert Hh.rel_l2(ysh.cpu().numpy(), esh) < 1e-5


@pytest.mark.gpu
@pytest.mark.parametrize("mode", [B.FFN_GEMV, B.FFN_GEMM])
def test_down_width_640_matches_oracle(mode):
    """I = 640, the down width the pages' model has ([P1] "step 4": rows 640
    wide): 20 scale blocks per down row (3-bit rows of 240 bytes, staged in
    16-byte columns; scale rows of 40 bytes, staged as bulk copies) through the
    streaming and the tensor-core paths, against the oracle."""
    cfg = LayerConfig("i640", H=2048, I=640, E=16, k=2, tiers=((8, 4), (4, 6), (3, 6)))
    T, seed = 8, 640
    layer = B.build_layer(cfg, seed, DEV)
    x = inputs.activations(T, cfg.H, seed=seed, device=DEV)
    ids = torch.stack([torch.randperm(cfg.E, generator=torch.Generator().manual_seed(31 + t))[: cfg.k]
                       for t in range(T)]).to(torch.int32).to(DEV)
    off, srt, pos, act = B.bucketize(ids, cfg.E)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    y, ysh = B.expert_ffn(layer, x, cfg.k, off, srt, act, mode=mode, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    ox = Hh.OracleExperts(cfg, seed, DEV)
    xn = x.float().cpu().numpy()
    idn = ids.cpu().numpy().reshape(-1)
    exp = np.stack([oracle.expert_ffn(xn[s // cfg.k: s // cfg.k + 1], *ox(int(idn[s])))[0]
                    for s in range(T * cfg.k)])
    esh = oracle.expert_ffn(xn, *ox.shared())
    tol = 1e-5 if mode == B.FFN_GEMV else Hh.REL_L2  # exact products vs fp16-staged tensor-core operands
    assert Hh.rel_l2(y.cpu().numpy(), exp) < tol
    assert Hh.rel_l2(ysh.cpu().numpy(), esh) < tol
