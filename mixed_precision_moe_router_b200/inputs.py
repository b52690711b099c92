"""Seeded synthetic inputs for the tiered MoE layer.

This module only draws random numbers.  It holds none of the layer's arithmetic
(no routing, quantisation or FFN), so that the CUDA path and the CPU oracle can
both consume exactly the same tensors.

The pages' workloads are a real model on real text; the trained weights and the
calibration statistics are not available, so these synthetic inputs stand in
for them, with the routing skew the pages measure:

* [P1] "step 2: the experts are not equal": in the average layer the busiest
  25% of experts handle 52% of the tokens.  A Zipf-shaped router bias
  ``b[e] = -alpha * ln(e + 1)`` (expert id = popularity rank) with
  ``alpha = 0.2266`` reproduces that share against the logit noise of
  N(0,1) activations times N(0, 0.02) router weights at hidden 2048.
* [P1] "step 4": experts are reordered hottest-first, so the tier tables are
  contiguous id ranges: ids [0,128) in 8-bit, [128,320) in 4-bit, [320,512) in
  3-bit for the 512-expert layer.
* [P5] "What the model actually is": 512 experts, 10 routed + 1 shared.
"""
from __future__ import annotations

import dataclasses
import math

import torch

ZIPF_ALPHA = 0.2266
W_STD = 0.02


@dataclasses.dataclass(frozen=True)
class LayerConfig:
    name: str
    H: int
    I: int
    E: int
    k: int
    tiers: tuple  # ((bits, n_experts), ...) in id order, hottest first
    shared: bool = True
    zipf_alpha: float = ZIPF_ALPHA
    shared_bits: object = 8  # a format, or a (gate_up, down) pair

    def tier_ranges(self):
        out, first = [], 0
        for bits, n in self.tiers:
            out.append((bits, first, n))
            first += n
        assert first == self.E
        return out


# The five workloads.  C0 has no router bias (its recipe names none).
TINY = LayerConfig("tiny", H=256, I=128, E=16, k=2, tiers=((8, 4), (4, 6), (3, 6)),
                   zipf_alpha=0.0)
DECODE = LayerConfig("decode", H=2048, I=512, E=512, k=10,
                     tiers=((8, 128), (4, 192), (3, 192)))
# FP4 (E2M1) shelves: the library numbers that format 5.  A shelf's format is
# one number, or a (gate_up, down) pair.  TINY_FP4 has every kind of FP4 shelf
# (gate_up and down, down only, a shared expert with an FP4 down); the
# ladder layer follows the pages' repacking recipe, whose down projections
# drop to MXFP4 on the rarest shelf while gate_up drops to 3 bits.
FP4 = 5
TINY_FP4 = LayerConfig("tiny_fp4", H=256, I=128, E=16, k=2,
                       tiers=((8, 4), (FP4, 4), ((3, FP4), 4), ((4, FP4), 4)),
                       zipf_alpha=0.0, shared_bits=(8, FP4))
DECODE_LADDER = LayerConfig("decode_fp4_down", H=2048, I=512, E=512, k=10,
                            tiers=((8, 128), (4, 192), ((3, FP4), 192)))
CONFIGS = {"tiny": TINY, "decode": DECODE}

TINY_SEED = 0
X_SEED = 7
LAYER_SEED0 = 1000
N_STACK = 48
PREFILL_T = 4096
VERIFY_T = 5
VERIFY_RHO = 0.82
SWEEP_T = (1, 2, 5, 16, 64, 256)


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) % (2 ** 63))
    return g


def _mix(*parts: int) -> int:
    h = 0x9E3779B97F4A7C15
    for p in parts:
        h = (h * 0x100000001B3 + (int(p) & 0xFFFFFFFF) + 1) % (2 ** 63)
    return h


def activations(T: int, H: int, seed: int = X_SEED, device="cpu") -> torch.Tensor:
    """x ~ N(0, 1) rounded to bf16, [T, H]."""
    g = _gen(_mix(seed, 1, T, H), device)
    return torch.randn(T, H, generator=g, device=device).to(torch.bfloat16)


def correlated_activations(T: int, H: int, rho: float = VERIFY_RHO, seed: int = X_SEED,
                           device="cpu") -> torch.Tensor:
    """A base token plus T-1 drafts: x_t = sqrt(rho) z_0 + sqrt(1-rho) z_t (t >= 1).

    Correlated drafts make the batch reuse experts, like a speculative-verify
    batch whose drafts follow the base token.
    """
    g = _gen(_mix(seed, 2, T, H), device)
    z = torch.randn(T, H, generator=g, device=device)
    x = z.clone()
    x[1:] = math.sqrt(rho) * z[0:1] + math.sqrt(1.0 - rho) * z[1:]
    return x.to(torch.bfloat16)


def router(cfg: LayerConfig, seed: int, device="cpu"):
    """(W_r bf16 [E, H] ~ N(0, 0.02), bias fp32 [E] = -alpha ln(e+1) or None)."""
    g = _gen(_mix(seed, 3, cfg.E, cfg.H), device)
    w = (torch.randn(cfg.E, cfg.H, generator=g, device=device) * W_STD).to(torch.bfloat16)
    if cfg.zipf_alpha == 0.0:
        return w, None
    e = torch.arange(cfg.E, device=device, dtype=torch.float64)
    bias = (-cfg.zipf_alpha * torch.log(e + 1.0)).to(torch.float32)
    return w, bias


def expert_source(cfg: LayerConfig, seed: int, expert: int, device="cpu"):
    """Source fp32 weights of one expert: (gate_up [2I, H], down [H, I]) ~ N(0, 0.02).

    ``expert`` = E selects the shared expert.  Each expert has its own stream,
    so any one of them can be regenerated alone.
    """
    g = _gen(_mix(seed, 4, expert, cfg.H, cfg.I), device)
    wgu = torch.randn(2 * cfg.I, cfg.H, generator=g, device=device) * W_STD
    wdn = torch.randn(cfg.H, cfg.I, generator=g, device=device) * W_STD
    return wgu, wdn


def layer_seed(cfg: LayerConfig, layer: int = 0) -> int:
    return TINY_SEED if cfg is TINY else LAYER_SEED0 + layer
