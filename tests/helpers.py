"""Test helpers: oracle-side expert preparation and comparison rules.

The oracle never receives anything the CUDA path computed: it gets the seeded
generator's source weights and activations and quantises them itself.
"""
import functools

import numpy as np
import torch

import oracle
from mixed_precision_moe_router_b200 import inputs

# Layer-output tolerance (bf16 outputs, fp32 accumulation against the fp64 oracle).
REL_L2 = 2e-3
MAX_ABS = 1e-2


def rel_l2(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def max_abs(a, b):
    return float(np.max(np.abs(np.asarray(a, np.float64) - np.asarray(b, np.float64)))) if np.size(a) else 0.0


def to_np(t):
    if t is None:
        return None
    if t.dtype == torch.bfloat16:
        t = t.float()
    return t.detach().cpu().numpy()


FP4 = 5  # the library's format number of an FP4 (E2M1) shelf


def formats(bits):
    """(gate_up, down) formats of a shelf given as one format or a pair."""
    return (bits, bits) if isinstance(bits, int) else (int(bits[0]), int(bits[1]))


def oracle_quantize_pack(w, fmt):
    return oracle.quantize_pack_fp4(w) if fmt == FP4 else oracle.quantize_pack(w, fmt)


def oracle_dequantize(q, s, fmt, K):
    return oracle.dequantize_fp4_f32(q, s, K) if fmt == FP4 else oracle.dequantize_f32(q, s, fmt, K)


def _prepare_expert(args):
    """Worker: oracle quantisation + dequantisation of one expert (runs in a
    spawned process; pure numpy, no GPU)."""
    wgu, wdn, bits, H, I = args
    gf, df = formats(bits)
    gq, gs = oracle_quantize_pack(wgu, gf)
    dq, ds = oracle_quantize_pack(wdn, df)
    return oracle_dequantize(gq, gs, gf, H), oracle_dequantize(dq, ds, df, I)


_POOL = None


def pool():
    """A process pool started with 'spawn' (safe after CUDA is initialised)."""
    global _POOL
    if _POOL is None:
        import concurrent.futures
        import multiprocessing
        import os
        n = max(1, min(32, (os.cpu_count() or 2) - 1))
        _POOL = concurrent.futures.ProcessPoolExecutor(n, mp_context=multiprocessing.get_context("spawn"))
    return _POOL


class OracleExperts:
    """Expert id -> dequantised fp32 weights, quantised by the oracle from the
    generator's source weights (drawn on ``device`` like the GPU layer's)."""

    def __init__(self, cfg, seed, device):
        self.cfg, self.seed, self.device = cfg, seed, device
        self._cache = {}
        self._packed = {}

    def prefetch(self, experts):
        """Prepare several experts in parallel (worker processes)."""
        todo = [int(e) for e in sorted(set(int(v) for v in experts)) if int(e) not in self._cache]
        if not todo:
            return
        jobs = []
        for e in todo:
            wgu, wdn = inputs.expert_source(self.cfg, self.seed, e, self.device)
            jobs.append((wgu.cpu().numpy(), wdn.cpu().numpy(), self.bits(e), self.cfg.H, self.cfg.I))
        for e, res in zip(todo, pool().map(_prepare_expert, jobs)):
            self._cache[e] = res

    def bits(self, e):
        if e == self.cfg.E:
            return self.cfg.shared_bits
        for bits, first, n in self.cfg.tier_ranges():
            if first <= e < first + n:
                return bits
        raise KeyError(e)

    def packed(self, e):
        if e not in self._packed:
            wgu, wdn = inputs.expert_source(self.cfg, self.seed, e, self.device)
            gf, df = formats(self.bits(e))
            self._packed[e] = (oracle_quantize_pack(wgu.cpu().numpy(), gf), oracle_quantize_pack(wdn.cpu().numpy(), df))
        return self._packed[e]

    def __call__(self, e):
        if e not in self._cache:
            (gq, gs), (dq, ds) = self.packed(e)
            gf, df = formats(self.bits(e))
            self._cache[e] = (oracle_dequantize(gq, gs, gf, self.cfg.H), oracle_dequantize(dq, ds, df, self.cfg.I))
        return self._cache[e]

    def shared(self):
        return self(self.cfg.E) if self.cfg.shared else None


def logit_error_bound(x, w_router, bias, factor=1.0):
    """Error bound used to certify routing decisions taken on fp32 logits.

    The GPU accumulates each logit in fp32 along H; a sequential fp32 sum of n
    terms is within gamma_n * sum|x_h w_h| of the exact value (gamma_n ~ n u).
    The CUDA-core routers sum at most 128 terms in sequence before a pairwise
    tree, so n_eff = 128 + log2(H) bounds them (factor 1).  The tensor-core
    router (64 tokens or more) adds the exact bf16 products into an fp32
    accumulator inside the MMA, whose alignment may truncate instead of
    rounding to nearest: factor 2 allows a whole ulp per addition.  Returns
    [T, E] bounds.
    """
    ax = np.abs(np.asarray(x, np.float64))
    aw = np.abs(np.asarray(w_router, np.float64))
    s = ax @ aw.T
    u = 2.0 ** -24
    n_eff = 128 + int(np.ceil(np.log2(max(ax.shape[1], 2))))
    b = factor * n_eff * u * s
    if bias is not None:
        b = b + u * np.abs(np.asarray(bias, np.float64))[None, :]
    return b


TENSOR_CORE_ROUTER_FACTOR = 2.0


def assert_few_near_ties(near, T, frac, what):
    """Report the near-tie count of a routing check and bound it: near ties
    are the tokens the bound cannot certify, a fraction set by the bound and
    the spacing of the top logits (about 5-13 % on these inputs)."""
    print(f"{what}: {near} of {T} tokens are near ties")
    assert near <= max(2, int(np.ceil(frac * T))), f"{what}: {near} near ties of {T}"


def check_routing(gpu_idx, gpu_w, ora_logits, k, bound):
    """Routing parity rule.

    Tokens whose oracle top-(k+1) gaps all exceed twice the bound are certified:
    their GPU indices must equal the oracle's exactly (same order) and weights
    match within 1e-5.  Others (near-ties) must be a valid choice: every chosen
    expert's exact logit is within 2*bound of the k-th largest, and the order is
    consistent within the bound.  Returns (n_certified, n_near_ties).
    """
    gi = np.asarray(gpu_idx)
    gw = np.asarray(gpu_w, np.float64)
    L = np.asarray(ora_logits, np.float64)
    T = L.shape[0]
    oi, ow = oracle.select_topk(L, k)
    cert = near = 0
    for t in range(T):
        order = np.lexsort((np.arange(L.shape[1]), -L[t]))[: k + 1]
        vals = L[t, order]
        gaps = vals[:-1] - vals[1:] if len(vals) > 1 else np.array([np.inf])
        tb = 2 * bound[t, order].max()
        if np.all(gaps > tb):
            cert += 1
            assert gi[t].tolist() == oi[t].tolist(), f"token {t}: {gi[t]} vs {oi[t]}"
            assert np.max(np.abs(gw[t] - ow[t])) < 1e-5
        else:
            near += 1
            kth = L[t, oi[t, -1]]
            assert len(set(gi[t].tolist())) == k
            assert np.all(L[t, gi[t]] >= kth - tb), f"token {t}: invalid near-tie choice"
            assert np.all(np.diff(L[t, gi[t]]) <= tb)
            assert abs(gw[t].sum() - 1) < 1e-5
    return cert, near


@functools.lru_cache(maxsize=None)
def sm100_available():
    if not torch.cuda.is_available():
        return False
    return torch.cuda.get_device_capability(0) >= (10, 0)
