"""GPU parity at the workloads' full sizes (decode layer, 48-layer stack, prefill,
speculative-verify batch and token sweep), against the CPU oracle.

Where the oracle cannot afford every output it checks sampled tokens (a token's
output depends only on its own input and the weights), and in stacks the GPU
runs each layer on the oracle's own layer inputs, so that every comparison is
made on identical inputs.
"""
import os

import numpy as np
import pytest
import torch

import oracle
from mixed_precision_moe_router_b200 import binding as B
from mixed_precision_moe_router_b200 import inputs
from tests import helpers as Hh

pytestmark = pytest.mark.gpu
DEV = "cuda"
STACK_LAYERS = int(os.environ.get("MOE_TEST_STACK_LAYERS", str(inputs.N_STACK)))


def _bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(DEV).to(torch.bfloat16)


def _oracle_layer(cfg, seed, n, x, ox):
    """Oracle layer on its own inputs n (normalised) and x (stream)."""
    wr, bias = inputs.router(cfg, seed, DEV)
    wrn, bn = wr.float().cpu().numpy(), None if bias is None else bias.cpu().numpy()
    idx, _ = oracle.select_topk(oracle.router_logits(n, wrn, bn), cfg.k)
    ox.prefetch(list(idx.reshape(-1)) + ([cfg.E] if cfg.shared else []))
    return oracle.moe_layer(n, wrn, bn, cfg.k, ox, ox.shared(), cfg.H, cfg.I, residual=x), wrn, bn


def _check_layer_outputs(got_out, res, wrn, bn, n, rows=None, got_idx=None, got_w=None):
    o = got_out.float().cpu().numpy()
    e = res["out"] if rows is None else res["out"][rows]
    assert Hh.rel_l2(o, e) < Hh.REL_L2, Hh.rel_l2(o, e)
    assert Hh.max_abs(o, e) < Hh.MAX_ABS, Hh.max_abs(o, e)
    if got_idx is not None:
        L = res["logits"] if rows is None else res["logits"][rows]
        nn = n if rows is None else n[rows]
        Hh.check_routing(got_idx, got_w, L, got_idx.shape[1], Hh.logit_error_bound(nn, wrn, bn))


@pytest.fixture(scope="module")
def decode_stack():
    cfg = inputs.DECODE
    layers = [B.build_layer(cfg, inputs.layer_seed(cfg, l), DEV) for l in range(STACK_LAYERS)]
    torch.cuda.synchronize()
    yield cfg, layers
    del layers
    torch.cuda.empty_cache()


def test_decode_layer_one_token(decode_stack):
    """Decode configuration, one layer, one token, every hot-path step."""
    cfg, layers = decode_stack
    seed = inputs.layer_seed(cfg, 0)
    ox = Hh.OracleExperts(cfg, seed, DEV)
    x = inputs.activations(1, cfg.H, seed=inputs.X_SEED, device=DEV).float().cpu().numpy()
    n = oracle.rms_norm(x).astype(np.float32)
    res, wrn, bn = _oracle_layer(cfg, seed, n, x, ox)
    wr, bias = inputs.router(cfg, seed, DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    out, xn, nn = B.layer_forward(layers[0], wr, bias, _bf16(n), cfg.k, residual=_bf16(x), status=status)
    idx, w, _ = B.router_topk(_bf16(n), wr, bias, cfg.k)
    torch.cuda.synchronize()
    assert status.item() == 0
    _check_layer_outputs(out, res, wrn, bn, n, got_idx=idx.cpu().numpy(), got_w=w.cpu().numpy())


def test_decode_stack_teacher_forced_and_free_running(decode_stack):
    """48 stacked layers, 1 token: every GPU layer on the oracle's layer inputs
    matches the oracle's layer output; the free-running GPU stack stays close
    to the free-running oracle stack."""
    cfg, layers = decode_stack
    x = inputs.activations(1, cfg.H, seed=inputs.X_SEED, device=DEV).float().cpu().numpy()
    n = oracle.rms_norm(x).astype(np.float32)
    g_x = _bf16(x)
    g_n = B.rmsnorm(g_x)
    assert np.array_equal(g_n.float().cpu().numpy(), n) or Hh.max_abs(g_n.float().cpu().numpy(), n) <= 2 ** -7
    for l in range(STACK_LAYERS):
        seed = inputs.layer_seed(cfg, l)
        ox = Hh.OracleExperts(cfg, seed, DEV)
        res, wrn, bn = _oracle_layer(cfg, seed, n, x, ox)
        wr, bias = inputs.router(cfg, seed, DEV)
        out, _, _ = B.layer_forward(layers[l], wr, bias, _bf16(n), cfg.k, residual=_bf16(x))
        idx, w, _ = B.router_topk(_bf16(n), wr, bias, cfg.k)
        _check_layer_outputs(out, res, wrn, bn, n, got_idx=idx.cpu().numpy(), got_w=w.cpu().numpy())
        # the free-running GPU chain
        _, g_x, g_n = B.layer_forward(layers[l], wr, bias, g_n, cfg.k, residual=g_x)
        x, n = res["x_next"].astype(np.float32), res["n_next"].astype(np.float32)
    drift = Hh.rel_l2(g_x.float().cpu().numpy(), x)
    assert drift < 2e-2, drift


def test_decode_stack_eight_tokens_batch_invariant(decode_stack):
    """The 8-token decode batch: every token's result equals its 1-token run
    (GEMV path), so the 1-token oracle comparison above covers it."""
    cfg, layers = decode_stack
    xs = inputs.activations(8, cfg.H, seed=inputs.X_SEED + 1, device=DEV)
    g_x, g_n = xs.clone(), B.rmsnorm(xs)
    ones = [(xs[t:t + 1].clone(), B.rmsnorm(xs[t:t + 1].contiguous())) for t in range(8)]
    for l in range(min(STACK_LAYERS, 6)):
        wr, bias = inputs.router(cfg, inputs.layer_seed(cfg, l), DEV)
        _, g_x, g_n = B.layer_forward(layers[l], wr, bias, g_n, cfg.k, residual=g_x, mode=B.FFN_GEMV)
        for t in range(8):
            one_x, one_n = ones[t]
            _, one_x, one_n = B.layer_forward(layers[l], wr, bias, one_n, cfg.k, residual=one_x, mode=B.FFN_GEMV)
            ones[t] = (one_x, one_n)
            assert torch.equal(g_x[t:t + 1], one_x), (l, t)


@pytest.mark.parametrize("T", [1, 2, 5, 16, 64, 256])
def test_token_sweep_one_layer(decode_stack, T):
    """Sweep of token counts on one layer: sampled tokens against the oracle."""
    cfg, layers = decode_stack
    seed = inputs.layer_seed(cfg, 1)
    ox = Hh.OracleExperts(cfg, seed, DEV)
    x = inputs.activations(T, cfg.H, seed=inputs.X_SEED + T, device=DEV)
    n = B.rmsnorm(x)
    nn = oracle.rms_norm(x.float().cpu().numpy()).astype(np.float32)
    wr, bias = inputs.router(cfg, seed, DEV)
    out = B.layer_forward(layers[1], wr, bias, _bf16(nn), cfg.k)
    rows = np.arange(T) if T <= 8 else np.linspace(0, T - 1, 8).astype(int)
    res, wrn, bn = _oracle_layer(cfg, seed, nn[rows], None, ox)
    _check_layer_outputs(out[torch.from_numpy(rows).to(DEV)], res, wrn, bn, nn[rows])


def test_verify_batch_correlated_drafts(decode_stack):
    """1 base token + 4 correlated drafts through the stack, every token on the
    oracle's own layer inputs: all five tokens' outputs and routing match the
    oracle at every layer, and the drafts share most of the base token's
    experts."""
    cfg, layers = decode_stack
    xs = inputs.correlated_activations(inputs.VERIFY_T, cfg.H, device=DEV)
    x = xs.float().cpu().numpy()
    n = oracle.rms_norm(x).astype(np.float32)
    overlaps = []
    for l in range(min(STACK_LAYERS, 6)):
        seed = inputs.layer_seed(cfg, l)
        ox = Hh.OracleExperts(cfg, seed, DEV)
        res, wrn, bn = _oracle_layer(cfg, seed, n, x, ox)
        wr, bias = inputs.router(cfg, seed, DEV)
        out, _, _ = B.layer_forward(layers[l], wr, bias, _bf16(n), cfg.k, residual=_bf16(x))
        idx, w, _ = B.router_topk(_bf16(n), wr, bias, cfg.k)
        d = idx.cpu().numpy()
        _check_layer_outputs(out, res, wrn, bn, n, got_idx=d, got_w=w.cpu().numpy())
        overlaps += [len(set(d[0]) & set(d[t])) / cfg.k for t in range(1, inputs.VERIFY_T)]
        x, n = res["x_next"].astype(np.float32), res["n_next"].astype(np.float32)
    assert 0.3 < np.mean(overlaps) < 0.9


def test_prefill_layer_4096_tokens():
    """Prefill: one decode-configuration layer on 4096 tokens; routing of all
    tokens is certified, sampled tokens' outputs compared."""
    cfg = inputs.DECODE
    seed = inputs.layer_seed(cfg, 0)
    layer = B.build_layer(cfg, seed, DEV)
    T = inputs.PREFILL_T
    x = inputs.activations(T, cfg.H, seed=inputs.X_SEED + 4096, device=DEV)
    nn = oracle.rms_norm(x.float().cpu().numpy()).astype(np.float32)
    wr, bias = inputs.router(cfg, seed, DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    out = B.layer_forward(layer, wr, bias, _bf16(nn), cfg.k, status=status)
    idx, w, _ = B.router_topk(_bf16(nn), wr, bias, cfg.k)
    torch.cuda.synchronize()
    assert status.item() == 0
    wrn, bn = wr.float().cpu().numpy(), bias.cpu().numpy()
    L = oracle.router_logits(nn, wrn, bn)
    bound = Hh.logit_error_bound(nn, wrn, bn, Hh.TENSOR_CORE_ROUTER_FACTOR)
    cert, near = Hh.check_routing(idx.cpu().numpy(), w.cpu().numpy(), L, cfg.k, bound)
    Hh.assert_few_near_ties(near, T, 0.15, "prefill router")
    # token -> expert lists: every slot once, counts sum to T*k, some experts carry hundreds of tokens
    off, srt, pos, act = B.bucketize(idx, cfg.E)
    off = off.cpu().numpy()
    assert off[-1] == T * cfg.k and np.array_equal(np.sort(srt.cpu().numpy()), np.arange(T * cfg.k))
    assert np.diff(off).max() > 300
    rows = np.linspace(0, T - 1, 48).astype(int)
    ox = Hh.OracleExperts(cfg, seed, DEV)
    res, _, _ = _oracle_layer(cfg, seed, nn[rows], None, ox)
    _check_layer_outputs(out[torch.from_numpy(rows).to(DEV)], res, wrn, bn, nn[rows])
