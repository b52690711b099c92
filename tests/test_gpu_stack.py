"""The persistent stack kernel (moe_stack_forward) against the CPU oracle.

A launch of one layer runs on the oracle's own layer inputs, so each layer is
compared on identical inputs; a launch of several layers is compared with the
free-running oracle stack (loosely: legal rounding differences accumulate)
and with the per-layer GPU path.
"""
import numpy as np
import pytest
import torch

import oracle
from mixed_precision_moe_router_b200 import binding as B
from mixed_precision_moe_router_b200 import inputs
from tests import helpers as Hh

pytestmark = pytest.mark.gpu
DEV = "cuda"
N_LAYERS = 6


def _bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(DEV).to(torch.bfloat16)


def _oracle_layer(cfg, seed, x):
    """The oracle's layer on its own residual stream x (bf16 values)."""
    n = oracle.rms_norm(x).astype(np.float32)
    wr, bias = inputs.router(cfg, seed, DEV)
    wrn, bn = wr.float().cpu().numpy(), None if bias is None else bias.cpu().numpy()
    ox = Hh.OracleExperts(cfg, seed, DEV)
    idx, _ = oracle.select_topk(oracle.router_logits(n, wrn, bn), cfg.k)
    ox.prefetch(list(idx.reshape(-1)) + ([cfg.E] if cfg.shared else []))
    return oracle.moe_layer(n, wrn, bn, cfg.k, ox, ox.shared(), cfg.H, cfg.I, residual=x)


def _check_stream(x_next_gpu, x, res):
    """The layer's output recovered from the GPU's new stream value against the
    oracle's: the only extra error over the layer tolerance is the final bf16
    rounding of x + out (half an ulp of x_next)."""
    xg = Hh.to_np(x_next_gpu).astype(np.float64)
    out_g = xg - np.asarray(x, np.float64)
    out_o = np.asarray(res["out"], np.float64)
    half_ulp = np.abs(np.asarray(res["x_next"], np.float64)) * 2.0 ** -8
    assert np.all(np.abs(out_g - out_o) <= Hh.MAX_ABS + 2 * half_ulp), Hh.max_abs(out_g, out_o)
    excess = np.maximum(np.abs(out_g - out_o) - 2 * half_ulp, 0.0)
    assert np.linalg.norm(excess) / np.linalg.norm(out_o) < Hh.REL_L2


@pytest.fixture(scope="module")
def decode_layers():
    cfg = inputs.DECODE
    layers = [B.build_layer(cfg, inputs.layer_seed(cfg, l), DEV) for l in range(N_LAYERS)]
    routers = [inputs.router(cfg, inputs.layer_seed(cfg, l), DEV) for l in range(N_LAYERS)]
    torch.cuda.synchronize()
    yield cfg, layers, routers
    del layers, routers
    torch.cuda.empty_cache()


@pytest.mark.parametrize("T", [1, 5, 8])
def test_stack_layer_on_oracle_inputs(decode_layers, T):
    """One-layer launches, each on the oracle's stream entering that layer."""
    cfg, layers, routers = decode_layers
    x = inputs.activations(T, cfg.H, seed=inputs.X_SEED + 3 * T, device=DEV).float().cpu().numpy()
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    for l in range(3):
        seed = inputs.layer_seed(cfg, l)
        res = _oracle_layer(cfg, seed, x)
        st = B.Stack([layers[l]], [routers[l]])
        norm = torch.empty(T, cfg.H, dtype=torch.bfloat16, device=DEV)
        got = B.stack_forward(st, _bf16(x), cfg.k, out_norm=norm, status=status)
        torch.cuda.synchronize()
        assert status.item() == 0, hex(status.item())
        _check_stream(got, x, res)
        # the normalised output is the next layer's input n, one bf16 ulp at most apart
        assert Hh.max_abs(Hh.to_np(norm), oracle.rms_norm(Hh.to_np(got))) <= 2.0 ** -7 * 8
        x = res["x_next"].astype(np.float32)


def test_stack_multi_layer_matches_layer_path_and_oracle(decode_layers):
    """Several layers in one launch: the stream at every layer boundary stays
    close to the per-layer GPU path (rmsnorm + moe_layer_forward, GEMV mode) and
    to the free-running oracle stack."""
    cfg, layers, routers = decode_layers
    T = 1
    x0 = inputs.activations(T, cfg.H, seed=inputs.X_SEED, device=DEV)
    st = B.Stack(layers, routers)
    xl = torch.empty(N_LAYERS + 1, T, cfg.H, dtype=torch.bfloat16, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    out = B.stack_forward(st, x0, cfg.k, x_layers=xl, status=status)
    g_x, g_n = x0.clone(), B.rmsnorm(x0)
    for l in range(N_LAYERS):
        wr, bias = routers[l]
        _, g_x, g_n = B.layer_forward(layers[l], wr, bias, g_n, cfg.k, residual=g_x, mode=B.FFN_GEMV)
        assert Hh.rel_l2(Hh.to_np(xl[l + 1]), Hh.to_np(g_x)) < 5e-3, l
    torch.cuda.synchronize()
    assert status.item() == 0
    assert torch.equal(xl[0], x0) and torch.equal(xl[N_LAYERS], out)
    x = x0.float().cpu().numpy()
    for l in range(N_LAYERS):
        x = _oracle_layer(cfg, inputs.layer_seed(cfg, l), x)["x_next"].astype(np.float32)
    assert Hh.rel_l2(Hh.to_np(out), x) < 2e-2


def test_stack_batch_invariant(decode_layers):
    """Each token of an 8-token launch gets exactly its 1-token result."""
    cfg, layers, routers = decode_layers
    st = B.Stack(layers[:4], routers[:4])
    xs = inputs.activations(8, cfg.H, seed=inputs.X_SEED + 1, device=DEV)
    all8 = B.stack_forward(st, xs, cfg.k)
    for t in range(8):
        one = B.stack_forward(st, xs[t:t + 1].contiguous(), cfg.k)
        assert torch.equal(all8[t:t + 1], one), t


def test_stack_tiny_configuration():
    """The tiny layer shape (H=256, I=128, 16 experts, top-2) through four
    layers, every layer on the oracle's inputs."""
    cfg = inputs.TINY
    x = inputs.activations(8, cfg.H, seed=5, device=DEV).float().cpu().numpy()
    for l in range(4):
        seed = inputs.layer_seed(cfg, l) if l else inputs.layer_seed(cfg)
        layer = B.build_layer(cfg, seed, DEV)
        router = inputs.router(cfg, seed, DEV)
        res = _oracle_layer(cfg, seed, x)
        got = B.stack_forward(B.Stack([layer], [router]), _bf16(x), cfg.k)
        torch.cuda.synchronize()
        _check_stream(got, x, res)
        x = res["x_next"].astype(np.float32)


def test_one_token_top_k_ties_resolve_to_the_lowest_id(decode_layers):
    """The one-token routing inside the kernels ranks 32-logit chunks first,
    then their candidates.  Three experts in different chunks are given the
    router row and bias of the k-th choice, so that they tie exactly for the
    last place: the lowest id must take it ([P1] "step 4": the router picks
    the best k; ties go to the lower id).  The stack and the fused layer path
    are checked against the oracle's layer, which a wrong pick fails (another
    expert's output)."""
    cfg, layers, routers = decode_layers
    k, E = cfg.k, cfg.E
    wr0, bias0 = routers[0]
    seed = inputs.layer_seed(cfg, 0)
    for s in range(20):  # a token whose k-th logit is clear of its neighbours
        x = inputs.activations(1, cfg.H, seed=inputs.X_SEED + 700 + s, device=DEV)
        n = B.rmsnorm(x)
        idx, _, lg = B.router_topk(n, wr0, bias0, k, want_logits=True)
        lg = lg[0].double().cpu()
        srt = torch.sort(lg, descending=True).values
        gap = float(min(srt[k - 2] - srt[k - 1], srt[k - 1] - srt[k]))
        if gap > 1e-3 * float(srt[k - 1].abs()) + 1e-4:
            break
    else:
        pytest.skip("no token with a clear k-th logit")
    chosen = set(idx[0].tolist())
    ek = int(idx[0, k - 1])
    others = [e for e in range(E) if e not in chosen and e // 32 != ek // 32]
    ea, eb = others[0], others[-1]  # the lowest and highest ids outside ek's chunk
    win = min(ea, ek, eb)
    wr = wr0.clone()
    wr[ea] = wr0[ek]
    wr[eb] = wr0[ek]
    bias = None
    if bias0 is not None:
        bias = bias0.clone()
        bias[ea] = bias0[ek]
        bias[eb] = bias0[ek]
    xn = x.float().cpu().numpy()
    nn = oracle.rms_norm(xn).astype(np.float32)
    wrn, bn = wr.float().cpu().numpy(), None if bias is None else bias.cpu().numpy()
    oidx, _ = oracle.select_topk(oracle.router_logits(nn, wrn, bn), k)
    tied = {ea, ek, eb}
    assert win in oidx[0] and not (tied - {win}) & set(oidx[0].tolist())  # the tie as built
    ox = Hh.OracleExperts(cfg, seed, DEV)
    ox.prefetch(list(oidx.reshape(-1)) + [E])
    res = oracle.moe_layer(nn, wrn, bn, k, ox, ox.shared(), cfg.H, cfg.I, residual=xn)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    got = B.stack_forward(B.Stack([layers[0]], [(wr, bias)]), x, k, status=status)
    _, x_next, _ = B.layer_forward(layers[0], wr, bias, n, k, residual=x, mode=B.FFN_GEMV, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    _check_stream(got, xn, res)
    _check_stream(x_next, xn, res)
