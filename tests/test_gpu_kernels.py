"""GPU parity: each hot-path call through the C ABI against the CPU oracle.

Integer and byte results (codes, scales, dequantised values, top-k ids, token
lists) must match bit for bit; floating-point outputs within stated bounds.
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


# ----------------------------------------------------------------------------
# quantise / dequantise: bit-exact
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("bits", [8, 4, 3])
@pytest.mark.parametrize("rows,K", [(37, 128), (64, 256), (130, 512), (5, 2048), (3, 640)])
def test_quantize_bytes_match_oracle(bits, rows, K):
    g = torch.Generator(device=DEV).manual_seed(rows * K + bits)
    w = torch.randn(rows, K, generator=g, device=DEV) * 0.02
    w[0, :32] = 0.0                       # zero block
    w[1, :32] *= 1e-4                     # subnormal-scale block
    w[2, 32:64] = torch.linspace(-3, 3, 32, device=DEV)  # values on half steps
    qs, sc = B.quantize(w, bits)
    oq, od = oracle.quantize_pack(w.cpu().numpy(), bits)
    assert np.array_equal(qs.cpu().numpy(), oq)
    assert np.array_equal(sc.cpu().numpy().view(np.uint16), od.view(np.uint16))
    f32, f16 = B.dequantize(qs, sc, K, bits, f32=True, f16=True)
    assert np.array_equal(f32.cpu().numpy(), oracle.dequantize_f32(oq, od, bits, K))
    assert np.array_equal(f16.cpu().numpy().view(np.uint16),
                          oracle.dequantize_f16(oq, od, bits, K).view(np.uint16))


def test_quantize_golden_cases_on_gpu():
    from tests import golden
    for case in golden.load("quant_examples.txt")[1]:
        w = np.zeros((1, 64), np.float32)
        ws = case["w"] if isinstance(case["w"], list) else [case["w"]]
        w[0, : len(ws)] = ws
        qs, sc = B.quantize(torch.from_numpy(w).to(DEV), case["bits"])
        assert float(np.float16(sc.cpu().numpy().view(np.float16)[0, 0])) == case["d"], case["name"]
        q = oracle.unpack_rows(qs.cpu().numpy(), case["bits"], 64)
        exp = case["q"] if isinstance(case["q"], list) else [case["q"]]
        assert q[0, : len(exp)].tolist() == exp, case["name"]


# ----------------------------------------------------------------------------
# top-k on given logits: bit-exact ids (same fp32 inputs on both sides)
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("T,E,k", [(1, 512, 10), (33, 512, 10), (8, 16, 2), (5, 24, 24), (6, 40, 32), (70, 1024, 32),
                                   (3, 1, 1), (0, 16, 2)])
def test_topk_softmax_matches_oracle(T, E, k):
    g = torch.Generator(device=DEV).manual_seed(T * 131 + E)
    L = torch.randn(T, E, generator=g, device=DEV)
    if T > 2 and E > 8:
        L[1, 3] = L[1, 5] = L[1, 7] = L[1].max() + 1.0      # a three-way tie at the top
        L[2] = torch.round(L[2] * 4) / 4                       # many ties
    idx, w = B.topk_softmax(L.contiguous(), k)
    if T == 0:
        return
    oi, ow = oracle.select_topk(L.cpu().numpy().astype(np.float64), k)
    assert np.array_equal(idx.cpu().numpy(), oi)
    assert np.max(np.abs(w.cpu().numpy() - ow)) < 1e-6


# ----------------------------------------------------------------------------
# router: logits within the fp32 bound, routing certified-exact
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("cfg,T", [(inputs.TINY, 8), (inputs.DECODE, 1), (inputs.DECODE, 40), (inputs.DECODE, 300)])
def test_router_topk_matches_oracle(cfg, T):
    seed = inputs.layer_seed(cfg)
    x = inputs.activations(T, cfg.H, seed=seed + 17, device=DEV)
    wr, bias = inputs.router(cfg, seed, DEV)
    idx, w, logits = B.router_topk(x, wr, bias, cfg.k, want_logits=True)
    xn, wn = x.float().cpu().numpy(), wr.float().cpu().numpy()
    bn = None if bias is None else bias.cpu().numpy()
    L = oracle.router_logits(xn, wn, bn)
    tensor = T >= 64  # logits on the tensor cores
    bound = Hh.logit_error_bound(xn, wn, bn, Hh.TENSOR_CORE_ROUTER_FACTOR if tensor else 1.0)
    assert np.all(np.abs(logits.cpu().numpy() - L) <= bound)
    cert, near = Hh.check_routing(idx.cpu().numpy(), w.cpu().numpy(), L, cfg.k, bound)
    assert cert + near == T
    Hh.assert_few_near_ties(near, T, 0.15 if tensor else 0.1, f"router T={T}")
    # the ids come from the GPU's own logits by the exact top-k rule
    oi, _ = oracle.select_topk(logits.cpu().numpy().astype(np.float64), cfg.k)
    assert np.array_equal(idx.cpu().numpy(), oi)


# ----------------------------------------------------------------------------
# bucketize: bit-exact
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("T,E,k", [(1, 512, 10), (8, 16, 2), (4096, 512, 10), (1000, 1024, 32), (7, 1, 1),
                                   (0, 16, 2), (3, 4, 4), (2000, 64, 1)])
def test_bucketize_matches_oracle(T, E, k):
    rng = np.random.default_rng(T + E + k)
    ids = np.array([rng.permutation(E)[:k] for _ in range(T)], np.int32).reshape(T, k)
    if T > 100:  # Zipf-like skew: many tokens on few experts
        ids = np.stack([np.sort(rng.choice(E, size=k, replace=False, p=np.arange(E, 0, -1) / (E * (E + 1) / 2)))
                        for _ in range(T)]).astype(np.int32)
    t_ids = torch.from_numpy(ids).to(DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    off, srt, pos, act = B.bucketize(t_ids, E, status)
    o_off, o_srt, o_pos = oracle.bucketize(ids, E)
    assert np.array_equal(off.cpu().numpy(), o_off)
    assert np.array_equal(srt.cpu().numpy(), o_srt)
    assert np.array_equal(pos.cpu().numpy(), o_pos)
    counts = np.diff(o_off)
    act = act.cpu().numpy()
    assert act[0] == np.count_nonzero(counts)
    assert np.array_equal(act[1: 1 + act[0]], np.nonzero(counts)[0])
    assert status.item() == 0


def test_bucketize_rejects_bad_ids_without_addressing_them():
    """[P1] the unsigned-ternary bug: a -1 "skip" must never become an address."""
    ids = np.array([[3, -1], [2, 3], [16, 0], [2147483647, -2147483648]], np.int32)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    off, srt, pos, act = B.bucketize(torch.from_numpy(ids).to(DEV), 16, status)
    assert status.item() & B.STATUS_BAD_EXPERT_ID
    good = [(int(e), s) for s, e in enumerate(ids.reshape(-1)) if 0 <= e < 16]
    off = off.cpu().numpy()
    assert off[16] == len(good)
    assert srt.cpu().numpy()[: len(good)].tolist() == [s for _, s in sorted(good)]
    p = pos.cpu().numpy()
    for s, e in enumerate(ids.reshape(-1)):
        if not 0 <= e < 16:
            assert p[s] == -1


# ----------------------------------------------------------------------------
# combine: bf16 outputs
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("T,k,H,shared,res", [(8, 2, 256, True, False), (5, 10, 2048, True, True),
                                              (33, 3, 128, False, True)])
def test_combine_matches_oracle(T, k, H, shared, res):
    g = torch.Generator(device=DEV).manual_seed(T * k + H)
    y = torch.randn(T * k, H, generator=g, device=DEV)
    ysh = torch.randn(T, H, generator=g, device=DEV) if shared else None
    w = torch.softmax(torch.randn(T, k, generator=g, device=DEV), dim=1).contiguous()
    r = torch.randn(T, H, generator=g, device=DEV).to(torch.bfloat16) if res else None
    got = B.combine(y, ysh, w, residual=r)
    out = got[0] if res else got
    exp = oracle.combine(y.cpu().numpy(), None if ysh is None else ysh.cpu().numpy(), w.cpu().numpy(),
                         residual=None if r is None else r.float().cpu().numpy())
    e_out = exp[0] if res else exp
    o = out.float().cpu().numpy()
    # fp32 vs fp64 sums before one bf16 rounding: identical or one bf16 step apart
    ulp = np.maximum(2.0 ** (np.floor(np.log2(np.maximum(np.abs(e_out), 1e-30))) - 7), 2.0 ** -133)
    assert np.all(np.abs(o - e_out) <= ulp)
    assert np.mean(o != e_out) < 0.01
    if res:
        xn = got[1].float().cpu().numpy()
        e_x = exp[1]
        # the residual add is exact: where out agrees, x_next agrees
        same = o == e_out
        assert np.array_equal(xn[same], e_x[same])
        nn = got[2].float().cpu().numpy()
        nulp = np.maximum(2.0 ** (np.floor(np.log2(np.maximum(np.abs(exp[2]), 1e-30))) - 7), 2.0 ** -133)
        assert np.all(np.abs(nn - exp[2]) <= 2 * nulp)
        assert np.mean(nn != exp[2]) < 0.02


@pytest.mark.parametrize("T,H", [(1, 2048), (7, 256), (300, 128)])
def test_rmsnorm_matches_oracle(T, H):
    g = torch.Generator(device=DEV).manual_seed(T + H)
    x = (torch.randn(T, H, generator=g, device=DEV) * 3).to(torch.bfloat16)
    n = B.rmsnorm(x).float().cpu().numpy()
    e = oracle.rms_norm(x.float().cpu().numpy())
    ulp = np.maximum(2.0 ** (np.floor(np.log2(np.maximum(np.abs(e), 1e-30))) - 7), 2.0 ** -133)
    assert np.all(np.abs(n - e) <= ulp)
    assert np.mean(n != e) < 0.01


# ----------------------------------------------------------------------------
# FFN and the whole layer on the tiny configuration
# ----------------------------------------------------------------------------

def _tiny():
    cfg = inputs.TINY
    seed = inputs.layer_seed(cfg)
    layer = B.build_layer(cfg, seed, DEV)
    return cfg, seed, layer


@pytest.mark.parametrize("mode", [B.FFN_GEMV, B.FFN_GEMM])
def test_ffn_tiny_matches_oracle(mode):
    cfg, seed, layer = _tiny()
    T = 8
    x = inputs.activations(T, cfg.H, seed=seed, device=DEV)
    ids = torch.stack([torch.randperm(cfg.E, generator=torch.Generator().manual_seed(t))[: cfg.k]
                       for t in range(T)]).to(torch.int32).to(DEV)
    off, srt, pos, act = B.bucketize(ids, cfg.E)
    y, ysh = B.expert_ffn(layer, x, cfg.k, off, srt, act, mode=mode)
    ox = Hh.OracleExperts(cfg, seed, DEV)
    xn = x.float().cpu().numpy()
    idn = ids.cpu().numpy()
    exp = np.stack([oracle.expert_ffn(xn[s // cfg.k: s // cfg.k + 1], *ox(int(idn.reshape(-1)[s])))[0]
                    for s in range(T * cfg.k)])
    tol = 1e-5 if mode == B.FFN_GEMV else 2e-3
    assert Hh.rel_l2(y.cpu().numpy(), exp) < tol
    esh = oracle.expert_ffn(xn, *ox.shared())
    assert Hh.rel_l2(ysh.cpu().numpy(), esh) < tol


def _layer_check(cfg, seed, layer, x, mode, ox=None):
    wr, bias = inputs.router(cfg, seed, DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    out, xn_gpu, nn_gpu = B.layer_forward(layer, wr, bias, x, cfg.k, residual=x, mode=mode, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    ox = ox or Hh.OracleExperts(cfg, seed, DEV)
    xn, wn = x.float().cpu().numpy(), wr.float().cpu().numpy()
    bn = None if bias is None else bias.cpu().numpy()
    res = oracle.moe_layer(xn, wn, bn, cfg.k, ox, ox.shared(), cfg.H, cfg.I, residual=xn)
    o = out.float().cpu().numpy()
    assert Hh.rel_l2(o, res["out"]) < Hh.REL_L2, Hh.rel_l2(o, res["out"])
    assert Hh.max_abs(o, res["out"]) < Hh.MAX_ABS
    # routing as the library computed it inside the layer
    idx, w, _ = B.router_topk(x, wr, bias, cfg.k)
    bound = Hh.logit_error_bound(xn, wn, bn)
    Hh.check_routing(idx.cpu().numpy(), w.cpu().numpy(), res["logits"], cfg.k, bound)
    return out, xn_gpu, res


@pytest.mark.parametrize("mode", [B.FFN_GEMV, B.FFN_AUTO, B.FFN_GEMM])
def test_layer_tiny_matches_oracle(mode):
    cfg, seed, layer = _tiny()
    x = inputs.activations(8, cfg.H, seed=seed, device=DEV)
    _layer_check(cfg, seed, layer, x, mode)


def test_layer_tiny_tier_split_is_bit_identical():
    """[P1] the shelf results simply add up: the same 8-bit weights in one table
    or in three tables give bit-identical layer output."""
    cfg = inputs.TINY
    seed = inputs.layer_seed(cfg)
    one = B.build_layer(cfg, seed, DEV, tier_ranges=[(8, 0, 16)])
    three = B.build_layer(cfg, seed, DEV, tier_ranges=[(8, 0, 5), (8, 5, 2), (8, 7, 9)])
    x = inputs.activations(8, cfg.H, seed=seed, device=DEV)
    wr, bias = inputs.router(cfg, seed, DEV)
    for mode in (B.FFN_GEMV, B.FFN_GEMM, B.FFN_AUTO):
        a = B.layer_forward(one, wr, bias, x, cfg.k, mode=mode)
        b = B.layer_forward(three, wr, bias, x, cfg.k, mode=mode)
        assert torch.equal(a, b), mode


def test_layer_tiny_edge_token_counts():
    cfg, seed, layer = _tiny()
    wr, bias = inputs.router(cfg, seed, DEV)
    for T in (1, 2, 3, 5, 17):
        x = inputs.activations(T, cfg.H, seed=seed + T, device=DEV)
        _layer_check(cfg, seed, layer, x, B.FFN_GEMV)
    # T = 0 is a no-op
    out = B.layer_forward(layer, wr, bias, torch.empty(0, cfg.H, dtype=torch.bfloat16, device=DEV), cfg.k)
    assert out.shape == (0, cfg.H)


def test_gemv_batch_invariance():
    """A token's GEMV-path output does not depend on the other tokens in the batch."""
    cfg, seed, layer = _tiny()
    wr, bias = inputs.router(cfg, seed, DEV)
    x = inputs.activations(9, cfg.H, seed=seed + 3, device=DEV)
    full = B.layer_forward(layer, wr, bias, x, cfg.k, mode=B.FFN_GEMV)
    for t in (0, 4, 8):
        one = B.layer_forward(layer, wr, bias, x[t:t + 1].contiguous(), cfg.k, mode=B.FFN_GEMV)
        assert torch.equal(one[0], full[t])


@pytest.mark.parametrize("T", [1, 13, 40, 300])
def test_gemm_path_matches_f16_staged_oracle(T):
    """The tensor-core path against the oracle's fp16-staged arithmetic: the same
    staged operands with exact accumulation, so only fp32 accumulation order
    separates them (tight bound), for token counts from 1 to several M tiles."""
    cfg, seed, layer = _tiny()
    x = inputs.activations(T, cfg.H, seed=seed + 100 + T, device=DEV)
    g = torch.Generator().manual_seed(T)
    ids = torch.stack([torch.randperm(cfg.E, generator=g)[: cfg.k] for _ in range(T)]).to(torch.int32).to(DEV)
    off, srt, pos, act = B.bucketize(ids, cfg.E)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    y, ysh = B.expert_ffn(layer, x, cfg.k, off, srt, act, mode=B.FFN_GEMM, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    ox = Hh.OracleExperts(cfg, seed, DEV)
    xn = x.float().cpu().numpy()
    idn = ids.cpu().numpy().reshape(-1)

    def staged(e, rows):
        (gq, gs), (dq, ds) = ox.packed(e)
        b = ox.bits(e)
        return oracle.expert_ffn_f16_staged(rows, oracle.dequantize_f16(gq, gs, b, cfg.H),
                                            oracle.dequantize_f16(dq, ds, b, cfg.I))
    exp = np.stack([staged(int(idn[s]), xn[s // cfg.k: s // cfg.k + 1])[0] for s in range(T * cfg.k)])
    got = y.cpu().numpy()
    scale = np.abs(exp).max()
    assert np.max(np.abs(got - exp)) < 5e-4 * scale, np.max(np.abs(got - exp)) / scale
    esh = staged(cfg.E, xn)
    assert np.max(np.abs(ysh.cpu().numpy() - esh)) < 5e-4 * np.abs(esh).max()
