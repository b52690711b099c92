"""Pins for the CPU oracle: it is checked here against things other than itself.

Each test compares the oracle with one of: a value the pages print, a
hand-derived worked example of the stated definition (tests/golden/), a closed
form, a library routine that computes the same mathematics a different way, or
brute force on tiny inputs.  All run on the CPU.
"""
import math
from fractions import Fraction

import numpy as np
import pytest
import scipy.special
import torch

import oracle
from mixed_precision_moe_router_b200 import inputs
from tests import golden


# ----------------------------------------------------------------------------
# byte accounting and block quantisation
# ----------------------------------------------------------------------------

def test_byte_accounting_matches_pages():
    hdr, _ = golden.load("byte_accounting.txt")
    bpw = oracle.bits_per_weight(hdr["bits"])
    assert bpw == hdr["bits_per_weight"]
    gb = hdr["params"] * bpw / 8 / 1e9
    assert abs(gb - hdr["gigabytes"]) < 0.005
    # the packed row size plus its scales gives the same cost per weight
    K = 2048
    per_row = oracle.packed_row_bytes(K, 4) + 2 * K // 32
    assert per_row * 8 / K == hdr["bits_per_weight"]
    assert oracle.packed_row_bytes(K, 3) * 8 / K == 3
    assert oracle.packed_row_bytes(K, 8) == K


def _block(ws):
    w = np.zeros((1, 32), np.float32)
    ws = ws if isinstance(ws, list) else [ws]
    w[0, : len(ws)] = np.asarray(ws, np.float32)
    return w


@pytest.mark.parametrize("case", golden.load("quant_examples.txt")[1], ids=lambda c: c["name"])
def test_quantize_hand_examples(case):
    w = _block(case["w"])
    q, d = oracle.quantize_rows(w, case["bits"])
    assert float(d[0, 0]) == case["d"]
    exp = case["q"] if isinstance(case["q"], list) else [case["q"]]
    assert q[0, : len(exp)].tolist() == exp
    assert not q[0, len(exp):].any()


@pytest.mark.parametrize("bits", [8, 4, 3])
def test_quantize_roundtrip_bound(bits):
    rng = np.random.default_rng(bits)
    w = (rng.standard_normal((64, 256)) * 0.02).astype(np.float32)
    w[3, :32] *= 1e-4  # a block with a tiny scale
    w[5, 32:64] = 0.0  # an all-zero block
    packed, d = oracle.quantize_pack(w, bits)
    back = oracle.dequantize_f32(packed, d, bits, 256)
    blocks = w.reshape(64, 8, 32)
    amax = np.abs(blocks).max(axis=2, keepdims=True).astype(np.float64)
    dd = d.astype(np.float64)[..., None]
    err = np.abs(back.reshape(64, 8, 32) - blocks.astype(np.float64))
    assert np.all(err <= dd / 2 + amax * 2.0 ** -11 + 1e-30)
    assert np.all(back.reshape(64, 8, 32)[5, 1] == 0)
    # every code stays within +-qmax and the block maximum reaches +-qmax
    q, _ = oracle.quantize_rows(w, bits)
    qmax = oracle.QMAX[bits]
    assert np.abs(q).max() <= qmax
    top = np.abs(q.reshape(64, 8, 32)).max(axis=2)
    # (only for normal fp16 scales: a subnormal scale is rounded coarsely)
    normal = d.astype(np.float64) >= 2.0 ** -14
    assert np.all(top[normal] == qmax)


def test_quantize_uses_division_not_reciprocal():
    """Find weights where w/d and w*(1/d) round to different codes; the definition
    (fp32 division, half away from zero) decides, and the oracle must follow it."""
    d = np.float32(np.float16(0.0999755859375))
    found = 0
    for n in range(1, 127):
        target = np.float32((n + 0.5) * float(d))
        for cand in (np.nextafter(target, np.float32(0)), target, np.nextafter(target, np.float32(1e9))):
            cand = np.float32(cand)
            by_div = np.float32(cand / d)
            by_rcp = np.float32(cand * np.float32(np.float32(1) / d))
            if by_div == by_rcp:
                continue
            # block: the maximum pins d to exactly fp16(0.1) * 127 / 127
            w = np.zeros((1, 32), np.float32)
            w[0, 0] = np.float32(127) * d
            w[0, 1] = cand
            q, dq = oracle.quantize_rows(w, 8)
            assert np.float32(dq[0, 0]) == d
            r = Fraction(float(by_div))
            expect = int(math.floor(r + Fraction(1, 2)))  # r > 0: half away from zero
            assert q[0, 1] == min(expect, 127)
            found += 1
    assert found > 0


# ----------------------------------------------------------------------------
# packing
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("case", golden.load("pack_examples.txt")[1], ids=lambda c: c["name"])
def test_pack_hand_examples(case):
    q = np.zeros((1, 32), np.int64)
    qs = case["q"] if isinstance(case["q"], list) else [case["q"]]
    q[0, : len(qs)] = qs
    packed = oracle.pack_rows(q, case["bits"])
    expect = [int(str(b), 16) for b in case["bytes"]]
    assert packed[0].tolist() == expect
    assert oracle.unpack_rows(packed, case["bits"], 32).tolist() == q.tolist()


@pytest.mark.parametrize("bits", [8, 4, 3])
def test_pack_roundtrip_all_codes(bits):
    qmax = oracle.QMAX[bits]
    rng = np.random.default_rng(10 + bits)
    q = rng.integers(-qmax, qmax + 1, size=(7, 256))
    q[0, : 2 * qmax + 1] = np.arange(-qmax, qmax + 1)
    packed = oracle.pack_rows(q, bits)
    assert packed.shape == (7, oracle.packed_row_bytes(256, bits))
    assert np.array_equal(oracle.unpack_rows(packed, bits, 256), q)


def test_dequant_is_exact_product():
    rng = np.random.default_rng(3)
    for bits in (8, 4, 3):
        w = (rng.standard_normal((4, 64)) * 0.02).astype(np.float32)
        q, d = oracle.quantize_rows(w, bits)
        packed = oracle.pack_rows(q, bits)
        f32 = oracle.dequantize_f32(packed, d, bits, 64)
        for r in range(4):
            for i in range(64):
                exact = Fraction(float(d[r, i // 32])) * int(q[r, i])
                assert Fraction(float(f32[r, i])) == exact
        f16 = oracle.dequantize_f16(packed, d, bits, 64)
        ref = torch.from_numpy(f32).to(torch.float16).numpy()  # library RNE fp32 -> fp16
        assert np.array_equal(f16.view(np.uint16), ref.view(np.uint16))


# ----------------------------------------------------------------------------
# router / top-k / weights
# ----------------------------------------------------------------------------

def _bf16_values(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(*shape, generator=g) * scale).to(torch.bfloat16).float().numpy()


def test_router_logits_exact_on_bf16_inputs():
    x = _bf16_values((3, 64), 1)
    w = _bf16_values((5, 64), 2, 0.02)
    b = np.array([0.5, -0.25, 0.0, 1.0, -2.0], np.float32)
    L = oracle.router_logits(x, w, b)
    for t in range(3):
        for e in range(5):
            exact = sum(Fraction(float(x[t, h])) * Fraction(float(w[e, h])) for h in range(64))
            exact += Fraction(float(b[e]))
            assert abs(Fraction(L[t, e]) - exact) <= abs(exact) * Fraction(1, 2 ** 50) + Fraction(1, 2 ** 80)


def test_topk_brute_force():
    rng = np.random.default_rng(5)
    for trial in range(20):
        E = int(rng.integers(2, 40))
        k = int(rng.integers(1, E + 1))
        L = np.round(rng.standard_normal((4, E)), 1)  # coarse values -> many ties
        idx, w = oracle.select_topk(L, k)
        for t in range(4):
            ranked = sorted(range(E), key=lambda e: (-L[t, e], e))[:k]
            assert idx[t].tolist() == ranked
            z = [math.exp(L[t, e]) for e in ranked]
            assert np.allclose(w[t], [v / math.fsum(z) for v in z], rtol=1e-13, atol=0)


def test_topk_ties_go_to_lower_id():
    L = np.array([[1.0, 3.0, 3.0, 2.0, 3.0, 0.0]])
    idx, w = oracle.select_topk(L, 4)
    assert idx[0].tolist() == [1, 2, 4, 3]
    assert np.allclose(w[0, :3], w[0, 0])


def test_topk_full_k_is_softmax():
    rng = np.random.default_rng(6)
    L = rng.standard_normal((3, 16)) * 3
    idx, w = oracle.select_topk(L, 16)
    p = scipy.special.softmax(L, axis=1)
    for t in range(3):
        assert np.allclose(w[t], p[t, idx[t]], rtol=1e-12, atol=0)


def test_topk_weights_renormalised_softmax():
    rng = np.random.default_rng(7)
    L = rng.standard_normal((5, 32))
    idx, w = oracle.select_topk(L, 6)
    p = scipy.special.softmax(L, axis=1)
    for t in range(5):
        sel = p[t, idx[t]]
        assert np.allclose(w[t], sel / sel.sum(), rtol=1e-12)
        assert abs(w[t].sum() - 1) < 1e-12
        assert np.all(np.diff(w[t]) <= 0)
    # a constant shift of all logits changes nothing
    idx2, w2 = oracle.select_topk(L + 123.0, 6)
    assert np.array_equal(idx, idx2) and np.allclose(w, w2, rtol=1e-12)


def test_topk_margin():
    L = np.array([[5.0, 4.0, 3.5, 3.4, 0.0]])
    assert oracle.topk_margin(L, 2)[0] == pytest.approx(0.5)
    assert oracle.topk_margin(L, 3)[0] == pytest.approx(0.1)


# ----------------------------------------------------------------------------
# bucketize
# ----------------------------------------------------------------------------

def test_bucketize_brute_force():
    rng = np.random.default_rng(8)
    for trial in range(30):
        E = int(rng.integers(1, 20))
        k = int(rng.integers(1, E + 1))
        T = int(rng.integers(0, 12))
        idx = np.array([rng.permutation(E)[:k] for _ in range(T)], np.int32).reshape(T, k)
        off, srt, pos = oracle.bucketize(idx, E)
        pairs = sorted((int(e), s) for s, e in enumerate(idx.reshape(-1)))
        assert srt.tolist() == [s for _, s in pairs]
        for e in range(E):
            assert off[e + 1] - off[e] == sum(1 for p in pairs if p[0] == e)
        assert off[0] == 0 and off[E] == T * k
        assert np.array_equal(srt[pos], np.arange(T * k))


# ----------------------------------------------------------------------------
# FFN, combine, rounding
# ----------------------------------------------------------------------------

def test_silu_closed_form():
    g = np.array([-30.0, -1.0, 0.0, 1.0, 2.5, 30.0])
    assert np.allclose(oracle.silu(g), g * scipy.special.expit(g), rtol=1e-15, atol=1e-300)
    assert oracle.silu(np.array([0.0]))[0] == 0.0
    assert oracle.silu(np.array([1.0]))[0] == pytest.approx(0.7310585786300049, rel=1e-15)


def test_ffn_identity_weights_closed_form():
    """With W_gate = c*I, W_up = I, W_down = I the layer is y = silu(c x) * x
    elementwise: a swapped gate/up, a transposed operand or a missing factor fails."""
    n = 8
    c = 1.7
    wgu = np.concatenate([c * np.eye(n), np.eye(n)])
    x = np.linspace(-3, 3, 2 * n).reshape(2, n)
    y = oracle.expert_ffn(x, wgu, np.eye(n))
    assert np.allclose(y, c * x * scipy.special.expit(c * x) * x, rtol=1e-14, atol=1e-15)
    # a permutation as W_down permutes the output
    P = np.eye(n)[::-1]
    assert np.allclose(oracle.expert_ffn(x, wgu, P), y[:, ::-1], rtol=1e-14)


def test_round_bf16_matches_library_on_fp32_values():
    rng = np.random.default_rng(9)
    v = np.concatenate([rng.standard_normal(5000) * 10.0 ** rng.integers(-30, 30, 5000),
                        [0.0, -0.0, 1e-40, -3e-39, 3.0e38]]).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.bfloat16).float().numpy().astype(np.float64)
    assert np.array_equal(oracle.round_bf16(v.astype(np.float64)), ref)


def test_round_bf16_ties_and_single_rounding():
    one = 1.0
    assert oracle.round_bf16(np.array([one + 2 ** -8]))[0] == 1.0  # tie -> even
    assert oracle.round_bf16(np.array([one + 3 * 2 ** -8]))[0] == 1 + 2 ** -6
    # just above the tie: a double rounding through fp32 would land on the tie and go
    # to even (1.0); the correct single rounding goes up
    v = one + 2 ** -8 + 2 ** -40
    assert oracle.round_bf16(np.array([v]))[0] == 1 + 2 ** -7


def test_combine_single_slot_is_rounding():
    rng = np.random.default_rng(10)
    y = rng.standard_normal((3, 16))
    out = oracle.combine(y, None, np.ones((3, 1)))
    assert np.array_equal(out, oracle.round_bf16(y))
    out2, nxt, nrm = oracle.combine(y, np.zeros((3, 16)), np.ones((3, 1)), residual=np.ones((3, 16)))
    assert np.array_equal(out2, out)
    assert np.array_equal(nxt, oracle.round_bf16(1.0 + out))
    assert np.array_equal(nrm, oracle.rms_norm(nxt))


def test_rms_norm_closed_forms_and_library():
    # a constant row normalises to ones (up to eps); sign and scale are preserved
    c = np.full((2, 64), 3.0)
    assert np.allclose(oracle.rms_norm(c), 1.0, atol=2 ** -8)
    v = np.array([[3.0, -4.0] * 8])          # rms = sqrt(12.5)
    assert np.allclose(oracle.rms_norm(v), oracle.round_bf16(v / np.sqrt(12.5 + oracle.NORM_EPS)), rtol=0)
    rng = np.random.default_rng(11)
    x = rng.standard_normal((5, 256)) * 7
    ref = torch.nn.functional.rms_norm(torch.from_numpy(x), (256,), eps=oracle.NORM_EPS).numpy()
    assert np.allclose(oracle.rms_norm(x), oracle.round_bf16(ref), rtol=0, atol=0) or \
        np.max(np.abs(oracle.rms_norm(x) - ref)) <= 2 ** -8 * np.max(np.abs(ref))
    assert np.array_equal(oracle.rms_norm(x * 2 ** 5), oracle.rms_norm(x))  # exact scale invariance


# ----------------------------------------------------------------------------
# the whole layer: brute-force dense evaluation and tier-split invariance
# ----------------------------------------------------------------------------

def _tiny_layer(shelf_split=None):
    cfg = inputs.TINY
    seed = inputs.layer_seed(cfg)
    x = inputs.activations(8, cfg.H, seed=seed).float().numpy()
    wr, bias = inputs.router(cfg, seed)
    wr = wr.float().numpy()
    src = [tuple(t.numpy() for t in inputs.expert_source(cfg, seed, e)) for e in range(cfg.E + 1)]
    ranges = shelf_split or cfg.tier_ranges()
    shelves = [oracle.build_shelf(bits, first, src[first:first + n]) for bits, first, n in ranges]
    shared = oracle.build_shelf(8, cfg.E, [src[cfg.E]])
    return cfg, x, wr, bias, shelves, shared


def test_layer_brute_force_dense():
    """Every expert evaluated for every token, masked by the top-k and weighted,
    must equal the sparse routed evaluation."""
    cfg, x, wr, bias, shelves, shared = _tiny_layer()
    res = oracle.moe_layer(x, wr, bias, cfg.k, oracle.shelves_lookup(shelves, cfg.H, cfg.I),
                           shared.weights(cfg.E, cfg.H, cfg.I), cfg.H, cfg.I)
    T = x.shape[0]
    # brute force: independent loops over (token, expert)
    logits = np.zeros((T, cfg.E))
    for t in range(T):
        for e in range(cfg.E):
            logits[t, e] = math.fsum(float(a) * float(b) for a, b in zip(x[t], wr[e]))
    dense = np.zeros((T, cfg.E, cfg.H))
    for e in range(cfg.E):
        wgu, wdn = oracle.shelf_of(shelves, e).weights(e, cfg.H, cfg.I)
        for t in range(T):
            g = wgu[: cfg.I].astype(np.float64) @ x[t]
            u = wgu[cfg.I:].astype(np.float64) @ x[t]
            h = g * scipy.special.expit(g) * u
            dense[t, e] = wdn.astype(np.float64) @ h
    wgu, wdn = shared.weights(cfg.E, cfg.H, cfg.I)
    total = np.zeros((T, cfg.H))
    for t in range(T):
        order = sorted(range(cfg.E), key=lambda e: (-logits[t, e], e))[: cfg.k]
        p = scipy.special.softmax(logits[t])
        mask = np.zeros(cfg.E)
        mask[order] = p[order] / p[order].sum()
        g = wgu[: cfg.I].astype(np.float64) @ x[t]
        u = wgu[cfg.I:].astype(np.float64) @ x[t]
        total[t] = mask @ dense[t] + wdn.astype(np.float64) @ (g * scipy.special.expit(g) * u)
        assert res["topk_idx"][t].tolist() == order
    pre = np.einsum("tj,tjh->th", res["topk_w"], res["y_slots"].reshape(T, cfg.k, -1)) + res["y_shared"]
    assert np.allclose(pre, total, rtol=1e-12, atol=1e-14)
    assert np.array_equal(res["out"], oracle.round_bf16(total)) or \
        np.max(np.abs(res["out"] - oracle.round_bf16(total))) <= 2 ** -8 * np.abs(total).max()
    assert np.allclose(res["topk_w"].sum(axis=1), 1.0, atol=1e-12)


def test_layer_tier_split_invariance():
    """The same 8-bit weights in one table or split over three tables give the same
    output: each shelf computes only its ids and the results add up."""
    cfg = inputs.TINY
    one = _tiny_layer(shelf_split=[(8, 0, 16)])
    three = _tiny_layer(shelf_split=[(8, 0, 5), (8, 5, 2), (8, 7, 9)])
    r1 = oracle.moe_layer(*one[1:4], cfg.k, oracle.shelves_lookup(one[4], cfg.H, cfg.I),
                          one[5].weights(cfg.E, cfg.H, cfg.I), cfg.H, cfg.I)
    r3 = oracle.moe_layer(*three[1:4], cfg.k, oracle.shelves_lookup(three[4], cfg.H, cfg.I),
                          three[5].weights(cfg.E, cfg.H, cfg.I), cfg.H, cfg.I)
    assert np.array_equal(r1["out"], r3["out"])


# ----------------------------------------------------------------------------
# the synthetic workload reproduces the pages' routing skew
# ----------------------------------------------------------------------------

def test_zipf_routing_share():
    hdr, _ = golden.load("routing_skew.txt")
    cfg = inputs.DECODE
    x = inputs.activations(4096, cfg.H, seed=inputs.X_SEED).float().numpy()
    wr, bias = inputs.router(cfg, inputs.layer_seed(cfg, 0))
    L = oracle.router_logits(x, wr.float().numpy(), bias.numpy())
    idx, _ = oracle.select_topk(L, cfg.k)
    counts = np.bincount(idx.reshape(-1), minlength=cfg.E)
    top = int(cfg.E * hdr["top_fraction"])
    share = np.sort(counts)[::-1][:top].sum() / counts.sum()
    assert abs(share - hdr["token_share"]) < hdr["tolerance"]
    # ids are popularity ranks: the 8-bit tier (ids < 128) carries that share
    assert abs(counts[:128].sum() / counts.sum() - hdr["token_share"]) < hdr["tolerance"] + 0.01


def test_draft_batch_overlap():
    """Correlated drafts share about 60% of the base token's top-10 experts."""
    cfg = inputs.DECODE
    wr, bias = inputs.router(cfg, inputs.layer_seed(cfg, 0))
    overlaps = []
    for s in range(8):
        x = inputs.correlated_activations(5, cfg.H, seed=100 + s).float().numpy()
        idx, _ = oracle.select_topk(oracle.router_logits(x, wr.float().numpy(), bias.numpy()), cfg.k)
        base = set(idx[0].tolist())
        overlaps += [len(base & set(idx[t].tolist())) / cfg.k for t in range(1, 5)]
    assert 0.45 < float(np.mean(overlaps)) < 0.75


def test_round_f16_matches_library():
    rng = np.random.default_rng(12)
    v = np.concatenate([rng.standard_normal(4000) * 10.0 ** rng.integers(-9, 5, 4000),
                        [0.0, 65504.0, 65520.0, 2.0 ** -24, 3 * 2.0 ** -26]]).astype(np.float32)
    ref = v.astype(np.float16).astype(np.float64)  # numpy: RNE fp32 -> fp16
    assert np.array_equal(oracle.round_f16(v.astype(np.float64)), ref)


def test_f16_staged_ffn_equals_exact_when_staging_is_lossless():
    """With integer weights (d = 1) and small integer activations every staged
    value is exactly representable, so the staged FFN equals the fp64 one up to
    the rounding of h, which is exact too when silu(g)*u is representable."""
    rng = np.random.default_rng(13)
    n, I = 64, 32
    wgu = rng.integers(-3, 4, size=(2 * I, n)).astype(np.float64)
    wdn = rng.integers(-3, 4, size=(n, I)).astype(np.float64)
    x = rng.integers(-2, 3, size=(5, n)).astype(np.float64)
    y_exact = oracle.expert_ffn(x, wgu, wdn)
    y_staged = oracle.expert_ffn_f16_staged(x, wgu, wdn)
    h = oracle.silu(x @ wgu[:I].T) * (x @ wgu[I:].T)
    assert np.allclose(y_staged, oracle.round_f16(h) @ wdn.T, rtol=0, atol=0)
    assert np.max(np.abs(y_staged - y_exact)) <= np.abs(h).max() * 2.0 ** -11 * np.abs(wdn).sum(axis=1).max()


def test_f16_staged_ffn_rounds_x_to_f16():
    """Activations that are not fp16 values: the staged FFN must round x to the
    nearest fp16 (ties to even) before the products.  With W_gate = 2I, W_up = I and
    W_down = I every product is exact, so y = fp16(silu(2X) * X) where X is the
    fp16 rounding of x, written out here by hand from the fp16 grid (step 2^-10 in
    [1, 2), 2^-9 in [2, 4), 2^-14 in [1/16, 1/8))."""
    n = 8
    x = np.array([[1 + 2.0 ** -12,       # quarter step above 1 -> 1
                   1 + 3 * 2.0 ** -12,   # three quarters of a step -> 1 + 2^-10
                   1 + 2.0 ** -11,       # tie between 1 and 1 + 2^-10 -> even: 1
                   1 + 3 * 2.0 ** -11,   # tie between 1 + 2^-10 and 1 + 2^-9 -> even: 1 + 2^-9
                   -(2 + 2.0 ** -11),    # quarter step beyond -2 -> -2
                   0.1,                  # 1638.4 * 2^-14 -> 1638 * 2^-14
                   3.14159,              # 1608.49 * 2^-9 -> 1608 * 2^-9
                   -0.75]])              # an fp16 value: unchanged
    X = np.array([[1.0, 1 + 2.0 ** -10, 1.0, 1 + 2.0 ** -9, -2.0, 1638 * 2.0 ** -14, 1608 * 2.0 ** -9, -0.75]])
    wgu = np.concatenate([2.0 * np.eye(n), np.eye(n)])
    y = oracle.expert_ffn_f16_staged(x, wgu, np.eye(n))
    expect = oracle.round_f16(oracle.silu(2.0 * X) * X)
    assert np.array_equal(y, expect)
    # the pin has teeth: skipping the rounding of x changes six of the eight outputs
    unrounded = oracle.round_f16(oracle.silu(2.0 * x) * x)
    assert np.sum(unrounded != expect) == 6


def _stack_layer_identity(n, c):
    """One routed expert (E = 1, k = 1) whose FFN is y = silu(c x) * x elementwise,
    and no shared expert: the layer is out = bf16(silu(c n) * n)."""
    wgu = np.concatenate([c * np.eye(n), np.eye(n)])
    wr = np.zeros((1, n), np.float32)
    return (wr, None, lambda e: (wgu, np.eye(n)), None)


def test_moe_stack_closed_form_recursion():
    """A stack of elementwise layers has a closed form: n_l = rms_norm(x_l),
    out_l = bf16(silu(c_l n_l) n_l), x_{l+1} = bf16(x_l + out_l).  Feeding x instead
    of n to a layer, or adding out to n instead of x, breaks it."""
    n = 16
    rng = np.random.default_rng(21)
    x0 = oracle.round_bf16(rng.standard_normal((3, n)) * 4.0)
    cs = [0.5, 2.0, 1.0, 4.0]
    res = oracle.moe_stack(x0, [_stack_layer_identity(n, c) for c in cs], 1, n, n)
    x = x0.copy()
    for l, c in enumerate(cs):
        nl = oracle.rms_norm(x)
        out = oracle.round_bf16(oracle.silu(c * nl) * nl)
        assert np.array_equal(res[l]["n"], nl)
        assert np.array_equal(res[l]["x"], x)
        assert np.array_equal(res[l]["out"], out)
        x = oracle.round_bf16(x + out)
        assert np.array_equal(res[l]["x_next"], x)
        assert np.array_equal(res[l]["n_next"], oracle.rms_norm(x))


def test_moe_stack_zero_experts_keep_the_stream():
    """With all-zero expert weights every layer adds 0: the stream stays x_0 exactly
    and each layer reads rms_norm(x_0)."""
    cfg = inputs.TINY
    rng = np.random.default_rng(22)
    x0 = oracle.round_bf16(rng.standard_normal((4, cfg.H)) * 3.0)
    wr = _bf16_values((cfg.E, cfg.H), 23, 0.02)
    zero = (np.zeros((2 * cfg.I, cfg.H)), np.zeros((cfg.H, cfg.I)))
    layer = (wr, None, lambda e: zero, zero)
    res = oracle.moe_stack(x0, [layer] * 3, cfg.k, cfg.H, cfg.I)
    for r in res:
        assert not np.any(r["out"])
        assert np.array_equal(r["x"], x0) and np.array_equal(r["x_next"], x0)
        assert np.array_equal(r["n"], oracle.rms_norm(x0))


def test_moe_stack_layers_read_the_normalised_stream():
    """The first layer's output does not change when x_0 is scaled by 2^5 (the
    normalised stream is exactly scale invariant), while the layer evaluated on the
    raw stream does change."""
    cfg, x, wr, bias, shelves, shared = _tiny_layer()
    lookup = oracle.shelves_lookup(shelves, cfg.H, cfg.I)
    sw = shared.weights(cfg.E, cfg.H, cfg.I)
    layer = (wr, bias, lookup, sw)
    a = oracle.moe_stack(x, [layer], cfg.k, cfg.H, cfg.I)[0]
    b = oracle.moe_stack(x * 32.0, [layer], cfg.k, cfg.H, cfg.I)[0]
    assert np.array_equal(a["out"], b["out"])
    assert np.array_equal(b["x_next"], oracle.round_bf16(32.0 * x + b["out"]))
    raw = oracle.moe_layer(x * 32.0, wr, bias, cfg.k, lookup, sw, cfg.H, cfg.I)
    assert not np.array_equal(raw["out"], a["out"])


# ---------------------------------------------------------------------------
# FP4 (E2M1) shelf: codes and scales derived by hand from the format (OCP MX:
# shared scale X = 2^(floor(log2 amax) - 2), nearest E2M1 value, ties to the
# even code, saturation at 6; stored as d = X / 2 and q = 2 * value)
# ---------------------------------------------------------------------------

def test_fp4_hand_derived_block():
    # amax = 3.0: floor(log2 3) = 1, X = 2^-1, v = 2w, d = 0.25
    w = np.zeros((1, 32), np.float32)
    w[0, :10] = [3.0, 0.125, 0.375, -1.25, 2.5, 0.7, -0.1, 1.6, 2.9, -3.0]
    # v:          6    0.25   0.75   -2.5   5    1.4   -0.2  3.2  5.8  -6
    # nearest:    6    0|0.5  0.5|1  2|3    4|6  1.5   0     3    6    -6
    #                  tie->0 tie->1 tie->2 tie->4
    codes, d = oracle.quantize_rows_fp4(w)
    assert d.tolist() == [[0.25]]
    assert codes[0, :10].tolist() == [7, 0, 2, 12, 6, 3, 0, 5, 7, 15]
    assert codes[0, 10:].tolist() == [0] * 22
    assert oracle.fp4_integers(codes[0, :10]).tolist() == [12, 0, 2, -4, 8, 3, 0, 6, 12, -12]
    back = oracle.dequantize_fp4_f32(oracle.pack_rows_fp4(codes), d, 32)[0, :10]
    assert back.tolist() == [3.0, 0.0, 0.5, -1.0, 2.0, 0.75, 0.0, 1.5, 3.0, -3.0]
    # the nibble order of the 4-bit shelf: weight 2m low, 2m+1 high
    assert oracle.pack_rows_fp4(codes)[0, :2].tolist() == [7 | (0 << 4), 2 | (12 << 4)]


def test_fp4_edge_blocks():
    w = np.zeros((4, 32), np.float32)
    w[0, 5] = 4.0            # amax a power of two: X = 1, d = 0.5, code 6
    w[1, 3] = 2.0 ** -30     # below fp16's range: d = 2^-24, X = 2^-23, v = 2^-7 -> 0
    w[3, :] = -7.9           # every weight saturates: amax/X = 7.9 / 1 -> 6
    codes, d = oracle.quantize_rows_fp4(w)
    assert float(d[0, 0]) == 0.5 and codes[0, 5] == 6 and codes[0].sum() == 6
    assert float(d[1, 0]) == 2.0 ** -24 and codes[1].sum() == 0
    assert float(d[2, 0]) == 0.0 and codes[2].sum() == 0          # a zero block
    assert float(d[3, 0]) == 0.5 and set(codes[3].tolist()) == {15}
    assert oracle.dequantize_fp4_f32(oracle.pack_rows_fp4(codes), d, 32)[3].tolist() == [-6.0] * 32


def test_fp4_codes_are_the_nearest_of_all_sixteen():
    """Brute force: at the block's scale, every weight's code gives the value
    nearest to it among all 16 codes (ties: the even magnitude index, and 0
    rather than -0), and the round trip is within half a grid step."""
    rng = np.random.default_rng(11)
    w = (rng.standard_normal((16, 64)) * rng.choice([1e-3, 0.02, 1.0, 50.0], size=(16, 1))).astype(np.float32)
    w[0, :4] = [0.0, -0.0, 1e-9, -1e-9]
    codes, d = oracle.quantize_rows_fp4(w)
    grid = np.array([(1 if c < 8 else -1) * oracle.FP4_VALUES[c & 7] for c in range(16)])
    for r in range(w.shape[0]):
        for i in range(w.shape[1]):
            X = 2.0 * float(d[r, i // 32])
            v = float(w[r, i]) / X
            dist = np.abs(grid - v)
            best = [c for c in range(16) if dist[c] == dist.min()]
            best = [c for c in best if c != 8] or best           # 0 rather than -0
            even = [c for c in best if (c & 7) % 2 == 0]
            assert codes[r, i] == (even or best)[0], (r, i, v, best)
            assert abs(v - grid[codes[r, i]]) <= (1.0 if abs(v) <= 6 else 2.0)


def test_fp4_scale_puts_the_block_max_in_the_top_binade():
    """The MX scale of a block with E2M1 elements (largest binade [4, 6]) is
    the power of two X with amax / X in [4, 8): the block's largest weight
    lands in the elements' top binade or just above it (saturating to 6).  A
    scale exponent one off in either direction fails this."""
    rng = np.random.default_rng(5)
    w = (rng.standard_normal((64, 256)) * 10.0 ** rng.uniform(-4, 3, size=(64, 1))).astype(np.float32)
    _, d = oracle.quantize_rows_fp4(w)
    amax = np.abs(w.reshape(64, 8, 32)).max(axis=2).astype(np.float64)
    X = 2.0 * d.astype(np.float64)
    ratio = amax / X
    assert np.all((ratio >= 4.0) & (ratio < 8.0)), ratio.min()
    assert np.all(np.log2(X) == np.round(np.log2(X)))  # powers of two


def test_fp4_sign_symmetry_and_power_of_two_equivariance():
    """Negating a block flips the sign bit of every nonzero code and keeps
    the scale; scaling it by 2^j keeps the codes and scales d by 2^j (away
    from the scale's clamps)."""
    rng = np.random.default_rng(9)
    w = (rng.standard_normal((8, 128)) * 0.05).astype(np.float32)
    c, d = oracle.quantize_rows_fp4(w)
    cn, dn = oracle.quantize_rows_fp4(-w)
    assert np.array_equal(dn, d)
    nz = (c & 7) != 0
    assert np.array_equal(cn[nz], c[nz] ^ 8) and np.array_equal(cn[~nz], c[~nz])
    for j in (-3, 1, 5):
        cj, dj = oracle.quantize_rows_fp4((w * np.float32(2.0 ** j)).astype(np.float32))
        assert np.array_equal(cj, c)
        assert np.array_equal(dj.astype(np.float64), d.astype(np.float64) * 2.0 ** j)
