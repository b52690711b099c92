"""FP4 (E2M1) shelves against the oracle.

[P1] "step 4": the repacker gives the down projections a ladder of their own
that ends in MXFP4 on the rarest shelf.  The library stores an FP4 shelf as
4-bit codes of E2M1 values with a power-of-two block scale (format MOE_FP4),
for gate_up, down or both, and decodes it inside the same kernels as the
integer shelves.  Checked here:

- quantisation: codes and scales bit-identical to the oracle's MX conversion
  (ties, saturation, zero, clamped and subnormal scales included), and the
  dequantised fp32 / fp16 weights too;
- the expert FFN through the streaming path (exact products: 1e-5) and the
  tensor-core path (fp16-staged operands) on a layer with every kind of FP4
  shelf, the shared expert included;
- the fused layer (routing inside the FFN kernel at one token) and the
  persistent stack on the decode-size ladder layer, each on the oracle's
  inputs.
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


def _edge_rows(K):
    """Rows of hand-made blocks: every midpoint of the E2M1 grid, saturation,
    a zero block, a scale clamped at each end and a subnormal-range block."""
    w = np.zeros((6, K), np.float32)
    # amax 7.5: X = 1, so w / X is w itself; 7.5 and 6.5 saturate at 6
    mids = [7.5, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25, -0.75, -1.25, -1.75, -2.5, -3.5, -5.0, 6.5,
            0.2, 0.3, 0.7, 0.8, 1.2, 1.3, 1.7, 1.8, 2.4, 2.6, 3.4, 3.6, 4.9, 5.1, -0.0, 1e-3]
    w[0, :32] = mids
    w[1, :32] = np.asarray(mids, np.float32) * 2.0 ** -20     # same ratios at a small scale
    w[2, 32:64] = np.linspace(-1, 1, 32) * 2.0 ** 18          # X = 2^16 (largest)
    w[3, :32] = np.linspace(-1, 1, 32) * 2.0 ** -30           # X clamped at 2^-23: all codes 0 or small
    w[4, :32] = np.linspace(-1, 1, 32) * 2.0 ** 20            # X clamped at 2^16: saturates
    w[5, 32:64] = 1e-40                                       # fp32 subnormal block
    return w


@pytest.mark.parametrize("rows,K", [(6, 64), (37, 256), (64, 640), (300, 2048)])
def test_fp4_quantize_bytes_match_oracle(rows, K):
    g = torch.Generator(device=DEV).manual_seed(rows * K + 5)
    w = torch.randn(rows, K, generator=g, device=DEV) * 0.02
    w[:6] = torch.from_numpy(_edge_rows(K)).to(DEV)[:rows]
    qs, sc = B.quantize(w, B.FP4)
    assert qs.shape == (rows, K // 2) and B.packed_row_bytes(K, B.FP4) == K // 2
    oq, od = oracle.quantize_pack_fp4(w.cpu().numpy())
    assert np.array_equal(qs.cpu().numpy(), oq)
    assert np.array_equal(sc.cpu().numpy().view(np.uint16), od.view(np.uint16))
    f32, f16 = B.dequantize(qs, sc, K, B.FP4, f32=True, f16=True)
    ref = oracle.dequantize_fp4_f32(oq, od, K)
    assert np.array_equal(f32.cpu().numpy(), ref)
    with np.errstate(over="ignore"):  # the 2^16-scale rows overflow fp16 on both sides
        assert np.array_equal(f16.cpu().numpy().view(np.uint16), ref.astype(np.float16).view(np.uint16))


def test_fp4_hand_derived_codes_on_gpu():
    """The first edge row's codes, derived by hand from the E2M1 grid: values
    on a midpoint go to the even magnitude index, beyond 6 saturate, and a
    negative zero is stored as code 0."""
    w = _edge_rows(64)[:1]
    qs, sc = B.quantize(torch.from_numpy(w).to(DEV), B.FP4)
    codes = oracle.unpack_rows_fp4(qs.cpu().numpy(), 64)[0, :32].tolist()
    assert codes == [7, 0, 2, 2, 4, 4, 6, 6, 0, 10, 10, 12, 12, 14, 14, 7,
                     0, 1, 1, 2, 2, 3, 3, 4, 4, 5, 5, 6, 6, 7, 0, 0]
    assert float(sc.cpu().numpy().view(np.float16)[0, 0]) == 0.5  # d = X / 2, X = 1


@pytest.fixture(scope="module")
def tiny_fp4():
    cfg = inputs.TINY_FP4
    seed = 4321
    layer = B.build_layer(cfg, seed, DEV)
    torch.cuda.synchronize()
    return cfg, seed, layer


@pytest.mark.parametrize("mode", [B.FFN_GEMV, B.FFN_GEMM])
@pytest.mark.parametrize("T", [1, 8, 40])
def test_fp4_expert_ffn_matches_oracle(tiny_fp4, mode, T):
    cfg, seed, layer = tiny_fp4
    x = inputs.activations(T, cfg.H, seed=seed + T, device=DEV)
    ids = torch.stack([torch.randperm(cfg.E, generator=torch.Generator().manual_seed(50 + t))[: cfg.k]
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
    tol = 1e-5 if mode == B.FFN_GEMV else Hh.REL_L2
    assert Hh.rel_l2(y.cpu().numpy(), exp) < tol
    assert Hh.rel_l2(ysh.cpu().numpy(), esh) < tol
    # every FP4 shelf took part
    shelves = {next(i for i, (b, f, n) in enumerate(cfg.tier_ranges()) if f <= e < f + n) for e in idn.tolist()}
    assert shelves >= {1, 2, 3} or T == 1


def test_fp4_tensor_core_path_stages_exact_weights(tiny_fp4):
    """Tensor-core path, one token per slot: against the oracle's FFN on the
    fp16 weights the path stages (d * q is exact in fp16 for FP4 codes)."""
    cfg, seed, layer = tiny_fp4
    T = 12
    x = inputs.activations(T, cfg.H, seed=seed + 77, device=DEV)
    ids = torch.stack([torch.randperm(cfg.E, generator=torch.Generator().manual_seed(90 + t))[: cfg.k]
                       for t in range(T)]).to(torch.int32).to(DEV)
    off, srt, pos, act = B.bucketize(ids, cfg.E)
    y, ysh = B.expert_ffn(layer, x, cfg.k, off, srt, act, mode=B.FFN_GEMM)
    torch.cuda.synchronize()
    ox = Hh.OracleExperts(cfg, seed, DEV)
    xn = x.float().cpu().numpy()
    idn = ids.cpu().numpy().reshape(-1)

    def staged(e, rows):
        (gq, gs), (dq, ds) = ox.packed(e)
        gf, df = Hh.formats(ox.bits(e))
        return oracle.expert_ffn_f16_staged(rows, Hh.oracle_dequantize(gq, gs, gf, cfg.H).astype(np.float16),
                                            Hh.oracle_dequantize(dq, ds, df, cfg.I).astype(np.float16))
    exp = np.stack([staged(int(idn[s]), xn[s // cfg.k: s // cfg.k + 1])[0] for s in range(T * cfg.k)])
    got = y.cpu().numpy()
    assert np.max(np.abs(got - exp)) < 5e-4 * np.abs(exp).max()
    esh = staged(cfg.E, xn)
    assert np.max(np.abs(ysh.cpu().numpy() - esh)) < 5e-4 * np.abs(esh).max()


def _oracle_layer(cfg, seed, x):
    n = oracle.rms_norm(x).astype(np.float32)
    wr, bias = inputs.router(cfg, seed, DEV)
    wrn, bn = wr.float().cpu().numpy(), None if bias is None else bias.cpu().numpy()
    ox = Hh.OracleExperts(cfg, seed, DEV)
    idx, _ = oracle.select_topk(oracle.router_logits(n, wrn, bn), cfg.k)
    ox.prefetch(list(idx.reshape(-1)) + ([cfg.E] if cfg.shared else []))
    return oracle.moe_layer(n, wrn, bn, cfg.k, ox, ox.shared(), cfg.H, cfg.I, residual=x)


def _check_stream(x_next_gpu, x, res):
    """Layer output recovered from the new stream value, against the oracle's;
    the bf16 rounding of x + out adds half an ulp of x_next."""
    xg = Hh.to_np(x_next_gpu).astype(np.float64)
    out_g = xg - np.asarray(x, np.float64)
    out_o = np.asarray(res["out"], np.float64)
    half_ulp = np.abs(np.asarray(res["x_next"], np.float64)) * 2.0 ** -8
    assert np.all(np.abs(out_g - out_o) <= Hh.MAX_ABS + 2 * half_ulp), Hh.max_abs(out_g, out_o)
    excess = np.maximum(np.abs(out_g - out_o) - 2 * half_ulp, 0.0)
    assert np.linalg.norm(excess) / np.linalg.norm(out_o) < Hh.REL_L2


def _bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(DEV).to(torch.bfloat16)


@pytest.mark.parametrize("T", [1, 8])
def test_fp4_tiny_layer_forward_and_stack(tiny_fp4, T):
    """The fused layer (T = 1: the FFN kernel routes the token itself) and a
    one-layer stack launch, both against the oracle's layer."""
    cfg, seed, layer = tiny_fp4
    wr, bias = inputs.router(cfg, seed, DEV)
    x = inputs.activations(T, cfg.H, seed=seed + 300 + T, device=DEV).float().cpu().numpy()
    res = _oracle_layer(cfg, seed, x)
    xb = _bf16(x)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    _, x_next, _ = B.layer_forward(layer, wr, bias, B.rmsnorm(xb), cfg.k, residual=xb, mode=B.FFN_GEMV,
                                   status=status)
    got = B.stack_forward(B.Stack([layer], [(wr, bias)]), xb, cfg.k, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0, hex(status.item())
    _check_stream(x_next, x, res)
    _check_stream(got, x, res)


@pytest.fixture(scope="module")
def ladder():
    cfg = inputs.DECODE_LADDER
    layers = [B.build_layer(cfg, inputs.layer_seed(cfg, l), DEV) for l in range(2)]
    routers = [inputs.router(cfg, inputs.layer_seed(cfg, l), DEV) for l in range(2)]
    torch.cuda.synchronize()
    yield cfg, layers, routers
    del layers, routers
    torch.cuda.empty_cache()


@pytest.mark.parametrize("T", [1, 5])
def test_fp4_down_ladder_stack_on_oracle_inputs(ladder, T):
    """Decode-size layers whose rarest shelf has 3-bit gate_up and FP4 down
    ([P1] "step 4"'s ladder): one-layer stack launches on the oracle's stream,
    and the two layers in one launch against the per-layer launches."""
    cfg, layers, routers = ladder
    x = inputs.activations(T, cfg.H, seed=inputs.X_SEED + 40 + T, device=DEV).float().cpu().numpy()
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    x0 = _bf16(x)
    for l in range(2):
        res = _oracle_layer(cfg, inputs.layer_seed(cfg, l), x)
        got = B.stack_forward(B.Stack([layers[l]], [routers[l]]), _bf16(x), cfg.k, status=status)
        torch.cuda.synchronize()
        assert status.item() == 0, hex(status.item())
        _check_stream(got, x, res)
        x = res["x_next"].astype(np.float32)
    one = B.stack_forward(B.Stack(layers[:1], routers[:1]), x0, cfg.k)
    both = B.stack_forward(B.Stack(layers, routers), x0, cfg.k)
    again = B.stack_forward(B.Stack(layers[1:], routers[1:]), one, cfg.k)
    torch.cuda.synchronize()
    assert torch.equal(both, again)
