"""Partitioning over several GPUs, checked on CPU with two gloo ranks.

The ranks compute with the oracle (no GPU), so what is checked is the
partitioning itself: the expert-parallel split (each rank's byte-balanced
range of expert ids, the shared expert on rank 0, one sum all-reduce of the
[T, H] partials) reproduces the whole layer, and so do the replicas' token
ranges gathered back in order; the timing reduction is the max over ranks.
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from mixed_precision_moe_router_b200 import ep, inputs

WORLD = 2
TOKENS = 8


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _tiny_weights(cfg, seed):
    """Every expert's dequantised fp32 weights (the oracle's quantiser), the
    shared expert at index E."""
    W = {}
    tiers = cfg.tier_ranges()
    for e in range(cfg.E + 1):
        wgu, wdn = inputs.expert_source(cfg, seed, e)
        bits = cfg.shared_bits if e == cfg.E else next(b for b, f, n in tiers if f <= e < f + n)
        gq, gs = oracle.quantize_pack(wgu.numpy(), bits)
        dq, ds = oracle.quantize_pack(wdn.numpy(), bits)
        W[e] = (oracle.dequantize_f32(gq, gs, bits, cfg.H), oracle.dequantize_f32(dq, ds, bits, cfg.I))
    return W


def _partial(res, k):
    """sum_j w_j y_j (+ y_shared) before combine's bf16 rounding."""
    T = res["topk_w"].shape[0]
    s = np.einsum("tj,tjh->th", res["topk_w"], res["y_slots"].reshape(T, k, -1))
    return s if res["y_shared"] is None else s + res["y_shared"]


def _worker(rank, port, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=WORLD, timeout=datetime.timedelta(seconds=60))
    try:
        cfg = inputs.TINY
        seed = inputs.layer_seed(cfg)
        W = _tiny_weights(cfg, seed)
        wr, bias = inputs.router(cfg, seed)
        wrn, bn = wr.float().numpy(), None if bias is None else bias.numpy()
        x = inputs.activations(TOKENS, cfg.H, seed=inputs.X_SEED + 3).float().numpy()
        n = oracle.rms_norm(x).astype(np.float32)
        full = oracle.moe_layer(n, wrn, bn, cfg.k, lambda e: W[e], W[cfg.E], cfg.H, cfg.I)

        # expert parallel: this rank's experts only (the others contribute zero)
        shards = ep.expert_shards(ep.layer_expert_bytes(cfg.H, cfg.I, cfg.tier_ranges()), WORLD)
        first, count = shards[rank]
        zero = (np.zeros((2 * cfg.I, cfg.H), np.float32), np.zeros((cfg.H, cfg.I), np.float32))
        res = oracle.moe_layer(n, wrn, bn, cfg.k, lambda e: W[e] if first <= e < first + count else zero,
                               W[cfg.E] if rank == 0 else None, cfg.H, cfg.I)
        local_slots = int(np.sum((full["topk_idx"] >= first) & (full["topk_idx"] < first + count)))
        part = torch.from_numpy(_partial(res, cfg.k))
        dist.all_reduce(part)  # sum over ranks
        ep_err = float(np.max(np.abs(part.numpy() - _partial(full, cfg.k))))
        ep_out_equal = bool(np.array_equal(oracle.round_bf16(part.numpy()), full["out"]))

        # replicas: this rank's tokens, gathered back in rank order
        lo, hi = ep.token_range(TOKENS, WORLD, rank)
        mine = oracle.moe_layer(n[lo:hi], wrn, bn, cfg.k, lambda e: W[e], W[cfg.E], cfg.H, cfg.I)["out"]
        gathered = [None] * WORLD
        dist.all_gather_object(gathered, (lo, hi, mine))
        rep = np.concatenate([o for _, _, o in sorted(gathered, key=lambda g: g[0])])
        rep_equal = bool(np.array_equal(rep, full["out"]))

        # the benchmark's timing reduction
        t = torch.tensor([float(rank + 1)], dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        out_q.put((rank, shards, local_slots, ep_err, ep_out_equal, rep_equal, float(t.item())))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_expert_parallel_and_replicas():
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, port, q)) for r in range(WORLD)]
    for p in procs:
        p.start()
    try:
        results = sorted(q.get(timeout=240) for _ in range(WORLD))
    finally:
        for p in procs:
            p.join(timeout=60)
    assert all(p.exitcode == 0 for p in procs)
    shards = results[0][1]
    assert all(r[1] == shards for r in results)  # every rank cut the same shards
    assert all(r[2] > 0 for r in results), "each rank should own some chosen slot"
    assert sum(r[2] for r in results) == TOKENS * inputs.TINY.k
    for rank, _, _, ep_err, ep_out_equal, rep_equal, tmax in results:
        assert ep_err < 1e-9, (rank, ep_err)
        assert ep_out_equal and rep_equal, rank
        assert tmax == WORLD


@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_expert_shards_cover_and_balance(world):
    cfg = inputs.DECODE
    nbytes = ep.layer_expert_bytes(cfg.H, cfg.I, cfg.tier_ranges())
    shards = ep.expert_shards(nbytes, world)
    assert len(shards) == world
    assert shards[0][0] == 0 and sum(c for _, c in shards) == cfg.E
    assert all(shards[r][0] + shards[r][1] == shards[r + 1][0] for r in range(world - 1))
    total = sum(nbytes)
    for first, count in shards:  # within one (largest) expert of an equal share
        assert abs(sum(nbytes[first:first + count]) - total / world) <= max(nbytes)
    assert [ep.shard_of(shards, e) for e in (0, cfg.E - 1)] == [0, world - 1]


def test_expert_bytes_match_the_shelf_format():
    # 8-bit: one byte per weight; 4-bit: half; 3-bit: 3/8; plus an fp16 scale per 32
    H, I = 2048, 512
    w = 3 * H * I
    assert ep.expert_bytes(H, I, 8) == w + w // 16
    assert ep.expert_bytes(H, I, 4) == w // 2 + w // 16
    assert ep.expert_bytes(H, I, 3) == 3 * w // 8 + w // 16
    # FP4 stores 4-bit codes; a (gate_up, down) pair counts each table at its own width
    assert ep.expert_bytes(H, I, 5) == ep.expert_bytes(H, I, 4)
    assert ep.expert_bytes(H, I, (3, 5)) == (2 * H * I * 3 + H * I * 4) // 8 + w // 16
    assert ep.expert_bytes(H, I, (8, 8)) == ep.expert_bytes(H, I, 8)


@pytest.mark.parametrize("T,world", [(1, 1), (8, 2), (5, 4), (3, 8), (4096, 8)])
def test_token_ranges_partition_the_batch(T, world):
    ranges = [ep.token_range(T, world, r) for r in range(world)]
    assert ranges[0][0] == 0 and ranges[-1][1] == T
    assert all(ranges[r][1] == ranges[r + 1][0] for r in range(world - 1))
    sizes = [b - a for a, b in ranges]
    assert max(sizes) - min(sizes) <= 1
