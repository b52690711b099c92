"""Host-side partitioning of the MoE layer over several GPUs.

Plain functions of sizes (no device work, no collectives), used by the
multi-process paths:

* Replicas: rank r of N takes the contiguous token range token_range(T, N, r)
  of a batch and runs every layer on its own tokens; the layer has no
  exchange step, so nothing crosses between ranks (the benchmark only
  max-reduces its timings).
* Expert parallel: rank r holds the contiguous range of expert ids
  expert_shards(...)[r], cut where the running total of the experts' bytes
  crosses r/N of the layer's total, so that each rank streams about the same
  number of weight bytes whatever the shelves' precisions (an 8-bit expert
  weighs about 2.7 times a 3-bit one).  The shared expert belongs to rank 0.
  Every rank routes every token (the router weights are small), runs the
  FFN of the slots whose experts it holds, and sums w_j * y_j over them (rank
  0 adds the shared expert): one sum all-reduce of these [T, H] partials gives
  each rank the layer output.
"""


def token_range(T, world, rank):
    """[start, stop) of rank's tokens: contiguous, sizes differ by at most one."""
    if not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside [0, {world})")
    return T * rank // world, T * (rank + 1) // world


def expert_bytes(H, I, bits, block=32):
    """Bytes of one expert's codes and fp16 block scales (gate_up [2I, H] and
    down [H, I], blocks of `block` weights along each row).  `bits` is one
    format for both or a (gate_up, down) pair; FP4 (5) stores 4-bit codes."""
    gu, dn = (bits, bits) if isinstance(bits, int) else bits
    code = {5: 4}
    weights = 2 * I * H + H * I
    return (2 * I * H * code.get(gu, gu) + H * I * code.get(dn, dn)) // 8 + (weights // block) * 2


def layer_expert_bytes(H, I, tiers):
    """Per-expert bytes of a layer whose shelves are (bits, first, count)."""
    out = {}
    for bits, first, count in tiers:
        for e in range(first, first + count):
            out[e] = expert_bytes(H, I, bits)
    E = len(out)
    if sorted(out) != list(range(E)):
        raise ValueError("shelves must cover expert ids 0..E-1 exactly once")
    return [out[e] for e in range(E)]


def expert_shards(nbytes, world):
    """Contiguous expert-id ranges [(first, count)] for `world` ranks: rank r
    starts at the first expert whose preceding bytes reach r/world of the
    total (integer comparison, so every rank computes the same cut)."""
    if world < 1:
        raise ValueError("world must be >= 1")
    total = sum(nbytes)
    starts, before, r = [0], 0, 1
    for e, b in enumerate(nbytes):
        while r < world and before * world >= r * total:
            starts.append(e)
            r += 1
        before += b
    while len(starts) < world:
        starts.append(len(nbytes))
    ends = starts[1:] + [len(nbytes)]
    return [(s, t - s) for s, t in zip(starts, ends)]


def shard_of(shards, e):
    """Rank holding expert e."""
    for r, (first, count) in enumerate(shards):
        if first <= e < first + count:
            return r
    raise ValueError(f"expert {e} is in no shard")
