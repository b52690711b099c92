"""The tier planner ([P1] "step 4": a greedy planner fills a byte budget,
each byte going to the expert where it removes the most expected error), on
CPU with synthetic frequencies and error models."""
import itertools

import numpy as np
import pytest

from mixed_precision_moe_router_b200 import ep, planner

H, I = 2048, 512
NB = {b: ep.expert_bytes(H, I, b) for b in (3, 4, 8)}
# squared error of absmax block-32 quantisation scales as (amax / qmax)^2
QMAX = {3: 3, 4: 7, 8: 127}


def _err(E, scale=None):
    scale = scale or [1.0] * E
    return [{b: scale[e] / QMAX[b] ** 2 for b in (3, 4, 8)} for e in range(E)]


def _zipf(E, alpha=0.8):
    f = 1.0 / np.arange(1, E + 1) ** alpha
    return list(f / f.sum())


def test_budget_bounds():
    E = 64
    f, err = _zipf(E), _err(E)
    lo, hi = E * NB[3], E * NB[8]
    assert planner.plan_tiers(f, err, NB, lo) == [3] * E
    assert planner.plan_tiers(f, err, NB, hi) == [8] * E
    with pytest.raises(ValueError):
        planner.plan_tiers(f, err, NB, lo - 1)
    for frac in (0.1, 0.3, 0.5, 0.8):
        B = lo + frac * (hi - lo)
        plan = planner.plan_tiers(f, err, NB, B)
        assert planner.plan_bytes(plan, NB) <= B
        # maximal: no single upgrade left that would still fit
        spare = B - planner.plan_bytes(plan, NB)
        steps = [NB[4] - NB[3] if b == 3 else NB[8] - NB[4] for b in plan if b != 8]
        assert not steps or min(steps) > spare


def test_error_falls_with_budget_and_shelves_follow_popularity():
    E = 512
    f, err = _zipf(E), _err(E)
    prev = None
    for frac in np.linspace(0.0, 1.0, 11):
        B = E * NB[3] + frac * E * (NB[8] - NB[3])
        plan = planner.plan_tiers(f, err, NB, B)
        e = planner.expected_error(plan, f, err)
        assert prev is None or e <= prev * (1 + 1e-12)
        prev = e
        # equal error models, falling frequency: precision falls with the id
        assert all(a >= b for a, b in zip(plan, plan[1:]))
        order, shelves = planner.shelves_from_bits(plan)
        assert order == list(range(E))
        assert sum(n for _, _, n in shelves) == E and shelves[0][1] == 0


def test_a_hard_expert_is_upgraded_out_of_popularity_order():
    E = 16
    scale = [1.0] * E
    scale[11] = 400.0  # outlier weights: a much larger error at every width
    f, err = _zipf(E), _err(E, scale)
    plan = planner.plan_tiers(f, err, NB, E * NB[3] + (NB[8] - NB[3]) + 4 * (NB[4] - NB[3]))
    assert plan[11] == 8
    order, shelves = planner.shelves_from_bits(plan)
    assert sorted(order) == list(range(E)) and order[0] == 11
    firsts = [s[1] for s in shelves]
    assert firsts == sorted(firsts) and [s[0] for s in shelves] == sorted({*plan}, reverse=True)
    for b, first, n in shelves:  # each shelf holds exactly the experts planned at its width
        assert all(plan[order[i]] == b for i in range(first, first + n))


def test_against_every_contiguous_layout_of_the_same_size():
    """On a small Zipf case the greedy plan does at least as well as 95 % of
    the 8/4/3 splits by popularity at each split's own budget, and never more
    than 20 % worse than any: greedy is not an exact knapsack solver (an
    upgrade that no longer fits leaves its bytes to smaller ones), the rule
    [P1] states."""
    E = 24
    f, err = _zipf(E, 1.1), _err(E)
    ratios = []
    for n8, n4 in itertools.product(range(E + 1), range(E + 1)):
        if n8 + n4 > E:
            continue
        split = [8] * n8 + [4] * n4 + [3] * (E - n8 - n4)
        plan = planner.plan_tiers(f, err, NB, planner.plan_bytes(split, NB))
        ratios.append(planner.expected_error(plan, f, err) / planner.expected_error(split, f, err))
    ratios = np.array(ratios)
    assert np.mean(ratios <= 1 + 1e-9) >= 0.95 and ratios.max() <= 1.2


def test_beats_the_configured_split_at_its_size():
    """At the byte size of the decode configuration's shelves (128 x 8-bit,
    192 x 4-bit, 192 x 3-bit) the planned layout's expected error is lower."""
    E = 512
    f, err = _zipf(E, 0.8), _err(E)
    split = [8] * 128 + [4] * 192 + [3] * 192
    plan = planner.plan_tiers(f, err, NB, planner.plan_bytes(split, NB))
    assert planner.plan_bytes(plan, NB) <= planner.plan_bytes(split, NB)
    assert planner.expected_error(plan, f, err) < planner.expected_error(split, f, err)


def test_format_pair_levels_plan_the_down_ladder():
    """Levels that are (gate_up, down) format pairs, as in the pages' repacker
    ladder (3-bit gate_up with FP4 down, 4/4, 8/8): the plan fits the
    budget, is maximal, falls with the id under equal error models, and its
    shelves are format-pair ranges in the library's order."""
    FP4 = 5
    levels = ((3, FP4), (4, 4), (8, 8))
    nb = {lv: ep.expert_bytes(H, I, lv) for lv in levels}
    assert nb[(3, FP4)] < nb[(4, 4)] < nb[(8, 8)]
    qerr = {3: 1 / 9, 4: 1 / 49, 8: 1 / 127 ** 2, FP4: 1 / 40}  # per weight, in units of amax^2
    E = 96
    f = _zipf(E)
    err = [{lv: 2 * qerr[lv[0]] + qerr[lv[1]] for lv in levels} for _ in range(E)]
    lo, hi = E * nb[(3, FP4)], E * nb[(8, 8)]
    B = lo + 0.4 * (hi - lo)
    plan = planner.plan_tiers(f, err, nb, B, bits=levels)
    assert planner.plan_bytes(plan, nb) <= B
    spare = B - planner.plan_bytes(plan, nb)
    steps = [nb[levels[levels.index(lv) + 1]] - nb[lv] for lv in plan if lv != levels[-1]]
    assert not steps or min(steps) > spare
    rank = [levels.index(lv) for lv in plan]
    assert all(a >= b for a, b in zip(rank, rank[1:]))
    order, shelves = planner.shelves_from_bits(plan)
    assert order == list(range(E))
    assert [lv for lv, _, _ in shelves] == sorted({lv for lv in plan}, reverse=True)
    assert sum(n for _, _, n in shelves) == E
    # an unpopular expert with a large error model is lifted and renumbered first
    err[E - 1] = {lv: 50 * v for lv, v in err[E - 1].items()}
    plan = planner.plan_tiers(f, err, nb, B, bits=levels)
    order, shelves = planner.shelves_from_bits(plan)
    assert plan[E - 1] != levels[0] and order.index(E - 1) < order.index(E - 2)
