"""Tier planner: which experts get which precision under a byte budget.

[P1] "step 4: three shelves, all on the GPU" describes the rule: a greedy
planner fills a memory budget, and every byte goes to the expert where it
removes the most expected error.  Here that is a host-side function of three
inputs the caller supplies:

* freq[e]  how often expert e is routed (any scale; the expected error of an
           expert counts in proportion to its use),
* err[e][b] the expected quantisation error of expert e stored at b bits
           (for instance the squared error of dequant(quant(W)) summed over
           its weights, measured with the library's own quantiser),
* nbytes[b] the bytes of one expert at b bits (codes plus block scales).

Every expert starts at the lowest precision; then, repeatedly, among the
upgrades that still fit the budget (3 -> 4 bits, 4 -> 8 bits) the one with the
largest freq * (error removed) / (bytes added) is taken, until none fits.
The library stores each precision as one shelf covering a contiguous id range
(moe_tier), so shelves_from_bits orders the experts by precision (ties by id)
and returns the permutation together with the shelf ranges; when the
planned precisions already fall with the expert id (hot experts first, as
their ids are popularity ranks) the permutation is the identity.

A level need not be one width: the pages' repacker gives the down
projections a ladder of their own (`--gu Q6_K,IQ4_XS,IQ3_XXS` beside `--dn
Q8_0,IQ4_NL,MXFP4`), so a level can be a (gate_up, down) format pair such as
(3, 5) for 3-bit gate_up with FP4 down; err and nbytes are then keyed by the
pairs, and the levels are ranked by their bytes.
"""
import heapq

BITS = (3, 4, 8)


def plan_tiers(freq, err, nbytes, budget, bits=BITS):
    """Per-expert bit widths (a list, one entry per expert) under `budget`
    bytes.  err[e] and nbytes map each width in `bits` (ascending) to the
    expert's expected error and bytes.  Raises if even the lowest precision
    does not fit."""
    E = len(freq)
    bits = tuple(sorted(bits, key=lambda b: nbytes[b]))  # ascending bytes
    level = [0] * E
    used = sum(nbytes[bits[0]] for _ in range(E))
    if used > budget:
        raise ValueError(f"budget {budget} B is below the lowest precision's {used} B")
    heap = []

    def push(e):
        lv = level[e]
        if lv + 1 < len(bits):
            b0, b1 = bits[lv], bits[lv + 1]
            cost = nbytes[b1] - nbytes[b0]
            gain = freq[e] * (err[e][b0] - err[e][b1])
            # largest gain per byte first; ties go to the lower id
            heapq.heappush(heap, (-gain / cost, e, lv))

    for e in range(E):
        push(e)
    while heap:
        _, e, lv = heapq.heappop(heap)
        if lv != level[e]:
            continue
        cost = nbytes[bits[lv + 1]] - nbytes[bits[lv]]
        if used + cost > budget:
            continue  # this expert stays; a cheaper upgrade elsewhere may still fit
        used += cost
        level[e] += 1
        push(e)
    return [bits[lv] for lv in level]


def plan_bytes(plan, nbytes):
    return sum(nbytes[b] for b in plan)


def expected_error(plan, freq, err):
    return sum(f * err[e][b] for e, (f, b) in enumerate(zip(freq, plan)))


def shelves_from_bits(plan):
    """(order, shelves): order[new_id] = old expert id, sorted by precision
    (highest first, widths or format pairs compared as values) then id;
    shelves = [(bits, first, count)] over the new ids, one per precision in
    use."""
    # a stable sort in descending order keeps equal precisions in id order
    order = sorted(range(len(plan)), key=lambda e: plan[e], reverse=True)
    shelves = []
    for new, e in enumerate(order):
        b = plan[e]
        if shelves and shelves[-1][0] == b:
            shelves[-1] = (b, shelves[-1][1], shelves[-1][2] + 1)
        else:
            shelves.append((b, new, 1))
    return order, shelves
