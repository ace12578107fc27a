"""CPU model of the decode kernel's work split and split-K bookkeeping.

A decode launch is a sequence of CTA steps: op o owns row_blocks(o) x su(o)
steps in row-block-major order (su = steps per row block, GPS groups of 128
each).  The host cuts the sequence into chunks, whole row blocks when there
are at least 4 per CTA (ops sorted by su, longest first), else runs of 2^c
steps.  A CTA walks the steps of each chunk it takes; at the last step of its
piece of a row block it emits: directly when the piece is the whole row
block, otherwise into partial slot (chunk, 0) when the row block started in an
earlier chunk and (chunk, 1) when it continues in a later one, then each of
the CTA's 4 warps adds 1 to counter 1 + w_first (w_first = the row block's
first chunk).  The warp that brings that counter to 4 x (number of chunks
holding a piece) adds the tail slot of chunk w_first and the head slots of
chunks w_first + 1 .. w_last in that order.

This model restates the host's chunk planning and the kernel's step flags
and emission, and checks over random stacks that every step is visited once,
no partial slot is written twice, every cut row block's pieces sit in the
consecutive chunks w_first .. w_last with the slots the reduction reads, its
counter reaches the kernel's threshold exactly once, and no two cut row
blocks share a counter.
"""
import bisect
import random

import pytest

WARPS = 4
MAX_COUNTERS = 256 * 1024 // 4


def geometry(bits, mt):
    rows = 16 * WARPS * (2 if (mt >= 4 and bits <= 4) else 1)
    gps = 1 if bits == 16 else (2 if (bits == 8 or mt >= 4) else 4)
    return rows, gps


def plan(ops, bits, mt, max_ctas):
    """Host chunk planning: per-op (step0, su, row_blocks) in launch order,
    total steps, log2c, chunk count, units flag."""
    rows, gps = geometry(bits, mt)
    rbs = [(N + rows - 1) // rows for (N, K) in ops]
    sus = [(K // 128 + gps - 1) // gps for (N, K) in ops]
    total = sum(r * s for r, s in zip(rbs, sus))
    units_total = sum(rbs)
    order = list(range(len(ops)))
    units, log2c = 0, 0
    if units_total >= 4 * max_ctas:
        units = 1
        n_chunks = units_total
        order.sort(key=lambda i: -sus[i])  # stable, like std::stable_sort
    elif total >= 16 * max_ctas:
        per = total // (12 * max_ctas)
        log2c = 2
        while log2c < 8 and (2 << log2c) <= per:
            log2c += 1
        n_chunks = (total + (1 << log2c) - 1) >> log2c
    else:
        per = (total + max_ctas - 1) // max_ctas
        while (1 << log2c) < per:
            log2c += 1
        n_chunks = (total + (1 << log2c) - 1) >> log2c
    launch, step0, unit0 = [], 0, 0
    for i in order:
        launch.append({"step0": step0, "unit0": unit0, "su": sus[i], "rb": rbs[i], "op": i})
        step0 += rbs[i] * sus[i]
        unit0 += rbs[i]
    return launch, total, log2c, n_chunks, units


def chunk_range(launch, total, log2c, units, k):
    if units:
        o = bisect.bisect_right([op["unit0"] for op in launch], k) - 1
        b = launch[o]["step0"] + (k - launch[o]["unit0"]) * launch[o]["su"]
        return b, b + launch[o]["su"]
    b = k << log2c
    return b, min(b + (1 << log2c), total)


def simulate(ops, bits, mt, max_ctas, arrivals=WARPS):
    launch, total, log2c, n_chunks, units = plan(ops, bits, mt, max_ctas)
    if not units:
        assert n_chunks + 1 <= MAX_COUNTERS - 2
    visited = [0] * total
    slots = {}       # (chunk, 0 | 1) -> row block
    counters = {}    # counter index -> [row block, arrivals]
    pieces = {}      # row block -> list of (chunk, slot or None)
    starts = [op["step0"] for op in launch]
    for k in range(n_chunks):
        begin, end = chunk_range(launch, total, log2c, units, k)
        for s in range(begin, end):
            visited[s] += 1
            o = bisect.bisect_right(starts, s) - 1  # last op with step0 <= s
            op = launch[o]
            local = s - op["step0"]
            rb, j = divmod(local, op["su"])
            unit_start = s - j
            last = j + 1 == op["su"] or s + 1 == end
            head = unit_start < begin
            tail = unit_start + op["su"] > end
            if not last:
                continue
            key = (o, rb)
            if not (head or tail):
                pieces.setdefault(key, []).append((k, None))
                continue
            slot = (k, 0 if head else 1)
            assert slot not in slots, f"partial slot {slot} written twice"
            slots[slot] = key
            pieces.setdefault(key, []).append((k, slot))
            w_first = unit_start >> log2c
            w_last = (unit_start + op["su"] - 1) >> log2c
            c = counters.setdefault(1 + w_first, [key, 0])
            assert c[0] == key, f"counter {1 + w_first} shared by row blocks {c[0]} and {key}"
            c[1] += arrivals
            if c[1] == WARPS * (w_last - w_first + 1):
                # the last arrival reduces: tail slot of w_first, head slots after it
                reads = [(w_first, 1)] + [(ww, 0) for ww in range(w_first + 1, w_last + 1)]
                assert all(slots.get(r) == key for r in reads), f"row block {key} reads slots it did not write"
                assert sorted(ch for ch, _ in pieces[key]) == list(range(w_first, w_last + 1))
            assert c[1] <= WARPS * (w_last - w_first + 1)
    assert visited == [1] * total
    for key, ps in pieces.items():
        if len(ps) > 1 or ps[0][1] is not None:
            op = launch[key[0]]
            w_first = (op["step0"] + key[1] * op["su"]) >> log2c
            assert counters[1 + w_first][1] == WARPS * len(ps), f"row block {key} never reduced"
    n_blocks = sum(op["rb"] for op in launch)
    assert len(pieces) == n_blocks
    return units, log2c, n_chunks


def test_known_stack_plans():
    """The 28-layer 7B-shaped INT4 stack at M = 1 on 148 SMs x 4 CTAs runs
    whole row blocks; a single small layer is split into short chunks."""
    qwen = [(4608, 3584), (3584, 3584), (37888, 3584), (3584, 18944)] * 28
    units, _, n_chunks = simulate(qwen, 4, 1, 148 * 4)
    assert units == 1 and n_chunks == sum((N + 63) // 64 for N, _ in qwen)
    units, log2c, n_chunks = simulate([(512, 512)], 4, 1, 148 * 4)
    assert units == 0 and (log2c, n_chunks) == (0, 8)


@pytest.mark.parametrize("seed", range(8))
def test_random_stacks(seed):
    rng = random.Random(seed)
    for _ in range(60):
        bits = rng.choice((2, 3, 4, 8, 16))
        mt = rng.choice((1, 2, 4))
        max_ctas = 148 * rng.choice((1, 2, 3, 4))
        ops = [(rng.randint(1, 12000), 128 * rng.randint(1, 160)) for _ in range(rng.randint(1, 12))]
        simulate(ops, bits, mt, max_ctas)


def test_the_model_catches_a_wrong_piece_count():
    """If each piece brought one arrival fewer than the kernel's threshold
    counts, a cut row block would never be reduced: the model must see it (so
    that it is not vacuous)."""
    ops = [(300, 128 * 37)]  # 5 row blocks of 10 steps, chunks of 1 step
    launch, total, log2c, n_chunks, units = plan(ops, 4, 1, 148)
    assert not units
    simulate(ops, 4, 1, 148)
    with pytest.raises(AssertionError, match="never reduced"):
        simulate(ops, 4, 1, 148, arrivals=WARPS - 1)
