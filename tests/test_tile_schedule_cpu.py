"""CPU model of the one-token-half tile plan's code-slot schedule.

The dequant warps walk their CTA's blocks of 128 codes of each row (one group
with groups of 128) through a ring of kS shared-memory slots: block j's codes are copied
into slot j % kS when it is issued, PD = kS - 1 blocks before it is consumed,
and its (scale | zero << 16) words are written into the same slot when block
j + 2 is issued, or, when block j is the second of a pair loaded with one
4-byte load (groups of 128, an even number of groups per row), when block
j + 1 is issued.  The kernel's loop is: issue blocks 0 .. PD - 1, then for
i = 0, 1, ...: issue block i + PD, consume block i.

This model replays that order over random tile sequences (each tile an op
with its own number of groups per row) for the slot counts of every plan, and
checks that (1) a slot's codes and words are overwritten only after the
block that held them was consumed, (2) a block's words are in its slot when
it is consumed, and (3) a pair never spans two tiles.
"""
import random

import pytest

# kSlots of the one-token-half plans: (bits, x rows per stage) -> slots
SLOTS = {(2, 64): 5, (3, 64): 4, (4, 64): 3, (2, 128): 6, (3, 128): 5, (4, 128): 4, (8, 128): 3}

ONE, SPLIT, PAIR, PAIR_SECOND = 1, 2, 3, 4


def block_modes(tiles):
    """Per block: (tile, block index in the tile, load mode), as the issue
    cursor assigns them; tiles = [(blocks of 128 codes per row, group size)]
    (with groups of 128 the block count is the group count)."""
    out = []
    for t, (G, group) in enumerate(tiles):
        pair2 = group == 128 and G % 2 == 0
        for gp in range(G):
            if group != 128:
                mode = SPLIT
            elif pair2:
                mode = PAIR if gp % 2 == 0 else PAIR_SECOND
            else:
                mode = ONE
            out.append((t, gp, mode))
    return out


def replay(blocks, kS, PD=None):
    PD = kS - 1 if PD is None else PD
    n = len(blocks)
    codes_of = [None] * kS     # block whose codes a slot holds
    words_of = [None] * kS     # block whose words a slot holds
    consumed = set()

    def write_words(b):
        s = b % kS
        prev = words_of[s]
        assert prev is None or prev in consumed or prev == b, f"words of block {prev} overwritten before use"
        assert codes_of[s] == b, f"slot {s} holds the codes of block {codes_of[s]}, not {b}"
        words_of[s] = b

    def issue(j):
        if j >= 2 and j - 2 < n:
            mode = blocks[j - 2][2]
            if mode in (ONE, SPLIT, PAIR):
                write_words(j - 2)
            if mode == PAIR:
                assert blocks[j - 1][0] == blocks[j - 2][0], "a pair spans two tiles"
                assert blocks[j - 1][2] == PAIR_SECOND
                write_words(j - 1)
        if j < n:
            s = j % kS
            prev = codes_of[s]
            assert prev is None or prev in consumed, f"codes of block {prev} overwritten before use"
            codes_of[s] = j

    def consume(i):
        s = i % kS
        assert codes_of[s] == i and words_of[s] == i, f"block {i}: slot {s} not ready"
        consumed.add(i)

    for j in range(PD):
        issue(j)
    for i in range(n):
        issue(i + PD)
        consume(i)
    return consumed


@pytest.mark.parametrize("plan", sorted(SLOTS))
def test_slot_schedule_random_tiles(plan):
    kS = SLOTS[plan]
    rng = random.Random(1000 + 10 * plan[0] + plan[1])
    for _ in range(300):
        tiles = []
        for _ in range(rng.randint(1, 6)):
            group = rng.choice((128, 128, 128, 64, 32))
            G = rng.randint(1, 12)  # blocks of 128 codes per row; odd and even
            tiles.append((G, group))
        blocks = block_modes(tiles)
        assert replay(blocks, kS) == set(range(len(blocks)))


def test_pairs_need_an_even_group_count():
    # 8 groups per row: 4 pairs; 3 groups per row: one group per load
    modes = [m for (_, _, m) in block_modes([(8, 128)])]
    assert modes == [PAIR, PAIR_SECOND] * 4
    assert [m for (_, _, m) in block_modes([(3, 128)])] == [ONE] * 3
    assert [m for (_, _, m) in block_modes([(4, 64)])] == [SPLIT] * 4


def test_the_model_catches_a_schedule_that_runs_too_far_ahead():
    """Issuing kS blocks ahead with kS slots overwrites the codes of a block
    not yet consumed; the model must see it (so that it is not vacuous)."""
    blocks = block_modes([(6, 128)])
    for kS in (3, 4, 5):
        with pytest.raises(AssertionError, match="overwritten before use"):
            replay(blocks, kS, PD=kS)
