"""The fused kernel's inter-chunk hand-off, modelled on the CPU.

A randomised model of the protocol that ``csrc/ssd_fused.cu`` runs between CTAs: the hand-out order of
``decode`` (the owners of a chunk one step ahead of the chunk before's other blocks), the chain without
look-back (the owner of chunk c waits for S~_{c-1} and reads it from its sequence's one fp32 slot, then
writes S~_c over it; the other blocks read bf16 tiles of S~ from 3 slots, stored by the owner's publisher
once the slot's earlier readers are done and flagged per slot) and with look-back over D chunks (local
states L_c published early, the owner starting from the most recent S~_j whose later L are out; 2D slots
of S~ and L, which the other blocks read too), and the slot-reuse counts (``cons``).  CTAs take units in hand-out order and interleave at random.
The test checks that every schedule finishes (no deadlock with one CTA or many) and that no read ever
finds its slot overwritten; planted mistakes in the reuse counts must be caught.  The model follows the
kernel's rules one for one; it is the argument behind the kernel's comments, executed.
"""
import random

import pytest


def decode(u, nc, halves, Mo, Mw):
    """(chunk, unit index within the role, row block) of hand-out position u, as the kernel's decode:
    Mo units per chunk of the other block (r = 0), Mw of the owners' block (r = 1)."""
    if halves == 1:
        return u // Mo, u % Mo, 0
    if u < Mw:
        return 0, u, 1
    v = u - Mw
    t, j = v // (Mw + Mo), v % (Mw + Mo)
    if t < nc - 1 and j < Mw:
        return t + 1, j, 1
    return t, (j - Mw if t < nc - 1 else j), 0


def run(nc, halves, M, heads, D, ctas, lastlen, seed, split=1, planted_undercount=False, planted_no_wait=False,
        planted_tile_count=False):
    # M units of `heads` heads per chunk for the other block; the owners' block in units of heads / split
    rnd = random.Random(seed)
    R = 3 if D == 1 else 2 * D
    # counted reads of a slot per use: the next chunk's other block (its tile), and with look-back the D
    # owners after it (S~ and L); without look-back the owners' reads of the one fp32 slot are ordered by
    # the chain itself and not counted
    rpu = (D if D > 1 else 0) + (1 if halves == 2 else 0) - (1 if planted_undercount else 0)
    nbh = M * heads
    inc = [[0] * R for _ in range(nbh)]
    agg = [[0] * R for _ in range(nbh)]
    cons = [[0] * R for _ in range(nbh)]
    tag_s = [[-1] * R for _ in range(nbh)]   # fp32 S~ (D = 1: slot 0 only)
    tag_l = [[-1] * R for _ in range(nbh)]   # fp32 L (look-back)
    tag_t = [[-1] * R for _ in range(nbh)]   # bf16 tile of S~
    tin = [[0] * R for _ in range(nbh)]      # per slot: c + 1 once the tile of S~_c is in it
    Mo, Mw, hw = M, M * split, heads // split
    n_units = nc * (Mo + Mw if halves == 2 else Mo)
    Q = 128 * halves
    counter = [0]

    def pause(k):
        # short random delays, and now and then a long one (a block that falls far behind)
        n = rnd.randint(20, 60) if rnd.random() < 0.05 else rnd.randint(0, k)
        for _ in range(n):
            yield None

    def flag(bh, c):  # the inc flag of chunk c: one count per sequence without look-back
        return (bh, 0) if D == 1 else (bh, c % R)

    def wait_slot_readers(bh, c):
        if c >= R and not planted_no_wait:
            while cons[bh][c % R] < (c // R) * rpu:
                yield None

    def unit(u):
        c, idx, r = decode(u, nc, halves, Mo, Mw)
        hu = hw if r == 1 else heads
        ln = Q if c < nc - 1 else lastlen
        if r * 128 >= ln:
            return
        owner = r == (ln - 1) // 128
        for hh in range(hu):  # a pipeline's heads, one after the other
            bh = idx * hu + hh
            yield from pause(3)
            writes = owner and c < nc - 1
            if not owner:
                if c > 0 and D == 1:  # the issuer waits for the tile of S~_{c-1}, loads it, counts the read
                    while tin[bh][0 if planted_tile_count else (c - 1) % R] < c:
                        yield None
                    assert tag_t[bh][(c - 1) % R] == c - 1, ("tile overwritten before it was read", c)
                    yield from pause(2)
                    cons[bh][(c - 1) % R] += 1
                elif c > 0:  # look-back: the warps read S~_{c-1} from its fp32 slot
                    b, s = flag(bh, c - 1)
                    while inc[b][s] < c:
                        yield None
                    assert tag_s[bh][(c - 1) % R] == c - 1, ("S~ overwritten before it was read", c)
                    yield from pause(2)
                    cons[bh][(c - 1) % R] += 1
                continue
            if D > 1 and writes:  # publish L_c early, once chunk c-R's readers are done
                yield from wait_slot_readers(bh, c)
                tag_l[bh][c % R] = c
                yield from pause(3)
                agg[bh][c % R] = c + 1
            if D > 1:  # look-back: the most recent S~_j whose later L are all out
                while True:
                    base = None
                    for l in range(D):
                        j = c - 1 - l
                        if j == -1:
                            base = -1
                            break
                        if j < -1:
                            break
                        if inc[bh][j % R] >= j + 1:
                            base = j
                            break
                        if agg[bh][j % R] < j + 1:
                            break
                    if base is not None:
                        break
                    yield None
                if base >= 0:
                    assert tag_s[bh][base % R] == base, ("S~ overwritten before it was read", c, base)
                for i in range(base + 1, c):
                    assert tag_l[bh][i % R] == i, ("L overwritten before it was read", c, i)
            elif c > 0:
                while inc[bh][0] < c:
                    yield None
                assert tag_s[bh][0] == c - 1, ("S~ overwritten before it was read", c)
            yield from pause(3)
            if writes:
                tag_s[bh][0 if D == 1 else c % R] = c
                yield from pause(2)
                b, s = flag(bh, c)
                inc[b][s] = c + 1
            if D > 1:
                for l in range(min(D, c)):
                    cons[bh][(c - 1 - l) % R] += 1
            if writes and halves == 2 and D == 1:  # the publisher's tile store, after the chain's release
                yield from pause(3)
                yield from wait_slot_readers(bh, c)
                tag_t[bh][c % R] = c
                yield from pause(2)
                tin[bh][0 if planted_tile_count else c % R] = c + 1

    def cta():
        while True:
            u = counter[0]
            counter[0] += 1
            if u >= n_units:
                return
            yield from unit(u)
            yield None

    alive = [cta() for _ in range(ctas)]
    steps = 0
    while alive:
        p = rnd.choice(alive)
        try:
            next(p)
        except StopIteration:
            alive.remove(p)
        steps += 1
        assert steps < 2_000_000, ("no progress", nc, halves, M, D, ctas)


def _cases(n, seed0):
    rnd = random.Random(seed0)
    for seed in range(n):
        halves = rnd.choice([1, 2])
        heads = rnd.choice([1, 2, 3, 4, 6])
        split = rnd.choice([d for d in (1, 2, 3) if heads % d == 0]) if halves == 2 else 1
        yield dict(nc=rnd.choice([1, 2, 3, 5, 9, 17, 33]), halves=halves, M=rnd.choice([1, 2, 3]),
                   heads=heads, split=split, D=rnd.choice([1, 4]), ctas=rnd.choice([1, 2, 3, 5, 8, 30]),
                   lastlen=rnd.choice([128 * halves, 1, 77] + ([129] if halves == 2 else [])), seed=seed)


@pytest.mark.parametrize("case", list(_cases(60, 7)), ids=lambda c: "nc{nc}_h{halves}_M{M}_H{heads}_s{split}_D{D}_cta{ctas}".format(**c))
def test_every_schedule_finishes_and_no_read_sees_an_overwritten_slot(case):
    run(**case)


@pytest.mark.parametrize("mistake", ["planted_undercount", "planted_no_wait", "planted_tile_count"])
@pytest.mark.parametrize("depth", [1, 4])
def test_a_planted_mistake_in_the_slot_reuse_is_caught(mistake, depth):
    # one read too few per use of a slot, an owner that overwrites a slot (L_c, or the tile of S~_c)
    # without waiting for its readers, or one tile count per sequence instead of a flag per slot (tile
    # stores may complete out of chunk order): some block then reads a slot that was overwritten or not
    # yet written
    if mistake == "planted_tile_count" and depth > 1:
        pytest.skip("with look-back the other blocks read the fp32 slots: there are no tiles")
    caught = 0
    for case in _cases(300, 11):
        if case["D"] != depth or case["nc"] < 9 or (depth == 1 and case["halves"] == 1):
            continue

        try:
            run(**case, **{mistake: True})
        except AssertionError:
            caught += 1
    assert caught >= 1
