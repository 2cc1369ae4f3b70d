"""The fused kernel's inter-chunk hand-off, modelled on the CPU.

A randomised model of the protocol that ``csrc/ssd_fused.cu`` runs between CTAs: the hand-out order of
``decode`` (the owners of a chunk one step ahead of the chunk before's other blocks), the chain without
look-back (the owner of chunk c waits for S~_{c-1}; slot c % 3) and with look-back over D chunks (local
states L_c published early, the owner starting from the most recent S~_j whose later L are out; 2D
slots), and the slot-reuse counts (``cons``).  CTAs take units in hand-out order and interleave at
random.  The test checks that every schedule finishes (no deadlock with one CTA or many) and that no
read ever finds its slot overwritten; a planted under-count of the reads must be caught.  The model
follows the kernel's rules one for one; it is the argument behind the kernel's comments, executed.
"""
import random

import pytest


def decode(u, nc, halves, M):
    """(chunk, unit index within the role, row block) of hand-out position u, as the kernel's decode."""
    if halves == 1:
        return u // M, u % M, 0
    if u < M:
        return 0, u, 1
    v = u - M
    t, j = v // (2 * M), v % (2 * M)
    if t < nc - 1 and j < M:
        return t + 1, j, 1
    return t, (j - M if t < nc - 1 else j), 0


def run(nc, halves, M, heads, D, ctas, lastlen, seed, planted_undercount=False, planted_no_wait=False):
    rnd = random.Random(seed)
    R = 3 if D == 1 else 2 * D
    count_owner_reads = D > 1  # without look-back an owner's read precedes the next owners' publications
    # reads of a slot per use: the next chunk's other block, and with look-back the D owners after it
    rpu = (D if count_owner_reads else 0) + (1 if halves == 2 else 0) - (1 if planted_undercount else 0)
    nbh = M * heads
    inc = [[0] * R for _ in range(nbh)]
    agg = [[0] * R for _ in range(nbh)]
    cons = [[0] * R for _ in range(nbh)]
    tag_s = [[-1] * R for _ in range(nbh)]
    tag_l = [[-1] * R for _ in range(nbh)]
    n_units = nc * M * halves
    Q = 128 * halves
    counter = [0]

    def pause(k):
        # short random delays, and now and then a long one (a block that falls far behind)
        n = rnd.randint(20, 60) if rnd.random() < 0.05 else rnd.randint(0, k)
        for _ in range(n):
            yield None

    def unit(u):
        c, idx, r = decode(u, nc, halves, M)
        ln = Q if c < nc - 1 else lastlen
        if r * 128 >= ln:
            return
        owner = r == (ln - 1) // 128
        for hh in range(heads):  # a pipeline's heads, one after the other
            bh = idx * heads + hh
            yield from pause(3)
            writes = owner and c < nc - 1
            if owner and D > 1 and writes:  # publish L_c early, once chunk c-R's readers are done
                if c >= R and not planted_no_wait:
                    while cons[bh][c % R] < (c // R) * rpu:
                        yield None
                tag_l[bh][c % R] = c
                yield from pause(3)
                agg[bh][c % R] = c + 1
            if owner and D > 1:  # look-back: the most recent S~_j whose later L are all out
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
            else:
                if c > 0:
                    while inc[bh][(c - 1) % R] < c:
                        yield None
                if writes and c >= R:
                    while cons[bh][c % R] < (c // R) * rpu:
                        yield None
                if c > 0:
                    assert tag_s[bh][(c - 1) % R] == c - 1, ("S~ overwritten before it was read", c)
            yield from pause(3)
            if owner:
                if writes:
                    tag_s[bh][c % R] = c
                yield from pause(2)
                if writes:
                    inc[bh][c % R] = c + 1
                if count_owner_reads:
                    for l in range(min(D, c)):
                        cons[bh][(c - 1 - l) % R] += 1
            elif c > 0:
                yield from pause(2)
                cons[bh][(c - 1) % R] += 1

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
        yield dict(nc=rnd.choice([1, 2, 3, 5, 9, 17, 33]), halves=halves, M=rnd.choice([1, 2, 3]),
                   heads=rnd.choice([1, 2, 3]), D=rnd.choice([1, 4]), ctas=rnd.choice([1, 2, 3, 5, 8, 30]),
                   lastlen=rnd.choice([128 * halves, 1, 77] + ([129] if halves == 2 else [])), seed=seed)


@pytest.mark.parametrize("case", list(_cases(60, 7)), ids=lambda c: "nc{nc}_h{halves}_M{M}_H{heads}_D{D}_cta{ctas}".format(**c))
def test_every_schedule_finishes_and_no_read_sees_an_overwritten_slot(case):
    run(**case)


@pytest.mark.parametrize("mistake", ["planted_undercount", "planted_no_wait"])
def test_a_planted_mistake_in_the_slot_reuse_is_caught(mistake):
    # one read too few per use of a slot, or an owner that publishes L_c without waiting for the slot's
    # readers: some block then reads a slot that was overwritten
    caught = 0
    for case in _cases(300, 11):
        if case["D"] == 1 or case["nc"] < 9:
            continue
        try:
            run(**case, **{mistake: True})
        except AssertionError:
            caught += 1
    assert caught >= 1
