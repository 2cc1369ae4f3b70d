"""Host model of the backward's head-summing scans' tile partition (``TilePart`` in csrc/ssd_bwd_tc.cu).

The dB and dC scans on the tensor cores sum their per-head terms over each group's heads: CTA i takes the
contiguous run of (chunk, 128-row block, head) tiles whose cost before them lies in [i, i + 1) * total / n
(the host works out each run's first tile), and stores one partial sum per (chunk, block, group) key it
touched, in slot i + key.  The reduce takes, for each key, the CTAs whose runs intersect the key's tiles.
This model restates the runs in integers and checks, over many shapes, that the two views agree: every
key's heads are covered once, by exactly the CTAs the reduce visits, in CTA order, that the runs balance
the cost, and that no two (CTA, key) pairs share a slot.  The GPU parity tests check the kernels
themselves against the oracle.
"""
import random

import pytest

ROWS = 128
MAX_CTAS = 256


class Part:
    def __init__(self, batch, T, H, G, Q, anti, n):
        self.H, self.Q, self.G = H, Q, G
        self.hpg = H // G
        self.nc = (T + Q - 1) // Q
        self.blocks = Q // ROWS
        self.len_last = T - (self.nc - 1) * Q
        self.anti, self.n, self.batch = anti, n, batch
        self.cfull = sum(self.cost_len(Q, rb) for rb in range(self.blocks))
        clast = sum(self.cost_len(self.len_last, rb) for rb in range(self.blocks))
        self.perseq = (self.nc - 1) * self.cfull + clast
        self.tiles = batch * self.nc * self.blocks * H
        self.ctot = batch * self.perseq * H

    def cost_len(self, length, rb):
        r0 = rb * ROWS
        if r0 >= length:
            return 0
        return 1 + ((self.Q - r0) if self.anti else (r0 + ROWS)) // ROWS

    def cost(self, c, rb):
        return self.cost_len(self.len_last if c == self.nc - 1 else self.Q, rb)

    def cum(self, t):
        blk, h = divmod(t, self.H)
        r, rb = divmod(blk, self.blocks)
        b, c = divmod(r, self.nc)
        before = b * self.perseq + c * self.cfull + sum(self.cost(c, q) for q in range(rb))
        return before * self.H + self.cost(c, rb) * h

    def beg(self, i):
        if i <= 0:
            return 0
        if i >= self.n:
            return self.tiles
        lo, hi = 0, self.tiles
        while lo < hi:
            mid = (lo + hi) // 2
            if self.cum(mid) * self.n >= i * self.ctot:
                hi = mid
            else:
                lo = mid + 1
        return lo

    def valid(self, t):
        blk = t // self.H
        r, rb = divmod(blk, self.blocks)
        c = r % self.nc
        return self.cost(c, rb) > 0


def kernel_view(p):
    """(CTA, key) -> heads of the key the CTA's run holds, from the scans' tile ranges."""
    seen = {}
    for i in range(p.n):
        for t in range(p.beg(i), p.beg(i + 1)):
            if not p.valid(t):
                continue
            key = t // p.hpg
            seen.setdefault((i, key), []).append(t % p.hpg)
    return seen


def reduce_view(p, table, key):
    """CTAs the reduce adds for one valid key (those whose runs intersect the key's tiles), with the heads
    the intersection holds, in visiting order."""
    blk, g = divmod(key, p.G)
    k0 = blk * p.H + g * p.hpg
    out = []
    for i in range(p.n):
        lo, hi = max(table[i], k0), min(table[i + 1], k0 + p.hpg)
        if lo < hi:
            out.append((i, list(range(lo - k0, hi - k0))))
    return out


def shapes():
    rng = random.Random(20240611)
    fixed = [(4, 2048, 80, 1, 256), (2, 600, 8, 2, 256), (1, 131072 // 64, 48, 8, 128), (1, 130, 2, 1, 128),
             (3, 1, 4, 4, 256), (1, 256, 1, 1, 256), (2, 383, 6, 3, 128)]
    for f in fixed:
        yield f
    for _ in range(60):
        G = rng.choice([1, 2, 4])
        H = G * rng.randint(1, 12)
        yield (rng.randint(1, 4), rng.randint(1, 1300), H, G, rng.choice([128, 256]))


@pytest.mark.parametrize("anti", [True, False])
def test_partition_and_reduce_agree(anti):
    rng = random.Random(7)
    for batch, T, H, G, Q in shapes():
        tiles = batch * ((T + Q - 1) // Q) * (Q // ROWS) * H
        for n in {1, min(tiles, 148), min(tiles, rng.randint(1, MAX_CTAS))}:
            p = Part(batch, T, H, G, Q, anti, n)
            table = [p.beg(i) for i in range(n + 1)]
            # the ranges cover every tile once, in order
            assert table[0] == 0 and table[n] == p.tiles
            assert all(table[i] <= table[i + 1] for i in range(n))
            seen = kernel_view(p)
            nkeys = p.tiles // p.hpg
            # slots are unique and inside the workspace's region
            slots = [i + key for (i, key) in seen]
            assert len(set(slots)) == len(slots)
            assert all(0 <= s < MAX_CTAS + nkeys for s in slots)
            # the reduce visits exactly the CTAs that hold part of each valid key, crediting the same heads
            for key in range(nkeys):
                if not p.valid(key * p.hpg):
                    continue
                want = sorted((i, sorted(hs)) for (i, k), hs in seen.items() if k == key)
                got = reduce_view(p, table, key)
                assert got == want, (batch, T, H, G, Q, n, key)
                assert sorted(h for _, hs in got for h in hs) == list(range(p.hpg))


def test_partition_balances_cost():
    # the 2.7B layer's dB scan (anti-causal: the chunk's first block has two halves) on 148 CTAs
    p = Part(4, 2048, 80, 1, 256, True, 148)
    costs = []
    for i in range(p.n):
        costs.append(sum(p.cost((t // p.H // p.blocks) % p.nc, (t // p.H) % p.blocks)
                         for t in range(p.beg(i), p.beg(i + 1))))
    assert sum(costs) == p.ctot
    assert max(costs) - min(costs) <= 2 * 3  # within two tiles' cost of each other


def _check(p, slot_of, reduce):
    """The agreement checks of test_partition_and_reduce_agree for one partition, with the slot rule and the
    reduce's view passed in (so that a planted mistake in either can be shown to fail)."""
    table = [p.beg(i) for i in range(p.n + 1)]
    seen = kernel_view(p)
    nkeys = p.tiles // p.hpg
    slots = [slot_of(i, key) for (i, key) in seen]
    if len(set(slots)) != len(slots) or not all(0 <= s < MAX_CTAS + nkeys for s in slots):
        return False
    for key in range(nkeys):
        if not p.valid(key * p.hpg):
            continue
        want = sorted((i, sorted(hs)) for (i, k), hs in seen.items() if k == key)
        if reduce(p, table, key) != want:
            return False
    return True


def _first_cta_only(p, table, key):
    # a mistake: the reduce takes only the CTA whose run holds the key's first head
    got = reduce_view(p, table, key)
    return got[:1]


def _off_by_one_end(p, table, key):
    # a mistake: a run's end taken as inclusive
    blk, g = divmod(key, p.G)
    k0 = blk * p.H + g * p.hpg
    out = []
    for i in range(p.n):
        lo, hi = max(table[i], k0), min(table[i + 1] + 1, k0 + p.hpg)
        if lo < hi:
            out.append((i, list(range(lo - k0, hi - k0))))
    return out


@pytest.mark.parametrize("mistake", ["slot_is_key", "first_cta_only", "inclusive_end"])
def test_a_planted_mistake_in_the_partition_is_caught(mistake):
    slot_of = (lambda i, key: key) if mistake == "slot_is_key" else (lambda i, key: i + key)
    reduce = {"first_cta_only": _first_cta_only, "inclusive_end": _off_by_one_end}.get(mistake, reduce_view)
    # the right rules pass on every shape; the planted one fails on at least one
    caught = False
    for batch, T, H, G, Q in list(shapes())[:20]:
        tiles = batch * ((T + Q - 1) // Q) * (Q // ROWS) * H
        for anti in (True, False):
            p = Part(batch, T, H, G, Q, anti, min(tiles, 148))
            assert _check(p, lambda i, key: i + key, reduce_view)
            if not _check(p, slot_of, reduce):
                caught = True
    assert caught, mistake
