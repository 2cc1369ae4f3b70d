"""Host model of the backward's head-summing scans' tile partition (``TilePart`` in csrc/ssd_bwd_tc.cu).

The dB and dC scans on the tensor cores sum their per-head terms over each group's heads: CTA i takes the
contiguous run of (chunk, 128-row block, head) tiles whose cost before them lies in [i, i + 1) * total / n,
and stores one partial sum per (chunk, block, group) key it touched, in slot i + key.  The reduce finds
the CTAs that touched a key from the same arithmetic, without a table.  This model restates both views in
integers and checks, over many shapes, that they agree: every key's heads are covered once, by exactly
the CTAs the reduce visits, in CTA order, and no two (CTA, key) pairs share a slot.  The GPU parity tests
check the kernels themselves against the oracle.
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

    def cta_of(self, t):
        return min(self.n - 1, self.cum(t) * self.n // self.ctot)

    def first_in(self, i, base, cb, n):
        num = i * self.ctot - base * self.n
        if num <= 0:
            return 0
        return min(n, -(-num // (cb * self.n)))

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


def reduce_view(p, key):
    """CTAs the reduce adds for one valid key, with the heads it credits to each, in visiting order."""
    blk, g = divmod(key, p.G)
    r, rb = divmod(blk, p.blocks)
    c = r % p.nc
    k0 = blk * p.H + g * p.hpg
    base, cb = p.cum(k0), p.cost(c, rb)
    i0, i1 = p.cta_of(k0), p.cta_of(k0 + p.hpg - 1)
    out = []
    f0 = p.first_in(i0, base, cb, p.hpg)
    for i in range(i0, i1 + 1):
        f1 = p.first_in(i + 1, base, cb, p.hpg)
        if f0 < f1:
            out.append((i, list(range(f0, f1))))
        f0 = f1
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
            # the ranges cover every tile once, in order
            assert p.beg(0) == 0 and p.beg(n) == p.tiles
            assert all(p.beg(i) <= p.beg(i + 1) for i in range(n))
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
                got = reduce_view(p, key)
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
