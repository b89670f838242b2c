"""Host model of the gather-attention kernel's pair schedule (PairPlan in
csrc/attention.cu), checked for the properties the three warp roles rely on.

A pair of neighbouring query blocks walks its tiles in steps: the first tb
tiles lie inside the shared segment and are gathered once for both rows; the
others are gathered per row (two gathers per step while both rows have one),
then the longer row's remaining tiles.  The model restates the kernel's
integer formulas; the GPU parity tests check the kernel's output itself.
Checked here, for every pair shape:
  - each row walks each of its tiles exactly once, in order;
  - a shared step walks the same tile with the same gather group for both rows;
  - gather groups are 0 .. groups-1, increasing along each row, and the
    producer's group -> (row, tile) inverse agrees with the forward map;
  - the K/V ring (5 slots at d = 128) cannot deadlock: the producer fills slot
    positions in order, each needing the position ST earlier released, and the
    MMA issuer's waits and releases follow the kernel's issue order
    (per step: row 0's PV and next S, then row 1's).
(Spreading the shared steps among the own steps instead passes the same
checks, but measured 16.8 ms against 10.7 at wan14b-720p: an own step's four
loads then wait for slots that the other row's MMAs release, which ties the
two rows' chains together.)
"""
import random

import pytest


class PairPlan:
    def __init__(self, nb, na, nc, has1, bpt):
        self.nb, self.na = nb, na
        self.L0 = nb + na
        self.L1 = nb + nc if has1 else 0
        self.n0 = -(-self.L0 // bpt)
        self.n1 = -(-self.L1 // bpt)
        self.tb = nb // bpt if has1 else 0
        self.m = max(0, min(self.n0, self.n1) - self.tb)
        self.groups = self.n0 + self.n1 - self.tb

    def n(self, s):
        return self.n1 if s else self.n0

    def is_shared(self, t):
        return t < self.tb

    def tile(self, t):
        return t

    def group(self, s, t):
        if t < self.tb:
            return t
        d = t - self.tb
        return self.tb + 2 * d + s if d < self.m else self.tb + 2 * self.m + (d - self.m)

    def tile_of(self, g):
        if g < self.tb:
            return -1, g
        r = g - self.tb
        if r < 2 * self.m:
            return r & 1, self.tb + (r >> 1)
        return (0 if self.n0 > self.n1 else 1), self.tb + self.m + (r - 2 * self.m)


def _check(nb, na, nc, has1, bpt, ST=5):
    P = PairPlan(nb, na, nc, has1, bpt)
    rows = [0, 1] if has1 else [0]
    groups = set()
    for r in rows:
        assert sorted(P.tile(t) for t in range(P.n(r))) == list(range(P.n(r)))
        gs = [P.group(r, t) for t in range(P.n(r))]
        assert all(b > a for a, b in zip(gs, gs[1:]))
        for t, g in enumerate(gs):
            sr, tl = P.tile_of(g)
            assert tl == P.tile(t)
            if P.is_shared(t):
                assert sr == -1 and tl < P.tb and P.group(1 - r, t) == g
            else:
                assert sr == r
            groups.add(g)
    assert sorted(groups) == list(range(P.groups))
    # the MMA issuer: first S of each row, then per step and row PV(t) and S(t+1)
    frees = lambda r, t: (not P.is_shared(t)) or r == 1
    ops = []
    for r in rows:
        if P.n(r):
            k = 2 * P.group(r, 0)
            ops.append(([k], [k] if frees(r, 0) else []))
    for t in range(max(P.n0, P.n1)):
        for r in rows:
            if t >= P.n(r):
                continue
            v = 2 * P.group(r, t) + 1
            more = t + 1 < P.n(r)
            waits = [v] + ([2 * P.group(r, t + 1)] if more else [])
            rel = ([v] if frees(r, t) else []) + ([2 * P.group(r, t + 1)] if more and frees(r, t + 1) else [])
            ops.append((waits, rel))
    nload = 2 * P.groups
    assert sorted(x for _, rl in ops for x in rl) == list(range(nload))
    released, loaded, i = set(), 0, 0
    while i < len(ops) or loaded < nload:
        progress = False
        while loaded < nload and (loaded < ST or loaded - ST in released):
            loaded += 1
            progress = True
        if i < len(ops) and all(w < loaded for w in ops[i][0]):
            released.update(ops[i][1])
            i += 1
            progress = True
        assert progress, f"ring deadlock at op {i} (nb={nb}, na={na}, nc={nc}, bpt={bpt})"
    return P


@pytest.mark.parametrize("bpt", [1, 2, 4, 8])
def test_small_pair_shapes(bpt):
    for nb in range(0, 26):
        for na in range(0, 14):
            for nc in sorted({0, 1, 7, 8, 9, na, max(0, na - 9), na + 9}):
                _check(nb, na, nc, True, bpt)
            _check(nb, na, 0, False, bpt)


def test_random_pair_shapes():
    rng = random.Random(7)
    for _ in range(1000):
        bpt = rng.choice((1, 2, 4, 8))
        _check(rng.randint(0, 800), rng.randint(0, 400), rng.randint(0, 400), True, bpt)


def test_wan14b_like_pair():
    # 257 shared blocks, 121 / 118 own, 8 blocks per tile: 32 shared steps, then
    # 15 steps with two gathers, then one more step of row 0
    P = _check(257, 121, 118, True, 8)
    assert (P.tb, P.m, P.n0, P.n1, P.groups) == (32, 15, 48, 47, 63)
