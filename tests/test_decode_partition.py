"""Host-side check of the decode attention's work partition and merge protocol (no GPU).

The decode attention lists the 128-key tiles of every (sequence, KV group) row, rows in
order, and gives CTA c of n the tiles [c T / n, (c + 1) T / n). A row split between CTAs
is merged by its first CTA: the others leave a partial in slot row + c and count it,
and the first CTA waits for that count. This test restates the index arithmetic of the
kernel (the tile prefix of the plan kernel, the CTA holding a tile, the walk over the
rows a CTA meets) and checks on random length mixes what the protocol relies on:

* every tile of every row is processed by exactly one CTA;
* a row is whole in a CTA exactly when its first and last tiles are in the same CTA;
* partial slots row + c are unique and fit the scratch (B * Hkv + n slots);
* the row's first CTA reaches the row last in its range (so it merges at its end), and
  the CTAs that publish are exactly the non-empty CTAs after it up to the row's last;
* a merger only waits for CTAs after it, so no wait cycle exists.
"""
import random

import pytest


def plan_of(lens, hkv, s_max):
    """plan[b]: first tile of sequence b's rows; no tiles for an invalid length."""
    plan = [0]
    for n_cached in lens:
        v = 0 if (n_cached < 0 or n_cached >= s_max) else hkv * ((n_cached + 1 + 127) // 128)
        plan.append(plan[-1] + v)
    return plan


def cta_of(t, T, n):
    """The CTA whose range [c T / n, (c + 1) T / n) holds tile t."""
    return ((t + 1) * n - 1) // T


def cta_empty(c, T, n):
    return T * c // n >= T * (c + 1) // n


def walk(plan, B, hkv, b0, tb, te):
    """The (b, g, tiles per row, first, end, row start) segments of the rows that meet
    [tb, te), in order; sequences with no tiles are skipped."""
    segs = []
    if tb >= te:
        return segs
    b = b0
    nt = (plan[b + 1] - plan[b]) // hkv
    g = (tb - plan[b]) // nt
    rs = plan[b] + g * nt
    while rs < te:
        segs.append((b, g, nt, max(tb, rs) - rs, min(te, rs + nt) - rs, rs))
        rs += nt
        g += 1
        if g == hkv:
            g = 0
            b += 1
            while b < B and plan[b + 1] == plan[b]:
                b += 1
            if b < B:
                nt = (plan[b + 1] - plan[b]) // hkv
            else:
                rs = te
    return segs


def check_mix(lens, hkv, s_max, n):
    B = len(lens)
    plan = plan_of(lens, hkv, s_max)
    T = plan[B]
    cover = {}
    slots = set()
    publishers = {}
    merger_of = {}
    n_other = {}  # the count a merger waits for: non-empty CTAs in (c_first, c_last]
    ctas_of = {}  # every CTA that processes some tile of the row
    waits = []  # (waiting CTA, CTA waited for)
    for c in range(n):
        tb, te = T * c // n, T * (c + 1) // n
        holders = [b for b in range(B) if plan[b] <= tb < plan[b + 1]]
        if tb < te:
            assert len(holders) == 1
        segs = walk(plan, B, hkv, holders[0] if holders else 0, tb, te)
        for i, (b, g, nt, j0, j1, rs) in enumerate(segs):
            assert 0 <= j0 < j1 <= nt and b < B and g < hkv and rs == plan[b] + g * nt
            row = b * hkv + g
            for j in range(j0, j1):
                assert (row, j) not in cover
                cover[(row, j)] = c
            ctas_of.setdefault(row, set()).add(c)
            c_first, c_last = cta_of(rs, T, n), cta_of(rs + nt - 1, T, n)
            assert c_first <= c <= c_last
            whole = j0 == 0 and j1 == nt
            assert whole == (c_first == c_last)
            if whole:
                continue
            if c == c_first:
                # the merger: the row is the last one it meets, so it merges at its end
                assert i == len(segs) - 1
                merger_of[row] = c
                others = [cc for cc in range(c_first + 1, c_last + 1) if not cta_empty(cc, T, n)]
                n_other[row] = len(others)
                waits.extend((c, cc) for cc in others)
            else:
                slot = row + c
                assert slot not in slots and slot < B * hkv + n
                slots.add(slot)
                publishers.setdefault(row, set()).add(c)
    for b in range(B):
        nt = (plan[b + 1] - plan[b]) // hkv
        for g in range(hkv):
            for j in range(nt):
                assert (b * hkv + g, j) in cover
    for row, c in merger_of.items():
        # the merger is the row's first CTA; every other CTA of the row publishes once,
        # and that is the count the merger waits for
        assert c == min(ctas_of[row])
        assert publishers[row] == ctas_of[row] - {c}
        assert n_other[row] == len(publishers[row])
    assert set(publishers) == set(merger_of)
    for waiter, waited in waits:
        assert waited > waiter  # waits only go forward: no cycle


@pytest.mark.parametrize("seed", range(6))
def test_decode_partition_and_merge_protocol(seed):
    rng = random.Random(seed)
    for _ in range(100):
        B = rng.choice([1, 2, 3, 7, 64, 100, 300])
        hkv = rng.choice([1, 2, 4, 8])
        s_max = rng.choice([8, 128, 300, 4224, 40000])
        n = rng.choice([1, 3, 148, 256])
        lens = [rng.choice([0, 1, 127, 128, 129, s_max - 1, s_max, rng.randrange(0, s_max + 2), -1])
                for _ in range(B)]
        check_mix(lens, hkv, s_max, n)


def test_decode_partition_bench_shape():
    """The B64 x 4097-position decode layer on 148 CTAs: 16896 tiles, 114-115 per CTA,
    every shared row split between two CTAs."""
    lens = [4096] * 64
    check_mix(lens, 8, 4224, 148)
    plan = plan_of(lens, 8, 4224)
    T = plan[-1]
    assert T == 64 * 8 * 33
    sizes = {T * (c + 1) // 148 - T * c // 148 for c in range(148)}
    assert sizes == {114, 115}
