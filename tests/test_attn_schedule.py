"""The attention's balanced tile schedule, checked on the CPU.

The kernels cut all units' key tiles, laid end to end, into one contiguous
range per CTA of a persistent grid; each CTA walks its range as segments (one
per unit it touches) and stores each segment's partial at slot u + c; the
CTA that completes a unit finds its CTAs by c(t) = ((t+1)*P - 1) // T and
merges them.  This restates that
integer arithmetic (attn_plan_kernel and the SegWalk of attn_kernel) and
checks it against brute force: every tile is run exactly once, slots are
distinct and inside the partial buffers, every walk starts at its first
tile's unit and reads no prefix sum past the end, each unit's CTA range is
exactly the CTAs that ran a piece of it, and the count the fix-up waits for
is the number of those CTAs.
"""
import numpy as np
import pytest

BN = 128


def plan(lengths, n_qtiles, Hkv, L_cap, P):
    units = len(lengths) * Hkv * n_qtiles
    n = [1 + (min(max(lengths[u // (Hkv * n_qtiles)], 0), L_cap) + BN - 1) // BN
         for u in range(units)]
    start = [0]
    for x in n:
        start.append(start[-1] + x)
    T = start[-1]
    first = [None] * P
    for u in range(units):
        s0, s1 = start[u], start[u + 1]
        c0, c1 = (s0 * P + T - 1) // T, (s1 * P + T - 1) // T
        for c in range(c0, min(c1, P)):
            first[c] = u
    return units, start, first


def walk(start, units, T, P, c, first):
    lo, hi = c * T // P, (c + 1) * T // P
    segs = []
    if lo >= hi:
        return segs
    t, u = lo, first[c]
    while t < hi:
        assert u + 1 <= units                      # start[u + 1] stays in the array
        s0, s1 = start[u], start[u + 1]
        assert s0 <= t < s1                        # the walk is on the unit holding t
        segs.append((u, t - s0, min(hi, s1) - s0))
        t = min(hi, s1)
        u += 1
    return segs


def unit_segments(start, T, P, u):
    """The CTAs that ran unit u, as the merges find them: c(t) of its first and
    last tile, skipping CTAs whose range is empty (fewer tiles than CTAs)."""
    t0, t1 = start[u], start[u + 1] - 1
    c0, c1 = ((t0 + 1) * P - 1) // T, ((t1 + 1) * P - 1) // T
    return {c for c in range(c0, c1 + 1) if c * T // P < (c + 1) * T // P}


def check(lengths, n_qtiles, Hkv, L_cap, P):
    units, start, first = plan(lengths, n_qtiles, Hkv, L_cap, P)
    T = start[-1]
    assert all(f is not None for f in first)       # every CTA has a first unit
    seen = np.zeros(T, np.int64)
    slots = set()
    ran = {u: set() for u in range(units)}
    for c in range(P):
        for u, a, b in walk(start, units, T, P, c, first):
            n_u = start[u + 1] - start[u]
            assert 0 <= a < b <= n_u
            seen[start[u] + a:start[u] + b] += 1
            slot = u + c
            assert slot not in slots and 0 <= slot < units + P - 1
            slots.add(slot)
            ran[u].add(c)
    assert (seen == 1).all()
    # an empty range lies in the CTA range [cf, cl] of at most one unit: the
    # one holding tile lo, when it starts before lo (that CTA writes an empty
    # record at slot unit + CTA for the merges)
    for c in range(P):
        lo, hi = c * T // P, (c + 1) * T // P
        if lo < hi:
            continue
        inside = [u for u in range(units)
                  if ((start[u] + 1) * P - 1) // T <= c <= (start[u + 1] * P - 1) // T]
        u0 = first[c]
        assert inside == ([u0] if start[u0] < lo else []), (c, inside, u0)
    # the fix-up's per-CTA list of completed units (a unit is completed by the
    # CTA holding its last tile) never exceeds the capacity the host sizes
    L_eff = max(L_cap, 0)
    cap = min(units, -(-units * (1 + -(-L_eff // BN)) // P) + 1)
    done = [0] * P
    for u in range(units):
        done[(start[u + 1] * P - 1) // T] += 1
    assert max(done) <= cap, (max(done), cap)
    for u in range(units):
        assert ran[u] == unit_segments(start, T, P, u), u
        # the fix-up's count of the CTAs holding a piece of the unit
        s0, s1 = start[u], start[u + 1]
        cf, cl = ((s0 + 1) * P - 1) // T, (s1 * P - 1) // T
        assert len(ran[u]) == (cl - cf + 1 if T >= P else s1 - s0), u


@pytest.mark.parametrize("lengths,n_qtiles,Hkv,L_cap,P", [
    ([4096] * 8, 1, 2, 4096, 148),            # mid: 16 units of 33 tiles
    ([8192] * 64, 1, 2, 8192, 148),           # the batch-64 loop: 128 units on 148 CTAs
    ([65536] * 4, 1, 2, 65536, 148),          # long: each unit over ~19 CTAs
    ([256], 1, 1, 256, 148),                  # tiny: 3 tiles, most CTAs idle
    ([0, 0, 0], 8, 1, 10, 148),               # empty contexts: block tiles only
    ([300, 77], 2, 1, 300, 1),                # one CTA runs everything
    ([1000, 777, 0], 1, 2, 1000, 5),
    ([-5, 70000], 1, 2, 65536, 16),           # out-of-range lengths are clamped
])
def test_schedule_cases(lengths, n_qtiles, Hkv, L_cap, P):
    check(lengths, n_qtiles, Hkv, L_cap, P)


def test_schedule_random_ragged_batches():
    rng = np.random.default_rng(5)
    for _ in range(300):
        B = int(rng.integers(1, 40))
        L_cap = int(rng.integers(0, 5000))
        lengths = rng.integers(0, L_cap + 1, B).tolist()
        check(lengths, int(rng.choice([1, 2, 8])), int(rng.choice([1, 2, 4])), L_cap,
              int(rng.integers(1, 200)))


def test_schedule_ragged_serving_batch():
    rng = np.random.default_rng(0)
    check(rng.integers(512, 32769, 128).tolist(), 2, 2, 32768, 148)
