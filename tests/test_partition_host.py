"""Host model of the stream-K partition of the decode stream kernel and of
the finish kernel's record lookup, checked on random ragged batches.

All quantised pages of all (sequence, head) pairs form one unit list; each
pair's units are its pages led by SETUP units. CTA c of n takes units
[U*c/n, U*(c+1)/n); every (pair, CTA) overlap is a segment whose record goes
to slot pair + c. The finish kernel of a pair reads slots pair + c for
c in [c_first, c_last], computed from the pair's first unit alone. These
tests restate those formulas and check the two properties the design rests
on: no two segments share a slot (and all slots fit pairs + max CTAs), and
the finish kernel's range is exactly the set of CTAs that wrote the pair."""

import numpy as np
import pytest

SETUP = 16          # units charged for a segment's setup (kSegmentUnits)
MAX_CTAS = 256      # record slots beyond the pairs (kMaxStreamCtas)


def pair_units(pages):
    return pages + SETUP if pages > 0 else 0


def segments(seq_pages, Hq, n_cta):
    """(pair, cta, first page, end page) of every segment, walking each CTA's range."""
    units = [(b, hq, pair_units(p)) for b, p in enumerate(seq_pages) for hq in range(Hq)]
    starts = np.cumsum([0] + [u for _, _, u in units])
    U = int(starts[-1])
    out = []
    for c in range(n_cta):
        lo, hi = U * c // n_cta, U * (c + 1) // n_cta
        for k, (b, hq, u) in enumerate(units):
            a, z = int(starts[k]), int(starts[k]) + u
            if u == 0 or z <= lo or a >= hi:
                continue
            pu0, pu1 = max(lo, a) - a, min(hi, z) - a          # units inside the pair
            out.append((b * Hq + hq, c, max(pu0 - SETUP, 0), max(pu1 - SETUP, 0)))
    return out, U


def finish_range(seq_pages, Hq, n_cta, b, hq, U):
    before = sum(pair_units(p) for p in seq_pages[:b])
    ub = pair_units(seq_pages[b])
    u0 = before * Hq + hq * ub
    return ((u0 + 1) * n_cta - 1) // U, ((u0 + ub) * n_cta - 1) // U


@pytest.mark.parametrize("seed", range(40))
def test_record_slots_are_unique_and_found_by_the_finish_kernel(seed):
    rng = np.random.default_rng(seed)
    B = int(rng.integers(1, 12))
    Hq = int(rng.integers(1, 6))
    seq_pages = [int(p) for p in rng.integers(0, 40, size=B)]
    if rng.random() < 0.3:
        seq_pages[int(rng.integers(0, B))] = 0
    if sum(seq_pages) == 0:
        seq_pages[0] = 1
    n_cta = int(rng.integers(1, MAX_CTAS + 1))
    segs, U = segments(seq_pages, Hq, n_cta)
    n_cta = min(n_cta, U)                    # the launcher never starts more CTAs than units
    segs, U = segments(seq_pages, Hq, n_cta)
    slots = [pair + c for pair, c, _, _ in segs]
    assert len(slots) == len(set(slots))
    assert max(slots) < B * Hq + MAX_CTAS
    # every page of every pair is streamed by exactly one segment
    for b in range(B):
        for hq in range(Hq):
            pair = b * Hq + hq
            got = sorted((p0, p1) for pr, _, p0, p1 in segs if pr == pair and p1 > p0)
            covered = [pg for p0, p1 in got for pg in range(p0, p1)]
            assert covered == list(range(seq_pages[b]))
            if seq_pages[b] == 0:
                continue
            c_first, c_last = finish_range(seq_pages, Hq, n_cta, b, hq, U)
            writers = {c for pr, c, _, _ in segs if pr == pair}
            nonempty = {c for c in range(c_first, c_last + 1)
                        if U * c // n_cta < U * (c + 1) // n_cta}
            assert writers == nonempty
