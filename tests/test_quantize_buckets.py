"""A property of the NF4 levels that the GPU quantiser's bucket lookup relies
on: split [-1, 1] into 32 buckets of width 1/16. Each of the 15 decision
thresholds (the level midpoints) then lies in its own bucket, at least 2^-10
from every bucket boundary. So the count of thresholds below a bucket plus
one compare with the single threshold inside it gives the code. An element
whose bucket index is off by one, from the rounding of p + 3, still gets the
right code. (The levels are the oracle's, pinned to the pages elsewhere.)"""
from fractions import Fraction

import oracle


def test_thresholds_one_per_sixteenth_and_clear_of_boundaries():
    lv = [Fraction(float(v)) for v in oracle.levels()]
    mids = [(a + b) / 2 for a, b in zip(lv, lv[1:])]
    assert len(mids) == 15
    buckets = [int((m + 1) * 16) for m in mids]          # floor: every midpoint is inside (-1, 1)
    assert len(set(buckets)) == 15                         # no bucket holds two
    for m in mids:
        nearest = min(abs(m - (Fraction(k, 16) - 1)) for k in range(33))
        assert nearest >= Fraction(1, 1024)
