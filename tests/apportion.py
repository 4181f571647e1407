"""Largest-remainder apportionment (Hamilton's method), written in the tests
from its textbook definition with exact rational arithmetic, independent of
the oracle's integer code.

The codec's frequency table gives each of the k present symbols one slot and
shares the other M - k slots out of M = 4096 in proportion to the counts: the
quota of symbol s is q_s = c_s (M - k) / n, every present symbol takes
1 + floor(q_s), and the slots left over go one each to the symbols with the
largest fractional parts q_s - floor(q_s), ties to the smaller symbol (the
table that drives the coder of the KVTC page, "rANS Makes the Last Mile
Smaller"; the pages fix no rule, this is the codec's)."""
from fractions import Fraction

M = 4096


def largest_remainder(counts):
    counts = [int(c) for c in counts]
    present = [s for s, c in enumerate(counts) if c > 0]
    k, n = len(present), sum(counts)
    f = [0] * len(counts)
    if k == 0:
        return f, 0
    if k == 1:
        f[present[0]] = M
        return f, 1
    quota = {s: Fraction(counts[s] * (M - k), n) for s in present}
    for s in present:
        f[s] = 1 + quota[s].numerator // quota[s].denominator
    left = M - sum(f)
    order = sorted(present, key=lambda s: (-(quota[s] - (quota[s].numerator // quota[s].denominator)), s))
    for s in order[:left]:
        f[s] += 1
    return f, k
