"""Packing of a record's rANS groups into warps, checked over every width mix
(CPU only).

A record's width streams (KVTC, "Bit Budget Is Not Fair": one stream per bit
width; "rANS Makes the Last Mile Smaller": each entropy coded) hold at most
128 rANS lanes in all, over at most eight streams, in groups of at most 32
lanes. Both transform entropy stages place those groups in warps of 32 lanes:
larger groups first, each into the first of warps 0..6 with room, warp 7
otherwise, without looking at warp 7's fill. Each group gets a refill ring
of 16 words per lane rounded up to a power of two, and the record's tables
hold at most 12 groups. This file checks, for every multiset of group sizes
the lane rule can produce, that warp 7 never overflows, and that the group
count and ring words stay within those tables.
"""
import numpy as np

LANES = 128      # rANS lanes of a record, at most
GROUP = 32       # lanes of a group, at most
STREAMS = 8      # width streams (bits 1..8)
WARPS = 8
MAX_GROUPS = 12  # entries of the record's packing table
RING_WORDS = 4096


def _lanes(n_symbols: int) -> int:
    """The code streams' lane rule: one lane per 512 symbols, 1 to 128."""
    return min(max(n_symbols // 512, 1), LANES)


def _groups(lanes: int) -> list[int]:
    return [min(GROUP, lanes - g) for g in range(0, lanes, GROUP)]


def _partitions(max_sum: int, k: int, largest: int) -> np.ndarray:
    """Every nonincreasing k-tuple of parts in [1, largest] with sum <= max_sum,
    one per row."""
    if k == 0:
        return np.zeros((1, 0), np.int16)
    rows = np.arange(min(largest, max_sum - (k - 1)), 0, -1, dtype=np.int16)[:, None]
    for i in range(1, k):
        used = rows.sum(axis=1, dtype=np.int32)
        cap = np.minimum(rows[:, -1].astype(np.int32), max_sum - used - (k - 1 - i))
        cap = np.maximum(cap, 0)
        rep = np.repeat(np.arange(rows.shape[0]), cap)
        start = np.repeat(np.cumsum(cap) - cap, cap)
        nxt = (np.repeat(cap, cap) - (np.arange(rep.size) - start)).astype(np.int16)
        rows = np.concatenate([rows[rep], nxt[:, None]], axis=1)
    return rows


def _pack(sizes: np.ndarray, warps: int = WARPS) -> np.ndarray:
    """The fills of each warp after placing groups (rows of sizes, largest
    first) into the first of warps 0..warps-2 with room, the last otherwise."""
    fill = np.zeros((sizes.shape[0], warps), np.int32)
    rows = np.arange(sizes.shape[0])
    for i in range(sizes.shape[1]):
        L = sizes[:, i].astype(np.int32)
        fits = fill[:, :warps - 1] + L[:, None] <= GROUP
        w = np.where(fits.any(axis=1), fits.argmax(axis=1), warps - 1)
        fill[rows, w] += L
    return fill


def _mixes(warps: int = WARPS):
    """Group-size multisets, largest first, of every width mix that could need
    more than warps - 1 warps before the last one: F full groups of 32 lanes and
    k remainder groups (at most one per stream) with F + k >= warps. Any mix
    with fewer groups puts at most one group in the last warp."""
    for F in range(LANES // GROUP + 1):
        for k in range(max(warps - F, 1), STREAMS + 1):
            rem = _partitions(LANES - GROUP * F, k, GROUP - 1)
            if rem.shape[0]:
                full = np.full((rem.shape[0], F), GROUP, np.int16)
                yield F, k, np.concatenate([full, rem], axis=1)


def test_partitions_are_complete():
    """The enumeration against brute force on small cases."""
    import itertools
    for max_sum, k, largest in ((10, 3, 5), (12, 4, 4), (7, 1, 31), (9, 5, 3)):
        want = {tuple(sorted(c, reverse=True))
                for c in itertools.product(range(1, largest + 1), repeat=k) if sum(c) <= max_sum}
        got = _partitions(max_sum, k, largest)
        assert len(got) == len(want) and {tuple(r) for r in got.tolist()} == want


def test_lane_rule_keeps_every_record_within_128_lanes_in_8_streams():
    """A stream of m components over a chunk of 1 to 512 tokens has at most m
    lanes, so the streams of a record's 128 components hold at most 128."""
    for m in range(1, 129):
        for tcc in range(1, 513):
            assert _lanes(m * tcc) <= m
    rng = np.random.default_rng(5)
    for _ in range(500):  # and their groups fill at most 11 entries
        tcc = int(rng.integers(1, 513))
        comps = rng.multinomial(128, rng.dirichlet(np.ones(STREAMS) * 0.3))
        lanes = [_lanes(int(m) * tcc) for m in comps if m]
        assert len(lanes) <= STREAMS and sum(lanes) <= LANES
        assert sum(len(_groups(L)) for L in lanes) <= MAX_GROUPS - 1


def test_last_warp_never_overflows():
    n_cases = 0
    for F, k, sizes in _mixes():
        fill = _pack(sizes)
        assert fill[:, -1].max() <= GROUP, (F, k, sizes[fill[:, -1].argmax()])
        assert (fill.sum(axis=1) == sizes.sum(axis=1, dtype=np.int32)).all()
        assert F + k <= MAX_GROUPS - 1
        n_cases += sizes.shape[0]
    assert n_cases > 7_000_000


def test_ring_words_fit():
    """16 words per lane rounded up to a power of two: pow2ceil(L) <= 2L - 1
    for every group size, so a record's rings take at most 16 (2 * 128 - 1)
    words."""
    for L in range(1, GROUP + 1):
        p2 = 1 << (L - 1).bit_length()
        assert L <= p2 <= 2 * L - 1
    assert 16 * (2 * LANES - 1) <= RING_WORDS


def test_two_warps_fewer_would_overflow():
    """Six warps are too few: six groups of 17 lanes open warps 0..4 and fill
    the last, and a group of 16 then overflows it (118 lanes in all). The
    fill check above sees such a placement."""
    sizes = np.array([[17] * 6 + [16]], np.int16)
    assert sizes.sum() <= LANES
    assert _pack(sizes, warps=6)[0, -1] == 33
    assert _pack(sizes)[0, -1] <= GROUP
