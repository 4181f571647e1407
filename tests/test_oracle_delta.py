"""Pins of the oracle's lane-delta candidate (QATQ "How it works": delta-XOR,
native 16-bit adjacent-XOR and shape-aware strided-XOR among the lossless
candidates; this codec's reading applies the XOR with the previous token of
the same channel within each rANS lane's range, on every byte plane of
lossless chunks)."""
import numpy as np
import pytest

import kvgen
import oracle


def _lane_ranges(n):
    """Contiguous lane ranges of a stream of n symbols (the stream format)."""
    N = min(128, max(1, n // 512))
    base, extra = divmod(n, N)
    out, start = [], 0
    for l in range(N):
        ln = base + (1 if l < extra else 0)
        out.append((start, ln))
        start += ln
    return out


SIZES = [1, 2, 511, 512, 1023, 1024, 1537, 65536, 70001]


@pytest.mark.parametrize("n", SIZES)
def test_lane_constant_sequence_deltas_to_lane_starts(n):
    """Closed form: a sequence constant on every lane has, after the delta,
    its lane's value at each lane start and zero everywhere else."""
    rng = np.random.default_rng(n)
    x = np.zeros(n, np.uint8)
    starts = []
    for start, ln in _lane_ranges(n):
        x[start:start + ln] = rng.integers(1, 256)
        starts.append(start)
    d = oracle.lane_delta(x)
    mask = np.zeros(n, bool)
    mask[starts] = True
    assert np.array_equal(d[mask], x[mask])
    assert not d[~mask].any()


@pytest.mark.parametrize("n", SIZES)
def test_undelta_inverts_delta(n):
    rng = np.random.default_rng(100 + n)
    x = rng.integers(0, 256, n).astype(np.uint8)
    assert np.array_equal(oracle.lane_undelta(oracle.lane_delta(x)), x)


def _random_walk(rng, n, step=3):
    return (np.cumsum(rng.integers(-step, step + 1, n)) % 256).astype(np.uint8)


@pytest.mark.parametrize("n", [1024, 4096, 65536])
def test_delta_chosen_only_when_strictly_smaller(n):
    rng = np.random.default_rng(7)
    smooth = _random_walk(rng, n)
    plain = oracle.stream_encode(smooth)
    rec = oracle.stream_encode_delta(smooth)
    assert rec[3] == 1 and rec[0] == 2  # RANS of lane deltas
    assert len(rec) < len(plain)
    st, y, used = oracle.stream_decode(rec, n)
    assert st == oracle.OK and used == len(rec) and np.array_equal(y, smooth)
    # independent symbols: the delta cannot win, the plain record comes out byte for byte
    iid = rng.choice(8, size=n, p=[.4, .2, .1, .1, .08, .06, .04, .02]).astype(np.uint8)
    assert oracle.stream_encode_delta(iid) == oracle.stream_encode(iid)
    uni = rng.integers(0, 256, n).astype(np.uint8)
    assert oracle.stream_encode_delta(uni) == oracle.stream_encode(uni)


def test_delta_never_worse_and_constant_planes():
    rng = np.random.default_rng(9)
    for n in [1, 3, 600, 5000]:
        for x in [np.full(n, 7, np.uint8), _random_walk(rng, n, 1), rng.integers(0, 256, n).astype(np.uint8)]:
            rec = oracle.stream_encode_delta(x)
            assert len(rec) <= len(oracle.stream_encode(x)) <= 16 + (n + 15) // 16 * 16
            st, y, _ = oracle.stream_decode(rec, n)
            assert st == oracle.OK and np.array_equal(y, x)


def test_flag_only_on_rans_records():
    x = np.full(100, 9, np.uint8)
    rec = bytearray(oracle.stream_encode_delta(x))  # CONST
    rec[3] = 1
    assert oracle.stream_decode(bytes(rec), 100)[0] == oracle.CORRUPT
    raw = bytearray(oracle.stream_encode(np.arange(100, dtype=np.uint8)))  # RAW
    raw[3] = 1
    assert oracle.stream_decode(bytes(raw), 100)[0] == oracle.CORRUPT


def test_lossless_workload_high_planes_take_the_delta():
    """The AR(1) workloads' high byte planes are smooth along tokens: the
    lossless containers carry lane-delta records, and round-trip."""
    w = kvgen.WORKLOADS["lossless-1x8x512x128-bf16"]
    plan = oracle.Plan.from_workload(w)
    x = kvgen.slices(w)
    c = oracle.encode_lossless(plan, x)
    n = int.from_bytes(c[36:40], "little")
    flags = []
    for i in range(n):
        e = 64 + 16 * i
        off = int.from_bytes(c[e:e + 8], "little")
        b0 = int.from_bytes(c[off + 4:off + 8], "little")
        flags.append((c[off + 3], c[off + b0 + 3]))
    assert all(f0 == 0 for f0, _ in flags)
    assert sum(f1 for _, f1 in flags) > 0
    st, y = oracle.decode_lossless(plan, c)
    assert st == oracle.OK and np.array_equal(y[:w.n_slices], x)


def _plane_records(c):
    """(offset, length) of every stream record of every chunk of a lossless
    container, in order."""
    import struct
    n_rec = struct.unpack_from("<I", c, 36)[0]
    out = []
    for r in range(n_rec):
        off, ln, _ = struct.unpack_from("<QII", c, 64 + 16 * r)
        p = off
        while p < off + ln:
            b = struct.unpack_from("<I", c, p + 4)[0]
            out.append((p, b))
            p += b
    return out


def test_low_plane_takes_the_delta_where_it_is_smaller():
    """16-bit XOR with the previous token of the channel: a ramp along tokens
    (value = 3 t + 17 c, fp16 bits) changes its low byte by a few steps per
    token, so the low plane's lane deltas compress far below its plain RANS
    record; the low plane takes the delta flag too, and the round trip holds."""
    w = kvgen.Workload("ramp", "lossless", 2, 1, 1, 1024, 64, 0.9, 1e4, 0)
    t = np.arange(1024)[:, None]
    ch = np.arange(64)[None, :]
    x = ((3 * t + 17 * ch + 4096) & 0xFFFF).astype(np.uint16)[None].repeat(2, 0)
    plan = oracle.Plan.from_workload(w)
    c = oracle.encode_lossless(plan, x)
    recs = _plane_records(c)
    assert len(recs) == 2 * 2  # two slices, one chunk each, two planes
    low = [recs[0], recs[2]]
    plane0 = np.ascontiguousarray(x[0].T).ravel() & 0xFF  # channel-major low bytes of a slice
    plain = oracle.stream_encode(plane0.astype(np.uint8))
    for off, ln in low:
        assert c[off] == 2 and c[off + 3] == 1  # RANS of lane deltas on the low plane
        assert ln < len(plain) and ln < (16 + 65536) // 2  # below the plain record and half of RAW
    st, y = oracle.decode_lossless(plan, c)
    assert st == oracle.OK and np.array_equal(y, x)


def _sq(a):
    c = np.bincount(np.asarray(a, np.int64), minlength=256)
    return int((c * c).sum())


def _lane_delta(sym):
    d = sym.copy()
    for a, ln in _lane_ranges(sym.size):
        d[a + 1:a + ln] = sym[a + 1:a + ln] ^ sym[a:a + ln - 1]
    return d


@pytest.mark.parametrize("kind", ["noise", "walk", "ramp", "runs"])
@pytest.mark.parametrize("n", [600, 4096, 65536])
def test_delta_gate_by_concentration(kind, n):
    """The lossless planes code the lane-delta candidate only when the deltas'
    squared counts sum strictly above the plane's and 181 times that sum
    exceeds n^2 (collision entropy under log2(181) bits; computed here from the
    tests' own lane ranges); otherwise the record is the plain one byte for
    byte, and with the gate open it is the plain or delta record, whichever
    the strict never-worse rule keeps."""
    rng = np.random.default_rng(n + len(kind))
    if kind == "noise":
        sym = rng.integers(0, 256, n).astype(np.uint8)
    elif kind == "walk":
        sym = (np.cumsum(rng.integers(-1, 2, n)) % 256).astype(np.uint8)
    elif kind == "ramp":
        sym = ((3 * np.arange(n)) % 256).astype(np.uint8)
    else:
        sym = np.repeat(rng.integers(0, 256, n // 16 + 1), 16)[:n].astype(np.uint8)
    rec = oracle.stream_encode_delta(sym)
    plain = oracle.stream_encode(sym)
    qd = _sq(_lane_delta(sym))
    if not (qd > _sq(sym) and 181 * qd > n * n):
        assert rec == plain
    else:
        assert rec[3] in (0, 1)
        assert len(rec) <= len(plain)
        if rec[3] == 1:
            assert len(rec) < len(plain)
    st, out, used = oracle.stream_decode(rec, n)
    assert st == oracle.OK and used == len(rec) and np.array_equal(out, sym)
