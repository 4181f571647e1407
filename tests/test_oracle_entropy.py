"""Pins for the oracle's integrity and entropy-coding layers (CPU only).

CRC-32 is pinned to the standard check value and to zlib; the frequency
normalisation to its invariants and hand cases; rANS to round trips, the
closed form of a uniform 2^k alphabet (exact bit packing), brute-force ideal
code lengths and the entropy bound on tiny inputs (container integrity: QATQ
page, "QATC v2 checksum validated"; entropy stage: KVTC page, "rANS Makes the
Last Mile Smaller").
"""
import math
import os
import zlib

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_kv(name):
    out = {}
    for line in open(os.path.join(GOLDEN, name)):
        line = line.strip()
        if line and not line.startswith("#"):
            k, v = line.split("=", 1)
            out[k] = v
    return out


def test_crc32_check_value():
    g = _golden_kv("crc32_check.txt")
    assert oracle.crc32(g["input_ascii"].encode()) == int(g["crc32"], 16)


@pytest.mark.parametrize("n", [0, 1, 2, 3, 15, 16, 17, 255, 4096, 100003])
def test_crc32_matches_zlib(n):
    rng = np.random.default_rng(n)
    data = rng.integers(0, 256, n, dtype=np.uint8).tobytes()
    assert oracle.crc32(data) == zlib.crc32(data)


def test_normalize_invariants_random():
    rng = np.random.default_rng(1)
    for trial in range(400):
        k = int(rng.integers(2, 257))
        syms = rng.choice(256, k, replace=False)
        counts = np.zeros(256, np.uint32)
        n = int(rng.integers(k, 70000))
        # skewed counts, every chosen symbol present
        w = rng.pareto(1.0 + rng.random(), k) + 1e-3
        c = np.maximum(1, np.floor(w / w.sum() * n)).astype(np.uint32)
        counts[syms] = c
        f, kk = oracle.normalize(counts)
        assert kk == k
        assert int(f.sum()) == 4096
        assert np.all((f > 0) == (counts > 0))
        # proportional within one slot of c*(M-k)/n + 1
        tot = int(counts.sum())
        ideal = counts.astype(np.float64) * (4096 - k) / tot + 1
        present = counts > 0
        assert np.all(np.abs(f[present] - ideal[present]) <= 1.0 + 1e-9)


def test_normalize_hand_cases():
    c = np.zeros(256, np.uint32)
    c[0], c[1] = 3, 1  # q = (12282, 4094), n = 4: f = 1 + (3070, 1023), r = (2, 2)
    f, k = oracle.normalize(c)  # d = 1 goes to the tie's smaller symbol
    assert k == 2 and f[0] == 3072 and f[1] == 1024
    c = np.zeros(256, np.uint32)
    c[7] = 10
    f, k = oracle.normalize(c)
    assert k == 1 and f[7] == 4096 and f.sum() == 4096
    c = np.zeros(256, np.uint32)
    c[[2, 5, 9]] = [1, 1, 1]  # q = 4093 each, n = 3: f = 1 + 1364, r = 1 each; d = 1
    f, k = oracle.normalize(c)
    assert (f[2], f[5], f[9]) == (1366, 1365, 1365)
    for kbits in range(1, 9):  # equal counts over 2^k symbols: exactly uniform
        c = np.zeros(256, np.uint32)
        c[: 1 << kbits] = 37
        f, _ = oracle.normalize(c)
        assert np.all(f[: 1 << kbits] == 4096 >> kbits) and np.all(f[1 << kbits:] == 0)


def test_normalize_remainder_not_on_largest_count():
    """Hand-worked tables where the slots left over go to the largest
    remainders, not to the largest counts (a rule that hands them to the
    largest counts fails both)."""
    c = np.zeros(256, np.uint32)
    c[[0, 1, 2]] = [10, 3, 2]
    # n = 15, k = 3, M - k = 4093: c (M - k) = 40930, 12279, 8186
    # floor / 15 = 2728, 818, 545 -> f = 2729, 819, 546 (sum 4094, d = 2)
    # remainders mod 15 = 10, 9, 11 -> symbols 2 and 0 take one more each
    f, k = oracle.normalize(c)
    assert k == 3 and (f[0], f[1], f[2]) == (2730, 819, 547)
    c = np.zeros(256, np.uint32)
    c[[0, 1, 2]] = [1, 2, 10]
    # n = 13: c (M - k) = 4093, 8186, 40930; floor / 13 = 314, 629, 3148
    # -> f = 315, 630, 3149 (sum 4094, d = 2 = k - 1); remainders 11, 9, 6:
    # the two smaller counts round up, the largest count stays
    f, k = oracle.normalize(c)
    assert k == 3 and (f[0], f[1], f[2]) == (316, 631, 3149)
    c = np.zeros(256, np.uint32)
    c[[40, 41, 200, 201]] = [7, 5, 5, 1]
    # n = 18, k = 4, M - k = 4092: c (M - k) = 28644, 20460, 20460, 4092
    # floor / 18 = 1591, 1136, 1136, 227 -> f = 1592, 1137, 1137, 228
    # (sum 4094, d = 2); remainders 6, 12, 12, 6: the tie at 12 takes both
    f, k = oracle.normalize(c)
    assert k == 4 and (f[40], f[41], f[200], f[201]) == (1592, 1138, 1138, 228)
    c = np.zeros(256, np.uint32)
    c[[3, 9, 250]] = [4, 4, 4]
    # equal counts, n = 12: 16372 / 12 = 1364 r 4 -> 1365 each (sum 4095),
    # d = 1, equal remainders: the smallest symbol takes it
    f, k = oracle.normalize(c)
    assert (f[3], f[9], f[250]) == (1366, 1365, 1365)


def test_normalize_quota_property():
    """Every present symbol gets 1 + floor(q) or 1 + ceil(q) of its quota
    q = c (M - k) / n; exactly M - sum(1 + floor(q)) symbols round up, and no
    symbol left at its floor has a larger remainder than one that rounded up
    (nor an equal remainder and a smaller symbol): the defining property of
    largest-remainder apportionment, checked with exact rationals."""
    from fractions import Fraction
    rng = np.random.default_rng(11)
    for trial in range(300):
        k = int(rng.integers(2, 257))
        counts = np.zeros(256, np.uint32)
        syms = rng.choice(256, k, replace=False)
        counts[syms] = rng.integers(1, int(rng.choice([3, 50, 5000])), k)
        n = int(counts.sum())
        f, kk = oracle.normalize(counts)
        assert kk == k
        q = {s: Fraction(int(counts[s]) * (4096 - k), n) for s in map(int, syms)}
        fl = {s: q[s].numerator // q[s].denominator for s in q}
        up = {s for s in q if int(f[s]) == 2 + fl[s]}
        assert all(int(f[s]) in (1 + fl[s], 2 + fl[s]) for s in q)
        assert len(up) == 4096 - sum(1 + fl[s] for s in q)
        down = set(q) - up
        for u in up:
            ru = q[u] - fl[u]
            for s in down:
                rs = q[s] - fl[s]
                assert rs < ru or (rs == ru and s > u)


@pytest.mark.parametrize("seed", range(6))
def test_normalize_equals_textbook_apportionment(seed):
    """The oracle's table equals Hamilton's largest-remainder method restated
    with exact rationals in tests/apportion.py, on skewed, flat, tiny and
    one-dominant count vectors."""
    from apportion import largest_remainder
    rng = np.random.default_rng(100 + seed)
    for trial in range(150):
        counts = np.zeros(256, np.uint32)
        k = int(rng.integers(1, 257))
        syms = rng.choice(256, k, replace=False)
        kind = trial % 4
        if kind == 0:
            counts[syms] = np.minimum(rng.geometric(0.05, k), 65536)
        elif kind == 1:
            counts[syms] = rng.integers(1, 4, k)
        elif kind == 2:
            counts[syms] = 1
            counts[syms[0]] = int(rng.integers(1, 65536))
        else:
            counts[syms] = rng.integers(1, 65536 // k + 2, k)
        f, kk = oracle.normalize(counts)
        want, wk = largest_remainder(counts)
        assert kk == wk
        assert f.astype(int).tolist() == want


def _roundtrip(sym):
    rec = oracle.stream_encode(sym)
    assert len(rec) % 16 == 0 and len(rec) <= 16 + (len(sym) + 15) // 16 * 16
    st, out, used = oracle.stream_decode(rec, len(sym))
    assert st == oracle.OK and used == len(rec)
    assert np.array_equal(out, sym)
    return rec


@pytest.mark.parametrize("n", [1, 2, 100, 511, 512, 513, 1023, 1024, 1025, 4095, 16384,
                               33333, 65535, 65536])
@pytest.mark.parametrize("dist", ["geom", "two", "uniform16", "random"])
def test_stream_roundtrip(n, dist):
    rng = np.random.default_rng(n * 7 + len(dist))
    if dist == "geom":
        sym = np.minimum(rng.geometric(0.3, n) - 1, 255).astype(np.uint8)
    elif dist == "two":
        sym = np.where(rng.random(n) < 0.99, 17, 200).astype(np.uint8)
    elif dist == "uniform16":
        sym = rng.integers(0, 16, n).astype(np.uint8)
    else:
        sym = rng.integers(0, 256, n).astype(np.uint8)
    rec = _roundtrip(sym)
    distinct = len(np.unique(sym))
    if distinct == 1:
        assert rec[0] == 1 and len(rec) == 16
    elif dist == "random" and n >= 4096:
        assert rec[0] == 0  # incompressible: raw fallback


def test_stream_const_and_raw_layout():
    rec = oracle.stream_encode(np.full(1000, 9, np.uint8))
    assert rec == bytes([1, 9, 0, 0]) + (16).to_bytes(4, "little") + (1000).to_bytes(4, "little") \
        + (1).to_bytes(4, "little")
    sym = np.array([5, 1, 4, 2], np.uint8)
    rec = oracle.stream_encode(sym)  # 4 distinct in 4: raw is smaller
    assert rec == bytes([0, 0, 0, 0]) + (32).to_bytes(4, "little") + (4).to_bytes(4, "little") \
        + bytes(4) + bytes([5, 1, 4, 2]) + bytes(12)


def _lanes(n):
    N = min(128, max(1, n // 512))
    base, extra = divmod(n, N)
    return [base + (l < extra) for l in range(N)]


@pytest.mark.parametrize("kbits", [1, 2, 3, 4, 5, 6, 7, 8])
@pytest.mark.parametrize("reps", [1, 3, 40, 257])
def test_rans_uniform_alphabet_is_bit_packing(kbits, reps):
    """With f = 2^(12-k) for all 2^k symbols, coding one symbol inserts exactly
    k bits into the state, so a lane of len symbols starting from the 17-bit
    state 2^16 holds 17 + k*len bits; the final state keeps 17..32 of them and
    the rest leave as 16-bit words: payload = sum_lanes (4 + 2*floor(k*len/16))."""
    rng = np.random.default_rng(kbits * 1000 + reps)
    sym = np.repeat(np.arange(1 << kbits, dtype=np.uint8), reps)
    rng.shuffle(sym)
    n = sym.size
    expect = sum(4 + 2 * ((kbits * ln) // 16) for ln in _lanes(n))
    assert oracle.rans_payload_bytes(sym) == expect
    _roundtrip(sym)


def _entropy_bits(sym):
    _, c = np.unique(sym, return_counts=True)
    n = sym.size
    return float(-(c * np.log2(c / n)).sum())


def _tiny_cases():
    rng = np.random.default_rng(5)
    cases = []
    for n in [16, 100, 257, 512, 777, 1023]:
        cases.append(("uniform", rng.integers(0, 256, n).astype(np.uint8)))
        cases.append(("uniform8", rng.integers(0, 8, n).astype(np.uint8)))
        cases.append(("geometric", np.minimum(rng.geometric(0.25, n) - 1, 255).astype(np.uint8)))
        z = rng.zipf(1.5, n)
        cases.append(("zipf", np.minimum(z - 1, 255).astype(np.uint8)))
        cases.append(("p0.99", np.where(rng.random(n) < 0.99, 3, 4).astype(np.uint8)))
        cases.append(("random", rng.integers(0, 256, n).astype(np.uint8)))
    return cases


@pytest.mark.parametrize("name,sym", _tiny_cases())
def test_rans_within_entropy_bound_on_tiny_inputs(name, sym):
    """rANS size (states + words) within 0.5% + 16 bytes of the exact empirical
    entropy for n <= 1023 symbols (one lane, 4-byte state flush)."""
    if len(np.unique(sym)) < 2:
        pytest.skip("single symbol: CONST stream, no rANS payload")
    payload = oracle.rans_payload_bytes(sym)
    h = _entropy_bits(sym)
    assert payload <= 1.005 * h / 8 + 16, (name, payload, h / 8)


@pytest.mark.parametrize("name,sym", _tiny_cases()[:18])
def test_rans_matches_ideal_code_length(name, sym):
    """Brute force: sum of -log2(f_s/4096) over the symbols, with the table the
    coder uses, is the ideal length; rANS must be within its state overhead."""
    if len(np.unique(sym)) < 2:
        pytest.skip("single symbol")
    counts = np.bincount(sym, minlength=256).astype(np.uint32)
    f, _ = oracle.normalize(counts)
    ideal = float(-np.log2(f[sym].astype(np.float64) / 4096).sum())
    bits = 8 * oracle.rans_payload_bytes(sym)
    assert ideal - 1 <= bits <= ideal + 32 + 16, (name, bits, ideal)


def test_stream_decoder_refuses_bad_records():
    rng = np.random.default_rng(9)
    sym = np.minimum(rng.geometric(0.2, 5000) - 1, 255).astype(np.uint8)
    rec = bytearray(oracle.stream_encode(sym))
    assert rec[0] == 2
    # wrong symbol count, truncated record, bad mode, broken frequency total
    assert oracle.stream_decode(bytes(rec), 4999)[0] != oracle.OK
    assert oracle.stream_decode(bytes(rec[:-16]), 5000)[0] != oracle.OK
    bad = bytearray(rec); bad[0] = 7
    assert oracle.stream_decode(bytes(bad), 5000)[0] != oracle.OK
    bad = bytearray(rec); bad[48] ^= 1
    assert oracle.stream_decode(bytes(bad), 5000)[0] != oracle.OK
    # flipped payload bits must not decode silently to the same length stream
    refused = 0
    for pos in range(len(rec) - 200, len(rec)):
        bad = bytearray(rec); bad[pos] ^= 0x5A
        st, out, _ = oracle.stream_decode(bytes(bad), 5000)
        refused += (st != oracle.OK) or (not np.array_equal(out, sym))
    assert refused > 150


def test_rans_words_lower_bound():
    """A lower bound on the words of an rANS record, used by the GPU side
    encoder to skip a variant that cannot beat RAW. Before each coding step the
    state x is at least 16 f (after renormalisation), so a step multiplies x by
    more than (M / f)(15/16); an emitted word removes at most 16 + log2(16/15)
    bits; the N final states hold at most 16 bits each beyond their start; and
    sum_s c_s log2(M / f_s) >= n H (Gibbs) for the empirical entropy H. Hence
    W >= (n H - n log2(16/15) - 16 N) / (16 + log2(16/15)). Checked on skewed,
    uniform, heavy-tailed and sorted streams, with the kernel's margins too."""
    rng = np.random.default_rng(17)
    d = math.log2(16 / 15)
    for trial in range(250):
        n = int(rng.integers(2, 70000))
        kind = trial % 5
        if kind == 0:
            s = rng.integers(0, int(rng.integers(2, 257)), n)
        elif kind == 1:
            s = np.minimum(rng.geometric(float(rng.uniform(0.05, 0.9)), n) - 1, 255)
        elif kind == 2:
            s = np.minimum(rng.zipf(1.5, n) - 1, 255)
        elif kind == 3:
            s = np.where(rng.random(n) < 0.99, 0, rng.integers(1, 256, n))
        else:
            s = np.sort(rng.integers(0, 256, n))
        s = s.astype(np.uint8)
        payload = oracle.rans_payload_bytes(s)
        if payload == 0:
            continue
        N = min(128, max(1, n // 512))
        W = (payload - 4 * N) / 2
        _, c = np.unique(s, return_counts=True)
        H = float((c * np.log2(n / c)).sum())
        assert W >= (H - d * n - 16 * N) / (16 + d) - 1e-9, (trial, n, kind)
        assert W >= (H * 0.9999 - 2.0 - 0.0932 * n - 16.0 * N) / (16.0 + 0.0932)  # the kernel's form
