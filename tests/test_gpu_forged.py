"""Forged records: a record changed on purpose and sealed again (its index CRC
and the header CRC recomputed, as a writer that does not follow the format
would), so that only the decoders' structural checks can refuse it. The GPU
decoders must take the oracle's decision on every such container, and where
both accept it, decode it to the oracle's values (QATQ "How it works": corrupt
or truncated input is rejected before restore; KVTC "rANS Makes the Last Mile
Smaller": the stream records these checks follow)."""
import dataclasses
import struct
import zlib

import numpy as np
import pytest

import kvgen
import oracle
import transform_codec_b200 as kvc
from kvc_gpu import decode, f32

pytestmark = pytest.mark.gpu


def _index(c, i):
    return struct.unpack_from("<QII", c, 64 + 16 * i)


def _reseal(c: bytearray, i: int) -> bytes:
    """Recompute record i's CRC in the index and the header CRC over header[0, 60) and the index."""
    n = struct.unpack_from("<I", c, 36)[0]
    off, ln, _ = _index(c, i)
    struct.pack_into("<I", c, 64 + 16 * i + 12, zlib.crc32(bytes(c[off:off + ln])))
    struct.pack_into("<I", c, 60, zlib.crc32(bytes(c[:60]) + bytes(c[64:64 + 16 * n])))
    return bytes(c)


def _streams(rec: bytes, count: int):
    """Offsets of the first `count` stream records of a record (from their byte lengths)."""
    out, o = [], 0
    for _ in range(count):
        if o + 16 > len(rec):
            break
        out.append(o)
        o += struct.unpack_from("<I", rec, o + 4)[0]
    return out


def _header_edits(base):
    """(position, new byte) pairs that rewrite the header fields of a stream record at base."""
    edits = [(base + 0, m) for m in (0, 1, 2, 3)]
    edits += [(base + 2, 0), (base + 2, 2), (base + 3, 1), (base + 3, 2)]
    edits += [(base + 4, None), (base + 8, None), (base + 12, None)]  # low byte of bytes, n, k: +-1 / +-16
    return edits


def _forgeries(c: bytes, i: int, n_streams: int, rng, n_random: int):
    """Forged copies of container c, each with one change inside record i."""
    off, ln, _ = _index(c, i)
    rec = c[off:off + ln]
    edits = []
    for o in _streams(rec, n_streams):
        edits += _header_edits(o)
        size = struct.unpack_from("<I", rec, o + 4)[0]
        if size > 16:
            edits += [(o + int(p), None) for p in rng.integers(16, size, 4)]
    edits += [(int(p), None) for p in rng.integers(0, ln, n_random)]
    for pos, val in edits:
        cc = bytearray(c)
        old = cc[off + pos]
        if val is None:
            delta = 16 if pos % 4 == 0 and rng.integers(2) else 1
            val = (old + delta) & 0xFF if rng.integers(2) else (old - delta) & 0xFF
        if val == old:
            continue
        cc[off + pos] = val
        yield pos, _reseal(cc, i)


def _close(got, want):
    """Reconstruction check for forged transform records that both sides accept:
    relative RMS 1e-3 over the values the oracle gives as finite and moderate."""
    a = f32(got).astype(np.float64)
    b = f32(want).astype(np.float64)
    keep = np.isfinite(b) & (np.abs(b) < 1e20)
    a, b = a[keep], b[keep]
    assert np.isfinite(a).all()
    err = np.sqrt(((a - b) ** 2).sum() / max((b ** 2).sum(), 1e-300))
    assert err <= 1e-3, err


def test_forged_lossless_records():
    w = kvgen.WORKLOADS["lossless-1x8x512x128-bf16"]
    x = kvgen.slices(w)
    oplan = oracle.Plan.from_workload(w)
    plan = kvc.Plan(kvc.Shape.from_workload(w))
    c = oracle.encode_lossless(oplan, x)
    rng = np.random.default_rng(21)
    seen = set()
    for i in (0, 5):
        for pos, cc in _forgeries(c, i, 2, rng, 40):
            want, wy = oracle.decode_lossless(oplan, cc)
            got, gy = decode(plan, kvc.LOSSLESS, cc, w.n_slices)
            assert got == want, (i, pos, got, want)
            if want == oracle.OK:
                assert np.array_equal(gy, wy), (i, pos)
            seen.add(want)
    assert seen == {oracle.OK, oracle.CORRUPT}  # raw-plane bytes decode to other values; the rest is refused


def test_forged_transform_records():
    base = dataclasses.replace(kvgen.WORKLOADS["transform-32x8x8192x128-bf16"], n_layers=1, n_heads=1)
    w = dataclasses.replace(base, n_tokens=1024)
    cal = kvgen.calibration(w)
    pcs = [oracle.pca(cal[s], s == 0, w.theta) for s in range(w.n_slices)]
    bases = np.stack([p[0] for p in pcs])
    lam = np.stack([p[1] for p in pcs])
    widths = oracle.allocate(lam, w.avg_bits, w.max_bits).reshape(lam.shape)
    plan = kvc.Plan(kvc.Shape.from_workload(w), bases=bases, widths=widths)
    oplan = oracle.Plan.from_workload(w, bases=bases, widths=widths)
    c = oracle.encode_transform(oplan, kvgen.slices(w))
    n_rec = struct.unpack_from("<I", c, 36)[0]
    assert n_rec == 2 * 3  # per slice: the raw record and two middle chunks
    rng = np.random.default_rng(22)
    statuses = []
    for i in (1, 2, 5):  # middle records: four side streams, then the width streams
        n_streams = 4 + len(set(widths[(i // 3)].tolist()) - {0})
        for pos, cc in _forgeries(c, i, n_streams, rng, 40):
            want, wy = oracle.decode_transform(oplan, cc)
            got, gy = decode(plan, kvc.TRANSFORM, cc, w.n_slices)
            assert got == want, (i, pos, got, want)
            if want == oracle.OK:
                _close(gy, wy)
            statuses.append(want)
    assert statuses.count(oracle.OK) < len(statuses)  # most forgeries are refused
