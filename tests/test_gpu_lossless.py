"""Lossless path on the GPU against the oracle: the GPU container must be the
oracle's container byte for byte, the GPU decoder must restore the oracle's
containers exactly, and damaged or truncated containers must be refused with
the oracle's status."""
import dataclasses

import numpy as np
import pytest

import kvgen
import oracle
import transform_codec_b200 as kvc
from kvc_gpu import decode, encode

pytestmark = pytest.mark.gpu


def _w(name, **kw):
    return dataclasses.replace(kvgen.WORKLOADS[name], **kw)


CASES = [
    _w("lossless-1x8x512x128-bf16"),
    _w("lossless-1x8x512x128-bf16", n_tokens=700),
    _w("lossless-12x12x1024x64-fp16", n_layers=1, n_heads=3, n_tokens=1500),
    _w("lossless-1x8x512x128-bf16", n_tokens=3, head_dim=10, values_per_chunk=16),
    _w("lossless-1x8x512x128-bf16", n_tokens=1000, head_dim=24, values_per_chunk=4096),
    _w("lossless-8x8x1536x128-bf16", n_layers=1, n_heads=2),
    _w("lossless-12x12x1024x64-fp16", n_layers=2, n_heads=2),
]


def _plans(w):
    s = kvc.Shape.from_workload(w)
    return kvc.Plan(s), oracle.Plan.from_workload(w)


@pytest.mark.parametrize("w", CASES, ids=lambda w: f"{w.n_layers}x{w.n_heads}x{w.n_tokens}x{w.head_dim}")
def test_lossless_parity(w):
    plan, oplan = _plans(w)
    x = kvgen.slices(w)
    want = oracle.encode_lossless(oplan, x)
    st, got = encode(plan, kvc.LOSSLESS, x)
    assert st == kvc.OK
    assert len(got) == len(want)
    assert got == want
    st, y = decode(plan, kvc.LOSSLESS, want, w.n_slices)
    assert st == kvc.OK and np.array_equal(y, x)


def test_lossless_subrange_and_empty():
    w = _w("lossless-1x8x512x128-bf16")
    plan, oplan = _plans(w)
    x = kvgen.slices(w, first=5, n=3)
    st, got = encode(plan, kvc.LOSSLESS, x, first_slice=5)
    assert st == kvc.OK and got == oracle.encode_lossless(oplan, x, first_slice=5)
    st, y = decode(plan, kvc.LOSSLESS, got, 3)
    assert st == kvc.OK and np.array_equal(y, x)
    e = np.zeros((0, w.n_tokens, w.head_dim), np.uint16)
    st, got = encode(plan, kvc.LOSSLESS, e)
    assert st == kvc.OK and got == oracle.encode_lossless(oplan, e)
    st, y = decode(plan, kvc.LOSSLESS, got, 1)
    assert st == kvc.OK and y.shape[0] == 0


def test_random_control_block_takes_raw():
    raw = kvgen.random_bytes(4 << 20)
    w = _w("lossless-12x12x1024x64-fp16", n_layers=1, n_heads=1, n_tokens=16384)
    plan, oplan = _plans(w)
    x = raw.view(np.uint16).reshape(2, 16384, 64)
    st, got = encode(plan, kvc.LOSSLESS, x)
    assert st == kvc.OK
    assert len(got) == raw.size + 64 + 48 * 32
    assert got == oracle.encode_lossless(oplan, x)
    st, y = decode(plan, kvc.LOSSLESS, got, 2)
    assert st == kvc.OK and np.array_equal(y, x)


def test_special_bit_patterns():
    rng = np.random.default_rng(3)
    pats = np.array([0x7FC0, 0xFFC0, 0x7F80, 0xFF80, 0x0000, 0x8000, 0x0001, 0x807F, 0x7F81],
                    np.uint16)
    x = rng.choice(pats, size=(2, 512, 128)).astype(np.uint16)
    x[1] = 0x3F80
    w = _w("lossless-1x8x512x128-bf16", n_heads=1)
    plan, oplan = _plans(w)
    st, got = encode(plan, kvc.LOSSLESS, x)
    assert st == kvc.OK and got == oracle.encode_lossless(oplan, x)
    st, y = decode(plan, kvc.LOSSLESS, got, 2)
    assert st == kvc.OK and np.array_equal(y, x)


def test_full_size_migration_block():
    """50,331,648 bytes (8 layers x 8 heads x 1536 x 128, K+V), bit exact."""
    w = kvgen.WORKLOADS["lossless-8x8x1536x128-bf16"]
    plan, oplan = _plans(w)
    x = kvgen.slices(w)
    assert x.nbytes == 50_331_648
    st, got = encode(plan, kvc.LOSSLESS, x)
    assert st == kvc.OK and got == oracle.encode_lossless(oplan, x)
    st, y = decode(plan, kvc.LOSSLESS, got, w.n_slices)
    assert st == kvc.OK and np.array_equal(y, x)


def test_full_size_frame_of_32k_cache():
    """One 64 MiB frame (one layer's K: 8 heads x 32768 x 128) of the 64-layer cache."""
    w = kvgen.WORKLOADS["lossless-64x8x32768x128-bf16"]
    plan, oplan = _plans(w)
    x = kvgen.slices(w, first=80, n=8)
    st, got = encode(plan, kvc.LOSSLESS, x, first_slice=80)
    assert st == kvc.OK and got == oracle.encode_lossless(oplan, x, first_slice=80)
    st, y = decode(plan, kvc.LOSSLESS, got, 8)
    assert st == kvc.OK and np.array_equal(y, x)


def test_damage_is_refused_with_oracle_status():
    w = _w("lossless-1x8x512x128-bf16", n_heads=2)
    plan, oplan = _plans(w)
    x = kvgen.slices(w)
    c = bytearray(oracle.encode_lossless(oplan, x))
    rng = np.random.default_rng(5)
    n_idx = 64 + 16 * 4
    positions = list(range(0, n_idx)) + list(rng.integers(n_idx, len(c), 120))
    for pos in positions:
        orig = c[pos]
        c[pos] = orig ^ int(rng.integers(1, 256))
        want, _ = oracle.decode_lossless(oplan, bytes(c))
        got, _ = decode(plan, kvc.LOSSLESS, bytes(c), w.n_slices)
        assert want != oracle.OK and got == want, (pos, got, want)
        c[pos] = orig
    for n in [0, 1, 63, 64, 100, n_idx, len(c) // 2, len(c) - 16, len(c) - 1]:
        got, _ = decode(plan, kvc.LOSSLESS, bytes(c[:n]), w.n_slices)
        assert got == kvc.ERR_TRUNCATED, n
    got, _ = decode(plan, kvc.LOSSLESS, bytes(c) + bytes(16), w.n_slices)
    assert got == kvc.ERR_CORRUPT


def test_plan_mismatch_and_capacity():
    w = _w("lossless-1x8x512x128-bf16", n_heads=1)
    plan, oplan = _plans(w)
    c = oracle.encode_lossless(oplan, kvgen.slices(w))
    other = kvc.Plan(kvc.Shape(kvc.BF16, 1, 1, 513, 128))
    assert decode(other, kvc.LOSSLESS, c, 2)[0] == kvc.ERR_PLAN_MISMATCH
    assert decode(plan, kvc.LOSSLESS, c, 1)[0] == kvc.ERR_CAPACITY


RAW, CONST, RANS = 0, 1, 2
_SKEW = np.array([.5, .2, .1, .08, .05, .04, .02, .01])


def _plane(rng, kind, shape):
    if kind == RAW:
        return rng.integers(0, 256, shape)
    if kind == CONST:
        return np.full(shape, 0x3F)
    return rng.choice(np.arange(8) * 29, size=shape, p=_SKEW)


def _records(c: bytes):
    """(offset, length) of every record of a container, from its index."""
    n = int.from_bytes(c[36:40], "little")
    out = []
    for i in range(n):
        e = 64 + 16 * i
        out.append((int.from_bytes(c[e:e + 8], "little"), int.from_bytes(c[e + 8:e + 12], "little")))
    return out


@pytest.mark.parametrize("D", [128, 64])
def test_full_chunk_mode_pairs_and_damage(D):
    """Full chunks (the token-synchronous decoder) with every pair of plane
    modes but two rANS planes, decoded exactly; damage in either stream's
    header or payload, or at the record's ends, is refused as the oracle does."""
    pairs = [(RAW, RANS), (RAW, RAW), (RAW, CONST), (RANS, RAW), (RANS, CONST), (CONST, RANS),
             (CONST, RAW), (CONST, CONST)]
    T = 65536 // D
    rng = np.random.default_rng(11 + D)
    x = np.stack([(_plane(rng, lo, (T, D)) | (_plane(rng, hi, (T, D)) << 8)).astype(np.uint16)
                  for lo, hi in pairs])
    w = _w("lossless-1x8x512x128-bf16", n_heads=4, n_tokens=T, head_dim=D)
    plan, oplan = _plans(w)
    c = bytearray(oracle.encode_lossless(oplan, x))
    recs = _records(c)
    assert len(recs) == len(pairs)
    for (off, ln), (lo, hi) in zip(recs, pairs):  # the encoder chose the intended modes
        b0 = int.from_bytes(c[off + 4:off + 8], "little")
        assert (c[off], c[off + b0]) == (lo, hi)
    st, y = decode(plan, kvc.LOSSLESS, bytes(c), len(pairs))
    assert st == kvc.OK and np.array_equal(y, x)
    for off, ln in recs:
        b0 = int.from_bytes(c[off + 4:off + 8], "little")
        spots = {off, off + 1, off + 12, off + 16, off + b0 // 2, off + b0 - 1, off + b0,
                 off + b0 + 16, off + (b0 + ln) // 2, off + ln - 1}
        for pos in sorted(p for p in spots if p < off + ln):
            orig = c[pos]
            c[pos] = orig ^ 0x5A
            want, _ = oracle.decode_lossless(oplan, bytes(c))
            got, _ = decode(plan, kvc.LOSSLESS, bytes(c), len(pairs))
            assert want != oracle.OK and got == want, (pos - off, got, want)
            c[pos] = orig


def _ramp(w, scale=3, dtype=np.uint16):
    t = np.arange(w.n_tokens)[None, :, None]
    ch = np.arange(w.head_dim)[None, None, :]
    s = np.arange(w.n_slices)[:, None, None]
    x = (scale * t + 17 * ch + 29 * s + 4096)
    return (x & (0xFFFF if dtype == np.uint16 else 0xFFFFFFFF)).astype(dtype)


@pytest.mark.parametrize("name,kw", [
    ("lossless-1x8x512x128-bf16", dict(n_heads=2)),                    # full chunks of 128 channels
    ("lossless-12x12x1024x64-fp16", dict(n_layers=1, n_heads=2)),      # full chunks of 64 channels
    ("lossless-1x8x512x128-bf16", dict(n_heads=1, n_tokens=700)),      # a full and a ragged chunk
])
def test_low_plane_lane_deltas_equal_oracle_bytes(name, kw):
    """Values that change by a few steps per token (a ramp along tokens) make
    the low byte plane's lane deltas the smallest record: the low plane takes
    the 16-bit XOR with the previous token of the channel too. The fast
    encoder hands such chunks to the general encoder; the container is the
    oracle's byte for byte and the GPU decoder restores it."""
    w = _w(name, **kw)
    plan, oplan = _plans(w)
    x = _ramp(w)
    want = oracle.encode_lossless(oplan, x)
    st, got = encode(plan, kvc.LOSSLESS, x)
    assert st == kvc.OK
    assert got == want
    n_rec = int.from_bytes(want[36:40], "little")
    off0 = int.from_bytes(want[64:72], "little")
    assert want[off0] == 2 and want[off0 + 3] == 1  # the first chunk's low plane: RANS of lane deltas
    st, y = decode(plan, kvc.LOSSLESS, got, w.n_slices)
    assert st == kvc.OK and np.array_equal(y, x)
    assert n_rec >= 1


def test_f32_low_planes_lane_deltas_equal_oracle_bytes():
    """f32: every byte plane may take the lane deltas (a ramp in the low bits)."""
    w = _w("lossless-1x8x512x128-bf16", dtype=kvgen.F32, n_heads=1, n_tokens=512, head_dim=64,
           values_per_chunk=8192)
    plan, oplan = _plans(w)
    x = _ramp(w, scale=5, dtype=np.uint32)
    want = oracle.encode_lossless(oplan, x)
    st, got = encode(plan, kvc.LOSSLESS, x)
    assert st == kvc.OK and got == want
    st, y = decode(plan, kvc.LOSSLESS, got, w.n_slices)
    assert st == kvc.OK and np.array_equal(y, x)
