"""f32 lossless on the GPU against the oracle (QATQ "qatq encode": f32, f16 and
bf16 tensors restored bit for bit; AT-1 "KV & tensor mode": fp32/fp16/bf16).
A chunk record is one stream per byte plane of the 4-byte value; the GPU
encoder must write the oracle's exact bytes, and the GPU decoder must restore
the oracle's containers exactly and refuse what the oracle refuses."""
import dataclasses
import struct
import zlib

import numpy as np
import pytest

import kvgen
import oracle
import transform_codec_b200 as kvc
from kvc_gpu import decode, encode

pytestmark = pytest.mark.gpu

BASE = kvgen.WORKLOADS["lossless-12x12x1024x64-f32"]
CASES = [
    dataclasses.replace(BASE, n_layers=1, n_heads=2),                                # full chunks, D = 64
    dataclasses.replace(BASE, n_layers=1, n_heads=1, n_tokens=1500),                 # ragged last chunk
    dataclasses.replace(BASE, n_layers=1, n_heads=2, n_tokens=700, head_dim=128),    # D = 128, ragged
    dataclasses.replace(BASE, n_layers=1, n_heads=1, n_tokens=37, head_dim=6, values_per_chunk=60),
    dataclasses.replace(BASE, n_layers=2, n_heads=1, n_tokens=256, rho=0.0),         # no token correlation
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: f"{w.n_slices}x{w.n_tokens}x{w.head_dim}-{w.values_per_chunk}")
def test_f32_container_equals_oracle_bytes_and_roundtrip(w):
    x = kvgen.slices(w)
    plan = kvc.Plan(kvc.Shape.from_workload(w))
    oplan = oracle.Plan.from_workload(w)
    want = oracle.encode_lossless(oplan, x)
    st, got = encode(plan, kvc.LOSSLESS, x)
    assert st == kvc.OK and got == want
    st, y = decode(plan, kvc.LOSSLESS, want, w.n_slices)
    assert st == kvc.OK and y.dtype == np.uint32 and np.array_equal(y, x)


def test_f32_random_bytes_take_raw_and_subrange():
    w = dataclasses.replace(BASE, n_layers=1, n_heads=2)
    x = kvgen.random_bytes(w.raw_bytes, seed=9).view(np.uint32).reshape(w.n_slices, w.n_tokens, w.head_dim)
    plan = kvc.Plan(kvc.Shape.from_workload(w))
    oplan = oracle.Plan.from_workload(w)
    st, got = encode(plan, kvc.LOSSLESS, x)
    assert st == kvc.OK and got == oracle.encode_lossless(oplan, x)
    assert len(got) == plan.max_encoded_bytes(kvc.LOSSLESS, w.n_slices)  # RAW everywhere: the bound exactly
    st, got = encode(plan, kvc.LOSSLESS, x[2:3], first_slice=2)
    assert st == kvc.OK and got == oracle.encode_lossless(oplan, x[2:3], first_slice=2)


def _reseal(c: bytearray, i: int) -> bytes:
    n = struct.unpack_from("<I", c, 36)[0]
    off, ln, _ = struct.unpack_from("<QII", c, 64 + 16 * i)
    struct.pack_into("<I", c, 64 + 16 * i + 12, zlib.crc32(bytes(c[off:off + ln])))
    struct.pack_into("<I", c, 60, zlib.crc32(bytes(c[:60]) + bytes(c[64:64 + 16 * n])))
    return bytes(c)


def test_f32_damage_and_forged_records():
    """Byte flips (the CRCs refuse them) and forged records (sealed again, so
    that the stream checks decide): the GPU decoder's status is the oracle's,
    and an accepted forgery decodes to the oracle's values."""
    w = dataclasses.replace(BASE, n_layers=1, n_heads=1, n_tokens=512)
    x = kvgen.slices(w)
    plan = kvc.Plan(kvc.Shape.from_workload(w))
    oplan = oracle.Plan.from_workload(w)
    c = oracle.encode_lossless(oplan, x)
    rng = np.random.default_rng(31)
    for pos in rng.integers(0, len(c), 40):
        cc = bytearray(c)
        cc[int(pos)] ^= int(rng.integers(1, 256))
        assert decode(plan, kvc.LOSSLESS, bytes(cc), w.n_slices)[0] == oracle.decode_lossless(oplan, bytes(cc))[0]
    off, ln, _ = struct.unpack_from("<QII", c, 64)
    seen = set()
    for pos in list(range(0, 16)) + [int(p) for p in rng.integers(16, ln, 60)]:
        cc = bytearray(c)
        cc[off + pos] = (cc[off + pos] + int(rng.integers(1, 256))) & 0xFF
        cc = _reseal(cc, 0)
        want, wy = oracle.decode_lossless(oplan, cc)
        got, gy = decode(plan, kvc.LOSSLESS, cc, w.n_slices)
        assert got == want, (pos, got, want)
        if want == oracle.OK:
            assert np.array_equal(gy, wy)
        seen.add(want)
    assert oracle.CORRUPT in seen
