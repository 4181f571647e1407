"""Pins for the oracle's container and lossless front-end (CPU only).

Bit-for-bit restore (QATQ page, "qatq encode"; AT-1 Memory page, "KV & tensor
mode"), never worse than raw plus the container overhead (AT-1 Memory, "What's
proven"), and refusal of corrupt or truncated input (QATQ page, "QATC v2
checksum validated"). The byte layout is pinned by a hand-worked container.
"""
import dataclasses
import struct
import zlib

import numpy as np
import pytest

import kvgen
import oracle


def test_hand_worked_container_2x2():
    """One slice of 2 tokens x 2 channels, chunks of 4 values (2 tokens):
    values (t, d): (0,0)=0x0102 (0,1)=0x0304 (1,0)=0x0506 (1,1)=0x0708.
    Channel-major order (d, t): 0x0102, 0x0506, 0x0304, 0x0708, so the low
    plane is 02 06 04 08 and the high plane 01 05 03 07; four distinct symbols
    in four make rANS larger than raw, so both planes are RAW records."""
    plan = oracle.Plan(oracle.BF16, 1, 1, 2, 2, values_per_chunk=4)
    src = np.array([[[0x0102, 0x0304], [0x0506, 0x0708]]], np.uint16)
    got = oracle.encode_lossless(plan, src)

    def raw_stream(b):
        return bytes([0, 0, 0, 0]) + struct.pack("<III", 32, 4, 0) + bytes(b) + bytes(12)

    record = raw_stream([0x02, 0x06, 0x04, 0x08]) + raw_stream([0x01, 0x05, 0x03, 0x07])
    n_rec, total = 1, 64 + 16 + len(record)
    head = b"KVC1" + struct.pack("<HBB", 1, 0, 1) + struct.pack(
        "<IIIIIIII", 1, 1, 2, 2, 0, 1, 2, n_rec) + struct.pack("<Q", total) + struct.pack(
        "<IHHHH", 0, 0, 0, 0, 0)
    index = struct.pack("<QII", 80, len(record), zlib.crc32(record))
    head += struct.pack("<I", zlib.crc32(head + index))
    expect = head + index + record
    assert got == expect
    st, back = oracle.decode_lossless(plan, got)
    assert st == oracle.OK and np.array_equal(back, src)


def _small(name, **kw):
    return dataclasses.replace(kvgen.WORKLOADS[name], **kw)


CASES = [
    _small("lossless-1x8x512x128-bf16"),
    _small("lossless-1x8x512x128-bf16", n_tokens=700),        # ragged last chunk
    _small("lossless-12x12x1024x64-fp16", n_layers=1, n_heads=3, n_tokens=1500),
    _small("lossless-1x8x512x128-bf16", n_tokens=3, head_dim=10, values_per_chunk=16),
    _small("lossless-8x8x1536x128-bf16", n_layers=1, n_heads=2),
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: f"{w.n_tokens}x{w.head_dim}")
def test_lossless_roundtrip_and_never_worse(w):
    plan = oracle.Plan.from_workload(w)
    x = kvgen.slices(w)
    c = oracle.encode_lossless(plan, x)
    assert len(c) <= oracle.lossless_bound(plan, w.n_slices)
    st, y = oracle.decode_lossless(plan, c)
    assert st == oracle.OK and np.array_equal(x, y)


def test_lossless_subrange_of_slices():
    w = _small("lossless-1x8x512x128-bf16")
    plan = oracle.Plan.from_workload(w)
    x = kvgen.slices(w, first=5, n=3)
    c = oracle.encode_lossless(plan, x, first_slice=5)
    assert struct.unpack_from("<II", c, 24) == (5, 3)
    st, y = oracle.decode_lossless(plan, c)
    assert st == oracle.OK and np.array_equal(x, y)


def test_random_control_block_takes_raw_exactly():
    """4 MiB of uniform random bytes viewed as fp16 with D = 64: every plane
    stream must fall back to RAW, so the size equals raw + 64 + 48 per chunk."""
    raw = kvgen.random_bytes(4 << 20)
    plan = oracle.Plan(oracle.FP16, 1, 1, 32768, 64)
    x = raw.view(np.uint16).reshape(1, 32768, 64)
    c = oracle.encode_lossless(plan, x)
    n_chunks = 32768 // 1024
    assert len(c) == raw.size + 64 + 48 * n_chunks
    st, y = oracle.decode_lossless(plan, c)
    assert st == oracle.OK and np.array_equal(x, y)


def test_special_bit_patterns_roundtrip():
    """NaN, infinities, signed zeros, subnormals and constant chunks go through
    unchanged: the lossless path never interprets the values."""
    rng = np.random.default_rng(3)
    pats = np.array([0x7FC0, 0xFFC0, 0x7F80, 0xFF80, 0x0000, 0x8000, 0x0001, 0x807F, 0x7F81],
                    np.uint16)
    x = rng.choice(pats, size=(2, 512, 128)).astype(np.uint16)
    x[1] = 0x3F80
    plan = oracle.Plan(oracle.BF16, 1, 1, 512, 128)
    c = oracle.encode_lossless(plan, x)
    st, y = oracle.decode_lossless(plan, c)
    assert st == oracle.OK and np.array_equal(x, y)
    # the constant slice is two CONST streams (16 bytes each) per chunk
    idx = struct.unpack_from("<QII", c, 64 + 16)
    assert idx[1] == 32


def test_empty_slice_range():
    plan = oracle.Plan(oracle.BF16, 1, 1, 64, 128)
    c = oracle.encode_lossless(plan, np.zeros((0, 64, 128), np.uint16))
    assert len(c) == 64
    st, y = oracle.decode_lossless(plan, c)
    assert st == oracle.OK and y.shape[0] == 0


def _tiny_container():
    w = _small("lossless-1x8x512x128-bf16", n_layers=1, n_heads=1, n_tokens=48)
    plan = oracle.Plan.from_workload(w)
    x = kvgen.slices(w)
    return plan, x, oracle.encode_lossless(plan, x)


def test_every_single_byte_change_is_refused():
    plan, x, c = _tiny_container()
    rng = np.random.default_rng(11)
    buf = bytearray(c)
    for pos in range(len(c)):
        orig = buf[pos]
        buf[pos] = orig ^ int(rng.integers(1, 256))
        st, _ = oracle.decode_lossless(plan, bytes(buf))
        assert st != oracle.OK, pos
        buf[pos] = orig


def test_every_truncation_is_refused():
    plan, x, c = _tiny_container()
    for n in range(len(c)):
        st, _ = oracle.decode_lossless(plan, c[:n])
        assert st == oracle.TRUNCATED, n
    st, _ = oracle.decode_lossless(plan, c + b"\0")
    assert st == oracle.CORRUPT


def test_sampled_byte_changes_refused_on_full_size_container():
    w = _small("lossless-1x8x512x128-bf16")
    plan = oracle.Plan.from_workload(w)
    c = bytearray(oracle.encode_lossless(plan, kvgen.slices(w)))
    rng = np.random.default_rng(12)
    for pos in list(range(64 + 16 * 16)) + list(rng.integers(0, len(c), 150)):
        orig = c[pos]
        c[pos] = orig ^ 0xFF
        assert oracle.decode_lossless(plan, bytes(c))[0] != oracle.OK
        c[pos] = orig


def test_plan_mismatch_and_capacity():
    plan, x, c = _tiny_container()
    other = oracle.Plan(oracle.BF16, 1, 1, 97, 128)
    assert oracle.decode_lossless(other, c)[0] == oracle.PLAN_MISMATCH
    assert oracle.decode_lossless(plan, c, n_slices_cap=0)[0] == oracle.CAPACITY


def test_hand_worked_container_f32_2x2():
    """f32 (QATQ and AT-1 code f32 tensors too): one slice of 2 tokens x 2
    channels, chunks of 4 values. Values (t, d) = (0,0) 0x04030201, (0,1)
    0x14131211, (1,0) 0x24232221, (1,1) 0x34333231; channel-major order (d, t)
    is (0,0), (1,0), (0,1), (1,1), so plane p holds byte p of 0x..01, 0x..21,
    0x..11, 0x..31 in that order: four RAW records, plane 0 first."""
    plan = oracle.Plan(oracle.F32, 1, 1, 2, 2, values_per_chunk=4)
    src = np.array([[[0x04030201, 0x14131211], [0x24232221, 0x34333231]]], np.uint32)
    got = oracle.encode_lossless(plan, src)

    def raw_stream(b):
        return bytes([0, 0, 0, 0]) + struct.pack("<III", 32, 4, 0) + bytes(b) + bytes(12)

    # byte p of value (t, d) is 0x01 + p + 0x10 * (2t + d); in channel-major order (0,0) (1,0) (0,1) (1,1)
    record = b"".join(raw_stream([0x01 + p + 0x10 * k for k in (0, 2, 1, 3)]) for p in range(4))
    n_rec, total = 1, 64 + 16 + len(record)
    head = b"KVC1" + struct.pack("<HBB", 1, 0, 3) + struct.pack(
        "<IIIIIIII", 1, 1, 2, 2, 0, 1, 2, n_rec) + struct.pack("<Q", total) + struct.pack(
        "<IHHHH", 0, 0, 0, 0, 0)
    index = struct.pack("<QII", 80, len(record), zlib.crc32(record))
    head += struct.pack("<I", zlib.crc32(head + index))
    assert got == head + index + record
    st, back = oracle.decode_lossless(plan, got)
    assert st == oracle.OK and np.array_equal(back, src)


F32_CASES = [
    _small("lossless-12x12x1024x64-f32", n_layers=1, n_heads=2),
    _small("lossless-12x12x1024x64-f32", n_layers=1, n_heads=1, n_tokens=1500),  # ragged last chunk
    _small("lossless-12x12x1024x64-f32", n_layers=1, n_heads=1, n_tokens=700, head_dim=128),
    _small("lossless-12x12x1024x64-f32", n_layers=1, n_heads=1, n_tokens=5, head_dim=6, values_per_chunk=12),
]


@pytest.mark.parametrize("w", F32_CASES, ids=lambda w: f"{w.n_tokens}x{w.head_dim}")
def test_f32_roundtrip_never_worse_and_planes(w):
    """Round trip; size within raw + container overhead; every record is four
    stream records whose lengths add up to the record; the sign/exponent plane
    of the AR(1) fixture takes a RANS record (it carries the structure) and the
    low mantissa plane is RAW."""
    plan = oracle.Plan.from_workload(w)
    x = kvgen.slices(w)
    assert x.dtype == np.uint32
    c = oracle.encode_lossless(plan, x)
    assert len(c) <= oracle.lossless_bound(plan, w.n_slices)
    st, y = oracle.decode_lossless(plan, c)
    assert st == oracle.OK and np.array_equal(x, y)
    n_rec = struct.unpack_from("<I", c, 36)[0]
    modes = []
    for i in range(n_rec):
        off, ln, _ = struct.unpack_from("<QII", c, 64 + 16 * i)
        o, m = 0, []
        for _ in range(4):
            m.append(c[off + o])
            o += struct.unpack_from("<I", c, off + o + 4)[0]
        assert o == ln
        modes.append(m)
    if w.n_tokens * w.head_dim >= 4096:
        assert modes[0][0] == 0 and modes[0][3] == 2


def test_f32_random_block_takes_raw_exactly():
    """Uniform random bytes viewed as f32: four RAW streams per chunk, so the
    size equals raw + 64 + (16 + 4 * 16) per chunk."""
    w = _small("lossless-12x12x1024x64-f32", n_layers=1, n_heads=1)
    plan = oracle.Plan.from_workload(w)
    x = kvgen.random_bytes(w.raw_bytes, seed=5).view(np.uint32).reshape(w.n_slices, w.n_tokens, w.head_dim)
    c = oracle.encode_lossless(plan, x)
    n_chunks = w.n_slices * (w.n_tokens // (65536 // w.head_dim))
    assert len(c) == w.raw_bytes + 64 + n_chunks * (16 + 4 * 16)
    st, y = oracle.decode_lossless(plan, c)
    assert st == oracle.OK and np.array_equal(x, y)


def test_f32_tamper_refused():
    w = _small("lossless-12x12x1024x64-f32", n_layers=1, n_heads=1, n_tokens=256)
    plan = oracle.Plan.from_workload(w)
    c = bytearray(oracle.encode_lossless(plan, kvgen.slices(w)))
    rng = np.random.default_rng(3)
    for pos in rng.integers(0, len(c), 60):
        old = c[int(pos)]
        c[int(pos)] = old ^ int(rng.integers(1, 256))
        assert oracle.decode_lossless(plan, bytes(c))[0] != oracle.OK
        c[int(pos)] = old
