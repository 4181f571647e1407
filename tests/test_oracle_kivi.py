"""Pins of the oracle's KIVI-style ranges (Codec-Gauge page, "Compression
Conditions": the KIVI-style path takes per-channel key ranges and per-token
value ranges). Reading: keys keep the codec's per-component block ranges
(per-channel ranges in the basis); values take one range per token over the
token's coded components: z = their minimum, r = fl(max - min), and a
component of width b quantises with s = fl(r / (2^b - 1)). The side
information of a value record is every token's z, then every token's r."""
import dataclasses

import numpy as np
import pytest

import kvgen
import oracle


def _bf16(f):
    return (np.asarray(f, np.float32).view(np.uint32) >> 16).astype(np.uint16)


def _f32(h):
    return (np.asarray(h, np.uint32) << 16).view(np.float32)


def _plan(T=200, D=16, ranges=oracle.RANGES_KIVI, widths=None, seed=0):
    rng = np.random.default_rng(seed)
    w = kvgen.Workload("kivi", "transform", 1, 1, 1, T, D, 0.9, 1e4, 0, n_sink=4, n_recent=16,
                       block_tokens=16, chunk_tokens=64, max_bits=8)
    bases = np.stack([np.eye(D, dtype=np.float32)] * w.n_slices)
    if widths is None:
        widths = rng.integers(0, 9, (w.n_slices, D)).astype(np.uint8)
    return w, oracle.Plan.from_workload(w, bases=bases, widths=widths, ranges=ranges), widths


def _quant(y, z, s, levels):
    if s == 0:
        return 0
    q = np.float32(np.float32(y - z) / s)
    r = np.rint(q)
    return int(min(max(r, 0), levels))


def test_value_codes_follow_per_token_ranges_by_hand():
    """Identity basis (y = x), so the value codes are computed here from the
    definition: per middle token, z and r over the coded components in
    ascending order, each component quantised in its own number of steps."""
    w, plan, widths = _plan()
    rng = np.random.default_rng(3)
    x = _bf16(rng.normal(0, 2, (w.n_slices, w.n_tokens, w.head_dim)).astype(np.float32))
    s_end, r_start = w.n_sink, w.n_tokens - w.n_recent
    sv = 1  # slice 1 is the value slice of layer 0, head 0
    codes, _, _ = oracle.transform_slice_codes(plan, sv, x[sv])
    ws = widths[sv]
    coded = np.flatnonzero(ws)
    for t in range(s_end, r_start):
        y = _f32(x[sv, t])
        z = np.float32(y[coded].min())
        mx = np.float32(y[coded].max())
        r = np.float32(mx - z)
        for j in range(w.head_dim):
            if ws[j] == 0:
                assert codes[t, j] == 0
                continue
            levels = (1 << int(ws[j])) - 1
            s = np.float32(0) if mx == z else np.float32(r / np.float32(levels))
            assert codes[t, j] == _quant(y[j], z, s, levels), (t, j)


def test_keys_keep_block_ranges():
    """The key slice's codes are those of the same plan with block ranges."""
    w, kplan, widths = _plan(ranges=oracle.RANGES_KIVI)
    _, bplan, _ = _plan(ranges=oracle.RANGES_BLOCK, widths=widths)
    x = _bf16(np.random.default_rng(4).normal(0, 1, (w.n_slices, w.n_tokens, w.head_dim)).astype(np.float32))
    ck, _, _ = oracle.transform_slice_codes(kplan, 0, x[0])
    cb, _, _ = oracle.transform_slice_codes(bplan, 0, x[0])
    assert np.array_equal(ck, cb)
    cv, _, _ = oracle.transform_slice_codes(kplan, 1, x[1])
    cvb, _, _ = oracle.transform_slice_codes(bplan, 1, x[1])
    assert not np.array_equal(cv, cvb)


@pytest.mark.parametrize("T", [200, 90, 70])
def test_kivi_container_roundtrip_error_bound_and_refusals(T):
    """Round trip within half a step of the token's range per value (identity
    basis, so x^ = y^ before the bf16 rounding); the side streams hold 2 tcc
    values per value record; the plan CRC differs from the block plan's, and
    a block plan refuses the container; a flipped byte is refused."""
    w, plan, widths = _plan(T=T)
    _, bplan, _ = _plan(T=T, ranges=oracle.RANGES_BLOCK, widths=widths)
    assert oracle.plan_crc(plan) != oracle.plan_crc(bplan)
    x = _bf16(np.random.default_rng(T).normal(0, 1, (w.n_slices, w.n_tokens, w.head_dim)).astype(np.float32))
    c = oracle.encode_transform(plan, x)
    st, y = oracle.decode_transform(plan, c)
    assert st == oracle.OK
    s_end, r_start = w.n_sink, w.n_tokens - w.n_recent
    ws = widths[1]
    coded = np.flatnonzero(ws)
    for t in range(s_end, r_start):
        xv = _f32(x[1, t]).astype(np.float64)
        yv = _f32(y[1, t]).astype(np.float64)
        rngv = xv[coded].max() - xv[coded].min()
        for j in coded:
            step = rngv / ((1 << int(ws[j])) - 1)
            assert abs(yv[j] - xv[j]) <= step / 2 * (1 + 1e-5) + abs(xv[j]) * 2 ** -8 + 1e-30
        for j in np.flatnonzero(ws == 0):
            assert yv[j] == 0
    assert oracle.decode_transform(bplan, c)[0] == oracle.PLAN_MISMATCH
    bad = bytearray(c)
    bad[len(bad) // 2] ^= 0x10
    assert oracle.decode_transform(plan, bytes(bad))[0] != oracle.OK
    # the first middle record of the value slice: 4 side streams of 2 * tcc symbols
    st, codes, zs = oracle.container_codes(plan, c, w.n_slices)
    assert st == oracle.OK
    tcc = min(w.chunk_tokens, r_start - s_end)
    zt = zs[1, 0].reshape(-1)[: 2 * tcc].reshape(tcc, 2)
    xv = _f32(x[1, s_end:s_end + tcc])[:, coded]
    assert np.array_equal(zt[:, 0], xv.min(1))
    assert np.array_equal(zt[:, 1], (xv.max(1) - xv.min(1)).astype(np.float32))


def test_kivi_on_the_workload_generator_with_pca():
    """A calibrated PCA plan on the synthetic generator: KIVI-style round trip
    status OK, and the key slices' records equal the block plan's."""
    w = dataclasses.replace(kvgen.WORKLOADS["transform-32x8x8192x128-bf16"], n_layers=1, n_heads=1,
                            n_tokens=700)
    cal = kvgen.calibration(w)
    pcs = [oracle.pca(cal[s], s == 0, w.theta) for s in range(w.n_slices)]
    bases = np.stack([p[0] for p in pcs])
    widths = oracle.allocate(np.stack([p[1] for p in pcs]), w.avg_bits, w.max_bits).reshape(w.n_slices, 128)
    x = kvgen.slices(w)
    kp = oracle.Plan.from_workload(w, bases=bases, widths=widths, ranges=oracle.RANGES_KIVI)
    bp = oracle.Plan.from_workload(w, bases=bases, widths=widths)
    ck = oracle.encode_transform(kp, x[0:1], first_slice=0)
    cb = oracle.encode_transform(bp, x[0:1], first_slice=0)
    assert ck[64:] == cb[64:]  # keys: the same index and records (the header carries the plan CRC)
    c = oracle.encode_transform(kp, x)
    st, y = oracle.decode_transform(kp, c)
    assert st == oracle.OK
