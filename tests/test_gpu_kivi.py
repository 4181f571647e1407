"""KIVI-style ranges on the GPU against the oracle (Codec-Gauge page,
"Compression Conditions": per-channel key ranges, per-token value ranges).
Keys keep the per-component block ranges; each value token takes one zero
point and range over its coded components. The encoder's tensor-core
projection reproduces the oracle's y where a decision needs it, so whole
containers equal the oracle's byte for byte."""
import dataclasses

import numpy as np
import pytest

import kvgen
import oracle
import transform_codec_b200 as kvc
from kvc_gpu import decode, encode, rel_rms

pytestmark = pytest.mark.gpu


def _setup(T, n_heads=2, seed=None):
    w = dataclasses.replace(kvgen.WORKLOADS["transform-32x8x8192x128-bf16"], n_layers=1, n_heads=n_heads,
                            n_tokens=T)
    cal = kvgen.calibration(w)
    pcs = [oracle.pca(cal[s], (s // w.n_heads) % 2 == 0, w.theta) for s in range(w.n_slices)]
    bases = np.stack([p[0] for p in pcs])
    widths = oracle.allocate(np.stack([p[1] for p in pcs]), w.avg_bits, w.max_bits).reshape(w.n_slices, 128)
    shape = dataclasses.replace(kvc.Shape.from_workload(w), range_mode=kvc.RANGES_KIVI)
    plan = kvc.Plan(shape, bases=bases, widths=widths)
    oplan = oracle.Plan.from_workload(w, bases=bases, widths=widths, ranges=oracle.RANGES_KIVI)
    return w, plan, oplan, bases, widths


@pytest.mark.parametrize("T", [1024, 644, 100])
def test_kivi_container_equals_oracle_bytes(T):
    w, plan, oplan, bases, widths = _setup(T)
    assert plan.crc == oracle.plan_crc(oplan)
    x = kvgen.slices(w)
    st, got = encode(plan, kvc.TRANSFORM, x)
    assert st == kvc.OK
    want = oracle.encode_transform(oplan, x)
    assert len(got) == len(want)
    assert got == want
    st, y = decode(plan, kvc.TRANSFORM, got, w.n_slices)
    assert st == kvc.OK
    st_o, yo = oracle.decode_transform(oplan, want)
    assert st_o == oracle.OK
    for s in range(w.n_slices):
        assert rel_rms(yo[s], y[s]) <= 1e-3


def test_kivi_extremes_equal_oracle_bytes():
    """Tokens of very different scales, all-zero tokens and repeated tokens."""
    w, plan, oplan, _, _ = _setup(644)
    x = kvgen.slices(w).copy()
    rng = np.random.default_rng(17)
    mid = np.arange(w.n_sink, w.n_tokens - w.n_recent)
    zero = rng.choice(mid, 30, replace=False)
    x[:, zero, :] = 0
    small = rng.choice(np.setdiff1d(mid, zero), 30, replace=False)
    f = (x[:, small, :].astype(np.uint32) << 16).view(np.float32) * np.float32(2.0 ** -60)
    x[:, small, :] = (f.view(np.uint32) >> 16).astype(np.uint16)
    big = rng.choice(np.setdiff1d(mid, np.union1d(zero, small)), 30, replace=False)
    f = (x[:, big, :].astype(np.uint32) << 16).view(np.float32) * np.float32(2.0 ** 40)
    x[:, big, :] = (f.view(np.uint32) >> 16).astype(np.uint16)
    x[:, mid[200:210], :] = x[:, mid[199:200], :]
    st, got = encode(plan, kvc.TRANSFORM, x)
    assert st == kvc.OK
    assert got == oracle.encode_transform(oplan, x)


def test_block_plan_refuses_a_kivi_container():
    w, plan, oplan, bases, widths = _setup(644, n_heads=1)
    x = kvgen.slices(w)
    st, got = encode(plan, kvc.TRANSFORM, x)
    assert st == kvc.OK
    bplan = kvc.Plan(kvc.Shape.from_workload(w), bases=bases, widths=widths)
    assert bplan.crc != plan.crc
    st, _ = decode(bplan, kvc.TRANSFORM, got, w.n_slices)
    assert st == kvc.ERR_PLAN_MISMATCH
