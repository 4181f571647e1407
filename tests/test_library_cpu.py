"""Host-side checks of libkvc.so that need no GPU: every symbol the C header
declares is exported, container bounds equal the oracle's, and the plan-time
host algorithms (greedy allocation, PCA calibration) agree with the oracle."""
import ctypes
import dataclasses
import os
import re

import numpy as np
import pytest

import kvgen
import oracle
import transform_codec_b200 as kvc

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    text = open(os.path.join(ROOT, "include", "kvc.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kvc_\w+)\s*\(", text)))


def test_every_declared_symbol_is_exported():
    names = _declared_functions()
    assert len(names) >= 16
    lib = ctypes.CDLL(kvc.LIB_PATH)
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing
    assert set(names) == set(kvc.EXPORTS)


def test_status_strings():
    for code in range(9):
        assert kvc.status_string(code) and kvc.status_string(code) != "unknown status"
    assert kvc.status_string(99) == "unknown status"


SHAPES = [
    kvc.Shape(kvc.BF16, 1, 8, 512, 128),
    kvc.Shape(kvc.BF16, 1, 8, 700, 128),
    kvc.Shape(kvc.FP16, 12, 12, 1024, 64),
    kvc.Shape(kvc.BF16, 1, 8, 3, 10, values_per_chunk=16),
    kvc.Shape(kvc.BF16, 64, 8, 32768, 128),
    kvc.Shape(kvc.F32, 12, 12, 1024, 64),
    kvc.Shape(kvc.F32, 1, 2, 700, 128),
]


@pytest.mark.parametrize("s", SHAPES, ids=lambda s: f"{s.n_tokens}x{s.head_dim}")
def test_lossless_bound_matches_oracle(s):
    plan = kvc.Plan(s)
    op = oracle.Plan(s.dtype, s.n_layers, s.n_heads, s.n_tokens, s.head_dim, s.values_per_chunk)
    for n in [0, 1, 3, s.n_slices]:
        assert plan.max_encoded_bytes(kvc.LOSSLESS, n) == oracle.lossless_bound(op, n)
    assert plan.workspace_bytes(kvc.LOSSLESS, False, 2) > 0
    assert plan.workspace_bytes(kvc.LOSSLESS, True, 0) >= 32
    assert plan.max_encoded_bytes(kvc.TRANSFORM, 1) == 0  # no bases: lossless-only plan
    assert kvc.stream_buffer_bytes(plan, kvc.LOSSLESS, 1) > 3 * plan.max_encoded_bytes(kvc.LOSSLESS, 1)
    assert kvc.stream_buffer_bytes(plan, kvc.LOSSLESS, 0) == 0


def test_plan_validation():
    with pytest.raises(kvc.KvcError) as e:
        kvc.Plan(kvc.Shape(kvc.BF16, 0, 8, 512, 128))
    assert e.value.status == kvc.ERR_INVALID
    with pytest.raises(kvc.KvcError):
        kvc.Plan(kvc.Shape(4, 1, 8, 512, 128))  # no such value type
    q = np.eye(128, dtype=np.float32)[None].repeat(16, 0)
    with pytest.raises(kvc.KvcError) as e:  # f32 is lossless only
        kvc.Plan(kvc.Shape(kvc.F32, 1, 8, 512, 128), bases=q, widths=np.ones((16, 128), np.uint8))
    assert e.value.status == kvc.ERR_INVALID
    with pytest.raises(kvc.KvcError):
        kvc.Plan(kvc.Shape(kvc.BF16, 1, 8, 512, 128, values_per_chunk=100000))


def test_allocation_matches_oracle():
    rng = np.random.default_rng(0)
    for trial in range(30):
        U = int(rng.integers(1, 3000))
        lam = np.exp(rng.standard_normal(U) * 3)
        if trial % 3 == 0:
            lam[rng.integers(0, U, U // 4)] = 1.0          # exact ties
        if trial % 4 == 1:
            lam[rng.integers(0, U, U // 5)] = 0.0          # no variance
            lam[rng.integers(0, U, 3)] = -1e-17            # round-off below zero
        for avg in [0.0, 0.7, 1.6, 2.0, 5.5]:
            mb = int(rng.integers(max(1, int(np.ceil(avg))), 9))
            got = kvc.allocate_bits(lam, avg, mb)
            want = oracle.allocate(lam, avg, mb)
            assert np.array_equal(got, want), (trial, avg, mb)


def test_allocation_on_calibrated_workload_matches_oracle():
    w = dataclasses.replace(kvgen.WORKLOADS["transform-32x8x8192x128-bf16"], n_layers=2)
    shape = kvc.Shape.from_workload(w)
    bases, lam = kvc.calibrate_pca(shape, kvgen.calibration(w))
    assert np.array_equal(kvc.allocate_bits(lam, w.avg_bits), oracle.allocate(lam, w.avg_bits))


@pytest.mark.parametrize("heads", [1])
def test_calibration_matches_oracle_pca(heads):
    w = dataclasses.replace(kvgen.WORKLOADS["transform-32x8x8192x128-bf16"], n_layers=1,
                            n_heads=heads)
    shape = kvc.Shape.from_workload(w)
    cal = kvgen.calibration(w)
    bases, lam = kvc.calibrate_pca(shape, cal)
    D = w.head_dim
    for s in range(w.n_slices):
        Qo, lo = oracle.pca(cal[s], (s // w.n_heads) % 2 == 0, w.theta)
        assert np.allclose(lam[s], lo, rtol=1e-9, atol=1e-9 * lo[0])
        Q = bases[s].astype(np.float64)
        assert np.abs(Q.T @ Q - np.eye(D)).max() < 1e-5
        gap = np.minimum(np.r_[np.inf, -np.diff(lo)], np.r_[-np.diff(lo), np.inf]) / lo[0]
        sep = gap > 1e-3
        # same sign convention, so separated components agree column by column
        assert np.abs(bases[s][:, sep] - Qo[:, sep]).max() < 1e-4


@pytest.mark.parametrize("kind", [kvc.BASIS_HADAMARD, kvc.BASIS_DCT])
def test_fixed_basis_calibration_matches_oracle_bit_for_bit(kind):
    """The library's calibration-free bases and component variances equal the
    oracle's exactly (same closed forms, same fp64 sums in the same order)."""
    for D in (8, 128):
        a = kvc.fixed_basis(kind, D)
        b = oracle.fixed_basis(kind, D)
        assert np.array_equal(a.view(np.uint32), b.view(np.uint32))
    w = dataclasses.replace(kvgen.WORKLOADS["transform-32x8x8192x128-bf16"], n_layers=1, n_heads=2)
    shape = kvc.Shape.from_workload(w)
    cal = kvgen.calibration(w)
    bases, lam = kvc.calibrate_basis(shape, kind, cal)
    for s in range(w.n_slices):
        assert np.array_equal(bases[s], oracle.fixed_basis(kind, w.head_dim))
        lo = oracle.basis_variances(cal[s], (s // w.n_heads) % 2 == 0, w.theta, bases[s])
        assert np.array_equal(lam[s].view(np.uint64), lo.view(np.uint64))
    widths = kvc.allocate_bits(lam, w.avg_bits, w.max_bits)
    owidths = oracle.allocate(lam, w.avg_bits, w.max_bits).reshape(lam.shape)
    assert np.array_equal(widths.reshape(lam.shape), owidths)


def test_fixed_basis_refusals():
    with pytest.raises(kvc.KvcError):
        kvc.fixed_basis(kvc.BASIS_HADAMARD, 96)
    with pytest.raises(kvc.KvcError):
        kvc.fixed_basis(9, 8)


def test_stream_host_argument_checks():
    """The host-streamed calls refuse bad arguments before touching a device:
    no frame size, a misaligned or too small device ring, too many slices."""
    import types

    import torch
    null = types.SimpleNamespace(cuda_stream=0)  # the legacy default stream; no CUDA context needed here
    plan = kvc.Plan(kvc.Shape(kvc.BF16, 1, 8, 512, 128))
    n = plan.shape.n_slices
    src = torch.zeros(n * 512 * 128, dtype=torch.int16)
    dst = torch.zeros(plan.max_encoded_bytes(kvc.LOSSLESS, n), dtype=torch.uint8)
    fb = torch.zeros(n, dtype=torch.int64)
    res = torch.zeros(n, 2, dtype=torch.int64)
    need = kvc.stream_buffer_bytes(plan, kvc.LOSSLESS, 4)
    assert need > 0 and kvc.stream_buffer_bytes(plan, kvc.LOSSLESS, n + 1) == 0
    assert kvc.stream_buffer_bytes(plan, kvc.TRANSFORM, 4) == 0  # no bases: lossless-only plan
    raw = torch.zeros(1024 + 256, dtype=torch.uint8)
    small = raw[(-raw.data_ptr()) % 256:][:1024]  # 256-byte aligned, far too small
    cases = [
        (lambda: kvc.stream_encode_host(plan, kvc.LOSSLESS, 0, n, 0, src, dst, fb, res, small, null), kvc.ERR_INVALID),
        (lambda: kvc.stream_encode_host(plan, kvc.LOSSLESS, 1, n, 4, src, dst, fb, res, small, null), kvc.ERR_INVALID),
        (lambda: kvc.stream_encode_host(plan, kvc.LOSSLESS, 0, n, 4, src, dst, fb, res, small, null), kvc.ERR_CAPACITY),
        (lambda: kvc.stream_decode_host(plan, kvc.LOSSLESS, n, 0, dst, fb, src, res, small, null), kvc.ERR_INVALID),
        (lambda: kvc.stream_decode_host(plan, kvc.LOSSLESS, n, 4, dst, fb, src, res, small, null), kvc.ERR_CAPACITY),
        (lambda: kvc.stream_encode_host(plan, kvc.TRANSFORM, 0, n, 4, src, dst, fb, res, small, null), kvc.ERR_UNSUPPORTED),
    ]
    for call, want in cases:
        with pytest.raises(kvc.KvcError) as e:
            call()
        assert e.value.status == want


def test_plan_held_until_interpreter_exit_is_released_quietly():
    # A plan still referenced by a module global is collected after the
    # binding's own globals are cleared; its destructor must not need them.
    import subprocess
    import sys
    # Importing torch first is what puts the binding's module teardown ahead
    # of the plan's collection.
    code = ("import torch\n"
            "import transform_codec_b200 as kvc\n"
            "p = kvc.Plan(kvc.Shape(kvc.BF16, 2, 2, 1024, 128))\n"
            "print(p.max_encoded_bytes(kvc.LOSSLESS, 4))\n")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    assert int(r.stdout.split()[-1]) > 0
    assert "Exception ignored" not in r.stderr, r.stderr
