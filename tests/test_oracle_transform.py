"""Pins for the oracle's transform-coding path (CPU only).

RoPE undo (KVTC page, "Why RoPE Has to Be Reversed First"), the per-head basis
projection and its inverse (Codec-Gauge, "Problem Statement and Overview"; the
G^-1 G round-trip sanity rows of "Evaluation Design"), greedy allocation (KVTC,
"Bit Budget Is Not Fair"), the block-uniform quantiser (Codec-Gauge,
"Compression Conditions") and the PCA/KLT basis (same section).
"""
import dataclasses
import itertools
import struct

import numpy as np
import pytest

import kvgen
from apportion import largest_remainder
import oracle


def _f32(h):
    return (np.asarray(h, np.uint32) << 16).view(np.float32)


def _bf16(f):
    return np.array([oracle.f32_to_bf16(float(v)) for v in np.ravel(f)], np.uint16).reshape(
        np.shape(f))


# --------------------------------------------------------------------------- RoPE
def test_rope_table_matches_numpy_within_one_ulp():
    T, D, theta = 300, 128, 5e5
    cs = oracle.rope_table(T, D, theta)
    i = np.arange(D // 2)
    ang = np.arange(T)[:, None] * theta ** (-(2.0 * i) / D)[None, :]
    ref = np.stack([np.cos(ang), np.sin(ang)], -1).astype(np.float32)
    ulp = np.spacing(np.abs(ref))
    assert np.all(np.abs(cs - ref) <= ulp)


def test_rope_unit_vectors_closed_form():
    """Forward rotation of e_i is c e_i + s e_(i+D/2); of e_(i+D/2) is
    -s e_i + c e_(i+D/2); the inverse uses the opposite angle."""
    D = 16
    cs = oracle.rope_table(40, D, 1e4)
    row = cs[37]
    for i in range(D // 2):
        c, s = row[i]
        e = np.zeros(D, np.float32); e[i] = 1
        f = oracle.rope_forward(row, e)
        assert f[i] == c and f[i + D // 2] == s and np.count_nonzero(f) <= 2
        g = oracle.rope_inverse(row, e)
        assert g[i] == c and g[i + D // 2] == -s
        e = np.zeros(D, np.float32); e[i + D // 2] = 1
        f = oracle.rope_forward(row, e)
        assert f[i] == -s and f[i + D // 2] == c


def test_rope_inverse_undoes_forward():
    rng = np.random.default_rng(0)
    D = 128
    cs = oracle.rope_table(8192, D, 5e5)
    for t in [0, 1, 5, 100, 4095, 8191]:
        for _ in range(20):
            x = (rng.standard_normal(D) * np.exp(rng.standard_normal(D))).astype(np.float32)
            y = oracle.rope_inverse(cs[t], oracle.rope_forward(cs[t], x))
            tol = 1e-6 * max(1.0, float(np.abs(x).max()))
            assert np.abs(y - x).max() <= tol
            if t == 0:
                assert np.array_equal(oracle.rope_forward(cs[t], x), x)
            xr = oracle.rope_forward(cs[t], x).astype(np.float64)
            assert abs(np.linalg.norm(xr) - np.linalg.norm(x)) <= 1e-6 * np.linalg.norm(x)


# --------------------------------------------------------------------- projection
def _random_orthogonal(rng, D):
    q, r = np.linalg.qr(rng.standard_normal((D, D)))
    return (q * np.sign(np.diag(r))).astype(np.float32)


def test_projection_identity_and_permutation_exact():
    rng = np.random.default_rng(1)
    D = 128
    x = rng.standard_normal(D).astype(np.float32)
    assert np.array_equal(oracle.project(np.eye(D, dtype=np.float32), x), x)
    perm = rng.permutation(D)
    P = np.zeros((D, D), np.float32)
    P[perm, np.arange(D)] = 1.0  # column j selects x[perm[j]]
    assert np.array_equal(oracle.project(P, x), x[perm])
    assert np.array_equal(oracle.unproject(P, x[perm]), x)


def test_projection_matches_fp64_matmul_and_parseval():
    rng = np.random.default_rng(2)
    D = 128
    Q = _random_orthogonal(rng, D)
    same = total = 0
    for _ in range(50):
        x = (rng.standard_normal(D) * 3).astype(np.float32)
        y = oracle.project(Q, x)
        ref = (Q.astype(np.float64).T @ x.astype(np.float64)).astype(np.float32)
        assert np.all(np.abs(y - ref) <= np.spacing(np.abs(ref)))
        same += int(np.sum(y == ref)); total += D
        nx, ny = np.linalg.norm(x.astype(np.float64)), np.linalg.norm(y.astype(np.float64))
        assert abs(nx - ny) <= 1e-6 * nx
        back = oracle.unproject(Q, y)
        assert np.sqrt(np.mean((back - x) ** 2) / np.mean(x ** 2)) <= 1e-6
    assert same >= 0.999 * total


# --------------------------------------------------------------------- allocation
def _distortion(lam, b):
    return float(np.sum(lam * 4.0 ** (-np.asarray(b, np.float64))))


def test_allocation_matches_brute_force():
    rng = np.random.default_rng(3)
    for trial in range(60):
        k = int(rng.integers(1, 5))
        lam = np.exp(rng.standard_normal(k) * 2)
        for budget in range(0, 8 * k + 1):
            w = oracle.allocate(lam, budget / k, 8)
            assert int(w.sum()) == budget and w.max(initial=0) <= 8
            best = min(_distortion(lam, b) for b in itertools.product(range(9), repeat=k)
                       if sum(b) == budget)
            assert _distortion(lam, w) <= best * (1 + 1e-12)


def _dp_min_distortion(lam, budget, max_bits=8):
    """Dynamic programming over units (KVTC "Bit Budget Is Not Fair": the
    reference path allocates by dynamic programming): best[c] is the least
    distortion of the units so far with exactly c bits spent."""
    best = np.full(budget + 1, np.inf)
    best[0] = 0.0
    for l in lam:
        nxt = np.full(budget + 1, np.inf)
        for b in range(max_bits + 1):
            if b > budget:
                break
            cand = best[: budget + 1 - b] + l * 4.0 ** (-b)
            nxt[b:] = np.minimum(nxt[b:], cand)
        best = nxt
    return best[budget]


@pytest.mark.parametrize("k", [16, 64, 200])
def test_allocation_equals_dynamic_programming(k):
    """The greedy allocation reaches the dynamic-programming optimum of
    sum lam * 4^-b at every budget (the marginal gains lam * 3/4 * 4^-b fall
    with b, so taking the largest gain first is exact)."""
    rng = np.random.default_rng(k)
    lam = np.exp(rng.standard_normal(k) * 3)
    lam[rng.integers(0, k, k // 8)] = lam[0]  # ties
    for avg in (0.25, 1.0, 1.6, 2.0, 4.5, 7.9):
        w = oracle.allocate(lam, avg, 8)
        budget = int(np.floor(avg * k + 0.5))
        assert int(w.sum()) == budget
        opt = _dp_min_distortion(lam, budget)
        assert abs(_distortion(lam, w) - opt) <= 1e-12 * max(opt, 1e-300) + 1e-300


def test_allocation_ties_go_to_lower_index_and_cap():
    w = oracle.allocate(np.ones(3), 4 / 3, 8)
    assert list(w) == [2, 1, 1]
    w = oracle.allocate(np.array([1.0, 1e6]), 9 / 2, 8)
    assert list(w) == [1, 8]
    w = oracle.allocate(np.array([5.0, 0.0, 5.0]), 1.0, 2)
    assert list(w) == [2, 0, 1]
    with pytest.raises(ValueError):
        oracle.allocate(np.ones(4), 9.0, 8)


def test_allocation_budget_rounding_and_monotone():
    rng = np.random.default_rng(4)
    lam = np.exp(rng.standard_normal(1000) * 3)
    w = oracle.allocate(lam, 1.6, 8)
    assert int(w.sum()) == int(np.floor(1.6 * 1000 + 0.5))
    order = np.argsort(-lam, kind="stable")
    assert np.all(np.diff(w[order].astype(int)) <= 0)


# ---------------------------------------------------------------------- quantiser
def _plan(T, D=128, L=1, H=1, sink=0, recent=0, block=64, chunk=64, theta=1e4, bases=None,
          widths=None):
    S = L * 2 * H
    if bases is None:
        bases = np.broadcast_to(np.eye(D, dtype=np.float32), (S, D, D)).copy()
    if widths is None:
        widths = np.full((S, D), 8, np.uint8)
    return oracle.Plan(oracle.BF16, L, H, T, D, n_sink=sink, n_recent=recent,
                       block_tokens=block, chunk_tokens=chunk, max_bits=8, rope_theta=theta,
                       bases=bases, widths=widths)


def test_quantiser_b8_hand_example():
    """V slice, Q = I: y = x. Component 0 holds 0, 1, ..., 63 (exact in bf16):
    z = 0, s = fl(63 / 255), codes = rint(t / s) = 0, 4, 8, ..., 125, 130, ..., 255."""
    T, D = 64, 4
    plan = _plan(T, D=D)
    x = np.zeros((T, D), np.float32)
    x[:, 0] = np.arange(T)
    src = _bf16(x)
    codes, qpre, zs = oracle.transform_slice_codes(plan, 1, src)
    assert zs[0, 0, 0, 0] == 0.0 and zs[0, 0, 0, 1] == np.float32(63) / np.float32(255)
    c = codes[:, 0]
    assert (c[0], c[1], c[2], c[31], c[32], c[63]) == (0, 4, 8, 125, 130, 255)
    assert np.all(codes[:, 1:] == 0) and np.all(zs[0, 1:, 0, 1] == 0)


@pytest.mark.parametrize("bits", [1, 2, 3, 5, 8])
def test_quantiser_properties(bits):
    rng = np.random.default_rng(bits)
    T, D = 250, 16
    plan = _plan(T, D=D, chunk=128, widths=np.full((2, D), bits, np.uint8))
    x = (rng.standard_normal((T, D)) * np.exp(rng.standard_normal(D))).astype(np.float32)
    src = _bf16(x)
    y = _f32(src)
    codes, qpre, zs = oracle.transform_slice_codes(plan, 1, src)
    levels = (1 << bits) - 1
    assert codes.max() <= levels
    for t0 in range(0, T, 64):
        c, blk = divmod(t0, 128)
        blk //= 64
        for j in range(D):
            seg = y[t0:t0 + 64, j]
            cs = codes[t0:t0 + 64, j]
            z, s = zs[c, j, blk]
            assert z == seg.min()
            assert cs[np.argmin(seg)] == 0 and cs[np.argmax(seg)] == levels
            yh = (cs.astype(np.float64) * s + z).astype(np.float32)  # = fmaf
            # s/2 from rounding to the nearest level, plus fp32 roundings of
            # y - z, the division and the fused dequantisation at the block's scale
            slack = 4 * np.spacing(np.float32(np.abs(seg).max() + abs(z)))
            assert np.all(np.abs(yh - seg) <= s / 2 + slack)


# ---------------------------------------------------------------------------- PCA
def test_jacobi_closed_forms():
    d = np.array([3.0, -1.0, 7.5, 0.25])
    V, w = oracle.jacobi_eigen(np.diag(d))
    assert np.array_equal(w, d) and np.array_equal(V, np.eye(4))
    a, b, c = 2.0, 0.7, -1.3
    V, w = oracle.jacobi_eigen(np.array([[a, b], [b, c]]))
    m, r = (a + c) / 2, np.hypot((a - c) / 2, b)
    assert np.allclose(sorted(w), [m - r, m + r], rtol=0, atol=1e-14)


@pytest.mark.parametrize("n", [3, 8, 32, 64])
def test_jacobi_vs_eigh(n):
    rng = np.random.default_rng(n)
    B = rng.standard_normal((n, n))
    A = B @ B.T + np.diag(rng.random(n))
    V, w = oracle.jacobi_eigen(A)
    assert np.allclose(np.sort(w), np.linalg.eigvalsh(A), rtol=1e-12, atol=1e-12)
    assert np.abs(V.T @ V - np.eye(n)).max() < 1e-12
    assert np.abs(A @ V - V * w).max() < 1e-10 * np.abs(A).max()
    assert abs(w.sum() - np.trace(A)) < 1e-10 * abs(np.trace(A))


@pytest.mark.parametrize("is_key", [True, False])
def test_pca_basis(is_key):
    w = dataclasses.replace(kvgen.WORKLOADS["transform-32x8x8192x128-bf16"], n_layers=1,
                            n_heads=1)
    cal = kvgen.calibration(w)[0 if is_key else 1]
    Q, lam = oracle.pca(cal, is_key, w.theta)
    D = 128
    assert np.abs(Q.astype(np.float64).T @ Q.astype(np.float64) - np.eye(D)).max() < 1e-5
    assert np.all(np.diff(lam) <= 0)
    amax = np.argmax(np.abs(Q), axis=0)
    assert np.all(Q[amax, np.arange(D)] > 0)
    cs = oracle.rope_table(cal.shape[0], D, w.theta)
    xs = np.stack([oracle.rope_inverse(cs[t], _f32(cal[t])) if is_key else _f32(cal[t])
                   for t in range(cal.shape[0])]).astype(np.float64)
    C = xs.T @ xs / xs.shape[0]
    ref = np.linalg.eigvalsh(C)[::-1]
    assert np.allclose(lam, ref, rtol=1e-9, atol=1e-9 * ref[0])
    _, vecs = np.linalg.eigh(C)
    vecs = vecs[:, ::-1]
    gap = np.minimum(np.r_[np.inf, -np.diff(ref)], np.r_[-np.diff(ref), np.inf]) / ref[0]
    sep = gap > 1e-3
    dots = np.abs(np.sum(vecs[:, sep] * Q[:, sep], axis=0))
    assert np.all(dots > 1 - 1e-5)


# ---------------------------------------------------------------- transform codec
def _workload(**kw):
    base = dataclasses.replace(kvgen.WORKLOADS["transform-32x8x8192x128-bf16"], n_layers=1,
                               n_heads=1)
    return dataclasses.replace(base, **kw)


def _pca_plan(w):
    cal = kvgen.calibration(w)
    Qs, lams = [], []
    for s in range(w.n_slices):
        Q, lam = oracle.pca(cal[s], (s // w.n_heads) % 2 == 0, w.theta)
        Qs.append(Q); lams.append(lam)
    lam = np.stack(lams)
    widths = oracle.allocate(lam, w.avg_bits, w.max_bits).reshape(lam.shape)
    return oracle.Plan.from_workload(w, bases=np.stack(Qs), widths=widths)


@pytest.mark.parametrize("T", [1024, 640, 100])
def test_transform_roundtrip_regions_and_codes(T):
    """T = 1024: middle 892 = 512 + 380 tokens (ragged chunk, 60-token last block);
    T = 100: no middle, everything raw."""
    w = _workload(n_tokens=T)
    plan = _pca_plan(w)
    x = kvgen.slices(w)
    c = oracle.encode_transform(plan, x)
    assert len(c) <= oracle.transform_bound(plan, w.n_slices)
    st, y = oracle.decode_transform(plan, c)
    assert st == oracle.OK
    s_end, r_start = min(4, T), max(min(4, T), T - 128)
    assert np.array_equal(y[:, :s_end], x[:, :s_end])
    assert np.array_equal(y[:, r_start:], x[:, r_start:])
    a, b = _f32(x).astype(np.float64), _f32(y).astype(np.float64)
    rel = np.sqrt(((a - b) ** 2).sum() / (a ** 2).sum())
    assert rel < 0.6  # reported, not a pin: 2.0 bits per value on this generator
    st, codes, zs = oracle.container_codes(plan, c, w.n_slices)
    assert st == oracle.OK
    for s in range(w.n_slices):
        cc, _, zz = oracle.transform_slice_codes(plan, s, x[s])
        assert np.array_equal(codes[s], cc) and np.array_equal(zs[s], zz)


def test_transform_eight_bits_identity_basis_is_near_lossless():
    """All components at 8 bits on the identity basis: |x^ - x| <= s/2 plus the
    rotation and bf16 roundings; the G^-1 G path alone (no quantisation) is
    checked by the projection round-trip pin above."""
    w = _workload(n_tokens=900)
    S, D = w.n_slices, 128
    plan = _plan(900, D=D, sink=4, recent=128, block=64, chunk=512, theta=w.theta)
    x = kvgen.slices(w)
    c = oracle.encode_transform(plan, x)
    st, y = oracle.decode_transform(plan, c)
    assert st == oracle.OK
    a, b = _f32(x).astype(np.float64), _f32(y).astype(np.float64)
    rng_blk = np.abs(a).max()
    assert np.abs(a - b).max() <= rng_blk * (1 / 255 + 2 ** -7)
    assert np.sqrt(((a - b) ** 2).sum() / (a ** 2).sum()) < 5e-3


def test_transform_refuses_tamper_truncation_and_plan_mismatch():
    w = _workload(n_tokens=700)
    plan = _pca_plan(w)
    x = kvgen.slices(w)
    c = bytearray(oracle.encode_transform(plan, x))
    rng = np.random.default_rng(7)
    for pos in list(range(0, 64 + 16 * 6, 3)) + list(rng.integers(0, len(c), 120)):
        orig = c[pos]
        c[pos] = orig ^ int(rng.integers(1, 256))
        assert oracle.decode_transform(plan, bytes(c))[0] != oracle.OK, pos
        c[pos] = orig
    for n in list(range(0, 200)) + list(rng.integers(200, len(c), 50)):
        assert oracle.decode_transform(plan, bytes(c[:n]))[0] == oracle.TRUNCATED
    other_w = plan.widths.copy()
    other_w[0, 0] ^= 1
    other = oracle.Plan.from_workload(w, bases=plan.bases, widths=other_w)
    assert oracle.decode_transform(other, bytes(c))[0] == oracle.PLAN_MISMATCH


# ------------------------------------------------- calibration-free bases (f4)
@pytest.mark.parametrize("D", [2, 8, 64, 128])
def test_hadamard_basis_is_sylvester_hadamard(D):
    """Sylvester Hadamard matrix / sqrt(D), against scipy's construction; its
    columns multiply elementwise as the XOR of their indices (Walsh functions)."""
    import scipy.linalg
    Q = oracle.fixed_basis(oracle.HADAMARD, D)
    want = (scipy.linalg.hadamard(D).astype(np.float64) / np.sqrt(D)).astype(np.float32)
    assert np.array_equal(Q, want)
    if D == 2:
        h = np.float32(1.0 / np.sqrt(2.0))
        assert np.array_equal(Q, np.array([[h, h], [h, -h]], np.float32))
    s = np.sign(Q).astype(np.int64)
    j, l = 3 % D, (D - 1)
    assert np.array_equal(s[:, j] * s[:, l], s[:, j ^ l])
    assert np.abs(Q.astype(np.float64).T @ Q.astype(np.float64) - np.eye(D)).max() < 1e-6


@pytest.mark.parametrize("D", [2, 8, 64, 128])
def test_dct_basis_is_orthonormal_dct2(D):
    """Q^T x is the orthonormal DCT-II of x (scipy.fft.dct, norm='ortho'); the
    first component is the mean direction; a cosine of frequency m has all its
    energy in component m."""
    import scipy.fft
    Q = oracle.fixed_basis(oracle.DCT, D).astype(np.float64)
    M = scipy.fft.dct(np.eye(D), type=2, norm="ortho", axis=0)  # y = M x
    assert np.abs(Q.T - M).max() < 1e-7
    assert np.abs(Q[:, 0] - 1.0 / np.sqrt(D)).max() < 1e-7  # fp32 rounding of 1/sqrt(D)
    m = D // 2 - 1 if D > 2 else 1
    x = np.cos(np.pi * (2 * np.arange(D) + 1) * m / (2 * D))
    y = Q.T @ x
    assert abs(y[m] - np.sqrt(D / 2.0)) < 1e-5
    assert np.abs(np.delete(y, m)).max() < 1e-5
    assert np.abs(Q.T @ Q - np.eye(D)).max() < 1e-6


def test_fixed_basis_refusals():
    with pytest.raises(ValueError):
        oracle.fixed_basis(oracle.HADAMARD, 96)  # not a power of two
    with pytest.raises(ValueError):
        oracle.fixed_basis(7, 8)


@pytest.mark.parametrize("kind", [oracle.HADAMARD, oracle.DCT])
@pytest.mark.parametrize("is_key", [True, False])
def test_basis_variances_are_coordinate_second_moments(kind, is_key):
    """lambda_j equals the mean of y_j^2 over the calibration tokens (y = Q^T x
    per token, keys de-rotated) and the variances sum to the trace of C."""
    w = dataclasses.replace(kvgen.WORKLOADS["transform-32x8x8192x128-bf16"], n_layers=1,
                            n_heads=1)
    cal = kvgen.calibration(w)[0 if is_key else 1][:256]
    D = 128
    Q = oracle.fixed_basis(kind, D)
    lam = oracle.basis_variances(cal, is_key, w.theta, Q)
    cs = oracle.rope_table(cal.shape[0], D, w.theta)
    xs = np.stack([oracle.rope_inverse(cs[t], _f32(cal[t])) if is_key else _f32(cal[t])
                   for t in range(cal.shape[0])]).astype(np.float64)
    y = xs @ Q.astype(np.float64)
    ref = (y ** 2).mean(axis=0)
    assert np.allclose(lam, ref, rtol=1e-10, atol=1e-12 * ref.max())
    trace = (xs ** 2).sum(axis=1).mean()
    assert abs(lam.sum() - trace) < 1e-5 * trace  # fp32 basis: orthonormal to ~1e-7


def test_side_information_streams_layout():
    """A middle record opens with four stream records: byte plane q (low to high)
    of V = every z, then every s (coded components ascending, blocks in order),
    each coded with the lane-delta candidate on the side lane rule; the code
    streams follow. Also: the
    side streams of the AR(1) workload are smaller than the raw fp32 values."""
    w = _workload(n_tokens=1024)
    plan = _pca_plan(w)
    x = kvgen.slices(w)
    c = oracle.encode_transform(plan, x)
    _, _, zs = oracle.transform_slice_codes(plan, 0, x[0])
    coded = np.flatnonzero(plan.widths.reshape(w.n_slices, 128)[0])
    entries = np.frombuffer(c, dtype=np.uint8)[64:64 + 16 * 3].reshape(3, 16)
    off = int(entries[1, :8].view(np.uint64)[0])
    length = int(entries[1, 8:12].view(np.uint32)[0])
    nb = 8  # first middle chunk: 512 tokens
    V = np.concatenate([zs[0][coded, :nb, 0].reshape(-1), zs[0][coded, :nb, 1].reshape(-1)]).astype(np.float32)
    planes = V.view(np.uint32)
    want = b"".join(oracle.side_stream_encode(((planes >> (8 * q)) & 0xFF).astype(np.uint8))
                    for q in range(4))
    assert c[off:off + len(want)] == want
    assert len(want) < 4 * (16 + V.size) and len(want) < length


def _side_lanes(n):
    N = min(32, max(1, n // 64))
    base, extra = divmod(n, N)
    return [base + (l < extra) for l in range(N)]


@pytest.mark.parametrize("n", [64, 127, 128, 200, 1000, 1600, 2047, 2048])
@pytest.mark.parametrize("kbits", [1, 3])
def test_side_stream_lane_rule_by_bit_packing(n, kbits):
    """Side streams take min(32, max(1, n // 64)) lanes in one group. With a
    uniform alphabet of 2^k symbols (f = 2^(12-k)) every symbol inserts exactly
    k bits, so the group's sub-stream is sum over lanes of 4 + 2 floor(k len / 16)
    bytes: the closed form fixes the lane count and the lane ranges."""
    reps = -(-n // (1 << kbits))
    sym = np.tile(np.arange(1 << kbits, dtype=np.uint8), reps)[:n]
    if n % (1 << kbits):
        return  # the closed form needs every symbol equally often
    rng = np.random.default_rng(n * 10 + kbits)
    rng.shuffle(sym)
    rec = oracle.side_stream_encode(sym)
    k = 1 << kbits
    sub_pred = sum(4 + 2 * ((kbits * ln) // 16) for ln in _side_lanes(n))
    rans_pred = (48 + 2 * k + 15) // 16 * 16 + 16 + (sub_pred + 15) // 16 * 16
    raw = 16 + (n + 15) // 16 * 16
    if rec[0] == 2 and rec[3] == 0:  # plain RANS: one group whose sub-stream has the closed-form length
        assert rec[2] == 1 and rans_pred < raw
        lens_at = (48 + 2 * k + 15) // 16 * 16
        assert int.from_bytes(rec[lens_at:lens_at + 4], "little") == sub_pred
    elif rec[0] == 0:
        assert rans_pred >= raw
    else:  # lane deltas, taken only when strictly smaller than both
        assert rec[0] == 2 and rec[2] == 1 and len(rec) < min(rans_pred, raw)
    st, out, used = oracle.side_stream_decode(rec, n)
    assert st == 0 and used == len(rec) and np.array_equal(out, sym)


@pytest.mark.parametrize("n", [1, 63, 64, 500, 2048])
def test_side_stream_roundtrip_and_refusals(n):
    """Round trip of smooth side planes (the lane delta is taken where it is
    strictly smaller); a side record read on the code streams' lane rule, or
    with one byte changed in its header, is refused."""
    rng = np.random.default_rng(n)
    x = (np.cumsum(rng.integers(-2, 3, n)) % 256).astype(np.uint8)
    rec = oracle.side_stream_encode(x)
    st, out, used = oracle.side_stream_decode(rec, n)
    assert st == 0 and used == len(rec) and np.array_equal(out, x)
    if rec[0] == 2 and n // 64 > 1:
        assert oracle.stream_decode(rec, n)[0] != 0  # other lane count: refused or wrong end state
    bad = bytearray(rec)
    bad[8] ^= 1  # symbol count
    assert oracle.side_stream_decode(bytes(bad), n)[0] != 0


def _rans_record_one_lane(sym, N=1):
    """A RANS stream record of N interleaved lanes (groups of 32), written
    here from the format (header, presence bitmap, frequencies, one sub-stream
    lengths, each group's final states and words) with a plain rANS encoder
    (J. Duda, arXiv:1311.2540; 32-bit state, L = 2^16, 16-bit words,
    M = 2^12; lane l codes the contiguous range [start_l, start_l + len_l),
    len_l = n // N + (l < n % N)), whatever its size against RAW. The decoder
    reads, step by step, the lanes in ascending order, so the encoder runs
    the steps backwards with the lanes in descending order and prepends its
    words."""
    n = sym.size
    counts = np.bincount(sym, minlength=256)
    freq, k = largest_remainder(counts)  # the tests' own restatement of the table rule
    freq = np.asarray(freq, np.int64)
    cum = np.concatenate([[0], np.cumsum(freq)[:-1]])
    base, extra = divmod(n, N)
    lens = [base + (1 if l < extra else 0) for l in range(N)]
    starts = np.concatenate([[0], np.cumsum(lens)[:-1]]).astype(int)
    syms = sym.tolist()
    pad = lambda b: b + bytes(-len(b) % 16)  # noqa: E731
    subs = []
    for g0 in range(0, N, 32):  # one sub-stream per group of 32 lanes
        lanes = range(g0, min(N, g0 + 32))
        x, words = {l: 1 << 16 for l in lanes}, []
        for tau in range(lens[g0] - 1, -1, -1):
            for l in reversed(lanes):
                if tau >= lens[l]:
                    continue
                s = syms[starts[l] + tau]
                f = int(freq[s])
                if x[l] >= f << 20:
                    words.append(x[l] & 0xFFFF)
                    x[l] >>= 16
                x[l] = ((x[l] // f) << 12) + (x[l] % f) + int(cum[s])
        words = words[::-1]  # the decoder reads the last emitted word first
        subs.append(b"".join(struct.pack("<I", x[l]) for l in lanes) + b"".join(struct.pack("<H", w) for w in words))
    bitmap = bytearray(32)
    for s in np.flatnonzero(freq):
        bitmap[s >> 3] |= 1 << (s & 7)
    table = pad(bytes(bitmap) + b"".join(struct.pack("<H", int(freq[s])) for s in np.flatnonzero(freq)))
    body = table + pad(b"".join(struct.pack("<I", len(b)) for b in subs)) + b"".join(pad(b) for b in subs)
    return bytes([2, 0, len(subs), 0]) + struct.pack("<III", 16 + len(body), n, int(k)) + body


def test_side_stream_longer_than_raw_refused():
    """A RANS record longer than RAW is valid as a code stream (the general
    decoder restores it) but never comes from the side-stream encoder, whose
    never-worse choice would have written RAW; the side decoder refuses it."""
    rng = np.random.default_rng(5)
    sym = rng.integers(0, 64, 100).astype(np.uint8)  # one lane under both lane rules
    rec = _rans_record_one_lane(sym)
    assert len(rec) > 16 + 112  # longer than the RAW record of 100 symbols
    st, out, used = oracle.stream_decode(rec, sym.size)
    assert st == oracle.OK and used == len(rec) and np.array_equal(out, sym)
    assert oracle.side_stream_decode(rec, sym.size)[0] == oracle.CORRUPT
    small = rng.choice(np.array([3, 3, 3, 3, 9], np.uint8), 100)  # compressible: RANS below RAW
    rec2 = _rans_record_one_lane(small)
    assert len(rec2) < 16 + 112
    assert oracle.side_stream_decode(rec2, small.size)[0] == oracle.OK


@pytest.mark.parametrize("n", [100, 300, 511, 1023])
def test_oracle_rans_records_equal_independent_encoder(n):
    """Where the oracle writes a one-lane RANS record (n < 1024, compressible
    symbols), its bytes equal those of the independent single-lane encoder
    above: the state update, the renormalisation, the word order and the
    record layout are pinned byte for byte."""
    rng = np.random.default_rng(n)
    sym = np.minimum(rng.geometric(0.35 if n > 400 else 0.8, n) - 1, 255).astype(np.uint8)
    if np.unique(sym).size < 2:
        sym[0] = sym[0] ^ 1
    rec = oracle.stream_encode(sym)
    assert rec[0] == 2  # RANS is the smaller record for these symbols
    assert rec == _rans_record_one_lane(sym)


@pytest.mark.parametrize("n", [1100, 5000, 16000])
def test_oracle_interleaved_rans_equals_independent_encoder(n):
    """Code streams of 2 to 31 lanes (n // 512, one group) and side streams of
    3 to 32 lanes (n // 64): the oracle's RANS records equal the independent
    interleaved encoder's byte for byte."""
    rng = np.random.default_rng(n)
    sym = np.minimum(rng.geometric(0.3, n) - 1, 255).astype(np.uint8)
    rec = oracle.stream_encode(sym)
    assert rec[0] == 2 and rec[2] == 1
    assert rec == _rans_record_one_lane(sym, min(128, max(1, n // 512)))
    m = min(n // 4, 2048)
    side = sym[:m].copy()
    srec = oracle.side_stream_encode(side)
    plain = _rans_record_one_lane(side, min(32, max(1, m // 64)))
    if srec[0] == 2 and srec[3] == 0:  # plain RANS: the same bytes
        assert srec == plain
    elif srec[0] == 0:  # RAW: the plain RANS record is not smaller
        assert len(plain) >= len(srec)
    else:  # lane deltas: strictly smaller than the plain record
        assert srec[0] == 2 and len(srec) < len(plain) and oracle.side_stream_decode(srec, m)[0] == oracle.OK


def test_oracle_lossless_plane_equals_independent_encoder():
    """A full 65,536-symbol lossless plane: 128 lanes in four groups; the
    oracle's RANS record equals the independent encoder's byte for byte."""
    rng = np.random.default_rng(65536)
    sym = np.minimum(rng.geometric(0.25, 65536) - 1, 255).astype(np.uint8)
    rec = oracle.stream_encode(sym)
    assert rec[0] == 2 and rec[2] == 4
    assert rec == _rans_record_one_lane(sym, 128)
