"""Host model of the encoder's exact projection and its error bound (CPU only).

The transform encoder quantises y = fl32(acc), acc the oracle's fp64 chain
sum over k ascending of Q[k][j] x_k (Codec-Gauge, "Problem Statement and
Overview": the per-head basis projection; KVTC, "How the Pipeline Works":
project, then quantise per block). On the GPU the projection is estimated from
exact integer byte products on the tensor cores, and every decision (a block's
or a token's extremes, a code near a rounding boundary) that the estimate's
error bound R leaves open is settled by running the fp64 chain itself. So the
encoder's containers equal the oracle's only if R really bounds |y - y~|.

This file restates the integer scheme in exact integer arithmetic: per token
X = rint(x 2^(29 - e)), per basis column J = rint(Q 2^(29 - f)), both split
into four two's-complement bytes (the top byte signed), the ten byte pairs
with a + b <= 3 summed into four levels, the levels combined in fp32 by
correctly rounded fused multiply-adds and scaled by 2^(e + f - 34). It then
checks, against the oracle's own projection, that |y - y~| <= R on random,
scaled, adversarial and PCA-of-cache inputs, for R per 64-token block and
column (block ranges) and per token over its coded columns (per-token ranges,
Codec-Gauge "Compression Conditions"), and that every level stays inside the
range its fp32 conversion is exact in.

The second half checks the rule by which a code is taken from the estimate
without the chain: with qa = RN(RN(y~ - z) RN(1/s)), a code is settled when the
distance from qa to the nearest half-integer exceeds RU(R RN(1/s) (1 + 2^-19))
+ |qa| 2^-19. The oracle's quantiser (q = rint(RN(RN(y - z) / s)), clamped to
[0, 2^b - 1]) is monotone in y, so a settled code is right for every fp32 y in
[y~ - R, y~ + R] exactly when the oracle's codes at the two ends of that set
equal rint(qa); that is checked on quotients placed next to half-integers.
"""
import dataclasses
import math

import numpy as np
import pytest

import kvgen
import oracle

D = 128
BLOCK = 64
# the six dropped pairs (a + b >= 4, both bytes unsigned, 128 terms each of at
# most 255^2, weights 2^16 (a + b = 4: three pairs), 2^8 (two) and 1 (one)),
# plus 96 units for rounding x and Q to integers
DROP_UNITS = 128 * 255 ** 2 * (3 * 2 ** 16 + 2 * 2 ** 8 + 1) + 96
SLACK = 1.0 + 2.0 ** -40
F32 = np.float32


def _ilogb(a):
    return np.frexp(np.asarray(a, np.float64))[1] - 1


def _f32_up(v: float) -> np.float32:
    """The least fp32 number >= v."""
    r = np.float32(v)
    if float(r) < v:
        r = np.nextafter(r, np.float32(np.inf))
    return r


def _l1_up(a: np.ndarray) -> np.ndarray:
    """Per row, an fp32 upper bound of sum |a| (the least the bound admits,
    up to one fp64 rounding of an exactly rounded sum)."""
    return np.array([_f32_up(math.fsum(np.abs(r.astype(np.float64))) * (1.0 + 2.0 ** -52))
                     for r in np.atleast_2d(a)], np.float32)


def _bytes(v: np.ndarray):
    """The four bytes of |v| <= 2^30 as two's complement: byte 0 (the top
    one) signed, bytes 1..3 unsigned."""
    u = np.asarray(v, np.int64) & 0xFFFFFFFF
    b = [(u >> (24 - 8 * p)) & 0xFF for p in range(4)]
    b[0] = np.where(b[0] >= 128, b[0] - 256, b[0])
    return b


def _integers(a: np.ndarray):
    """Per row of a (fp32): exponent ilogb(max |a|) (None for an all-zero
    row) and the integers rint(a 2^(29 - e))."""
    a64 = a.astype(np.float64)
    m = np.abs(a64).max(axis=1)
    zero = m == 0.0
    e = np.where(zero, 0, _ilogb(np.where(zero, 1.0, m)))
    ints = np.rint(a64 * np.ldexp(1.0, 29 - e)[:, None]).astype(np.int64)
    return e, ints, zero


def _estimate(Q: np.ndarray, x: np.ndarray):
    """The encoder's estimate y~ (T, D) of x (T, D) projected on the columns of
    Q (D, D), with the exponents, 1-norm bounds and levels its bound uses."""
    et, X, zt = _integers(x)
    fj, J, zj = _integers(np.ascontiguousarray(Q.T))
    assert np.abs(X).max() <= 2 ** 30 and np.abs(J).max() <= 2 ** 30
    dx, dq = _bytes(X), _bytes(J)
    for d, v in ((dx, X), (dq, J)):  # the bytes recompose the integer
        assert np.array_equal(((d[0] * 256 + d[1]) * 256 + d[2]) * 256 + d[3], v)
    P = [np.zeros((x.shape[0], D), np.int64) for _ in range(4)]
    for a in range(4):
        for b in range(4 - a):
            # byte products summed over k: below 2^23 in magnitude, exact in fp64
            P[a + b] += np.rint(dx[a].astype(np.float64) @ dq[b].astype(np.float64).T).astype(np.int64)
    # the ranges the fp32 conversions of the levels rely on
    assert np.abs(P[0]).max() <= 2 ** 19 and np.abs(P[1]).max() < 2 ** 22
    assert np.abs(P[2]).max() < 2 ** 24 and np.abs(P[3]).max() < 2 ** 25
    f0 = P[0].astype(np.float64)
    f1 = P[1].astype(np.float64)
    f2 = ((P[2] >> 2) * 4).astype(np.float64)
    f3 = ((P[3] >> 3) * 8).astype(np.float64)
    # fused multiply-adds in fp32: each exact sum of integers below 2^53 in
    # fp64, rounded once to fp32
    v = np.float32(f0 * 256.0 + f1).astype(np.float64)
    v = np.float32(v * 256.0 + f2).astype(np.float64)
    v = np.float32(v * 256.0 + f3)
    V = ((P[0] * 256 + P[1]) * 256 + P[2]) * 256 + P[3]
    # the combination is within 2^-22 |v| + 2^11 of the exact V
    assert np.all(np.abs(v.astype(np.float64) - V) <= 2.0 ** -22 * np.abs(v.astype(np.float64)) + 2.0 ** 11)
    k = et[:, None] + fj[None, :] - 34
    # v 2^k in fp32; below the normal range in two steps, as the kernel does
    big = np.float32(v.astype(np.float64) * np.ldexp(1.0, np.maximum(k, -126)))
    small = np.float32(np.float32(v.astype(np.float64) * np.ldexp(1.0, k + 64)) * np.float32(2.0 ** -64))
    yv = np.where(k >= -126, big, small)
    yv = np.where(zt[:, None] | zj[None, :], np.float32(0.0), yv)
    return yv, et, zt, _l1_up(x), fj, zj, _l1_up(Q.T)


def _r(e, f, x1, q1, Ma):
    """R from the block's (or token's) exponent e and 1-norm bound x1, the
    column's (or slice's) f and q1, and the largest estimate magnitude Ma."""
    E = (math.ldexp(DROP_UNITS, e + f - 58) + float(x1) * (math.ldexp(1.0, f - 30) + math.ldexp(1.0, f - 45))
         + float(q1) * math.ldexp(1.0, e - 30))
    dl = Ma * 2.0 ** -21 + math.ldexp(1.0, e + f - 22) + 2.0 ** -148
    E *= SLACK
    M = Ma * (1.0 + 2.0 ** -21) + E + dl
    lm = math.frexp(M)[1] - 1 if M > 0.0 else -1000
    return float(_f32_up((E + dl + math.ldexp(1.0, max(lm - 23, -149))) * SLACK))


def _scan_bits(vals: np.ndarray):
    """The oracle's sequential scan for the smallest and largest value (a
    later value replaces the current one only when strictly beyond it), as
    fp32 bit patterns, so that -0 and +0 are told apart."""
    lo, hi = F32(np.inf), F32(-np.inf)
    for v in vals.astype(np.float32):
        if v < lo:
            lo = v
        if v > hi:
            hi = v
    return int(np.float32(lo).view(np.uint32)), int(np.float32(hi).view(np.uint32))


def _extremes_agree(y_f32, v_f32, exact, R, reach=2.0):
    """Candidates: estimates within reach R (2R in the encoder) of the
    smallest or largest estimate (thresholds rounded outward in fp32). The scan
    over exact values for candidates and exact entries, estimates elsewhere,
    must give the oracle's smallest and largest value bit for bit."""
    mn, mx = F32(v_f32.min()), F32(v_f32.max())
    two = F32(reach) * F32(R)
    lo_thr = _round_dir(np.array([mn]), np.array([two]), up=True)[0]
    hi_thr = _round_dir(np.array([mx]), np.array([-two]), up=False)[0]
    cand = (v_f32 <= lo_thr) | (v_f32 >= hi_thr)
    used = np.where(cand | exact, y_f32, v_f32)
    return _scan_bits(used) == _scan_bits(y_f32), int(cand.sum())


def _oracle_y(Q, x):
    return np.stack([oracle.project(Q, x[t]) for t in range(x.shape[0])])


def _check_block_ranges(Q, x, reach=2.0):
    """Block ranges: R per 64-token block and column, from the block's largest
    token exponent and 1-norm bound. Returns the largest |y - y~| / R."""
    y = _oracle_y(Q, x).astype(np.float64)
    yv, et, zt, x1, fj, zj, q1 = _estimate(Q, x)
    worst = 0.0
    for b0 in range(0, x.shape[0], BLOCK):
        live = ~zt[b0:b0 + BLOCK]
        assert np.all(yv[b0:b0 + BLOCK][~live] == 0) and np.all(y[b0:b0 + BLOCK][~live] == 0)
        if not live.any():
            continue
        em = int(et[b0:b0 + BLOCK][live].max())
        xm = x1[b0:b0 + BLOCK][live].max()
        for j in range(D):
            yb = y[b0:b0 + BLOCK, j][live]
            vb = yv[b0:b0 + BLOCK, j][live].astype(np.float64)
            if zj[j]:
                assert np.all(yb == 0) and np.all(vb == 0)
                continue
            R = _r(em, int(fj[j]), xm, q1[j], float(np.abs(yv[b0:b0 + BLOCK, j]).max()))
            err = np.abs(yb - vb).max()
            assert err <= R, (b0, j, err, R)
            worst = max(worst, err / R)
            agree, _ = _extremes_agree(y[b0:b0 + BLOCK, j].astype(np.float32), yv[b0:b0 + BLOCK, j],
                                       zt[b0:b0 + BLOCK], R, reach)
            assert agree, (b0, j)
    return worst


def _check_token_ranges(Q, x, coded):
    """Per-token ranges: R per token over its coded columns, from the token's
    own exponent and 1-norm bound and the coded columns' largest f and q1."""
    y = _oracle_y(Q, x).astype(np.float64)
    yv, et, zt, x1, fj, zj, q1 = _estimate(Q, x)
    cols = np.flatnonzero(coded)
    live_cols = cols[~zj[cols]]
    fmax = int(fj[live_cols].max())
    qmax = q1[cols].max()
    worst = 0.0
    for t in range(x.shape[0]):
        if zt[t]:
            assert np.all(y[t, cols] == 0) and np.all(yv[t, cols] == 0)
            continue
        R = _r(int(et[t]), fmax, x1[t], qmax, float(np.abs(yv[t, cols]).max()))
        err = np.abs(y[t, live_cols] - yv[t, live_cols].astype(np.float64)).max()
        assert err <= R, (t, err, R)
        worst = max(worst, err / R)
        agree, _ = _extremes_agree(y[t, cols].astype(np.float32), yv[t, cols], zj[cols], R)
        assert agree, t
    return worst


def _orthonormal(rng):
    return np.linalg.qr(rng.standard_normal((D, D)))[0].astype(np.float32)


def _mixed_tokens(rng, T):
    """Heavy-tailed channels, per-token scales over six decades, all-zero
    tokens, one-hot tokens and exact zeros inside tokens."""
    x = rng.standard_normal((T, D)) * np.exp(rng.standard_normal((T, D)))
    x *= 10.0 ** rng.uniform(-3, 3, (T, 1))
    x[rng.random((T, D)) < 0.05] = 0.0
    x[::29] = 0.0
    for t in range(5, T, 37):
        x[t] = 0.0
        x[t, rng.integers(D)] = rng.standard_normal()
    return x.astype(np.float32)


def test_block_ranges_bound_random_orthonormal():
    rng = np.random.default_rng(11)
    worst = max(_check_block_ranges(_orthonormal(rng), _mixed_tokens(rng, 320)) for _ in range(3))
    assert 0.01 < worst <= 1.0  # a bound that holds, and not a vacuous one


def test_block_ranges_bound_with_extreme_digits():
    """Largest magnitudes just below a power of two (top bytes at their limit,
    integers near 2^30), every lower byte populated by entries spread over
    twenty binades, and a block whose tokens differ by 2^20 in scale (the
    small tokens measured against the block's largest exponent)."""
    rng = np.random.default_rng(12)
    Q = _orthonormal(rng)
    Q[:, 0] = np.float32(1.0)  # a column of ones: |Q| at an exact power of two
    Q[:, 1] = 0.0
    Q[3, 1] = np.float32(2.0 - 2.0 ** -23)  # one entry just below 2
    Q[:, 2] = np.float32(-(1.0 - 2.0 ** -24))  # all entries just below 1 in magnitude
    T = 192
    sign = np.where(rng.random((T, D)) < 0.5, -1.0, 1.0)
    x = sign * np.ldexp(1.0 + rng.random((T, D)), -rng.integers(0, 20, (T, D)))
    x[:, 0] = sign[:, 0] * (2.0 - 2.0 ** -23)  # each token's max just below 2
    x[64:128] *= np.ldexp(1.0, -rng.integers(0, 21, (64, 1)))
    x[128:192:2] *= 2.0 ** -20
    assert _check_block_ranges(Q, x.astype(np.float32)) <= 1.0


def test_block_ranges_bound_tiny_tokens():
    """Tokens below 2^-98 (scaled in fp64 by the kernel) and estimates that
    fall below fp32's normal range (scaled in two steps)."""
    rng = np.random.default_rng(13)
    Q = _orthonormal(rng) * np.float32(2.0 ** -20)
    x = (rng.standard_normal((128, D)) * 2.0 ** -110).astype(np.float32)
    x[64:] = (rng.standard_normal((64, D)) * 2.0 ** -60).astype(np.float32)
    assert _check_block_ranges(Q, x) <= 1.0


def _near_ties(rng):
    """Two blocks of one token with a few entries moved by one ulp each, and a
    block of one token repeated: the block extremes lie within R of many
    other tokens, and the repeated block ties everywhere."""
    base = (rng.standard_normal(D) * 3).astype(np.float32)
    x = np.repeat(base[None], 3 * BLOCK, 0)
    for t in range(2 * BLOCK):
        idx = rng.integers(0, D, 4)
        way = np.where(rng.random(4) < 0.5, np.inf, -np.inf).astype(np.float32)
        x[t, idx] = np.nextafter(x[t, idx], way)
    x[2 * BLOCK:] = x[2 * BLOCK]
    return x


def test_block_extremes_among_near_ties():
    rng = np.random.default_rng(31)
    assert _check_block_ranges(_orthonormal(rng), _near_ties(rng)) <= 1.0


def test_extremes_without_candidates_are_caught():
    """With no reach (only the smallest and largest estimate run the chain),
    the scan misses true extremes among near ties: the check sees it."""
    rng = np.random.default_rng(31)
    with pytest.raises(AssertionError):
        _check_block_ranges(_orthonormal(rng), _near_ties(rng), reach=0.0)


@pytest.mark.parametrize("is_key", [True, False])
def test_block_and_token_ranges_bound_on_pca_of_the_cache(is_key):
    """The cache workload's own inputs: a slice of the 8k-token cache (keys
    with RoPE undone) on the oracle's PCA basis of its calibration tokens."""
    w = dataclasses.replace(kvgen.WORKLOADS["transform-32x8x8192x128-bf16"], n_layers=1, n_heads=1)
    s = 0 if is_key else 1
    Q, lam = oracle.pca(kvgen.calibration(w)[s], is_key, w.theta)
    raw = kvgen.slices(w, s, 1)[0][:384]
    x = (np.asarray(raw, np.uint32) << 16).view(np.float32)
    if is_key:
        cs = oracle.rope_table(raw.shape[0], D, w.theta)
        x = np.stack([oracle.rope_inverse(cs[t], x[t]) for t in range(x.shape[0])]).astype(np.float32)
    worst = _check_block_ranges(Q, x)
    assert 0.01 < worst <= 1.0
    coded = oracle.allocate(lam, w.avg_bits, w.max_bits) > 0
    assert coded.any() and not coded.all()
    assert _check_token_ranges(Q, x, coded) <= 1.0


def test_token_ranges_bound_random():
    rng = np.random.default_rng(14)
    Q = _orthonormal(rng)
    x = _mixed_tokens(rng, 256)
    coded = rng.random(D) < 0.7
    assert 0.001 < _check_token_ranges(Q, x, coded) <= 1.0


def test_a_planted_mistake_in_the_bound_is_caught():
    """R without its dropped-pair term no longer bounds the error on these
    inputs: the check above is sharp enough to see a missing term."""
    rng = np.random.default_rng(11)
    Q, x = _orthonormal(rng), _mixed_tokens(rng, 320)
    global DROP_UNITS
    saved = DROP_UNITS
    try:
        DROP_UNITS = 96
        with pytest.raises(AssertionError):
            _check_block_ranges(Q, x)
    finally:
        DROP_UNITS = saved


# ------------------------------------------------------------ settling codes
MAGIC = F32(12582912.0)  # 1.5 * 2^23: adding it rounds |q| < 2^22 to an integer


def _round_dir(a: np.ndarray, b: np.ndarray, up: bool) -> np.ndarray:
    """a + b (fp32 arrays) rounded to fp32 toward +inf (up) or -inf, from the
    exact sum as an unevaluated pair of fp64 numbers (two-sum)."""
    a64, b64 = a.astype(np.float64), b.astype(np.float64)
    s = a64 + b64
    bb = s - a64
    err = (a64 - (s - bb)) + (b64 - bb)
    r = s.astype(np.float32)
    r64 = r.astype(np.float64)
    if up:
        low = (r64 < s) | ((r64 == s) & (err > 0))
        return np.where(low, np.nextafter(r, F32(np.inf)), r)
    high = (r64 > s) | ((r64 == s) & (err < 0))
    return np.where(high, np.nextafter(r, F32(-np.inf)), r)


def _mul_up(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """a b (fp32) rounded toward +inf: the fp64 product of two fp32 numbers is exact."""
    p = a.astype(np.float64) * b.astype(np.float64)
    r = p.astype(np.float32)
    return np.where(r.astype(np.float64) < p, np.nextafter(r, F32(np.inf)), r)


def _oracle_code(y, z, s, levels):
    """The block-uniform quantiser of the oracle (Codec-Gauge, "Compression
    Conditions"): rint(RN(RN(y - z) / s)) clamped to [0, levels]."""
    q = np.rint((y - z) / s)
    return np.clip(q, 0, levels).astype(np.int64)


def _settle(v, z, s, R, exact, interval=True, quotient=True):
    """The encoder's decision from the estimate v: (settled, code). The two
    flags leave out the margin's interval term or its quotient term."""
    rs = F32(1.0) / s
    qa = (v - z) * rs
    mg = qa + MAGIC
    iq = mg.view(np.int32).astype(np.int64) - 0x4B400000
    d = F32(0.5) - np.abs(qa - (mg - MAGIC))
    mR = _mul_up(_mul_up(R, rs), np.full_like(R, F32(1.0 + 2.0 ** -19)))
    mR = mR if interval else np.zeros_like(R)
    mq = _mul_up(np.abs(qa), np.full_like(qa, F32(2.0 ** -19)))
    mq = mq if quotient else np.zeros_like(qa)
    m = _round_dir(np.where(exact, F32(0.0), mR), mq, up=True)
    return d > m, iq


def _settling_cases(rng, n):
    """Block ranges of random widths and offsets, quotients next to
    half-integers (offsets from 2^-30 to 1/2 of a code on either side, below
    0 and above the top code too), error bounds from 10^-9 to 10^-1 of a
    code, and exact estimates (R = 0)."""
    bits = rng.integers(1, 9, n)
    levels = (1 << bits) - 1
    z = (rng.standard_normal(n) * 10.0 ** rng.uniform(-4, 3, n)).astype(np.float32)
    span = (10.0 ** rng.uniform(-4, 3, n)).astype(np.float32)
    zx = (z + span).astype(np.float32)
    s = ((zx - z) / levels.astype(np.float32)).astype(np.float32)
    k = rng.integers(-1, levels + 1)
    off = np.where(rng.random(n) < 0.5, -1.0, 1.0) * 2.0 ** rng.uniform(-30, -1, n)
    v = (z.astype(np.float64) + (k + 0.5 + off) * s.astype(np.float64)).astype(np.float32)
    R = (s.astype(np.float64) * 10.0 ** rng.uniform(-9, -1, n)).astype(np.float32)
    exact = rng.random(n) < 0.2
    R = np.where(exact, F32(0.0), R)
    ok = (s > 0) & (F32(1.0) / s < F32(2.0 ** 126))
    return v[ok], z[ok], s[ok], R[ok], exact[ok], levels[ok]


def _settling_errors(v, z, s, R, exact, levels, **kw):
    settled, iq = _settle(v, z, s, R, exact, **kw)
    lo = _round_dir(v, -R, up=True)   # the fp32 numbers in [v - R, v + R] run
    hi = _round_dir(v, R, up=False)   # from RU(v - R) to RD(v + R)
    want = np.clip(iq, 0, levels)
    bad = settled & ((_oracle_code(lo, z, s, levels) != want) | (_oracle_code(hi, z, s, levels) != want))
    return settled, bad


def test_settled_codes_equal_the_oracles_on_the_whole_interval():
    rng = np.random.default_rng(21)
    v, z, s, R, exact, levels = _settling_cases(rng, 400_000)
    settled, bad = _settling_errors(v, z, s, R, exact, levels)
    assert not bad.any(), np.flatnonzero(bad)[:5]
    # both outcomes occur, and settled codes close to their margin are among them
    assert 0.2 < settled.mean() < 0.95
    rs = F32(1.0) / s
    qa = (v - z) * rs
    d = F32(0.5) - np.abs(qa - np.rint(qa))
    assert np.count_nonzero(settled & (d < 2 * (R * rs + np.abs(qa) * 2.0 ** -19))) > 1000


@pytest.mark.parametrize("interval,quotient", [(False, True), (True, False)])
def test_settling_without_a_margin_term_is_caught(interval, quotient):
    """Without the estimate's interval term (R / s), or without the term for
    the quotient's own rounding (|qa| 2^-19), some settled codes differ from
    the oracle's: the check sees either term go missing."""
    rng = np.random.default_rng(21)
    cases = _settling_cases(rng, 400_000)
    _, bad = _settling_errors(*cases, interval=interval, quotient=quotient)
    assert bad.any()
