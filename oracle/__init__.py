"""CPU oracle for the KV codec — TEST INFRASTRUCTURE.

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg
may import this package. It wraps ``libkvco.so`` (plain single-threaded C, see
kvco.c), which shares no code with the GPU library.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kvco.c")
_HDR = os.path.join(_HERE, "kvco.h")
_LIB = os.path.join(_HERE, "libkvco.so")
_lib = None

BF16, FP16, F32 = 1, 2, 3
OK, INVALID, CAPACITY, CORRUPT, TRUNCATED, PLAN_MISMATCH = 0, 1, 2, 3, 4, 5


def compile_command() -> list[str]:
    return ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fPIC", "-shared",
            "-o", _LIB, _SRC, "-lm"]


def build() -> str:
    newest = max(os.path.getmtime(_SRC), os.path.getmtime(_HDR))
    if not os.path.exists(_LIB) or os.path.getmtime(_LIB) < newest:
        subprocess.check_call(compile_command())
    return _LIB


class Desc(ctypes.Structure):
    _fields_ = [
        ("dtype", ctypes.c_uint32), ("n_layers", ctypes.c_uint32),
        ("n_heads", ctypes.c_uint32), ("n_tokens", ctypes.c_uint32),
        ("head_dim", ctypes.c_uint32), ("values_per_chunk", ctypes.c_uint32),
        ("n_sink", ctypes.c_uint32), ("n_recent", ctypes.c_uint32),
        ("block_tokens", ctypes.c_uint32), ("chunk_tokens", ctypes.c_uint32),
        ("max_bits", ctypes.c_uint32), ("rope_theta", ctypes.c_double),
        ("bases", ctypes.c_void_p), ("widths", ctypes.c_void_p),
        ("plan_crc", ctypes.c_uint32), ("plan_crc_set", ctypes.c_uint32),
        ("ranges", ctypes.c_uint32),
    ]


RANGES_BLOCK, RANGES_KIVI = 0, 1


def _load():
    global _lib
    if _lib is not None:
        return _lib
    build()
    lib = ctypes.CDLL(_LIB)
    vp, sz, u32, u64, i32, dbl = (ctypes.c_void_p, ctypes.c_size_t, ctypes.c_uint32,
                                  ctypes.c_uint64, ctypes.c_int, ctypes.c_double)
    P = ctypes.POINTER
    sig = {
        "kvco_crc32": ([vp, sz], u32),
        "kvco_normalize": ([vp, vp], i32),
        "kvco_stream_bound": ([u32], sz),
        "kvco_stream_encode": ([vp, u32, vp], sz),
        "kvco_stream_encode_delta": ([vp, u32, vp], sz),
        "kvco_side_stream_encode": ([vp, u32, vp], sz),
        "kvco_side_stream_decode": ([vp, sz, u32, vp, P(sz)], i32),
        "kvco_lane_delta": ([vp, u32, vp], None),
        "kvco_lane_undelta": ([vp, u32], None),
        "kvco_stream_decode": ([vp, sz, u32, vp, P(sz)], i32),
        "kvco_rans_payload_bytes": ([vp, u32], sz),
        "kvco_lossless_bound": ([P(Desc), u32], sz),
        "kvco_encode_lossless": ([P(Desc), u32, u32, vp, vp, sz], sz),
        "kvco_decode_lossless": ([P(Desc), vp, sz, vp, sz, P(u64)], i32),
        "kvco_rope_table": ([u32, u32, dbl, vp], None),
        "kvco_rope_inverse": ([vp, u32, vp], None),
        "kvco_rope_forward": ([vp, u32, vp], None),
        "kvco_project": ([vp, u32, vp, vp], None),
        "kvco_unproject": ([vp, u32, vp, vp], None),
        "kvco_allocate": ([vp, u64, dbl, u32, vp], i32),
        "kvco_plan_crc": ([P(Desc)], u32),
        "kvco_transform_bound": ([P(Desc), u32], sz),
        "kvco_encode_transform": ([P(Desc), u32, u32, vp, vp, sz], sz),
        "kvco_decode_transform": ([P(Desc), vp, sz, vp, sz, P(u64)], i32),
        "kvco_transform_slice_codes": ([P(Desc), u32, vp, vp, vp, vp], i32),
        "kvco_record_codes": ([P(Desc), u32, vp, u32, u32, vp, vp], i32),
        "kvco_container_codes": ([P(Desc), vp, sz, u32, vp, vp, P(u32)], i32),
        "kvco_pca": ([vp, u32, u32, u32, i32, dbl, vp, vp], i32),
        "kvco_jacobi_eigen": ([vp, u32, vp, vp], i32),
        "kvco_fixed_basis": ([u32, u32, vp], i32),
        "kvco_basis_variances": ([vp, u32, u32, u32, i32, dbl, vp, vp], i32),
        "kvco_bf16_to_f32": ([ctypes.c_uint16], ctypes.c_float),
        "kvco_f32_to_bf16": ([ctypes.c_float], ctypes.c_uint16),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    _lib = lib
    return lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def _buf(b) -> np.ndarray:
    return np.frombuffer(bytes(b), dtype=np.uint8) if not isinstance(b, np.ndarray) else b


class Plan:
    """A kvco_desc plus the arrays it points at (kept alive here)."""

    def __init__(self, dtype, n_layers, n_heads, n_tokens, head_dim, values_per_chunk=65536,
                 n_sink=4, n_recent=128, block_tokens=64, chunk_tokens=512, max_bits=8,
                 rope_theta=1e4, bases=None, widths=None, ranges=RANGES_BLOCK):
        self.bases = None if bases is None else np.ascontiguousarray(bases, dtype=np.float32)
        self.widths = None if widths is None else np.ascontiguousarray(widths, dtype=np.uint8)
        self.desc = Desc(dtype, n_layers, n_heads, n_tokens, head_dim, values_per_chunk,
                         n_sink, n_recent, block_tokens, chunk_tokens, max_bits, rope_theta,
                         None if self.bases is None else _ptr(self.bases),
                         None if self.widths is None else _ptr(self.widths))
        self._bound = {}
        self.desc.ranges = ranges
        if self.bases is not None and self.widths is not None:
            # the plan CRC every transform container carries, computed once here
            self.desc.plan_crc = _load().kvco_plan_crc(ctypes.byref(self.desc))
            self.desc.plan_crc_set = 1

    @property
    def n_slices(self):
        return self.desc.n_layers * 2 * self.desc.n_heads

    @classmethod
    def from_workload(cls, w, bases=None, widths=None, ranges=RANGES_BLOCK):
        return cls(w.dtype, w.n_layers, w.n_heads, w.n_tokens, w.head_dim, w.values_per_chunk,
                   w.n_sink, w.n_recent, w.block_tokens, w.chunk_tokens, w.max_bits, w.theta,
                   bases, widths, ranges)


def crc32(data) -> int:
    a = _buf(data)
    return _load().kvco_crc32(_ptr(a) if a.size else None, a.size)


def normalize(counts) -> tuple[np.ndarray, int]:
    c = np.ascontiguousarray(counts, dtype=np.uint32)
    f = np.zeros(256, dtype=np.uint16)
    k = _load().kvco_normalize(_ptr(c), _ptr(f))
    return f, k


def stream_encode(sym: np.ndarray) -> bytes:
    s = np.ascontiguousarray(sym, dtype=np.uint8)
    lib = _load()
    out = np.zeros(lib.kvco_stream_bound(s.size), dtype=np.uint8)
    n = lib.kvco_stream_encode(_ptr(s) if s.size else None, s.size, _ptr(out))
    return out[:n].tobytes()


def stream_encode_delta(sym: np.ndarray) -> bytes:
    """Stream record with the lane-delta candidate (the lossless planes' coder)."""
    s = np.ascontiguousarray(sym, dtype=np.uint8)
    lib = _load()
    out = np.zeros(lib.kvco_stream_bound(s.size), dtype=np.uint8)
    n = lib.kvco_stream_encode_delta(_ptr(s) if s.size else None, s.size, _ptr(out))
    return out[:n].tobytes()


def side_stream_encode(sym: np.ndarray) -> bytes:
    """Side stream record (a byte plane of a middle record's zero points and
    scales): the lane-delta choice on min(32, max(1, n // 64)) lanes."""
    s = np.ascontiguousarray(sym, dtype=np.uint8)
    lib = _load()
    out = np.zeros(lib.kvco_stream_bound(s.size), dtype=np.uint8)
    n = lib.kvco_side_stream_encode(_ptr(s) if s.size else None, s.size, _ptr(out))
    return out[:n].tobytes()


def side_stream_decode(rec: bytes, n: int):
    """(status, symbols, bytes used) of a side stream record of n symbols."""
    buf = np.frombuffer(bytes(rec), dtype=np.uint8).copy()
    out = np.zeros(max(n, 1), dtype=np.uint8)
    used = ctypes.c_size_t(0)
    st = _load().kvco_side_stream_decode(_ptr(buf) if buf.size else None, buf.size, n, _ptr(out),
                                         ctypes.byref(used))
    return st, out[:n], used.value


def lane_delta(sym: np.ndarray) -> np.ndarray:
    s = np.ascontiguousarray(sym, dtype=np.uint8)
    out = np.zeros_like(s)
    if s.size:
        _load().kvco_lane_delta(_ptr(s), s.size, _ptr(out))
    return out


def lane_undelta(sym: np.ndarray) -> np.ndarray:
    s = np.array(sym, dtype=np.uint8, copy=True)
    if s.size:
        _load().kvco_lane_undelta(_ptr(s), s.size)
    return s


def stream_decode(rec, n: int):
    r = _buf(rec)
    out = np.zeros(max(n, 1), dtype=np.uint8)
    used = ctypes.c_size_t(0)
    st = _load().kvco_stream_decode(_ptr(r) if r.size else None, r.size, n, _ptr(out),
                                    ctypes.byref(used))
    return st, out[:n], used.value


def rans_payload_bytes(sym: np.ndarray) -> int:
    s = np.ascontiguousarray(sym, dtype=np.uint8)
    return _load().kvco_rans_payload_bytes(_ptr(s), s.size)


def lossless_bound(plan: Plan, n_slices: int) -> int:
    return _load().kvco_lossless_bound(ctypes.byref(plan.desc), n_slices)


def _vtype(plan: Plan):
    """numpy type of one value's bits: uint32 for f32, else uint16."""
    return np.uint32 if plan.desc.dtype == F32 else np.uint16


def encode_lossless(plan: Plan, src: np.ndarray, first_slice: int = 0) -> bytes:
    s = np.ascontiguousarray(src, dtype=_vtype(plan))
    n_slices = s.size // (plan.desc.n_tokens * plan.desc.head_dim)
    lib = _load()
    cap = lib.kvco_lossless_bound(ctypes.byref(plan.desc), n_slices)
    out = np.zeros(max(cap, 1), dtype=np.uint8)
    n = lib.kvco_encode_lossless(ctypes.byref(plan.desc), first_slice, n_slices,
                                 _ptr(s) if s.size else None, _ptr(out), cap)
    if n == 0:
        raise ValueError("oracle lossless encode refused its arguments")
    return out[:n].tobytes()


def _decode(fn, plan, buf, n_slices_cap):
    b = _buf(buf)
    D, T = plan.desc.head_dim, plan.desc.n_tokens
    out = np.zeros(max(n_slices_cap * T * D, 1), dtype=_vtype(plan))
    written = ctypes.c_uint64(0)
    st = fn(ctypes.byref(plan.desc), _ptr(b) if b.size else None, b.size, _ptr(out),
            out.nbytes if n_slices_cap else 0, ctypes.byref(written))
    ns = written.value // (T * D * out.itemsize)
    return st, out[: ns * T * D].reshape(ns, T, D)


def decode_lossless(plan: Plan, buf, n_slices_cap: int | None = None):
    cap = plan.n_slices if n_slices_cap is None else n_slices_cap
    return _decode(_load().kvco_decode_lossless, plan, buf, cap)


def rope_table(T: int, D: int, theta: float) -> np.ndarray:
    cs = np.zeros(T * (D // 2) * 2, dtype=np.float32)
    _load().kvco_rope_table(T, D, theta, _ptr(cs))
    return cs.reshape(T, D // 2, 2)


def rope_inverse(cs_row: np.ndarray, x: np.ndarray) -> np.ndarray:
    c = np.ascontiguousarray(cs_row, dtype=np.float32)
    y = np.array(x, dtype=np.float32, copy=True)
    _load().kvco_rope_inverse(_ptr(c), y.size, _ptr(y))
    return y


def rope_forward(cs_row: np.ndarray, x: np.ndarray) -> np.ndarray:
    c = np.ascontiguousarray(cs_row, dtype=np.float32)
    y = np.array(x, dtype=np.float32, copy=True)
    _load().kvco_rope_forward(_ptr(c), y.size, _ptr(y))
    return y


def project(Q: np.ndarray, x: np.ndarray) -> np.ndarray:
    q = np.ascontiguousarray(Q, dtype=np.float32)
    xv = np.ascontiguousarray(x, dtype=np.float32)
    y = np.zeros(xv.size, dtype=np.float32)
    _load().kvco_project(_ptr(q), xv.size, _ptr(xv), _ptr(y))
    return y


def unproject(Q: np.ndarray, y: np.ndarray) -> np.ndarray:
    q = np.ascontiguousarray(Q, dtype=np.float32)
    yv = np.ascontiguousarray(y, dtype=np.float32)
    x = np.zeros(yv.size, dtype=np.float32)
    _load().kvco_unproject(_ptr(q), yv.size, _ptr(yv), _ptr(x))
    return x


def allocate(lam: np.ndarray, avg_bits: float, max_bits: int = 8) -> np.ndarray:
    l = np.ascontiguousarray(lam, dtype=np.float64).ravel()
    w = np.zeros(l.size, dtype=np.uint8)
    st = _load().kvco_allocate(_ptr(l), l.size, avg_bits, max_bits, _ptr(w))
    if st != OK:
        raise ValueError("oracle allocation refused its arguments")
    return w


def plan_crc(plan: Plan) -> int:
    return _load().kvco_plan_crc(ctypes.byref(plan.desc))


def transform_bound(plan: Plan, n_slices: int) -> int:
    return _load().kvco_transform_bound(ctypes.byref(plan.desc), n_slices)


def encode_transform(plan: Plan, src: np.ndarray, first_slice: int = 0) -> bytes:
    s = np.ascontiguousarray(src, dtype=np.uint16)
    n_slices = s.size // (plan.desc.n_tokens * plan.desc.head_dim)
    lib = _load()
    if n_slices not in plan._bound:
        plan._bound[n_slices] = lib.kvco_transform_bound(ctypes.byref(plan.desc), n_slices)
    cap = plan._bound[n_slices]
    out = np.zeros(max(cap, 1), dtype=np.uint8)
    n = lib.kvco_encode_transform(ctypes.byref(plan.desc), first_slice, n_slices,
                                  _ptr(s) if s.size else None, _ptr(out), cap)
    if n == 0:
        raise ValueError("oracle transform encode refused its arguments")
    return out[:n].tobytes()


def decode_transform(plan: Plan, buf, n_slices_cap: int | None = None):
    cap = plan.n_slices if n_slices_cap is None else n_slices_cap
    return _decode(_load().kvco_decode_transform, plan, buf, cap)


def _n_mid(plan: Plan) -> int:
    d = plan.desc
    s_end = min(d.n_sink, d.n_tokens)
    r_start = max(s_end, d.n_tokens - d.n_recent if d.n_tokens > d.n_recent else 0)
    return (r_start - s_end + d.chunk_tokens - 1) // d.chunk_tokens


def transform_slice_codes(plan: Plan, slice_index: int, src_slice: np.ndarray):
    d = plan.desc
    s = np.ascontiguousarray(src_slice, dtype=np.uint16)
    codes = np.zeros((d.n_tokens, d.head_dim), dtype=np.uint8)
    qpre = np.zeros((d.n_tokens, d.head_dim), dtype=np.float32)
    nbmax = d.chunk_tokens // d.block_tokens
    zs = np.zeros((max(_n_mid(plan), 1), d.head_dim, nbmax, 2), dtype=np.float32)
    st = _load().kvco_transform_slice_codes(ctypes.byref(d), slice_index, _ptr(s),
                                            _ptr(codes), _ptr(qpre), _ptr(zs))
    if st != OK:
        raise ValueError("oracle transform_slice_codes refused its arguments")
    return codes, qpre, zs[: _n_mid(plan)]


def record_codes(plan: Plan, slice_index: int, rec: bytes, tcc: int):
    d = plan.desc
    r = np.frombuffer(bytes(rec), dtype=np.uint8) if len(rec) else np.zeros(1, np.uint8)
    codes = np.zeros((tcc, d.head_dim), dtype=np.uint8)
    zs = np.zeros((d.head_dim, d.chunk_tokens // d.block_tokens, 2), dtype=np.float32)
    st = _load().kvco_record_codes(ctypes.byref(d), slice_index, _ptr(r), len(rec), tcc,
                                   _ptr(codes), _ptr(zs))
    return st, codes, zs


def container_codes(plan: Plan, buf, n_slices: int):
    d = plan.desc
    b = _buf(buf)
    nbmax = d.chunk_tokens // d.block_tokens
    nm = _n_mid(plan)
    codes = np.zeros((max(n_slices, 1), d.n_tokens, d.head_dim), dtype=np.uint8)
    zs = np.zeros((max(n_slices, 1), max(nm, 1), d.head_dim, nbmax, 2), dtype=np.float32)
    got = ctypes.c_uint32(0)
    st = _load().kvco_container_codes(ctypes.byref(d), _ptr(b), b.size, 0, _ptr(codes),
                                      _ptr(zs), ctypes.byref(got))
    return st, codes[:n_slices], zs[:n_slices, :nm]


def pca(calib: np.ndarray, is_key: bool, theta: float):
    c = np.ascontiguousarray(calib, dtype=np.uint16)
    n_tok, D = c.shape
    Q = np.zeros((D, D), dtype=np.float32)
    lam = np.zeros(D, dtype=np.float64)
    st = _load().kvco_pca(_ptr(c), n_tok, D, BF16, int(is_key), theta, _ptr(Q), _ptr(lam))
    if st != OK:
        raise ValueError("oracle PCA refused its arguments")
    return Q, lam


HADAMARD, DCT = 1, 2


def fixed_basis(kind: int, D: int) -> np.ndarray:
    """Calibration-free basis [D][D] fp32 (element [k][j]: channel k of component j)."""
    Q = np.zeros((D, D), dtype=np.float32)
    if _load().kvco_fixed_basis(kind, D, _ptr(Q)) != OK:
        raise ValueError("oracle refused the basis kind or size")
    return Q


def basis_variances(calib: np.ndarray, is_key: bool, theta: float, Q: np.ndarray) -> np.ndarray:
    """Second moment of each component of basis Q over the calibration tokens."""
    c = np.ascontiguousarray(calib, dtype=np.uint16)
    q = np.ascontiguousarray(Q, dtype=np.float32)
    n_tok, D = c.shape
    lam = np.zeros(D, dtype=np.float64)
    if _load().kvco_basis_variances(_ptr(c), n_tok, D, BF16, int(is_key), theta, _ptr(q), _ptr(lam)) != OK:
        raise ValueError("oracle refused its arguments")
    return lam


def jacobi_eigen(A: np.ndarray):
    a = np.ascontiguousarray(A, dtype=np.float64)
    n = a.shape[0]
    V = np.zeros((n, n), dtype=np.float64)
    w = np.zeros(n, dtype=np.float64)
    _load().kvco_jacobi_eigen(_ptr(a), n, _ptr(V), _ptr(w))
    return V, w


def bf16_to_f32(h: int) -> float:
    return _load().kvco_bf16_to_f32(h)


def f32_to_bf16(f: float) -> int:
    return _load().kvco_f32_to_bf16(f)
