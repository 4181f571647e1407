"""Python binding of libkvc.so, the B200 KV-cache codec (C ABI in include/kvc.h).

Argument marshalling only: every step of encoding and decoding runs in the
library's CUDA kernels. PyTorch supplies device memory and streams. There is no
CPU fallback: importing this package fails loudly when libkvc.so is missing.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
# KVC_BUILD_VARIANT=<name> loads the in-tree test build libkvc_<name>.so (see
# build.VARIANTS) instead of libkvc.so; a missing library fails the import.
_VARIANT = os.environ.get("KVC_BUILD_VARIANT", "")
if _VARIANT and not _VARIANT.isidentifier():
    raise ImportError(f"bad KVC_BUILD_VARIANT {_VARIANT!r}")
LIB_PATH = os.path.join(_HERE, f"libkvc_{_VARIANT}.so" if _VARIANT else "libkvc.so")

OK, ERR_INVALID, ERR_CAPACITY, ERR_CORRUPT, ERR_TRUNCATED, ERR_PLAN_MISMATCH = 0, 1, 2, 3, 4, 5
ERR_TIMEOUT, ERR_CUDA, ERR_UNSUPPORTED = 6, 7, 8
BF16, FP16, F32 = 1, 2, 3  # value types (f32: lossless only)
DTYPE_F32 = F32
LOSSLESS, TRANSFORM = 0, 1
ABI_VERSION = 2
RANGES_BLOCK, RANGES_KIVI = 0, 1  # transform value ranges: per block, or KIVI-style per-token values

EXPORTS = [
    "kvc_plan", "kvc_plan_create", "kvc_plan_destroy", "kvc_plan_widths", "kvc_plan_crc",
    "kvc_max_encoded_bytes", "kvc_workspace_bytes",
    "kvc_encode_lossless", "kvc_decode_lossless", "kvc_encode_transform", "kvc_decode_transform",
    "kvc_status_string", "kvc_calibrate_pca", "kvc_allocate_bits",
    "kvc_fixed_basis", "kvc_calibrate_basis",
    "kvc_stage_crc32", "kvc_stage_stream_encode", "kvc_stage_stream_decode",
    "kvc_stage_stream_encode_noalloc",
    "kvc_profile_begin", "kvc_profile_end",
    "kvc_batch_workspace_bytes", "kvc_encode_batch", "kvc_decode_batch",
    "kvc_stream_buffer_bytes", "kvc_stream_encode_host", "kvc_stream_decode_host",
]


class KvcError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})" if what else status_string(status))


class PlanDesc(ctypes.Structure):
    _fields_ = [
        ("abi_version", ctypes.c_uint32), ("dtype", ctypes.c_uint32),
        ("n_layers", ctypes.c_uint32), ("n_heads", ctypes.c_uint32),
        ("n_tokens", ctypes.c_uint32), ("head_dim", ctypes.c_uint32),
        ("values_per_chunk", ctypes.c_uint32),
        ("n_sink", ctypes.c_uint32), ("n_recent", ctypes.c_uint32),
        ("block_tokens", ctypes.c_uint32), ("chunk_tokens", ctypes.c_uint32),
        ("max_bits", ctypes.c_uint32),
        ("rope_theta", ctypes.c_double), ("avg_bits", ctypes.c_double),
        ("bases", ctypes.c_void_p), ("eigvals", ctypes.c_void_p), ("widths", ctypes.c_void_p),
        ("range_mode", ctypes.c_uint32), ("reserved", ctypes.c_uint32),
    ]


class Frame(ctypes.Structure):
    _fields_ = [("first_slice", ctypes.c_uint32), ("n_slices", ctypes.c_uint32),
                ("src", ctypes.c_void_p), ("src_bytes", ctypes.c_size_t),
                ("dst", ctypes.c_void_p), ("dst_cap", ctypes.c_size_t),
                ("res", ctypes.c_void_p)]


class KernelTime(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 40), ("launches", ctypes.c_uint32),
                ("total_ms", ctypes.c_double)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing; build it with transform_codec_b200.build.build()")
    lib = ctypes.CDLL(LIB_PATH)
    vp, sz, u32, i32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_uint32, ctypes.c_int
    sig = {
        "kvc_plan": ([ctypes.POINTER(PlanDesc), ctypes.POINTER(vp)], i32),
        "kvc_plan_create": ([ctypes.POINTER(PlanDesc), ctypes.POINTER(vp)], i32),
        "kvc_plan_destroy": ([vp], None),
        "kvc_plan_widths": ([vp, vp, sz], i32),
        "kvc_plan_crc": ([vp], u32),
        "kvc_max_encoded_bytes": ([vp, i32, u32], sz),
        "kvc_workspace_bytes": ([vp, i32, i32, u32], sz),
        "kvc_encode_lossless": ([vp, u32, u32, vp, vp, sz, vp, sz, vp, vp], i32),
        "kvc_decode_lossless": ([vp, vp, sz, vp, sz, vp, sz, vp, vp], i32),
        "kvc_encode_transform": ([vp, u32, u32, vp, vp, sz, vp, sz, vp, vp], i32),
        "kvc_decode_transform": ([vp, vp, sz, vp, sz, vp, sz, vp, vp], i32),
        "kvc_status_string": ([i32], ctypes.c_char_p),
        "kvc_calibrate_pca": ([ctypes.POINTER(PlanDesc), vp, u32, vp, vp, i32], i32),
        "kvc_allocate_bits": ([vp, ctypes.c_uint64, ctypes.c_double, u32, vp], i32),
        "kvc_fixed_basis": ([i32, u32, vp], i32),
        "kvc_calibrate_basis": ([ctypes.POINTER(PlanDesc), i32, vp, u32, vp, vp, i32], i32),
        "kvc_batch_workspace_bytes": ([vp, i32, i32, u32, u32], sz),
        "kvc_encode_batch": ([vp, i32, ctypes.POINTER(Frame), u32, vp, sz, vp], i32),
        "kvc_decode_batch": ([vp, i32, ctypes.POINTER(Frame), u32, u32, vp, sz, vp], i32),
        "kvc_stream_buffer_bytes": ([vp, i32, u32], sz),
        "kvc_stream_encode_host": ([vp, i32, u32, u32, u32, vp, vp, sz, vp, vp, vp, sz, vp], i32),
        "kvc_stream_decode_host": ([vp, i32, u32, u32, vp, vp, vp, sz, vp, vp, sz, vp], i32),
        "kvc_profile_begin": ([], i32),
        "kvc_profile_end": ([ctypes.POINTER(KernelTime), i32, ctypes.POINTER(i32)], i32),
        "kvc_stage_crc32": ([vp, sz, vp, vp], i32),
        "kvc_stage_stream_encode": ([vp, u32, vp, vp, vp, vp], i32),
        "kvc_stage_stream_decode": ([vp, u32, u32, vp, vp, vp], i32),
        "kvc_stage_stream_encode_noalloc": ([vp, u32, vp, vp, vp], i32),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    return lib


_lib = _load()


def lib():
    return _lib


def status_string(status: int) -> str:
    return _lib.kvc_status_string(int(status)).decode()


def _check(status: int, what: str):
    if status != OK:
        raise KvcError(status, what)


def _np_ptr(a):
    return None if a is None else a.ctypes.data


def _stream(stream):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


@dataclass
class Shape:
    dtype: int
    n_layers: int
    n_heads: int
    n_tokens: int
    head_dim: int
    values_per_chunk: int = 65536
    n_sink: int = 4
    n_recent: int = 128
    block_tokens: int = 64
    chunk_tokens: int = 512
    max_bits: int = 8
    rope_theta: float = 1e4
    avg_bits: float = 2.0
    range_mode: int = 0  # RANGES_BLOCK or RANGES_KIVI

    @property
    def n_slices(self) -> int:
        return self.n_layers * 2 * self.n_heads

    @classmethod
    def from_workload(cls, w) -> "Shape":
        return cls(w.dtype, w.n_layers, w.n_heads, w.n_tokens, w.head_dim, w.values_per_chunk,
                   w.n_sink, w.n_recent, w.block_tokens, w.chunk_tokens, w.max_bits, w.theta,
                   w.avg_bits)

    def desc(self, bases=None, eigvals=None, widths=None) -> PlanDesc:
        return PlanDesc(ABI_VERSION, self.dtype, self.n_layers, self.n_heads, self.n_tokens,
                        self.head_dim, self.values_per_chunk, self.n_sink, self.n_recent,
                        self.block_tokens, self.chunk_tokens, self.max_bits, self.rope_theta,
                        self.avg_bits, _np_ptr(bases), _np_ptr(eigvals), _np_ptr(widths), self.range_mode, 0)


class Plan:
    """A kvc plan on the current CUDA device. Lossless-only when bases is None."""

    def __init__(self, shape: Shape, bases=None, eigvals=None, widths=None):
        self.shape = shape
        b = None if bases is None else np.ascontiguousarray(bases, dtype=np.float32)
        e = None if eigvals is None else np.ascontiguousarray(eigvals, dtype=np.float64)
        w = None if widths is None else np.ascontiguousarray(widths, dtype=np.uint8)
        desc = shape.desc(b, e, w)
        h = ctypes.c_void_p()
        _check(_lib.kvc_plan(ctypes.byref(desc), ctypes.byref(h)), "kvc_plan")
        self._h = h
        # Held by the object: at interpreter exit the module's globals may be
        # cleared before the last plan is collected.
        self._destroy = _lib.kvc_plan_destroy
        self.has_transform = b is not None

    def __del__(self):
        h = getattr(self, "_h", None)
        destroy = getattr(self, "_destroy", None)
        if h is not None and h.value and destroy is not None:
            destroy(h)
            self._h = None

    @property
    def handle(self):
        return self._h

    @property
    def crc(self) -> int:
        return _lib.kvc_plan_crc(self._h)

    def widths(self) -> np.ndarray:
        s = self.shape
        out = np.zeros((s.n_slices, s.head_dim), np.uint8)
        _check(_lib.kvc_plan_widths(self._h, out.ctypes.data, out.size), "kvc_plan_widths")
        return out

    def max_encoded_bytes(self, path: int, n_slices: int) -> int:
        return _lib.kvc_max_encoded_bytes(self._h, path, n_slices)

    def workspace_bytes(self, path: int, decode: bool, n_slices: int) -> int:
        return _lib.kvc_workspace_bytes(self._h, path, int(decode), n_slices)


class Codec:
    """Owns output, workspace and result buffers for repeated calls of one size."""

    def __init__(self, plan: Plan, path: int, n_slices: int, device=None):
        import torch
        self.plan, self.path, self.n_slices = plan, path, n_slices
        dev = torch.device("cuda") if device is None else device
        s = plan.shape
        self.cap = plan.max_encoded_bytes(path, n_slices)
        self.out_elems = n_slices * s.n_tokens * s.head_dim
        vt = torch.int32 if s.dtype == DTYPE_F32 else torch.int16  # one element per value
        self.container = torch.empty(max(self.cap, 16), dtype=torch.uint8, device=dev)
        self.ws_enc = torch.empty(max(plan.workspace_bytes(path, False, n_slices), 256),
                                  dtype=torch.uint8, device=dev)
        self.ws_dec = torch.empty(max(plan.workspace_bytes(path, True, n_slices), 256),
                                  dtype=torch.uint8, device=dev)
        self.res = torch.zeros(4, dtype=torch.int64, device=dev)  # kvc_result (16 bytes) x 2
        self.decoded = torch.empty(max(self.out_elems, 8), dtype=vt, device=dev)

    def encode(self, src, first_slice: int = 0, stream=None, res=None):
        fn = _lib.kvc_encode_lossless if self.path == LOSSLESS else _lib.kvc_encode_transform
        r = self.res[0:2] if res is None else res
        st = fn(self.plan.handle, first_slice, self.n_slices, _dptr(src), _dptr(self.container),
                self.container.numel(), _dptr(self.ws_enc), self.ws_enc.numel(), _dptr(r),
                _stream(stream))
        _check(st, "encode")
        return r

    def decode(self, container, nbytes: int, out=None, stream=None, res=None):
        fn = _lib.kvc_decode_lossless if self.path == LOSSLESS else _lib.kvc_decode_transform
        r = self.res[2:4] if res is None else res
        dst = self.decoded if out is None else out
        cap = dst.numel() * dst.element_size()
        st = fn(self.plan.handle, _dptr(container), nbytes, _dptr(dst), cap, _dptr(self.ws_dec),
                self.ws_dec.numel(), _dptr(r), _stream(stream))
        _check(st, "decode")
        return r


def batch_workspace_bytes(plan: Plan, path: int, decode: bool, n_frames: int,
                          max_slices_per_frame: int) -> int:
    return _lib.kvc_batch_workspace_bytes(plan.handle, path, int(decode), n_frames,
                                          max_slices_per_frame)


def _frames(items):
    arr = (Frame * max(len(items), 1))()
    for i, it in enumerate(items):
        arr[i] = Frame(*it)
    return arr


def encode_batch(plan: Plan, path: int, frames, ws, stream=None):
    """frames: sequence of (first_slice, n_slices, src_tensor, dst_tensor, res_tensor)."""
    items = [(fs, ns, src.data_ptr() if src is not None and src.numel() else None, 0,
              dst.data_ptr(), dst.numel() * dst.element_size(), res.data_ptr())
             for fs, ns, src, dst, res in frames]
    _check(_lib.kvc_encode_batch(plan.handle, path, _frames(items), len(items), _dptr(ws),
                                 ws.numel() * ws.element_size(), _stream(stream)),
           "kvc_encode_batch")


def decode_batch(plan: Plan, path: int, frames, ws, max_slices_per_frame: int = 0, stream=None):
    """frames: sequence of (src_tensor, src_bytes, dst_tensor, res_tensor)."""
    items = [(0, 0, src.data_ptr(), nbytes, dst.data_ptr(), dst.numel() * dst.element_size(),
              res.data_ptr()) for src, nbytes, dst, res in frames]
    _check(_lib.kvc_decode_batch(plan.handle, path, _frames(items), len(items),
                                 max_slices_per_frame, _dptr(ws), ws.numel() * ws.element_size(),
                                 _stream(stream)), "kvc_decode_batch")


def stream_buffer_bytes(plan: Plan, path: int, frame_slices: int) -> int:
    return _lib.kvc_stream_buffer_bytes(plan.handle, path, frame_slices)


def _nbytes(t):
    return t.numel() * t.element_size()


def stream_encode_host(plan: Plan, path: int, first_slice: int, n_slices: int, frame_slices: int,
                       h_src, h_dst, h_frame_bytes, h_results, d_buf, stream=None):
    """kvc_stream_encode_host (blocking): h_src / h_dst host tensors (pinned for
    overlap), h_frame_bytes host int64 [n_frames], h_results host int64
    [n_frames, 2] (kvc_result), d_buf device uint8 of stream_buffer_bytes."""
    _check(_lib.kvc_stream_encode_host(plan.handle, path, first_slice, n_slices, frame_slices, _dptr(h_src),
                                       _dptr(h_dst), _nbytes(h_dst), _dptr(h_frame_bytes), _dptr(h_results),
                                       _dptr(d_buf), _nbytes(d_buf), _stream(stream)), "kvc_stream_encode_host")


def stream_decode_host(plan: Plan, path: int, n_slices: int, frame_slices: int, h_src, h_frame_bytes, h_dst,
                       h_results, d_buf, stream=None):
    """kvc_stream_decode_host (blocking); arguments as for stream_encode_host."""
    _check(_lib.kvc_stream_decode_host(plan.handle, path, n_slices, frame_slices, _dptr(h_src),
                                       _dptr(h_frame_bytes), _dptr(h_dst), _nbytes(h_dst), _dptr(h_results),
                                       _dptr(d_buf), _nbytes(d_buf), _stream(stream)), "kvc_stream_decode_host")


def read_result(res) -> tuple[int, int]:
    """(status, bytes) from a device kvc_result (synchronises with its stream)."""
    v = res.cpu().numpy()
    return int(v[0] & 0xFFFFFFFF), int(v[1])


def calibrate_pca(shape: Shape, calib: np.ndarray, n_threads: int = 0):
    """Host PCA per slice: bases [S][D][D] fp32 and eigenvalues [S][D]."""
    c = np.ascontiguousarray(calib, dtype=np.uint16)
    S, n_calib, D = c.shape
    bases = np.zeros((S, D, D), np.float32)
    lam = np.zeros((S, D), np.float64)
    desc = shape.desc()
    _check(_lib.kvc_calibrate_pca(ctypes.byref(desc), c.ctypes.data, n_calib, bases.ctypes.data,
                                  lam.ctypes.data, n_threads), "kvc_calibrate_pca")
    return bases, lam


BASIS_PCA, BASIS_HADAMARD, BASIS_DCT = 0, 1, 2


def fixed_basis(kind: int, D: int) -> np.ndarray:
    """Calibration-free basis [D][D] fp32 (Hadamard or DCT-II)."""
    q = np.zeros((D, D), np.float32)
    _check(_lib.kvc_fixed_basis(kind, D, q.ctypes.data), "kvc_fixed_basis")
    return q


def calibrate_basis(shape: Shape, kind: int, calib: np.ndarray, n_threads: int = 0):
    """Bases [S][D][D] and component variances [S][D] for a basis kind."""
    c = np.ascontiguousarray(calib, dtype=np.uint16)
    S, n_calib, D = c.shape
    bases = np.zeros((S, D, D), np.float32)
    lam = np.zeros((S, D), np.float64)
    desc = shape.desc()
    _check(_lib.kvc_calibrate_basis(ctypes.byref(desc), kind, c.ctypes.data, n_calib, bases.ctypes.data,
                                    lam.ctypes.data, n_threads), "kvc_calibrate_basis")
    return bases, lam


def allocate_bits(eigvals: np.ndarray, avg_bits: float, max_bits: int = 8) -> np.ndarray:
    lam = np.ascontiguousarray(eigvals, dtype=np.float64).ravel()
    w = np.zeros(lam.size, np.uint8)
    _check(_lib.kvc_allocate_bits(lam.ctypes.data, lam.size, avg_bits, max_bits, w.ctypes.data),
           "kvc_allocate_bits")
    return w


def profile_begin():
    _check(_lib.kvc_profile_begin(), "kvc_profile_begin")


def profile_end() -> dict:
    """{kernel name: (launches, total ms)} for the launches since profile_begin()."""
    arr = (KernelTime * 64)()
    n = ctypes.c_int(0)
    _check(_lib.kvc_profile_end(arr, 64, ctypes.byref(n)), "kvc_profile_end")
    return {arr[i].name.decode(): (int(arr[i].launches), float(arr[i].total_ms))
            for i in range(n.value)}


def stage_crc32(src, n: int, out, stream=None):
    _check(_lib.kvc_stage_crc32(_dptr(src), n, _dptr(out), _stream(stream)), "kvc_stage_crc32")


def stage_stream_encode(sym, n: int, out, scratch, res, stream=None):
    _check(_lib.kvc_stage_stream_encode(_dptr(sym), n, _dptr(out), _dptr(scratch), _dptr(res),
                                        _stream(stream)), "kvc_stage_stream_encode")


def stage_stream_encode_noalloc(sym, n: int, out, res, stream=None):
    """kvc_stage_stream_encode with the library's own fixed scratch (n <= 65536);
    allocates nothing. Overlapping calls on one device share that scratch."""
    _check(_lib.kvc_stage_stream_encode_noalloc(_dptr(sym), n, _dptr(out), _dptr(res),
                                                _stream(stream)), "kvc_stage_stream_encode_noalloc")


def stage_stream_decode(rec, rec_bytes: int, n: int, sym, res, stream=None):
    _check(_lib.kvc_stage_stream_decode(_dptr(rec), rec_bytes, n, _dptr(sym), _dptr(res),
                                        _stream(stream)), "kvc_stage_stream_decode")
