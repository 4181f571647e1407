"""Seeded synthetic KV-cache inputs, shared by the oracle tests and the GPU codec.

This module only makes inputs (see kvgen.c for the generator's definition); it
holds none of the codec's arithmetic. The workload table below gives the shapes
the codec is exercised on; they stand in for the exported caches the pages
measure (GPT-2-sized fp16 KV, a 50,331,648-byte live-migration block, a
Llama-8B-shaped and a Qwen3-32B-shaped cache), which are not available here.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kvgen.c")
_LIB = os.path.join(_HERE, "libkvgen.so")
_lib = None

BF16, FP16, F32 = 1, 2, 3


def compile_command() -> list[str]:
    return ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread", "-o", _LIB, _SRC, "-lm"]


def build() -> str:
    if not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(compile_command())
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        u32, u64, i32, dbl, vp = (ctypes.c_uint32, ctypes.c_uint64, ctypes.c_int,
                                  ctypes.c_double, ctypes.c_void_p)
        lib.kvgen_slices.argtypes = [u64, u32, u32, u32, u32, i32, dbl, dbl, u32, u32, i32, vp]
        lib.kvgen_slices.restype = i32
        lib.kvgen_calibration.argtypes = [u64, u32, u32, u32, u32, i32, dbl, dbl, i32, vp]
        lib.kvgen_calibration.restype = i32
        lib.kvgen_random_bytes.argtypes = [u64, u64, vp]
        lib.kvgen_random_bytes.restype = None
        _lib = lib
    return _lib


@dataclass(frozen=True)
class Workload:
    name: str
    path: str            # "lossless" or "transform"
    dtype: int           # BF16, FP16 or F32
    n_layers: int
    n_heads: int
    n_tokens: int
    head_dim: int
    rho: float
    theta: float
    seed: int = 0
    values_per_chunk: int = 65536
    n_sink: int = 4
    n_recent: int = 128
    block_tokens: int = 64
    chunk_tokens: int = 512
    avg_bits: float = 2.0
    max_bits: int = 8
    slices_per_frame: int = 0   # 0: the whole cache is one container
    control_bytes: int = 0      # uniform random control block (lossless only)

    @property
    def n_slices(self) -> int:
        return self.n_layers * 2 * self.n_heads

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == F32 else 2

    @property
    def raw_bytes(self) -> int:
        return self.n_slices * self.n_tokens * self.head_dim * self.elem_bytes


WORKLOADS = {
    # 1 layer K+V, 8 heads x 512 tokens x 128, bf16, rho 0.9
    "lossless-1x8x512x128-bf16": Workload(
        "lossless-1x8x512x128-bf16", "lossless", BF16, 1, 8, 512, 128, 0.9, 1e4),
    # GPT-2-small-shaped KV: 12 layers x 12 heads x 1024 x 64, fp16, rho 0.8,
    # plus a 4 MiB uniform-random control block
    "lossless-12x12x1024x64-fp16": Workload(
        "lossless-12x12x1024x64-fp16", "lossless", FP16, 12, 12, 1024, 64, 0.8, 1e4,
        control_bytes=4 << 20),
    # the GPT-2-small shape at fp32 (QATQ and AT-1 code f32 tensors too)
    "lossless-12x12x1024x64-f32": Workload(
        "lossless-12x12x1024x64-f32", "lossless", F32, 12, 12, 1024, 64, 0.8, 1e4),
    # live-migration block of 50,331,648 bytes: 8 layers x 8 heads x 1536 x 128
    "lossless-8x8x1536x128-bf16": Workload(
        "lossless-8x8x1536x128-bf16", "lossless", BF16, 8, 8, 1536, 128, 0.95, 1e4),
    # the same generator at 3072 tokens (100,663,296 bytes)
    "lossless-8x8x3072x128-bf16": Workload(
        "lossless-8x8x3072x128-bf16", "lossless", BF16, 8, 8, 3072, 128, 0.95, 1e4),
    # Llama-8B-shaped: 32 layers x 8 heads x 8192 x 128, transform at 2.0 bits
    "transform-32x8x8192x128-bf16": Workload(
        "transform-32x8x8192x128-bf16", "transform", BF16, 32, 8, 8192, 128, 0.9, 5e5,
        avg_bits=2.0),
    # Qwen3-32B-shaped at 32k tokens: 64 layers x 8 heads x 32768 x 128, 64 MiB frames
    "lossless-64x8x32768x128-bf16": Workload(
        "lossless-64x8x32768x128-bf16", "lossless", BF16, 64, 8, 32768, 128, 0.9, 5e5,
        slices_per_frame=8),
    "transform-64x8x32768x128-bf16": Workload(
        "transform-64x8x32768x128-bf16", "transform", BF16, 64, 8, 32768, 128, 0.9, 5e5,
        avg_bits=1.6, slices_per_frame=8),
}


def slices(w: Workload, first: int = 0, n: int | None = None, out=None, n_threads: int = 0):
    """Slices [first, first+n) as [n][T][D] value bits (uint16, or uint32 for F32);
    out may be a preallocated (e.g. pinned) buffer with room for n*T*D values
    (numpy or ctypes address)."""
    lib = _load()
    n = w.n_slices - first if n is None else n
    count = n * w.n_tokens * w.head_dim
    if out is None:
        arr = np.empty(count, dtype=np.uint32 if w.dtype == F32 else np.uint16)
        ptr = arr.ctypes.data
    elif isinstance(out, int):
        arr, ptr = None, out
    else:
        arr, ptr = out, out.ctypes.data
    rc = lib.kvgen_slices(w.seed, w.n_layers, w.n_heads, w.n_tokens, w.head_dim, w.dtype,
                          w.rho, w.theta, first, n, n_threads, ptr)
    if rc != 0:
        raise ValueError("kvgen_slices: bad shape")
    return None if arr is None else arr[:count].reshape(n, w.n_tokens, w.head_dim)


def calibration(w: Workload, n_calib: int = 1024, n_threads: int = 0) -> np.ndarray:
    """Calibration draw [L*2*H][n_calib][D]: same channel parameters, separate noise."""
    lib = _load()
    arr = np.empty(w.n_slices * n_calib * w.head_dim, dtype=np.uint16)
    rc = lib.kvgen_calibration(w.seed, w.n_layers, w.n_heads, n_calib, w.head_dim, w.dtype,
                               w.rho, w.theta, n_threads, arr.ctypes.data)
    if rc != 0:
        raise ValueError("kvgen_calibration: bad shape")
    return arr.reshape(w.n_slices, n_calib, w.head_dim)


def random_bytes(n: int, seed: int = 0) -> np.ndarray:
    lib = _load()
    arr = np.empty(n, dtype=np.uint8)
    lib.kvgen_random_bytes(seed, n, arr.ctypes.data)
    return arr
