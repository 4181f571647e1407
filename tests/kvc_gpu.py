"""Helpers for the GPU parity tests: run the library through its Python binding
on numpy inputs and bring containers and outputs back to the host."""
import numpy as np
import torch

import transform_codec_b200 as kvc


def dev_u16(x: np.ndarray) -> torch.Tensor:
    """Value bits on the device: int16 elements, or int32 for 4-byte values."""
    x = np.ascontiguousarray(x)
    return torch.from_numpy(x.view(np.int32 if x.itemsize == 4 else np.int16).ravel()).cuda()


def encode(plan, path, x, first_slice=0):
    """Container bytes and status of the GPU encode of x [n][T][D] (uint16)."""
    n = x.shape[0]
    codec = kvc.Codec(plan, path, n)
    src = dev_u16(x) if x.size else torch.empty(0, dtype=torch.int16, device="cuda")
    res = codec.encode(src, first_slice)
    st, nbytes = kvc.read_result(res)
    data = codec.container[:nbytes].cpu().numpy().tobytes() if st == kvc.OK else b""
    return st, data


def decode(plan, path, container: bytes, n_slices_cap: int):
    """Status and decoded [n][T][D] value bits (uint16, or uint32 for f32) of the
    GPU decode of a container."""
    s = plan.shape
    wide = s.dtype == kvc.F32
    codec = kvc.Codec(plan, path, max(n_slices_cap, 1))
    buf = torch.zeros(max(len(container), 16), dtype=torch.uint8, device="cuda")
    if container:
        buf[: len(container)] = torch.frombuffer(bytearray(container), dtype=torch.uint8).cuda()
    out = torch.zeros(max(n_slices_cap * s.n_tokens * s.head_dim, 8),
                      dtype=torch.int32 if wide else torch.int16, device="cuda")
    res = codec.decode(buf, len(container), out=out[: n_slices_cap * s.n_tokens * s.head_dim]
                       if n_slices_cap else out[:0])
    st, nbytes = kvc.read_result(res)
    n = nbytes // ((4 if wide else 2) * s.n_tokens * s.head_dim)
    y = out[: n * s.n_tokens * s.head_dim].cpu().numpy().view(np.uint32 if wide else np.uint16)
    return st, y.reshape(n, s.n_tokens, s.head_dim)


def f32(h):
    return (np.asarray(h, np.uint32) << 16).view(np.float32)


def rel_rms(a, b):
    a = f32(a).astype(np.float64)
    b = f32(b).astype(np.float64)
    return float(np.sqrt(((a - b) ** 2).sum() / max((a ** 2).sum(), 1e-300)))
