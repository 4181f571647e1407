"""Host-streamed coding (QATQ "Measured evidence": raw blocks streamed through
the codec) against the oracle: kvc_stream_encode_host codes a slice range from
host memory frame by frame, each frame a container equal to the oracle's for
its slices; kvc_stream_decode_host restores them, and a damaged frame is
refused on its own."""
import dataclasses

import numpy as np
import pytest
import torch

import kvgen
import oracle
import transform_codec_b200 as kvc
from kvc_gpu import rel_rms

pytestmark = pytest.mark.gpu


def _host(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.uint8).ravel().copy()).pin_memory()


def _round_trip(plan, path, x, fs, want_frame):
    n = x.shape[0]
    nf = -(-n // fs)
    src = _host(x)
    cap = sum(plan.max_encoded_bytes(path, min(fs, n - f * fs)) for f in range(nf))
    dst = torch.zeros(cap, dtype=torch.uint8).pin_memory()
    fb = torch.zeros(nf, dtype=torch.int64)
    res = torch.zeros(nf, 2, dtype=torch.int64).pin_memory()
    buf = torch.empty(kvc.stream_buffer_bytes(plan, path, fs), dtype=torch.uint8, device="cuda")
    kvc.stream_encode_host(plan, path, 0, n, fs, src, dst, fb, res, buf)
    assert not (res[:, 0] & 0xFFFFFFFF).any()
    sizes = fb.tolist()
    cont = dst.numpy().tobytes()
    off = 0
    for f in range(nf):
        s0, ns = f * fs, min(fs, n - f * fs)
        assert sizes[f] == res[f, 1].item()
        assert cont[off:off + sizes[f]] == want_frame(s0, ns), f
        off += sizes[f]
    back = torch.zeros_like(src)
    res2 = torch.zeros(nf, 2, dtype=torch.int64).pin_memory()
    kvc.stream_decode_host(plan, path, n, fs, dst, fb, back, res2, buf)
    assert not (res2[:, 0] & 0xFFFFFFFF).any()
    return back.numpy(), src.numpy(), dst, fb, buf


@pytest.mark.parametrize("fs", [1, 3, 16])
def test_stream_lossless_frames_equal_oracle(fs):
    w = kvgen.WORKLOADS["lossless-1x8x512x128-bf16"]
    x = kvgen.slices(w)
    plan = kvc.Plan(kvc.Shape.from_workload(w))
    op = oracle.Plan.from_workload(w)
    back, src, _, _, _ = _round_trip(plan, kvc.LOSSLESS, x, fs,
                                     lambda s0, ns: oracle.encode_lossless(op, x[s0:s0 + ns], first_slice=s0))
    assert np.array_equal(back, src)


def test_stream_f32_and_damaged_frame():
    w = dataclasses.replace(kvgen.WORKLOADS["lossless-12x12x1024x64-f32"], n_layers=1, n_heads=3)
    x = kvgen.slices(w)
    plan = kvc.Plan(kvc.Shape.from_workload(w))
    op = oracle.Plan.from_workload(w)
    back, src, dst, fb, buf = _round_trip(plan, kvc.LOSSLESS, x, 4,
                                          lambda s0, ns: oracle.encode_lossless(op, x[s0:s0 + ns], first_slice=s0))
    assert np.array_equal(back, src)
    sizes = fb.tolist()
    bad = dst.clone().pin_memory()
    bad[sizes[0] + 200] ^= 0x5A  # inside frame 1
    out = torch.zeros_like(torch.from_numpy(src)).pin_memory()
    res = torch.zeros(len(sizes), 2, dtype=torch.int64).pin_memory()
    kvc.stream_decode_host(plan, kvc.LOSSLESS, x.shape[0], 4, bad, fb, out, res, buf)
    st = (res[:, 0] & 0xFFFFFFFF).tolist()
    assert st[1] == kvc.ERR_CORRUPT and st[0] == kvc.OK and all(s == kvc.OK for s in st[2:])
    per = 4 * w.n_tokens * w.head_dim * 4
    assert np.array_equal(out.numpy()[:per], src[:per])
    assert np.array_equal(out.numpy()[2 * per:], src[2 * per:])


def test_stream_transform_frames_equal_oracle():
    base = dataclasses.replace(kvgen.WORKLOADS["transform-32x8x8192x128-bf16"], n_layers=1, n_heads=2)
    w = dataclasses.replace(base, n_tokens=640)
    cal = kvgen.calibration(w)
    pcs = [oracle.pca(cal[s], (s // w.n_heads) % 2 == 0, w.theta) for s in range(w.n_slices)]
    bases = np.stack([p[0] for p in pcs])
    lam = np.stack([p[1] for p in pcs])
    widths = oracle.allocate(lam, w.avg_bits, w.max_bits).reshape(lam.shape)
    plan = kvc.Plan(kvc.Shape.from_workload(w), bases=bases, widths=widths)
    op = oracle.Plan.from_workload(w, bases=bases, widths=widths)
    x = kvgen.slices(w)
    back, src, _, _, _ = _round_trip(plan, kvc.TRANSFORM, x, 3,
                                     lambda s0, ns: oracle.encode_transform(op, x[s0:s0 + ns], first_slice=s0))
    st, want = oracle.decode_transform(op, oracle.encode_transform(op, x))
    assert st == oracle.OK
    assert rel_rms(back.view(np.uint16), want.ravel()) <= 1e-3  # the transform path's reconstruction rule


def test_stream_capacity_errors():
    w = kvgen.WORKLOADS["lossless-1x8x512x128-bf16"]
    x = kvgen.slices(w)
    plan = kvc.Plan(kvc.Shape.from_workload(w))
    src = _host(x)
    buf = torch.empty(kvc.stream_buffer_bytes(plan, kvc.LOSSLESS, 4), dtype=torch.uint8, device="cuda")
    fb = torch.zeros(4, dtype=torch.int64)
    res = torch.zeros(4, 2, dtype=torch.int64).pin_memory()
    with pytest.raises(kvc.KvcError) as e:
        kvc.stream_encode_host(plan, kvc.LOSSLESS, 0, 16, 4, src, torch.zeros(1000, dtype=torch.uint8), fb, res, buf)
    assert e.value.status == kvc.ERR_CAPACITY
    with pytest.raises(kvc.KvcError) as e:
        kvc.stream_encode_host(plan, kvc.LOSSLESS, 0, 16, 4, src, torch.zeros(10 ** 7, dtype=torch.uint8), fb, res,
                               buf[:1024])
    assert e.value.status == kvc.ERR_CAPACITY
