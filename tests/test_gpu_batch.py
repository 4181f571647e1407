"""Batches of frames (independent containers) through one call: every frame's
container must equal the oracle's and decode back exactly; a damaged frame
fails alone with the oracle's status."""
import dataclasses

import numpy as np
import pytest
import torch

import kvgen
import oracle
import transform_codec_b200 as kvc
from kvc_gpu import dev_u16, rel_rms

pytestmark = pytest.mark.gpu


def _run_batch(plan, path, x_frames, firsts, oplan, encoder):
    n = len(x_frames)
    caps = [plan.max_encoded_bytes(path, xf.shape[0]) for xf in x_frames]
    conts = [torch.zeros(max(c, 16), dtype=torch.uint8, device="cuda") for c in caps]
    res = torch.zeros(n, 2, dtype=torch.int64, device="cuda")
    srcs = [dev_u16(xf) if xf.size else torch.empty(0, dtype=torch.int16, device="cuda")
            for xf in x_frames]
    ms = max(xf.shape[0] for xf in x_frames)
    ws = torch.empty(kvc.batch_workspace_bytes(plan, path, False, n, ms), dtype=torch.uint8,
                     device="cuda")
    kvc.encode_batch(plan, path, [(firsts[i], x_frames[i].shape[0], srcs[i], conts[i], res[i])
                                  for i in range(n)], ws)
    r = res.cpu().numpy()
    assert np.all((r[:, 0] & 0xFFFFFFFF) == 0)
    got = [conts[i][: r[i, 1]].cpu().numpy().tobytes() for i in range(n)]
    want = [encoder(oplan, x_frames[i], first_slice=firsts[i]) for i in range(n)]
    return got, want, ms


def _decode_batch(plan, path, blobs, shapes, ms):
    n = len(blobs)
    s = plan.shape
    bufs = [torch.zeros(max(len(c), 16), dtype=torch.uint8, device="cuda") for c in blobs]
    for b_, c in zip(bufs, blobs):
        if c:
            b_[: len(c)] = torch.frombuffer(bytearray(c), dtype=torch.uint8).cuda()
    outs = [torch.zeros(max(k * s.n_tokens * s.head_dim, 8), dtype=torch.int16, device="cuda")
            for k in shapes]
    res = torch.zeros(n, 2, dtype=torch.int64, device="cuda")
    ws = torch.empty(kvc.batch_workspace_bytes(plan, path, True, n, ms), dtype=torch.uint8,
                     device="cuda")
    kvc.decode_batch(plan, path, [(bufs[i], len(blobs[i]), outs[i], res[i]) for i in range(n)],
                     ws, ms)
    r = res.cpu().numpy()
    ys = [outs[i][: shapes[i] * s.n_tokens * s.head_dim].cpu().numpy().view(np.uint16)
          .reshape(shapes[i], s.n_tokens, s.head_dim) for i in range(n)]
    return (r[:, 0] & 0xFFFFFFFF).tolist(), ys


def test_lossless_batch_parity_and_damage():
    w = dataclasses.replace(kvgen.WORKLOADS["lossless-1x8x512x128-bf16"], n_layers=2,
                            n_tokens=1100)
    plan = kvc.Plan(kvc.Shape.from_workload(w))
    oplan = oracle.Plan.from_workload(w)
    firsts = [0, 3, 16, 31, 5, 7]
    counts = [3, 5, 1, 1, 0, 9]
    xs = [kvgen.slices(w, first=f, n=c) for f, c in zip(firsts, counts)]
    got, want, ms = _run_batch(plan, kvc.LOSSLESS, xs, firsts, oplan, oracle.encode_lossless)
    assert got == want
    bad = bytearray(want[1])
    bad[len(bad) // 2] ^= 0x40
    blobs = list(want)
    blobs[1] = bytes(bad)
    st, ys = _decode_batch(plan, kvc.LOSSLESS, blobs, counts, ms)
    want_bad, _ = oracle.decode_lossless(oplan, blobs[1])
    assert st[1] == want_bad != 0
    for i in range(len(xs)):
        if i != 1:
            assert st[i] == 0 and np.array_equal(ys[i], xs[i])


def test_transform_batch_parity():
    w = dataclasses.replace(kvgen.WORKLOADS["transform-32x8x8192x128-bf16"], n_layers=1,
                            n_heads=2, n_tokens=1024)
    cal = kvgen.calibration(w)
    pcs = [oracle.pca(cal[s], (s // w.n_heads) % 2 == 0, w.theta) for s in range(w.n_slices)]
    bases = np.stack([p[0] for p in pcs])
    lam = np.stack([p[1] for p in pcs])
    widths = oracle.allocate(lam, w.avg_bits, w.max_bits).reshape(lam.shape)
    plan = kvc.Plan(kvc.Shape.from_workload(w), bases=bases, widths=widths)
    oplan = oracle.Plan.from_workload(w, bases=bases, widths=widths)
    firsts, counts = [0, 1, 2], [1, 3, 2]
    xs = [kvgen.slices(w, first=f, n=c) for f, c in zip(firsts, counts)]
    got, want, ms = _run_batch(plan, kvc.TRANSFORM, xs, firsts, oplan, oracle.encode_transform)
    for i in range(len(xs)):
        st, codes, _ = oracle.container_codes(oplan, got[i], counts[i])
        assert st == oracle.OK
        for k in range(counts[i]):
            oc, _, _ = oracle.transform_slice_codes(oplan, firsts[i] + k, xs[i][k])
            assert np.mean(codes[k] == oc) >= 0.99999
    st, ys = _decode_batch(plan, kvc.TRANSFORM, got, counts, ms)
    assert st == [0, 0, 0]
    for i in range(len(xs)):
        ost, yo = oracle.decode_transform(oplan, want[i], n_slices_cap=counts[i])
        assert ost == oracle.OK and rel_rms(yo, ys[i]) <= 1e-3
