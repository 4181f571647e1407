"""The codec's device waits (the transform encoder's and decoder's waits for
their own tensor-core MMAs) are bounded: when one gives up, the frame reports
KVC_ERR_TIMEOUT in its device result instead of spinning, and the context
stays usable.

The waits are made to run out on purpose with the library's "wait0" test
build (the first completion wait gives up without polling; the drain wait that
follows keeps its long bound, so the MMAs have finished before the block frees
their tensor memory). Nothing faults: the kernel only takes its error path.
The build runs in a child process, since a process loads one libkvc."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import dataclasses, sys
import numpy as np
import torch
sys.path.insert(0, ROOT)
sys.path.insert(0, ROOT + "/tests")
import kvgen, oracle
import transform_codec_b200 as kvc
from kvc_gpu import decode, encode
assert kvc.LIB_PATH.endswith("libkvc_wait0.so"), kvc.LIB_PATH
w = dataclasses.replace(kvgen.WORKLOADS["transform-32x8x8192x128-bf16"], n_layers=1,
                        n_heads=1, n_tokens=900)
cal = kvgen.calibration(w)
pcs = [oracle.pca(cal[s], s == 0, w.theta) for s in range(w.n_slices)]
bases = np.stack([p[0] for p in pcs])
widths = oracle.allocate(np.stack([p[1] for p in pcs]), w.avg_bits, w.max_bits).reshape(w.n_slices, 128)
x = kvgen.slices(w)
plan = kvc.Plan(kvc.Shape.from_workload(w), bases=bases, widths=widths)
# the encoder's projection waits for its MMAs too: the frame reports the timeout
for _ in range(2):
    st, _ = encode(plan, kvc.TRANSFORM, x)
    assert st == kvc.ERR_TIMEOUT, kvc.status_string(st)
# the decoder's tensor stage, on the oracle's container
oplan = oracle.Plan.from_workload(w, bases=bases, widths=widths)
c = oracle.encode_transform(oplan, x)
for _ in range(2):
    st, _ = decode(plan, kvc.TRANSFORM, c, w.n_slices)
    assert st == kvc.ERR_TIMEOUT, kvc.status_string(st)
# the context is still usable: a lossless round trip after the timeouts
wl = kvgen.WORKLOADS["lossless-1x8x512x128-bf16"]
xl = kvgen.slices(wl)
lplan = kvc.Plan(kvc.Shape.from_workload(wl))
st, cl = encode(lplan, kvc.LOSSLESS, xl)
assert st == kvc.OK
st, yl = decode(lplan, kvc.LOSSLESS, cl, wl.n_slices)
assert st == kvc.OK and np.array_equal(yl, xl)
torch.cuda.synchronize()
print("timeout-child: ok")
"""


def test_mma_wait_timeout_reports_status():
    lib = os.path.join(ROOT, "transform_codec_b200", "libkvc_wait0.so")
    assert os.path.exists(lib), "the wait0 test build is missing (build.build_all())"
    env = dict(os.environ, KVC_BUILD_VARIANT="wait0")
    r = subprocess.run([sys.executable, "-c", f"ROOT = {ROOT!r}\n" + CHILD], env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    assert "timeout-child: ok" in r.stdout
