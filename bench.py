#!/usr/bin/env python
"""Benchmark of the B200 KV-cache codec.

One step = the whole hot path over one synthetic Qwen3-32B-shaped cache at 32k
tokens (64 layers x 8 KV heads x 32768 tokens x 128, bf16 K+V, 8.59 GB),
streamed through HBM as 128 frames of 64 MiB (one layer's K or V each):
lossless encode, transform encode (1.6 bits per value), lossless decode and
transform decode of every frame. The metric is codec throughput in GB/s of raw
KV bytes (4 x raw bytes per step / step time), reported with per-operation
GB/s, compression ratios and the HBM roofline of the dominant kernel.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl kvc|reference]
For N > 1 launch with torch.distributed.run: every rank codes its own full
cache (weak scaling, no data-path collective); timing is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

WORKLOAD_L = "lossless-64x8x32768x128-bf16"
WORKLOAD_T = "transform-64x8x32768x128-bf16"
METRIC = "KV codec encode/decode GB/s (raw bytes) vs HBM roofline; compression ratio"

# Algorithmic work per step of each kernel with a roofline, given the step's
# raw bytes R, its container bytes C and its middle (transform-coded) values V:
# bytes for the lossless kernels (raw + container) and for the transform
# entropy stages (a code byte per middle value + the records), and 2 * 128
# flops per middle value for the transform contraction, counted once although
# the kernels split it into several tensor-core products (ten int8 byte-pair
# products in the encoder's projection, three bf16 hi/lo products in the
# decoder). The third field is the dtype whose tensor peak bounds the kernel.
KERNEL_WORK = {
    "lossless_encode": ("hbm", lambda R, C, V: R + C, None),
    "lossless_decode": ("hbm", lambda R, C, V: R + C, None),
    "transform_project": ("tensor", lambda R, C, V: 2 * 128 * V, "i8"),
    "transform_entropy": ("hbm", lambda R, C, V: V + C, None),          # codes in, records out
    "transform_decode_codes": ("hbm", lambda R, C, V: C + V, None),     # records in, codes out
    "transform_decode": ("tensor", lambda R, C, V: 2 * 128 * V, "bf16"),
}

# Dense tensor peak of a dtype as a multiple of the measured bf16 figure
# (nominal B200 ratios: int8 and fp8 run at twice the bf16 rate).
TENSOR_RATIO = {"bf16": 1.0, "i8": 2.0}

# DRAM bytes (read + write) per frame of 64 MiB, from one ncu capture of each
# kernel over 4 frames (larger than L2; the traffic of these kernels grows
# with the frames a launch covers). A kernel changed after its capture has no
# entry.
DRAM_BYTES_PER_FRAME = {
    "lossless_encode": (717.4e6 + 345.0e6) / 4,
    "transform_project": (328.1e6 + 106.2e6) / 4,
    "transform_side": (14.0e6 + 0.0e6) / 4,
    "transform_entropy": (126.2e6 + 21.8e6) / 4,
    "lossless_decode": (200.7e6 + 217.5e6) / 4,
    "transform_decode": (200.7e6 + 217.0e6) / 4,
}


def measured_peaks():
    """(HBM GB/s, sustained bf16 TFLOP/s, max SM MHz, source): the driver's
    measurements, else the pool's earlier figures."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return (float(p["hbm_gbs"]), float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                float(p.get("sm_max_mhz", 1965.0)), "measured")
    except (OSError, KeyError, ValueError):
        return 6650.0, 1400.0, 1965.0, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        self.f.flush()
        self.f.seek(0)
        rows = [r.split(",") for r in self.f.read().strip().splitlines() if r.strip()]
        os.unlink(self.f.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(r[1]) for r in rows if len(r) > 2 and r[1].strip().replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if len(r) > 2 and r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in rows:
            for i, n in enumerate(names):
                if len(r) > 5 + i and r[5 + i].strip().lower() == "active":
                    reasons.add(n)
        loaded = sorted(sm)[len(sm) // 2:] if sm else []
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(rows)}


def dist_setup(backend: str = "nccl"):
    """Rank, world and local rank from the launcher's environment; for more than
    one rank, the process group (NCCL on the GPUs; gloo runs the same code on
    the CPU). The only collectives are the timing reductions below."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(minutes=5))
    return world, rank, local


def max_over_ranks(values, world):
    """Element-wise maximum of each rank's values (device timings), on every rank."""
    if world == 1:
        return list(values)
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor(list(values), dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.cpu().tolist()


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ------------------------------------------------------------------ the codec
BASES = {"pca": 0, "hadamard": 1, "dct": 2}  # transform basis: calibrated PCA, or a fixed one


class Job:
    def __init__(self, w_l, w_t, n_frames=None, basis="pca"):
        import torch

        import kvgen
        import transform_codec_b200 as kvc
        self.kvc, self.torch = kvc, torch
        self.w_l, self.w_t = w_l, w_t
        self.spf = w_l.slices_per_frame
        self.frames = w_l.n_slices // self.spf if n_frames is None else n_frames
        self.T, self.D = w_l.n_tokens, w_l.head_dim
        self.frame_vals = self.spf * self.T * self.D
        self.frame_bytes = self.frame_vals * 2
        self.raw_bytes = self.frames * self.frame_bytes
        t0 = time.time()
        self.host = torch.empty(self.frames * self.frame_vals, dtype=torch.int16).pin_memory()
        kvgen.slices(w_l, 0, self.frames * self.spf, out=self.host.data_ptr())
        self.gen_s = time.time() - t0
        self.x = self.host.cuda()
        t0 = time.time()
        shape_t = kvc.Shape.from_workload(w_t)
        bases, lam = kvc.calibrate_basis(shape_t, BASES[basis], kvgen.calibration(w_t))
        self.plan_t = kvc.Plan(shape_t, bases=bases, eigvals=lam)
        self.plan_l = kvc.Plan(kvc.Shape.from_workload(w_l))
        self.bases = bases
        self.plan_s = time.time() - t0
        self.codec_l = kvc.Codec(self.plan_l, kvc.LOSSLESS, self.spf)
        self.codec_t = kvc.Codec(self.plan_t, kvc.TRANSFORM, self.spf)
        self.cap_l, self.cap_t = self.codec_l.cap, self.codec_t.cap
        self.cont_l = torch.empty(self.frames * self.cap_l, dtype=torch.uint8, device="cuda")
        self.cont_t = torch.empty(self.frames * self.cap_t, dtype=torch.uint8, device="cuda")
        self.out = torch.empty(self.frames * self.frame_vals, dtype=torch.int16, device="cuda")
        self.res = torch.zeros(self.frames * 4, 2, dtype=torch.int64, device="cuda")
        # batch workspaces: encode groups of up to 16 frames, decode up to 64 frames per launch
        grp = min(16, self.frames)
        self.ws_enc_l = torch.empty(kvc.batch_workspace_bytes(self.plan_l, kvc.LOSSLESS, False, grp,
                                                              self.spf), dtype=torch.uint8, device="cuda")
        self.ws_enc_t = torch.empty(kvc.batch_workspace_bytes(self.plan_t, kvc.TRANSFORM, False, grp,
                                                              self.spf), dtype=torch.uint8, device="cuda")
        self.ws_dec = torch.empty(max(kvc.batch_workspace_bytes(self.plan_l, kvc.LOSSLESS, True,
                                                                self.frames, self.spf),
                                      kvc.batch_workspace_bytes(self.plan_t, kvc.TRANSFORM, True,
                                                                self.frames, self.spf)),
                                  dtype=torch.uint8, device="cuda")
        self.sizes_l = self.sizes_t = None
        # middle values per frame (transform path)
        s_end = min(w_t.n_sink, self.T)
        r_start = max(s_end, self.T - w_t.n_recent)
        self.mid_vals = self.spf * (r_start - s_end) * self.D

    def _frame(self, t, f, cap):
        return t[f * cap:(f + 1) * cap]

    def encode_all(self, path):
        kvc = self.kvc
        cont, cap, base, plan, ws = ((self.cont_l, self.cap_l, 0, self.plan_l, self.ws_enc_l)
                                     if path == kvc.LOSSLESS else
                                     (self.cont_t, self.cap_t, self.frames, self.plan_t, self.ws_enc_t))
        frames = [(f * self.spf, self.spf, self.x[f * self.frame_vals:(f + 1) * self.frame_vals],
                   self._frame(cont, f, cap), self.res[base + f]) for f in range(self.frames)]
        kvc.encode_batch(plan, path, frames, ws)

    def read_sizes(self):
        r = self.res[: 2 * self.frames].cpu().numpy()
        st = (r[:, 0] & 0xFFFFFFFF).astype(np.int64)
        if np.any(st != 0):
            raise RuntimeError(f"encode failed: statuses {sorted(set(st.tolist()))}")
        self.sizes_l = r[: self.frames, 1].tolist()
        self.sizes_t = r[self.frames:, 1].tolist()

    def decode_all(self, path):
        kvc = self.kvc
        cont, cap, sizes, base, plan = (
            (self.cont_l, self.cap_l, self.sizes_l, 2 * self.frames, self.plan_l)
            if path == kvc.LOSSLESS else
            (self.cont_t, self.cap_t, self.sizes_t, 3 * self.frames, self.plan_t))
        frames = [(self._frame(cont, f, cap), sizes[f],
                   self.out[f * self.frame_vals:(f + 1) * self.frame_vals], self.res[base + f])
                  for f in range(self.frames)]
        kvc.decode_batch(plan, path, frames, self.ws_dec, self.spf)

    def step(self, ev):
        kvc = self.kvc
        ev[0].record()
        self.encode_all(kvc.LOSSLESS)
        ev[1].record()
        self.encode_all(kvc.TRANSFORM)
        ev[2].record()
        self.read_sizes()
        ev[3].record()
        self.decode_all(kvc.LOSSLESS)
        ev[4].record()
        self.decode_all(kvc.TRANSFORM)
        ev[5].record()

    def statuses_ok(self):
        """Every encode and decode of the last step reported OK."""
        st = self.res[:, 0].cpu().numpy() & 0xFFFFFFFF
        return bool(np.all(st == 0))

    def check(self, oracle_slices=(0, 13)):
        """Lossless decode restores the input exactly; transform decode of the
        whole cache is measured against the input (relative RMS); on sampled
        slices the transform codes are checked against the oracle's under the
        parity rule (at least 99.999% identical, any mismatch +-1 within 1e-4
        of a rounding boundary) and the reconstruction against the oracle's
        own encode and decode (relative RMS <= 1e-3); every call reported OK."""
        import struct

        import oracle
        torch, kvc = self.torch, self.kvc
        self.encode_all(kvc.LOSSLESS)
        self.encode_all(kvc.TRANSFORM)
        self.read_sizes()
        self.decode_all(kvc.LOSSLESS)
        torch.cuda.synchronize()
        exact = bool(torch.equal(self.out, self.x))
        self.decode_all(kvc.TRANSFORM)
        torch.cuda.synchronize()
        ok = exact and self.statuses_ok()
        num = den = 0.0
        for f in range(self.frames):  # relative RMS of the transform path against the input
            sl = slice(f * self.frame_vals, (f + 1) * self.frame_vals)
            a = self.x[sl].view(torch.bfloat16).double()
            b = self.out[sl].view(torch.bfloat16).double()
            num += float(((a - b) ** 2).sum())
            den += float((a ** 2).sum())
        T, D, spf = self.T, self.D, self.spf
        w = self.w_t
        s_end = min(w.n_sink, T)
        r_start = max(s_end, T - w.n_recent)
        rps = 1 + (r_start - s_end + w.chunk_tokens - 1) // w.chunk_tokens
        widths = self.plan_t.widths()
        op = oracle.Plan.from_workload(w, bases=self.bases, widths=widths)
        total = mism = 0
        near = True
        rr = 0.0
        for s in oracle_slices:
            f = s // spf
            if f >= self.frames:
                continue
            blob = self.cont_t[f * self.cap_t:f * self.cap_t + self.sizes_t[f]].cpu().numpy().tobytes()
            n_rec = struct.unpack_from("<I", blob, 36)[0]
            idx = [struct.unpack_from("<QII", blob, 64 + 16 * i) for i in range(n_rec)]
            xs = self.x[s * T * D:(s + 1) * T * D].cpu().numpy().view(np.uint16).reshape(T, D)
            ys = self.out[s * T * D:(s + 1) * T * D].cpu().numpy().view(np.uint16).reshape(T, D)
            oc, qp, _ = oracle.transform_slice_codes(op, s, xs)
            i0 = (s - f * spf) * rps
            coded = widths[s] > 0
            for c in range(rps - 1):
                t0 = s_end + c * w.chunk_tokens
                tcc = min(w.chunk_tokens, r_start - t0)
                off, ln, _ = idx[i0 + 1 + c]
                st, cc, _ = oracle.record_codes(op, s, blob[off:off + ln], tcc)
                ok = ok and st == oracle.OK
                a = cc[:, coded].astype(np.int32)
                b = oc[t0:t0 + tcc][:, coded].astype(np.int32)
                d = a != b
                total += a.size
                mism += int(d.sum())
                if d.any():
                    q = qp[t0:t0 + tcc][:, coded].astype(np.float64)[d]
                    near = near and bool(np.all(np.abs(a[d] - b[d]) == 1)) and \
                        bool(np.all(np.abs(q - (np.floor(q) + 0.5)) <= 1e-4))
            st, yo = oracle.decode_transform(op, oracle.encode_transform(op, xs[None], first_slice=s),
                                             n_slices_cap=1)
            ok = ok and st == oracle.OK
            fa = (yo[0].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
            fb = (ys.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
            rr = max(rr, float(np.sqrt(((fa - fb) ** 2).sum() / (fa ** 2).sum())))
        match = 1.0 - mism / max(total, 1)
        self.transform_check = {
            "rel_rms_vs_input": round(float(np.sqrt(num / den)), 6),
            "oracle_slices": [s for s in oracle_slices if s // spf < self.frames],
            "code_match_vs_oracle": round(match, 7), "mismatches_near_boundary": near,
            "rel_rms_vs_oracle": float(f"{rr:.3g}"),
        }
        return ok and match >= 0.99999 and near and rr <= 1e-3


def run_e2e(job, steps, warmup):
    """Host to host through the library's host-streamed calls, the calls a user
    with the cache in host memory makes: per step kvc_stream_encode_host for
    the lossless and the transform path (pinned H2D of each 64 MiB frame, its
    encode, D2H of its container) and kvc_stream_decode_host for both (H2D of
    each container, its decode, D2H of the restored frame). Each call overlaps
    its copies with the codec on three streams and returns when its last copy
    has landed. Device-timed with events around the four calls; every frame's
    status is checked and both restored caches are compared with the input
    after the timed steps."""
    torch, kvc = job.torch, job.kvc
    F, spf, n = job.frames, job.spf, job.frames * job.spf
    stream = torch.cuda.Stream()
    size_l, size_t = sum(job.sizes_l), sum(job.sizes_t)
    h_cont_l = torch.empty(size_l, dtype=torch.uint8).pin_memory()
    h_cont_t = torch.empty(size_t, dtype=torch.uint8).pin_memory()
    h_back = torch.empty_like(job.host).pin_memory()
    fb_l, fb_t = torch.zeros(F, dtype=torch.int64), torch.zeros(F, dtype=torch.int64)
    res = torch.zeros(4, F, 2, dtype=torch.int64).pin_memory()
    buf = torch.empty(max(kvc.stream_buffer_bytes(job.plan_l, kvc.LOSSLESS, spf),
                          kvc.stream_buffer_bytes(job.plan_t, kvc.TRANSFORM, spf)),
                      dtype=torch.uint8, device="cuda")
    exact = True

    def one_step(check):
        nonlocal exact
        kvc.stream_encode_host(job.plan_l, kvc.LOSSLESS, 0, n, spf, job.host, h_cont_l, fb_l, res[0], buf,
                               stream=stream)
        kvc.stream_encode_host(job.plan_t, kvc.TRANSFORM, 0, n, spf, job.host, h_cont_t, fb_t, res[1], buf,
                               stream=stream)
        kvc.stream_decode_host(job.plan_l, kvc.LOSSLESS, n, spf, h_cont_l, fb_l, h_back, res[2], buf,
                               stream=stream)
        if check:
            exact = exact and bool(torch.equal(h_back, job.host))
        kvc.stream_decode_host(job.plan_t, kvc.TRANSFORM, n, spf, h_cont_t, fb_t, h_back, res[3], buf,
                               stream=stream)

    for _ in range(warmup):
        one_step(False)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        one_step(False)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    st = res[:, :, 0].numpy() & 0xFFFFFFFF
    if st.any():
        raise RuntimeError(f"end-to-end step: codec status {set(st.ravel().tolist())}")
    one_step(True)  # untimed: the lossless restore is bit-exact
    if not exact or fb_l.tolist() != job.sizes_l or fb_t.tolist() != job.sizes_t:
        raise RuntimeError("end-to-end step: restored cache or container sizes differ")
    h2d = 2 * job.raw_bytes + size_l + size_t
    d2h = size_l + size_t + 2 * job.raw_bytes + res.numel() * 8
    return ms, h2d, d2h


# The oracle's bounded sample, the same in the CPU-baseline leg and the
# reference arm: one key slice and one value slice of the cache (layer 0, head
# 0), each coded on its own, all four operations, single-threaded.
ORACLE_SLICES = (0, 8)
ORACLE_SAMPLE = ("slices 0 (K) and 8 (V) of 32768x128 bf16 (16 MiB), each lossless and "
                 "transform encoded and decoded on its own, one thread")


def cpu_info():
    """(CPU model, logical CPUs) of this host."""
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.lower().startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return model, os.cpu_count()


def oracle_step(pl, pt, xs):
    """One pass of the oracle over the sample: per slice, lossless and transform
    encode and decode. xs: {slice index: [T][D] uint16}."""
    import oracle
    for s, x in xs.items():
        c = oracle.encode_lossless(pl, x[None], first_slice=s)
        st, y = oracle.decode_lossless(pl, c, n_slices_cap=1)
        ct = oracle.encode_transform(pt, x[None], first_slice=s)
        st2, _ = oracle.decode_transform(pt, ct, n_slices_cap=1)
        if st or st2 or not np.array_equal(y[0], x):
            raise RuntimeError("oracle sample failed")


def oracle_sample(job):
    """The oracle on the bounded sample, timed once. Returns (seconds, raw bytes)."""
    import oracle
    TD = job.T * job.D
    xs = {s: job.host[s * TD:(s + 1) * TD].numpy().view(np.uint16).reshape(job.T, job.D)
          for s in ORACLE_SLICES}
    pl = oracle.Plan.from_workload(job.w_l)
    pt = oracle.Plan.from_workload(job.w_t, bases=job.bases, widths=job.plan_t.widths())
    t0 = time.perf_counter()
    oracle_step(pl, pt, xs)
    return time.perf_counter() - t0, sum(x.nbytes for x in xs.values())


def run_kvc(args):
    import torch

    import kvgen
    import transform_codec_b200 as kvc
    world, rank, local = dist_setup()
    torch.cuda.set_device(local)
    w_l, w_t = kvgen.WORKLOADS[WORKLOAD_L], kvgen.WORKLOADS[WORKLOAD_T]
    job = Job(w_l, w_t, n_frames=args.frames, basis=args.basis)
    ok = job.check(() if args.no_oracle_check else (0, 13))
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
    for _ in range(args.warmup):
        job.step(ev)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    phase = np.zeros(5)
    kvc.profile_begin()
    with ClockSampler(torch.cuda.current_device()) as clk:
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        t_start.record()
        for _ in range(args.steps):
            job.step(ev)
            torch.cuda.synchronize()
            phase += [ev[0].elapsed_time(ev[1]), ev[1].elapsed_time(ev[2]),
                      ev[3].elapsed_time(ev[4]), ev[4].elapsed_time(ev[5]),
                      ev[0].elapsed_time(ev[5])]
        t_end.record()
        torch.cuda.synchronize()
    kernels = kvc.profile_end()
    timed_ok = job.statuses_ok()
    total_ms = t_start.elapsed_time(t_end)
    barrier(world)
    torch.cuda.synchronize()
    total_ms, = max_over_ranks([total_ms], world)
    phase = np.array(max_over_ranks((phase / args.steps).tolist(), world))
    ms_step = total_ms / args.steps
    raw = job.raw_bytes
    cont_l, cont_t = sum(job.sizes_l), sum(job.sizes_t)
    value = world * 4 * raw / (ms_step * 1e-3) / 1e9
    hbm_peak, bf16_peak, sm_max, peak_kind = measured_peaks()
    launches = sum(n for n, _ in kernels.values())
    step_cont = {"lossless_encode": cont_l, "lossless_decode": cont_l, "transform_project": cont_t,
                 "transform_entropy": cont_t, "transform_decode_codes": cont_t, "transform_decode": cont_t}
    kern_out = {}
    total_kern_ms = sum(t for _, t in kernels.values()) or 1.0
    for name, (n, t) in kernels.items():
        entry = {"launches": n, "total_ms": round(t, 3), "share": round(t / total_kern_ms, 4)}
        if name in KERNEL_WORK and n:
            bound, fn, dt = KERNEL_WORK[name]
            work = fn(raw, step_cont[name], job.mid_vals * job.frames) * args.steps
            secs = t * 1e-3
            if bound == "hbm":
                ach = work / secs / 1e9
                entry.update(bound="hbm", achieved=round(ach, 1), peak=hbm_peak, unit="GB/s",
                             frac=round(ach / hbm_peak, 4),
                             algorithmic_bytes_per_launch=int(work / n))
            else:
                ach = work / secs / 1e12
                peak = bf16_peak * TENSOR_RATIO[dt]
                entry.update(bound=bound, achieved=round(ach, 3), peak=round(peak, 2),
                             unit="TFLOP/s", frac=round(ach / peak, 4), dtype=dt,
                             algorithmic_flops_per_launch=int(work / n))
        if name in DRAM_BYTES_PER_FRAME and n:
            entry["traffic"] = int(DRAM_BYTES_PER_FRAME[name] * job.frames * args.steps / n)
        kern_out[name] = entry
    dominant = max(kern_out, key=lambda k: kern_out[k]["total_ms"]) if kern_out else None
    roof = None
    if dominant and "bound" in kern_out[dominant]:
        d = kern_out[dominant]
        roof = {"kernel": dominant, "bound": d["bound"], "achieved": d["achieved"],
                "peak": d["peak"], "unit": d["unit"], "frac": d["frac"], "traffic": d.get("traffic"),
                "peak_source": (peak_kind + " copy bandwidth" if d["bound"] == "hbm" else
                                peak_kind + " sustained cuBLAS bf16"
                                + (" x 2 (nominal int8/bf16 ratio)" if d.get("dtype") == "i8" else ""))}
    e2e = None
    if not args.no_e2e:
        e_ms, h2d, d2h = run_e2e(job, max(1, min(args.steps, 3)), 1)
        e_ms, = max_over_ranks([e_ms], world)
        e2e = {"value": round(world * 4 * raw / (e_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": round(e_ms, 2)}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        dt, nbytes = oracle_sample(job)
        model, ncpu = cpu_info()
        cpu = {"value": round(4 * nbytes / dt / 1e9, 5), "unit": "GB/s", "cores": 1,
               "kind": "oracle", "sample": f"{ORACLE_SAMPLE}, {dt:.1f} s",
               "cpu": model, "nproc": ncpu}
    if rank == 0:
        gbs = lambda ms: round(raw / (ms * 1e-3) / 1e9, 1)
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded per-channel AR(1) KV, RoPE'd keys)",
            "config": {"workload": "qwen3-32b-shaped cache 64x8x32768x128 bf16 K+V, "
                                   "128 frames of 64 MiB, lossless + transform at 1.6 bits",
                       "basis": args.basis, "raw_bytes": raw, "frames": job.frames, "frame_bytes": job.frame_bytes,
                       "l2": "inputs larger than L2 (8.59 GB per step)",
                       "value_definition": "4 x raw bytes per step / step time, all ranks"},
            "ops": {"lossless_encode_gbs": gbs(phase[0]), "transform_encode_gbs": gbs(phase[1]),
                    "lossless_decode_gbs": gbs(phase[2]), "transform_decode_gbs": gbs(phase[3]),
                    "lossless_ratio": round(raw / cont_l, 4), "transform_ratio": round(raw / cont_t, 4),
                    "lossless_bits_per_value": round(8 * cont_l / (raw / 2), 4),
                    "transform_bits_per_value": round(8 * cont_t / (raw / 2), 4),
                    "checks_passed": ok, "timed_statuses_ok": timed_ok,
                    "transform_check": job.transform_check},
            "roofline": roof, "kernels": kern_out, "gpu_launches": launches,
            "cpu_baseline": cpu, "e2e": e2e, "clocks": clk.summary(),
            "setup_s": {"generate": round(job.gen_s, 1), "plan": round(job.plan_s, 1)},
        }
        print(json.dumps(line), flush=True)
    barrier(world)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def _oracle_basis_one(args):
    """Oracle basis and component variances of one slice (a pool task)."""
    import oracle
    cal, is_key, theta, kind, D = args
    if kind == 0:
        return oracle.pca(cal, is_key, theta)
    Q = oracle.fixed_basis(kind, D)
    return Q, oracle.basis_variances(cal, is_key, theta, Q)


def oracle_plan_inputs(w, kind):
    """Bases and widths of the transform plan from the oracle alone: each
    slice's basis from its calibration draw (a pool of spawned processes, plan
    time only), then the oracle's greedy allocation over every component."""
    import multiprocessing as mp

    import kvgen
    import oracle
    cal = kvgen.calibration(w)
    tasks = [(cal[s], (s // w.n_heads) % 2 == 0, w.theta, kind, w.head_dim) for s in range(w.n_slices)]
    with mp.get_context("spawn").Pool(max(1, min(32, os.cpu_count() or 1))) as pool:
        out = pool.map(_oracle_basis_one, tasks, chunksize=8)
    bases = np.stack([o[0] for o in out])
    lam = np.stack([o[1] for o in out])
    return bases, oracle.allocate(lam, w.avg_bits, w.max_bits).reshape(lam.shape)


def run_reference(args):
    """The oracle as the reference arm: each step codes the bounded sample (a
    key and a value slice of the same workload, all four operations) on one
    host core. The plan's bases and widths come from the oracle too."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import kvgen
    import oracle
    w_l, w_t = kvgen.WORKLOADS[WORKLOAD_L], kvgen.WORKLOADS[WORKLOAD_T]
    t0 = time.time()
    bases, widths = oracle_plan_inputs(w_t, BASES[args.basis])
    plan_s = time.time() - t0
    xs = {s: kvgen.slices(w_l, s, 1)[0] for s in ORACLE_SLICES}
    pl = oracle.Plan.from_workload(w_l)
    pt = oracle.Plan.from_workload(w_t, bases=bases, widths=widths)
    for _ in range(args.warmup):
        oracle_step(pl, pt, xs)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(pl, pt, xs)
    dt = (time.perf_counter() - t0) / args.steps
    nbytes = sum(x.nbytes for x in xs.values())
    value = 4 * nbytes / dt / 1e9
    model, ncpu = cpu_info()
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 5), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt * 1e3, 1), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "qwen3-32b-shaped cache 64x8x32768x128 bf16 K+V, "
                               "128 frames of 64 MiB, lossless + transform at 1.6 bits",
                   "basis": args.basis, "sample": ORACLE_SAMPLE},
        "cpu_baseline": {"kind": "oracle", "cores": 1, "sample": ORACLE_SAMPLE, "value": round(value, 5),
                         "unit": "GB/s", "cpu": model, "nproc": ncpu},
        "e2e": {"value": round(value, 5), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "setup_s": {"oracle_plan": round(plan_s, 1)},
    }
    print(json.dumps(line), flush=True)


def run_migration(args):
    """Host-streamed migration of the 50,331,648-byte live-migration block
    (QATQ "Measured evidence": raw streamed blocks against the codec's
    transferred bytes), lossless, through the library's host-streamed calls:
    send = kvc_stream_encode_host (pinned H2D of each frame of
    `--migration-slices` slices, encode, D2H of its container), receive =
    kvc_stream_decode_host (H2D of each container, decode, D2H of the restored
    frame); each call overlaps the copies with the codec on three streams.
    Device-timed with events around each blocking call; the restored bytes are
    checked against the input."""
    import torch

    import kvgen
    import transform_codec_b200 as kvc
    w = kvgen.WORKLOADS["lossless-8x8x1536x128-bf16"]
    spf = args.migration_slices
    n = w.n_slices
    F = -(-n // spf)
    host = torch.empty(n * w.n_tokens * w.head_dim, dtype=torch.int16).pin_memory()
    kvgen.slices(w, 0, n, out=host.data_ptr())
    plan = kvc.Plan(kvc.Shape.from_workload(w))
    cap = sum(plan.max_encoded_bytes(kvc.LOSSLESS, min(spf, n - f * spf)) for f in range(F))
    h_cont = torch.empty(cap, dtype=torch.uint8).pin_memory()
    h_back = torch.empty_like(host).pin_memory()
    fb = torch.zeros(F, dtype=torch.int64)
    res = torch.zeros(F, 2, dtype=torch.int64).pin_memory()
    buf = torch.empty(kvc.stream_buffer_bytes(plan, kvc.LOSSLESS, spf), dtype=torch.uint8, device="cuda")
    stream = torch.cuda.Stream()

    def send():
        kvc.stream_encode_host(plan, kvc.LOSSLESS, 0, n, spf, host, h_cont, fb, res, buf, stream=stream)

    def receive():
        kvc.stream_decode_host(plan, kvc.LOSSLESS, n, spf, h_cont, fb, h_back, res, buf, stream=stream)

    def timed(fn, steps, warmup):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / steps

    ms_send = timed(send, args.steps, args.warmup)
    sent = int(fb.sum())
    ms_recv = timed(receive, args.steps, args.warmup)
    exact = bool(torch.equal(h_back, host)) and not bool((res[:, 0] & 0xFFFFFFFF).any())
    raw = n * w.n_tokens * w.head_dim * 2
    print(json.dumps({
        "metric": "host-streamed migration, lossless: GB/s of raw bytes from and to pinned host memory",
        "workload": f"live-migration block {w.n_layers}x{w.n_heads}x{w.n_tokens}x{w.head_dim} bf16 K+V "
                    f"({raw} bytes), {F} frames of {spf} slices",
        "send_gbs": round(raw / (ms_send * 1e-3) / 1e9, 2), "send_ms": round(ms_send, 3),
        "receive_gbs": round(raw / (ms_recv * 1e-3) / 1e9, 2), "receive_ms": round(ms_recv, 3),
        "raw_bytes": raw, "transferred_bytes": sent, "ratio_vs_raw": round(sent / raw, 4),
        "exact": exact, "steps": args.steps, "warmup": args.warmup, "data": "synthetic"}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["kvc", "reference"], default="kvc")
    ap.add_argument("--frames", type=int, default=None, help="limit frames (debug only)")
    ap.add_argument("--no-oracle-check", action="store_true",
                    help="skip the sampled transform check against the oracle")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--migration", action="store_true",
                    help="instead of the bench step: the host-streamed migration workload")
    ap.add_argument("--migration-slices", type=int, default=32, help="slices per streamed frame")
    ap.add_argument("--basis", choices=sorted(BASES), default="pca",
                    help="transform basis: calibrated PCA (default) or a fixed Hadamard / DCT-II")
    args = ap.parse_args()
    if args.warmup < 3 and args.frames is None:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    elif args.migration:
        run_migration(args)
    else:
        run_kvc(args)


if __name__ == "__main__":
    main()
