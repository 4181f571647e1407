"""The codec and stage entry points refuse bad arguments before any launch
(CPU only).

Each call in include/kvc.h states its error channel: KVC_ERR_INVALID for a
missing or misaligned pointer or a slice range outside the plan,
KVC_ERR_CAPACITY for an output or workspace below the stated bound,
KVC_ERR_UNSUPPORTED for a path the plan cannot code; nothing is launched then.
These checks run on the host, so they are exercised here through the C ABI
with device addresses that are never dereferenced. The calls run in a child
process that sees no CUDA device, so that a missing check could only fail to
launch, never touch memory.
"""
import json
import os
import subprocess
import sys

import transform_codec_b200 as kvc

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import ctypes, json
import transform_codec_b200 as kvc

lib = kvc._lib
A = 0x7F0000000000                     # a 256-byte aligned address, never read
MIS = A + 8                            # 8-byte aligned only
vp = ctypes.c_void_p
plan = kvc.Plan(kvc.Shape(kvc.BF16, 1, 2, 512, 128))   # lossless-only, 4 slices
P, S, L, T = plan.handle, plan.shape.n_slices, kvc.LOSSLESS, kvc.TRANSFORM
cap = plan.max_encoded_bytes(L, 1)
ws_enc = lib.kvc_batch_workspace_bytes(P, L, 0, 2, 1)
ws_dec = lib.kvc_batch_workspace_bytes(P, L, 1, 1, 1)   # one frame of one slice
out = {}

def enc(name, frames, path=L, ws=A, ws_bytes=None, plan_h=P, n=None):
    arr = kvc._frames(frames) if frames is not None else None
    out[name] = lib.kvc_encode_batch(plan_h, path, arr, len(frames) if n is None else n, vp(ws),
                                     ws_enc if ws_bytes is None else ws_bytes, None)

def dec(name, frames, ws=A, ws_bytes=None, path=L):
    out[name] = lib.kvc_decode_batch(P, path, kvc._frames(frames), len(frames), 1, vp(ws),
                                     ws_dec if ws_bytes is None else ws_bytes, None)

good = (0, 1, A, 0, A + (1 << 20), cap, A + (2 << 20))
def frame(**kw):
    f = dict(zip(("first_slice", "n_slices", "src", "src_bytes", "dst", "dst_cap", "res"), good))
    f.update(kw)
    return tuple(f.values())

enc("enc_null_plan", [good], plan_h=None)
enc("enc_transform_on_lossless_plan", [good], path=T)
enc("enc_unknown_path", [good], path=7)
enc("enc_null_ws", [good], ws=None)
enc("enc_misaligned_ws", [good], ws=MIS)
enc("enc_null_frames", None, n=1)
enc("enc_first_slice_past_end", [frame(first_slice=S)])
enc("enc_range_past_end", [frame(n_slices=S + 1, dst_cap=plan.max_encoded_bytes(L, S + 1))])
enc("enc_null_dst", [frame(dst=None)])
enc("enc_null_res", [frame(res=None)])
enc("enc_null_src", [frame(src=None)])
enc("enc_misaligned_src", [frame(src=MIS)])
enc("enc_misaligned_dst", [frame(dst=MIS)])
enc("enc_misaligned_res", [frame(res=MIS)])
enc("enc_dst_below_bound", [frame(dst_cap=cap - 1)])
enc("enc_second_frame_bad", [good, frame(first_slice=1, res=None)])
out["enc_single_ws_below_bound"] = lib.kvc_encode_lossless(
    P, 0, 1, vp(A), vp(A + (1 << 20)), cap, vp(A), lib.kvc_workspace_bytes(P, L, 0, 1) - 1,
    vp(A + (2 << 20)), None)
out["enc_single_transform"] = lib.kvc_encode_transform(
    P, 0, 1, vp(A), vp(A + (1 << 20)), cap, vp(A), 1 << 30, vp(A + (2 << 20)), None)

dgood = (0, 0, A, cap, A + (1 << 20), 512 * 128 * 2, A + (2 << 20))
def dframe(**kw):
    f = dict(zip(("first_slice", "n_slices", "src", "src_bytes", "dst", "dst_cap", "res"), dgood))
    f.update(kw)
    return tuple(f.values())

dec("dec_ws_below_bound", [dgood], ws_bytes=ws_dec - 1)
dec("dec_null_ws", [dgood], ws=None)
dec("dec_transform_on_lossless_plan", [dgood], path=T)
dec("dec_null_src", [dframe(src=None)])
dec("dec_null_res", [dframe(res=None)])
dec("dec_null_dst_with_capacity", [dframe(dst=None)])
dec("dec_misaligned_src", [dframe(src=MIS)])
dec("dec_misaligned_dst", [dframe(dst=MIS)])
dec("dec_misaligned_res", [dframe(res=MIS)])
out["dec_single_ws_below_one_slice"] = lib.kvc_decode_lossless(
    P, vp(A), cap, vp(A + (1 << 20)), 1 << 20, vp(A), 256, vp(A + (2 << 20)), None)

out["crc_null_src"] = lib.kvc_stage_crc32(None, 16, vp(A), None)
out["crc_null_out"] = lib.kvc_stage_crc32(vp(A), 16, None, None)
out["enc_stage_empty"] = lib.kvc_stage_stream_encode(vp(A), 0, vp(A), vp(A), vp(A), None)
out["enc_stage_too_long"] = lib.kvc_stage_stream_encode(vp(A), 65537, vp(A), vp(A), vp(A), None)
out["enc_stage_misaligned_out"] = lib.kvc_stage_stream_encode(vp(A), 16, vp(MIS), vp(A), vp(A), None)
out["enc_stage_odd_scratch"] = lib.kvc_stage_stream_encode(vp(A), 16, vp(A), vp(A + 1), vp(A), None)
out["dec_stage_empty"] = lib.kvc_stage_stream_decode(vp(A), 64, 0, vp(A), vp(A), None)
out["dec_stage_misaligned_rec"] = lib.kvc_stage_stream_decode(vp(MIS), 64, 16, vp(A), vp(A), None)
out["noalloc_too_long"] = lib.kvc_stage_stream_encode_noalloc(vp(A), 65537, vp(A), vp(A), None)
out["noalloc_empty"] = lib.kvc_stage_stream_encode_noalloc(vp(A), 0, vp(A), vp(A), None)
out["noalloc_misaligned_out"] = lib.kvc_stage_stream_encode_noalloc(vp(A), 16, vp(MIS), vp(A), None)
print(json.dumps(out))
'''

EXPECT = {
    "enc_null_plan": kvc.ERR_INVALID,
    "enc_transform_on_lossless_plan": kvc.ERR_UNSUPPORTED,
    "enc_unknown_path": kvc.ERR_UNSUPPORTED,
    "enc_null_ws": kvc.ERR_INVALID,
    "enc_misaligned_ws": kvc.ERR_INVALID,
    "enc_null_frames": kvc.ERR_INVALID,
    "enc_first_slice_past_end": kvc.ERR_INVALID,
    "enc_range_past_end": kvc.ERR_INVALID,
    "enc_null_dst": kvc.ERR_INVALID,
    "enc_null_res": kvc.ERR_INVALID,
    "enc_null_src": kvc.ERR_INVALID,
    "enc_misaligned_src": kvc.ERR_INVALID,
    "enc_misaligned_dst": kvc.ERR_INVALID,
    "enc_misaligned_res": kvc.ERR_INVALID,
    "enc_dst_below_bound": kvc.ERR_CAPACITY,
    "enc_second_frame_bad": kvc.ERR_INVALID,
    "enc_single_ws_below_bound": kvc.ERR_CAPACITY,
    "enc_single_transform": kvc.ERR_UNSUPPORTED,
    "dec_ws_below_bound": kvc.ERR_CAPACITY,
    "dec_null_ws": kvc.ERR_INVALID,
    "dec_transform_on_lossless_plan": kvc.ERR_UNSUPPORTED,
    "dec_null_src": kvc.ERR_INVALID,
    "dec_null_res": kvc.ERR_INVALID,
    "dec_null_dst_with_capacity": kvc.ERR_INVALID,
    "dec_misaligned_src": kvc.ERR_INVALID,
    "dec_misaligned_dst": kvc.ERR_INVALID,
    "dec_misaligned_res": kvc.ERR_INVALID,
    "dec_single_ws_below_one_slice": kvc.ERR_CAPACITY,
    "crc_null_src": kvc.ERR_INVALID,
    "crc_null_out": kvc.ERR_INVALID,
    "enc_stage_empty": kvc.ERR_INVALID,
    "enc_stage_too_long": kvc.ERR_INVALID,
    "enc_stage_misaligned_out": kvc.ERR_INVALID,
    "enc_stage_odd_scratch": kvc.ERR_INVALID,
    "dec_stage_empty": kvc.ERR_INVALID,
    "dec_stage_misaligned_rec": kvc.ERR_INVALID,
    "noalloc_too_long": kvc.ERR_CAPACITY,
    "noalloc_empty": kvc.ERR_INVALID,
    "noalloc_misaligned_out": kvc.ERR_INVALID,
}


def test_entry_points_refuse_bad_arguments_before_launching():
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, "-c", CHILD], cwd=ROOT, env=env, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    got = json.loads(r.stdout.strip().splitlines()[-1])
    assert set(got) == set(EXPECT)
    wrong = {k: (got[k], EXPECT[k]) for k in EXPECT if got[k] != EXPECT[k]}
    assert not wrong, wrong
