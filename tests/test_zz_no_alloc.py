"""kvc_stage_stream_encode_noalloc: the rANS stage encoder on the library's own
fixed scratch must give the bytes and result of kvc_stage_stream_encode (the
entry point with a caller-provided scratch) on two calls in a row, and refuse
sizes past its scratch. Kept in a file of its own that runs after the others,
so it is seen both in a fresh process and after every other test."""
import numpy as np
import pytest

import transform_codec_b200 as kvc

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _cases():
    rng = np.random.default_rng(23)
    skew = np.array([.45, .25, .12, .08, .05, .03, .015, .005])
    return [
        ("skewed-64k", rng.choice(np.arange(8) * 31, size=65536, p=skew).astype(np.uint8)),
        ("uniform-64k", rng.integers(0, 256, 65536).astype(np.uint8)),
        ("skewed-1000", rng.choice(np.arange(8), size=1000, p=skew).astype(np.uint8)),
        ("const-4096", np.full(4096, 7, np.uint8)),
        ("one", np.array([200], np.uint8)),
    ]


def _encode_with_scratch(d_sym, n):
    out = torch.zeros(16 + (n + 15) // 16 * 16, dtype=torch.uint8, device="cuda")
    scratch = torch.zeros(2 * n + 64, dtype=torch.uint8, device="cuda")
    res = torch.zeros(2, dtype=torch.int64, device="cuda")
    kvc.stage_stream_encode(d_sym, n, out, scratch, res)
    st, nbytes = kvc.read_result(res)
    return st, out[:nbytes].cpu().numpy().tobytes()


@pytest.mark.parametrize("name,sym", _cases(), ids=[c[0] for c in _cases()])
def test_noalloc_matches_scratch_entry_point_twice(name, sym):
    n = sym.size
    d_sym = torch.from_numpy(sym.copy()).cuda()
    st_ref, want = _encode_with_scratch(d_sym, n)
    assert st_ref == kvc.OK
    outs = [torch.full((16 + (n + 15) // 16 * 16,), 0xA5, dtype=torch.uint8, device="cuda")
            for _ in range(2)]
    ress = [torch.zeros(2, dtype=torch.int64, device="cuda") for _ in range(2)]
    for i in range(2):
        if i == 1:  # after the first call's set-up, a call takes no device memory
            torch.cuda.synchronize()
            free_before = torch.cuda.mem_get_info()[0]
        kvc.stage_stream_encode_noalloc(d_sym, n, outs[i], ress[i])
        if i == 1:
            torch.cuda.synchronize()
            assert torch.cuda.mem_get_info()[0] == free_before
        st, nbytes = kvc.read_result(ress[i])
        assert st == kvc.OK
        assert outs[i][:nbytes].cpu().numpy().tobytes() == want


def test_noalloc_refuses_sizes_past_its_scratch():
    d_sym = torch.zeros(65537, dtype=torch.uint8, device="cuda")
    out = torch.zeros(16 + 65552, dtype=torch.uint8, device="cuda")
    res = torch.zeros(2, dtype=torch.int64, device="cuda")
    with pytest.raises(kvc.KvcError) as e:
        kvc.stage_stream_encode_noalloc(d_sym, 65537, out, res)
    assert e.value.status == kvc.ERR_CAPACITY
    with pytest.raises(kvc.KvcError) as e:
        kvc.stage_stream_encode_noalloc(d_sym, 0, out, res)
    assert e.value.status == kvc.ERR_INVALID
