"""Stage parity on the GPU: CRC-32 against zlib, and the rANS stream coder
bit-exact against the oracle from the same symbols (encode) and on the oracle's
records (decode)."""
import zlib

import numpy as np
import pytest
import torch

import oracle
import transform_codec_b200 as kvc

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("n", [0, 1, 3, 4, 5, 15, 16, 17, 255, 1000, 65536, 262145, 3_000_001])
def test_stage_crc32_matches_zlib(n):
    rng = np.random.default_rng(n)
    data = rng.integers(0, 256, max(n, 1), dtype=np.uint8)[:n]
    src = torch.from_numpy(data.copy()).cuda() if n else torch.empty(16, dtype=torch.uint8, device="cuda")
    out = torch.zeros(1, dtype=torch.int32, device="cuda")
    kvc.stage_crc32(src, n, out)
    got = int(out.cpu().numpy().view(np.uint32)[0])
    assert got == zlib.crc32(data.tobytes())


def _symbols():
    rng = np.random.default_rng(42)
    out = []
    for n in [1, 2, 7, 100, 511, 512, 513, 1023, 1024, 1025, 4095, 16384, 33333, 65535, 65536]:
        out.append((f"geom{n}", np.minimum(rng.geometric(0.3, n) - 1, 255).astype(np.uint8)))
        out.append((f"two{n}", np.where(rng.random(n) < 0.99, 17, 200).astype(np.uint8)))
        out.append((f"u16_{n}", rng.integers(0, 16, n).astype(np.uint8)))
        out.append((f"rand{n}", rng.integers(0, 256, n).astype(np.uint8)))
        out.append((f"const{n}", np.full(n, 77, np.uint8)))
    z = np.minimum(rng.zipf(1.3, 65536) - 1, 255).astype(np.uint8)
    out.append(("zipf", z))
    # every symbol present, one dominant: exercises the remainder ranking
    s = np.full(65536, 5, np.uint8)
    s[:256] = np.arange(256)
    rng.shuffle(s)
    out.append(("all256", s))
    return out


@pytest.mark.parametrize("name,sym", _symbols(), ids=[n for n, _ in _symbols()])
def test_stage_stream_encode_bit_exact(name, sym):
    n = sym.size
    want = oracle.stream_encode(sym)
    d_sym = torch.from_numpy(sym.copy()).cuda()
    out = torch.zeros(16 + (n + 15) // 16 * 16, dtype=torch.uint8, device="cuda")
    scratch = torch.zeros(2 * n + 64, dtype=torch.uint8, device="cuda")
    res = torch.zeros(2, dtype=torch.int64, device="cuda")
    kvc.stage_stream_encode(d_sym, n, out, scratch, res)
    st, nbytes = kvc.read_result(res)
    assert st == kvc.OK
    got = out[:nbytes].cpu().numpy().tobytes()
    assert got == want


@pytest.mark.parametrize("name,sym", _symbols(), ids=[n for n, _ in _symbols()])
def test_stage_stream_decode_oracle_records(name, sym):
    n = sym.size
    rec = oracle.stream_encode(sym)
    d_rec = torch.frombuffer(bytearray(rec), dtype=torch.uint8).cuda()
    d_sym = torch.zeros(n, dtype=torch.uint8, device="cuda")
    res = torch.zeros(2, dtype=torch.int64, device="cuda")
    kvc.stage_stream_decode(d_rec, len(rec), n, d_sym, res)
    st, used = kvc.read_result(res)
    assert st == kvc.OK and used == len(rec)
    assert np.array_equal(d_sym.cpu().numpy(), sym)


def test_stage_stream_decode_refuses_damage():
    rng = np.random.default_rng(9)
    sym = np.minimum(rng.geometric(0.2, 20000) - 1, 255).astype(np.uint8)
    rec = bytearray(oracle.stream_encode(sym))
    assert rec[0] == 2
    res = torch.zeros(2, dtype=torch.int64, device="cuda")
    d_sym = torch.zeros(20000, dtype=torch.uint8, device="cuda")
    checked = 0
    for pos in list(range(0, 64)) + list(rng.integers(64, len(rec), 60)):
        bad = bytearray(rec)
        bad[pos] ^= 0x5A
        want_st, want_sym, _ = oracle.stream_decode(bytes(bad), 20000)
        kvc.stage_stream_decode(torch.frombuffer(bad, dtype=torch.uint8).cuda(), len(bad), 20000,
                                d_sym, res)
        st, _ = kvc.read_result(res)
        assert (st == kvc.OK) == (want_st == oracle.OK), pos
        if st == kvc.OK:
            assert np.array_equal(d_sym.cpu().numpy(), want_sym)
        checked += 1
    assert checked > 100
