"""Host fuzz of the oracle under AddressSanitizer and UndefinedBehaviorSanitizer:
every single-byte change and every truncation of bf16 / f32 lossless and bf16
transform containers is refused (QATQ page: corrupt or truncated input is
rejected before restore; AT-1 page, "What's proven": single-byte tamper
refusal), and forged records (changed and sealed again with fresh CRCs) and
garbage inputs meet the stream parsers without any read or write outside
their buffers. The driver is tests/fuzz_oracle.c."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.timeout(600)
def test_oracle_fuzz_under_sanitizers(tmp_path):
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not found")
    exe = str(tmp_path / "fuzz_oracle")
    subprocess.check_call([gcc, "-O2", "-g", "-std=c11", "-ffp-contract=off",
                           "-fsanitize=address,undefined", "-fno-sanitize-recover=all",
                           "-fno-omit-frame-pointer", os.path.join(ROOT, "tests", "fuzz_oracle.c"),
                           os.path.join(ROOT, "oracle", "kvco.c"), "-lm", "-o", exe])
    r = subprocess.run([exe], capture_output=True, text=True, timeout=540)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    assert r.stdout.strip().endswith("ok"), r.stdout[-2000:]
    assert "forged records accepted" in r.stdout
