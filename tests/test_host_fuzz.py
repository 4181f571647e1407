"""Host-side code of the library under AddressSanitizer and
UndefinedBehaviorSanitizer: api.cpp (plan validation and sizing, the greedy
allocation, the calibration solvers) is compiled here with the sanitizers and
driven by tests/fuzz_host.cpp with valid, extreme and invalid arguments; the
device objects are linked as built. Every call must return a status without a
read or write outside its buffers."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")


@pytest.mark.timeout(600)
def test_host_library_under_sanitizers(tmp_path):
    gxx = shutil.which("g++")
    if gxx is None or not os.path.isdir(os.path.join(CUDA, "include")):
        pytest.skip("g++ or the CUDA headers not found")
    import importlib.util
    spec = importlib.util.spec_from_file_location("_kvc_build", os.path.join(ROOT, "transform_codec_b200", "build.py"))
    build = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(build)
    build.build()  # the device objects
    objs = [os.path.join(build.BUILD, f + ".o") for f in ("container.cu", "lossless.cu", "transform.cu")]
    san = ["-std=c++17", "-O1", "-g", "-fsanitize=address,undefined", "-fno-sanitize-recover=all",
           "-fno-omit-frame-pointer", "-I", os.path.join(ROOT, "include"), "-I", os.path.join(CUDA, "include")]
    api = str(tmp_path / "api.o")
    subprocess.check_call([gxx, *san, "-I", build.CSRC, "-c", os.path.join(build.CSRC, "api.cpp"), "-o", api])
    exe = str(tmp_path / "fuzz_host")
    subprocess.check_call([gxx, *san, os.path.join(ROOT, "tests", "fuzz_host.cpp"), api, *objs,
                           "-L", os.path.join(CUDA, "lib64"), "-lcudart", "-lpthread", "-o", exe])
    # the CUDA runtime maps memory in ASan's shadow gap on machines with a GPU,
    # and keeps its own allocations until exit
    env = dict(os.environ, ASAN_OPTIONS="protect_shadow_gap=0:detect_leaks=0")
    r = subprocess.run([exe], capture_output=True, text=True, timeout=540, env=env)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    assert r.stdout.strip().endswith("ok"), r.stdout[-2000:]
