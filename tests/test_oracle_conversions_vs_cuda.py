"""The oracle's own fp16 and bf16 converters against NVIDIA's.

The oracle converts fp32 to binary16 with directed rounding (zero points
rounded down, scales rounded up) and to bfloat16 with round-to-nearest-even,
in its own code.  tests/emu/f16_crosscheck.cpp calls those functions and the
CUDA headers' host implementations of __float2half_rn / _rd / _ru and
__float2bfloat16_rn on every fp32 pattern whose magnitude lies in
[2^-25, 2^17) (both signs, all three modes) and on a dense stride of all
2^32 patterns, and counts disagreements (NaN only has to stay NaN)."""
import os
import shutil
import subprocess

import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "emu", "f16_crosscheck.cpp")


def test_oracle_conversions_match_cuda_host_conversions(tmp_path):
    import emu_harness
    inc, gxx = emu_harness.cuda_include(), shutil.which("g++")
    if not inc or not gxx:
        pytest.skip("g++ or the CUDA headers are missing")
    exe = str(tmp_path / "f16_crosscheck")
    r = subprocess.run([gxx, "-std=c++17", "-O2", "-fopenmp", "-I", inc, SRC, "-o", exe, "-ldl"],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr[-3000:]
    oracle.lib()
    r = subprocess.run([exe, oracle.LIB, "61"], capture_output=True, text=True, timeout=1200)
    checked, bad = (int(x) for x in r.stdout.split())
    assert checked > 2_000_000_000
    assert bad == 0 and r.returncode == 0
