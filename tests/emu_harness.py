"""Builds and runs tests/emu/kernel_emu.cpp: the library's emulatable CUDA
kernel bodies executed as host C++ (one thread per CUDA thread) under
AddressSanitizer and UndefinedBehaviorSanitizer, on arrays in the library's
storage format.  Test infrastructure only: neither the oracle nor a fallback
of the library."""
from __future__ import annotations

import os
import shutil
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(HERE, "emu", "kernel_emu.cpp")
CSRC = os.path.join(ROOT, "mixed_precision_quantized_kvq_b200", "csrc")

MODE_ATTENTION, MODE_APPEND_PC, MODE_DEQUANT_PC = 0, 1, 2


def cuda_include():
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    inc = os.path.join(os.path.dirname(os.path.dirname(os.path.realpath(nvcc))), "include")
    return inc if os.path.exists(os.path.join(inc, "cuda_fp16.h")) else None


def build(out_dir: str) -> str | None:
    """Compile the emulator into out_dir; None when g++ or the CUDA headers are missing."""
    inc, gxx = cuda_include(), shutil.which("g++")
    if not inc or not gxx:
        return None
    exe = os.path.join(out_dir, "kernel_emu")
    cmd = [gxx, "-std=c++20", "-O1", "-g", "-fsanitize=address,undefined", "-fno-sanitize-recover=all",
           "-fno-omit-frame-pointer", "-frounding-math", "-ffp-contract=off", "-I", inc, "-I", CSRC,
           "-I", os.path.join(HERE, "emu"), SRC, "-o", exe, "-pthread"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(r.stderr[-4000:])
    return exe


def run(exe: str, tmp: str, params: dict, arrays: dict, outputs: dict) -> dict:
    """Write params and arrays to tmp, run the emulator, read `outputs`
    ({name: (dtype, shape)}) back."""
    with open(os.path.join(tmp, "params.txt"), "w") as f:
        for k, v in params.items():
            f.write(f"{k} {float(v)!r}\n")
    for k, a in arrays.items():
        if a is not None:
            np.ascontiguousarray(a).tofile(os.path.join(tmp, k + ".bin"))
    env = dict(os.environ, ASAN_OPTIONS="detect_leaks=0")
    r = subprocess.run([exe, str(tmp)], capture_output=True, text=True, timeout=900, env=env)
    if r.returncode != 0:
        raise AssertionError((r.stdout + r.stderr)[-4000:])
    return {k: np.fromfile(os.path.join(tmp, k + ".bin"), dt).reshape(shape) for k, (dt, shape) in outputs.items()}


def cache_params(c) -> tuple[dict, dict]:
    """Layout scalars and cache arrays of an oracle.Cache, for the emulator."""
    lay = c.layout
    params = dict(d=lay.head_dim, hq=lay.num_q_heads, hkv=lay.num_kv_heads, kb=lay.k_bits, vb=lay.v_bits,
                  kg=lay.k_group, vg=lay.v_group, W=lay.window, rotate=int(lay.rotate_keys),
                  kpc=int(getattr(lay, "k_per_channel", False)), batch=c.batch,
                  max_pages=c.page_table.shape[1], num_pages=c.num_pages)
    arrays = dict(k_codes=c.k_codes, v_codes=c.v_codes, k_meta=c.k_meta, v_meta=c.v_meta, k_win=c.k_win,
                  v_win=c.v_win, page_table=c.page_table)
    return params, arrays
