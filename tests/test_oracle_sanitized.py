"""The oracle's pin tests, once more with the oracle built under
AddressSanitizer and UndefinedBehaviorSanitizer (KVQO_SANITIZE=1, libasan
preloaded into a child Python process): every access of the plain-C
reference stays inside its buffers and no undefined behaviour is hit on
the pinned cases."""
import os
import subprocess
import sys

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
PINS = ["test_oracle_numerics.py", "test_oracle_quantizer.py", "test_oracle_attention.py",
        "test_oracle_cache.py", "test_oracle_prefill.py", "test_oracle_per_channel.py"]


def _runtime(name):
    try:
        path = subprocess.run(["gcc", f"-print-file-name={name}"], capture_output=True, text=True).stdout.strip()
    except OSError:
        return None
    return path if os.path.isabs(path) and os.path.exists(path) else None


def test_oracle_pins_under_sanitizers():
    asan, ubsan = _runtime("libasan.so"), _runtime("libubsan.so")
    if not asan or not ubsan:
        pytest.skip("gcc sanitizer runtimes are missing")
    env = dict(os.environ, KVQO_SANITIZE="1", LD_PRELOAD=f"{asan} {ubsan}",
               ASAN_OPTIONS="detect_leaks=0:verify_asan_link_order=0")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        *[os.path.join(HERE, p) for p in PINS]],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=1200)
    assert r.returncode == 0, (r.stdout + r.stderr)[-4000:]
    assert "passed" in r.stdout
