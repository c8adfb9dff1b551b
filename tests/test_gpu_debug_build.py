"""The bounds-checked debug build (libqlora_nf4_debug.so, compiled with
QLORA_DEBUG; selected by QLORA_LIBRARY=debug): device-side checks of the
computed store indices record QLORA_ERR_BOUNDS instead of trapping.  The
guard-byte, variant, small-M and fused-projection tests run against it in a
child process; every one of them checks the status word after its calls,
so a failed bounds check fails them."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
pytestmark = pytest.mark.gpu


def test_debug_build_passes_guard_and_parity_tests(cuda):
    from bit_nf4_quantized_08_b200 import build
    build.build(debug=True)
    env = dict(os.environ, QLORA_LIBRARY="debug")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider",
                        "tests/test_gpu_canary.py", "tests/test_gpu_variants.py", "tests/test_gpu_fused.py",
                        "tests/test_gpu_linear.py"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=1800)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]
    assert "passed" in r.stdout
