import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")


@pytest.fixture(scope="session")
def O():
    """The CPU oracle (test infrastructure)."""
    from oracle import oracle
    oracle.build()
    return oracle


@pytest.fixture(scope="session")
def Q():
    """The CUDA library's torch binding (built in-tree if stale)."""
    from bit_nf4_quantized_08_b200 import build
    build.build()
    import bit_nf4_quantized_08_b200 as q
    return q


@pytest.fixture(scope="session")
def cuda():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch.device("cuda:0")


def assert_close_tol(out, ref, name=""):
    """max|d| <= 1e-2 max|ref| and ||d||_F / ||ref||_F <= 5e-3."""
    out = np.asarray(out, np.float64)
    ref = np.asarray(ref, np.float64)
    assert out.shape == ref.shape, (name, out.shape, ref.shape)
    assert np.all(np.isfinite(out)), f"{name}: non-finite output"
    d = out - ref
    mref = np.max(np.abs(ref)) if ref.size else 0.0
    fref = np.linalg.norm(ref)
    md = np.max(np.abs(d)) if d.size else 0.0
    fd = np.linalg.norm(d)
    assert md <= 1e-2 * mref + 1e-30, f"{name}: max|d|={md:.3e} > 1e-2*max|ref|={1e-2 * mref:.3e}"
    assert fd <= 5e-3 * fref + 1e-30, f"{name}: ||d||/||ref|| = {fd / max(fref, 1e-300):.3e} > 5e-3"
