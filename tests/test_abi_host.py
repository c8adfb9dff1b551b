"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every function include/qlora_nf4.h declares, answers workspace queries, and
rejects bad arguments before launching anything."""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qlora_nf4.h")

FAKE = 0x7F0000000000  # 256-byte aligned stand-in pointer; never dereferenced


def _declared_functions():
    txt = open(HEADER).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    names = re.findall(r"\b(qlora_[a-z0-9_]+)\s*\(", txt)
    return sorted(set(names))


def test_header_and_exports(Q):
    from bit_nf4_quantized_08_b200 import _lib
    lib = _lib.lib()
    declared = _declared_functions()
    assert set(declared) == set(_lib.EXPORTS)
    for name in declared:
        assert hasattr(lib, name), f"{name} not exported"


def test_debug_build_loads_and_exports():
    """The bounds-checked build (QLORA_DEBUG) loads without a GPU and exports
    the same C ABI."""
    from bit_nf4_quantized_08_b200 import build
    path = build.build(debug=True)
    dbg = ctypes.CDLL(path)
    for name in _declared_functions():
        assert hasattr(dbg, name), f"{name} not exported by the debug build"
    dbg.qlora_get_last_error.argtypes = [ctypes.c_void_p]
    dbg.qlora_get_last_error.restype = ctypes.c_int32


def test_nf4_table_matches_oracle(Q, O):
    np.testing.assert_array_equal(np.array(Q.qlora_nf4_table(), np.float32).view(np.uint32),
                                  O.nf4_table().view(np.uint32))


def _w(rows=256, cols=256, dq=1, blocksize=64, codes=FAKE, code_type=0, dq_type=0):
    from bit_nf4_quantized_08_b200._lib import CNF4Weight
    return CNF4Weight(rows, cols, blocksize, dq, codes, FAKE, FAKE, FAKE, FAKE, code_type, dq_type)


def test_quantize_workspace_sizes(Q):
    from bit_nf4_quantized_08_b200._lib import lib
    L = lib()
    assert L.qlora_nf4_quantize_workspace(4096, 4096, 64, 0) == 0
    n = 4096 * 4096
    nb, ng = n // 64, n // 16384
    assert L.qlora_nf4_quantize_workspace(4096, 4096, 64, 1) == nb * 4 + ng * 8
    assert L.qlora_nf4_quantize_workspace(4096, 4096, 32, 1) == 0
    assert L.qlora_nf4_quantize_workspace(4096, 4096, 128, 1) == (n // 128) * 4 + ng * 8
    assert L.qlora_nf4_quantize_workspace(4096, 4096, 256, 1) == (n // 256) * 4 + ng * 8
    assert L.qlora_nf4_quantize_workspace(-1, 4, 64, 1) == 0

    def a256(x):
        return (x + 255) // 256 * 256

    # more than 8192 group sums: one fp64 partial per 4096 leaves of the
    # zero-padded power-of-two leaf array of the offset tree
    for rows, cols, partials in ((16384, 16384, 4), (9000, 16384, 4), (8192, 16384, 0)):
        n = rows * cols
        nb, ng = -(-n // 64), -(-n // 16384)
        want = a256(nb * 4) + a256(ng * 8) + a256(partials * 8)
        assert L.qlora_nf4_quantize_workspace(rows, cols, 64, 1) == want, (rows, cols)


def test_quantize_rejects(Q):
    from bit_nf4_quantized_08_b200._lib import lib, QLORA_ERR_INVALID_ARG, QLORA_ERR_UNSUPPORTED, QLORA_BF16
    L = lib()
    ws = FAKE
    big = 1 << 30
    assert L.qlora_nf4_quantize(FAKE, QLORA_BF16, None, ws, big, None) == QLORA_ERR_INVALID_ARG
    assert L.qlora_nf4_quantize(FAKE, QLORA_BF16, ctypes.byref(_w(blocksize=32)), ws, big, None) == QLORA_ERR_UNSUPPORTED
    assert L.qlora_nf4_quantize(FAKE, QLORA_BF16, ctypes.byref(_w(blocksize=512)), ws, big, None) == QLORA_ERR_UNSUPPORTED
    assert L.qlora_nf4_quantize(FAKE, QLORA_BF16, ctypes.byref(_w(code_type=2)), ws, big, None) == QLORA_ERR_INVALID_ARG
    assert L.qlora_nf4_quantize(FAKE, QLORA_BF16, ctypes.byref(_w(dq_type=-1)), ws, big, None) == QLORA_ERR_INVALID_ARG
    assert L.qlora_nf4_quantize(None, QLORA_BF16, ctypes.byref(_w()), ws, big, None) == QLORA_ERR_INVALID_ARG
    assert L.qlora_nf4_quantize(FAKE + 8, QLORA_BF16, ctypes.byref(_w()), ws, big, None) == QLORA_ERR_INVALID_ARG
    assert L.qlora_nf4_quantize(FAKE, 7, ctypes.byref(_w()), ws, big, None) == QLORA_ERR_INVALID_ARG
    assert L.qlora_nf4_quantize(FAKE, QLORA_BF16, ctypes.byref(_w()), ws, 16, None) == QLORA_ERR_INVALID_ARG
    assert L.qlora_nf4_quantize(FAKE, QLORA_BF16, ctypes.byref(_w(dq=2)), ws, big, None) == QLORA_ERR_INVALID_ARG
    assert L.qlora_nf4_quantize(FAKE, QLORA_BF16, ctypes.byref(_w(rows=-3)), ws, big, None) == QLORA_ERR_INVALID_ARG
    assert L.qlora_nf4_quantize(FAKE, QLORA_BF16, ctypes.byref(_w(codes=FAKE + 4)), ws, big, None) == QLORA_ERR_INVALID_ARG
    # an empty tensor is valid and enqueues nothing
    assert L.qlora_nf4_quantize(None, QLORA_BF16, ctypes.byref(_w(rows=0)), None, 0, None) == 0


def test_linear_rejects(Q):
    from bit_nf4_quantized_08_b200._lib import lib, QLORA_ERR_INVALID_ARG, QLORA_ERR_UNSUPPORTED
    L = lib()
    big = 1 << 34
    f = L.qlora_linear_fwd
    w = _w(256, 256)
    assert f(FAKE, 16, ctypes.byref(_w(256, 200)), FAKE, FAKE, 8, 2.0, FAKE, FAKE, big, None) == QLORA_ERR_UNSUPPORTED
    assert f(FAKE, 16, ctypes.byref(_w(260, 256)), FAKE, FAKE, 8, 2.0, FAKE, FAKE, big, None) == QLORA_ERR_UNSUPPORTED
    assert f(FAKE, 16, ctypes.byref(w), FAKE, FAKE, 12, 2.0, FAKE, FAKE, big, None) == QLORA_ERR_UNSUPPORTED
    assert f(FAKE, 16, ctypes.byref(w), FAKE, FAKE, 264, 2.0, FAKE, FAKE, big, None) == QLORA_ERR_UNSUPPORTED
    assert f(FAKE, 16, ctypes.byref(w), FAKE, FAKE, -8, 2.0, FAKE, FAKE, big, None) == QLORA_ERR_INVALID_ARG
    assert f(FAKE, -1, ctypes.byref(w), FAKE, FAKE, 8, 2.0, FAKE, FAKE, big, None) == QLORA_ERR_INVALID_ARG
    assert f(None, 16, ctypes.byref(w), FAKE, FAKE, 8, 2.0, FAKE, FAKE, big, None) == QLORA_ERR_INVALID_ARG
    assert f(FAKE, 16, ctypes.byref(w), None, FAKE, 8, 2.0, FAKE, FAKE, big, None) == QLORA_ERR_INVALID_ARG
    assert f(FAKE, 16, ctypes.byref(w), FAKE, FAKE, 8, 2.0, FAKE + 2, FAKE, big, None) == QLORA_ERR_INVALID_ARG
    assert f(FAKE, 16, ctypes.byref(w), FAKE, FAKE, 8, 2.0, FAKE, FAKE, 64, None) == QLORA_ERR_INVALID_ARG
    assert f(FAKE, 16, ctypes.byref(_w(256, 256, blocksize=32)), FAKE, FAKE, 8, 2.0, FAKE, FAKE, big, None) == QLORA_ERR_UNSUPPORTED
    b = L.qlora_linear_bwd
    assert b(FAKE, FAKE, 16, ctypes.byref(w), FAKE, FAKE, 8, 2.0, FAKE, None, FAKE, FAKE, big, None) == QLORA_ERR_INVALID_ARG
    assert b(FAKE, FAKE, 16, ctypes.byref(w), FAKE, FAKE, 8, 2.0, FAKE + 2, FAKE, FAKE, FAKE, big, None) == QLORA_ERR_INVALID_ARG
    assert b(FAKE, FAKE, 16, ctypes.byref(_w(256, 100)), FAKE, FAKE, 8, 2.0, FAKE, FAKE, FAKE, FAKE, big, None) == QLORA_ERR_UNSUPPORTED
    # M == 0 forward: valid, nothing to do
    assert f(None, 0, ctypes.byref(w), FAKE, FAKE, 8, 2.0, None, FAKE, big, None) == 0


def test_merge_rejects(Q):
    from bit_nf4_quantized_08_b200._lib import lib, QLORA_ERR_INVALID_ARG, QLORA_ERR_UNSUPPORTED
    L = lib()
    m, u = L.qlora_lora_merge, L.qlora_lora_unmerge
    w = _w(256, 256)
    assert m(ctypes.byref(w), FAKE, FAKE, 12, 2.0, FAKE, None) == QLORA_ERR_UNSUPPORTED
    assert m(ctypes.byref(w), FAKE, FAKE, 264, 2.0, FAKE, None) == QLORA_ERR_UNSUPPORTED
    assert m(ctypes.byref(w), FAKE, FAKE, 0, 2.0, FAKE, None) == QLORA_ERR_INVALID_ARG
    assert m(ctypes.byref(_w(256, 200)), FAKE, FAKE, 8, 2.0, FAKE, None) == QLORA_ERR_UNSUPPORTED
    assert m(ctypes.byref(_w(260, 256)), FAKE, FAKE, 8, 2.0, FAKE, None) == QLORA_ERR_UNSUPPORTED
    assert m(ctypes.byref(w), None, FAKE, 8, 2.0, FAKE, None) == QLORA_ERR_INVALID_ARG
    assert m(ctypes.byref(w), FAKE, FAKE, 8, 2.0, FAKE + 8, None) == QLORA_ERR_INVALID_ARG
    assert m(None, FAKE, FAKE, 8, 2.0, FAKE, None) == QLORA_ERR_INVALID_ARG
    assert u(FAKE, 256, 256, FAKE, FAKE, 12, 2.0, FAKE, None) == QLORA_ERR_UNSUPPORTED
    assert u(None, 256, 256, FAKE, FAKE, 8, 2.0, FAKE, None) == QLORA_ERR_INVALID_ARG
    assert u(FAKE, -1, 256, FAKE, FAKE, 8, 2.0, FAKE, None) == QLORA_ERR_INVALID_ARG
    assert u(FAKE, 256, 100, FAKE, FAKE, 8, 2.0, FAKE, None) == QLORA_ERR_UNSUPPORTED
    # empty: valid, nothing to do
    assert u(None, 0, 256, FAKE, FAKE, 8, 2.0, FAKE, None) == 0


def test_adamw_and_paged_reject(Q):
    from bit_nf4_quantized_08_b200._lib import lib, CAdamWConfig, QLORA_ERR_INVALID_ARG
    L = lib()
    good = CAdamWConfig(1e-3, 0.9, 0.999, 1e-8, 0.0, 1.0, 1)
    for bad in (CAdamWConfig(1e-3, 0.9, 0.999, 1e-8, 0.0, 1.0, 0), CAdamWConfig(-1.0, 0.9, 0.999, 1e-8, 0.0, 1.0, 1),
                CAdamWConfig(1e-3, 1.0, 0.999, 1e-8, 0.0, 1.0, 1), CAdamWConfig(1e-3, 0.9, 0.999, 0.0, 0.0, 1.0, 1)):
        assert L.qlora_adamw_step(FAKE, FAKE, FAKE, FAKE, None, 16, ctypes.byref(bad), None) == QLORA_ERR_INVALID_ARG
    assert L.qlora_adamw_step(FAKE + 4, FAKE, FAKE, FAKE, None, 16, ctypes.byref(good), None) == QLORA_ERR_INVALID_ARG
    assert L.qlora_adamw_step(FAKE, FAKE, FAKE, FAKE, FAKE + 2, 16, ctypes.byref(good), None) == QLORA_ERR_INVALID_ARG
    assert L.qlora_adamw_step(None, None, None, None, None, 0, ctypes.byref(good), None) == 0
    assert L.qlora_adamw_step(FAKE, FAKE, FAKE, FAKE, None, 16, None, None) == QLORA_ERR_INVALID_ARG
    assert L.qlora_paged_alloc(16, None) == QLORA_ERR_INVALID_ARG
    p = ctypes.c_void_p(1)
    assert L.qlora_paged_alloc(0, ctypes.byref(p)) == 0 and not p.value
    assert L.qlora_paged_free(None) == 0
    assert L.qlora_paged_prefetch(None, 16, 1, None) == QLORA_ERR_INVALID_ARG


def test_linear_workspace_queries(Q):
    from bit_nf4_quantized_08_b200._lib import lib
    L = lib()
    w = _w(4096, 4096)
    fwd = L.qlora_linear_workspace(2048, ctypes.byref(w), 64, 0)
    bwd = L.qlora_linear_workspace(2048, ctypes.byref(w), 64, 1)
    # the expanded block constants alone: (K/64) x N fp32
    assert fwd >= 64 * 4096 * 4 and bwd >= fwd
    assert L.qlora_linear_workspace(2048, ctypes.byref(_w(4096, 100)), 64, 0) == 0
    assert L.qlora_linear_workspace(2048, ctypes.byref(w), 12, 0) == 0


def test_missing_library_fails_loudly(Q, tmp_path, monkeypatch):
    from bit_nf4_quantized_08_b200 import _lib
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "nope.so"))
    monkeypatch.setattr(_lib, "_lib", None)
    with pytest.raises(RuntimeError, match="no CPU fallback"):
        _lib.lib()


def test_product_does_not_import_oracle():
    pkg = os.path.join(ROOT, "bit_nf4_quantized_08_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h")):
                txt = open(os.path.join(dirpath, fn)).read()
                assert "import oracle" not in txt and "from oracle" not in txt, fn
                assert "qlora_oracle" not in txt, fn
