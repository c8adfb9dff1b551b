"""NumPy front end of the CPU oracle (``qlora_oracle.c``).

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the bench's
CPU-baseline leg are the only callers.  Nothing in the product package may
import this module, and this module imports nothing from the product.

Every function takes and returns host NumPy arrays.  bf16 tensors travel as
their raw ``uint16`` bit patterns so that no library rounding sits between the
caller and the oracle's own arithmetic.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "qlora_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

GCC_FLAGS = ["-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-shared", "-fPIC", "-std=c11"]


def build(force: bool = False, src: str = _SRC, out: str = _LIB) -> str:
    """Compile the oracle source into a shared library (plain gcc, fp-contract off)."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        tmp = out + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", *GCC_FLAGS, "-o", tmp, src, "-lm"])
        os.replace(tmp, out)
    return out


_lib = None


def _declare(L: ctypes.CDLL) -> ctypes.CDLL:
    p, i64, i32, f64, u32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_double, ctypes.c_uint32
    L.oracle_normal_quantile.argtypes = [f64]
    L.oracle_normal_quantile.restype = f64
    L.oracle_nf4_table.argtypes = [p]
    L.oracle_t8_table.argtypes = [p]
    L.oracle_nf4_nearest.argtypes = [ctypes.c_float]
    L.oracle_nf4_nearest.restype = i32
    L.oracle_nf4_nearest_bits.argtypes = [u32, i64, p]
    L.oracle_nf4_quantize.argtypes = [p, i32, i64, i32, p, p, p, p, p]
    L.oracle_nf4_dequantize.argtypes = [i64, i32, p, p, p, p, ctypes.c_float, p]
    L.oracle_quantize_ex.argtypes = [p, i32, i64, i32, i32, i32, i32, p, p, p, p, p]
    L.oracle_dequantize_ex.argtypes = [i64, i32, i32, i32, i32, p, p, p, p, ctypes.c_float, p]
    L.oracle_fp4_table.argtypes = [p]
    L.oracle_dq_nearest_bits.argtypes = [u32, i64, i32, p]
    L.oracle_dq_nearest_bits.restype = None
    L.oracle_e4m3_table.argtypes = [p]
    L.oracle_e4m3_table.restype = i32
    L.oracle_linear_fwd.argtypes = [i64, i64, i64, i32, f64, p, p, p, p, p, i64, p]
    L.oracle_linear_bwd.argtypes = [i64, i64, i64, i32, f64, p, p, p, p, p, p, i64, p, p, p]
    L.oracle_num_threads.restype = i32
    L.oracle_set_num_threads.argtypes = [i32]
    L.oracle_set_num_threads.restype = None
    L.oracle_adamw_step.argtypes = [i64, f64, f64, f64, f64, f64, f64, i64, p, p, p, p]
    L.oracle_adamw_step.restype = None
    L.oracle_lora_merge.argtypes = [i64, i64, i32, f64, i32, p, p, p, p, p]
    L.oracle_lora_merge.restype = None
    L.oracle_t8_nearest.argtypes = [ctypes.c_float]
    L.oracle_t8_nearest.restype = i32
    return L


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        _lib = _declare(ctypes.CDLL(build()))
    return _lib


def use_library(path: str) -> None:
    """Point this module at another build of the oracle source (the mutation
    tests load deliberately broken copies to show that the pins catch them)."""
    global _lib
    _lib = _declare(ctypes.CDLL(path))


def t8_nearest(y: float) -> int:
    return int(lib().oracle_t8_nearest(ctypes.c_float(y)))


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    return int(lib().oracle_num_threads())


def set_num_threads(n: int) -> None:
    """Threads the oracle's OpenMP loops use from now on."""
    lib().oracle_set_num_threads(int(n))


def normal_quantile(p: float) -> float:
    return float(lib().oracle_normal_quantile(float(p)))


def nf4_table() -> np.ndarray:
    out = np.zeros(16, np.float32)
    lib().oracle_nf4_table(_ptr(out))
    return out


def t8_table() -> np.ndarray:
    out = np.zeros(255, np.float32)
    lib().oracle_t8_table(_ptr(out))
    return out


def nf4_nearest(x: float) -> int:
    return int(lib().oracle_nf4_nearest(ctypes.c_float(x)))


def nf4_nearest_bits(start: int, n: int) -> np.ndarray:
    """Nearest-code index of the n consecutive fp32 bit patterns from ``start``."""
    out = np.zeros(n, np.uint8)
    lib().oracle_nf4_nearest_bits(ctypes.c_uint32(start), n, _ptr(out))
    return out


def fp4_table() -> np.ndarray:
    out = np.zeros(16, np.float32)
    lib().oracle_fp4_table(_ptr(out))
    return out


def e4m3_table() -> np.ndarray:
    out = np.zeros(256, np.float32)
    k = lib().oracle_e4m3_table(_ptr(out))
    return out[:k].copy()


CODE_TYPES = {"nf4": 0, "fp4": 1}
DQ_TYPES = {"int8": 0, "e4m3": 1}


def dq_nearest_bits(start: int, n: int, dq_type: str = "int8") -> np.ndarray:
    """Nearest 8-bit code (brute force) of the n fp32 bit patterns from ``start``."""
    out = np.zeros(n, np.uint8)
    lib().oracle_dq_nearest_bits(ctypes.c_uint32(start), n, DQ_TYPES[dq_type], _ptr(out))
    return out


def nf4_quantize(w: np.ndarray, double_quant: bool = True, blocksize: int = 64, code_type: str = "nf4",
                 dq_type: str = "int8") -> dict:
    """Blockwise 4-bit quantization (+ double quantization) of a flat tensor.

    ``w`` is either ``uint16`` (bf16 bit patterns) or ``float32``.
    Returns ``codes`` (uint8, ceil(n/2)), ``absmax`` (float32, ceil(n/bs)) and,
    with double quantization, ``q8`` (uint8, nb), ``c1`` (float32, ceil(nb/256))
    and ``offset`` (float).  The defaults are the NF4 / linear 8-bit / block
    64 format; ``code_type`` "fp4", ``dq_type`` "e4m3" and block sizes 128 and
    256 are the variants.
    """
    w = np.ascontiguousarray(w).reshape(-1)
    if w.dtype == np.uint16:
        is_bf16 = 1
    elif w.dtype == np.float32:
        is_bf16 = 0
    else:
        raise TypeError("w must be uint16 (bf16 bits) or float32")
    n = w.size
    nb = (n + blocksize - 1) // blocksize
    nb2 = (nb + 255) // 256
    codes = np.zeros((n + 1) // 2, np.uint8)
    absmax = np.zeros(nb, np.float32)
    q8 = np.zeros(nb, np.uint8)
    c1 = np.zeros(nb2, np.float32)
    off = np.zeros(1, np.float32)
    lib().oracle_quantize_ex(_ptr(w), is_bf16, n, int(bool(double_quant)), int(blocksize), CODE_TYPES[code_type],
                             DQ_TYPES[dq_type], _ptr(codes), _ptr(absmax), _ptr(q8), _ptr(c1), _ptr(off))
    out = {"codes": codes, "absmax": absmax}
    if double_quant:
        out.update(q8=q8, c1=c1, offset=float(off[0]))
    return out


def nf4_dequantize(n: int, q: dict, double_quant: bool = True, blocksize: int = 64, code_type: str = "nf4",
                   dq_type: str = "int8") -> np.ndarray:
    """doubleDequant: bf16 bit patterns (uint16, n) of the dequantized tensor."""
    out = np.zeros(n, np.uint16)
    codes = np.ascontiguousarray(q["codes"], np.uint8)
    ct, dt = CODE_TYPES[code_type], DQ_TYPES[dq_type]
    if double_quant:
        q8 = np.ascontiguousarray(q["q8"], np.uint8)
        c1 = np.ascontiguousarray(q["c1"], np.float32)
        lib().oracle_dequantize_ex(n, 1, int(blocksize), ct, dt, _ptr(codes), None, _ptr(q8), _ptr(c1),
                                   ctypes.c_float(q["offset"]), _ptr(out))
    else:
        absmax = np.ascontiguousarray(q["absmax"], np.float32)
        lib().oracle_dequantize_ex(n, 0, int(blocksize), ct, dt, _ptr(codes), _ptr(absmax), None, None,
                                   ctypes.c_float(0.0), _ptr(out))
    return out


def _bits(a: np.ndarray) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError("expected bf16 bit patterns (uint16)")
    return a


def linear_fwd(X: np.ndarray, W: np.ndarray, A: np.ndarray, B: np.ndarray, s: float,
               rows: np.ndarray | None = None) -> np.ndarray:
    """Y = X W^T + s (X A^T) B^T in fp64 (all inputs bf16 bits, 2-D).

    ``rows`` selects rows of Y (int64 indices); None computes all of them.
    """
    X, W, A, B = map(_bits, (X, W, A, B))
    M, K = X.shape
    N = W.shape[0]
    r = A.shape[0]
    assert W.shape == (N, K) and A.shape == (r, K) and B.shape == (N, r)
    if rows is not None:
        rows = np.ascontiguousarray(rows, np.int64)
        nrows = rows.size
    else:
        nrows = M
    Y = np.zeros((nrows, N), np.float64)
    lib().oracle_linear_fwd(M, N, K, r, float(s), _ptr(X), _ptr(W), _ptr(A), _ptr(B),
                            _ptr(rows), nrows, _ptr(Y))
    return Y


def linear_bwd(dY: np.ndarray, X: np.ndarray, W: np.ndarray, A: np.ndarray, B: np.ndarray,
               s: float, rows: np.ndarray | None = None, want_dx: bool = True):
    """(dX, dA, dB) in fp64.  dX only for ``rows`` (all when None); dX is None
    when ``want_dx`` is false.  There is no dW: the frozen weight has no
    gradient."""
    dY, X, W, A, B = map(_bits, (dY, X, W, A, B))
    M, K = X.shape
    N = W.shape[0]
    r = A.shape[0]
    assert dY.shape == (M, N) and W.shape == (N, K) and A.shape == (r, K) and B.shape == (N, r)
    if rows is not None:
        rows = np.ascontiguousarray(rows, np.int64)
        nrows = rows.size
    else:
        nrows = M
    dX = np.zeros((nrows, K), np.float64) if want_dx else None
    dA = np.zeros((r, K), np.float64)
    dB = np.zeros((N, r), np.float64)
    lib().oracle_linear_bwd(M, N, K, r, float(s), _ptr(dY), _ptr(X), _ptr(W), _ptr(A), _ptr(B),
                            _ptr(rows), nrows, _ptr(dX), _ptr(dA), _ptr(dB))
    return dX, dA, dB


def lora_merge(W: np.ndarray, A: np.ndarray, B: np.ndarray, s: float, sign: int = 1,
               want_exact: bool = False):
    """bf16 bits of W + sign * s * B A, rounded once from fp64 (merge: W the
    dequantized base, sign +1; unmerge: W the merged weight, sign -1).
    With ``want_exact`` also returns the fp64 value before the rounding."""
    W, A, B = map(_bits, (W, A, B))
    N, K = W.shape
    r = A.shape[0]
    assert A.shape == (r, K) and B.shape == (N, r)
    out = np.zeros((N, K), np.uint16)
    exact = np.zeros((N, K), np.float64) if want_exact else None
    lib().oracle_lora_merge(N, K, r, float(s), int(sign), _ptr(W), _ptr(A), _ptr(B), _ptr(out), _ptr(exact))
    return (out, exact) if want_exact else out


def fused_linear_fwd(X: np.ndarray, W: np.ndarray, A: np.ndarray, B: np.ndarray, s: float, nseg: int,
                     rows: np.ndarray | None = None) -> np.ndarray:
    """Fused projection of nseg linears sharing X: row segment i of W with
    adapter (A rows i*r.., B rows of segment i); Y is the concatenation of
    the segments' outputs (each one linear_fwd)."""
    N = W.shape[0]
    r = A.shape[0] // nseg
    S = N // nseg
    parts = [linear_fwd(X, W[i * S:(i + 1) * S], A[i * r:(i + 1) * r], B[i * S:(i + 1) * S], s, rows)
             for i in range(nseg)]
    return np.concatenate(parts, axis=1)


def fused_linear_bwd(dY: np.ndarray, X: np.ndarray, W: np.ndarray, A: np.ndarray, B: np.ndarray, s: float,
                     nseg: int, rows: np.ndarray | None = None):
    """(dX, dA, dB) of the fused projection: dX is the sum (fp64) of the
    segments' input gradients, dA and dB the segments' adapter gradients
    stacked in segment order."""
    N = W.shape[0]
    r = A.shape[0] // nseg
    S = N // nseg
    dX, dA, dB = None, [], []
    for i in range(nseg):
        gx, ga, gb = linear_bwd(dY[:, i * S:(i + 1) * S], X, W[i * S:(i + 1) * S], A[i * r:(i + 1) * r],
                                B[i * S:(i + 1) * S], s, rows)
        dX = gx if dX is None else dX + gx
        dA.append(ga)
        dB.append(gb)
    return dX, np.concatenate(dA, axis=0), np.concatenate(dB, axis=0)


def adamw_step(p: np.ndarray, m: np.ndarray, v: np.ndarray, grad: np.ndarray, *, lr: float, step: int,
               beta1: float = 0.9, beta2: float = 0.999, eps: float = 1e-8, weight_decay: float = 0.0,
               grad_scale: float = 1.0) -> None:
    """One AdamW step in fp64, in place on the float64 arrays p, m, v."""
    for a in (p, m, v):
        assert a.dtype == np.float64 and a.flags["C_CONTIGUOUS"]
    g = np.ascontiguousarray(grad, np.float64)
    lib().oracle_adamw_step(p.size, float(lr), float(beta1), float(beta2), float(eps), float(weight_decay),
                            float(grad_scale), int(step), _ptr(p), _ptr(m), _ptr(v), _ptr(g))
