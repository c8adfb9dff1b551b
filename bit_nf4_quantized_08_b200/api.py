"""Torch-facing wrappers of the C ABI, same names as the C entry points.

PyTorch supplies device memory and the current stream; every step of the
path runs in the library's CUDA kernels.  Functions that produce tensors
allocate them with ``torch.empty`` (outputs and the workspace the library asks
for) unless the caller passes them in, which the bench does to keep
allocation out of the timed region.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass

import torch

from . import _lib
from ._lib import CAdamWConfig, CNF4Weight, CODE_TYPES, DQ_TYPES, QLORA_BF16, QLORA_F32, check, lib

BLOCKSIZE = 64
DQ_BLOCK = 256


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream: torch.cuda.Stream | None = None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


@dataclass
class NF4Weight:
    """A quantized frozen weight W [rows = N, cols = K] and its constants.

    codes [ceil(N*K/2)] uint8 (element 2i in the high nibble of byte i);
    without double quantization ``absmax`` [nb] fp32; with it ``absmax_q8``
    [nb] uint8, ``absmax_scale`` [ceil(nb/256)] fp32 and ``absmax_offset``
    [1] fp32; nb = ceil(N*K / blocksize).  ``code_type`` "nf4" or "fp4",
    ``dq_type`` "int8" or "e4m3" (the 8-bit code book of the constants).
    """

    rows: int
    cols: int
    double_quant: bool
    codes: torch.Tensor
    absmax: torch.Tensor | None = None
    absmax_q8: torch.Tensor | None = None
    absmax_scale: torch.Tensor | None = None
    absmax_offset: torch.Tensor | None = None
    blocksize: int = BLOCKSIZE
    code_type: str = "nf4"
    dq_type: str = "int8"

    @property
    def nblocks(self) -> int:
        return (self.rows * self.cols + self.blocksize - 1) // self.blocksize

    def c_struct(self) -> CNF4Weight:
        return CNF4Weight(self.rows, self.cols, self.blocksize, int(self.double_quant),
                          _ptr(self.codes), _ptr(self.absmax), _ptr(self.absmax_q8),
                          _ptr(self.absmax_scale), _ptr(self.absmax_offset),
                          CODE_TYPES[self.code_type], DQ_TYPES[self.dq_type])

    def storage_bytes(self) -> int:
        t = [self.codes, self.absmax, self.absmax_q8, self.absmax_scale, self.absmax_offset]
        return sum(x.numel() * x.element_size() for x in t if x is not None)

    @staticmethod
    def empty(rows: int, cols: int, double_quant: bool = True, device="cuda", blocksize: int = BLOCKSIZE,
              code_type: str = "nf4", dq_type: str = "int8") -> "NF4Weight":
        n = rows * cols
        nb = (n + blocksize - 1) // blocksize
        codes = torch.empty((n + 1) // 2, dtype=torch.uint8, device=device)
        fmt = dict(blocksize=blocksize, code_type=code_type, dq_type=dq_type)
        if double_quant:
            return NF4Weight(rows, cols, True, codes,
                             absmax_q8=torch.empty(nb, dtype=torch.uint8, device=device),
                             absmax_scale=torch.empty((nb + DQ_BLOCK - 1) // DQ_BLOCK, dtype=torch.float32, device=device),
                             absmax_offset=torch.empty(1, dtype=torch.float32, device=device), **fmt)
        return NF4Weight(rows, cols, False, codes, absmax=torch.empty(nb, dtype=torch.float32, device=device), **fmt)


def _workspace(nbytes: int, device, ws: torch.Tensor | None) -> torch.Tensor:
    if ws is not None and ws.numel() >= nbytes:
        return ws
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


def qlora_nf4_quantize_workspace(rows: int, cols: int, double_quant: bool = True,
                                 blocksize: int = BLOCKSIZE) -> int:
    return int(lib().qlora_nf4_quantize_workspace(rows, cols, blocksize, int(double_quant)))


def qlora_nf4_quantize(W: torch.Tensor, double_quant: bool = True, out: NF4Weight | None = None,
                       ws: torch.Tensor | None = None, blocksize: int = BLOCKSIZE, code_type: str = "nf4",
                       dq_type: str = "int8") -> NF4Weight:
    """Blockwise NF4 quantization (+ 8-bit double quantization) of a 2-D
    bf16 or fp32 CUDA tensor.  blocksize, code_type and dq_type choose the
    variants (used only when ``out`` is not given; ``out`` carries its own)."""
    if W.dim() != 2 or not W.is_cuda or not W.is_contiguous():
        raise ValueError("W must be a contiguous 2-D CUDA tensor")
    if W.dtype == torch.bfloat16:
        dt = QLORA_BF16
    elif W.dtype == torch.float32:
        dt = QLORA_F32
    else:
        raise TypeError("W must be bf16 or fp32")
    rows, cols = W.shape
    if out is None:
        out = NF4Weight.empty(rows, cols, double_quant, W.device, blocksize, code_type, dq_type)
    need = qlora_nf4_quantize_workspace(rows, cols, out.double_quant, out.blocksize)
    wsb = _workspace(need, W.device, ws) if need else None
    cw = out.c_struct()
    check(lib().qlora_nf4_quantize(_ptr(W), dt, ctypes.byref(cw), _ptr(wsb), need, _stream()),
          "qlora_nf4_quantize")
    return out


def qlora_nf4_quantize_static(W: torch.Tensor, out: NF4Weight) -> NF4Weight:
    """qlora_nf4_quantize into caller-allocated outputs, with the library's
    fixed internal scratch instead of a workspace (at most
    QLORA_STATIC_QUANTIZE_MAX_ELEMS elements; calls on one device must not
    overlap)."""
    if W.dim() != 2 or not W.is_cuda or not W.is_contiguous():
        raise ValueError("W must be a contiguous 2-D CUDA tensor")
    if W.dtype == torch.bfloat16:
        dt = QLORA_BF16
    elif W.dtype == torch.float32:
        dt = QLORA_F32
    else:
        raise TypeError("W must be bf16 or fp32")
    if (out.rows, out.cols) != tuple(W.shape):
        raise ValueError("out does not match the shape of W")
    cw = out.c_struct()
    check(lib().qlora_nf4_quantize_static(_ptr(W), dt, ctypes.byref(cw), _stream()),
          "qlora_nf4_quantize_static")
    return out


def qlora_nf4_dequantize(w: NF4Weight, out: torch.Tensor | None = None) -> torch.Tensor:
    """doubleDequant: the bf16 weight [rows, cols] the layer multiplies with."""
    if out is None:
        out = torch.empty(w.rows, w.cols, dtype=torch.bfloat16, device=w.codes.device)
    cw = w.c_struct()
    check(lib().qlora_nf4_dequantize(ctypes.byref(cw), _ptr(out), _stream()), "qlora_nf4_dequantize")
    return out


def qlora_linear_workspace(M: int, w: NF4Weight, r: int, bwd: bool) -> int:
    cw = w.c_struct()
    return int(lib().qlora_linear_workspace(M, ctypes.byref(cw), r, int(bwd)))


def qlora_linear_fwd(X: torch.Tensor, w: NF4Weight, A: torch.Tensor | None, B: torch.Tensor | None,
                     scale: float, Y: torch.Tensor | None = None,
                     ws: torch.Tensor | None = None) -> torch.Tensor:
    """Y = X dequant(W)^T + scale (X A^T) B^T (bf16 in/out, fp32 accumulate)."""
    M = X.shape[0]
    r = 0 if A is None else A.shape[0]
    if Y is None:
        Y = torch.empty(M, w.rows, dtype=torch.bfloat16, device=X.device)
    need = qlora_linear_workspace(M, w, r, False)
    wsb = _workspace(need, X.device, ws)
    cw = w.c_struct()
    check(lib().qlora_linear_fwd(_ptr(X), M, ctypes.byref(cw), _ptr(A), _ptr(B), r, float(scale),
                                 _ptr(Y), _ptr(wsb), wsb.numel(), _stream()), "qlora_linear_fwd")
    return Y


def qlora_linear_bwd(dY: torch.Tensor, X: torch.Tensor, w: NF4Weight, A: torch.Tensor | None,
                     B: torch.Tensor | None, scale: float, dX: torch.Tensor | None = None,
                     dA: torch.Tensor | None = None, dB: torch.Tensor | None = None,
                     ws: torch.Tensor | None = None, want_dx: bool = True):
    """(dX, dA, dB) of the layer; the frozen weight gets no gradient."""
    M = X.shape[0]
    r = 0 if A is None else A.shape[0]
    if want_dx and dX is None:
        dX = torch.empty(M, w.cols, dtype=torch.bfloat16, device=X.device)
    if r > 0:
        if dA is None:
            dA = torch.empty(r, w.cols, dtype=torch.float32, device=X.device)
        if dB is None:
            dB = torch.empty(w.rows, r, dtype=torch.float32, device=X.device)
    need = qlora_linear_workspace(M, w, r, True)
    wsb = _workspace(need, X.device, ws)
    cw = w.c_struct()
    check(lib().qlora_linear_bwd(_ptr(dY), _ptr(X), M, ctypes.byref(cw), _ptr(A), _ptr(B), r,
                                 float(scale), _ptr(dX) if want_dx else None, _ptr(dA), _ptr(dB),
                                 _ptr(wsb), wsb.numel(), _stream()), "qlora_linear_bwd")
    return dX, dA, dB


def qlora_fused_linear_workspace(M: int, w: NF4Weight, nseg: int, r: int, bwd: bool) -> int:
    cw = w.c_struct()
    return int(lib().qlora_fused_linear_workspace(M, ctypes.byref(cw), nseg, r, int(bwd)))


def qlora_fused_linear_fwd(X: torch.Tensor, w: NF4Weight, nseg: int, A: torch.Tensor | None,
                           B: torch.Tensor | None, scale: float, Y: torch.Tensor | None = None,
                           ws: torch.Tensor | None = None) -> torch.Tensor:
    """Forward of a fused projection: nseg linears stored as the row segments
    of one NF4 weight, sharing X; A [nseg*r, K], B [N, r]."""
    M = X.shape[0]
    r = 0 if A is None else A.shape[0] // nseg
    if Y is None:
        Y = torch.empty(M, w.rows, dtype=torch.bfloat16, device=X.device)
    need = qlora_fused_linear_workspace(M, w, nseg, r, False)
    wsb = _workspace(need, X.device, ws)
    cw = w.c_struct()
    check(lib().qlora_fused_linear_fwd(_ptr(X), M, ctypes.byref(cw), nseg, _ptr(A), _ptr(B), r, float(scale),
                                       _ptr(Y), _ptr(wsb), wsb.numel(), _stream()), "qlora_fused_linear_fwd")
    return Y


def qlora_fused_linear_bwd(dY: torch.Tensor, X: torch.Tensor, w: NF4Weight, nseg: int, A: torch.Tensor | None,
                           B: torch.Tensor | None, scale: float, dX: torch.Tensor | None = None,
                           dA: torch.Tensor | None = None, dB: torch.Tensor | None = None,
                           ws: torch.Tensor | None = None, want_dx: bool = True):
    """(dX, dA, dB) of a fused projection; dX sums every segment's input
    gradient, dA [nseg*r, K] and dB [N, r] hold every adapter's."""
    M = X.shape[0]
    r = 0 if A is None else A.shape[0] // nseg
    if want_dx and dX is None:
        dX = torch.empty(M, w.cols, dtype=torch.bfloat16, device=X.device)
    if r > 0:
        if dA is None:
            dA = torch.empty(nseg * r, w.cols, dtype=torch.float32, device=X.device)
        if dB is None:
            dB = torch.empty(w.rows, r, dtype=torch.float32, device=X.device)
    need = qlora_fused_linear_workspace(M, w, nseg, r, True)
    wsb = _workspace(need, X.device, ws)
    cw = w.c_struct()
    check(lib().qlora_fused_linear_bwd(_ptr(dY), _ptr(X), M, ctypes.byref(cw), nseg, _ptr(A), _ptr(B), r,
                                       float(scale), _ptr(dX) if want_dx else None, _ptr(dA), _ptr(dB),
                                       _ptr(wsb), wsb.numel(), _stream()), "qlora_fused_linear_bwd")
    return dX, dA, dB


def qlora_lora_merge(w: NF4Weight, A: torch.Tensor, B: torch.Tensor, scale: float,
                     out: torch.Tensor | None = None) -> torch.Tensor:
    """W_merged = bf16(dequant(W) + scale B A), the dense bf16 weight with the
    adapter folded in."""
    if out is None:
        out = torch.empty(w.rows, w.cols, dtype=torch.bfloat16, device=w.codes.device)
    cw = w.c_struct()
    check(lib().qlora_lora_merge(ctypes.byref(cw), _ptr(A), _ptr(B), A.shape[0], float(scale), _ptr(out),
                                 _stream()), "qlora_lora_merge")
    return out


def qlora_lora_unmerge(W_merged: torch.Tensor, A: torch.Tensor, B: torch.Tensor, scale: float,
                       out: torch.Tensor | None = None) -> torch.Tensor:
    """bf16(W_merged - scale B A): the base weight back from a merged one."""
    rows, cols = W_merged.shape
    if out is None:
        out = torch.empty(rows, cols, dtype=torch.bfloat16, device=W_merged.device)
    check(lib().qlora_lora_unmerge(_ptr(W_merged), rows, cols, _ptr(A), _ptr(B), A.shape[0], float(scale),
                                   _ptr(out), _stream()), "qlora_lora_unmerge")
    return out


class PagedBuffer:
    """Paged (unified) memory from qlora_paged_alloc for optimizer state:
    reachable from the host and the device through one pointer; its pages
    migrate on demand or on prefetch().  Freed with free() or when the
    object is collected."""

    def __init__(self, nbytes: int):
        p = ctypes.c_void_p()
        check(lib().qlora_paged_alloc(int(nbytes), ctypes.byref(p)), "qlora_paged_alloc")
        self.ptr = p.value or 0
        self.nbytes = int(nbytes)

    def prefetch(self, to_host: bool, stream: torch.cuda.Stream | None = None) -> None:
        check(lib().qlora_paged_prefetch(self.ptr, self.nbytes, int(bool(to_host)), _stream(stream)),
              "qlora_paged_prefetch")

    def host_view(self, dtype=None):
        """NumPy view of the buffer on the host (synchronize the device first)."""
        import numpy as np
        buf = (ctypes.c_uint8 * self.nbytes).from_address(self.ptr)
        return np.frombuffer(buf, dtype=dtype or np.uint8)

    def data_ptr(self) -> int:
        return self.ptr

    def free(self) -> None:
        if self.ptr:
            check(lib().qlora_paged_free(self.ptr), "qlora_paged_free")
            self.ptr = 0

    def __del__(self):
        try:
            self.free()
        except Exception:
            pass


def qlora_adamw_step(param: torch.Tensor, exp_avg, exp_avg_sq, grad: torch.Tensor,
                     param_bf16: torch.Tensor | None = None, *, lr: float, step: int, beta1: float = 0.9,
                     beta2: float = 0.999, eps: float = 1e-8, weight_decay: float = 0.0,
                     grad_scale: float = 1.0) -> None:
    """One AdamW step on fp32 param (in place) with fp32 moments exp_avg,
    exp_avg_sq (tensors or PagedBuffer) and fp32 grad; param_bf16 receives
    the bf16 copy."""
    n = param.numel()
    cfg = CAdamWConfig(lr, beta1, beta2, eps, weight_decay, grad_scale, int(step))
    check(lib().qlora_adamw_step(param.data_ptr(), exp_avg.data_ptr(), exp_avg_sq.data_ptr(), grad.data_ptr(),
                                 _ptr(param_bf16), n, ctypes.byref(cfg), _stream()), "qlora_adamw_step")


def qlora_get_last_error(stream: torch.cuda.Stream | None = None) -> int:
    return int(lib().qlora_get_last_error(_stream(stream)))


def qlora_nf4_table() -> list[float]:
    buf = (ctypes.c_float * 16)()
    lib().qlora_nf4_table(buf)
    return list(buf)


def qlora_nf4_encode(x: torch.Tensor, codes: torch.Tensor | None = None) -> torch.Tensor:
    """Nearest-NF4-code index of every fp32 element of x (one code per byte)."""
    if codes is None:
        codes = torch.empty(x.numel(), dtype=torch.uint8, device=x.device)
    check(lib().qlora_nf4_encode(_ptr(x), x.numel(), _ptr(codes), _stream()), "qlora_nf4_encode")
    return codes


def qlora_dq_encode(y: torch.Tensor, dq_type: str = "int8", codes: torch.Tensor | None = None) -> torch.Tensor:
    """Nearest 8-bit code (double quantization) of every fp32 element of y."""
    if codes is None:
        codes = torch.empty(y.numel(), dtype=torch.uint8, device=y.device)
    check(lib().qlora_dq_encode(_ptr(y), y.numel(), _ptr(codes), DQ_TYPES[dq_type], _stream()), "qlora_dq_encode")
    return codes


def qlora_set_wait_timeout_ns(ns: int) -> None:
    lib().qlora_set_wait_timeout_ns(int(ns))


def qlora_debug_inject(mode: int) -> None:
    lib().qlora_debug_inject(int(mode))


def qlora_kernel_launches() -> int:
    return int(lib().qlora_kernel_launches())


def qlora_profile_enable(on: bool) -> None:
    lib().qlora_profile_enable(int(bool(on)))


def qlora_profile_read(kind: str) -> tuple[float, int]:
    """(summed device ms, launches) recorded for one tracked kernel kind."""
    ms = ctypes.c_double()
    n = ctypes.c_int64()
    check(lib().qlora_profile_read(_lib.KERNEL_KINDS[kind], ctypes.byref(ms), ctypes.byref(n)),
          "qlora_profile_read")
    return ms.value, n.value
