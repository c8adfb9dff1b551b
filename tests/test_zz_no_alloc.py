"""qlora_nf4_quantize_static (fixed internal scratch, no workspace, no
allocation) against qlora_nf4_quantize on the same inputs: every code, 8-bit
constant and fp32 constant equal, on calls made back to back, up to the
largest accepted size; a larger tensor is refused before anything runs.
Collected last so that it also runs after every other GPU test."""
import ctypes

import pytest
import torch

from bit_nf4_quantized_08_b200 import _lib
from bit_nf4_quantized_08_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _same(a, b, what):
    assert a.rows == b.rows and a.cols == b.cols
    assert torch.equal(a.codes, b.codes), f"{what}: codes differ"
    if a.double_quant:
        assert torch.equal(a.absmax_q8, b.absmax_q8), f"{what}: absmax_q8 differ"
        assert torch.equal(a.absmax_scale.view(torch.int32), b.absmax_scale.view(torch.int32)), \
            f"{what}: absmax_scale differ"
        assert torch.equal(a.absmax_offset.view(torch.int32), b.absmax_offset.view(torch.int32)), \
            f"{what}: absmax_offset differ"
    else:
        assert torch.equal(a.absmax.view(torch.int32), b.absmax.view(torch.int32)), f"{what}: absmax differ"


CASES = [
    # (rows, cols, dtype, double_quant): ragged last group and last block,
    # several groups, fp32 and bf16, and the largest accepted size
    (1001, 640, torch.bfloat16, True),
    (37, 200, torch.float32, True),
    (4096, 4096, torch.bfloat16, True),
    (300, 128, torch.bfloat16, False),
    (8192, 8192, torch.bfloat16, True),
]


def test_static_matches_workspace_entry_point(Q, cuda):
    ref, got = [], []
    for i, (rows, cols, dt, dq) in enumerate(CASES):
        W = wl.weight(rows, cols, seed=40 + i, dtype=dt, device=cuda)
        ref.append(Q.qlora_nf4_quantize(W, double_quant=dq))
        got.append((W, Q.NF4Weight.empty(rows, cols, dq, cuda)))
    torch.cuda.synchronize()
    # back to back on one stream, each reusing the scratch the previous wrote
    before = torch.cuda.memory_allocated(cuda)
    for W, out in got:
        Q.qlora_nf4_quantize_static(W, out)
    assert torch.cuda.memory_allocated(cuda) == before
    torch.cuda.synchronize()
    assert Q.qlora_get_last_error() == 0
    for (rows, cols, dt, dq), r, (_, g) in zip(CASES, ref, got):
        _same(g, r, f"{rows}x{cols} {dt} dq={dq}")


def test_static_two_calls_in_a_row(Q, cuda):
    """The same weight twice, then a different one, then the first again:
    every result equals the workspace entry point's."""
    W1 = wl.weight(2048, 1536, seed=50, dtype=torch.bfloat16, device=cuda)
    W2 = wl.weight(77, 4096, seed=51, dtype=torch.float32, device=cuda, outlier_frac=0.01)
    r1 = Q.qlora_nf4_quantize(W1)
    r2 = Q.qlora_nf4_quantize(W2)
    outs = []
    for W in (W1, W1, W2, W1):
        o = Q.NF4Weight.empty(W.shape[0], W.shape[1], True, cuda)
        Q.qlora_nf4_quantize_static(W, o)
        outs.append(o)
    torch.cuda.synchronize()
    assert Q.qlora_get_last_error() == 0
    for o, r in zip(outs, (r1, r1, r2, r1)):
        _same(o, r, "repeat")


def test_static_refuses_sizes_above_the_limit(Q, cuda):
    """rows*cols one row above the limit: QLORA_ERR_WORKSPACE, nothing enqueued
    (the output pointers only need to be valid and aligned)."""
    L = _lib.lib()
    buf = torch.zeros(1024, dtype=torch.uint8, device=cuda)
    p = buf.data_ptr()
    cols = 8192
    rows = _lib.QLORA_STATIC_QUANTIZE_MAX_ELEMS // cols + 1
    cw = _lib.CNF4Weight(rows, cols, 64, 1, p, p, p, p, p)
    st = L.qlora_nf4_quantize_static(ctypes.c_void_p(p), _lib.QLORA_BF16, ctypes.byref(cw), None)
    assert st == _lib.QLORA_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert int(buf.abs().sum()) == 0
    assert Q.qlora_get_last_error() == 0
