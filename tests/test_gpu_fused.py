"""GPU parity of the fused projection (nseg linears sharing X as row
segments of one NF4 weight, one rank-r adapter per segment; q/k/v and
gate/up of a decoder block) against the oracle, per linear: every segment's
Y, dA and dB, and dX summed over the segments."""
import numpy as np
import pytest
import torch

from bit_nf4_quantized_08_b200 import workloads as wl
from conftest import assert_close_tol

pytestmark = pytest.mark.gpu


def _setup(Q, O, M, nseg, S, K, r, seed, b_std=0.05, dq=True):
    N = nseg * S
    W = wl.weight(N, K, seed=seed, dtype=torch.bfloat16)
    inp = wl.fused_inputs(M, nseg, S, K, r, seed=seed, b_std=b_std)
    q = Q.qlora_nf4_quantize(W.cuda(), double_quant=dq)
    ref_q = O.nf4_quantize(wl.bits(W).reshape(-1), double_quant=dq)
    Wd = O.nf4_dequantize(N * K, ref_q, double_quant=dq).reshape(N, K)
    return q, inp, Wd


def _check(Q, O, q, inp, Wd, nseg, r, s, rows, tag, mode=0):
    X, dY, A, B = (inp[k].cuda() for k in ("X", "dY", "A", "B"))
    Q.qlora_debug_inject(mode)
    try:
        Y = Q.qlora_fused_linear_fwd(X, q, nseg, A, B, s)
        dX, dA, dB = Q.qlora_fused_linear_bwd(dY, X, q, nseg, A, B, s)
        torch.cuda.synchronize()
        assert Q.qlora_get_last_error() == 0
    finally:
        Q.qlora_debug_inject(0)
    Xb, dYb, Ab, Bb = (wl.bits(inp[k]) for k in ("X", "dY", "A", "B"))
    rY = O.fused_linear_fwd(Xb, Wd, Ab, Bb, s, nseg, rows=rows)
    rdX, rdA, rdB = O.fused_linear_bwd(dYb, Xb, Wd, Ab, Bb, s, nseg, rows=rows)
    S = Wd.shape[0] // nseg
    Yc = Y.float().cpu().numpy()[rows]
    for i in range(nseg):
        assert_close_tol(Yc[:, i * S:(i + 1) * S], rY[:, i * S:(i + 1) * S], f"Y seg {i} {tag}")
        assert_close_tol(dA.cpu().numpy()[i * r:(i + 1) * r], rdA[i * r:(i + 1) * r], f"dA seg {i} {tag}")
        assert_close_tol(dB.cpu().numpy()[i * S:(i + 1) * S], rdB[i * S:(i + 1) * S], f"dB seg {i} {tag}")
    assert_close_tol(dX.float().cpu().numpy()[rows], rdX, f"dX {tag}")


@pytest.mark.parametrize("M,nseg,S,K,r", [
    (300, 3, 256, 512, 16),      # r < 64: segments' adapter columns inside one 64-wide load
    (300, 2, 512, 256, 64),
    (129, 3, 256, 192, 8),
    (1100, 2, 768, 1024, 32),
    (16, 3, 1024, 2048, 32),     # small-M kernel
    (7, 2, 512, 1024, 64),
    (64, 4, 256, 512, 64),       # nseg * r = 256
    (2048, 3, 4096, 4096, 64),   # LLaMA-7B q/k/v
    (2048, 2, 11008, 4096, 64),  # LLaMA-7B gate/up
])
def test_fused_projection_parity(Q, O, cuda, M, nseg, S, K, r):
    q, inp, Wd = _setup(Q, O, M, nseg, S, K, r, seed=50 + nseg)
    _check(Q, O, q, inp, Wd, nseg, r, 2.0, wl.sample_rows(M, 64, seed=M), f"M={M} nseg={nseg} S={S} K={K} r={r}")


@pytest.mark.parametrize("mode", [2, 3, 4, 6], ids=["streamk7", "single_cta_grid", "pair_streamk4", "serial_bwd"])
def test_fused_projection_alternate_schedules(Q, O, cuda, mode):
    M, nseg, S, K, r = 600, 3, 256, 512, 16
    q, inp, Wd = _setup(Q, O, M, nseg, S, K, r, seed=60)
    _check(Q, O, q, inp, Wd, nseg, r, 2.0, wl.sample_rows(M, 64, seed=60), f"mode {mode}", mode=mode)


def test_fused_projection_llama65b_qkv(Q, O, cuda):
    """The LLaMA-65B q/k/v projection (3 x 8192 rows, K = 8192) at 2048 tokens."""
    c = wl.FUSED_GROUPS["llama65b"][0]
    _, nseg, S, K = c
    q, inp, Wd = _setup(Q, O, 2048, nseg, S, K, 64, seed=0, b_std=0.01)
    _check(Q, O, q, inp, Wd, nseg, 64, 0.25, wl.sample_rows(2048, 64, seed=0), "65B qkv")


def test_fused_nseg1_is_the_plain_linear(Q, O, cuda):
    M, N, K, r = 300, 512, 256, 16
    q, inp, _ = _setup(Q, O, M, 1, N, K, r, seed=61)
    X, dY, A, B = (inp[k].cuda() for k in ("X", "dY", "A", "B"))
    a = Q.qlora_fused_linear_fwd(X, q, 1, A, B, 2.0)
    b = Q.qlora_linear_fwd(X, q, A, B, 2.0)
    ga = Q.qlora_fused_linear_bwd(dY, X, q, 1, A, B, 2.0)
    gb = Q.qlora_linear_bwd(dY, X, q, A, B, 2.0)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    for x, y in zip(ga, gb):
        assert torch.equal(x.view(torch.int32 if x.dtype == torch.float32 else torch.int16),
                           y.view(torch.int32 if y.dtype == torch.float32 else torch.int16))


def test_fused_rejects_unaligned_segments(Q, cuda):
    W = wl.weight(3 * 200, 256, seed=62, dtype=torch.bfloat16).cuda()
    q = Q.qlora_nf4_quantize(W)
    X = torch.zeros(16, 256, dtype=torch.bfloat16, device="cuda")
    A = torch.zeros(3 * 16, 256, dtype=torch.bfloat16, device="cuda")
    B = torch.zeros(600, 16, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(Q.QloraError) as e:
        Q.qlora_fused_linear_fwd(X, q, 3, A, B, 1.0)
    assert e.value.status == Q.QLORA_ERR_UNSUPPORTED
