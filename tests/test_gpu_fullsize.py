"""GPU parity against the fp64 CPU oracle at the workloads' own sizes.

The layer shapes of the LLaMA-7B and LLaMA-65B decoder blocks (q/k/v/o,
gate/up, down at 2048 tokens, r = 64), the stress forward (4096 x 4096 with
outliers, 2048 tokens, r = 16), the 22016 x 8192 weight at every token count
of the small-M sweep, and the standalone quantize/dequantize of a 2^30-element
tensor, on the same seeded inputs (same generator indices) that the benchmark
feeds the library.

Quantization outputs are compared bit for bit.  Y and dX are compared on 64
sampled token rows (the first, the last and 62 seeded ones; every row when
M <= 64) and dA, dB in full, at max|d| <= 1e-2 max|ref| and
||d||_F <= 5e-3 ||ref||_F."""
import numpy as np
import pytest
import torch

from bit_nf4_quantized_08_b200 import workloads as wl
from conftest import assert_close_tol

pytestmark = pytest.mark.gpu


def _quantize_both(Q, O, W, dq=True):
    """Quantize on the GPU and in the oracle; check every output bit-exact;
    return the GPU weight and the oracle's dequantized bf16 weight."""
    q = Q.qlora_nf4_quantize(W.cuda(), double_quant=dq)
    torch.cuda.synchronize()
    assert Q.qlora_get_last_error() == 0
    N, K = W.shape
    ref = O.nf4_quantize(wl.bits(W).reshape(-1), double_quant=dq)
    assert np.array_equal(q.codes.cpu().numpy(), ref["codes"]), "codes"
    if dq:
        assert np.array_equal(q.absmax_q8.cpu().numpy(), ref["q8"]), "q8"
        assert np.array_equal(q.absmax_scale.cpu().numpy().view(np.uint32), ref["c1"].view(np.uint32)), "c1"
        assert q.absmax_offset.cpu().numpy().view(np.uint32)[0] == np.float32(ref["offset"]).view(np.uint32)
    else:
        assert np.array_equal(q.absmax.cpu().numpy().view(np.uint32), ref["absmax"].view(np.uint32)), "absmax"
    Wd = O.nf4_dequantize(N * K, ref, double_quant=dq).reshape(N, K)
    return q, Wd


def _check_fwd(Q, O, q, Wd, inp, s, rows, tag):
    X, A, B = inp["X"], inp["A"], inp["B"]
    Y = Q.qlora_linear_fwd(X.cuda(), q, A.cuda(), B.cuda(), s)
    torch.cuda.synchronize()
    assert Q.qlora_get_last_error() == 0
    ref = O.linear_fwd(wl.bits(X), Wd, wl.bits(A), wl.bits(B), s, rows=rows)
    got = Y.float().cpu().numpy()[rows]
    assert_close_tol(got, ref, f"Y {tag}")


def _check_bwd(Q, O, q, Wd, inp, s, rows, tag):
    X, dY, A, B = inp["X"], inp["dY"], inp["A"], inp["B"]
    dX, dA, dB = Q.qlora_linear_bwd(dY.cuda(), X.cuda(), q, A.cuda(), B.cuda(), s)
    torch.cuda.synchronize()
    assert Q.qlora_get_last_error() == 0
    rdX, rdA, rdB = O.linear_bwd(wl.bits(dY), wl.bits(X), Wd, wl.bits(A), wl.bits(B), s, rows=rows)
    assert_close_tol(dX.float().cpu().numpy()[rows], rdX, f"dX {tag}")
    assert_close_tol(dA.cpu().numpy(), rdA, f"dA {tag}")
    assert_close_tol(dB.cpu().numpy(), rdB, f"dB {tag}")


def _block_cases():
    """(config, layer index, name, N, K) of every distinct linear shape of the
    two decoder blocks; the layer index picks the benchmark's generator
    indices (10 per layer)."""
    out = []
    for cfg in ("llama7b", "llama65b"):
        seen = set()
        for li, (name, N, K) in enumerate(wl.CONFIGS[cfg]["linears"]):
            if (N, K) in seen:
                continue
            seen.add((N, K))
            out.append((cfg, li, name, N, K))
    return out


@pytest.mark.parametrize("cfg,li,name,N,K", _block_cases(),
                         ids=[f"{c}-{n}-{N}x{K}" for c, _, n, N, K in _block_cases()])
def test_block_linear_fullsize(Q, O, cuda, cfg, li, name, N, K):
    """One linear of a decoder block at 2048 tokens, r = 64, alpha = 16:
    quantize bit-exact, then forward and backward within tolerance."""
    c = wl.CONFIGS[cfg]
    M, r, s = c["M"], c["r"], c["alpha"] / c["r"]
    base = 10 * li
    W = wl.weight(N, K, seed=0, dtype=torch.bfloat16, index_base=base)
    inp = wl.linear_inputs(M, N, K, r, seed=0, index_base=base)
    q, Wd = _quantize_both(Q, O, W)
    del W
    rows = wl.sample_rows(M, 64, seed=li)
    _check_fwd(Q, O, q, Wd, inp, s, rows, f"{cfg} {name}")
    _check_bwd(Q, O, q, Wd, inp, s, rows, f"{cfg} {name}")


def test_stress_forward_fullsize(Q, O, cuda):
    """Quantizer stress weight (4096 x 4096 bf16 with 0.1 % N(0, 0.5)
    outliers), forward at 2048 tokens, r = 16, alpha = 32."""
    c = wl.CONFIGS["stress"]
    (_, N, K), = c["linears"]
    M, r, s = c["M"], c["r"], c["alpha"] / c["r"]
    W = wl.weight(N, K, seed=0, dtype=torch.bfloat16, outlier_frac=c["outlier_frac"],
                  outlier_std=c["outlier_std"])
    inp = wl.linear_inputs(M, N, K, r, seed=0)
    q, Wd = _quantize_both(Q, O, W)
    _check_fwd(Q, O, q, Wd, inp, s, wl.sample_rows(M, 64, seed=99), "stress")


@pytest.fixture(scope="module")
def sweep_weight(Q, O):
    c = wl.CONFIGS["sweep"]
    (_, N, K), = c["linears"]
    W = wl.weight(N, K, seed=0, dtype=torch.bfloat16)
    q, Wd = _quantize_both(Q, O, W)
    return q, Wd


@pytest.mark.parametrize("M", wl.CONFIGS["sweep"]["Ms"])
def test_small_m_sweep_fullsize(Q, O, cuda, sweep_weight, M):
    """The 22016 x 8192 NF4 weight at every token count of the sweep (the
    small-M kernel), r = 64, alpha = 16: every row of Y."""
    c = wl.CONFIGS["sweep"]
    (_, N, K), = c["linears"]
    r, s = c["r"], c["alpha"] / c["r"]
    q, Wd = sweep_weight
    inp = wl.linear_inputs(M, N, K, r, seed=0)
    _check_fwd(Q, O, q, Wd, inp, s, np.arange(M, dtype=np.int64), f"sweep M={M}")


def test_quantize_dequantize_2e30(Q, O, cuda):
    """Standalone NF4 + double quantization and dequantization of the 2^30
    element bf16 tensor of the sweep (131072 x 8192): codes, 8-bit constants,
    c1, the offset and every dequantized bf16 value equal the oracle's.  At
    this size (65536 groups of 16384 elements) the offset is formed from the
    partial subtree sums of many CTAs."""
    n = wl.CONFIGS["sweep"]["big_numel"]
    W = wl.weight(n // 8192, 8192, seed=0, dtype=torch.bfloat16)
    Wg = W.cuda()
    q = Q.qlora_nf4_quantize(Wg, double_quant=True)
    deq = Q.qlora_nf4_dequantize(q)
    torch.cuda.synchronize()
    assert Q.qlora_get_last_error() == 0
    del Wg
    ref = O.nf4_quantize(wl.bits(W).reshape(-1), double_quant=True)
    del W
    assert np.array_equal(q.codes.cpu().numpy(), ref["codes"]), "codes"
    assert np.array_equal(q.absmax_q8.cpu().numpy(), ref["q8"]), "q8"
    assert np.array_equal(q.absmax_scale.cpu().numpy().view(np.uint32), ref["c1"].view(np.uint32)), "c1"
    assert q.absmax_offset.cpu().numpy().view(np.uint32)[0] == np.float32(ref["offset"]).view(np.uint32)
    ref_deq = O.nf4_dequantize(n, ref)
    got = wl.bits(deq).reshape(-1)
    del deq
    assert np.array_equal(got, ref_deq), "dequantized bf16"


@pytest.mark.parametrize("M,N,K,r", [(2048, 11008, 4096, 64), (1100, 1280, 1024, 32), (16, 4096, 4096, 64),
                                     (3, 1000, 512, 8)])
def test_linear_without_double_quant(Q, O, cuda, M, N, K, r):
    """fp32 block maxima (no double quantization) through the large-M
    (CTA-pair) and small-M kernels: forward and backward."""
    W = wl.weight(N, K, seed=21, dtype=torch.bfloat16)
    inp = wl.linear_inputs(M, N, K, r, seed=21, b_std=0.05)
    q, Wd = _quantize_both(Q, O, W, dq=False)
    rows = wl.sample_rows(M, 64, seed=21)
    _check_fwd(Q, O, q, Wd, inp, 2.0, rows, f"no-DQ M={M}")
    _check_bwd(Q, O, q, Wd, inp, 2.0, rows, f"no-DQ M={M}")
