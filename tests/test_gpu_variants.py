"""GPU parity of the data-type variants (QLoRA paper digest, sec. 6 "Float4
(FP4)" against NFloat4; sec. 4 "c2^FP8" double quantization; block sizes 128
and 256 besides the pages' 64) against the oracle: quantize and dequantize bit
for bit for every combination, and the linear forward / backward, the small-M
forward and the merge within the parity tolerance."""
import itertools

import numpy as np
import pytest
import torch

from bit_nf4_quantized_08_b200 import workloads as wl
from conftest import assert_close_tol
from test_gpu_merge import _assert_rounded_like_oracle

pytestmark = pytest.mark.gpu

FORMATS = list(itertools.product([64, 128, 256], ["nf4", "fp4"], ["int8", "e4m3"]))
FMT_IDS = [f"bs{b}-{c}-{d}" for b, c, d in FORMATS]


def _threshold_tensor(O, code_type):
    """Blocks of absmax 1 whose other values sit on and beside every midpoint
    of the code book (fp32)."""
    t = (O.fp4_table() if code_type == "fp4" else O.nf4_table()).astype(np.float64)
    vals = []
    for j in range(15):
        m = (t[j] + t[j + 1]) / 2
        f = np.float32(m)
        vals += [f, np.nextafter(f, np.float32(2)), np.nextafter(f, np.float32(-2)), np.float32(t[j])]
    vals = np.array(vals, np.float32)
    body = np.tile(vals, -(-255 * 256 // vals.size))[:255 * 256].reshape(255, 256)
    return np.concatenate([np.ones((255, 1), np.float32), body[:, :255]], axis=1)


def _quant_both(Q, O, W, dq, bs, ct, dt):
    q = Q.qlora_nf4_quantize(W.cuda(), double_quant=dq, blocksize=bs, code_type=ct, dq_type=dt)
    deq = Q.qlora_nf4_dequantize(q)
    torch.cuda.synchronize()
    assert Q.qlora_get_last_error() == 0
    host = wl.bits(W).reshape(-1) if W.dtype == torch.bfloat16 else W.numpy().reshape(-1)
    ref = O.nf4_quantize(host, double_quant=dq, blocksize=bs, code_type=ct, dq_type=dt)
    np.testing.assert_array_equal(q.codes.cpu().numpy(), ref["codes"], err_msg="codes")
    if dq:
        np.testing.assert_array_equal(q.absmax_q8.cpu().numpy(), ref["q8"], err_msg="q8")
        np.testing.assert_array_equal(q.absmax_scale.cpu().numpy().view(np.uint32), ref["c1"].view(np.uint32),
                                      err_msg="c1")
        assert q.absmax_offset.cpu().numpy().view(np.uint32)[0] == np.float32(ref["offset"]).view(np.uint32)
    else:
        np.testing.assert_array_equal(q.absmax.cpu().numpy().view(np.uint32), ref["absmax"].view(np.uint32),
                                      err_msg="absmax")
    ref_deq = O.nf4_dequantize(W.numel(), ref, double_quant=dq, blocksize=bs, code_type=ct, dq_type=dt)
    np.testing.assert_array_equal(wl.bits(deq).reshape(-1), ref_deq, err_msg="dequant")
    return q, ref_deq


@pytest.mark.parametrize("bs,ct,dt", FORMATS, ids=FMT_IDS)
def test_variant_quantize_bit_exact(Q, O, cuda, bs, ct, dt):
    W = wl.weight(1024, 4096, seed=70, dtype=torch.bfloat16, outlier_frac=0.001)
    _quant_both(Q, O, W, True, bs, ct, dt)
    if dt == "int8":  # without double quantization the 8-bit code book plays no part
        _quant_both(Q, O, W, False, bs, ct, dt)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_variant_ring_refill_and_tail(Q, O, cuda, dtype):
    """FP4 with blocks of 256 and FP8 double quantization on a tensor with
    more whole 16384-element groups than the quantizer's ring holds per CTA
    (bf16: 6 stages, fp32: 3) and a ragged last group."""
    W = wl.weight(11, 1411587, seed=72, dtype=dtype)  # 947 whole groups + 11809 elements
    _quant_both(Q, O, W, True, 256, "fp4", "e4m3")


@pytest.mark.parametrize("ct", ["nf4", "fp4"])
@pytest.mark.parametrize("bs", [64, 256])
def test_variant_thresholds_and_ragged(Q, O, cuda, ct, bs):
    """Values on and beside every decision midpoint (fp32 input), a ragged
    tensor with a partial last block, and zero blocks."""
    _quant_both(Q, O, torch.from_numpy(_threshold_tensor(O, ct)), True, bs, ct, "e4m3")
    rng = np.random.default_rng(71)
    ragged = rng.normal(0, 0.02, (7, 1000)).astype(np.float32)
    ragged[2, :300] = 0.0
    _quant_both(Q, O, torch.from_numpy(ragged), True, bs, ct, "int8")
    _quant_both(Q, O, torch.from_numpy(ragged), False, bs, ct, "int8")


@pytest.mark.parametrize("bs,ct,dt", [(128, "fp4", "e4m3"), (256, "nf4", "e4m3"), (64, "fp4", "int8"),
                                      (128, "nf4", "int8")])
@pytest.mark.parametrize("M", [300, 16, 40])
def test_variant_linear(Q, O, cuda, bs, ct, dt, M):
    """Forward and backward on each format: the CTA-pair GEMMs (M = 300),
    the warp-MMA small-M kernel (16) and the tcgen05 small-M kernel (40)."""
    N, K, r, s = 768, 1024, 16, 2.0
    W = wl.weight(N, K, seed=72, dtype=torch.bfloat16)
    inp = wl.linear_inputs(M, N, K, r, seed=72, b_std=0.05)
    q, deq = _quant_both(Q, O, W, True, bs, ct, dt)
    Wd = deq.reshape(N, K)
    X, dY, A, B = (inp[k] for k in ("X", "dY", "A", "B"))
    Y = Q.qlora_linear_fwd(X.cuda(), q, A.cuda(), B.cuda(), s)
    dX, dA, dB = Q.qlora_linear_bwd(dY.cuda(), X.cuda(), q, A.cuda(), B.cuda(), s)
    torch.cuda.synchronize()
    assert Q.qlora_get_last_error() == 0
    rows = wl.sample_rows(M, 64, seed=72)
    Xb, dYb, Ab, Bb = (wl.bits(t) for t in (X, dY, A, B))
    assert_close_tol(Y.float().cpu().numpy()[rows], O.linear_fwd(Xb, Wd, Ab, Bb, s, rows=rows), "Y")
    rdX, rdA, rdB = O.linear_bwd(dYb, Xb, Wd, Ab, Bb, s, rows=rows)
    assert_close_tol(dX.float().cpu().numpy()[rows], rdX, "dX")
    assert_close_tol(dA.cpu().numpy(), rdA, "dA")
    assert_close_tol(dB.cpu().numpy(), rdB, "dB")


@pytest.mark.parametrize("bs,ct,dt", [(128, "fp4", "e4m3"), (256, "nf4", "int8")])
def test_variant_merge(Q, O, cuda, bs, ct, dt):
    """Merge on a variant base equals the merge of its dequantized weight (the
    oracle's bf16 weight, then the same one-rounding merge)."""
    N, K, r, s = 512, 768, 16, 1.0
    W = wl.weight(N, K, seed=73, dtype=torch.bfloat16)
    inp = wl.linear_inputs(8, N, K, r, seed=73, b_std=0.05)
    q, deq = _quant_both(Q, O, W, True, bs, ct, dt)
    Wm = Q.qlora_lora_merge(q, inp["A"].cuda(), inp["B"].cuda(), s)
    torch.cuda.synchronize()
    Wd, Ab, Bb = deq.reshape(N, K), wl.bits(inp["A"]), wl.bits(inp["B"])
    ref, exact = O.lora_merge(Wd, Ab, Bb, s, 1, want_exact=True)
    _assert_rounded_like_oracle(wl.bits(Wm), ref, exact, Wd, Ab, Bb, s, r, "merge")
