"""GPU parity of the NF4 quantizer, double quantization and dequantization
against the CPU oracle: bit-exact on every byte, code and fp32 constant."""
import numpy as np
import pytest
import torch

from bit_nf4_quantized_08_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _edge_tensor(kind: str) -> np.ndarray:
    rng = np.random.default_rng(7)
    if kind == "zero_blocks":
        w = rng.normal(0, 0.02, 64 * 300).astype(np.float32)
        w[64 * 5:64 * 6] = 0.0
        w[64 * 17:64 * 18] = -0.0
        w[64 * 299:] = 0.0
        return w.reshape(300, 64)
    if kind == "subnormal":
        w = rng.normal(0, 0.02, 64 * 40).astype(np.float32)
        w[:64] = (rng.normal(0, 1, 64) * 1e-39).astype(np.float32)      # subnormal block
        w[64:128] = np.float32(1.4e-45) * rng.integers(-3, 4, 64)        # tiny multiples of the min subnormal
        w[128:192] = (rng.normal(0, 1, 64) * 1e-37).astype(np.float32)   # normal but tiny
        return w.reshape(40, 64)
    if kind == "equal_absmax":
        a = np.float32(0.0371)
        w = (rng.uniform(-1, 1, (512, 64)) * a).astype(np.float32)
        w[:, 3] = a
        return w
    if kind == "on_thresholds":
        nf4 = np.array(wl_table(), np.float64)
        mids = (nf4[:-1] + nf4[1:]) / 2
        vals = []
        for m in mids:
            f = np.float32(m)
            vals += [f, np.nextafter(f, np.float32(2)), np.nextafter(f, np.float32(-2))]
        vals = np.array(vals, np.float32)
        reps = int(np.ceil(63 * 200 / vals.size))
        body = np.tile(vals, reps)[:63 * 200].reshape(200, 63)
        w = np.concatenate([np.ones((200, 1), np.float32), body], axis=1)  # absmax 1 per block
        return w.astype(np.float32)
    if kind == "ragged":
        return rng.normal(0, 0.02, (7, 153)).astype(np.float32)  # n = 1071: partial block, odd n
    if kind == "multi_group_partial":
        return rng.normal(0, 0.02, (3, 64 * 256 + 64 * 7 + 32)).astype(np.float32)
    raise KeyError(kind)


def wl_table():
    from oracle import oracle
    return oracle.nf4_table()


def _run_both(Q, O, W: torch.Tensor, dq: bool):
    Wd = W.cuda()
    q = Q.qlora_nf4_quantize(Wd, double_quant=dq)
    deq = Q.qlora_nf4_dequantize(q)
    torch.cuda.synchronize()
    assert Q.qlora_get_last_error() == 0
    if W.dtype == torch.bfloat16:
        host = wl.bits(W).reshape(-1)
    else:
        host = W.numpy().reshape(-1)
    ref = O.nf4_quantize(host, double_quant=dq)
    n = W.numel()
    ref_deq = O.nf4_dequantize(n, ref, double_quant=dq)
    np.testing.assert_array_equal(q.codes.cpu().numpy(), ref["codes"], err_msg="codes")
    if dq:
        np.testing.assert_array_equal(q.absmax_q8.cpu().numpy(), ref["q8"], err_msg="q8")
        np.testing.assert_array_equal(q.absmax_scale.cpu().numpy().view(np.uint32),
                                      ref["c1"].view(np.uint32), err_msg="c1")
        got_off = q.absmax_offset.cpu().numpy().view(np.uint32)[0]
        assert got_off == np.float32(ref["offset"]).view(np.uint32), "offset"
    else:
        np.testing.assert_array_equal(q.absmax.cpu().numpy().view(np.uint32),
                                      ref["absmax"].view(np.uint32), err_msg="absmax")
    np.testing.assert_array_equal(wl.bits(deq).reshape(-1), ref_deq, err_msg="dequant")
    return q, ref


@pytest.mark.parametrize("dq", [True, False])
def test_tiny_fp32(Q, O, cuda, dq):
    W = wl.weight(256, 256, seed=0, dtype=torch.float32)
    _run_both(Q, O, W, dq)


@pytest.mark.parametrize("dq", [True, False])
def test_stress_outliers_bf16(Q, O, cuda, dq):
    c = wl.CONFIGS["stress"]
    W = wl.weight(4096, 4096, seed=0, dtype=torch.bfloat16, outlier_frac=c["outlier_frac"],
                  outlier_std=c["outlier_std"])
    _run_both(Q, O, W, dq)


@pytest.mark.parametrize("kind", ["zero_blocks", "subnormal", "equal_absmax", "on_thresholds",
                                  "ragged", "multi_group_partial"])
@pytest.mark.parametrize("dq", [True, False])
def test_edge_cases(Q, O, cuda, kind, dq):
    W = torch.from_numpy(_edge_tensor(kind))
    _run_both(Q, O, W, dq)
    _run_both(Q, O, W.to(torch.bfloat16), dq)


@pytest.mark.parametrize("dq", [True, False])
def test_persistent_ragged_tail_bf16(Q, O, cuda, dq):
    """More 16384-element groups than resident CTAs (592 on 148 SMs) and a
    ragged last group: a CTA that codes a whole group loads the partial last
    group as its next one (n = 11469717 = 700 whole groups + 917 elements,
    an odd tail inside a block)."""
    W = wl.weight(7, 1638531, seed=5, dtype=torch.bfloat16)
    _run_both(Q, O, W, dq)


@pytest.mark.parametrize("dq", [True, False])
def test_persistent_ring_fp32(Q, O, cuda, dq):
    """fp32 input (three 64 KB ring stages of two TMA boxes each) with more
    than three whole groups per CTA, so every stage is refilled, and a
    ragged last group (n = 9831419 = 600 whole groups + 1019 elements)."""
    W = wl.weight(13, 756263, seed=6, dtype=torch.float32)
    _run_both(Q, O, W, dq)


def test_equal_absmax_is_lossless(Q, O, cuda):
    W = torch.from_numpy(_edge_tensor("equal_absmax"))
    q_dq, _ = _run_both(Q, O, W, True)
    q_nodq, _ = _run_both(Q, O, W, False)
    a = Q.qlora_nf4_dequantize(q_dq)
    b = Q.qlora_nf4_dequantize(q_nodq)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert float(q_dq.absmax_scale.abs().max()) == 0.0


def test_empty(Q, cuda):
    W = torch.empty(0, 64, device="cuda", dtype=torch.bfloat16)
    q = Q.qlora_nf4_quantize(W)
    assert q.codes.numel() == 0
    assert Q.qlora_get_last_error() == 0


def test_determinism(Q, cuda):
    W = wl.weight(1024, 4096, seed=3, dtype=torch.bfloat16, device="cuda")
    a = Q.qlora_nf4_quantize(W)
    b = Q.qlora_nf4_quantize(W)
    for x, y in [(a.codes, b.codes), (a.absmax_q8, b.absmax_q8), (a.absmax_scale, b.absmax_scale),
                 (a.absmax_offset, b.absmax_offset)]:
        assert torch.equal(x, y)


def test_encode_exhaustive(Q, O, cuda):
    """The fast nearest-code search equals the oracle's brute-force argmin on
    every fp32 value in [-1.0001, 1.0001] (both signs, zeros and subnormals)."""
    hi = int(np.float32(1.0001).view(np.uint32))
    chunk = 1 << 26
    for sign in (0, 0x80000000):
        start = 0
        while start <= hi:
            n = min(chunk, hi + 1 - start)
            first = sign | start
            xb = torch.arange(first, first + n, dtype=torch.int64, device="cuda").to(torch.int32)
            x = xb.view(torch.float32)
            got = Q.qlora_nf4_encode(x)
            exp = torch.from_numpy(O.nf4_nearest_bits(first, n)).to("cuda")
            bad = int((got != exp).sum())
            assert bad == 0, f"{bad} mismatches in chunk starting at {first:#x}"
            start += n


@pytest.mark.parametrize("shape", [(4096, 4096), (37, 200), (1, 16384 * 3 + 64), (4096, 8192)])
def test_separate_offset_kernel_matches(Q, O, cuda, shape):
    """The double-quantization offset formed by the 8-bit pass itself and by
    its own kernel (test mode 5) are the same fp32 value, and both match the
    oracle."""
    W = wl.weight(shape[0], shape[1], seed=11, dtype=torch.bfloat16)
    q_fused, ref = _run_both(Q, O, W, True)
    Q.qlora_debug_inject(5)
    try:
        q_sep = Q.qlora_nf4_quantize(W.cuda(), double_quant=True)
        torch.cuda.synchronize()
        assert Q.qlora_get_last_error() == 0
    finally:
        Q.qlora_debug_inject(0)
    for x, y in [(q_fused.codes, q_sep.codes), (q_fused.absmax_q8, q_sep.absmax_q8),
                 (q_fused.absmax_scale.view(torch.int32), q_sep.absmax_scale.view(torch.int32)),
                 (q_fused.absmax_offset.view(torch.int32), q_sep.absmax_offset.view(torch.int32))]:
        assert torch.equal(x, y)


@pytest.mark.parametrize("shape", [(16384, 16384), (9000, 16384)])
def test_partial_offset_tree_matches_single_cta(Q, cuda, shape):
    """More than 8192 group sums: the offset from aligned 4096-leaf partial
    subtrees (many CTAs) and from the one-CTA tree over all sums (test mode 5)
    are the same fp32 value (same pairwise tree), so every output is equal."""
    W = wl.weight(shape[0], shape[1], seed=12, dtype=torch.bfloat16, device="cuda")
    q_part = Q.qlora_nf4_quantize(W, double_quant=True)
    torch.cuda.synchronize()
    assert Q.qlora_get_last_error() == 0
    Q.qlora_debug_inject(5)
    try:
        q_one = Q.qlora_nf4_quantize(W, double_quant=True)
        torch.cuda.synchronize()
        assert Q.qlora_get_last_error() == 0
    finally:
        Q.qlora_debug_inject(0)
    for x, y in [(q_part.codes, q_one.codes), (q_part.absmax_q8, q_one.absmax_q8),
                 (q_part.absmax_scale.view(torch.int32), q_one.absmax_scale.view(torch.int32)),
                 (q_part.absmax_offset.view(torch.int32), q_one.absmax_offset.view(torch.int32))]:
        assert torch.equal(x, y)


def test_dq_encode_exhaustive_int8(Q, O, cuda):
    """The 8-bit search of the double quantization (fp32 thresholds around the
    rint candidate) equals the oracle's brute-force argmin over the 255-entry
    code book on every fp32 value in [-1, 1] (both signs, zeros, subnormals)."""
    hi = int(np.float32(1.0).view(np.uint32))
    chunk = 1 << 26
    for sign in (0, 0x80000000):
        start = 0
        while start <= hi:
            n = min(chunk, hi + 1 - start)
            first = sign | start
            y = torch.arange(first, first + n, dtype=torch.int64, device="cuda").to(torch.int32).view(torch.float32)
            got = Q.qlora_dq_encode(y, "int8")
            exp = torch.from_numpy(O.dq_nearest_bits(first, n, "int8")).to("cuda")
            bad = int((got != exp).sum())
            assert bad == 0, f"{bad} mismatches in chunk starting at {first:#x}"
            start += n


def test_dq_encode_e4m3_near_every_midpoint(Q, O, cuda):
    """The FP8 (E4M3) search equals the oracle's brute force on every fp32
    within 2^16 units in the last place of each of the 252 midpoints of the
    code book, and on 2^24 spread values of [-1, 1]."""
    t = O.e4m3_table().astype(np.float64)
    mids = np.float32((t[:-1] + t[1:]) / 2).view(np.uint32)
    for m in mids.tolist():
        first = max(0, (m & 0x7FFFFFFF) - (1 << 16)) | (m & 0x80000000)
        n = 1 << 17
        y = torch.arange(first, first + n, dtype=torch.int64, device="cuda").to(torch.int32).view(torch.float32)
        got = Q.qlora_dq_encode(y, "e4m3").cpu().numpy()
        exp = O.dq_nearest_bits(first, n, "e4m3")
        assert np.array_equal(got, exp), f"mismatch near midpoint bits {m:#x}"
    hi = int(np.float32(1.0).view(np.uint32))
    stride = hi // (1 << 23)
    for sign in (0, 0x80000000):
        bits = (np.arange(1 << 23, dtype=np.uint64) * stride).astype(np.uint32) | np.uint32(sign)
        y = torch.from_numpy(bits.view(np.float32)).cuda()
        got = Q.qlora_dq_encode(y, "e4m3").cpu().numpy()
        exp = np.concatenate([O.dq_nearest_bits(int(b), 1, "e4m3") for b in bits[:: 1 << 12]])
        assert np.array_equal(got[:: 1 << 12], exp)
