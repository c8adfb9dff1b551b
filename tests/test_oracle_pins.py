"""Pins of the CPU oracle to things other than itself: library routines,
brute force, closed forms and invariants the pages fix, and hand-worked
examples under tests/golden/.  CPU only."""
import math
import os
import statistics
from fractions import Fraction

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _f32bits(a):
    return np.asarray(a, np.float32).view(np.uint32)


# ---------------------------------------------------------------------------
# NF4 code book
# ---------------------------------------------------------------------------

def _library_table(ppf):
    """The code-book reading built from a library quantile function."""
    d = 0.5 * (1 / 32 + 1 / 30)
    pos = [ppf(p) for p in np.linspace(0.5, 1 - d, 9)[1:]]
    neg = [ppf(p) for p in np.linspace(d, 0.5, 8)[:-1]]
    return np.array([x / -ppf(d) for x in neg] + [0.0] + [x / ppf(1 - d) for x in pos]).astype(np.float32)


def test_nf4_table_invariants(O):
    """Spec invariants: 16 sorted distinct values, min -1, max +1, an
    exact zero (digest sec. 4: asymmetric so 0 is exact)."""
    t = O.nf4_table()
    assert t.shape == (16,)
    assert np.all(np.diff(t) > 0)
    assert t[0] == -1.0 and t[-1] == 1.0
    assert np.count_nonzero(t == 0.0) == 1 and t[7] == 0.0
    assert np.count_nonzero(t < 0) == 7 and np.count_nonzero(t > 0) == 8


def test_nf4_table_matches_library_quantiles(O):
    """The oracle's own bisection on erfc reproduces the fp32 code book that
    SciPy's ndtri and Python's NormalDist.inv_cdf give, bit for bit."""
    from scipy.special import ndtri
    t = O.nf4_table()
    np.testing.assert_array_equal(_f32bits(t), _f32bits(_library_table(lambda p: float(ndtri(p)))))
    np.testing.assert_array_equal(_f32bits(t), _f32bits(_library_table(statistics.NormalDist().inv_cdf)))


@pytest.mark.parametrize("p", [1e-6, 0.0322917, 0.1, 0.3, 0.5, 0.7, 0.9677083, 0.999999])
def test_normal_quantile_vs_scipy(O, p):
    from scipy.special import ndtri
    q = O.normal_quantile(p)
    ref = float(ndtri(p))
    assert abs(q - ref) <= 1e-13 * max(1.0, abs(ref))


def test_nf4_codes_are_quantile_midpoint_like(O):
    """Each positive code lies between the two normal quantiles whose
    probability bins it represents (digest quantile equation: a code is the
    middle of its bin), after normalization."""
    from scipy.special import ndtri
    t = O.nf4_table().astype(np.float64)
    d = 0.5 * (1 / 32 + 1 / 30)
    qmax = ndtri(1 - d)
    # codes are increasing quantiles of equally spaced probabilities
    p = np.array([0.5 + i * (0.5 - d) / 8 for i in range(1, 9)])
    np.testing.assert_allclose(t[8:] * qmax, ndtri(p), rtol=1e-6)


# ---------------------------------------------------------------------------
# nearest-code search
# ---------------------------------------------------------------------------

def test_nearest_exhaustive_vs_exact_midpoints(O):
    """Brute-force argmin (oracle) equals the count of exact midpoints
    strictly below x (ties to the lower index) for EVERY fp32 x in
    [-1.0001, 1.0001]."""
    t = O.nf4_table().astype(np.float64)
    mids = (t[:-1] + t[1:]) / 2  # exact in fp64
    hi = int(np.float32(1.0001).view(np.uint32))
    chunk = 1 << 26
    for sign in (0, 0x80000000):
        start = 0
        while start <= hi:
            n = min(chunk, hi + 1 - start)
            first = sign | start
            got = O.nf4_nearest_bits(first, n)
            x = (np.arange(n, dtype=np.uint64) + first).astype(np.uint32).view(np.float32).astype(np.float64)
            exp = np.searchsorted(mids, x, side="left").astype(np.uint8)
            bad = np.flatnonzero(got != exp)
            assert bad.size == 0, f"mismatch at bits {first + int(bad[0]):#x}"
            start += n


def test_nearest_ties_go_low(O):
    t = O.nf4_table().astype(np.float64)
    for j in range(15):
        m = (t[j] + t[j + 1]) / 2
        f = np.float32(m)
        if float(f) == m:  # representable midpoint: an exact tie
            assert O.nf4_nearest(float(f)) == j


def test_t8_table(O):
    """8-bit constant code book: 255 symmetric levels k/127, exact 0 in the
    middle, ends at -1 and +1 (reading of the digest's 8-bit c2)."""
    t8 = O.t8_table().astype(np.float64)
    assert t8.shape == (255,)
    assert t8[0] == -1 and t8[127] == 0 and t8[254] == 1
    np.testing.assert_array_equal(t8, -t8[::-1])
    np.testing.assert_allclose(np.diff(t8), 1 / 127, rtol=0, atol=1.2e-7)  # fp32 rounding of each level


# ---------------------------------------------------------------------------
# quantize / dequantize
# ---------------------------------------------------------------------------

def _read_golden(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, *v = line.split()
            out[k] = v
    return out


def test_packing_golden(O):
    g = _read_golden("nf4_packing_example.txt")
    a = np.float32(g["absmax"][0])
    idx = [int(x) for x in g["indices"]]
    t = O.nf4_table()
    w = np.zeros(64, np.float32)
    w[:4] = [t[i] * a for i in idx]
    q = O.nf4_quantize(w, double_quant=False)
    assert q["absmax"][0] == a
    np.testing.assert_array_equal(q["codes"], np.array([int(b, 16) for b in g["bytes"]], np.uint8))


def test_roundtrip_lossless_without_dq(O):
    """Spec invariant: a block whose elements are exactly table values
    times its absmax (with at least one +-absmax) round-trips losslessly."""
    rng = np.random.default_rng(0)
    t = O.nf4_table()
    nb = 300
    idx = rng.integers(0, 16, (nb, 64))
    idx[:, 5] = 15
    a = rng.uniform(1e-3, 3.0, nb).astype(np.float32)
    w = (t[idx] * a[:, None]).astype(np.float32)
    q = O.nf4_quantize(w.reshape(-1), double_quant=False)
    np.testing.assert_array_equal(q["absmax"], a)
    codes = np.empty(nb * 64, np.uint8)
    codes[0::2] = q["codes"] >> 4
    codes[1::2] = q["codes"] & 15
    np.testing.assert_array_equal(codes, idx.reshape(-1))
    deq = O.nf4_dequantize(w.size, q, double_quant=False)
    # torch's own fp32 -> bf16 rounding of the exact input values
    ref = torch.from_numpy(w.reshape(-1)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(deq, ref)


def test_equal_absmax_dq_is_lossless(O):
    """With every block sharing one absmax, offset = absmax exactly, c1 = 0,
    q8 = 127, and double quantization loses nothing."""
    rng = np.random.default_rng(1)
    a = np.float32(0.0371)
    w = (rng.uniform(-1, 1, (1000, 64)) * a).astype(np.float32)
    w[:, 9] = -a
    q = O.nf4_quantize(w.reshape(-1), double_quant=True)
    assert np.float32(q["offset"]) == a
    assert np.all(q["c1"] == 0) and np.all(q["q8"] == 127)
    d1 = O.nf4_dequantize(w.size, q, double_quant=True)
    q0 = O.nf4_quantize(w.reshape(-1), double_quant=False)
    d0 = O.nf4_dequantize(w.size, q0, double_quant=False)
    np.testing.assert_array_equal(d1, d0)


def test_zero_and_partial_blocks(O):
    w = np.zeros(64 * 3 + 5, np.float32)
    w[64:128] = np.linspace(-1, 1, 64)
    w[-5:] = [0.1, -0.2, 0.0, 0.3, -0.4]
    q = O.nf4_quantize(w, double_quant=False)
    assert q["codes"].size == (w.size + 1) // 2 and q["absmax"].size == 4
    assert np.all(q["codes"][:32] == 0x77) and q["absmax"][0] == 0
    assert q["absmax"][3] == np.float32(0.4)
    assert q["codes"][-1] & 15 == 0  # padding nibble of the odd tail
    deq = O.nf4_dequantize(w.size, q, double_quant=False)
    assert np.all(deq[:64] == 0)
    empty = O.nf4_quantize(np.zeros(0, np.float32))
    assert empty["codes"].size == 0


def test_error_bound(O):
    """|x - nf4[code]| is at most the largest half-gap of the code book."""
    rng = np.random.default_rng(2)
    w = rng.normal(0, 0.02, 64 * 2000).astype(np.float32)
    q = O.nf4_quantize(w, double_quant=False)
    deq = O.nf4_dequantize(w.size, q, double_quant=False)
    d = torch.from_numpy(deq.view(np.int16)).view(torch.bfloat16).float().numpy()
    t = O.nf4_table().astype(np.float64)
    half_gap = np.max(np.diff(t)) / 2
    a = np.repeat(q["absmax"].astype(np.float64), 64)
    assert np.all(np.abs(w - d) <= half_gap * a + np.abs(d) * 2.0 ** -8 + 1e-12)


def test_dq_offset_is_mean(O):
    """offset = fl32(mean(absmax)); for these inputs the fp64 tree sum is exact,
    so it equals the correctly rounded sum (math.fsum)."""
    rng = np.random.default_rng(3)
    w = rng.normal(0, 0.02, 64 * 5000 + 17).astype(np.float32)
    q = O.nf4_quantize(w, double_quant=True)
    nb = q["absmax"].size
    mean = math.fsum(q["absmax"].astype(np.float64).tolist()) / nb
    assert np.float32(q["offset"]) == np.float32(mean)


def test_dq_constant_error_bound(O):
    """|a - a'| <= c1/254 plus rounding, per 256-block group."""
    rng = np.random.default_rng(4)
    w = rng.normal(0, 0.02, 64 * 3000).astype(np.float32)
    q = O.nf4_quantize(w, double_quant=True)
    t8 = O.t8_table().astype(np.float64)
    a = q["absmax"].astype(np.float64)
    c1 = np.repeat(q["c1"].astype(np.float64), 256)[:a.size]
    a2 = t8[q["q8"]] * c1 + q["offset"]
    assert np.all(np.abs(a - a2) <= c1 / 254 * (1 + 1e-6) + 4 * np.finfo(np.float32).eps * np.abs(a))


def test_q8_nearest_exact_rationals(O):
    """The 8-bit code picked for each centred constant is the nearest level in
    exact rational arithmetic (ties to the lower index)."""
    rng = np.random.default_rng(5)
    w = rng.normal(0, 0.02, 64 * 256 * 4).astype(np.float32)
    w[: 64 * 30] *= 5.0
    q = O.nf4_quantize(w, double_quant=True)
    t8 = [Fraction(float(v)) for v in O.t8_table()]
    off = np.float32(q["offset"])
    for b in range(0, q["absmax"].size, 7):
        d = np.float32(q["absmax"][b] - off)
        c = np.float32(q["c1"][b // 256])
        y = np.float32(d * np.float32(np.float32(1) / c))
        fy = Fraction(float(y))
        dist = [abs(fy - v) for v in t8]
        best = min(range(255), key=lambda k: (dist[k], k))
        assert q["q8"][b] == best


def test_dq_bits_per_param(O):
    """Constant overhead with double quantization: 8/64 + 32/(64*256) bits per
    parameter (digest sec. 4), from this layout's actual byte counts."""
    g = _read_golden("pages_closed_forms.txt")
    n = 64 * 256 * 64
    w = np.random.default_rng(6).normal(0, 0.02, n).astype(np.float32)
    q = O.nf4_quantize(w, double_quant=True)
    const_bits = (q["q8"].nbytes + q["c1"].nbytes) * 8 / n
    assert abs(const_bits - float(g["dq_const_bits_per_param"][0])) <= float(g["dq_const_bits_per_param"][1])
    assert const_bits == 8 / 64 + 32 / (64 * 256)
    q0 = O.nf4_quantize(w, double_quant=False)
    nodq = q0["absmax"].nbytes * 8 / n
    assert nodq == float(g["nodq_const_bits_per_param"][0])
    assert abs((nodq - const_bits) - float(g["dq_saving_bits_per_param"][0])) <= float(g["dq_saving_bits_per_param"][1])
    assert q["codes"].nbytes * 8 / n == 4


def test_memory_closed_forms(O):
    """Tutorial 11.3 memory figures for a 70B model from this layout."""
    g = _read_golden("pages_closed_forms.txt")
    n = 70e9
    weights_gb = n * 0.5 / 1e9
    consts_gb = n / 64 * 4 / 1e9
    dq_consts_gb = n * (8 / 64 + 32 / (64 * 256)) / 8 / 1e9
    for key, val in (("weights_70b_gb", weights_gb), ("consts_70b_gb", consts_gb),
                     ("dq_saving_70b_gb", consts_gb - dq_consts_gb)):
        ref, tol = float(g[key][0]), float(g[key][1])
        assert abs(val - ref) <= tol, (key, val)


# ---------------------------------------------------------------------------
# linear forward / backward
# ---------------------------------------------------------------------------

def _bf16(rng, shape, std):
    t = torch.from_numpy((rng.normal(0, std, shape)).astype(np.float32)).to(torch.bfloat16)
    return t, t.view(torch.int16).numpy().view(np.uint16)


def _case(seed=0, M=16, N=48, K=64, r=8):
    rng = np.random.default_rng(seed)
    X, Xb = _bf16(rng, (M, K), 1.0)
    W, Wb = _bf16(rng, (N, K), 0.02)
    A, Ab = _bf16(rng, (r, K), 1.0 / r)
    B, Bb = _bf16(rng, (N, r), 0.05)
    dY, dYb = _bf16(rng, (M, N), 1.0)
    return (X, W, A, B, dY), (Xb, Wb, Ab, Bb, dYb)


def test_fwd_vs_torch_linear(O):
    """Forward = F.linear(x, W0) + s * F.linear(F.linear(x, A), B), the
    loralib composition the reproduction blog describes, in fp64."""
    (X, W, A, B, _), (Xb, Wb, Ab, Bb, _) = _case(0, M=37, N=72, K=128, r=16)
    s = 2.0
    Y = O.linear_fwd(Xb, Wb, Ab, Bb, s)
    F = torch.nn.functional
    x, w, a, b = (t.double() for t in (X, W, A, B))
    ref = F.linear(x, w) + s * F.linear(F.linear(x, a), b)
    np.testing.assert_allclose(Y, ref.numpy(), rtol=1e-12, atol=1e-12)
    rows = np.array([0, 5, 36], np.int64)
    np.testing.assert_allclose(O.linear_fwd(Xb, Wb, Ab, Bb, s, rows=rows), ref.numpy()[rows], rtol=1e-12, atol=1e-12)


def test_bwd_vs_autograd(O):
    """dX, dA, dB equal torch.autograd's gradients of sum(Y * dY) in fp64; the
    frozen weight takes no gradient."""
    (X, W, A, B, dY), (Xb, Wb, Ab, Bb, dYb) = _case(1, M=29, N=40, K=192, r=8)
    s = 0.25
    x = X.double().requires_grad_(True)
    a = A.double().requires_grad_(True)
    b = B.double().requires_grad_(True)
    w = W.double()  # frozen
    F = torch.nn.functional
    y = F.linear(x, w) + s * F.linear(F.linear(x, a), b)
    (y * dY.double()).sum().backward()
    assert w.grad is None
    dX, dA, dB = O.linear_bwd(dYb, Xb, Wb, Ab, Bb, s)
    np.testing.assert_allclose(dX, x.grad.numpy(), rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(dA, a.grad.numpy(), rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(dB, b.grad.numpy(), rtol=1e-11, atol=1e-11)
    rows = np.array([3, 28], np.int64)
    dXr, _, _ = O.linear_bwd(dYb, Xb, Wb, Ab, Bb, s, rows=rows)
    np.testing.assert_allclose(dXr, x.grad.numpy()[rows], rtol=1e-11, atol=1e-11)


def test_bwd_finite_differences(O):
    """Central finite differences of L = sum(Y * dY) on the tiny shape
    (d = 256, M = 16), using the oracle's own forward."""
    rng = np.random.default_rng(2)
    M, N, K, r, s = 16, 256, 256, 8, 2.0
    Xf = rng.normal(0, 1, (M, K))
    Wb = torch.from_numpy(rng.normal(0, 0.02, (N, K)).astype(np.float32)).to(torch.bfloat16)
    Ab = torch.from_numpy(rng.normal(0, 1 / r, (r, K)).astype(np.float32)).to(torch.bfloat16)
    Bb = torch.from_numpy(rng.normal(0, 0.05, (N, r)).astype(np.float32)).to(torch.bfloat16)
    dYb = torch.from_numpy(rng.normal(0, 1, (M, N)).astype(np.float32)).to(torch.bfloat16)
    bits = lambda t: t.view(torch.int16).numpy().view(np.uint16)
    Xb = torch.from_numpy(Xf.astype(np.float32)).to(torch.bfloat16)
    dX, dA, dB = O.linear_bwd(bits(dYb), bits(Xb), bits(Wb), bits(Ab), bits(Bb), s)
    # the loss is linear in each of X, A, B separately, so a central
    # difference over the applied step is exact up to fp64 rounding
    dy = dYb.double().numpy()

    def loss(Xv, Av, Bv):
        Y = O.linear_fwd(bits(Xv), bits(Wb), bits(Av), bits(Bv), s)
        return float(np.sum(Y * dy))

    h = 2.0 ** -4
    for (which, i, j) in [("A", 0, 3), ("A", 7, 200), ("B", 5, 1), ("B", 255, 7), ("X", 0, 0), ("X", 15, 255)]:
        T = {"A": Ab, "B": Bb, "X": Xb}[which].clone()
        base = float(T[i, j])
        Tp, Tm = T.clone(), T.clone()
        Tp[i, j] = base + h
        Tm[i, j] = base - h
        step = float(Tp[i, j]) - float(Tm[i, j])  # the bf16-rounded perturbation actually applied
        assert step > 0
        args_p = {"A": (Xb, Tp, Bb), "B": (Xb, Ab, Tp), "X": (Tp, Ab, Bb)}[which]
        args_m = {"A": (Xb, Tm, Bb), "B": (Xb, Ab, Tm), "X": (Tm, Ab, Bb)}[which]
        fd = (loss(*args_p) - loss(*args_m)) / step
        an = {"A": dA, "B": dB, "X": dX}[which][i, j]
        assert abs(fd - an) <= 1e-9 * max(1.0, abs(an)), (which, i, j, fd, an)


def test_zero_B_noop_and_zero_dA(O):
    """Reproduction blog: with B = 0 at step 0 the output equals the frozen
    base path; then G = dY B = 0, so dA = 0 while dB is not."""
    (X, W, A, B, dY), (Xb, Wb, Ab, Bb, dYb) = _case(3, M=20, N=64, K=128, r=8)
    B0 = np.zeros_like(Bb)
    y0 = O.linear_fwd(Xb, Wb, Ab, B0, 2.0)
    base = O.linear_fwd(Xb, Wb, np.zeros((0, 128), np.uint16), np.zeros((64, 0), np.uint16), 2.0)
    np.testing.assert_array_equal(y0, base)
    np.testing.assert_allclose(base, torch.nn.functional.linear(X.double(), W.double()).numpy(), rtol=1e-12, atol=1e-12)
    _, dA, dB = O.linear_bwd(dYb, Xb, Wb, Ab, B0, 2.0)
    assert np.all(dA == 0) and np.any(dB != 0)


def test_lora_parameter_count():
    """Reproduction blog invariant: adapter parameters = r (d_in + d_out);
    the worked example is 8 * (4096 + 4096) = 65536 against ~16.77M."""
    from bit_nf4_quantized_08_b200 import workloads as wl
    g = _read_golden("pages_closed_forms.txt")
    inp = wl.linear_inputs(2, 4096, 4096, 8)
    assert inp["A"].numel() + inp["B"].numel() == int(g["lora_params_4096_r8"][0])
    assert 4096 * 4096 == int(g["full_params_4096"][0])


def test_no_dw_output(O):
    """The frozen weight's gradient is empty: the backward returns exactly
    (dX, dA, dB) and nothing of W's shape."""
    (X, W, A, B, dY), (Xb, Wb, Ab, Bb, dYb) = _case(4)
    out = O.linear_bwd(dYb, Xb, Wb, Ab, Bb, 1.0)
    assert len(out) == 3
    assert [o.shape for o in out] == [Xb.shape, Ab.shape, Bb.shape]


def test_q8_ties_go_low(O):
    """At an exactly representable midpoint between two 8-bit levels the
    lower index wins (the tie reading shared with the NF4 search)."""
    t8 = O.t8_table().astype(np.float64)
    checked = 0
    for k in range(254):
        m = (t8[k] + t8[k + 1]) / 2
        if float(np.float32(m)) == m:
            assert O.t8_nearest(float(m)) == k
            assert O.t8_nearest(float(np.nextafter(np.float32(m), np.float32(2)))) == k + 1
            checked += 1
    assert checked > 100


# ---------------------------------------------------------------------------
# LoRA merge / unmerge
# ---------------------------------------------------------------------------

def _bf16_value(h: int) -> Fraction:
    """Exact value of a finite bf16 code."""
    return Fraction(float(np.array([h << 16], np.uint32).view(np.float32)[0]))


def _bf16_nearest_even(x: Fraction) -> int:
    """Brute force: the finite bf16 code nearest to the exact rational x, ties
    to the code with an even last bit (positive codes enumerated; the sign is
    symmetric)."""
    neg = x < 0
    ax = -x if neg else x
    best, bd = None, None
    # candidates: every positive finite code (0x0000 .. 0x7F7F); the search
    # narrows to the two around ax through the order of the codes
    lo, hi = 0, 0x7F7F
    while hi - lo > 1:
        mid = (lo + hi) // 2
        if _bf16_value(mid) <= ax:
            lo = mid
        else:
            hi = mid
    for h in (lo, hi):
        d = abs(_bf16_value(h) - ax)
        if bd is None or d < bd or (d == bd and h % 2 == 0):
            best, bd = h, d
    return best | (0x8000 if neg and best != 0 else 0)


def _bits_of(vals):
    return (np.asarray(vals, np.float32).view(np.uint32) >> 16).astype(np.uint16)


def test_lora_merge_brute_force(O):
    """Merge and unmerge against exact rational arithmetic: every output is
    the bf16 code nearest to W + sign s sum_j B A (ties to even), on random
    bf16 inputs plus constructed exact ties (normal and subnormal)."""
    rng = np.random.default_rng(5)
    N, K, r = 6, 64, 8
    W = _bits_of(rng.normal(0, 0.02, (N, K)))
    A = _bits_of(rng.normal(0, 1 / r, (r, K)))
    B = _bits_of(rng.normal(0, 0.05, (N, r)))
    # row 0: exact ties (s = 2).  W = 1.0 and 1.0078125 with s B A = 2^-8,
    # half a unit in the last place of both; W = 0 with s B A = 1.5 * 2^-133,
    # halfway between the two smallest subnormals
    # (row 1 carries the subnormal case, so that its tiny B entry meets no
    # other term that would land on a midpoint)
    B[0:2, :] = 0
    A[:, :4] = 0
    W[0, 0] = 0x3F80
    W[0, 1] = 0x3F81
    W[1, 2] = 0x0000
    B[0, 0] = _bits_of([2.0 ** -4])[0]
    A[0, 0] = _bits_of([2.0 ** -5])[0]
    A[0, 1] = _bits_of([2.0 ** -5])[0]
    B[1, 1] = _bits_of([2.0 ** -67])[0]
    A[1, 2] = _bits_of([1.5 * 2.0 ** -67])[0]
    s = 2.0
    for sign in (1, -1):
        got = O.lora_merge(W, A, B, s, sign)
        Wf, Af, Bf = (np.array(x, np.uint32) for x in (W, A, B))
        for n in range(N):
            for k in range(K):
                acc = sum(_bf16_value(int(Bf[n, j])) * _bf16_value(int(Af[j, k])) for j in range(r))
                x = _bf16_value(int(Wf[n, k])) + sign * Fraction(s) * acc
                assert int(got[n, k]) == _bf16_nearest_even(x), (sign, n, k)
    got = O.lora_merge(W, A, B, s, 1)
    assert got[0, 0] == 0x3F80   # 1 + 2^-8: tie, to the even code (1.0)
    assert got[0, 1] == 0x3F82   # 1.0078125 + 2^-8: tie, to the even code
    assert got[1, 2] == 0x0002   # 1.5 * 2^-133: tie, to the even subnormal


def test_lora_merge_zero_B_is_identity(O):
    """B = 0 (the adapter's initial state): the merged weight is the base."""
    rng = np.random.default_rng(6)
    W = _bits_of(rng.normal(0, 0.02, (16, 128)))
    A = _bits_of(rng.normal(0, 0.1, (8, 128)))
    B = np.zeros((16, 8), np.uint16)
    np.testing.assert_array_equal(O.lora_merge(W, A, B, 2.0), W)


# ---------------------------------------------------------------------------
# fused projections (q/k/v or gate/up sharing X, one adapter per segment)
# ---------------------------------------------------------------------------

def test_fused_projection_vs_autograd(O):
    """The oracle's fused projection against torch autograd in fp64 on the
    explicit per-segment model: Y[:, seg i] = X W_i^T + s (X A_i^T) B_i^T,
    loss = sum(Y * dY); dX, dA, dB from backward (dX summed over the
    segments by autograd itself)."""
    rng = np.random.default_rng(8)
    M, S, K, r, nseg, s = 7, 12, 64, 4, 3, 1.5
    N = nseg * S
    X, W, A, B, dY = (_bits_of(rng.normal(0, sd, shp)) for sd, shp in
                      ((1.0, (M, K)), (0.05, (N, K)), (0.2, (nseg * r, K)), (0.1, (N, r)), (1.0, (M, N))))

    def t(b, grad=False):
        v = torch.from_numpy((np.asarray(b, np.uint32) << 16).view(np.float32).astype(np.float64))
        return v.requires_grad_(grad)

    Xt, At, Bt = t(X, True), t(A, True), t(B, True)
    Wt, dYt = t(W), t(dY)
    Y = torch.cat([Xt @ Wt[i * S:(i + 1) * S].T + s * (Xt @ At[i * r:(i + 1) * r].T) @ Bt[i * S:(i + 1) * S].T
                   for i in range(nseg)], dim=1)
    (Y * dYt).sum().backward()
    np.testing.assert_allclose(O.fused_linear_fwd(X, W, A, B, s, nseg), Y.detach().numpy(), rtol=1e-12, atol=1e-12)
    gx, ga, gb = O.fused_linear_bwd(dY, X, W, A, B, s, nseg)
    np.testing.assert_allclose(gx, Xt.grad.numpy(), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(ga, At.grad.numpy(), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(gb, Bt.grad.numpy(), rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------------------
# adapter optimizer step
# ---------------------------------------------------------------------------

def test_adamw_vs_torch_optim(O):
    """The oracle's AdamW step against torch.optim.AdamW in fp64 over four
    steps with weight decay and a gradient scale."""
    rng = np.random.default_rng(9)
    n = 257
    p0 = rng.normal(0, 0.1, n)
    grads = [rng.normal(0, 1e-3, n) for _ in range(4)]
    lr, b1, b2, eps, wd, gs = 2e-4, 0.9, 0.999, 1e-8, 0.01, 0.5
    pt = torch.tensor(p0.copy(), dtype=torch.float64, requires_grad=True)
    opt = torch.optim.AdamW([pt], lr=lr, betas=(b1, b2), eps=eps, weight_decay=wd)
    p, m, v = p0.copy(), np.zeros(n), np.zeros(n)
    for t, g in enumerate(grads, start=1):
        pt.grad = torch.tensor(g * gs, dtype=torch.float64)
        opt.step()
        O.adamw_step(p, m, v, g, lr=lr, step=t, beta1=b1, beta2=b2, eps=eps, weight_decay=wd, grad_scale=gs)
        np.testing.assert_allclose(p, pt.detach().numpy(), rtol=1e-13, atol=1e-16)
        st = opt.state[pt]
        np.testing.assert_allclose(m, st["exp_avg"].numpy(), rtol=1e-13, atol=1e-20)
        np.testing.assert_allclose(v, st["exp_avg_sq"].numpy(), rtol=1e-13, atol=1e-24)


# ---------------------------------------------------------------------------
# data-type variants: FP4 codes, FP8 (E4M3) double quantization, block sizes
# ---------------------------------------------------------------------------

def test_fp4_table_closed_form(O):
    """FP4 = 1 sign, 2 exponent (bias 1), 1 mantissa bit: magnitudes 0, 0.5,
    1, 1.5, 2, 3, 4, 6 divided by 6, both signs, sorted; -0 and +0 at 7, 8."""
    mags = []
    for e in range(4):
        for m in range(2):
            mags.append(Fraction(m, 2) if e == 0 else (1 + Fraction(m, 2)) * Fraction(2) ** (e - 1))
    mags = sorted(mags)
    assert mags == [Fraction(x) for x in (0, 0.5, 1, 1.5, 2, 3, 4, 6)]
    want = [-float(x / 6) for x in reversed(mags)] + [float(x / 6) for x in mags]
    t = O.fp4_table()
    np.testing.assert_array_equal(_f32bits(t), _f32bits(np.array(want, np.float32)))
    assert np.signbit(t[7]) and not np.signbit(t[8]) and t[7] == 0 and t[8] == 0


def test_e4m3_table_vs_torch(O):
    """The E4M3 code book: every finite value of torch.float8_e4m3fn (a
    library routine), zeros merged, sorted, divided by 448, in fp32."""
    v = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).to(torch.float64)
    v = v[~torch.isnan(v)].unique().numpy()  # unique also merges -0 and +0
    want = (np.sort(v) / 448.0).astype(np.float32)
    want[want == 0] = 0.0  # the one merged zero is +0
    t = O.e4m3_table()
    assert t.size == 253 and want.size == 253
    np.testing.assert_array_equal(_f32bits(t), _f32bits(want))


@pytest.mark.parametrize("bs", [64, 128, 256])
@pytest.mark.parametrize("code_type", ["nf4", "fp4"])
def test_variant_roundtrip_lossless(O, bs, code_type):
    """Blocks of bs elements that are exactly code-book values times their
    absmax round-trip: the constant of block b is the max over elements
    [b bs, (b+1) bs), every code comes back, and the dequantized bf16 value
    is the bf16 of the input."""
    rng = np.random.default_rng(bs)
    t = O.fp4_table() if code_type == "fp4" else O.nf4_table()
    usable = [j for j in range(16) if not (code_type == "fp4" and j == 8)]  # +0 is never chosen (ties low)
    nb = 40
    idx = rng.choice(usable, (nb, bs))
    idx[:, 3] = 15
    a = rng.uniform(1e-3, 3.0, nb).astype(np.float32)
    w = (t[idx] * a[:, None]).astype(np.float32)
    q = O.nf4_quantize(w.reshape(-1), double_quant=False, blocksize=bs, code_type=code_type)
    np.testing.assert_array_equal(q["absmax"], a)
    np.testing.assert_array_equal(q["absmax"], np.abs(w).max(axis=1))
    codes = np.empty(nb * bs, np.uint8)
    codes[0::2] = q["codes"] >> 4
    codes[1::2] = q["codes"] & 15
    np.testing.assert_array_equal(codes, idx.reshape(-1))
    deq = O.nf4_dequantize(w.size, q, double_quant=False, blocksize=bs, code_type=code_type)
    ref = torch.from_numpy(w.reshape(-1)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(deq, ref)


def test_fp4_zero_ties_to_negative_zero(O):
    """With two zeros in the FP4 code book, an exact tie goes to the lower
    index: 0 and values nearer to 0 than to 1/12 get code 7 (-0)."""
    w = np.array([1.0, 0.0, 1e-30, -1e-30, 0.04, 0.0417, -0.04] + [0.5] * 57, np.float32)
    q = O.nf4_quantize(w, double_quant=False, code_type="fp4")
    codes = np.empty(64, np.uint8)
    codes[0::2] = q["codes"] >> 4
    codes[1::2] = q["codes"] & 15
    assert list(codes[:7]) == [15, 7, 7, 7, 7, 9, 7]


@pytest.mark.parametrize("bs", [64, 256])
def test_e4m3_double_quant(O, bs):
    """FP8 (E4M3) double quantization: the 8-bit codes index the 253-value
    code book; each code is the nearest entry (exact rationals, ties low);
    equal block maxima stay lossless (c1 = 0, code of 0)."""
    rng = np.random.default_rng(3)
    w = rng.normal(0, 0.02, bs * 700).astype(np.float32)
    q = O.nf4_quantize(w, double_quant=True, blocksize=bs, dq_type="e4m3")
    t = O.e4m3_table()
    assert q["q8"].max() < 253
    absmax = np.abs(w.reshape(-1, bs)).max(axis=1)
    off = np.float32(q["offset"])
    for b in range(0, absmax.size, 37):
        c = q["c1"][b // 256]
        d = np.float32(absmax[b] - off)
        y = np.float32(d * np.float32(np.float32(1.0) / c))
        dist = [abs(Fraction(float(y)) - Fraction(float(x))) for x in t]
        best = min(range(len(t)), key=lambda k: (dist[k], k))
        assert q["q8"][b] == best
    a = np.float32(0.0371)
    w2 = (rng.uniform(-1, 1, (300, bs)) * a).astype(np.float32)
    w2[:, 1] = a
    q2 = O.nf4_quantize(w2.reshape(-1), double_quant=True, blocksize=bs, dq_type="e4m3")
    assert float(q2["c1"].max()) == 0.0 and np.all(q2["q8"] == 126)
    d2 = O.nf4_dequantize(w2.size, q2, double_quant=True, blocksize=bs, dq_type="e4m3")
    q0 = O.nf4_quantize(w2.reshape(-1), double_quant=False, blocksize=bs)
    np.testing.assert_array_equal(d2, O.nf4_dequantize(w2.size, q0, double_quant=False, blocksize=bs))
