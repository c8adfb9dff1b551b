"""GPU parity of LoRA merge / unmerge against the fp64 oracle, and the merge
check of the LoRA reproduction blog's acceptance protocol: the dense forward
with the merged weight gives the fused NF4 + adapter forward's outputs.

The GPU sums the rank-r product in fp32 on the tensor cores, the oracle in
fp64; both round once to bf16.  Every output code must equal the oracle's,
except where the exact value lies so close to a bf16 rounding boundary that
the fp32 error bound of the GPU's arithmetic reaches across it: there the
GPU's code must be the rounding of a value within that bound, and such codes
must be rare."""
import numpy as np
import pytest
import torch

from bit_nf4_quantized_08_b200 import workloads as wl
from conftest import assert_close_tol

pytestmark = pytest.mark.gpu


def _f(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _half_ulp(x):
    """Half the bf16 spacing at each |x| (2^-134 in the subnormal range)."""
    ax = np.abs(x)
    e = np.floor(np.log2(np.maximum(ax, 2.0 ** -126)))
    return np.ldexp(1.0, (e - 8).astype(np.int64))


def _assert_rounded_like_oracle(got, ref, exact, W, A, B, s, r, what, rare=1e-4):
    """got, ref: bf16 codes; exact: the oracle's fp64 value before rounding.
    Where got differs from the oracle's code, got must still be the rounding
    of some value within the error bound of the GPU's fp32 arithmetic around
    the exact value (so only values that sit that close to a rounding
    boundary may round the other way), and such codes must be rare."""
    bad = np.nonzero(got != ref)
    if bad[0].size == 0:
        return
    g = _f(got[bad])
    v = exact[bad]
    n, k = bad
    # bound of the GPU's error before its final rounding: the fp32 sum of the
    # r products in any order (2 r u sum|t|) and the final fma (2 u |v|)
    absBA = np.einsum("ij,ji->i", np.abs(_f(B)[n, :]), np.abs(_f(A)[:, k]))
    u = 2.0 ** -24
    bound = 2 * r * u * abs(s) * absBA + 2 * u * np.abs(v)
    ok = np.abs(g - v) <= bound + _half_ulp(g)
    assert ok.all(), f"{what}: {int((~ok).sum())} of {got.size} codes differ from the oracle beyond the bound"
    assert bad[0].size <= max(10, rare * got.size), f"{what}: {bad[0].size} near-boundary differences"


def _inputs(N, K, r, seed, dq=True):
    W = wl.weight(N, K, seed=seed, dtype=torch.bfloat16)
    inp = wl.linear_inputs(16, N, K, r, seed=seed, b_std=0.05)
    return W, inp


@pytest.mark.parametrize("N,K,r,dq", [(264, 320, 16, True), (1000, 768, 8, False), (4096, 4096, 64, True),
                                      (136, 192, 256, True), (8192, 8192, 64, True)])
def test_merge_unmerge_parity(Q, O, cuda, N, K, r, dq):
    W, inp = _inputs(N, K, r, seed=31, dq=dq)
    A, B = inp["A"], inp["B"]
    s = 16.0 / r
    q = Q.qlora_nf4_quantize(W.cuda(), double_quant=dq)
    Wm = Q.qlora_lora_merge(q, A.cuda(), B.cuda(), s)
    Wb = Q.qlora_lora_unmerge(Wm, A.cuda(), B.cuda(), s)
    torch.cuda.synchronize()
    assert Q.qlora_get_last_error() == 0
    ref_q = O.nf4_quantize(wl.bits(W).reshape(-1), double_quant=dq)
    Wd = O.nf4_dequantize(N * K, ref_q, double_quant=dq).reshape(N, K)
    Ab, Bb = wl.bits(A), wl.bits(B)
    ref_m, ex_m = O.lora_merge(Wd, Ab, Bb, s, 1, want_exact=True)
    got_m = wl.bits(Wm)
    _assert_rounded_like_oracle(got_m, ref_m, ex_m, Wd, Ab, Bb, s, r, "merge")
    # unmerge of the GPU's merged weight against the oracle's unmerge of it.
    # The exact unmerged value is the base plus the merge's rounding error,
    # which puts far more values near a rounding midpoint than a generic sum
    # (about 0.3 % within the fp32 error of the midpoint with fp32 products,
    # also when emulated on the host), so such differences are less rare
    ref_b, ex_b = O.lora_merge(got_m, Ab, Bb, s, -1, want_exact=True)
    _assert_rounded_like_oracle(wl.bits(Wb), ref_b, ex_b, got_m, Ab, Bb, s, r, "unmerge", rare=1e-2)


def test_merge_with_zero_B_is_the_dequantized_weight(Q, O, cuda):
    """B = 0 (the adapter's initial state): the merged weight equals the
    dequantized base."""
    N, K, r = 512, 1024, 16
    W, inp = _inputs(N, K, r, seed=32)
    q = Q.qlora_nf4_quantize(W.cuda())
    Wm = Q.qlora_lora_merge(q, inp["A"].cuda(), torch.zeros(N, r, dtype=torch.bfloat16, device="cuda"), 2.0)
    Wd = Q.qlora_nf4_dequantize(q)
    torch.cuda.synchronize()
    assert torch.equal(Wm.float(), Wd.float())


@pytest.mark.parametrize("M,N,K,r", [(2048, 4096, 4096, 64), (16, 1024, 2048, 16)])
def test_merge_check_logits(Q, O, cuda, M, N, K, r):
    """Merge check (reproduction blog, acceptance protocol): Y of the dense
    merged weight, X W_merged^T (fp64 oracle), matches the fused NF4 +
    adapter forward of the library within the parity tolerance."""
    W = wl.weight(N, K, seed=33, dtype=torch.bfloat16)
    inp = wl.linear_inputs(M, N, K, r, seed=33, b_std=0.05)
    s = 16.0 / r
    X, A, B = inp["X"], inp["A"], inp["B"]
    q = Q.qlora_nf4_quantize(W.cuda())
    Wm = Q.qlora_lora_merge(q, A.cuda(), B.cuda(), s)
    Y = Q.qlora_linear_fwd(X.cuda(), q, A.cuda(), B.cuda(), s)
    torch.cuda.synchronize()
    assert Q.qlora_get_last_error() == 0
    rows = wl.sample_rows(M, 64, seed=33)
    empty_A = np.zeros((0, K), np.uint16)
    empty_B = np.zeros((N, 0), np.uint16)
    Y_merged = O.linear_fwd(wl.bits(X), wl.bits(Wm), empty_A, empty_B, 0.0, rows=rows)
    assert_close_tol(Y.float().cpu().numpy()[rows], Y_merged, "fused Y vs merged dense Y")


def test_merge_rejects_bad_arguments(Q, cuda):
    W = wl.weight(256, 256, seed=34, dtype=torch.bfloat16).cuda()
    q = Q.qlora_nf4_quantize(W)
    A = torch.zeros(12, 256, dtype=torch.bfloat16, device="cuda")
    B = torch.zeros(256, 12, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(Q.QloraError) as e:
        Q.qlora_lora_merge(q, A, B, 1.0)
    assert e.value.status == Q.QLORA_ERR_UNSUPPORTED
