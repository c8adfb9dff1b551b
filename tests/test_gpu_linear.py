"""GPU parity of the fused NF4-dequant + LoRA linear forward and backward
against the fp64 CPU oracle, on seeded inputs that span several tiles and a
ragged tail, plus the invariants of the pages (B = 0 is a no-op, no dW)."""
import numpy as np
import pytest
import torch

from bit_nf4_quantized_08_b200 import workloads as wl
from conftest import assert_close_tol

pytestmark = pytest.mark.gpu


def _setup(Q, O, M, N, K, r, seed=0, dq=True, b_std=0.01):
    W = wl.weight(N, K, seed=seed, dtype=torch.bfloat16)
    inp = wl.linear_inputs(M, N, K, r, seed=seed, b_std=b_std)
    q = Q.qlora_nf4_quantize(W.cuda(), double_quant=dq)
    ref_q = O.nf4_quantize(wl.bits(W).reshape(-1), double_quant=dq)
    Wd_ref = O.nf4_dequantize(N * K, ref_q, double_quant=dq).reshape(N, K)
    return q, inp, Wd_ref


def _fwd_both(Q, O, q, inp, Wd_ref, s, r):
    X = inp["X"]
    A, B = inp["A"], inp["B"]
    Y = Q.qlora_linear_fwd(X.cuda(), q, None if r == 0 else A.cuda(), None if r == 0 else B.cuda(), s)
    assert Q.qlora_get_last_error() == 0
    K = X.shape[1]
    N = Wd_ref.shape[0]
    Ab = wl.bits(A) if r else np.zeros((0, K), np.uint16)
    Bb = wl.bits(B) if r else np.zeros((N, 0), np.uint16)
    ref = O.linear_fwd(wl.bits(X), Wd_ref, Ab, Bb, s)
    return Y.float().cpu().numpy(), ref


FWD_CASES = [
    # (M, N, K, r): several tiles + ragged tails; small-M path for M <= 64
    (300, 640, 512, 16),
    (129, 264, 256, 8),
    (65, 512, 64, 64),
    (257, 256, 1024, 0),
    (64, 640, 512, 16),
    (17, 384, 256, 8),
    (3, 1000, 512, 64),
    (1, 256, 128, 8),
    (33, 136, 192, 32),
    (300, 640, 512, 128),
    (200, 264, 192, 256),
    (17, 384, 256, 128),
    # small M over many tiles: stream-K shares cut tiles between CTAs
    (5, 2000, 2048, 64),
    (48, 1096, 1024, 16),
    (64, 296, 4096, 0),
    # long per-CTA unit ranges: the stage and operand rings wrap many times,
    # LoRA steps fall in the middle of ranges
    (16, 4096, 8192, 64),
    (40, 2048, 4096, 128),
]


@pytest.mark.parametrize("M,N,K,r", FWD_CASES)
def test_fwd_parity(Q, O, cuda, M, N, K, r):
    q, inp, Wd_ref = _setup(Q, O, M, N, K, r, seed=1)
    s = 16.0 / max(r, 1)
    got, ref = _fwd_both(Q, O, q, inp, Wd_ref, s, r)
    assert_close_tol(got, ref, f"Y M={M} N={N} K={K} r={r}")


@pytest.mark.parametrize("M,N,K,r", [(300, 640, 512, 16), (129, 264, 256, 8), (65, 512, 128, 64),
                                     (200, 256, 320, 0), (7, 264, 192, 8), (130, 520, 256, 24),
                                     (200, 264, 192, 128), (96, 136, 128, 256), (1100, 264, 1088, 64)])
def test_bwd_parity(Q, O, cuda, M, N, K, r):
    q, inp, Wd_ref = _setup(Q, O, M, N, K, r, seed=2, b_std=0.05)
    s = 2.0
    X, dY, A, B = inp["X"], inp["dY"], inp["A"], inp["B"]
    dX, dA, dB = Q.qlora_linear_bwd(dY.cuda(), X.cuda(), q, None if r == 0 else A.cuda(),
                                    None if r == 0 else B.cuda(), s)
    assert Q.qlora_get_last_error() == 0
    Ab = wl.bits(A) if r else np.zeros((0, K), np.uint16)
    Bb = wl.bits(B) if r else np.zeros((N, 0), np.uint16)
    rdX, rdA, rdB = O.linear_bwd(wl.bits(dY), wl.bits(X), Wd_ref, Ab, Bb, s)
    assert_close_tol(dX.float().cpu().numpy(), rdX, "dX")
    if r:
        assert_close_tol(dA.cpu().numpy(), rdA, "dA")
        assert_close_tol(dB.cpu().numpy(), rdB, "dB")


def test_bwd_serial_path_matches(Q, O, cuda):
    """The serial backward (test mode 6: sU and sG in one split-K launch, dX
    GEMM, then dA and dB) and the default one (sG alone, dX GEMM beside it,
    sU, dA and dB on the side stream) both match the oracle.  The two sum sG
    in different orders, so they are not bitwise equal."""
    M, N, K, r = 1100, 1280, 1024, 32
    q, inp, Wd_ref = _setup(Q, O, M, N, K, r, seed=12, b_std=0.05)
    X, dY, A, B = (inp[k].cuda() for k in ("X", "dY", "A", "B"))
    s = 2.0
    Q.qlora_debug_inject(6)
    try:
        serial = Q.qlora_linear_bwd(dY, X, q, A, B, s)
        assert Q.qlora_get_last_error() == 0
    finally:
        Q.qlora_debug_inject(0)
    forked = Q.qlora_linear_bwd(dY, X, q, A, B, s)
    assert Q.qlora_get_last_error() == 0
    rdX, rdA, rdB = O.linear_bwd(wl.bits(inp["dY"]), wl.bits(inp["X"]), Wd_ref, wl.bits(inp["A"]),
                                 wl.bits(inp["B"]), s)
    for tag, g in (("serial", serial), ("side stream", forked)):
        assert_close_tol(g[0].float().cpu().numpy(), rdX, f"dX {tag}")
        assert_close_tol(g[1].cpu().numpy(), rdA, f"dA {tag}")
        assert_close_tol(g[2].cpu().numpy(), rdB, f"dB {tag}")


@pytest.mark.parametrize("mode", [0, 6], ids=["side_stream", "serial"])
def test_back_to_back_calls_share_workspace(Q, O, cuda, mode):
    """Forward and backward calls of two layers issued back to back on one
    stream with one workspace (the kernels of a call may start while the
    call before finishes) give bitwise the results of the same calls run
    one at a time with their own workspaces."""
    shapes = [(600, 1024, 512, 32), (600, 512, 1024, 32)]
    layers = []
    for i, (M, N, K, r) in enumerate(shapes):
        q, inp, _ = _setup(Q, O, M, N, K, r, seed=40 + i, b_std=0.05)
        layers.append((q, {k: v.cuda() for k, v in inp.items()}))
    ws_bytes = max(max(Q.qlora_linear_workspace(M, q, r, True), Q.qlora_linear_workspace(M, q, r, False))
                   for (M, N, K, r), (q, _) in zip(shapes, layers))
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    Q.qlora_debug_inject(mode)
    try:
        chained = []
        for q, t in layers:
            chained.append(Q.qlora_linear_fwd(t["X"], q, t["A"], t["B"], 2.0, ws=ws))
        for q, t in reversed(layers):
            chained.extend(Q.qlora_linear_bwd(t["dY"], t["X"], q, t["A"], t["B"], 2.0, ws=ws))
        torch.cuda.synchronize()
        single = []
        for q, t in layers:
            single.append(Q.qlora_linear_fwd(t["X"], q, t["A"], t["B"], 2.0))
            torch.cuda.synchronize()
        for q, t in reversed(layers):
            single.extend(Q.qlora_linear_bwd(t["dY"], t["X"], q, t["A"], t["B"], 2.0))
            torch.cuda.synchronize()
        assert Q.qlora_get_last_error() == 0
    finally:
        Q.qlora_debug_inject(0)
    for i, (a_, b_) in enumerate(zip(chained, single)):
        assert torch.equal(a_.view(torch.int32 if a_.dtype == torch.float32 else torch.int16),
                           b_.view(torch.int32 if b_.dtype == torch.float32 else torch.int16)), f"output {i}"


def test_bwd_graph_replay(Q, O, cuda):
    """The backward captured in a CUDA graph, with dA and dB forked onto the
    side stream and joined back inside the capture, replayed on new inputs:
    every replay is bitwise equal to the eager call on the same inputs."""
    M, N, K, r = 600, 1024, 512, 64
    q, inp, _ = _setup(Q, O, M, N, K, r, seed=13, b_std=0.05)
    X, dY, A, B = (inp[k].cuda() for k in ("X", "dY", "A", "B"))
    dX = torch.empty(M, K, dtype=torch.bfloat16, device="cuda")
    dA = torch.empty(r, K, dtype=torch.float32, device="cuda")
    dB = torch.empty(N, r, dtype=torch.float32, device="cuda")
    ws = torch.empty(Q.qlora_linear_workspace(M, q, r, True), dtype=torch.uint8, device="cuda")
    Q.qlora_linear_bwd(dY, X, q, A, B, 2.0, dX=dX, dA=dA, dB=dB, ws=ws)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        Q.qlora_linear_bwd(dY, X, q, A, B, 2.0, dX=dX, dA=dA, dB=dB, ws=ws)
    for rep in range(3):
        new = wl.linear_inputs(M, N, K, r, seed=30 + rep)
        X.copy_(new["X"].cuda())
        dY.copy_(new["dY"].cuda())
        g.replay()
        torch.cuda.synchronize()
        got = [t.clone() for t in (dX, dA, dB)]
        ref = Q.qlora_linear_bwd(dY, X, q, A, B, 2.0)
        torch.cuda.synchronize()
        for a_, b_ in zip(got, ref):
            assert torch.equal(a_.view(torch.int32 if a_.dtype == torch.float32 else torch.int16),
                               b_.view(torch.int32 if b_.dtype == torch.float32 else torch.int16)), f"replay {rep}"
    assert Q.qlora_get_last_error() == 0


@pytest.mark.parametrize("M", [5, 300])
def test_zero_B_is_noop(Q, O, cuda, M):
    """Reproduction blog invariant: B = 0 at step 0 gives the frozen base
    output; bitwise equal to the call with the adapter scaled by 0."""
    N, K, r = 512, 256, 16
    q, inp, _ = _setup(Q, O, M, N, K, r, seed=3)
    X, A = inp["X"].cuda(), inp["A"].cuda()
    B0 = torch.zeros(N, r, dtype=torch.bfloat16, device="cuda")
    y0 = Q.qlora_linear_fwd(X, q, A, B0, 2.0)
    y_s0 = Q.qlora_linear_fwd(X, q, A, inp["B"].cuda(), 0.0)
    y_none = Q.qlora_linear_fwd(X, q, None, None, 2.0)
    assert torch.equal(y0.view(torch.int16), y_none.view(torch.int16))
    assert torch.equal(y_s0.view(torch.int16), y_none.view(torch.int16))


def test_fwd_bwd_deterministic(Q, O, cuda):
    M, N, K, r = 300, 640, 512, 16
    q, inp, _ = _setup(Q, O, M, N, K, r, seed=4)
    X, dY, A, B = (inp[k].cuda() for k in ("X", "dY", "A", "B"))
    y1 = Q.qlora_linear_fwd(X, q, A, B, 1.5)
    y2 = Q.qlora_linear_fwd(X, q, A, B, 1.5)
    g1 = Q.qlora_linear_bwd(dY, X, q, A, B, 1.5)
    g2 = Q.qlora_linear_bwd(dY, X, q, A, B, 1.5)
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
    for a, b in zip(g1, g2):
        assert torch.equal(a.view(torch.int32 if a.dtype == torch.float32 else torch.int16),
                           b.view(torch.int32 if b.dtype == torch.float32 else torch.int16))


def test_empty_tokens(Q, O, cuda):
    N, K, r = 256, 128, 8
    q, inp, _ = _setup(Q, O, 1, N, K, r, seed=5)
    X = torch.empty(0, K, dtype=torch.bfloat16, device="cuda")
    dY = torch.empty(0, N, dtype=torch.bfloat16, device="cuda")
    A, B = inp["A"].cuda(), inp["B"].cuda()
    Y = Q.qlora_linear_fwd(X, q, A, B, 2.0)
    assert Y.shape == (0, N)
    dA = torch.full((r, K), 7.0, device="cuda")
    dB = torch.full((N, r), 7.0, device="cuda")
    dX, dA, dB = Q.qlora_linear_bwd(dY, X, q, A, B, 2.0, dA=dA, dB=dB)
    torch.cuda.synchronize()
    assert float(dA.abs().max()) == 0.0 and float(dB.abs().max()) == 0.0


def test_timeout_is_reported_and_recovers(Q, O, cuda):
    """Failure detection without a GPU fault: the producer skips its loads,
    the consumers' bounded waits run out, the status word reports TIMEOUT,
    and the next normal call on the same context is correct."""
    M, N, K, r = 256, 256, 128, 8
    q, inp, Wd_ref = _setup(Q, O, M, N, K, r, seed=6)
    X, A, B = inp["X"].cuda(), inp["A"].cuda(), inp["B"].cuda()
    Q.qlora_get_last_error()
    Q.qlora_set_wait_timeout_ns(20_000_000)
    Q.qlora_debug_inject(1)
    try:
        Q.qlora_linear_fwd(X, q, A, B, 2.0)
        st = Q.qlora_get_last_error()
    finally:
        Q.qlora_debug_inject(0)
        Q.qlora_set_wait_timeout_ns(0)
    assert st == Q.QLORA_ERR_TIMEOUT
    got, ref = _fwd_both(Q, O, q, inp, Wd_ref, 2.0, r)
    assert_close_tol(got, ref, "Y after recovery")


@pytest.mark.parametrize("mode", [2, 3, 4], ids=["streamk7", "single_cta_grid", "pair_streamk4"])
@pytest.mark.parametrize("M,N,K,r", [(300, 640, 512, 16), (513, 264, 256, 8), (257, 512, 192, 64),
                                     (1100, 1280, 1024, 32), (200, 256, 1024, 8)])
def test_alternate_schedule_parity(Q, O, cuda, mode, M, N, K, r):
    """Forward and dX on the single-CTA kernel, on the stream-K schedule
    (forced onto 7 CTAs, so that tiles are split across CTAs and merged) and
    on the grid schedule, and on the CTA-pair kernel with stream-K forced onto
    4 pairs, match the oracle and are bitwise reproducible."""
    q, inp, Wd_ref = _setup(Q, O, M, N, K, r, seed=7, b_std=0.05)
    X, dY, A, B = (inp[k].cuda() for k in ("X", "dY", "A", "B"))
    s = 2.0
    Q.qlora_debug_inject(mode)
    try:
        Y1 = Q.qlora_linear_fwd(X, q, A, B, s)
        Y2 = Q.qlora_linear_fwd(X, q, A, B, s)
        dX1, dA1, dB1 = Q.qlora_linear_bwd(dY, X, q, A, B, s)
        dX2, _, _ = Q.qlora_linear_bwd(dY, X, q, A, B, s)
        assert Q.qlora_get_last_error() == 0
    finally:
        Q.qlora_debug_inject(0)
    assert torch.equal(Y1.view(torch.int16), Y2.view(torch.int16))
    assert torch.equal(dX1.view(torch.int16), dX2.view(torch.int16))
    ref = O.linear_fwd(wl.bits(inp["X"]), Wd_ref, wl.bits(inp["A"]), wl.bits(inp["B"]), s)
    assert_close_tol(Y1.float().cpu().numpy(), ref, "Y alternate schedule")
    rdX, rdA, rdB = O.linear_bwd(wl.bits(inp["dY"]), wl.bits(inp["X"]), Wd_ref, wl.bits(inp["A"]),
                                 wl.bits(inp["B"]), s)
    assert_close_tol(dX1.float().cpu().numpy(), rdX, "dX alternate schedule")
    # the default (CTA-pair) kernel gives the same values up to fp32 summation order
    Y3 = Q.qlora_linear_fwd(X, q, A, B, s)
    assert_close_tol(Y3.float().cpu().numpy(), ref, "Y default")


def test_small_m_graph_replay(Q, O, cuda):
    """The small-M forward captured in a CUDA graph and replayed on new
    inputs: every replay matches the oracle (the partial-tile flags of one
    replay are never taken for the next one's)."""
    M, N, K, r = 7, 1536, 2048, 32
    q, inp, Wd_ref = _setup(Q, O, M, N, K, r, seed=8)
    X = inp["X"].cuda()
    A, B = inp["A"].cuda(), inp["B"].cuda()
    Y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(Q.qlora_linear_workspace(M, q, r, False), dtype=torch.uint8, device="cuda")
    Q.qlora_linear_fwd(X, q, A, B, 2.0, Y=Y, ws=ws)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        Q.qlora_linear_fwd(X, q, A, B, 2.0, Y=Y, ws=ws)
    for rep in range(3):
        Xn = wl.linear_inputs(M, N, K, r, seed=20 + rep)["X"]
        X.copy_(Xn.cuda())
        g.replay()
        torch.cuda.synchronize()
        ref = O.linear_fwd(wl.bits(Xn), Wd_ref, wl.bits(inp["A"]), wl.bits(inp["B"]), 2.0)
        assert_close_tol(Y.float().cpu().numpy(), ref, f"Y replay {rep}")
    assert Q.qlora_get_last_error() == 0


@pytest.mark.parametrize("M", [16, 24])
def test_small_m_timeout_is_reported_and_recovers(Q, O, cuda, M):
    """Failure detection on the small-M kernels (M = 16: the warp-MMA kernel,
    M = 24: the tcgen05 kernel): skipped loads make the bounded waits run
    out, TIMEOUT is reported, the next call is correct."""
    N, K, r = 1024, 1024, 16
    q, inp, Wd_ref = _setup(Q, O, M, N, K, r, seed=9)
    X, A, B = inp["X"].cuda(), inp["A"].cuda(), inp["B"].cuda()
    Q.qlora_get_last_error()
    Q.qlora_set_wait_timeout_ns(20_000_000)
    Q.qlora_debug_inject(1)
    try:
        Q.qlora_linear_fwd(X, q, A, B, 2.0)
        st = Q.qlora_get_last_error()
    finally:
        Q.qlora_debug_inject(0)
        Q.qlora_set_wait_timeout_ns(0)
    assert st == Q.QLORA_ERR_TIMEOUT
    got, ref = _fwd_both(Q, O, q, inp, Wd_ref, 2.0, r)
    assert_close_tol(got, ref, "Y after recovery")


@pytest.mark.parametrize("M,N,K,r", [(1, 768, 1024, 16), (5, 2000, 2048, 64), (16, 4096, 8192, 64)])
def test_small_m_tcgen05_kernel_for_few_tokens(Q, O, cuda, M, N, K, r):
    """Test mode 8: the tcgen05 small-M kernel (bit-exact bf16 weight tiles)
    for M <= 16, where the default is the warp-MMA kernel."""
    q, inp, Wd_ref = _setup(Q, O, M, N, K, r, seed=91)
    Q.qlora_debug_inject(8)
    try:
        got, ref = _fwd_both(Q, O, q, inp, Wd_ref, 2.0, r)
        torch.cuda.synchronize()
        assert Q.qlora_get_last_error() == 0
    finally:
        Q.qlora_debug_inject(0)
    assert_close_tol(got, ref, f"Y tcgen05 M={M}")


@pytest.mark.parametrize("M,N,K,r,nseg,dq", [(1, 256, 128, 8, 1, True), (3, 1000, 512, 64, 1, True),
                                             (8, 22016, 8192, 64, 1, True), (16, 4096, 8192, 64, 1, True),
                                             (17, 384, 256, 128, 1, True), (32, 2048, 4096, 32, 1, True),
                                             (16, 3 * 1024, 2048, 32, 3, True), (5, 2000, 2048, 64, 1, True),
                                             (16, 2 * 768, 1024, 16, 2, True), (24, 3 * 768, 1024, 16, 3, True),
                                             (12, 1000, 1024, 24, 1, False), (30, 520, 640, 40, 1, False),
                                             (16, 2 * 1792, 1024, 32, 2, True), (5, 3 * 1792, 512, 64, 3, True)])
def test_small_m_warp_mma_kernel(Q, O, cuda, M, N, K, r, nseg, dq):
    """The register-fed warp-MMA small-M kernel (test mode 7: block constant
    applied to each 64-element block's fp32 partial, bf16 table values times
    a fixed prescale) against the oracle; the fused projection cases check
    its segment columns of sU, also where one 512-row group spans two
    adapters (segments of 768 rows); two cases without double quantization
    and with a partial last adapter tile (r = 24, 40); segments of 1792 rows
    (a whole number of 224-row units: the wide unit with an adapter per
    segment; 768 and 1024 take the 128-row unit)."""
    S = N // nseg
    W = wl.weight(N, K, seed=90, dtype=torch.bfloat16)
    inp = wl.fused_inputs(M, nseg, S, K, r, seed=90, b_std=0.05)
    q = Q.qlora_nf4_quantize(W.cuda(), double_quant=dq)
    ref_q = O.nf4_quantize(wl.bits(W).reshape(-1), double_quant=dq)
    Wd = O.nf4_dequantize(N * K, ref_q, double_quant=dq).reshape(N, K)
    Q.qlora_debug_inject(7)
    try:
        Y = Q.qlora_fused_linear_fwd(inp["X"].cuda(), q, nseg, inp["A"].cuda(), inp["B"].cuda(), 2.0)
        Y2 = Q.qlora_fused_linear_fwd(inp["X"].cuda(), q, nseg, inp["A"].cuda(), inp["B"].cuda(), 2.0)
        torch.cuda.synchronize()
        assert Q.qlora_get_last_error() == 0
    finally:
        Q.qlora_debug_inject(0)
    assert torch.equal(Y.view(torch.int16), Y2.view(torch.int16))
    ref = O.fused_linear_fwd(wl.bits(inp["X"]), Wd, wl.bits(inp["A"]), wl.bits(inp["B"]), 2.0, nseg)
    assert_close_tol(Y.float().cpu().numpy(), ref, f"Y warp-MMA M={M}")
