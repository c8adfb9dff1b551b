"""Out-of-bounds write detection without a sanitizer: every output of every
entry point is a view into a larger buffer whose guard bytes before and after
the view hold a known pattern; after the call (ragged shapes that end inside
tiles and blocks) the guards must be untouched and the device status clean."""
import numpy as np
import pytest
import torch

from bit_nf4_quantized_08_b200 import workloads as wl

pytestmark = pytest.mark.gpu

GUARD = 4096  # bytes on each side
PATTERN = 0xA5


class Guarded:
    """A tensor of `shape`/`dtype` at a 256-byte aligned offset inside a
    buffer padded with GUARD pattern bytes on both sides."""

    def __init__(self, shape, dtype):
        n = int(np.prod(shape)) if len(shape) else 1
        esize = torch.empty(0, dtype=dtype).element_size()
        nbytes = n * esize
        self.buf = torch.full((GUARD + nbytes + GUARD + 256,), PATTERN, dtype=torch.uint8, device="cuda")
        self.lo = GUARD
        self.hi = GUARD + nbytes
        self.t = self.buf[self.lo:self.hi].view(dtype).view(*shape) if n else self.buf[self.lo:self.lo].view(dtype)

    def check(self, what):
        b = self.buf.cpu().numpy()
        assert np.all(b[:self.lo] == PATTERN), f"{what}: write before the buffer"
        assert np.all(b[self.hi:] == PATTERN), f"{what}: write past the buffer"


def _guarded_weight(Q, rows, cols, dq, bs=64, ct="nf4", dt="int8"):
    n = rows * cols
    nb = (n + bs - 1) // bs
    g = {"codes": Guarded(((n + 1) // 2,), torch.uint8)}
    if dq:
        g["absmax_q8"] = Guarded((nb,), torch.uint8)
        g["absmax_scale"] = Guarded(((nb + 255) // 256,), torch.float32)
        g["absmax_offset"] = Guarded((1,), torch.float32)
        w = Q.NF4Weight(rows, cols, True, g["codes"].t, absmax_q8=g["absmax_q8"].t, absmax_scale=g["absmax_scale"].t,
                        absmax_offset=g["absmax_offset"].t, blocksize=bs, code_type=ct, dq_type=dt)
    else:
        g["absmax"] = Guarded((nb,), torch.float32)
        w = Q.NF4Weight(rows, cols, False, g["codes"].t, absmax=g["absmax"].t, blocksize=bs, code_type=ct,
                        dq_type=dt)
    return w, g


def _check_all(Q, guards, what):
    torch.cuda.synchronize()
    assert Q.qlora_get_last_error() == 0
    for k, g in guards.items():
        g.check(f"{what} {k}")


@pytest.mark.parametrize("rows,cols,dq,bs", [(7, 1000, True, 64), (3, 64 * 256 + 64 * 7 + 32, True, 128),
                                             (129, 320, False, 256), (1, 17, True, 64)])
def test_quantize_dequantize_guards(Q, cuda, rows, cols, dq, bs):
    W = wl.weight(rows, cols, seed=80, dtype=torch.bfloat16).cuda()
    w, g = _guarded_weight(Q, rows, cols, dq, bs)
    Q.qlora_nf4_quantize(W, dq, out=w)
    _check_all(Q, g, "quantize")
    out = Guarded((rows, cols), torch.bfloat16)
    Q.qlora_nf4_dequantize(w, out=out.t)
    _check_all(Q, {"out": out}, "dequantize")


@pytest.mark.parametrize("M,N,K,r", [(300, 264, 320, 24), (17, 136, 192, 8), (40, 520, 256, 16), (3, 1000, 512, 64),
                                     (129, 768, 1088, 32)])
def test_linear_guards(Q, cuda, M, N, K, r):
    W = wl.weight(N, K, seed=81, dtype=torch.bfloat16).cuda()
    inp = {k: v.cuda() for k, v in wl.linear_inputs(M, N, K, r, seed=81).items()}
    w = Q.qlora_nf4_quantize(W)
    Y = Guarded((M, N), torch.bfloat16)
    dX = Guarded((M, K), torch.bfloat16)
    dA = Guarded((r, K), torch.float32)
    dB = Guarded((N, r), torch.float32)
    ws_f = Guarded((Q.qlora_linear_workspace(M, w, r, False),), torch.uint8)
    ws_b = Guarded((Q.qlora_linear_workspace(M, w, r, True),), torch.uint8)
    Q.qlora_linear_fwd(inp["X"], w, inp["A"], inp["B"], 2.0, Y=Y.t, ws=ws_f.t)
    _check_all(Q, {"Y": Y, "ws": ws_f}, "fwd")
    Q.qlora_linear_bwd(inp["dY"], inp["X"], w, inp["A"], inp["B"], 2.0, dX=dX.t, dA=dA.t, dB=dB.t, ws=ws_b.t)
    _check_all(Q, {"dX": dX, "dA": dA, "dB": dB, "ws": ws_b}, "bwd")


@pytest.mark.parametrize("M", [300, 16])
def test_fused_merge_adamw_guards(Q, cuda, M):
    nseg, S, K, r = 3, 256, 320, 16
    N = nseg * S
    W = wl.weight(N, K, seed=82, dtype=torch.bfloat16).cuda()
    inp = {k: v.cuda() for k, v in wl.fused_inputs(M, nseg, S, K, r, seed=82).items()}
    w = Q.qlora_nf4_quantize(W)
    Y = Guarded((M, N), torch.bfloat16)
    dX = Guarded((M, K), torch.bfloat16)
    dA = Guarded((nseg * r, K), torch.float32)
    dB = Guarded((N, r), torch.float32)
    Q.qlora_fused_linear_fwd(inp["X"], w, nseg, inp["A"], inp["B"], 2.0, Y=Y.t)
    Q.qlora_fused_linear_bwd(inp["dY"], inp["X"], w, nseg, inp["A"], inp["B"], 2.0, dX=dX.t, dA=dA.t, dB=dB.t)
    _check_all(Q, {"Y": Y, "dX": dX, "dA": dA, "dB": dB}, "fused")
    Wm = Guarded((N, K), torch.bfloat16)
    Wb = Guarded((N, K), torch.bfloat16)
    A0, B0 = inp["A"][:r].contiguous(), inp["B"]
    Q.qlora_lora_merge(w, A0, B0, 2.0, out=Wm.t)
    Q.qlora_lora_unmerge(Wm.t, A0, B0, 2.0, out=Wb.t)
    _check_all(Q, {"merged": Wm, "unmerged": Wb}, "merge")
    n = 1003
    p, m, v, g = (Guarded((n,), torch.float32) for _ in range(4))
    for x in (p, m, v, g):
        x.t.zero_()
    pb = Guarded((n,), torch.bfloat16)
    Q.qlora_adamw_step(p.t, m.t, v.t, g.t, pb.t, lr=1e-3, step=1)
    _check_all(Q, {"p": p, "m": m, "v": v, "pb": pb}, "adamw")
