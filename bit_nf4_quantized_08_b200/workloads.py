"""Seeded synthetic inputs shaped like the QLoRA pages' workloads.

This module only draws random numbers and names shapes; it holds none of the
method's arithmetic, so both the CUDA path and the CPU oracle can be fed the
same arrays from it.  Every tensor is drawn in fp32 from its own
``torch.Generator`` seeded with ``seed * 1000 + index`` and then rounded to its
storage dtype.  ``N(0, s)`` means standard deviation s.

Workloads (LLaMA-shaped linear layers; the pages finetune LLaMA 7B-65B with
LoRA on every linear layer, r up to 64):
  tiny      one 256x256 linear, W fp32, M=16, r=8, alpha=16
  stress    W 4096x4096 bf16 with 0.1% N(0, 0.5) outliers, M=2048, r=16, alpha=32
  llama7b   q/k/v/o 4096x4096, gate/up 11008x4096, down 4096x11008, M=2048, r=64, alpha=16
  llama65b  q/k/v/o 8192x8192, gate/up 22016x8192, down 8192x22016, M=2048, r=64, alpha=16
  sweep     W 22016x8192, M in 1..64, r=64 (alpha 16); quantize/dequant of 2^30 elements
"""
from __future__ import annotations

import torch

TENSOR_INDEX = {"W": 0, "X": 1, "A": 2, "B": 3, "dY": 4, "outlier_pos": 5, "outlier_val": 6}

LLAMA7B_LINEARS = [("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096), ("o", 4096, 4096),
                   ("gate", 11008, 4096), ("up", 11008, 4096), ("down", 4096, 11008)]
LLAMA65B_LINEARS = [("q", 8192, 8192), ("k", 8192, 8192), ("v", 8192, 8192), ("o", 8192, 8192),
                    ("gate", 22016, 8192), ("up", 22016, 8192), ("down", 8192, 22016)]

CONFIGS = {
    "tiny": dict(linears=[("w", 256, 256)], M=16, r=8, alpha=16.0, w_dtype=torch.float32),
    "stress": dict(linears=[("w", 4096, 4096)], M=2048, r=16, alpha=32.0, w_dtype=torch.bfloat16,
                   outlier_frac=0.001, outlier_std=0.5),
    "llama7b": dict(linears=LLAMA7B_LINEARS, M=2048, r=64, alpha=16.0, w_dtype=torch.bfloat16),
    "llama65b": dict(linears=LLAMA65B_LINEARS, M=2048, r=64, alpha=16.0, w_dtype=torch.bfloat16),
    "sweep": dict(linears=[("w", 22016, 8192)], Ms=[1, 2, 4, 8, 16, 32, 64], r=64, alpha=16.0,
                  w_dtype=torch.bfloat16, big_numel=1 << 30),
}


# The same blocks as fused projections: (name, nseg, rows per segment, K).
# q/k/v share the attention input and gate/up the MLP input, so each group is
# one weight of nseg row segments with one adapter per segment.
FUSED_GROUPS = {
    "llama7b": [("qkv", 3, 4096, 4096), ("o", 1, 4096, 4096), ("gate_up", 2, 11008, 4096),
                ("down", 1, 4096, 11008)],
    "llama65b": [("qkv", 3, 8192, 8192), ("o", 1, 8192, 8192), ("gate_up", 2, 22016, 8192),
                 ("down", 1, 8192, 22016)],
}


def _gen(seed: int, index: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) * 1000 + int(index))
    return g


def normal(shape, std: float, seed: int, index: int, dtype=torch.bfloat16, device="cpu") -> torch.Tensor:
    g = _gen(seed, index, device)
    t = torch.randn(shape, generator=g, dtype=torch.float32, device=device)
    return (t * std).to(dtype)


def weight(rows: int, cols: int, seed: int = 0, dtype=torch.bfloat16, std: float = 0.02,
           outlier_frac: float = 0.0, outlier_std: float = 0.5, device="cpu",
           index_base: int = 0) -> torch.Tensor:
    """W ~ N(0, std); with outliers, exactly round(frac * n) positions drawn
    without replacement are replaced by N(0, outlier_std) draws."""
    W = normal((rows, cols), std, seed, index_base + TENSOR_INDEX["W"], torch.float32, device)
    if outlier_frac > 0:
        n = rows * cols
        k = int(round(outlier_frac * n))
        pos = torch.randperm(n, generator=_gen(seed, index_base + TENSOR_INDEX["outlier_pos"], device),
                             device=device)[:k]
        vals = torch.randn(k, generator=_gen(seed, index_base + TENSOR_INDEX["outlier_val"], device),
                           device=device) * outlier_std
        W.view(-1)[pos] = vals
    return W.to(dtype)


def linear_inputs(M: int, N: int, K: int, r: int, seed: int = 0, device="cpu", index_base: int = 0,
                  b_std: float = 0.01) -> dict:
    """X ~ N(0,1) [M,K], A ~ N(0, 1/r) [r,K], B ~ N(0, b_std) [N,r], dY ~ N(0,1) [M,N] (bf16)."""
    out = {
        "X": normal((M, K), 1.0, seed, index_base + TENSOR_INDEX["X"], device=device),
        "dY": normal((M, N), 1.0, seed, index_base + TENSOR_INDEX["dY"], device=device),
    }
    if r > 0:
        out["A"] = normal((r, K), 1.0 / r, seed, index_base + TENSOR_INDEX["A"], device=device)
        out["B"] = normal((N, r), b_std, seed, index_base + TENSOR_INDEX["B"], device=device)
    else:
        out["A"] = None
        out["B"] = None
    return out


def fused_inputs(M: int, nseg: int, S: int, K: int, r: int, seed: int = 0, device="cpu", index_base: int = 0,
                 b_std: float = 0.01) -> dict:
    """Inputs of a fused projection of nseg linears of S rows each sharing X:
    X ~ N(0,1) [M,K], dY ~ N(0,1) [M, nseg*S], A ~ N(0, 1/r) [nseg*r, K]
    (one rank-r adapter per segment), B ~ N(0, b_std) [nseg*S, r] (bf16)."""
    N = nseg * S
    return {
        "X": normal((M, K), 1.0, seed, index_base + TENSOR_INDEX["X"], device=device),
        "dY": normal((M, N), 1.0, seed, index_base + TENSOR_INDEX["dY"], device=device),
        "A": normal((nseg * r, K), 1.0 / r, seed, index_base + TENSOR_INDEX["A"], device=device),
        "B": normal((N, r), b_std, seed, index_base + TENSOR_INDEX["B"], device=device),
    }


def sample_rows(M: int, n: int = 64, seed: int = 0):
    """Token rows on which outputs of a full-size layer are compared with the
    oracle: the first and the last row plus n - 2 distinct rows drawn (seeded,
    without replacement) from the ones in between; all rows when M <= n.
    Returns a sorted int64 NumPy array."""
    import numpy as np
    if M <= n:
        return np.arange(M, dtype=np.int64)
    g = _gen(seed, 900, "cpu")
    mid = torch.randperm(M - 2, generator=g)[: n - 2] + 1
    rows = sorted({0, M - 1, *mid.tolist()})
    return np.asarray(rows, dtype=np.int64)


def bits(t: torch.Tensor):
    """Raw bit pattern of a bf16 tensor as a NumPy uint16 array (CPU copy)."""
    import numpy as np
    assert t.dtype == torch.bfloat16
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def from_bits(a, device="cpu") -> torch.Tensor:
    """bf16 tensor from a NumPy uint16 bit-pattern array."""
    import numpy as np
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)
