#!/usr/bin/env python3
"""Benchmark of the QLoRA NF4 frozen-linear hot path on B200.

One step = one pass of the whole hot path over one batch of the
LLaMA-65B-shaped decoder block (q/k/v/o 8192x8192, gate/up 22016x8192, down
8192x22016; M = 1 x 2048 tokens; LoRA r = 64, alpha = 16 on all seven):
  1. blockwise NF4 quantization + double quantization of the 7 bf16 weights
  2. forward Y = X W'^T + s (X A^T) B^T of the 7 linears
  3. backward dX, dA, dB of the 7 linears (no dW)
value = algorithmic fwd+bwd FLOPs of the step / device time of the step.

Timing: W warm-up steps, then K steps each bracketed by CUDA events on the
launching stream, L2 flushed (256 MiB write) between steps, barrier + device
synchronize around the timed region, max over ranks.  Under torchrun every
rank runs an independent replica (the layer does not shard: weak scaling).

Also reported: the roofline of the dominant kernel (live CUDA-event times of
its launches), an end-to-end figure through the C ABI with pinned host
buffers (every input copied in and every result copied out inside the timed
region), the CPU oracle on a bounded sample (all cores and one core) with its
outputs compared against the GPU's, sampled SM clocks, and extra measurements
outside the step (the LLaMA-7B block, the stress forward, the small-M forward
sweep on a 22016x8192 weight, standalone quantize and dequantize of 2^30
elements).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "fused NF4-dequant+LoRA linear fwd/bwd TFLOP/s and weight GB/s vs B200 roofline"
HEADLINE = "llama65b"
WORKLOADS = {
    "llama65b": "llama65b-decoder-block: 7 NF4+DQ linears (q,k,v,o 8192x8192; gate,up 22016x8192; "
                "down 8192x22016) with a LoRA adapter each, M=2048 (1 x 2048 tokens), r=64, alpha=16; "
                "quantize+fwd+bwd; q/k/v and gate/up as fused projections sharing their input",
    "llama7b": "llama7b-decoder-block: 7 NF4+DQ linears (q,k,v,o 4096x4096; gate,up 11008x4096; "
               "down 4096x11008) with a LoRA adapter each, M=2048 (4 x 512 tokens), r=64, alpha=16; "
               "quantize+fwd+bwd; q/k/v and gate/up as fused projections sharing their input",
}
WORKLOAD = WORKLOADS[HEADLINE]
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
WEIGHT_BYTES_PER_ELEM = 0.5 + 1 / 64 + 4 / (64 * 256)  # NF4 codes + q8 + c1 (DQ)


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-extras", action="store_true", help="skip the small-M sweep and 2^30 quantize/dequant")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--profile-case", choices=["fwd", "dx", "quantize", "dequantize", "smallm",
                                               "fwd_block", "dx_block"],
                    help="run one small case three times, untimed (for ncu captures); "
                         "*_block runs each projection of one decoder block once")
    ap.add_argument("--block", choices=sorted(WORKLOADS), default=HEADLINE,
                    help="decoder block of the *_block profile cases")
    return ap.parse_args()


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------

def fwd_flops(M, N, K, r):
    return 2 * M * N * K + 2 * M * r * (K + N)


def bwd_flops(M, N, K, r):
    return 2 * M * N * K + 4 * M * r * (K + N)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during a region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-f", self.path], stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def source_hash(files=None):
    """sha256 (first 16 hex digits) over the named kernel sources, or over
    every file of the CUDA source tree when no list is given."""
    h = hashlib.sha256()
    d = os.path.join(ROOT, "bit_nf4_quantized_08_b200", "csrc")
    for fn in sorted(files if files else os.listdir(d)):
        with open(os.path.join(d, fn), "rb") as f:
            h.update(fn.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def load_traffic(kind):
    """Per-launch DRAM bytes of a kernel from a committed ncu capture, or None
    when absent or taken on different kernel sources (the entry names the
    source files its hash covers)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(kind)
    if not e or e.get("source_hash") != source_hash(e.get("files")):
        return None
    return e.get("dram_bytes_per_launch")


# ---------------------------------------------------------------------------
# the workload
# ---------------------------------------------------------------------------

class Block:
    """One decoder block with every buffer preallocated.  fused=True: the
    block as its four projections, q/k/v and gate/up each one NF4 weight
    whose row segments share the input (one adapter per segment, one
    qlora_fused_linear call per projection); fused=False: the seven linears
    as separate weights and calls.  Group g draws its tensors from generator
    indices 10*g + (0..9) on the host (the oracle's arrays)."""

    def __init__(self, torch, Q, wl, device, cfg=HEADLINE, seed=0, fused=True):
        c = wl.CONFIGS[cfg]
        self.cfg, self.fused = cfg, fused
        self.M, self.r, self.s = c["M"], c["r"], c["alpha"] / c["r"]
        self.layers = []
        ws_need = 0
        for gi, (name, nseg, S, K) in enumerate(block_groups(wl, cfg, fused)):
            base = 10 * gi
            N = nseg * S
            W = wl.weight(N, K, seed=seed, dtype=torch.bfloat16, index_base=base).to(device)
            inp = {k: v.to(device) for k, v in
                   wl.fused_inputs(self.M, nseg, S, K, self.r, seed=seed, index_base=base).items()}
            w = Q.NF4Weight.empty(N, K, True, device)
            L = dict(name=name, nseg=nseg, S=S, N=N, K=K, W=W, w=w, X=inp["X"], dY=inp["dY"], A=inp["A"],
                     B=inp["B"],
                     Y=torch.empty(self.M, N, dtype=torch.bfloat16, device=device),
                     dX=torch.empty(self.M, K, dtype=torch.bfloat16, device=device),
                     dA=torch.empty(nseg * self.r, K, dtype=torch.float32, device=device),
                     dB=torch.empty(N, self.r, dtype=torch.float32, device=device))
            self.layers.append(L)
        for L in self.layers:
            ws_need = max(ws_need, Q.qlora_nf4_quantize_workspace(L["N"], L["K"], True),
                          Q.qlora_fused_linear_workspace(self.M, L["w"], L["nseg"], self.r, False),
                          Q.qlora_fused_linear_workspace(self.M, L["w"], L["nseg"], self.r, True))
        self.ws = torch.empty(ws_need, dtype=torch.uint8, device=device)
        self.Q = Q
        self.flops = block_flops(wl, cfg)
        M, r = self.M, self.r
        self.fwd_gemm_flops = sum(2 * M * L["N"] * L["K"] + 2 * M * r * L["N"] for L in self.layers)
        self.dx_gemm_flops = sum(2 * M * L["N"] * L["K"] + 2 * M * L["nseg"] * r * L["K"] for L in self.layers)
        self.quant_bytes = sum(L["N"] * L["K"] * (2 + WEIGHT_BYTES_PER_ELEM) for L in self.layers)
        # LoRA skinny GEMMs per step: forward U; backward U and G; dA and dB
        self.lora_bytes = 0
        for L in self.layers:
            rt, N, K = L["nseg"] * r, L["N"], L["K"]
            self.lora_bytes += ((2 * M * K + 2 * rt * K + 2 * M * rt)
                                + (2 * M * K + 2 * rt * K + 2 * M * N + 2 * N * r + 4 * M * rt)
                                + (2 * M * K + 2 * M * N + 4 * M * rt + 4 * rt * K + 4 * N * r))

    def step(self, adapter=True):
        Q, ws = self.Q, self.ws
        for L in self.layers:
            Q.qlora_nf4_quantize(L["W"], True, out=L["w"], ws=ws)
        for L in self.layers:
            A, B = (L["A"], L["B"]) if adapter else (None, None)
            Q.qlora_fused_linear_fwd(L["X"], L["w"], L["nseg"], A, B, self.s, Y=L["Y"], ws=ws)
        for L in reversed(self.layers):
            if adapter:
                Q.qlora_fused_linear_bwd(L["dY"], L["X"], L["w"], L["nseg"], L["A"], L["B"], self.s, dX=L["dX"],
                                         dA=L["dA"], dB=L["dB"], ws=ws)
            else:
                Q.qlora_fused_linear_bwd(L["dY"], L["X"], L["w"], L["nseg"], None, None, self.s, dX=L["dX"],
                                         ws=ws)


def block_groups(wl, cfg, fused=True):
    """(name, nseg, rows per segment, K) of the block's projections."""
    if fused:
        return wl.FUSED_GROUPS[cfg]
    return [(name, 1, N, K) for name, N, K in wl.CONFIGS[cfg]["linears"]]


def block_flops(wl, cfg):
    c = wl.CONFIGS[cfg]
    return sum(fwd_flops(c["M"], N, K, c["r"]) + bwd_flops(c["M"], N, K, c["r"]) for _, N, K in c["linears"])


def max_over_ranks(torch, value, world, device):
    """The largest of the ranks' values (the slowest rank's time); every rank
    gets it.  One collective, the same on every rank."""
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(flops_per_replica_step, world, ms_per_step):
    """Weak scaling over independent replicas: all ranks' flops per step over
    the slowest rank's step time."""
    return flops_per_replica_step * world / (ms_per_step * 1e-3) / 1e12


def time_steps(torch, fn, steps, flush, dist_barrier):
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    dist_barrier()
    torch.cuda.synchronize()
    for i in range(steps):
        flush()
        starts[i].record()
        fn()
        ends[i].record()
    torch.cuda.synchronize()
    dist_barrier()
    return [s.elapsed_time(e) for s, e in zip(starts, ends)]


def graph_of(torch, fn):
    """A CUDA graph of fn() captured after one untimed run on a side stream."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fn()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    g.replay()
    torch.cuda.synchronize()
    return g


def replay_ms(torch, g, reps, flush):
    """Median device time (ms) of reps graph replays, L2 flushed before each."""
    times = []
    for _ in range(reps):
        flush()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        g.replay()
        e1.record()
        e1.synchronize()
        times.append(e0.elapsed_time(e1))
    return statistics.median(times)


# ---------------------------------------------------------------------------
# end to end through the C ABI
# ---------------------------------------------------------------------------

def e2e_measure(torch, blk, steps, flush, barrier, world, device):
    """The step through the library's C entry points (ctypes, raw pointers),
    with every input copied in from pinned host buffers (W, X, dY of the seven
    linears) and every result copied out to pinned host buffers (Y, dX, dA,
    dB) inside the timed region.  Inputs stream in on one copy stream in the
    order the step uses them, results stream out on another as each call
    finishes; each call waits only for its own inputs."""
    import ctypes
    from bit_nf4_quantized_08_b200 import _lib
    lib = _lib.lib()
    layers = blk.layers
    cws = [L["w"].c_struct() for L in layers]
    hin = {}
    for i, L in enumerate(layers):
        for k in ("W", "X", "dY"):
            h = torch.empty(L[k].shape, dtype=L[k].dtype, pin_memory=True)
            h.copy_(L[k])
            hin[(i, k)] = h
    hout = {(i, k): torch.empty(L[k].shape, dtype=L[k].dtype, pin_memory=True)
            for i, L in enumerate(layers) for k in ("Y", "dX", "dA", "dB")}
    h2d = sum(h.numel() * h.element_size() for h in hin.values())
    d2h = sum(h.numel() * h.element_size() for h in hout.values())
    order = ([(i, "W") for i in range(len(layers))] + [(i, "X") for i in range(len(layers))] +
             [(i, "dY") for i in reversed(range(len(layers)))])
    ev_in = {k: torch.cuda.Event() for k in order}
    ev_fwd = [torch.cuda.Event() for _ in layers]
    ev_bwd = [torch.cuda.Event() for _ in layers]
    up, down = torch.cuda.Stream(device=device), torch.cuda.Stream(device=device)
    ws, ws_bytes = blk.ws.data_ptr(), blk.ws.numel()
    M, r, s = blk.M, blk.r, blk.s

    def call(st, what):
        if st != 0:
            raise RuntimeError(f"{what}: status {st}")

    def step():
        cur = torch.cuda.current_stream()
        hs = ctypes.c_void_p(cur.cuda_stream)
        up.wait_stream(cur)  # the previous step is done with the device buffers
        with torch.cuda.stream(up):
            for key in order:
                i, k = key
                layers[i][k].copy_(hin[key], non_blocking=True)
                ev_in[key].record(up)
        for i, L in enumerate(layers):
            cur.wait_event(ev_in[(i, "W")])
            call(lib.qlora_nf4_quantize(L["W"].data_ptr(), _lib.QLORA_BF16, ctypes.byref(cws[i]), ws, ws_bytes,
                                        hs), "qlora_nf4_quantize")
        for i, L in enumerate(layers):
            cur.wait_event(ev_in[(i, "X")])
            call(lib.qlora_fused_linear_fwd(L["X"].data_ptr(), M, ctypes.byref(cws[i]), L["nseg"],
                                            L["A"].data_ptr(), L["B"].data_ptr(), r, ctypes.c_float(s),
                                            L["Y"].data_ptr(), ws, ws_bytes, hs), "qlora_fused_linear_fwd")
            ev_fwd[i].record(cur)
            down.wait_event(ev_fwd[i])
            with torch.cuda.stream(down):
                hout[(i, "Y")].copy_(L["Y"], non_blocking=True)
        for i in reversed(range(len(layers))):
            L = layers[i]
            cur.wait_event(ev_in[(i, "dY")])
            call(lib.qlora_fused_linear_bwd(L["dY"].data_ptr(), L["X"].data_ptr(), M, ctypes.byref(cws[i]),
                                            L["nseg"], L["A"].data_ptr(), L["B"].data_ptr(), r, ctypes.c_float(s),
                                            L["dX"].data_ptr(), L["dA"].data_ptr(), L["dB"].data_ptr(), ws,
                                            ws_bytes, hs), "qlora_fused_linear_bwd")
            ev_bwd[i].record(cur)
            down.wait_event(ev_bwd[i])
            with torch.cuda.stream(down):
                for k in ("dX", "dA", "dB"):
                    hout[(i, k)].copy_(L[k], non_blocking=True)
        cur.wait_stream(down)  # the results are on the host when the step ends

    step()
    torch.cuda.synchronize()
    n = max(3, min(steps, 5))
    times = time_steps(torch, step, n, flush, barrier)
    ms = max_over_ranks(torch, statistics.mean(times), world, device)
    # the copied-out results are the device results
    for i, L in enumerate(layers):
        for k in ("Y", "dX", "dA", "dB"):
            assert torch.equal(hout[(i, k)].view(torch.int16 if L[k].dtype == torch.bfloat16 else torch.int32),
                               L[k].cpu().view(torch.int16 if L[k].dtype == torch.bfloat16 else torch.int32))
    return {"value": round(whole_job_tflops(blk.flops, world, ms), 2), "unit": "TFLOP/s",
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "ms_per_step": round(ms, 3),
            "method": "C ABI entry points called with raw device pointers (ctypes); W, X, dY of the block's "
                      "projections copied in from pinned host memory on one stream in the order of use, Y, dX, dA, dB "
                      "copied out to pinned host memory on another as each call ends, all inside the timed "
                      "region; the copied-out results equal the device results"}


# ---------------------------------------------------------------------------
# CPU oracle: bounded samples (reported baseline, the reference arm) and the
# check of the GPU's outputs
# ---------------------------------------------------------------------------

def _cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def oracle_sample(torch, wl, cfg, layers=None, rows_n=16, seed=0, fused=True):
    """The oracle on a bounded sample of the block step: for each selected
    projection (default: all of them), full NF4+DQ quantize and dequantize
    of its weight, Y and dX on rows_n sampled token rows, dA and dB in full
    (all M rows).  Input generation is not timed.  Returns a dict with the
    sample's flops, its seconds (quantize/dequantize and the products
    separately), the sampled rows and, per projection, the oracle's outputs."""
    from oracle import oracle as O
    O.build()
    c = wl.CONFIGS[cfg]
    M, r, s = c["M"], c["r"], c["alpha"] / c["r"]
    rows = wl.sample_rows(M, rows_n, seed=seed)
    R = rows.size
    out = {"flops": 0, "quant_s": 0.0, "gemm_s": 0.0, "rows": rows, "layers": {}}
    for gi, (name, nseg, S, K) in enumerate(block_groups(wl, cfg, fused)):
        if layers is not None and gi not in layers:
            continue
        base = 10 * gi
        N = nseg * S
        W = wl.weight(N, K, seed=seed, dtype=torch.bfloat16, index_base=base)
        inp = wl.fused_inputs(M, nseg, S, K, r, seed=seed, index_base=base)
        Xb, dYb, Ab, Bb = (wl.bits(inp[k]) for k in ("X", "dY", "A", "B"))
        Wbits = wl.bits(W).reshape(-1)
        del W, inp
        t0 = time.perf_counter()
        q = O.nf4_quantize(Wbits, double_quant=True)
        Wd = O.nf4_dequantize(N * K, q).reshape(N, K)
        t1 = time.perf_counter()
        Y = O.fused_linear_fwd(Xb, Wd, Ab, Bb, s, nseg, rows=rows)
        dX, dA, dB = O.fused_linear_bwd(dYb, Xb, Wd, Ab, Bb, s, nseg, rows=rows)
        t2 = time.perf_counter()
        out["quant_s"] += t1 - t0
        out["gemm_s"] += t2 - t1
        out["flops"] += nseg * (R * (2 * S * K + 2 * r * (K + S))      # forward rows
                                + R * (2 * S * K + 2 * r * K)          # dX rows
                                + 2 * M * r * (K + S)                  # U and G over all rows
                                + 2 * M * r * K + 2 * M * S * r)       # dA, dB
        out["layers"][gi] = {"codes": q["codes"], "q8": q["q8"], "Y": Y, "dX": dX, "dA": dA, "dB": dB}
    out["seconds"] = out["quant_s"] + out["gemm_s"]
    return out


def _ratios(got, ref):
    import numpy as np
    d = np.asarray(got, np.float64) - ref
    return (float(np.max(np.abs(d)) / max(np.max(np.abs(ref)), 1e-300)),
            float(np.linalg.norm(d) / max(np.linalg.norm(ref), 1e-300)))


def oracle_check(blk, sample):
    """GPU outputs of the step against the oracle sample: codes and 8-bit
    constants bit for bit, Y and dX on the sampled rows, dA and dB in full,
    at max|d| <= 1e-2 max|ref| and ||d||_F <= 5e-3 ||ref||_F."""
    import numpy as np
    rows = sample["rows"]
    worst = {"max_ratio": 0.0, "frob_ratio": 0.0}
    bitexact = True
    for li, ref in sample["layers"].items():
        L = blk.layers[li]
        bitexact &= bool(np.array_equal(L["w"].codes.cpu().numpy(), ref["codes"]))
        bitexact &= bool(np.array_equal(L["w"].absmax_q8.cpu().numpy(), ref["q8"]))
        for k in ("Y", "dX", "dA", "dB"):
            got = L[k].float().cpu().numpy()
            if k in ("Y", "dX"):
                got = got[rows]
            mr, fr = _ratios(got, ref[k])
            worst["max_ratio"] = max(worst["max_ratio"], mr)
            worst["frob_ratio"] = max(worst["frob_ratio"], fr)
    ok = bitexact and worst["max_ratio"] <= 1e-2 and worst["frob_ratio"] <= 5e-3
    return {"ok": ok, "quantize_bit_exact": bitexact, "worst_max_abs_err_over_max_ref": round(worst["max_ratio"], 6),
            "worst_frob_err_over_frob_ref": round(worst["frob_ratio"], 6),
            "compared": f"codes and q8 of all {len(sample['layers'])} projection weights bit for bit; Y and dX on "
                        f"{rows.size} sampled token rows, dA and dB in full"}


def cpu_baseline(torch, wl, cfg, gpu_block=None):
    """The oracle timed on the host's cores: the bounded sample on all cores
    (its outputs also checked against the GPU's when a block is given), the
    first linear's sample on one core, and the full step's time extrapolated
    from the all-core rates (labelled as such)."""
    from oracle import oracle as O
    O.build()
    threads = O.num_threads()
    smp = oracle_sample(torch, wl, cfg)
    check = oracle_check(gpu_block, smp) if gpu_block is not None else None
    O.set_num_threads(1)
    try:
        one = oracle_sample(torch, wl, cfg, layers=[1])
    finally:
        O.set_num_threads(threads)
    c = wl.CONFIGS[cfg]
    full_flops = block_flops(wl, cfg)
    sampled_gemm_rate = smp["flops"] / smp["gemm_s"]
    extrap_s = smp["quant_s"] + full_flops / sampled_gemm_rate
    base = {"value": smp["flops"] / smp["seconds"] / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
            "sample": f"every projection of the {cfg} block (7 linears as q/k/v, o, gate/up, down; M={c['M']}, "
                      f"r={c['r']}): full NF4+DQ quantize and dequantize of W, Y and dX on {smp['rows'].size} "
                      f"of {c['M']} token rows, dA and dB in full",
            "seconds": round(smp["seconds"], 2), "cpu_model": _cpu_model(), "nproc": os.cpu_count(),
            "single_thread": {"value": one["flops"] / one["seconds"] / 1e12, "unit": "TFLOP/s", "cores": 1,
                              "seconds": round(one["seconds"], 2),
                              "sample": "the same sample for the o projection (8192x8192 for the 65B block) only"},
            "all_cores": {"value": smp["flops"] / smp["seconds"] / 1e12, "unit": "TFLOP/s", "cores": threads},
            "full_step_seconds_extrapolated": round(extrap_s, 1),
            "extrapolation": "extrapolated: measured quantize+dequantize time of the block's weights plus the full "
                             "step's fwd+bwd flops at the sample's all-core product rate"}
    return base, check


# ---------------------------------------------------------------------------
# extras: 7B block, stress forward, small-M sweep, 2^30 quantize / dequantize
# ---------------------------------------------------------------------------

def extras(torch, Q, wl, device, flush, peaks):
    out = {}
    # the LLaMA-7B decoder block (the same step, smaller shapes), and both
    # blocks as seven separate linears (one weight and one call each)
    for key, cfg, fused in (("llama7b_block_step_cuda_graph", "llama7b", True),
                            ("llama7b_block_7_separate_linears_cuda_graph", "llama7b", False),
                            ("llama65b_block_7_separate_linears_cuda_graph", "llama65b", False)):
        blk = Block(torch, Q, wl, device, cfg=cfg, fused=fused)
        for _ in range(3):
            blk.step()
        g = graph_of(torch, blk.step)
        ms = replay_ms(torch, g, 10, flush)
        del g
        tf = blk.flops / (ms * 1e-3) / 1e12
        out[key] = {"workload": WORKLOADS[cfg] if fused else WORKLOADS[cfg].split(";")[0] + "; separate calls",
                    "ms": round(ms, 4), "TFLOPs": round(tf, 1), "frac_bf16_peak": round(tf / peaks["bf16_tflops"], 3)}
        del blk
        torch.cuda.empty_cache()

    # stress forward: 4096x4096 weight with outliers, 2048 tokens, r = 16
    c = wl.CONFIGS["stress"]
    (_, N, K), = c["linears"]
    M, r, s = c["M"], c["r"], c["alpha"] / c["r"]
    W = wl.weight(N, K, seed=0, dtype=torch.bfloat16, outlier_frac=c["outlier_frac"],
                  outlier_std=c["outlier_std"]).to(device)
    w = Q.qlora_nf4_quantize(W)
    inp = {k: v.to(device) for k, v in wl.linear_inputs(M, N, K, r, seed=0).items()}
    Y = torch.empty(M, N, dtype=torch.bfloat16, device=device)
    ws = torch.empty(Q.qlora_linear_workspace(M, w, r, False), dtype=torch.uint8, device=device)
    fn = lambda: Q.qlora_linear_fwd(inp["X"], w, inp["A"], inp["B"], s, Y=Y, ws=ws)  # noqa: E731
    for _ in range(3):
        fn()
    g = graph_of(torch, fn)
    ms = replay_ms(torch, g, 20, flush)
    del g
    tf = fwd_flops(M, N, K, r) / (ms * 1e-3) / 1e12
    out["stress_fwd_4096x4096_M2048_r16_cuda_graph"] = {
        "us": round(ms * 1e3, 2), "TFLOPs": round(tf, 1), "frac_bf16_peak": round(tf / peaks["bf16_tflops"], 3)}
    del W, w, inp, Y, ws

    c = wl.CONFIGS["sweep"]
    (_, N, K), = c["linears"]
    r, s = c["r"], c["alpha"] / c["r"]
    W = wl.weight(N, K, seed=0, dtype=torch.bfloat16).to(device)
    w = Q.qlora_nf4_quantize(W)
    del W
    sweep = {}
    for M in c["Ms"]:
        inp = {k: v.to(device) for k, v in wl.linear_inputs(M, N, K, r, seed=0).items()}
        X, A, B = inp["X"], inp["A"], inp["B"]
        Y = torch.empty(M, N, dtype=torch.bfloat16, device=device)
        ws = torch.empty(Q.qlora_linear_workspace(M, w, r, False), dtype=torch.uint8, device=device)
        fn = lambda: Q.qlora_linear_fwd(X, w, A, B, s, Y=Y, ws=ws)  # noqa: E731
        for _ in range(3):
            fn()
        g = graph_of(torch, fn)
        ms = replay_ms(torch, g, 20, flush)
        del g
        wbytes = N * K * WEIGHT_BYTES_PER_ELEM
        total = wbytes + M * K * 2 + r * K * 2 + N * r * 2 + M * N * 2
        sweep[str(M)] = {"us": round(ms * 1e3, 2), "weight_GBps": round(wbytes / ms / 1e6, 1),
                         "total_GBps": round(total / ms / 1e6, 1),
                         "frac_hbm": round(total / ms / 1e6 / peaks["hbm_gbs"], 3)}
    out["small_m_fwd_22016x8192_r64_cuda_graph"] = sweep

    # LoRA merge of the same weight (dequantize + s B A, bf16 out)
    A = wl.linear_inputs(1, N, K, r, seed=0)["A"].to(device)
    B = wl.linear_inputs(1, N, K, r, seed=0)["B"].to(device)
    Wm = torch.empty(N, K, dtype=torch.bfloat16, device=device)
    fn = lambda: Q.qlora_lora_merge(w, A, B, s, out=Wm)  # noqa: E731
    for _ in range(3):
        fn()
    g = graph_of(torch, fn)
    ms = replay_ms(torch, g, 20, flush)
    del g
    mbytes = N * K * (WEIGHT_BYTES_PER_ELEM + 2) + (N + K) * r * 2
    out["lora_merge_22016x8192_r64_cuda_graph"] = {
        "us": round(ms * 1e3, 1), "GBps": round(mbytes / ms / 1e6, 1),
        "frac_hbm": round(mbytes / ms / 1e6 / peaks["hbm_gbs"], 3), "algorithmic_bytes": int(mbytes)}
    del Wm, A, B, w

    # AdamW step over every adapter parameter of the LLaMA-65B block (A and B
    # of the 7 linears as one flat buffer): 16 B read + 14 B written each
    npar = sum(nseg * 64 * K + nseg * S * 64 for _, nseg, S, K in block_groups(wl, "llama65b"))
    pf = torch.randn(npar, device=device) * 0.01
    mf, vf, gf = torch.zeros_like(pf), torch.zeros_like(pf), torch.randn(npar, device=device) * 1e-3
    pb = torch.empty(npar, dtype=torch.bfloat16, device=device)
    fn = lambda: Q.qlora_adamw_step(pf, mf, vf, gf, pb, lr=1e-4, step=10, weight_decay=0.01)  # noqa: E731
    for _ in range(3):
        fn()
    g = graph_of(torch, fn)
    ms = replay_ms(torch, g, 20, flush)
    del g
    abytes = 30 * npar
    out["adamw_llama65b_block_adapters_cuda_graph"] = {
        "params": int(npar), "us": round(ms * 1e3, 1), "GBps": round(abytes / ms / 1e6, 1),
        "frac_hbm": round(abytes / ms / 1e6 / peaks["hbm_gbs"], 3), "algorithmic_bytes": int(abytes)}
    del pf, mf, vf, gf, pb

    n = c["big_numel"]
    Wbig = wl.weight(n // 8192, 8192, seed=0, dtype=torch.bfloat16).to(device)
    qb = Q.NF4Weight.empty(n // 8192, 8192, True, device)
    wsq = torch.empty(Q.qlora_nf4_quantize_workspace(n // 8192, 8192, True), dtype=torch.uint8, device=device)
    deq = torch.empty(n // 8192, 8192, dtype=torch.bfloat16, device=device)
    algo = n * (2 + WEIGHT_BYTES_PER_ELEM)
    for name, fn in (("quantize_2^30_bf16", lambda: Q.qlora_nf4_quantize(Wbig, True, out=qb, ws=wsq)),
                     ("dequantize_2^30_bf16", lambda: Q.qlora_nf4_dequantize(qb, out=deq))):
        for _ in range(3):
            fn()
        # one call captured in a CUDA graph and replayed, as the step: device
        # time of the call's kernels, without the host's launch cost
        g = graph_of(torch, fn)
        ms = replay_ms(torch, g, 5, flush)
        del g
        out[name + "_cuda_graph"] = {"us": round(ms * 1e3, 1), "GBps": round(algo / ms / 1e6, 1),
                                     "frac_hbm": round(algo / ms / 1e6 / peaks["hbm_gbs"], 3),
                                     "algorithmic_bytes": int(algo)}
    del Wbig, qb, deq, wsq
    return out


# ---------------------------------------------------------------------------

def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        return run_reference(args, world, rank)
    if args.profile_case:
        return run_profile_case(args.profile_case, args.block)

    import torch
    import torch.distributed as dist
    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=device)

    def barrier():
        if world > 1:
            dist.barrier()

    from bit_nf4_quantized_08_b200 import build as qbuild
    if rank == 0 or world == 1:
        qbuild.build()
    barrier()
    import bit_nf4_quantized_08_b200 as Q
    from bit_nf4_quantized_08_b200 import workloads as wl

    peaks, peak_src = load_peaks()
    flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device=device)

    def flush():
        flush_buf.fill_(1)

    blk = Block(torch, Q, wl, device, cfg=HEADLINE, seed=rank)
    for _ in range(max(3, args.warmup)):
        blk.step()
    torch.cuda.synchronize()
    assert Q.qlora_get_last_error() == 0

    # kernels of one step (the host launch counter of an eager step)
    l0 = Q.qlora_kernel_launches()
    blk.step()
    launches_per_step = Q.qlora_kernel_launches() - l0
    # eager steps: the host launches every kernel of the step
    eager_times = time_steps(torch, blk.step, min(args.steps, 5), flush, barrier)
    # the timed steps replay one CUDA graph of the step (no host launch cost)
    graph = graph_of(torch, blk.step)

    clocks = ClockSampler(local_rank)
    clocks.start()
    times = time_steps(torch, graph.replay, args.steps, flush, barrier)
    clk = clocks.stop()
    launches = launches_per_step * args.steps
    status = Q.qlora_get_last_error()
    assert status == 0, f"device status {status}"
    del graph
    # the same step without the adapter (r = 0), also a graph replay: the
    # difference is the step time the LoRA GEMMs still add
    base_graph = graph_of(torch, lambda: blk.step(adapter=False))
    base_ms = max_over_ranks(torch, sum(time_steps(torch, base_graph.replay, args.steps, flush, barrier)),
                             world, device) / args.steps
    del base_graph
    # per-kernel device times from a separate eager pass with launch events
    Q.qlora_profile_enable(True)
    time_steps(torch, blk.step, args.steps, flush, barrier)
    prof = {k: Q.qlora_profile_read(k) for k in ("quantize", "fwd_gemm", "dx_gemm", "lora_gemm")}
    Q.qlora_profile_enable(False)

    total_ms = max_over_ranks(torch, sum(times), world, device)
    ms_per_step = total_ms / args.steps
    value = whole_job_tflops(blk.flops, world, ms_per_step)

    # dominant kernel: the tracked kind with the largest device time
    dom = max(("fwd_gemm", "dx_gemm"), key=lambda k: prof[k][0])
    dom_ms, dom_n = prof[dom]
    dom_flops = (blk.fwd_gemm_flops if dom == "fwd_gemm" else blk.dx_gemm_flops) * args.steps
    achieved = dom_flops / (dom_ms * 1e-3) / 1e12
    peak = peaks["bf16_tflops"]
    traffic = load_traffic(dom)
    roofline = {"bound": "tensor", "kernel": f"k_gemm_pair ({dom.replace('_', ' ')}, NF4 dequant in producer)",
                "achieved": round(achieved, 1), "peak": peak, "unit": "TFLOP/s",
                "frac": round(achieved / peak, 4), "traffic": traffic,
                "peak_source": f"{peak_src} bf16 dense (burst)",
                "frac_of_sustained": round(achieved / peaks.get("bf16_tflops_sustained", peak), 4),
                "launches": dom_n, "avg_launch_us": round(dom_ms / max(dom_n, 1) * 1e3, 2)}
    breakdown = {}
    qms, qn = prof["quantize"]
    if qn:
        breakdown["quantize_GBps"] = round(blk.quant_bytes * args.steps / (qms * 1e-3) / 1e9, 1)
        breakdown["quantize_frac_hbm"] = round(breakdown["quantize_GBps"] / peaks["hbm_gbs"], 3)
    lms, ln = prof["lora_gemm"]
    if ln:
        # event times of kernels that run beside the dequant GEMMs (dependent
        # launch, side stream): their sum overlaps the GEMMs' times
        breakdown["lora_gemm_GBps"] = round(blk.lora_bytes * args.steps / (lms * 1e-3) / 1e9, 1)
        breakdown["lora_gemm_frac_hbm"] = round(breakdown["lora_gemm_GBps"] / peaks["hbm_gbs"], 3)
        breakdown["lora_gemm_overlapped_share"] = round(lms / total_ms, 3)
    breakdown["step_ms_without_adapter"] = round(base_ms, 4)
    breakdown["adapter_added_ms"] = round(ms_per_step - base_ms, 4)
    for k in ("fwd_gemm", "dx_gemm"):
        ms_k, n_k = prof[k]
        fl = (blk.fwd_gemm_flops if k == "fwd_gemm" else blk.dx_gemm_flops) * args.steps
        if n_k:
            breakdown[k + "_TFLOPs"] = round(fl / (ms_k * 1e-3) / 1e12, 1)
            breakdown[k + "_share_of_step"] = round(ms_k / total_ms, 3)

    e2e = e2e_measure(torch, blk, args.steps, flush, barrier, world, device)

    # the oracle on the host cores (rank 0 only), its outputs compared with
    # the GPU's outputs of this step
    cpu, check = None, None
    if rank == 0 and not args.no_cpu:
        blk.step()
        torch.cuda.synchronize()
        cpu, check = cpu_baseline(torch, wl, HEADLINE, gpu_block=blk)

    extra = None
    if not args.no_extras:
        del blk
        torch.cuda.empty_cache()
        extra = extras(torch, Q, wl, device, flush, peaks)

    if world > 1:
        dist.barrier()
    if rank == 0:
        c = wl.CONFIGS[HEADLINE]
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": round(ms_per_step, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": WORKLOAD, "global_batch": c["M"] * world, "seq_len": c["M"],
                       "flops_per_step": block_flops(wl, HEADLINE), "l2": "flushed between steps (256 MiB write)",
                       "parallelism": f"replicas x{world}" if world > 1 else "1 GPU",
                       "launch": "one CUDA graph per step (captured from the library calls)",
                       "eager_ms_per_step": round(sum(eager_times) / len(eager_times), 4)},
            "roofline": roofline, "breakdown": breakdown, "cpu_baseline": cpu, "oracle_check": check,
            "e2e": e2e, "gpu_launches": int(launches), "clocks": clk, "extra": extra,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def run_profile_case(case, block_cfg):
    """A small case of one kernel, launched three times: the gate-shaped
    linear (11008x4096, M=2048, r=64) for the GEMMs, 2^26 elements for the
    quantizer, the 22016x8192 weight at M=16 for the small-M forward; the
    *_block cases run each linear of one decoder block once."""
    import torch
    from bit_nf4_quantized_08_b200 import build as qbuild
    qbuild.build()
    import bit_nf4_quantized_08_b200 as Q
    from bit_nf4_quantized_08_b200 import workloads as wl
    dev = torch.device("cuda", 0)
    if case in ("fwd_block", "dx_block"):
        cfg = wl.CONFIGS[block_cfg]
        M, r, s = cfg["M"], cfg["r"], cfg["alpha"] / cfg["r"]
        for i, (_, nseg, S, K) in enumerate(block_groups(wl, block_cfg)):
            W = wl.weight(nseg * S, K, seed=0, dtype=torch.bfloat16, device=dev, index_base=10 * i)
            w = Q.qlora_nf4_quantize(W)
            del W
            inp = wl.fused_inputs(M, nseg, S, K, r, seed=0, device=dev, index_base=10 * i)
            if case == "dx_block":
                Q.qlora_fused_linear_bwd(inp["dY"], inp["X"], w, nseg, inp["A"], inp["B"], s)
            else:
                Q.qlora_fused_linear_fwd(inp["X"], w, nseg, inp["A"], inp["B"], s)
            del w, inp
    elif case in ("quantize", "dequantize"):
        W = wl.weight(1 << 13, 1 << 13, seed=0, dtype=torch.bfloat16, device=dev)
        w = Q.qlora_nf4_quantize(W)
        for _ in range(3):
            if case == "quantize":
                Q.qlora_nf4_quantize(W, True, out=w)
            else:
                Q.qlora_nf4_dequantize(w)
    else:
        N, K, M = (22016, 8192, 16) if case == "smallm" else (11008, 4096, 2048)
        r, s = 64, 0.25
        W = wl.weight(N, K, seed=0, dtype=torch.bfloat16, device=dev)
        w = Q.qlora_nf4_quantize(W)
        inp = wl.linear_inputs(M, N, K, r, seed=0, device=dev)
        for _ in range(3):
            if case == "dx":
                Q.qlora_linear_bwd(inp["dY"], inp["X"], w, inp["A"], inp["B"], s)
            else:
                Q.qlora_linear_fwd(inp["X"], w, inp["A"], inp["B"], s)
    torch.cuda.synchronize()
    assert Q.qlora_get_last_error() == 0
    print("profile case", case, "ok")
    return 0


def run_reference(args, world, rank):
    """Reference arm: the CPU oracle, as it stands, on the host cores.  Each
    step is the oracle's bounded sample of one linear of the block (the seven
    in turn): full quantize + dequantize of its weight, Y and dX on 16 sampled
    token rows, dA and dB in full.  Rank 0 only."""
    if rank != 0:
        return 0
    import torch
    from bit_nf4_quantized_08_b200 import workloads as wl
    from oracle import oracle as O
    O.build()
    nlin = len(block_groups(wl, HEADLINE))
    for i in range(max(0, min(args.warmup, 1))):
        oracle_sample(torch, wl, HEADLINE, layers=[i % nlin])
    tot_flops, tot_s = 0, 0.0
    for i in range(args.steps):
        smp = oracle_sample(torch, wl, HEADLINE, layers=[i % nlin])
        tot_flops += smp["flops"]
        tot_s += smp["seconds"]
    value = tot_flops / tot_s / 1e12
    threads = O.num_threads()
    desc = ("per step, one projection of the block in turn (q/k/v, o, gate/up, down; M=2048, r=64): full NF4+DQ "
            "quantize and dequantize of its weight, Y and dX on 16 of 2048 token rows, dA and dB in full")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": tot_s / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": WORKLOAD + " (bounded CPU sample per step)"},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": desc,
                             "cpu_model": _cpu_model()},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main() or 0)
