#!/usr/bin/env python
"""Throughput of the chunkwise linear-recurrence layer, forward + backward.

One step = the forward sub-sequence driver (sf_fwd_seq) and the backward one
(sf_bwd_seq) over one batch of the workload, the gated delta rule with H=32,
d=128, T=65536 cut into 16 sub-sequences of 4096 by default.  Prints one JSON
line (rank 0).  ``--impl reference`` times the fp64 CPU oracle instead.

Multi-GPU: one process per GPU (torchrun); every rank runs its own independent
copy of the workload (heads and batches are independent, so there is no
exchange on the data path): weak scaling, value = all ranks' tokens / the
slowest rank's time.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from chunked_linear_recurrence_chunkwise_b200 import inputs  # noqa: E402

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}


# ------------------------------------------------------------------ host logic
def parse_args(argv=None):
    p = argparse.ArgumentParser(description=__doc__)
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=10)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", default="sf", choices=["sf", "reference"])
    p.add_argument("--workload", default=inputs.BENCH_WORKLOAD, choices=list(inputs.WORKLOADS))
    p.add_argument("--mode", default="keep", choices=["keep", "recompute"],
                   help="keep: the forward keeps its intermediates for the backward; recompute: "
                        "the backward recomputes every piece from its stored entering state")
    p.add_argument("--no-other-mode", action="store_true",
                   help="do not time the other driver form beside the headline one")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-graph", action="store_true",
                   help="time the driver calls launched eagerly instead of a CUDA-graph replay of them "
                        "(the eager time is reported beside the graph one otherwise)")
    p.add_argument("--memory-study", default=None, metavar="T1,T2,...",
                   help="instead of the bench line: the layer's device memory and step time for these "
                        "sequence lengths at a fixed piece length of 4096 tokens (one JSON line)")
    p.add_argument("--no-plan", action="store_true",
                   help="skip timing the profile-guided cut (sf_plan_cut) beside the workload's own cut")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-sample-tokens", type=int, default=16384)
    p.add_argument("--tokens", type=int, default=None,
                   help="override T (a smaller case of the same workload, e.g. for ncu captures)")
    p.add_argument("--heads", type=int, default=None, help="override H")
    return p.parse_args(argv)


def dist_env():
    """(rank, world, local_rank) from the torchrun environment."""
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def rank_workload(w, rank: int):
    """Each rank gets an independent problem of the same shape (its own seed)."""
    return w if rank == 0 else w.scaled(seed=w.seed + 7919 * rank)


def reduce_max(value: float, group=None, device=None) -> float:
    """Max of a float over the ranks of the default process group (identity if none)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())


def job_tokens_per_s(world: int, B: int, T: int, ms_max: float) -> float:
    """Whole-job throughput: every rank processed B*T tokens; the slowest rank sets the time."""
    return world * B * T / (ms_max / 1e3)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return pk, "measured"
    except OSError:
        return dict(PEAKS_FALLBACK), "fallback"


def tc_path(w) -> bool:
    """The tensor-core kernels serve bf16 with d_k = d_v = 128; everything else is SIMT."""
    return w.dtype == "bf16" and w.d == 128


# Per token-head, with C = 64 and d = d_k = d_v: u = 2 C d and v = 2 d^2 flops.  The
# method's algorithmic work is counted triangle-aware (a product with a causal C x C
# factor at half its square size), step by step of the chunkwise algorithm:
#   forward:  A = K K^T, W, U (1.5 u); state pass W S and Ktil^T Delta (2 v);
#             output P = Q K^T and P Delta (u), Q S (v)            -> 2.5 u + 3 v
#   backward: reverse pass P^T dO (0.5 u), Ktil dS', Qtil^T dO, W^T dDelta (3 v);
#             gradients dP, F K, F^T Q, dKhat, dVhat, dA (two), (E + E^T) K (4.5 u),
#             dO S^T, dDelta S^T, Delta dS'^T (3 v)                 -> 5 u + 6 v
# (linear attention drops the delta-rule terms).  These are the canonical counts of
# the workload's headline TFLOP/s; what a kernel issues on full tiles is reported
# beside them.
def canonical_flops(name: str, w) -> float:
    """Triangle-aware algorithmic flops of one chunk-head (64 tokens of one head)
    that kernel `name` carries, from the per-token-head counts above."""
    C, d = 64, w.d
    u, v = 2.0 * C * d, 2.0 * d * d
    delta = w.has_beta
    per_token = {
        "intra_fwd": 1.5 * u if delta else 0.0,
        "intra_bwd": (1.5 * u if delta else 0.0) + 0.5 * u,   # also forms P
        "state_fwd": 2 * v if delta else v,
        "output": u + v,
        "output_p": 0.5 * u + v,                               # P read, not formed
        "state_bwd": 0.5 * u + (3 * v if delta else 2 * v),
        "grad_fused": 4.5 * u + 3 * v,
        "grad_attn": 1.5 * u + 2 * v,
    }.get(name, 0.0)
    return per_token * C


def layer_io_bytes_per_token_head(w) -> dict:
    """The layer's own I/O per token-head (the minimum traffic of an ideally fused
    layer): forward reads q, k, v, g, beta and writes o; backward reads q, k, v, g,
    beta, dO and writes dq, dk, dv, dg, dbeta."""
    e = 2 if w.dtype == "bf16" else 4
    dk = dv = w.d
    gb = 4 * (int(w.has_g) + int(w.has_beta))
    fwd = (2 * dk + dv) * e + gb + dv * e
    bwd = (2 * dk + 2 * dv) * e + gb + (2 * dk + dv) * e + gb
    return {"fwd": fwd, "bwd": bwd, "total": fwd + bwd}


def kernel_units(name: str, w, mode: str = "keep") -> dict:
    """Bytes and flops of one chunk-head (64 tokens of one head) per kernel.

    io_bytes: the layer I/O tensors (q, k, v, g, beta, dO read; o, dq, dk, dv, dg,
    dbeta written) that this kernel reads or writes, each once: the kernel's share
    of the layer's minimum traffic.  design_bytes: every tensor the kernel must read
    or write once at the precision the path stores it, intermediates included
    (W^T, U^T, chunk states, Delta, P, T ... in bf16 on the tensor-core path; g,
    beta, the cumulative decay fp32).  flops: the canonical triangle-aware count
    (canonical_flops); flops_issued: 2 x the multiply-adds of the products as the
    kernel issues them on full tiles.
    """
    C, d = 64, w.d
    f = 4
    gb = C * f * (int(w.has_g) + int(w.has_beta))   # g and beta of one chunk-head
    if tc_path(w) and name == "output" and mode == "keep":
        name = "output_p"  # the forward that keeps P runs the output kernel that reads it
    if tc_path(w):
        e = 2                       # bf16 I/O and intermediates
        tile = C * d * e            # one 64 x 128 bf16 tile: 16 KB
        st = d * d * e              # one chunk state, bf16: 32 KB
        mm = lambda m, n, k: 2 * m * n * k
        # (io_bytes, design_bytes, issued flops)
        tab = {
            # read k, v, g, beta; write G, W^T, U^T
            "intra_fwd": (2 * tile + gb, 2 * tile + 2 * C * f + C * f + 2 * tile,
                          mm(C, C, d) + 2 * mm(d, C, C)),
            # as intra_fwd, also reading q and writing P (and T for the delta rule)
            "intra_bwd": (3 * tile + gb, 3 * tile + 2 * C * f + C * f + 2 * tile
                          + (2 if w.has_beta else 1) * C * C * e,
                          mm(2 * C, C, d) + 2 * mm(d, C, C)),
            # read W^T, U^T, k, decay table; write S^T, Delta^T
            "state_fwd": (tile, 3 * tile + 2 * C * f + st + tile, mm(d, C, d) + mm(d, d, C)),
            # read q, k, S^T, Delta^T, G; write o (P recomputed on chip)
            "output": (3 * tile, 2 * tile + st + tile + C * f + tile,
                       mm(C, C, d) + mm(d, C, d) + mm(d, C, C)),
            # read q, S^T, Delta^T, the stored P, G; write o
            "output_p": (2 * tile, tile + st + tile + C * C * e + C * f + tile,
                         mm(d, C, d) + mm(d, C, C)),
            # read k, dO, q, W^T, P, G; write dS'^T, dDelta^T
            "state_bwd": (3 * tile, 4 * tile + C * C * e + C * f + st + tile,
                          mm(d, C, d) + mm(d, C, C) + 2 * mm(d, d, C)),
            # read q, k, dO, Delta^T (= V^T), S^T, dS'^T, G; write dq, dk, dg
            "grad_attn": (4 * tile + C * f + 2 * tile + C * f,
                          4 * tile + 2 * st + C * f + 2 * tile + C * f,
                          2 * mm(C, C, d) + 2 * mm(C, d, d) + 2 * mm(C, d, C)),
            # read q, k, v, dO, T, Delta^T, dDelta^T, S^T, dS'^T, G, beta;
            # write dq, dk, dv, dg, dbeta
            "grad_fused": (4 * tile + gb + 3 * tile + gb,
                           6 * tile + C * C * e + 2 * st + 2 * C * f + 3 * tile + 2 * C * f,
                           4 * mm(C, C, d) + 3 * mm(C, d, d) + 4 * mm(C, d, C)),
        }
    else:
        e = 2 if w.dtype == "bf16" else 4
        t1 = C * d * e
        tri_s = C * (C - 1) // 2
        tri_i = C * (C + 1) // 2
        tab = {
            "intra_fwd": (2 * t1 + gb, 2 * C * d * e + 3 * C * f + 2 * C * d * e, tri_s * 2 * d * 3),
            "state_fwd": (t1, 3 * C * d * e + C * f + d * d * e + C * d * e, 4 * C * d * d),
            "output": (2 * t1, 3 * C * d * e + C * f + d * d * e + C * d * e, tri_i * 4 * d + 2 * C * d * d),
            "dd_pre": (2 * t1, 3 * C * d * e + C * f + C * d * e, tri_i * 4 * d),
            "state_bwd": (3 * t1, 5 * C * d * e + C * f + d * d * e + C * d * e, 6 * C * d * d),
            "grad_delta": (2 * t1 + gb + t1 + C * f, 6 * C * d * e + d * d * e + C * d * f + 3 * C * f,
                           tri_s * 12 * d + 2 * C * d * d),
            "grad_attn": (3 * t1 + C * f + 2 * t1 + C * f, 5 * C * d * e + 2 * d * d * e + C * d * f + 2 * C * f,
                          tri_i * 8 * d + 4 * C * d * d),
        }
    io, design, fl = tab.get(name, (0, 0, 0))
    return {"io_bytes": io, "design_bytes": design, "flops": canonical_flops(name, w), "flops_issued": fl}


# DRAM bytes (read + write) per launch of one 4096-token piece of the 32-head, d = 128
# workload (2048 chunk-heads) from an ncu capture, per kernel, with `source_sha` of the
# source file the kernel was built from at the time of the capture (its code, comments
# left out).  A kernel whose code has changed since reports traffic null.
NCU_TRAFFIC_2048 = {
    # name: (bytes per 2048 chunk-heads, source file, source_sha); profiles/<kernel>_*.md
    "grad_fused": (432559104, "sf_tc_grad_fused.cu", "1eb9c2de37a51998"),
    "grad_attn": (321560320, "sf_tc_grad.cu", "48e6df666c2d3748"),
    "state_fwd": (163520512, "sf_tc_state.cu", "bcaa1eef5ea3178a"),
    "state_bwd": (224162304, "sf_tc_state.cu", "bcaa1eef5ea3178a"),
}
KERNEL_SOURCE = {
    "grad_fused": "sf_tc_grad_fused.cu", "state_fwd": "sf_tc_state.cu", "state_bwd": "sf_tc_state.cu",
    "intra_bwd": "sf_tc_chunk.cu", "intra_fwd": "sf_tc_chunk.cu", "output": "sf_tc_chunk.cu",
    "grad_attn": "sf_tc_grad.cu",
}


def code_of(text: str) -> str:
    """C/CUDA source without its comments, whitespace runs collapsed to one space
    (string and character literals kept as written)."""
    out, i, n = [], 0, len(text)
    while i < n:
        ch = text[i]
        if ch in "\"'":
            j = i + 1
            while j < n and text[j] != ch:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
        else:
            out.append(ch)
            i += 1
    return " ".join("".join(out).split())


def source_sha(fname: str) -> str | None:
    """sha256 (first 16 hex digits) of a kernel source's code, comments left out, so
    that the traffic of a capture stays attached to its code through comment edits."""
    import hashlib
    path = os.path.join(ROOT, "chunked_linear_recurrence_chunkwise_b200", "csrc", fname)
    try:
        with open(path, encoding="utf-8") as f:
            return hashlib.sha256(code_of(f.read()).encode()).hexdigest()[:16]
    except OSError:
        return None


def measured_traffic(name: str, units_per_launch: float, w, mode: str):
    """DRAM bytes per launch from the committed capture, or None when there is none for
    this kernel on this path or the kernel's source has changed since it was taken."""
    ent = NCU_TRAFFIC_2048.get(name)
    if not ent or not tc_path(w):
        return None
    nbytes, fname, sha = ent
    if source_sha(fname) != sha:
        return None
    return round(nbytes * units_per_launch / 2048)


def kernel_rooflines(timing: dict, w, steps: int, peaks: dict, mode: str = "keep") -> dict:
    """Every kernel of the serialized pass: launches and time per step, and per launch
    its bandwidth on the layer's own I/O (io) and on everything it moves (design), and
    its canonical and issued tensor throughput, with fractions of the measured peaks
    (HBM copy bandwidth; burst bf16 GEMM rate: the timed pass runs well under a second
    at full clock)."""
    chunk_heads = w.B * w.H * ((w.T + 63) // 64)
    units_per_launch = chunk_heads / w.n_sub
    hbm = float(peaks["hbm_gbs"])
    bf16 = float(peaks.get("bf16_tflops", 1590.0))
    out = {}
    for name, (launches, ms) in timing.items():
        if launches <= 0:
            continue
        u = kernel_units(name, w, mode)
        per_launch_s = ms / 1e3 / launches
        io = u["io_bytes"] * units_per_launch / per_launch_s / 1e9
        des = u["design_bytes"] * units_per_launch / per_launch_s / 1e9
        tfs = u["flops"] * units_per_launch / per_launch_s / 1e12
        tfi = u["flops_issued"] * units_per_launch / per_launch_s / 1e12
        out[name] = {"launches": launches // max(1, steps), "ms_per_step": round(ms / steps, 4),
                     "us_per_launch": round(per_launch_s * 1e6, 1),
                     "io_gbs": round(io, 1), "io_frac": round(io / hbm, 4),
                     "design_gbs": round(des, 1), "design_frac": round(des / hbm, 4),
                     "tflops": round(tfs, 2), "tensor_frac": round(tfs / bf16, 4),
                     "tflops_issued": round(tfi, 2)}
    return out


def roofline(timing: dict, w, steps: int, peaks: dict, peaks_src: str, clocks: dict,
             mode: str = "keep"):
    """Roofline object of the kernel with the largest total time (serialized pass).

    achieved = the kernel's algorithmic bytes per launch (its share of the layer's
    own I/O, kernel_units io_bytes, x the chunk-heads one launch covers) / the
    average launch duration, against the measured HBM copy bandwidth.  The bytes
    it moves with the split design's intermediates (design_bytes) and its canonical
    tensor throughput against the burst bf16 peak are reported beside it.
    """
    if not timing:
        return None
    name, (launches, ms) = max(timing.items(), key=lambda kv: kv[1][1])
    if launches == 0 or ms <= 0:
        return None
    chunk_heads = w.B * w.H * ((w.T + 63) // 64)  # per step, over all pieces
    # every launch processes one piece (all heads, batch rows); a launch covers
    # chunk_heads / n_sub chunk-heads on average
    units_per_launch = chunk_heads / w.n_sub
    u = kernel_units(name, w, mode)
    per_launch_s = ms / 1e3 / launches
    gbs = u["io_bytes"] * units_per_launch / per_launch_s / 1e9
    des = u["design_bytes"] * units_per_launch / per_launch_s / 1e9
    tfs = u["flops"] * units_per_launch / per_launch_s / 1e12
    hbm = float(peaks["hbm_gbs"])
    bf16 = float(peaks.get("bf16_tflops", 1590.0))
    obj = {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm, "unit": "GB/s",
           "frac": round(gbs / hbm, 4),
           "traffic": measured_traffic(name, units_per_launch, w, mode),
           "kernel": name, "launches": launches, "avg_launch_ms": round(ms / launches, 4),
           "chunk_heads_per_launch": units_per_launch,
           "bytes_per_chunk_head": u["io_bytes"],
           "bytes_per_launch": int(u["io_bytes"] * units_per_launch),
           "design_bytes_per_launch": int(u["design_bytes"] * units_per_launch),
           "design_gbs": round(des, 1), "design_frac": round(des / hbm, 4),
           "tensor_tflops": round(tfs, 2), "tensor_peak": bf16, "tensor_frac": round(tfs / bf16, 4),
           "peak_source": peaks_src + " (hbm_gbs for bytes; bf16_tflops, burst, for tensor_frac)",
           "share_of_kernel_time": round(ms / sum(v[1] for v in timing.values()), 4)}
    return obj


def step_roofline(w, ms: float, peaks: dict) -> dict:
    """Whole-step figures: canonical TFLOP/s of forward + backward and the fraction of
    the layer's HBM floor (its own I/O at the measured bandwidth) the step reaches."""
    C = 64
    token_heads = w.B * w.T * w.H
    fl = sum(canonical_flops(n, w) for n in ("intra_bwd", "state_fwd", "output_p", "state_bwd",
                                              "grad_fused" if w.has_beta else "grad_attn")) / C
    io = layer_io_bytes_per_token_head(w)["total"]
    hbm = float(peaks["hbm_gbs"])
    bf16 = float(peaks.get("bf16_tflops", 1590.0))
    s = ms / 1e3
    return {"flops_per_token_head": fl, "tflops": round(fl * token_heads / s / 1e12, 2),
            "tensor_frac": round(fl * token_heads / s / 1e12 / bf16, 4),
            "io_bytes_per_token_head": io, "hbm_floor_ms": round(io * token_heads / (hbm * 1e9) * 1e3, 4),
            "hbm_floor_frac": round(io * token_heads / s / 1e9 / hbm, 4)}


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 200 ms while running."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=5)
        return summarize_clocks(self.lines)


def summarize_clocks(lines) -> dict:
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    sm, mx, reasons = [], [], set()
    for ln in lines:
        parts = [x.strip() for x in ln.split(",")]
        if len(parts) < 9:
            continue
        try:
            sm.append(float(parts[1]))
            mx.append(float(parts[2]))
        except ValueError:
            continue
        for nm, val in zip(names, parts[5:9]):
            if val.lower().startswith("active"):
                reasons.add(nm)
    return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
            "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ oracle timing
def time_oracle(w, heads: int, tokens: int, nthreads: int | None = None):
    """fp64 oracle fwd + bwd on a bounded sample of workload w: the first `tokens`
    tokens of the first `heads` heads.  Returns (layer tokens/s, info); a layer token
    covers all H heads, so the sample's rate is scaled by heads / H."""
    import oracle
    cores = nthreads or oracle.max_threads()
    hs = list(range(min(heads, w.H)))
    x = inputs.generate(w, 0, tokens, heads=hs, with_grad=True)
    t0 = time.perf_counter()
    o, S = oracle.fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], nthreads=cores)
    oracle.bwd(x["q"], x["k"], x["v"], x["g"], x["beta"], None, x["dO"], nthreads=cores)
    dt = time.perf_counter() - t0
    layer_tokens = w.B * tokens * len(hs) / w.H  # a layer token covers all H heads
    return layer_tokens / dt, {
        "cores": cores, "seconds": round(dt, 3), "token_heads": w.B * tokens * len(hs),
        "sample": f"B={w.B} x {tokens} tokens x {len(hs)} of {w.H} heads, fwd+bwd, fp64 token loop; "
                  f"tokens/s counts a token as all {w.H} heads",
    }


def cpu_baseline(w, tokens: int) -> dict:
    """The oracle on every host core over a bounded sample of all heads, plus the same
    oracle on one thread over a smaller sample (one head per 16 of the workload's heads)."""
    val, info = time_oracle(w, heads=w.H, tokens=tokens)
    h1 = max(1, w.H // 16)
    v1, info1 = time_oracle(w, heads=h1, tokens=min(tokens, 4096), nthreads=1)
    return {"value": round(val, 3), "unit": "tokens/s", "cores": info["cores"], "kind": "oracle",
            "sample": info["sample"], "seconds": info["seconds"],
            "one_thread": {"value": round(v1, 3), "unit": "tokens/s", "cores": 1,
                           "sample": info1["sample"], "seconds": info1["seconds"]}}


def bench_config(w, lens, world: int, mode: str) -> dict:
    """The `config` object of a bench line (the reference arm uses the same one)."""
    return {"workload": w.name, "B": w.B, "T": w.T, "H": w.H, "d": w.d, "n_sub": len(lens),
            "chunk": 64, "variant": w.variant, "l2": "inputs larger than L2, no flush",
            "parallelism": f"replicas{world}", "mode": mode}


def run_reference(args, w, rank, world):
    """The reference arm: the fp64 oracle as it stands, on this host's cores.  Each step
    is a bounded sample (4096 tokens of as many heads as there are cores), timed; the
    line's value is the sample's rate in layer tokens/s, ms_per_step the sample's own
    measured time per step.  What the whole layer would take at that rate is reported
    as an extrapolation, not as a measured time."""
    if rank != 0:
        return 0
    import oracle
    cores = oracle.max_threads()
    heads = max(1, min(w.H, cores))
    tokens = min(w.T, 4096)
    vals, secs = [], []
    for i in range(args.warmup + args.steps):
        v, info = time_oracle(w, heads, tokens)
        if i >= args.warmup:
            vals.append(v)
            secs.append(info["seconds"])
    val = statistics.median(vals)
    sample_ms = statistics.median(secs) * 1e3
    line = {
        "impl": "reference", "metric": "fwd+bwd tokens/s per layer", "value": round(val, 3),
        "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(sample_ms, 3),
        "ms_per_step_is": "measured time of one step's bounded sample (see cpu_baseline.sample)",
        "full_layer_ms_extrapolated": round(w.B * w.T / val * 1e3, 3),
        "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": bench_config(w, inputs.sub_lengths(w), world, args.mode),
        "cpu_baseline": {"value": round(val, 3), "unit": "tokens/s", "cores": info["cores"],
                         "kind": "oracle", "sample": info["sample"] + "; each step one sample",
                         "seconds_per_sample": round(sample_ms / 1e3, 3)},
        "e2e": {"value": round(val, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ GPU arm
def workspace(torch, nbytes: int, dev):
    """A library workspace: its head (the device error word) starts zeroed."""
    ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    ws[:min(nbytes, 256)].zero_()
    return ws


def capture_graph(torch, fn, dev):
    """A CUDA graph of one step's driver calls: fn(stream) issues them with `stream` as
    their main stream (captured on a side stream; the drivers' aux and critical streams
    join the capture through their event waits)."""
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream(device=dev)
    torch.cuda.synchronize(dev)
    # thread-local: other threads of the process (a process group's watchdog) may keep
    # making CUDA calls while this thread captures
    with torch.cuda.graph(g, stream=s, capture_error_mode="thread_local"):
        fn(s)
    torch.cuda.synchronize(dev)
    return g


def time_planned_cut(args, sf, torch, sh, lens, x, timing, dev, main, aux, outs):
    """Device time of the keep drivers on the cut sf_plan_cut picks from the measured costs."""
    n_chunks = sum(-(-n // 64) for n in lens)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    from chunked_linear_recurrence_chunkwise_b200 import layer
    costs = layer.chunk_costs(timing, args.steps, n_chunks, sh.B * sh.H, sms)
    plan = sf.sf_plan_cut(sh, len(lens), costs)
    res = {"lens": plan, "model_ms": round(sf.sf_model_seq_us(sh, plan, costs) / 1e3, 4),
           "model_ms_own_cut": round(sf.sf_model_seq_us(sh, lens, costs) / 1e3, 4),
           "costs_us_per_chunk": {"intra": round(costs.intra_us, 4), "output": round(costs.output_us, 4),
                                  "grad": round(costs.grad_us, 4), "state_fwd": round(costs.state_fwd_us, 4),
                                  "state_bwd": round(costs.state_bwd_us, 4), "sms": sms,
                                  "min_chunks": costs.min_chunks}}
    ws_f = workspace(torch, sf.sf_seq_workspace_bytes(sh, plan, sf.SF_OP_FWD), dev)
    ws_b = workspace(torch, sf.sf_seq_workspace_bytes(sh, plan, sf.SF_OP_BWD), dev)
    keep = torch.empty(sf.sf_keep_bytes(sh, plan), dtype=torch.uint8, device=dev)

    def step(sm=None):
        sm = sm or main
        sf.sf_fwd_seq_keep(sh, plan, x["q"], x["k"], x["v"], x["g"], x["beta"], None, outs["o"],
                           outs["S_out"], keep, ws_f, stream_main=sm, stream_aux=aux)
        sf.sf_bwd_seq_keep(sh, plan, x["q"], x["k"], x["v"], x["g"], x["beta"], keep, x["dO"], None,
                           outs["dq"], outs["dk"], outs["dv"], outs["dg"], outs["dbeta"], outs["dS_in"],
                           ws_b, stream_main=sm, stream_aux=aux)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if not args.no_graph:  # timed as the headline is: a CUDA-graph replay of the two calls
        try:
            g = capture_graph(torch, step, dev)

            def step():
                with torch.cuda.stream(main):
                    g.replay()

            for _ in range(args.warmup):
                step()
        except RuntimeError:
            pass
        torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(main)
    for _ in range(args.steps):
        step()
    e1.record(main)
    torch.cuda.synchronize()
    sf.sf_check(ws_f, main)
    sf.sf_check(ws_b, main)
    ms = e0.elapsed_time(e1) / args.steps
    res["ms_per_step"] = round(ms, 4)
    res["value"] = round(sh.B * sh.T / (ms * 1e-3), 1)
    del keep, ws_f, ws_b
    return res


def run_sf(args, w, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from chunked_linear_recurrence_chunkwise_b200 import layer, sf

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    wr = rank_workload(w, rank)
    lens = inputs.sub_lengths(wr)
    host = inputs.to_torch(wr, pin=True)  # pinned host copies (end-to-end leg)
    x = {k_: (None if t is None else t.to(dev, non_blocking=True)) for k_, t in host.items()}
    torch.cuda.synchronize()
    B, T, H, d = wr.B, wr.T, wr.H, wr.d
    sh = sf.shape_of(x["q"], x["v"])
    ws_f = workspace(torch, sf.sf_seq_workspace_bytes(sh, lens, sf.SF_OP_FWD), dev)
    ws_b = workspace(torch, sf.sf_seq_workspace_bytes(sh, lens, sf.SF_OP_BWD), dev)
    main = torch.cuda.Stream(device=dev)
    aux = torch.cuda.Stream(device=dev)
    o = torch.empty_like(x["v"])
    S_out = torch.empty((B, H, d, d), dtype=torch.float32, device=dev)
    S_saved = torch.empty((len(lens), B, H, d, d), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(x["q"]), torch.empty_like(x["k"]), torch.empty_like(x["v"])
    dg = None if x["g"] is None else torch.empty_like(x["g"])
    db = None if x["beta"] is None else torch.empty_like(x["beta"])
    dS_in = torch.empty((B, H, d, d), dtype=torch.float32, device=dev)
    keep = torch.empty(sf.sf_keep_bytes(sh, lens), dtype=torch.uint8, device=dev)

    outs_main = {"o": o, "dq": dq, "dk": dk, "dv": dv, "S_out": S_out, "dS_in": dS_in, "dg": dg,
                 "dbeta": db}

    def step(src, serial=False, mode=None, out=None, sm=None):
        sm = sm or main
        sa = sm if serial else aux
        r = out or outs_main
        if (mode or args.mode) == "keep":
            sf.sf_fwd_seq_keep(sh, lens, src["q"], src["k"], src["v"], src["g"], src["beta"], None, r["o"],
                               r["S_out"], keep, ws_f, stream_main=sm, stream_aux=sa)
            sf.sf_bwd_seq_keep(sh, lens, src["q"], src["k"], src["v"], src["g"], src["beta"], keep,
                               src["dO"], None, r["dq"], r["dk"], r["dv"], r["dg"], r["dbeta"], r["dS_in"],
                               ws_b, stream_main=sm, stream_aux=sa)
            return
        sf.sf_fwd_seq(sh, lens, src["q"], src["k"], src["v"], src["g"], src["beta"], None, r["o"],
                      r["S_out"], S_saved, ws_f, stream_main=sm, stream_aux=sa)
        sf.sf_bwd_seq(sh, lens, src["q"], src["k"], src["v"], src["g"], src["beta"], S_saved,
                      src["dO"], None, r["dq"], r["dk"], r["dv"], r["dg"], r["dbeta"], r["dS_in"], ws_b,
                      stream_main=sm, stream_aux=sa)

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local_rank])

    for _ in range(args.warmup):
        step(x)
    torch.cuda.synchronize()
    sf.sf_check(ws_f, main)
    sf.sf_check(ws_b, main)

    # ---- the eager driver calls, timed (reported beside the headline, or as it)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    e0.record(main)
    for _ in range(args.steps):
        step(x)
    e1.record(main)
    torch.cuda.synchronize()
    barrier()
    ms_eager = reduce_max(e0.elapsed_time(e1) / args.steps, device=dev)
    sf.sf_check(ws_f, main)
    sf.sf_check(ws_b, main)

    # ---- the headline: one step's two driver calls captured into a CUDA graph and
    # replayed (the same kernels in the same order; launch gaps shrink)
    graph, launch = None, "eager"
    if not args.no_graph:
        try:
            graph = capture_graph(torch, lambda s: step(x, sm=s), dev)
            launch = "cuda_graph"
        except RuntimeError as e:  # time the eager step instead, and say so
            torch.cuda.synchronize()
            launch = f"eager (graph capture failed: {str(e)[:120]})"
    if graph is not None:
        for _ in range(args.warmup):
            with torch.cuda.stream(main):
                graph.replay()
        torch.cuda.synchronize()

    # ---- device-timed region (inputs resident in HBM; they exceed L2, so no flush)
    clk = ClockSampler(local_rank)
    barrier()
    torch.cuda.synchronize()
    clk.start()
    time.sleep(0.3)
    e0.record(main)
    for _ in range(args.steps):
        if graph is not None:
            with torch.cuda.stream(main):
                graph.replay()
        else:
            step(x)
    e1.record(main)
    torch.cuda.synchronize()
    clocks = clk.stop()
    barrier()
    ms = e0.elapsed_time(e1) / args.steps
    ms_max = reduce_max(ms, device=dev)
    sf.sf_check(ws_f, main)
    sf.sf_check(ws_b, main)
    del graph

    # ---- the other driver form, timed the same way (reported beside the headline)
    other = "recompute" if args.mode == "keep" else "keep"
    ms_other = None
    if not args.no_other_mode:
        for _ in range(args.warmup):
            step(x, mode=other)
        barrier()
        torch.cuda.synchronize()
        e0.record(main)
        for _ in range(args.steps):
            step(x, mode=other)
        e1.record(main)
        torch.cuda.synchronize()
        barrier()
        ms_other = reduce_max(e0.elapsed_time(e1) / args.steps, device=dev)
        sf.sf_check(ws_f, main)
        sf.sf_check(ws_b, main)

    # ---- per-kernel durations: the same steps with both driver streams on one
    # stream, every launch bracketed by CUDA events on its stream (with two
    # streams an event pair also counts time spent queued behind the other one)
    sf.sf_timing_reset()
    sf.sf_timing_enable(True)
    for _ in range(args.steps):
        step(x, serial=True)
    torch.cuda.synchronize()
    sf.sf_timing_enable(False)
    timing = sf.sf_timing_read()
    launches = sum(v[0] for v in timing.values()) // max(1, args.steps)

    # ---- the profile-guided cut: per-chunk kernel costs from the serialized pass above,
    # the cut sf_plan_cut chooses for them, and the same steps timed on that cut.  The
    # headline keeps the workload's own cut; this is reported beside it.
    planned = None
    if args.mode == "keep" and not args.no_plan and world == 1 and len(lens) > 1:
        planned = time_planned_cut(args, sf, torch, sh, lens, x, timing, dev, main, aux, outs_main)

    # ---- end to end: pinned host inputs -> device -> fwd+bwd -> results back to host.
    # Every step copies its inputs in and its results out inside the timed region; the
    # copies run on their own streams with two device buffer sets, so that the inputs of
    # step k+1 cross PCIe while the results of step k travel the other way (the two
    # directions of the link and the two copy engines work at once), as a host-fed
    # training loop would pipeline them.
    e2e = None
    if not args.no_e2e:
        names_out = ["o", "dq", "dk", "dv", "S_out", "dS_in"] + (["dg"] if dg is not None else []) \
            + (["dbeta"] if db is not None else [])
        outs_h = {n: torch.empty(outs_main[n].shape, dtype=outs_main[n].dtype, pin_memory=True)
                  for n in names_out}
        xs = [x, {n: (None if t is None else torch.empty_like(t)) for n, t in x.items()}]
        outs = [outs_main, {n: (None if t is None else torch.empty_like(t)) for n, t in outs_main.items()}]
        h2d = sum(t.numel() * t.element_size() for t in host.values() if t is not None)
        d2h = sum(t.numel() * t.element_size() for t in outs_h.values())
        e2e_steps = max(2, args.steps)
        copy_in = torch.cuda.Stream(device=dev)
        copy_out = torch.cuda.Stream(device=dev)
        ev = lambda: torch.cuda.Event()
        ev_in, ev_comp, ev_out = [ev(), ev()], [ev(), ev()], [ev(), ev()]
        barrier()
        torch.cuda.synchronize()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(main)
        copy_in.wait_event(f0)
        copy_out.wait_event(f0)
        for k_ in range(e2e_steps):
            b_ = k_ % 2
            if k_ >= 2:
                copy_in.wait_event(ev_comp[b_])  # step k-2 has finished reading this input set
                main.wait_event(ev_out[b_])      # and its results in this set have left
            with torch.cuda.stream(copy_in):
                for n_, t in host.items():
                    if t is not None:
                        xs[b_][n_].copy_(t, non_blocking=True)
            ev_in[b_].record(copy_in)
            main.wait_event(ev_in[b_])
            step(xs[b_], out=outs[b_])
            ev_comp[b_].record(main)
            copy_out.wait_event(ev_comp[b_])
            with torch.cuda.stream(copy_out):
                for n_ in names_out:
                    outs_h[n_].copy_(outs[b_][n_], non_blocking=True)
            ev_out[b_].record(copy_out)
        main.wait_event(ev_out[(e2e_steps - 1) % 2])
        main.wait_event(ev_out[e2e_steps % 2])
        f1.record(main)
        torch.cuda.synchronize()
        barrier()
        e_ms = reduce_max(f0.elapsed_time(f1) / e2e_steps, device=dev)
        e2e = {"value": round(job_tokens_per_s(world, B, T, e_ms), 1), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(e_ms, 3),
               "steps": e2e_steps}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, min(w.T, args.cpu_sample_tokens))

    if rank == 0:
        peaks, src = load_peaks()
        line = {
            "metric": "fwd+bwd tokens/s per layer", "value": round(job_tokens_per_s(world, B, T, ms_max), 1),
            "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms_max, 4), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16" if w.dtype == "bf16" else "f32",
            "data": "synthetic",
            "config": dict(bench_config(w, lens, world, args.mode), launch=launch),
            "modes": {args.mode: {"ms_per_step": round(ms_max, 4),
                                  "value": round(job_tokens_per_s(world, B, T, ms_max), 1)},
                      args.mode + "_eager": {"ms_per_step": round(ms_eager, 4),
                                             "value": round(job_tokens_per_s(world, B, T, ms_eager), 1)},
                      other: None if ms_other is None else
                      {"ms_per_step": round(ms_other, 4),
                       "value": round(job_tokens_per_s(world, B, T, ms_other), 1)}},
            "clocks": clocks,
            "gpu_launches": launches,
            "e2e": e2e,
            "roofline": roofline(timing, w, args.steps, peaks, src, clocks, args.mode),
            "step": step_roofline(w, ms_max, peaks),
            "keep_bytes": keep.numel(),
            "kernels": kernel_rooflines(timing, w, args.steps, peaks, args.mode),
            "kernel_timing": "serialized pass (driver streams merged), CUDA events per launch",
            "cpu_baseline": cpu,
            "planned_cut": planned,
        }
        print(json.dumps(line), flush=True)
    return 0


def run_memory_study(args, w):
    """Device memory the layer needs beside its inputs and outputs, against T at a fixed
    piece length (Sequence Accumulation, Key results: memory flat in the sequence length).

    For each T the workload's variant, heads and head size are kept and the sequence is
    cut into pieces of 4096 tokens.  Per driver form: the bytes the caller allocates for
    the layer (workspaces, plus the saved piece states of the recompute form or the kept
    intermediates of the keep form), the change of free device memory across a
    fwd+bwd call (the library allocates nothing itself), and the device time of one
    fwd+bwd after a warm-up.  Inputs are drawn on the device with the workload's value
    distributions (their values do not change the memory)."""
    import torch
    import torch.nn.functional as F
    from chunked_linear_recurrence_chunkwise_b200 import sf

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    rows = []
    for T in [int(x) for x in args.memory_study.split(",")]:
        lens = [4096] * (T // 4096) + ([T % 4096] if T % 4096 else [])
        gen = torch.Generator(device=dev).manual_seed(w.seed)
        rn = lambda *shape: torch.randn(*shape, device=dev, generator=gen)
        B, H, d = w.B, w.H, w.d
        q, k = F.normalize(rn(B, T, H, d), dim=-1).to(dt), F.normalize(rn(B, T, H, d), dim=-1).to(dt)
        v, dO = rn(B, T, H, d).to(dt), rn(B, T, H, d).to(dt)
        g = (-0.1 * F.softplus(rn(B, T, H))) if w.has_g else None
        beta = torch.sigmoid(rn(B, T, H)) if w.has_beta else None
        o, dq, dk, dv = (torch.empty_like(v) for _ in range(4))
        dg = None if g is None else torch.empty_like(g)
        db = None if beta is None else torch.empty_like(beta)
        S_out = torch.empty((B, H, d, d), dtype=torch.float32, device=dev)
        dS_in = torch.empty_like(S_out)
        sh = sf.shape_of(q, v)
        main_s, aux_s = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        row = {"T": T, "n_sub": len(lens)}
        for form in ("recompute", "keep"):
            ws_f = workspace(torch, sf.sf_seq_workspace_bytes(sh, lens, sf.SF_OP_FWD), dev)
            ws_b = workspace(torch, sf.sf_seq_workspace_bytes(sh, lens, sf.SF_OP_BWD), dev)
            if form == "keep":
                extra = torch.empty(sf.sf_keep_bytes(sh, lens), dtype=torch.uint8, device=dev)
            else:
                extra = torch.empty((len(lens), B, H, d, d), dtype=torch.float32, device=dev)

            def step():
                if form == "keep":
                    sf.sf_fwd_seq_keep(sh, lens, q, k, v, g, beta, None, o, S_out, extra, ws_f,
                                       stream_main=main_s, stream_aux=aux_s)
                    sf.sf_bwd_seq_keep(sh, lens, q, k, v, g, beta, extra, dO, None, dq, dk, dv, dg, db,
                                       dS_in, ws_b, stream_main=main_s, stream_aux=aux_s)
                else:
                    sf.sf_fwd_seq(sh, lens, q, k, v, g, beta, None, o, S_out, extra, ws_f,
                                  stream_main=main_s, stream_aux=aux_s)
                    sf.sf_bwd_seq(sh, lens, q, k, v, g, beta, extra, dO, None, dq, dk, dv, dg, db,
                                  dS_in, ws_b, stream_main=main_s, stream_aux=aux_s)

            torch.cuda.synchronize()
            free0 = torch.cuda.mem_get_info(dev)[0]
            step()
            torch.cuda.synchronize()
            free1 = torch.cuda.mem_get_info(dev)[0]
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(main_s)
            step()
            e1.record(main_s)
            torch.cuda.synchronize()
            sf.sf_check(ws_f, main_s)
            sf.sf_check(ws_b, main_s)
            row[f"{form}_layer_bytes"] = ws_f.numel() + ws_b.numel() + extra.numel() * extra.element_size()
            row[f"{form}_free_delta_bytes"] = free0 - free1
            row[f"{form}_ms"] = round(e0.elapsed_time(e1), 3)
            del ws_f, ws_b, extra
        rows.append(row)
        del q, k, v, dO, o, dq, dk, dv, g, beta, dg, db
        torch.cuda.empty_cache()
    print(json.dumps({"memory_study": {"workload": w.name, "variant": w.variant, "B": w.B, "H": w.H,
                                       "d": w.d, "dtype": w.dtype, "piece_tokens": 4096, "rows": rows}}),
          flush=True)
    return 0


def main(argv=None):
    args = parse_args(argv)
    rank, world, local_rank = dist_env()
    w = inputs.WORKLOADS[args.workload]
    if args.tokens or args.heads:
        T = args.tokens or w.T
        w = w.scaled(T=T, H=args.heads or w.H, n_sub=max(1, min(w.n_sub, T // 4096)))
    if args.impl == "reference":
        return run_reference(args, w, rank, world)
    if args.memory_study:
        return run_memory_study(args, w) if rank == 0 else 0
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        return run_sf(args, w, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
