"""Benchmark of the KDA operator on B200: prefill tokens/s (headline) and
decode tokens/s, each with its roofline, as ONE JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...      # the fp64 CPU oracle, timed

A step is one kda_prefill call over the prefill workload's batch (all chunks,
all heads, final state written).  The headline workload is the long
single-sequence prefill (131072 tokens, 32 heads, d = 128), the largest
single-GPU configuration; the 4096-token / 16-head prefill and the packed
16-sequence varlen batch are timed the same way as the extra objects
"prefill_T4096" and "varlen".  Inputs are resident in HBM when timing starts;
L2 is flushed (a 256 MiB write) before every timed step, outside the timed
interval.  The decode figures time chained kda_decode_step calls on the
decode workload (state 512 MiB, larger than L2, so no flush is needed).  The
"gdn_prefill" object times gdn_prefill (Gated DeltaNet: one gate value per
token and head) and "layer_prefill" times kda_layer_prefill (raw activations,
the layer's prologue and epilogue fused) on the headline workload the same
way; "backward" times the backward pass (the gradients, given seeded upstream
gradients; kda_backward_chunked for bf16 d = 128) on the 4096-token workload,
"backward_long" on the headline workload.
Under torchrun every rank runs the same workload as an independent replica
(the operator needs no exchange between GPUs); value = all ranks' tokens over
the slowest rank's time.
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
sys.path.insert(0, ROOT)

METRIC = "KDA prefill tokens/s and decode tokens/s at 1 B200; fraction of tensor/HBM roofline"
PREFILL_DEFAULT = "prefill_T131072_H32_d128"
EXTRA_PREFILL = (("prefill_T4096", "prefill_T4096_H16_d128"),
                 ("varlen", "varlen_16seq_256to16384_H32_d128"))
BACKWARD_DEFAULT = "prefill_T4096_H16_d128"
DECODE_DEFAULT = "decode_B256_H32_d128"
# DRAM bytes (read + write) of one whole kda_prefill call, from an ncu
# application-range capture over one call of the 16384-token, 32-head workload
# (597.9 MB read + 694.3 MB written), scaled by the token count to the
# 131072-token workload, which runs the same plan and per-chunk schedule
# (profiles/kda_prefill_T131072_H32_d128.md); null for other workloads.
CALL_TRAFFIC = {"prefill_T131072_H32_d128": (597.9e6 + 694.3e6) * 131072 / 16384}
# the oracle's sample: whole heads of the first sequence, at most this many
# of its first tokens (its cost is linear in (token, head) pairs)
ORACLE_PREFIX = 32768
DECODE_STEPS = 1000

# Algorithmic work per (token, head) for prefill with chunk C and d_k = d_v = d:
#   FLOP  = 6 d_k d_v + C (3 d_k + 2 d_v)          (state products + chunk products)
#   bytes = (3 d_k + 2 d_v) * io_bytes + io_bytes  (q, k, log_alpha, v in; o out; beta in)
# plus per (sequence, head) the fp32 state: read if an initial state is given,
# written always.
CHUNK = 64


def prefill_work(w, lengths, scalar_gate=False, layer=False):
    """Algorithmic work of one prefill call; with ``scalar_gate`` (Gated
    DeltaNet) log_alpha is one value per (token, head) instead of d_k; with
    ``layer`` the fused layer also reads the output gate (d_v per token)."""
    T = sum(lengths)
    n = len(lengths)
    eb = 2 if w.dtype == "bf16" else 4
    per_tok_flop = 6 * w.d_k * w.d_v + CHUNK * (3 * w.d_k + 2 * w.d_v)
    per_tok_bytes = (3 * w.d_k + 2 * w.d_v) * eb + eb
    if scalar_gate:
        per_tok_bytes -= (w.d_k - 1) * eb
    if layer:
        per_tok_bytes += w.d_v * eb
    state_bytes = n * w.H * w.d_k * w.d_v * 4 * (2 if w.init_std > 0 else 1)
    return dict(tokens=T, flop=per_tok_flop * T * w.H,
                bytes=per_tok_bytes * T * w.H + state_bytes)


# Backward pass, per (token, head) with a d_k x d_v state: one forward step
# (decay, r, update: 5 FLOP per state element) and the backward step (q do^T,
# dq, du, dk, the erase term, dk's second term, dg, the decay of dS, Sp and
# S_t again: 18 FLOP per element), on CUDA cores in fp32.  Bytes: q, k,
# log_alpha, v, do read in the I/O dtype, beta read; dq, dk, dlog_alpha, dv,
# dbeta written in fp32; per (sequence, head) the initial state and dL/dS_T
# read and dL/dS_0 written.
BWD_FLOP_PER_ELEM = 5 + 18
# fp32 CUDA-core peak: 148 SMs x 128 FP32 lanes x 2 FLOP (FMA) x 1.965 GHz
FP32_SIMT_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


# The chunk form of the backward pass (bf16, d = 128, C = 64) on the tensor
# cores: per (chunk, head) the products its algebra takes, 2 m n k FLOP each.
#   records:          [Ktil; Qtil] Khat^T, YT = Kbar^T T_beta, ZB = P T_beta,
#                     MP = -YT Ktil, ZB Ktil
#   forward scan:     MP S, YT V
#   reverse scan:     MP^T dS, QP^T dO
#   chunk gradients:  [Ktil; Qtil] Khat^T, Ktil S, Kbar dS_C, P^T dO,
#                     T_beta R, T_beta^T dU, dU R^T, U dS_C^T, dO U^T, dT T^T,
#                     dO S^T, dR S^T, T^T Z, dP Khat, BdA Khat, dP^T Qtil, BdA^T Ktil
def _mm(m, n, k):
    return 2 * m * n * k


def chunk_backward_flop(C=64, d=128):
    rec = _mm(2 * C, C, d) + _mm(d, C, C) + _mm(C, C, C) + _mm(d, d, C) + _mm(C, d, C)
    scans = 2 * (_mm(d, d, d) + _mm(d, d, C))
    local = _mm(2 * C, C, d) + 5 * _mm(C, d, d) + 9 * _mm(C, C, d) + 2 * _mm(C, C, C)
    return rec + scans + local


def backward_work(w, lengths):
    T, n = sum(lengths), len(lengths)
    eb = 2 if w.dtype == "bf16" else 4
    per_tok = (3 * w.d_k + 2 * w.d_v) * eb + eb + (3 * w.d_k + w.d_v + 1) * 4
    states = n * w.H * w.d_k * w.d_v * 4 * 3
    chunks = sum((L + 63) // 64 for L in lengths)
    return dict(tokens=T, flop=BWD_FLOP_PER_ELEM * w.d_k * w.d_v * T * w.H,
                chunk_flop=chunk_backward_flop() * chunks * w.H,
                bytes=per_tok * T * w.H + states)


def backward_roofline(work, ms, peaks, src):
    """The chunked pass against the bf16 tensor peak (its chunk-form
    products), the sequential one against the fp32 CUDA-core rate."""
    if work.get("chunked"):
        tf = work["chunk_flop"] / (ms * 1e-3) / 1e12
        return {"bound": "tensor", "achieved": tf, "peak": peaks["bf16"], "unit": "TFLOP/s",
                "frac": tf / peaks["bf16"], "traffic": None, "peak_source": src + " (bf16 burst)",
                "kernel": "kda_backward_chunked", "algorithmic_flop_per_launch": work["chunk_flop"],
                "algorithmic_bytes_per_launch": work["bytes"],
                "hbm_frac": work["bytes"] / (ms * 1e-3) / 1e9 / peaks["hbm"]}
    tf = work["flop"] / (ms * 1e-3) / 1e12
    return {"bound": "alu", "achieved": tf, "peak": FP32_SIMT_TFLOPS, "unit": "TFLOP/s",
            "frac": tf / FP32_SIMT_TFLOPS, "traffic": None,
            "peak_source": "nominal fp32 CUDA-core rate (148 SMs x 128 lanes x 2 x 1.965 GHz)",
            "kernel": "kda_backward", "algorithmic_flop_per_launch": work["flop"],
            "algorithmic_bytes_per_launch": work["bytes"],
            "hbm_frac": work["bytes"] / (ms * 1e-3) / 1e9 / peaks["hbm"]}


def decode_work(w):
    eb = 2 if w.dtype == "bf16" else 4
    units = w.batch * w.H
    return dict(tokens=w.batch,
                flop=units * (6 * w.d_k * w.d_v + 2 * w.d_k),
                bytes=units * (2 * w.d_k * w.d_v * 4 + (3 * w.d_k + 2 * w.d_v) * eb + eb))


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return dict(hbm=float(p["hbm_gbs"]), bf16=float(p["bf16_tflops"]),
                    bf16_sustained=float(p["bf16_tflops_sustained"]), source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


class ClockSampler:
    """nvidia-smi samples every 200 ms while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=5)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# --- distributed plumbing -------------------------------------------------------

def dist_setup():
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """The largest x over the ranks (the slowest rank's time); on the group's
    own device (CUDA for NCCL, the host for gloo)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# --- the GPU arm -------------------------------------------------------------------

def time_prefill(w, steps, warmup, world, scalar_gate=False, layer=False, profile_range=False):
    """kda_prefill (or, with ``scalar_gate``, gdn_prefill with channel 0 of
    the gate draw as the per-head gate; with ``layer``, kda_layer_prefill on
    raw activations) on the workload, L2 flushed."""
    import torch
    from gated_delta_rule_69_b200 import inputs as kin
    from gated_delta_rule_69_b200 import kda
    inp = kin.generate(w, device="cuda")
    q, k, v, g, b = (inp[x] for x in ("q", "k", "v", "log_alpha", "beta"))
    fn = kda.kda_prefill
    if scalar_gate:
        g = g[..., 0].contiguous()
        fn = kda.gdn_prefill
    if layer:
        # raw activations of the same shapes: q, k ~ N(0, 2^2), gate
        # pre-activation ~ N(-1, 1), A_log ~ N(0, 0.25^2), beta logits and
        # output-gate pre-activations ~ N(0, 1), RMSNorm weight 1 + N(0, 0.1^2)
        gen = torch.Generator(device="cuda").manual_seed(w.seed + 7)
        T0, H0, dk0 = q.shape
        rn = lambda *sh: torch.randn(*sh, generator=gen, device="cuda")
        q = (rn(T0, H0, dk0) * 2.0).to(q.dtype)
        k = (rn(T0, H0, dk0) * 2.0).to(q.dtype)
        g = (rn(T0, H0, dk0) - 1.0).to(q.dtype)
        b = rn(T0, H0).to(q.dtype)
        A_log = rn(H0) * 0.25
        out_gate = rn(T0, H0, v.shape[-1]).to(q.dtype)
        norm_weight = 1.0 + 0.1 * rn(v.shape[-1])

        def fn(q, k, v, g, b, **kw):
            return kda.kda_layer_prefill(q, k, v, g, A_log, b, out_gate=out_gate,
                                         norm_weight=norm_weight, **kw)
    T, H, dk = q.shape
    dv = v.shape[-1]
    n = len(inp["lengths"])
    o = torch.empty((T, H, dv), dtype=q.dtype, device="cuda")
    fs = torch.empty((n, H, dk, dv), dtype=torch.float32, device="cuda")
    need = (kda.kda_layer_prefill_workspace_size(n, T, H, dk, dv) if layer
            else kda.kda_prefill_workspace_size(n, T, H, dk, dv))
    ws = torch.empty(max(256, need), dtype=torch.uint8, device="cuda")
    flush = torch.empty(256 * 2 ** 20, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    def step():
        fn(q, k, v, g, b, init_state=inp["init_state"], cu_seqlens=inp["cu_seqlens"],
           o=o, final_state=fs, workspace=ws, stream=stream)

    for _ in range(warmup):
        flush.fill_(1)
        step()
    torch.cuda.synchronize()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    barrier(world)
    torch.cuda.synchronize()
    for i in range(steps):
        flush.fill_(i & 0xFF)                 # L2 flush, outside the timed interval
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    torch.cuda.synchronize()
    barrier(world)
    ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    if profile_range:   # one more call, alone inside a profiler range
        flush.fill_(7)
        torch.cuda.synchronize()
        torch.cuda.profiler.start()
        step()
        torch.cuda.synchronize()
        torch.cuda.profiler.stop()
    if kda.kda_check_workspace_error(ws) != kda.KDA_OK:
        raise RuntimeError("device-side check failed during the benchmark")
    # each call with a full workspace on bf16 d = 128 launches three kernels:
    # the plan, the preparation and the state chain (the layer two more: its
    # prologue pass and its epilogue)
    per_call = 3 if (w.dtype == "bf16" and w.d_k == 128 and w.d_v == 128) else 2
    if layer:
        per_call += 2
    return dict(ms_total=sum(ms), ms=ms, inputs=inp, launches=steps * per_call)


def time_backward(w, steps, warmup, world):
    """kda_backward on the prefill workload with seeded upstream gradients,
    L2 flushed before each step."""
    import torch
    from gated_delta_rule_69_b200 import inputs as kin
    from gated_delta_rule_69_b200 import kda
    inp = kin.generate(w, device="cuda")
    ct = kin.cotangents(w, inp["lengths"], device="cuda")
    q, k, v, g, b = (inp[x] for x in ("q", "k", "v", "log_alpha", "beta"))
    T, H, dk = q.shape
    dv = v.shape[-1]
    n = len(inp["lengths"])
    # bf16 with d = 128: the chunked backward (plan, preparation, two scans,
    # chunk steps: five kernels); otherwise the sequential one (one kernel)
    chunked = w.dtype == "bf16" and dk == 128 and dv == 128
    fn = kda.kda_backward_chunked if chunked else kda.kda_backward
    need = (kda.kda_backward_chunked_workspace_size(n, T, H) if chunked
            else kda.kda_backward_workspace_size(n, T, H, dk, dv))
    ws = torch.empty(max(256, need), dtype=torch.uint8, device="cuda")
    flush = torch.empty(256 * 2 ** 20, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    def step():
        fn(q, k, v, g, b, ct["d_o"], init_state=inp["init_state"],
           d_final_state=ct["d_final_state"], cu_seqlens=inp["cu_seqlens"],
           workspace=ws, stream=stream)

    for _ in range(warmup):
        flush.fill_(1)
        step()
    torch.cuda.synchronize()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    barrier(world)
    torch.cuda.synchronize()
    for i in range(steps):
        flush.fill_(i & 0xFF)
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    torch.cuda.synchronize()
    barrier(world)
    if kda.kda_check_workspace_error(ws) != kda.KDA_OK:
        raise RuntimeError("device-side check failed during the backward benchmark")
    ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    # chunked: the plan, the preparation, the two scans (one grid), the
    # tensor-core chunk kernel and the step kernel for the chunks it leaves
    return dict(ms_total=sum(ms), ms=ms, lengths=inp["lengths"], chunked=chunked,
                launches=steps * (5 if chunked else 1))


def time_prefill_e2e(w, steps, warmup):
    """Same workload through the public call, with each step's inputs copied
    from pinned host memory and o + final state read back.  Steps alternate
    between two streams with their own device buffers and workspace, so one
    step's copies overlap the other's compute and copies, as a caller
    streaming batches would run it; every step still moves all its bytes."""
    import torch
    from gated_delta_rule_69_b200 import inputs as kin
    from gated_delta_rule_69_b200 import kda
    inp = kin.generate(w, device="cuda")
    names = ("q", "k", "v", "log_alpha", "beta")
    host = {x: inp[x].cpu().pin_memory() for x in names}
    T, H, dk = inp["q"].shape
    dv = inp["v"].shape[-1]
    n = len(inp["lengths"])
    s0 = inp["init_state"]
    ws_bytes = max(kda.kda_prefill_workspace_size(n, T, H, dk, dv), 256)
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    bufs = []
    for _ in range(2):
        bufs.append(dict(
            dev={x: torch.empty_like(inp[x]) for x in names},
            o=torch.empty((T, H, dv), dtype=inp["q"].dtype, device="cuda"),
            fs=torch.empty((n, H, dk, dv), dtype=torch.float32, device="cuda"),
            ws=torch.empty(ws_bytes, dtype=torch.uint8, device="cuda"),
            o_h=torch.empty((T, H, dv), dtype=inp["q"].dtype).pin_memory(),
            fs_h=torch.empty((n, H, dk, dv), dtype=torch.float32).pin_memory()))
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = bufs[0]["o_h"].numel() * bufs[0]["o_h"].element_size() + bufs[0]["fs_h"].numel() * 4

    def step(i):
        s, b = streams[i % 2], bufs[i % 2]
        with torch.cuda.stream(s):
            for x in names:
                b["dev"][x].copy_(host[x], non_blocking=True)
            kda.kda_prefill(b["dev"]["q"], b["dev"]["k"], b["dev"]["v"], b["dev"]["log_alpha"],
                            b["dev"]["beta"], init_state=s0, cu_seqlens=inp["cu_seqlens"],
                            o=b["o"], final_state=b["fs"], workspace=b["ws"], stream=s)
            b["o_h"].copy_(b["o"], non_blocking=True)
            b["fs_h"].copy_(b["fs"], non_blocking=True)

    cur = torch.cuda.current_stream()
    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(cur)
    for s in streams:
        s.wait_stream(cur)
    for i in range(steps):
        step(i)
    for s in streams:
        cur.wait_stream(s)
    e1.record(cur)
    torch.cuda.synchronize()
    return dict(ms_per_step=e0.elapsed_time(e1) / steps, h2d=h2d, d2h=d2h)


def time_decode(w, steps, warmup, world):
    import torch
    from gated_delta_rule_69_b200 import inputs as kin
    from gated_delta_rule_69_b200 import kda
    inp = kin.generate(w, device="cuda")
    q, k, v, g, b, state = (inp[x] for x in ("q", "k", "v", "log_alpha", "beta", "init_state"))
    o = torch.empty((w.batch, w.H, w.d_v), dtype=q.dtype, device="cuda")
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        kda.kda_decode_step(q, k, v, g, b, state, o=o, stream=stream)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(steps):
        kda.kda_decode_step(q, k, v, g, b, state, o=o, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    return dict(ms_total=e0.elapsed_time(e1), launches=steps)


# --- the oracle on the host cores ------------------------------------------------------

def oracle_prefill_sample(w, inp, budget_s=10.0, max_heads=None, total_tokens=None):
    """Time the fp64 oracle on heads of the first sequence (its first
    ORACLE_PREFIX tokens at most), adding heads (as many per batch as there
    are oracle threads) until ``budget_s`` of CPU work has run or every head is
    done.  Returns the oracle's tokens/s extrapolated to the whole workload
    (``total_tokens`` of it, default the tokens in ``inp``), and a description
    of the sample."""
    import numpy as np
    import oracle
    from gated_delta_rule_69_b200.inputs import as_float64
    cu = inp["cu_seqlens"].cpu().numpy()
    L0 = min(int(cu[1] - cu[0]), ORACLE_PREFIX)
    threads = oracle.max_threads()
    H = w.H if max_heads is None else min(w.H, max_heads)
    done, t_total = 0, 0.0
    while done < H and (done == 0 or t_total < budget_s):
        hs = list(range(done, min(H, done + threads)))
        sel = lambda t: as_float64(t[:L0, hs])
        s0 = None if inp["init_state"] is None else as_float64(inp["init_state"][:1, hs])
        args = [sel(inp[x]) for x in ("q", "k", "v", "log_alpha", "beta")]
        t0 = time.perf_counter()
        oracle.kda_recurrence(*args, init_state=s0, cu_seqlens=np.array([0, L0]))
        t_total += time.perf_counter() - t0
        done += len(hs)
    if total_tokens is None:
        total_tokens = sum(inp["lengths"])
    # the oracle's cost is linear in (tokens x heads): scale the sampled rate
    units_done = done * L0
    units_all = total_tokens * w.H
    value = total_tokens / (t_total * units_all / units_done)
    sample = (f"{done} of {w.H} heads x the first {L0} tokens of sequence 0 "
              f"({units_done} (token, head) pairs of {units_all}); tokens/s scaled by the pair count")
    return value, threads, sample, t_total


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import torch
    from gated_delta_rule_69_b200 import inputs as kin
    # the sample's inputs only: the first sequence's first ORACLE_PREFIX
    # tokens, drawn with the workload's seed and distributions (drawing the
    # whole 131072-token batch on the host would take longer than timing it)
    lengths = kin.seq_lengths(w)
    inp = kin.generate(w, device="cpu", lengths=[min(lengths[0], ORACLE_PREFIX)])
    import oracle
    threads = oracle.max_threads()
    vals, secs = [], []
    for i in range(args.warmup + args.steps):
        v, thr, sample, t = oracle_prefill_sample(w, inp, budget_s=0.0, max_heads=threads,
                                                  total_tokens=sum(lengths))
        if i >= args.warmup:
            vals.append(v)
            secs.append(t)
    value = statistics.median(vals)
    work = prefill_work(w, lengths)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * work["tokens"] / value, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(w, lengths, args.gpus),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def config_of(w, lengths, n_gpus):
    c = {"workload": w.name, "tokens": sum(lengths), "num_seqs": len(lengths), "H": w.H,
         "d_k": w.d_k, "d_v": w.d_v, "chunk": CHUNK, "io_dtype": w.dtype,
         "state_dtype": "fp32", "init_state": "N(0, 0.02)" if w.init_std > 0 else "zeros",
         "seed": w.seed,
         "parallelism": f"replicas x{n_gpus}" if n_gpus > 1 else "single GPU",
         "l2": "flushed by a 256 MiB write before each timed prefill step"}
    return c


# --- main -------------------------------------------------------------------------------

def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=PREFILL_DEFAULT)
    ap.add_argument("--decode-workload", default=DECODE_DEFAULT)
    ap.add_argument("--backward-workload", default=BACKWARD_DEFAULT)
    ap.add_argument("--decode-steps", type=int, default=DECODE_STEPS)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--profile-range", action="store_true",
                    help="with --prefill-only: after the timed steps, one more prefill call "
                         "bracketed by cudaProfilerStart / cudaProfilerStop (for a profiler's "
                         "range replay over the whole call)")
    ap.add_argument("--backward-only", action="store_true",
                    help="time only the backward pass on --backward-workload (a lighter command "
                         "for profiler captures); prints a line without the other objects")
    ap.add_argument("--prefill-only", action="store_true",
                    help="time only the prefill workload (a lighter command for profiler captures); "
                         "prints a line without the extra objects")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    from gated_delta_rule_69_b200 import inputs as kin
    w = kin.WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w)

    import torch
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the library has no CPU path)")
    rank, world, local = dist_setup()
    from gated_delta_rule_69_b200 import build
    if rank == 0:
        build.build()
    barrier(world)
    peaks = load_peaks()

    sampler = ClockSampler(local)
    sampler.start()
    if args.backward_only:
        bw = kin.WORKLOADS[args.backward_workload]
        bwd = time_backward(bw, args.steps, args.warmup, world)
        clocks = sampler.stop()
        bwork = backward_work(bw, bwd["lengths"])
        bms = max_over_ranks(bwd["ms_total"] / len(bwd["ms"]), world)
        if rank == 0:
            print(json.dumps({"metric": "backward tokens/s", "value": world * bwork["tokens"] / (bms * 1e-3),
                              "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
                              "warmup": args.warmup, "ms_per_step": bms,
                              "config": config_of(bw, bwd["lengths"], world),
                              "gpu_launches": bwd["launches"], "clocks": clocks}), flush=True)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return 0
    pf = time_prefill(w, args.steps, args.warmup, world, profile_range=args.profile_range)
    if args.prefill_only:
        clocks = sampler.stop()
        work = prefill_work(w, pf["inputs"]["lengths"])
        ms_step = max_over_ranks(pf["ms_total"] / args.steps, world)
        if rank == 0:
            print(json.dumps({"metric": METRIC, "value": world * work["tokens"] / (ms_step * 1e-3),
                              "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
                              "warmup": args.warmup, "ms_per_step": ms_step,
                              "config": config_of(w, pf["inputs"]["lengths"], world),
                              "gpu_launches": pf["launches"], "clocks": clocks}), flush=True)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return 0
    extra = []
    for key, name in EXTRA_PREFILL:
        if name != w.name:
            ew = kin.WORKLOADS[name]
            extra.append((key, ew, time_prefill(ew, args.steps, args.warmup, world)))
    dw = kin.WORKLOADS[args.decode_workload]
    dec = time_decode(dw, args.decode_steps, args.warmup, world)
    gdn = time_prefill(w, args.steps, args.warmup, world, scalar_gate=True)
    lay = time_prefill(w, args.steps, args.warmup, world, layer=True)
    bw = kin.WORKLOADS[args.backward_workload]
    bwd = time_backward(bw, max(3, args.steps // 4), args.warmup, world)
    # the backward on the headline workload too, with few steps (about 0.2 s a call)
    bwd_long = time_backward(w, 3, 3, world) if w.name != bw.name else None
    clocks = sampler.stop()

    lengths = pf["inputs"]["lengths"]
    work = prefill_work(w, lengths)
    ms_step = max_over_ranks(pf["ms_total"] / args.steps, world)
    value = world * work["tokens"] / (ms_step * 1e-3)
    gbs = work["bytes"] / (ms_step * 1e-3) / 1e9
    tfs = work["flop"] / (ms_step * 1e-3) / 1e12
    dwork = decode_work(dw)
    dms = max_over_ranks(dec["ms_total"] / args.decode_steps, world)
    dgbs = dwork["bytes"] / (dms * 1e-3) / 1e9
    gwork = prefill_work(w, lengths, scalar_gate=True)
    gms = max_over_ranks(gdn["ms_total"] / args.steps, world)
    ggbs = gwork["bytes"] / (gms * 1e-3) / 1e9
    lwork = prefill_work(w, lengths, layer=True)
    lms = max_over_ranks(lay["ms_total"] / args.steps, world)
    lgbs = lwork["bytes"] / (lms * 1e-3) / 1e9
    bwork = backward_work(bw, bwd["lengths"])
    bwork["chunked"] = bwd["chunked"]
    bms = max_over_ranks(bwd["ms_total"] / len(bwd["ms"]), world)
    src = "of " + peaks["source"]

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if w.dtype == "bf16" else "f32", "data": "synthetic",
        "config": config_of(w, lengths, world),
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm"], "unit": "GB/s",
                     "frac": gbs / peaks["hbm"], "traffic": CALL_TRAFFIC.get(w.name),
                     "traffic_unit": "bytes per call (DRAM read + write)", "peak_source": src,
                     "kernel": "kda_prefill", "algorithmic_bytes_per_launch": work["bytes"],
                     "tensor_tflops": tfs, "tensor_frac": tfs / peaks["bf16"],
                     "algorithmic_flop_per_launch": work["flop"]},
        "decode": {"workload": dw.name, "value": world * dwork["tokens"] / (dms * 1e-3),
                   "unit": "tokens/s", "ms_per_step": dms, "steps": args.decode_steps,
                   "roofline": {"bound": "hbm", "achieved": dgbs, "peak": peaks["hbm"],
                                "unit": "GB/s", "frac": dgbs / peaks["hbm"], "traffic": None,
                                "peak_source": src, "kernel": "kda_decode_step",
                                "algorithmic_bytes_per_launch": dwork["bytes"]}},
        "gdn_prefill": {"workload": w.name + " with one gate value per (token, head)",
                        "value": world * gwork["tokens"] / (gms * 1e-3), "unit": "tokens/s",
                        "ms_per_step": gms, "steps": args.steps,
                        "roofline": {"bound": "hbm", "achieved": ggbs, "peak": peaks["hbm"],
                                     "unit": "GB/s", "frac": ggbs / peaks["hbm"], "traffic": None,
                                     "peak_source": src, "kernel": "gdn_prefill",
                                     "algorithmic_bytes_per_launch": gwork["bytes"]}},
        "layer_prefill": {"workload": w.name + ", raw activations, layer prologue and epilogue fused",
                          "value": world * lwork["tokens"] / (lms * 1e-3), "unit": "tokens/s",
                          "ms_per_step": lms, "steps": args.steps,
                          "roofline": {"bound": "hbm", "achieved": lgbs, "peak": peaks["hbm"],
                                       "unit": "GB/s", "frac": lgbs / peaks["hbm"],
                                       "traffic": None, "peak_source": src,
                                       "kernel": "kda_layer_prefill",
                                       "algorithmic_bytes_per_launch": lwork["bytes"]}},
        "backward": {"workload": bw.name + ", backward pass (kda_backward_chunked for bf16 d = 128), seeded upstream gradients",
                     "value": world * bwork["tokens"] / (bms * 1e-3), "unit": "tokens/s",
                     "ms_per_step": bms, "steps": len(bwd["ms"]),
                     "roofline": backward_roofline(bwork, bms, peaks, src)},
        "gpu_launches": pf["launches"] + dec["launches"] + gdn["launches"] + lay["launches"]
                        + bwd["launches"] + sum(x[2]["launches"] for x in extra)
                        + (bwd_long["launches"] if bwd_long else 0),
        "clocks": clocks,
    }
    if bwd_long:
        lwk = backward_work(w, bwd_long["lengths"])
        lwk["chunked"] = bwd_long["chunked"]
        lbms = max_over_ranks(bwd_long["ms_total"] / len(bwd_long["ms"]), world)
        line["backward_long"] = {
            "workload": w.name + ", backward pass (kda_backward_chunked), seeded upstream gradients",
            "value": world * lwk["tokens"] / (lbms * 1e-3), "unit": "tokens/s", "ms_per_step": lbms,
            "steps": len(bwd_long["ms"]),
            "roofline": backward_roofline(lwk, lbms, peaks, src)}
    for key, ew, r in extra:
        ework = prefill_work(ew, r["inputs"]["lengths"])
        ems = max_over_ranks(r["ms_total"] / args.steps, world)
        egbs = ework["bytes"] / (ems * 1e-3) / 1e9
        etfs = ework["flop"] / (ems * 1e-3) / 1e12
        line[key] = {"workload": ew.name, "config": config_of(ew, r["inputs"]["lengths"], world),
                     "value": world * ework["tokens"] / (ems * 1e-3), "unit": "tokens/s",
                     "ms_per_step": ems, "steps": args.steps,
                     "roofline": {"bound": "hbm", "achieved": egbs, "peak": peaks["hbm"],
                                  "unit": "GB/s", "frac": egbs / peaks["hbm"], "traffic": None,
                                  "peak_source": src, "kernel": "kda_prefill",
                                  "algorithmic_bytes_per_launch": ework["bytes"],
                                  "tensor_tflops": etfs, "tensor_frac": etfs / peaks["bf16"],
                                  "algorithmic_flop_per_launch": ework["flop"]}}
    if not args.no_e2e:
        e2e = time_prefill_e2e(w, max(6, args.steps), args.warmup)
        e_ms = max_over_ranks(e2e["ms_per_step"], world)
        line["e2e"] = {"value": world * work["tokens"] / (e_ms * 1e-3), "unit": "tokens/s",
                       "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"]}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, thr, sample, _ = oracle_prefill_sample(w, pf["inputs"], budget_s=10.0)
        line["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": thr, "kind": "oracle",
                                "sample": sample}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
