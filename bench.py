#!/usr/bin/env python
"""Benchmark of the KDA hot path on B200: long-context prefill tokens/s and
decode-step state GB/s, each against its roofline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One "step" is one chunked prefill of the long-context workload (B=1, H=32,
T=131072, d=128, bf16 q/k/v, fp32 gates, zero S0): the chunk-parallel kernel
and the sequential carry kernel. The other workloads are reported under their
own keys: the chunked (B=4, H=16, T=4096) and varlen (8 packed sequences) prefills,
the decode workload (256 sequences x 32 heads, 128 x 128 fp32 state, bf16
q/k/v) as a chain of 1000 steps with fresh inputs per step, the multi-token
decode, the one-gate-per-head prefill and the backward. Inputs are seeded
synthetic tensors resident in HBM before the timed region; every workload's
inputs are larger than the 126 MB L2, so no flush is needed between
iterations. Under torchrun each rank runs its own independent problem (weak
scaling, no collective on the data path) and the time is the max over ranks.

``--impl reference`` times the fp64 CPU oracle on the host cores instead, on a
bounded sample of the same workload per step (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from gated_delta_rule_132_b200 import inputs as I  # noqa: E402

METRIC = ("KDA prefill tokens/s (H=32,d=128) & decode-step state GB/s vs HBM peak, "
          "1×B200")
# DRAM traffic per (chunk, head) record (dram__bytes_read.sum +
# dram__bytes_write.sum of one ncu capture of each kernel on the chunked
# workload, 4096 records per launch); traffic grows in proportion to the
# records a launch processes. None: no capture of the current kernel yet.
TRAFFIC_PER_RECORD = {"prepare": 162_201, "carry": 113_586, "gdn_prepare": 128_265}
# Algorithmic work of the prefill per token and head at d = 128, chunk 64: bytes
# the operation must move (q, k, v bf16 in, log_alpha and beta fp32 in, o bf16
# out; the states are added per sequence) and tensor-core flops of the chunked
# form, split into the intra-chunk contractions (A, P and the solve's products:
# 10 C d) and the inter-chunk state carry (6 d^2).
PREFILL_IN_BYTES = 3 * 128 * 2 + 128 * 4 + 4
PREFILL_OUT_BYTES = 128 * 2
INTRA_FLOP = 10 * 64 * 128
CARRY_FLOP = 6 * 128 * 128
# The pages' own claims, quoted as context only: whole-model ratios of Kimi
# Linear against full attention (no hardware or precision stated).
PAGE_CLAIMS = {
    "decode_speed_1M_tokens": "about 6x faster decoding than full attention at 1M tokens",
    "decode_speedup_128k_1M": "4.8x at 128k and 6.3x at 1M tokens",
    "kv_cache": "up to 75% less KV cache",
    "long_context_speed": "2.9x faster on 100k-token long-context work",
    "note": "whole-model ratios from the pages, not kernel numbers; context only",
}
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------------------------- helpers
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


def dist_setup(gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """The largest of the ranks' values (the job's time is its slowest rank's)."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: float, ms_max: float, world: int) -> float:
    """Whole-job rate under weak scaling: every rank processes units_per_rank
    units, and the job takes as long as its slowest rank (ms_max)."""
    return units_per_rank * world / (ms_max / 1e3)


class ClockSampler:
    """nvidia-smi clock/throttle samples every 200 ms while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.dev = device_index

    def __enter__(self):
        try:
            uuid = "GPU-" + str(torch.cuda.get_device_properties(self.dev).uuid)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", uuid, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:  # noqa: BLE001 - clocks are best effort
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.out = ""
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except Exception:  # noqa: BLE001
                self.proc.kill()

    def summary(self):
        rows = []
        for line in (getattr(self, "out", "") or "").splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                rows.append((float(parts[0]), float(parts[1]), parts[4:8]))
            except ValueError:
                continue
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, flags in rows for i, f in enumerate(flags)
                          if f.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows),
                "sm_max_mhz": max(r[1] for r in rows), "reasons": reasons,
                "samples": len(rows)}


LAUNCHES = {"count": 0}  # the library's kernel launches inside every timed region


def time_region(fn_step, steps, stream, marks=0):
    """Run ``fn_step(i, events)`` for i < steps between two events on ``stream``.
    ``marks`` extra events per step are handed to fn_step to bracket kernels.
    Returns (total ms, [[ms between consecutive marks] per step]); the library's
    kernel launches inside the region are added to LAUNCHES."""
    from gated_delta_rule_132_b200 import kda
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(marks)] for _ in range(steps)]
    n0 = kda.kda_launch_count()
    start.record(stream)
    for i in range(steps):
        fn_step(i, evs[i])
    end.record(stream)
    torch.cuda.synchronize()
    LAUNCHES["count"] += kda.kda_launch_count() - n0
    per = [[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(marks - 1)]
           for i in range(steps)]
    return start.elapsed_time(end), per


# ----------------------------------------------------------------------------- our arm
def bench_prefill(preset, steps, warmup, world, rank, dev, peaks):
    from gated_delta_rule_132_b200 import kda
    if rank == 0:
        x = I.make_preset(preset, device=f"cuda:{dev}")
    else:  # an independent problem of the same shape on every other rank
        lengths = None
        if preset.n_varlen:
            lengths = I.varlen_lengths(preset.n_varlen, preset.varlen_min, preset.varlen_max,
                                       preset.seed)
        x = I.make_prefill(preset.B, preset.T, preset.H, preset.d, preset.dtype,
                           preset.gate_shift, preset.s0_std, preset.seed + 1000 * rank,
                           lengths=lengths, device=f"cuda:{dev}")
    call = kda.ChunkFwdCall(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"],
                            x["cu_seqlens"], x["scale"])
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        call.run()
    torch.cuda.synchronize()
    barrier(world)

    def step(i, ev):
        ev[0].record(stream)
        call.prepare()
        ev[1].record(stream)
        call.carry()
        ev[2].record(stream)

    n0 = LAUNCHES["count"]
    total_ms, per = time_region(step, steps, stream, marks=3)
    launches = LAUNCHES["count"] - n0
    barrier(world)
    ms = max_over_ranks(total_ms / steps, world)
    prep_ms = statistics.mean(p[0] for p in per)
    carry_ms = statistics.mean(p[1] for p in per)
    tokens = x["q"].shape[0] * x["q"].shape[1]
    token_heads = tokens * preset.H
    d = preset.d
    in_b = PREFILL_IN_BYTES                               # q,k,v + log_alpha + beta
    out_b = PREFILL_OUT_BYTES                             # o
    n_seq = preset.B if x["cu_seqlens"] is None else x["cu_seqlens"].numel() - 1
    state_b = n_seq * preset.H * d * d * 4 * (2 if x["S0"] is not None else 1)
    op_bytes = token_heads * (in_b + out_b) + state_b
    ws_bytes = call.workspace.numel()
    if x["cu_seqlens"] is None:
        chunks = preset.B * ((x["q"].shape[1] + 63) // 64)
    else:
        cu = x["cu_seqlens"].cpu().tolist()
        chunks = sum((cu[i + 1] - cu[i] + 63) // 64 for i in range(len(cu) - 1))
    return dict(x=x, call=call, ms=ms, prep_ms=prep_ms, carry_ms=carry_ms, tokens=tokens,
                launches=launches, n_seq=n_seq,
                token_heads=token_heads, op_bytes=op_bytes, in_bytes=token_heads * in_b,
                out_bytes=token_heads * out_b + state_b, ws_bytes=ws_bytes,
                records=chunks * preset.H)


def bench_gdn(pre, steps, warmup, world):
    """The same prefill with one gate per token and head (kda_gdn_chunk_fwd): the
    gate is channel 0 of the workload's per-channel gate; the KDA call's
    workspace is reused."""
    from gated_delta_rule_132_b200 import kda
    x = pre["x"]
    la = x["log_alpha"][..., 0].contiguous()
    call = kda.ChunkFwdCall(x["q"], x["k"], x["v"], la, x["beta"], x["S0"], x["cu_seqlens"],
                            x["scale"], workspace=pre["call"].workspace, gate="head")
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        call.run()
    torch.cuda.synchronize()
    barrier(world)

    def step(i, ev):
        ev[0].record(stream)
        call.prepare()
        ev[1].record(stream)
        call.carry()
        ev[2].record(stream)

    total_ms, per = time_region(step, steps, stream, marks=3)
    barrier(world)
    d = x["q"].shape[-1]
    in_b = pre["token_heads"] * (3 * d * x["q"].element_size() + 4 + 4)
    return dict(ms=max_over_ranks(total_ms / steps, world),
                prep_ms=statistics.mean(p[0] for p in per),
                carry_ms=statistics.mean(p[1] for p in per), in_bytes=in_b)


# The backward (kda_chunk_bwd_ex, both algorithms: the token walk under the key
# "backward", the chunk-parallel default under "backward_chunked") on the long
# workload's shape cut to its first 8192 tokens: fp32 CUDA-core arithmetic; the
# token walk does ~28 dk*dv flop per token and head (two forward replays and the
# reverse step), which both keys count as the algorithmic work.
BWD_T = 8192
BWD_FLOP_PER_TOKEN_HEAD = 28 * 128 * 128
# DRAM bytes (read + write) of bwd_kernel per token and head: one ncu capture at
# T = 1024 (163.7 MB read + 1573.9 MB written), scaled by token-heads. Most of it
# is the per-block replay buffer written back from L2.
BWD_TRAFFIC_PER_TOKEN_HEAD = 53_027
# fp32 FMA peak from the SM count, FP32 lanes per SM and the maximum SM clock:
# 148 x 128 x 2 flop x 1.965 GHz.
FP32_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def bench_backward(steps, warmup, world, rank, dev, T_b=BWD_T, algo="token"):
    from gated_delta_rule_132_b200 import kda
    P = I.LONG
    devs = f"cuda:{dev}"
    x = I.make_prefill(1, T_b, P.H, P.d, P.dtype, P.gate_shift, 0.0, P.seed + 1000 * rank,
                       device=devs)
    g = torch.Generator(device=devs).manual_seed(P.seed + 7 + 1000 * rank)
    dO = torch.randn(x["v"].shape, generator=g, device=devs).to(P.dtype)
    need = kda.lib().kda_chunk_bwd_workspace_size_ex(1, T_b, P.H, P.d, P.d, 0, 1,
                                                     kda.BWD_ALGOS[algo])
    ws = torch.empty(int(need), dtype=torch.uint8, device=devs)
    args = (x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], dO)
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        kda.kda_chunk_bwd(*args, workspace=ws, algo=algo)
    torch.cuda.synchronize()
    barrier(world)

    def step(i, ev):
        ev[0].record(stream)
        kda.kda_chunk_bwd(*args, workspace=ws, algo=algo)
        ev[1].record(stream)

    total_ms, per = time_region(step, steps, stream, marks=2)
    barrier(world)
    return dict(ms=max_over_ranks(total_ms / steps, world),
                kern_ms=statistics.mean(p[0] for p in per), tokens=T_b,
                token_heads=T_b * P.H, workload=f"long_bf16_B1_H{P.H}_T{T_b}_d{P.d}")


def bench_decode(P, warmup, world, rank, dev, steps=None):
    """The decode workload as a chain of P.steps (1000) steps: every step's
    token inputs (fresh seeded q, k, v and gates per step) are generated on the
    device before the timed region, the state is carried from step to step,
    and every step is bracketed by events. GB/s = bytes per step / median step
    time."""
    from gated_delta_rule_132_b200 import kda
    devs = f"cuda:{dev}"
    S0 = I.make_decode_state(P.N, P.H, P.d, P.s_std, P.seed + 1000 * rank, device=devs)
    n_steps = P.steps if steps is None else steps
    toks = [I.make_decode_token(P.N, P.H, P.d, P.dtype, P.gate_shift,
                                seed=P.step_seed0 + i + 100000 * rank, device=devs)
            for i in range(n_steps)]
    o = torch.empty(P.N, P.H, P.d, dtype=P.dtype, device=devs)
    S = S0.clone()
    stream = torch.cuda.current_stream()
    for i in range(warmup):
        kda.kda_decode_step(**toks[i], S=S, o=o)
    S.copy_(S0)  # the timed chain starts from the workload's state
    torch.cuda.synchronize()
    barrier(world)

    def step(i, ev):
        ev[0].record(stream)
        kda.kda_decode_step(**toks[i], S=S, o=o)
        ev[1].record(stream)

    total_ms, per = time_region(step, n_steps, stream, marks=2)
    barrier(world)
    per = [p[0] for p in per]
    med = max_over_ranks(statistics.median(per), world)
    units = P.N * P.H
    state_b = 2 * units * P.d * P.d * 4
    io_b = units * (3 * P.d * 2 + 4 * P.d + 4 + P.d * 2)
    del toks
    return dict(ms=max_over_ranks(total_ms / n_steps, world), kern_ms=med, min_ms=min(per),
                steps=n_steps, bytes=state_b + io_b, state_bytes=state_b)


# The time-split prefill: one 1M-token sequence with few heads (B=1, H=4,
# T=2^20, d=128, bf16, the long workload's gates), where the plain sequential
# walk keeps 2 H = 8 SMs busy.
SPLIT_H, SPLIT_T = 4, 1 << 20


def bench_timesplit(steps, warmup, world, rank, dev):
    """kda_chunk_fwd_timesplit with the automatic segment count against the
    same call without a split (segments = 1), whole calls timed."""
    from gated_delta_rule_132_b200 import kda
    P = I.LONG
    x = I.make_prefill(1, SPLIT_T, SPLIT_H, P.d, P.dtype, P.gate_shift, 0.0,
                       P.seed + 11 + 1000 * rank, device=f"cuda:{dev}")
    L = kda.lib()
    auto = None
    for seg in range(2, 65):  # the count AUTO picks: the one whose workspace matches
        if (L.kda_chunk_fwd_timesplit_workspace_size(1, SPLIT_T, SPLIT_H, P.d, P.d, 0, 1, seg) ==
                L.kda_chunk_fwd_timesplit_workspace_size(1, SPLIT_T, SPLIT_H, P.d, P.d, 0, 1, 0)):
            auto = seg
            break
    stream = torch.cuda.current_stream()
    out = {}
    for name, seg in (("sequential", 1), ("split", 0)):
        ws = torch.empty(int(L.kda_chunk_fwd_timesplit_workspace_size(
            1, SPLIT_T, SPLIT_H, P.d, P.d, 0, 1, seg)), dtype=torch.uint8, device=x["q"].device)
        a = (x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], None, None, x["scale"])
        for _ in range(warmup):
            kda.kda_chunk_fwd_timesplit(*a, segments=seg, workspace=ws)
        torch.cuda.synchronize()
        barrier(world)

        def step(i, ev):
            ev[0].record(stream)
            kda.kda_chunk_fwd_timesplit(*a, segments=seg, workspace=ws)
            ev[1].record(stream)

        total_ms, per = time_region(step, steps, stream, marks=2)
        barrier(world)
        ms = max_over_ranks(total_ms / steps, world)
        out[name] = ms
        del ws
    chains = SPLIT_H
    nseg = auto or 1
    # two CTAs (one SM each, the two 64-column halves) per (sequence, head) in the
    # walk; the split's first pass runs 2 + 4 (P - 1) per chain, its second 2 (P - 1)
    return dict(ms_seq=out["sequential"], ms_split=out["split"], segments=nseg,
                tokens=SPLIT_T, ctas_seq=2 * chains,
                ctas_pass1=chains * (2 + 4 * (nseg - 1)), ctas_pass2=chains * 2 * (nseg - 1))


DECODE_TOKENS_T = 8  # tokens per multi-token decode call


def bench_decode_tokens(P, T, steps, warmup, world, rank, dev):
    """kda_decode_tokens on the decode workload's state with T tokens per call;
    four input sets of the call's shape are cycled (the 537 MB state, touched
    once each way per call, dominates the bytes)."""
    from gated_delta_rule_132_b200 import kda
    devs = f"cuda:{dev}"
    S = I.make_decode_state(P.N, P.H, P.d, P.s_std, P.seed + 2000 + 1000 * rank, device=devs)
    names = ("q", "k", "v", "log_alpha", "beta")
    pool = []
    for i in range(4):
        x = I.make_prefill(P.N, T, P.H, P.d, P.dtype, gate_shift=P.gate_shift,
                           seed=P.step_seed0 + 50000 + i + 100000 * rank, device=devs)
        pool.append({n: x[n] for n in names})
    o = torch.empty(P.N, T, P.H, P.d, dtype=P.dtype, device=devs)
    stream = torch.cuda.current_stream()
    for i in range(warmup):
        kda.kda_decode_tokens(**pool[i % 4], S=S, o=o)
    torch.cuda.synchronize()
    barrier(world)

    def step(i, ev):
        ev[0].record(stream)
        kda.kda_decode_tokens(**pool[i % 4], S=S, o=o)
        ev[1].record(stream)

    total_ms, per = time_region(step, steps, stream, marks=2)
    barrier(world)
    ms = max_over_ranks(total_ms / steps, world)
    kern_ms = statistics.mean(p[0] for p in per)
    units = P.N * P.H
    state_b = 2 * units * P.d * P.d * 4
    io_b = units * T * (3 * P.d * 2 + 4 * P.d + 4 + P.d * 2)
    return dict(ms=ms, kern_ms=kern_ms, bytes=state_b + io_b, T=T, tokens=P.N * T)


def bench_e2e(pre, steps, stream):
    """The same prefill through the public call with host buffers: every step
    copies its inputs in from pinned host memory, runs kda_chunk_fwd and copies
    o and S_final out. The uploads run on a second stream into two alternating
    device input sets, so step i+1's upload overlaps step i's prefill and
    download (PCIe carries the two directions at once); the timed region still
    holds every step's copies both ways."""
    from gated_delta_rule_132_b200 import kda
    x, call = pre["x"], pre["call"]
    names = ["q", "k", "v", "log_alpha", "beta"]
    host = {n: x[n].cpu().pin_memory() for n in names}
    dev = [{n: x[n] for n in names}, {n: torch.empty_like(x[n]) for n in names}]
    o_h = torch.empty(call.o.shape, dtype=call.o.dtype, pin_memory=True)
    s_h = torch.empty(call.S_final.shape, dtype=torch.float32, pin_memory=True)
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = o_h.numel() * o_h.element_size() + s_h.numel() * 4
    up = torch.cuda.Stream(device=x["q"].device)
    ready = [torch.cuda.Event() for _ in range(2)]
    free = [torch.cuda.Event() for _ in range(2)]
    used = [False, False]

    def one(i):
        b = i % 2
        if i == 0:
            up.wait_stream(stream)  # the first upload starts inside the timed region
        if used[b]:
            up.wait_event(free[b])  # the prefill that read this input set has finished
        with torch.cuda.stream(up):
            for n in names:
                dev[b][n].copy_(host[n], non_blocking=True)
        ready[b].record(up)
        stream.wait_event(ready[b])
        d = dev[b]
        kda.kda_chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], x["S0"],
                          x["cu_seqlens"], x["scale"], o=call.o, S_final=call.S_final,
                          workspace=call.workspace, stream=stream)
        free[b].record(stream)
        used[b] = True
        with torch.cuda.stream(stream):
            o_h.copy_(call.o, non_blocking=True)
            s_h.copy_(call.S_final, non_blocking=True)

    one(0)
    torch.cuda.synchronize()
    total_ms, _ = time_region(lambda i, ev: one(i), steps, stream)
    return dict(ms=total_ms / steps, h2d=h2d, d2h=d2h)


def cpu_baseline(pre_x, preset, budget_s=12.0):
    """The fp64 oracle as it stands on this host's cores, on the first tokens of
    the same workload (all heads), sized to roughly ``budget_s`` seconds."""
    import oracle
    cores = oracle.num_threads(0)
    xs = {k: (v.cpu() if torch.is_tensor(v) else v) for k, v in pre_x.items()}

    def run(T):
        sl = lambda t: t[:, :T]
        t0 = time.perf_counter()
        oracle.forward(sl(xs["q"]), sl(xs["k"]), sl(xs["v"]), sl(xs["log_alpha"]),
                       sl(xs["beta"]), xs["S0"], None, xs["scale"], n_threads=0)
        return time.perf_counter() - t0

    T = 256
    dt = run(T)
    T = int(min(preset.T, max(256, T * budget_s / max(dt, 1e-3))))
    T = max(64, T // 64 * 64)
    dt = run(T)
    used = min(cores, preset.H * xs["q"].shape[0])
    return {"value": T * xs["q"].shape[0] / dt, "unit": "tokens/s", "cores": used,
            "kind": "oracle",
            "sample": f"first {T} tokens x {preset.H} heads of the workload "
                      f"({dt:.1f} s, fp64 token-by-token, {used} threads)"}


def prefill_summary(pre, preset, hbm, tc_peak):
    """Throughput and roofline figures of one prefill measurement."""
    kernels = {
        "prepare": {"ms": pre["prep_ms"], "bytes": pre["in_bytes"],
                    "flop": pre["token_heads"] * INTRA_FLOP},
        "carry": {"ms": pre["carry_ms"], "bytes": pre["out_bytes"],
                  "flop": pre["token_heads"] * CARRY_FLOP},
    }
    flop = pre["token_heads"] * (INTRA_FLOP + CARRY_FLOP)
    op_ach = pre["op_bytes"] / (pre["ms"] / 1e3) / 1e9
    tc_ach = flop / (pre["ms"] / 1e3) / 1e12
    return {
        "workload": preset.name, "tokens": int(pre["tokens"]),
        "ms_per_step": round(pre["ms"], 4),
        "kernels_ms": {n: round(v["ms"], 4) for n, v in kernels.items()},
        "op_roofline": {"bound": "hbm", "achieved": round(op_ach, 1), "peak": hbm,
                        "unit": "GB/s", "frac": round(op_ach / hbm, 4),
                        "bytes_per_step": pre["op_bytes"],
                        "note": "algorithmic bytes of the whole prefill (q,k,v,log_alpha,beta "
                                "in, o out, states) / step time"},
        "tc": {"bound": "tensor", "achieved": round(tc_ach, 2), "peak": tc_peak,
               "unit": "TFLOP/s", "frac": round(tc_ach / tc_peak, 4),
               "flop_per_token_head": INTRA_FLOP + CARRY_FLOP,
               "intra_chunk_frac_of_prepare": round(
                   kernels["prepare"]["flop"] / (kernels["prepare"]["ms"] / 1e3) / 1e12 /
                   tc_peak, 4),
               "note": "tensor-core flops of the chunked form / step time, against the "
                       "sustained bf16 peak"},
    }, kernels


def run_ours(args, world, rank, dev):
    from gated_delta_rule_132_b200 import kda
    kda.lib()
    peaks, peak_kind = load_peaks()
    hbm = peaks["hbm_gbs"]
    tc_peak = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    preset = {"long": I.LONG, "chunked": I.CHUNKED, "varlen": I.VARLEN}[args.workload]
    clocks = ClockSampler(dev)
    extra = {}
    with clocks:
        pre = bench_prefill(preset, args.steps, args.warmup, world, rank, dev, peaks)
        if not args.no_configs:
            for other in (I.CHUNKED, I.VARLEN):
                if other is preset:
                    continue
                o = bench_prefill(other, args.config_steps, args.warmup, world, rank, dev, peaks)
                extra[other.name] = o
                del o["x"], o["call"]
                torch.cuda.empty_cache()
        dec = None if args.no_decode else bench_decode(I.DECODE, args.warmup, world, rank, dev,
                                                       args.decode_steps)
        dtok = None if args.no_decode else bench_decode_tokens(
            I.DECODE, DECODE_TOKENS_T, args.steps, args.warmup, world, rank, dev)
        gdn = None if args.no_gdn else bench_gdn(pre, args.steps, args.warmup, world)
        tsp = None if args.no_timesplit else bench_timesplit(
            min(args.steps, 5), args.warmup, world, rank, dev)
        bwd = None if args.no_backward else bench_backward(
            min(args.steps, 3), args.warmup, world, rank, dev, args.bwd_tokens)
        bwd_c = None if args.no_backward else bench_backward(
            min(args.steps, 3), args.warmup, world, rank, dev, args.bwd_tokens, algo="chunked")
    value = job_throughput(pre["tokens"], pre["ms"], world)
    summ, kernels = prefill_summary(pre, preset, hbm, tc_peak)

    # Roofline of the dominant prefill kernel: the operation's algorithmic bytes
    # (1540 B per token and head plus the states) over that kernel's time, and
    # the DRAM traffic ncu measured for it (per record x records) against its
    # own algorithmic bytes.
    dom = max(kernels, key=lambda n: kernels[n]["ms"])
    ach = pre["op_bytes"] / (kernels[dom]["ms"] / 1e3) / 1e9
    traffic = {n: (TRAFFIC_PER_RECORD[n] * pre["records"] if TRAFFIC_PER_RECORD[n] else None)
               for n in kernels}
    known = all(v is not None for v in traffic.values())
    roof = {"kernel": dom, "bound": "hbm", "achieved": round(ach, 1), "peak": hbm,
            "unit": "GB/s", "frac": round(ach / hbm, 4), "traffic": traffic[dom],
            "peak_source": peak_kind,
            "bytes_per_launch": pre["op_bytes"], "ms_per_launch": round(kernels[dom]["ms"], 4),
            "note": "algorithmic bytes of the whole prefill / the dominant kernel's time",
            "traffic_vs_algorithmic": {
                dom: (round(traffic[dom] / kernels[dom]["bytes"], 3)
                      if traffic[dom] is not None else None),
                "prefill": (round(sum(traffic.values()) / pre["op_bytes"], 3)
                            if known else None)},
            "traffic_note": "ncu DRAM bytes per record on the chunked workload x records"}
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(pre["ms"], 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; q,k L2-normalised, beta=sigmoid(N), "
                "log_alpha=-softplus(N-3))",
        "config": {"workload": preset.name, "B": preset.B, "T": int(pre["tokens"]), "H": preset.H,
                   "d_k": preset.d, "d_v": preset.d, "chunk": 64,
                   "l2": "inputs larger than L2 (no flush needed)",
                   "parallelism": f"independent problem per GPU x{world}"},
        "roofline": roof,
        "op_roofline": summ["op_roofline"],
        "tc": summ["tc"],
        "kernels_ms": summ["kernels_ms"],
        "gpu_launches": pre["launches"],
        "gpu_launches_note": "library kernel launches counted inside the timed prefill "
                             "region (kda_launch_count)",
    }
    for name, o in extra.items():
        sm, _ = prefill_summary(o, I.PRESETS[name], hbm, tc_peak)
        sm["value"] = round(job_throughput(o["tokens"], o["ms"], world), 1)
        sm["unit"] = "tokens/s"
        sm["steps"] = args.config_steps
        line[name.split("_")[0]] = sm
    if dec is not None:
        dec_ach = dec["bytes"] / (dec["kern_ms"] / 1e3) / 1e9
        line["decode"] = {"workload": I.DECODE.name, "value": round(dec_ach, 1), "unit": "GB/s",
                          "steps": dec["steps"], "chained": True,
                          "ms_per_step": round(dec["kern_ms"], 4),
                          "ms_per_step_min": round(dec["min_ms"], 4),
                          "ms_per_step_mean": round(dec["ms"], 4),
                          "roofline": {"kernel": "decode", "bound": "hbm",
                                       "achieved": round(dec_ach, 1), "peak": hbm,
                                       "unit": "GB/s", "frac": round(dec_ach / hbm, 4),
                                       "frac_of_nominal_8tbs": round(dec_ach / 8000.0, 4),
                                       "traffic": None, "bytes_per_launch": dec["bytes"]},
                          "note": "median over the chained steps; inputs of every step "
                                  "generated on the device before the timed region"}
    if dtok is not None:
        t_ach = dtok["bytes"] / (dtok["kern_ms"] / 1e3) / 1e9
        line["decode_tokens"] = {
            "workload": f"{I.DECODE.name}_T{dtok['T']}", "value": round(t_ach, 1),
            "unit": "GB/s", "tokens_per_s": round(dtok["tokens"] / (dtok["kern_ms"] / 1e3), 1),
            "ms_per_call": round(dtok["kern_ms"], 4),
            "vs_single_steps": (round(dtok["T"] * dec["kern_ms"] / dtok["kern_ms"], 3)
                                if dec is not None else None),
            "roofline": {"kernel": "decode (T tokens per call)", "bound": "hbm",
                         "achieved": round(t_ach, 1), "peak": hbm, "unit": "GB/s",
                         "frac": round(t_ach / hbm, 4), "traffic": None,
                         "bytes_per_launch": dtok["bytes"]}}
    if gdn is not None:
        g_ach = (gdn["in_bytes"] + pre["out_bytes"]) / (gdn["ms"] / 1e3) / 1e9
        line["gdn"] = {
            "workload": preset.name + "_gate_per_head",
            "value": round(job_throughput(pre["tokens"], gdn["ms"], world), 1),
            "unit": "tokens/s",
            "ms_per_step": round(gdn["ms"], 4),
            "kernels_ms": {"prepare": round(gdn["prep_ms"], 4), "carry": round(gdn["carry_ms"], 4)},
            "op_roofline": {"bound": "hbm", "achieved": round(g_ach, 1), "peak": hbm,
                            "unit": "GB/s", "frac": round(g_ach / hbm, 4),
                            "traffic": (TRAFFIC_PER_RECORD["gdn_prepare"] * pre["records"]
                                        if TRAFFIC_PER_RECORD["gdn_prepare"] else None),
                            "bytes_per_step": gdn["in_bytes"] + pre["out_bytes"]}}
    if tsp is not None:
        line["timesplit"] = {
            "workload": f"long_bf16_B1_H{SPLIT_H}_T{SPLIT_T}_d128",
            "value": round(job_throughput(tsp["tokens"], tsp["ms_split"], world), 1),
            "unit": "tokens/s", "ms_per_step": round(tsp["ms_split"], 4),
            "segments": tsp["segments"],
            "sequential": {"value": round(job_throughput(tsp["tokens"], tsp["ms_seq"], world), 1),
                           "ms_per_step": round(tsp["ms_seq"], 4),
                           "sms_busy_in_walk": tsp["ctas_seq"]},
            "sms_busy_in_walk": {"pass1": min(148, tsp["ctas_pass1"]),
                                 "pass2": min(148, tsp["ctas_pass2"])},
            "speedup": round(tsp["ms_seq"] / tsp["ms_split"], 3),
            "note": "whole kda_chunk_fwd_timesplit calls (prep + walk); one CTA per SM in the "
                    "sequential walk"}
    if bwd is not None:
        tf = bwd["token_heads"] * BWD_FLOP_PER_TOKEN_HEAD / (bwd["kern_ms"] / 1e3) / 1e12
        line["backward"] = {
            "workload": bwd["workload"] + "_backward",
            "value": round(job_throughput(bwd["tokens"], bwd["ms"], world), 1),
            "unit": "tokens/s", "ms_per_step": round(bwd["ms"], 3),
            "steps": min(args.steps, 3), "warmup": args.warmup,
            "roofline": {"kernel": "backward (fp32 CUDA cores)", "bound": "alu",
                         "achieved": round(tf, 3), "peak": round(FP32_PEAK_TFLOPS, 1),
                         "unit": "TFLOP/s", "frac": round(tf / FP32_PEAK_TFLOPS, 4),
                         "traffic": BWD_TRAFFIC_PER_TOKEN_HEAD * bwd["token_heads"],
                         "peak_source": "derived: 148 SMs x 128 fp32 lanes x 2 flop x 1.965 GHz",
                         "timed": "whole kda_chunk_bwd_ex call with the token walk (plan, "
                                  "bwd_kernel, reduction)"}}
    if bwd_c is not None:
        tf = bwd_c["token_heads"] * BWD_FLOP_PER_TOKEN_HEAD / (bwd_c["kern_ms"] / 1e3) / 1e12
        line["backward_chunked"] = {
            "workload": bwd_c["workload"] + "_backward",
            "value": round(job_throughput(bwd_c["tokens"], bwd_c["ms"], world), 1),
            "unit": "tokens/s", "ms_per_step": round(bwd_c["ms"], 3),
            "steps": min(args.steps, 3), "warmup": args.warmup,
            "vs_token_walk": round(bwd["ms"] / bwd_c["ms"], 3),
            "roofline": {"kernel": "chunk-parallel backward (fp32 CUDA cores)", "bound": "alu",
                         "achieved": round(tf, 3), "peak": round(FP32_PEAK_TFLOPS, 1),
                         "unit": "TFLOP/s", "frac": round(tf / FP32_PEAK_TFLOPS, 4),
                         "traffic": None,
                         "peak_source": "derived: 148 SMs x 128 fp32 lanes x 2 flop x 1.965 GHz",
                         "note": "the token walk's algorithmic flops (28 dk dv per token and "
                                 "head) over the call's time; the chunked form does more",
                         "timed": "whole kda_chunk_bwd_ex call (plan, record prep, two chunk "
                                  "walks, two token-gradient kernels)"}}
    line["clocks"] = clocks.summary()
    if not args.no_e2e:
        e = bench_e2e(pre, max(1, args.e2e_steps), torch.cuda.current_stream())
        e_ms = max_over_ranks(e["ms"], world)
        line["e2e"] = {"value": round(job_throughput(pre["tokens"], e_ms, world), 1),
                       "unit": "tokens/s", "h2d_bytes_per_step": e["h2d"],
                       "d2h_bytes_per_step": e["d2h"], "ms_per_step": round(e_ms, 3),
                       "steps": max(1, args.e2e_steps),
                       "note": "kda_chunk_fwd with pinned host buffers; each step's upload on "
                               "a second stream overlaps the previous step's prefill and "
                               "download"}
    line["page_claims"] = PAGE_CLAIMS
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(pre["x"], preset)
    if rank == 0:
        print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- reference arm
def run_reference(args, world, rank):
    """The fp64 oracle as the reference implementation, on the host cores."""
    if rank != 0:
        return
    import oracle
    preset = I.LONG
    T_s = args.ref_tokens
    x = I.make_prefill(1, T_s, preset.H, preset.d, preset.dtype, preset.gate_shift, 0.0,
                       preset.seed, device="cpu")
    cores = oracle.num_threads(0)

    def step():
        oracle.forward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], None, None,
                       x["scale"], n_threads=0)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = (time.perf_counter() - t0) / args.steps
    value = T_s / dt
    used = min(cores, preset.H)
    sample = (f"first {T_s} tokens x {preset.H} heads of {preset.name} per step "
              f"(fp64 token-by-token, {used} threads)")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 2), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
        "config": {"workload": preset.name, "B": preset.B, "T": preset.T, "H": preset.H,
                   "d_k": preset.d, "d_v": preset.d},
        "cpu_baseline": {"value": round(value, 2), "unit": "tokens/s", "cores": used,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 2), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["long", "chunked", "varlen"], default="long",
                    help="prefill workload (default: the long-context one)")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--decode-steps", type=int, default=None,
                    help="chained decode steps (default: the workload's 1000)")
    ap.add_argument("--no-backward", action="store_true",
                    help="skip the backward (kda_chunk_bwd) measurement")
    ap.add_argument("--bwd-tokens", type=int, default=BWD_T,
                    help="tokens of the backward measurement (all 32 heads)")
    ap.add_argument("--no-timesplit", action="store_true",
                    help="skip the time-split prefill measurement (B=1, H=4, T=2^20)")
    ap.add_argument("--no-gdn", action="store_true",
                    help="skip the one-gate-per-head (GDN) variant of the prefill")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the chunked and varlen prefill workloads")
    ap.add_argument("--config-steps", type=int, default=10,
                    help="timed steps of the chunked and varlen prefill workloads")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ref-tokens", type=int, default=1024,
                    help="tokens per reference-arm step (all 32 heads)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, world, rank)
        return
    world, rank, dev = dist_setup(args.gpus)
    try:
        run_ours(args, world, rank, dev)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
