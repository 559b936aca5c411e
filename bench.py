#!/usr/bin/env python
"""Benchmark of the KDA recurrence hot path on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

A step is one chunked prefill (gate cumsum, intra-chunk products, triangular
solve, WY build, state recall/correction, output, state update, varlen state
I/O) of the 8192-token, 32-head, d=128 bf16 workload through ``kda_prefill``.
``value`` is tokens/s with inputs resident in HBM; ``e2e`` is the same metric
with the step's inputs copied from pinned host memory and its outputs read back
inside the timed region (beside it, the uploads alone timed the same way: the host
link's bound on that number). The decode step (256 sequences x 32 heads, fp32 state
of 512 MiB streamed once in and once out) is measured in the same run and
reported under ``decode``; speculative decode on the same states (verify 4 draft
tokens, commit them, and the fused commit + verify step) under
``speculative_decode``; the varlen-24 and 1M-token prefills and the headline
prefill on raw inputs through the fused prologue under
``other_prefill_workloads``. Inputs (404 MB prefill, 512 MiB decode state) are
larger than L2, so no L2 flush is done between timed iterations.

Multi-GPU (torchrun): every rank runs its own replica of the workload (sequences
shard with no exchange), value = all ranks' tokens / max-over-ranks time.

``--impl reference`` times the fp64 CPU oracle (the only other place this file
runs it) on a bounded sample of the same workload, on the host's cores.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from gated_delta_rule_62_b200 import workloads as W  # noqa: E402

METRIC = "KDA tokens/s: chunked prefill (TC util %) and decode step (HBM GB/s % of peak)"
# Algorithmic work per token-head at C = 64, d_k = d_v = 128 (intra-chunk QK^T and KK^T,
# WY build, recall, output, state update); the 64x64 triangular solve is not counted.
FLOP_PER_TOKEN_HEAD = 180224
# Minimum HBM bytes per token-head for prefill: q, k, v (bf16) + log_alpha (fp32) + beta + out.
PREFILL_BYTES_PER_TOKEN_HEAD = 3 * 128 * 2 + 128 * 4 + 4 + 128 * 2
# dram__bytes_read.sum + dram__bytes_write.sum of one split_kernel launch on the headline workload,
# from one ncu capture; reported only while the kernel's sources are the ones it was taken on.
SPLIT_TRAFFIC_BYTES = 336.804608e6 + 50.913024e6
SPLIT_TRAFFIC_SOURCES_SHA256 = "7683404149faad35199e5ccbd9a0e4dd95ec1ce1c2eee23bbcabf33862b6a71d"


def measured_traffic():
    import hashlib
    h = hashlib.sha256()
    for f in ("kda_chunk_split.cu", "kda_chunk_common.cuh", "sm100.cuh"):
        with open(os.path.join(ROOT, "gated_delta_rule_62_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return SPLIT_TRAFFIC_BYTES if h.hexdigest() == SPLIT_TRAFFIC_SOURCES_SHA256 else None
# Decode: state read + write (fp32) + q, k, v + log_alpha + beta + out.
DECODE_BYTES_PER_TOKEN_HEAD = 2 * 128 * 128 * 4 + 3 * 128 * 2 + 128 * 4 + 4 + 128 * 2
# dram__bytes_read.sum + dram__bytes_write.sum of one launch of each decode-side kernel on the
# decode workload (ncu, one capture each), reported while kda_decode.cu and kda_internal.cuh hash
# to the sources they were taken on.
DECODE_SIDE_TRAFFIC = {"decode": 547.598e6 + 477.494e6, "verify": 580.534e6 + 5.976e6,
                       "commit": 591.556e6 + 475.534e6,
                       "commit_verify": 801.722e6 + 502.169e6}
DECODE_SIDE_SOURCES_SHA256 = "acacbb0fe0ec21eb1a777d768e3e51901ad5783020300f3fc7625988517b8e0a"


def decode_side_traffic(kernel):
    import hashlib
    h = hashlib.sha256()
    for f in ("kda_decode.cu", "kda_internal.cuh"):
        with open(os.path.join(ROOT, "gated_delta_rule_62_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return DECODE_SIDE_TRAFFIC[kernel] if h.hexdigest() == DECODE_SIDE_SOURCES_SHA256 else None


# Speculative decode, per (sequence, head) and draft token: verify reads the state once and per
# token q, k, v (bf16), log_alpha, beta, writes out (bf16) and u (fp32); commit reads and writes the
# state once and per accepted token reads k, log_alpha and u.
DRAFT_TOKENS = 4
VERIFY_STATE_BYTES, VERIFY_TOKEN_BYTES = 128 * 128 * 4, 3 * 128 * 2 + 128 * 4 + 4 + 128 * 2 + 128 * 4
COMMIT_STATE_BYTES, COMMIT_TOKEN_BYTES = 2 * 128 * 128 * 4, 128 * 2 + 128 * 4 + 128 * 4


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap,"
         "clocks.mem,temperature.memory")

    def __init__(self, index, tag="", interval_ms=200):
        self.index = index
        self.interval_ms = interval_ms
        self.proc = None
        out_dir = os.environ.get("KDA_CLOCKS_DIR") or tempfile.gettempdir()
        self.path = os.path.join(out_dir, f"kda_clocks{tag}_rank{index}.csv")

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", str(self.interval_ms)],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return None
        rows = [r.split(",") for r in open(self.path).read().strip().splitlines() if r.strip()]
        sm, mx, reasons, pw, mem, mtemp = [], None, set(), [], [], []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            r = [x.strip() for x in r]
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
                pw.append(float(r[3]))
            except ValueError:
                continue
            for n, v in zip(names, r[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
            for col, dst in ((9, mem), (10, mtemp)):  # may read N/A on some boards
                try:
                    dst.append(float(r[col]))
                except (IndexError, ValueError):
                    pass
        if not sm:
            return None
        load = [s for s in sm if s > 0.5 * (mx or max(sm))] or sm
        return {"sm_mhz": statistics.median(load), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "power_w": statistics.median(pw) if pw else None,
                "mem_mhz": statistics.median(mem) if mem else None,
                "mem_temp_c": max(mtemp) if mtemp else None}


def dist_setup(args):
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    if args.impl == "reference":
        # The oracle runs on rank 0's host cores only; no process group is needed.
        return int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")), ws
    if ws > 1:
        import datetime
        import torch.distributed as dist
        rank = int(os.environ["RANK"])
        local = int(os.environ.get("LOCAL_RANK", rank))
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
        return rank, local, ws
    torch.cuda.set_device(0)
    return 0, 0, 1


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, ws):
    if ws == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def cpu_oracle_sample(wl, seconds_target=15.0, max_tokens=None):
    """Time the fp64 oracle on the first tokens of every head of the workload (CPU generator)."""
    import oracle
    oracle.build()
    # A calibration run sizes the sample to roughly `seconds_target` seconds.
    T0 = 256
    sample = W.custom((T0,), wl.H, wl.dk, wl.dv, wl.dtype, seed=wl.seed)
    inp = W.make_inputs(sample, "cpu")
    arrs = [W.to_f64_numpy(inp[n]) for n in ("q", "k", "v", "log_alpha", "beta")]
    t = time.perf_counter()
    oracle.forward(*arrs)
    dt = time.perf_counter() - t
    T = int(min(wl.seqlens[0], max(T0, T0 * seconds_target / max(dt, 1e-6))))
    if max_tokens:
        T = min(T, max_tokens)
    sample = W.custom((T,), wl.H, wl.dk, wl.dv, wl.dtype, seed=wl.seed)
    inp = W.make_inputs(sample, "cpu")
    arrs = [W.to_f64_numpy(inp[n]) for n in ("q", "k", "v", "log_alpha", "beta")]
    t = time.perf_counter()
    oracle.forward(*arrs)
    dt = time.perf_counter() - t
    return {"value": T / dt, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"first {T} tokens x {wl.H} heads of {wl.name} (fp64, OpenMP over heads), {dt:.1f} s"}


def run_reference(args, rank, ws):
    if rank != 0:
        return
    import oracle
    oracle.build()
    wl = W.WORKLOADS[args.workload]
    Ts = args.ref_tokens
    sample = W.custom((Ts,), wl.H, wl.dk, wl.dv, wl.dtype, seed=wl.seed)
    inp = W.make_inputs(sample, "cpu")
    arrs = [W.to_f64_numpy(inp[n]) for n in ("q", "k", "v", "log_alpha", "beta")]
    for _ in range(args.warmup):
        oracle.forward(*arrs)
    t = time.perf_counter()
    for _ in range(args.steps):
        oracle.forward(*arrs)
    dt = (time.perf_counter() - t) / args.steps
    v = Ts / dt
    line = {"metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": wl.name, "global_batch": 1, "seq_len": wl.seqlens[0],
                       "heads": wl.H, "d_k": wl.dk, "d_v": wl.dv,
                       "parallelism": "replicas (sequences shard, no exchange)"},
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": oracle.num_threads(),
                             "kind": "oracle",
                             "sample": f"each step: first {Ts} tokens x {wl.H} heads of {wl.name}"},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def time_events(fn, steps, stream):
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(steps):
        fn()
    end.record(stream)
    end.synchronize()
    return start.elapsed_time(end) / steps  # ms


def bench_decode(args, K, stream, ws):
    """Decode-step throughput on the 256-sequence, 32-head workload."""
    wl = W.DECODE_256
    inp = W.make_inputs(wl, "cuda", seed=wl.seed + 7919 * args.rank)
    _, state = K.prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], None,
                         inp["cu_seqlens"], inp["cu_seqlens_dev"])
    nsteps = args.decode_steps
    steps = W.make_decode_steps(wl, inp["_gen"], nsteps, "cuda")
    del inp
    saved = state.clone()
    out = torch.empty(nsteps, wl.num_seqs, wl.H, wl.dv, dtype=torch.bfloat16, device="cuda")
    i = [0]

    def step():
        t = i[0] % nsteps
        K.decode_step(steps["q"][t], steps["k"][t], steps["v"][t], steps["log_alpha"][t],
                      steps["beta"][t], state, out=out[t], stream=stream)
        i[0] += 1

    for _ in range(3):
        step()
    state.copy_(saved)
    i[0] = 0
    torch.cuda.synchronize()
    barrier(ws)
    ms = time_events(step, nsteps, stream)
    ms = max_over_ranks(ms, ws)
    th = wl.num_seqs * wl.H
    gbs = DECODE_BYTES_PER_TOKEN_HEAD * th / (ms * 1e-3) / 1e9
    pk = peaks()
    return {"workload": wl.name, "steps": nsteps, "ms_per_step": ms,
            "tokens_per_s": wl.num_seqs * ws / (ms * 1e-3),
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / pk["hbm_gbs"], "traffic": decode_side_traffic("decode"),
                         "bytes_per_token_head": DECODE_BYTES_PER_TOKEN_HEAD,
                         "peak_source": pk["source"]},
            "gpu_launches": nsteps}


def bench_speculative(args, K, stream, ws, decode_ms):
    """Speculative decode on the decode workload's states with DRAFT_TOKENS draft tokens per
    sequence, all accepted: the verify and commit calls timed alone, and the steady-state step
    (commit the previous draft while verifying the next, one pass over the states), compared with
    as many single decode steps."""
    wl = W.DECODE_256
    inp = W.make_inputs(wl, "cuda", seed=wl.seed + 7919 * args.rank)
    _, state = K.prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], None,
                         inp["cu_seqlens"], inp["cu_seqlens_dev"])
    N, H, T, sets = wl.num_seqs, wl.H, DRAFT_TOKENS, 8
    steps = W.make_decode_steps(wl, inp["_gen"], sets * T, "cuda")
    del inp
    # [sets * T, N, ...] -> per set [N, T, ...]
    x = {n: t.reshape(sets, T, N, *t.shape[2:]).transpose(1, 2).contiguous() for n, t in steps.items()}
    del steps
    out = torch.empty(sets, N, T, H, wl.dv, dtype=torch.bfloat16, device="cuda")
    u = torch.empty(sets, N, T, H, wl.dv, dtype=torch.float32, device="cuda")
    acc = torch.full((N,), T, dtype=torch.int32, device="cuda")
    work = torch.empty(256, dtype=torch.uint8, device="cuda")
    i = [0]

    def verify():
        j = i[0] % sets
        K.decode_verify(x["q"][j], x["k"][j], x["v"][j], x["log_alpha"][j], x["beta"][j], state,
                        out=out[j], u_cache=u[j], workspace=work, stream=stream)
        i[0] += 1

    def commit():
        j = i[0] % sets
        K.decode_commit(x["k"][j], x["log_alpha"][j], u[j], state, acc, workspace=work, stream=stream)
        i[0] += 1

    def fused():  # steady state: commit the previous draft (all accepted) while verifying this one
        j = i[0] % sets
        jp = (j - 1) % sets
        K.decode_commit_verify(x["k"][jp], x["log_alpha"][jp], u[jp], acc, x["q"][j], x["k"][j],
                               x["v"][j], x["log_alpha"][j], x["beta"][j], state, out=out[j],
                               u_cache=u[j], workspace=work, stream=stream)
        i[0] += 1

    nsteps = max(8, args.decode_steps // 4)
    timed = {}
    for name, fn in (("verify", verify), ("commit", commit), ("commit_verify", fused)):
        i[0] = 0
        for _ in range(sets):
            fn()
        torch.cuda.synchronize()
        barrier(ws)
        timed[name] = max_over_ranks(time_events(fn, nsteps, stream), ws)
    pk = peaks()

    def roof(state_b, tok_b, ms, kernel):
        gbs = N * H * (state_b + T * tok_b) / (ms * 1e-3) / 1e9
        return {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": gbs / pk["hbm_gbs"], "traffic": decode_side_traffic(kernel),
                "peak_source": pk["source"]}

    del x, out, u, state
    torch.cuda.empty_cache()
    ms = timed["commit_verify"]
    return {"workload": f"{wl.name} states, {T} draft tokens per sequence, all accepted",
            "draft_tokens": T, "steps": nsteps, "verify_ms": timed["verify"],
            "commit_ms": timed["commit"], "ms_per_step": ms,
            "tokens_per_s": N * T * ws / (ms * 1e-3),
            "speedup_vs_single_steps": None if decode_ms is None else T * decode_ms / ms,
            "roofline": roof(COMMIT_STATE_BYTES, VERIFY_TOKEN_BYTES + COMMIT_TOKEN_BYTES, ms,
                             "commit_verify"),
            "verify_roofline": roof(VERIFY_STATE_BYTES, VERIFY_TOKEN_BYTES, timed["verify"], "verify"),
            "commit_roofline": roof(COMMIT_STATE_BYTES, COMMIT_TOKEN_BYTES, timed["commit"], "commit"),
            "gpu_launches": 3 * nsteps}


def bench_prefill_workload(wl, K, stream, steps, warmup, rank, prologue=0, segments=0, inp=None):
    """Device-timed kda_prefill of one workload (inputs resident in HBM); returns a summary dict.
    With ``prologue`` flags: kda_prefill_prologue on the same draws before activation. With
    ``segments`` > 0: kda_prefill_cp (context parallelism, each sequence cut into that many
    segments)."""
    if inp is None:
        inp = W.make_inputs(wl, "cuda", seed=wl.seed + 7919 * rank, raw=bool(prologue))
    N, T, H = wl.num_seqs, wl.total_tokens, wl.H
    out = torch.empty(T, H, wl.dv, dtype=wl.torch_dtype, device="cuda")
    fs = torch.empty(N, H, wl.dk, wl.dv, dtype=torch.float32, device="cuda")
    if segments:
        import ctypes
        wsz = int(K.lib().kda_prefill_cp_workspace_size(N, ctypes.c_void_p(inp["cu_seqlens"].data_ptr()), H,
                                                        wl.dk, wl.dv, K.KDA_BF16, segments))
    else:
        wsz = K.workspace_size(N, T, H, wl.dk, wl.dv, wl.torch_dtype)
    work = torch.empty(wsz, dtype=torch.uint8, device="cuda")

    def step():
        if segments:
            K.prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["initial_state"],
                      inp["cu_seqlens"], inp["cu_seqlens_dev"], out=out, final_state=fs, workspace=work,
                      stream=stream, algo="cp", segments=segments)
            return
        K.prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["initial_state"],
                  inp["cu_seqlens"], inp["cu_seqlens_dev"], out=out, final_state=fs, workspace=work,
                  stream=stream, prologue=prologue, gate_scale=W.GATE_SCALE)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device(), tag="_" + wl.name[:12], interval_ms=50) as clk:
        ms = time_events(step, steps, stream)
    th = T * H
    pk = peaks()
    del inp, out, fs, work
    torch.cuda.empty_cache()
    name = wl.name + (" raw inputs, fused prologue (q/k L2 norm, gate -softplus, beta sigmoid)"
                      if prologue else "")
    if segments:
        name += f" context-parallel, {segments} segments per sequence (kda_prefill_cp)"
    return {"workload": name, "tokens": T, "heads": H, "sequences": N, "ms_per_step": ms,
            "tokens_per_s": T / (ms * 1e-3),
            "tc_frac": FLOP_PER_TOKEN_HEAD * th / (ms * 1e-3) / 1e12 / pk["bf16_tflops"],
            "hbm_frac": PREFILL_BYTES_PER_TOKEN_HEAD * th / (ms * 1e-3) / 1e9 / pk["hbm_gbs"],
            "clocks": clk.summary()}


def run_ours(args, rank, local, ws):
    from gated_delta_rule_62_b200 import build
    from gated_delta_rule_62_b200 import kda as K
    if rank == 0:
        build.build()
    barrier(ws)
    wl = W.WORKLOADS[args.workload]
    stream = torch.cuda.current_stream()
    inp = W.make_inputs(wl, "cuda", seed=wl.seed + 7919 * rank)
    N, T, H = wl.num_seqs, wl.total_tokens, wl.H
    out = torch.empty(T, H, wl.dv, dtype=wl.torch_dtype, device="cuda")
    fs = torch.empty(N, H, wl.dk, wl.dv, dtype=torch.float32, device="cuda")
    wsz = K.workspace_size(N, T, H, wl.dk, wl.dv, wl.torch_dtype)
    work = torch.empty(wsz, dtype=torch.uint8, device="cuda")
    s0 = inp["initial_state"]

    def step():
        K.prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], s0,
                  inp["cu_seqlens"], inp["cu_seqlens_dev"], out=out, final_state=fs,
                  workspace=work, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    barrier(ws)
    with ClockSampler(local) as clk:
        torch.cuda.synchronize()
        ms = time_events(step, args.steps, stream)
        torch.cuda.synchronize()
    kernels_per_step_measured = K.last_launch_count()  # this library's kernels in one step
    barrier(ws)
    ms = max_over_ranks(ms, ws)
    clocks = clk.summary()

    # Per-launch duration of the prefill kernel, events on its stream, same timed loop shape.
    kern_ms = ms
    th = T * H
    pk = peaks()
    gbs = PREFILL_BYTES_PER_TOKEN_HEAD * th / (kern_ms * 1e-3) / 1e9
    tflops = FLOP_PER_TOKEN_HEAD * th / (kern_ms * 1e-3) / 1e12

    # End to end: pinned host inputs -> device, prefill, outputs -> pinned host, every step.
    # Pipelined over two device buffer sets and three streams: step i+1's upload overlaps step i's
    # kernel and download (PCIe is full duplex; the kernel runs on the compute stream). The serial
    # order (one stream) is timed as well and reported beside it.
    names = ("q", "k", "v", "log_alpha", "beta")
    host = {n: inp[n].cpu().pin_memory() for n in names}
    host_s0 = s0.cpu().pin_memory() if s0 is not None else None
    host_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    host_fs = torch.empty(fs.shape, dtype=fs.dtype).pin_memory()
    h2d = sum(host[n].numel() * host[n].element_size() for n in names)
    h2d += host_s0.numel() * 4 if host_s0 is not None else 0
    d2h = host_out.numel() * host_out.element_size() + host_fs.numel() * 4
    bufs = [{n: torch.empty_like(inp[n]) for n in names} for _ in range(2)]
    bufs_s0 = [torch.empty_like(s0) if s0 is not None else None for _ in range(2)]
    outs = [out, torch.empty_like(out)]
    fss = [fs, torch.empty_like(fs)]
    s_up, s_down = torch.cuda.Stream(), torch.cuda.Stream()
    ev = {k: [torch.cuda.Event(), torch.cuda.Event()] for k in ("up", "comp", "down")}
    for k in ev:  # every event starts out recorded (nothing pending)
        for e in ev[k]:
            e.record(stream)
    it = [0]

    def e2e_step(pipelined=True):
        b = it[0] % 2 if pipelined else 0
        it[0] += 1
        up = s_up if pipelined else stream
        down = s_down if pipelined else stream
        dev, dev_s0 = bufs[b], bufs_s0[b]
        up.wait_event(ev["comp"][b])         # the kernel two steps back has read these buffers
        with torch.cuda.stream(up):
            for n in names:
                dev[n].copy_(host[n], non_blocking=True)
            if dev_s0 is not None:
                dev_s0.copy_(host_s0, non_blocking=True)
        ev["up"][b].record(up)
        stream.wait_event(ev["up"][b])
        stream.wait_event(ev["down"][b])     # the download two steps back has read out / fs
        K.prefill(dev["q"], dev["k"], dev["v"], dev["log_alpha"], dev["beta"], dev_s0,
                  inp["cu_seqlens"], inp["cu_seqlens_dev"], out=outs[b], final_state=fss[b],
                  workspace=work, stream=stream)
        ev["comp"][b].record(stream)
        down.wait_event(ev["comp"][b])
        with torch.cuda.stream(down):
            host_out.copy_(outs[b], non_blocking=True)
            host_fs.copy_(fss[b], non_blocking=True)
        ev["down"][b].record(down)

    def timed_e2e(pipelined, steps):
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record(stream)
        s_up.wait_event(start)
        s_down.wait_event(start)
        for _ in range(steps):
            e2e_step(pipelined)
        for b in range(2):
            stream.wait_event(ev["down"][b])
        end.record(stream)
        end.synchronize()
        return start.elapsed_time(end) / steps

    def timed_upload(steps):  # the step's host -> device copies alone: the link's own bound
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record(s_up)
        for i in range(steps):
            dev = bufs[i % 2]
            with torch.cuda.stream(s_up):
                for n in names:
                    dev[n].copy_(host[n], non_blocking=True)
                if host_s0 is not None:
                    bufs_s0[i % 2].copy_(host_s0, non_blocking=True)
        end.record(s_up)
        end.synchronize()
        return start.elapsed_time(end) / steps

    e2e_ms = e2e_serial_ms = upload_ms = None
    if not args.no_e2e:
        n_e2e = max(4, args.steps // 2)
        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        barrier(ws)
        e2e_ms = max_over_ranks(timed_e2e(True, n_e2e), ws)
        torch.cuda.synchronize()
        barrier(ws)
        e2e_serial_ms = max_over_ranks(timed_e2e(False, n_e2e), ws)
        torch.cuda.synchronize()
        barrier(ws)
        upload_ms = max_over_ranks(timed_upload(n_e2e), ws)
        torch.cuda.synchronize()
    del host, bufs, bufs_s0, outs, fss

    dec = bench_decode(args, K, stream, ws) if not args.no_decode else None
    spec = None if args.no_decode else bench_speculative(args, K, stream, ws, dec["ms_per_step"])
    extra = None
    if not args.no_extra:
        extra = [bench_prefill_workload(W.VARLEN_24, K, stream, 10, 3, rank)]
        inp_1m = W.make_inputs(W.PREFILL_1M, "cuda", seed=W.PREFILL_1M.seed + 7919 * rank)
        for segs in (0, 2, 4):  # the million-token prefill without and with context parallelism
            extra.append(bench_prefill_workload(W.PREFILL_1M, K, stream, 6, 3, rank, segments=segs,
                                                inp=inp_1m))
        del inp_1m
        torch.cuda.empty_cache()
        extra.append(bench_prefill_workload(wl, K, stream, 20, 3, rank, prologue=K.PROLOGUE_ALL))

    if rank != 0:
        return
    cpu = None
    if ws == 1 and not args.no_cpu_baseline:
        cpu = cpu_oracle_sample(wl, seconds_target=args.cpu_seconds)
    kernels_per_step = kernels_per_step_measured
    in_mb = wl.total_tokens * H * (PREFILL_BYTES_PER_TOKEN_HEAD - wl.dv * 2) / 1e6  # inputs, no out
    line = {
        "metric": METRIC, "value": T * ws / (ms * 1e-3), "unit": "tokens/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": wl.name, "global_batch": N * ws, "seq_len": T, "heads": H,
                   "d_k": wl.dk, "d_v": wl.dv, "chunk": 64,
                   "parallelism": f"replicas x{ws} (sequences shard, no exchange)",
                   "l2": f"inputs ({in_mb:.0f} MB) larger than L2; no flush" if in_mb > 126 else
                         f"inputs ({in_mb:.0f} MB) fit in L2; no flush"},
        "tc_util": {"achieved_tflops": tflops, "peak_tflops": pk["bf16_tflops"],
                    "frac": tflops / pk["bf16_tflops"], "flop_per_token_head": FLOP_PER_TOKEN_HEAD,
                    "peak_source": pk["source"] + " burst"},
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                     "frac": gbs / pk["hbm_gbs"],
                     # the ncu counters were taken on the 8192 x 32 workload's split kernel
                     "traffic": args.traffic if args.traffic is not None else
                                (measured_traffic() if wl is W.PREFILL_8K else None),
                     "bytes_per_token_head": PREFILL_BYTES_PER_TOKEN_HEAD,
                     "kernel_ms": kern_ms, "peak_source": pk["source"]},
        "e2e": None if e2e_ms is None else {
            "value": T * ws / (e2e_ms * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
            "copies": "pipelined: step i+1's upload overlaps step i's kernel and download "
                      "(two buffer sets, three streams)",
            "serial_ms_per_step": e2e_serial_ms,
            "serial_value": T * ws / (e2e_serial_ms * 1e-3),
            # the uploads alone, timed the same way: the host link's bound on this step
            "upload_only_ms_per_step": upload_ms,
            "upload_gbs": h2d / (upload_ms * 1e-3) / 1e9,
            "frac_of_upload_bound": upload_ms / e2e_ms},
        "decode": dec,
        "speculative_decode": spec,
        "other_prefill_workloads": extra,
        "gpu_launches": args.steps * kernels_per_step,
        "clocks": clocks,
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=W.PREFILL_8K.name, choices=sorted(W.WORKLOADS))
    ap.add_argument("--decode-steps", type=int, default=1024)
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the varlen-24 and 1M-token prefill measurements")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--ref-tokens", type=int, default=2048)
    ap.add_argument("--traffic", type=float, default=None,
                    help="ncu dram bytes (read+write) per launch of the prefill kernel, if measured")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    rank, local, ws = dist_setup(args)
    args.rank = rank
    try:
        if args.impl == "reference":
            run_reference(args, rank, ws)
        else:
            run_ours(args, rank, local, ws)
    finally:
        if ws > 1 and args.impl == "ours":
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
