#!/usr/bin/env python
"""Benchmark of the DiT attention-block hot path on B200.

One step = one pass of the whole path over one batch of the workload:
  u        = dit_adaln_modulate(x, gamma, beta)          (adaLN, memory-bound)
  q_r, k_r = dit_rope3d_qk(q, k, 3D-RoPE)                (RoPE pass, memory-bound)
  o        = dit_attn_fwd(q_r, k_r, v)                   (tensor-core bound)
  out      = dit_gated_residual(x, o, alpha)             (adaLN-Zero gate, memory-bound)
(--rope-mode fused rotates inside the attention kernel instead.) The q/k/v
projections around the path are not part of it; q, k, v, x and the adaLN parameters
are seeded synthetic bf16 tensors with the workload's shapes. Timed separately and
reported as components, not in the step: the Euler step, the block's linear layers
(bf16 and E4M3), and the E4M3 attention modes.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 480p] [--impl reference]

Prints one JSON line (rank 0). `value` is attention TFLOP/s over the whole step
(algorithmic 4*L^2*d*H FLOPs of every sequence, all ranks, / max-over-ranks time).
With N > 1 (torchrun), every rank runs its own batch (weak scaling, no collective
on the data path). `--impl reference` times the fp64 CPU oracle instead, on a
bounded sample of the same workload.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "3D-RoPE attention TFLOP/s & % BF16 peak; adaLN GB/s & % HBM peak (1xB200)"
UNIT = "TFLOP/s"
# DRAM bytes per head of one attention launch at the 480P geometry, from an ncu capture
# with 16 heads (dram__bytes_read.sum + dram__bytes_write.sum = 410.445 + 118.815 MB, over
# 16), keyed by RoPE mode ("prepass" and "none" run the same kernel, without in-kernel
# RoPE; the in-kernel RoPE mode has no capture of the current kernel: null). Heads are
# independent, so a launch's traffic is this times its head count. Other workloads
# report null.
ATTN_DRAM_BYTES_PER_HEAD_480P = {"prepass": 529.260544e6 / 16, "none": 529.260544e6 / 16,
                                 "fused": None}


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        # nvidia-smi takes a moment to start: wait (bounded) for its first sample so that
        # even a short timed region is covered
        deadline = time.time() + 5.0
        while self.proc is not None and time.time() < deadline and self.proc.poll() is None:
            if os.path.getsize(self.path) > 0:
                break
            time.sleep(0.05)
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = []
        try:
            for line in open(self.path):
                parts = [s.strip() for s in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        finally:
            os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        def num(x):
            try:
                return float(x)
            except ValueError:
                return None

        sm = [v for v in (num(r[1]) for r in rows) if v is not None]
        watts = [v for v in (num(r[3]) for r in rows) if v is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        mask = 0
        for r in rows:  # union of the active-reasons bitmasks (0x4: software power cap)
            try:
                mask |= int(r[4], 16)
            except ValueError:
                pass
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": num(rows[0][2]),
                "reasons": reasons, "active_mask": hex(mask),
                "power_w": statistics.median(watts) if watts else None, "samples": len(rows)}


def widen_qkv(inp):
    """The oracle's fp64 copies of q, k, v (made once, outside any timed region)."""
    from diffusion_transformer_video_b200 import workloads as wl
    return tuple(wl.bf16_bits_to_f64(inp[n]) for n in ("q", "k", "v"))


def cpu_oracle_attention(w, qkv64, n_rows: int, seed: int = 0):
    """Time the oracle's 3D-RoPE attention on `n_rows` sampled query rows (all heads, all
    keys of their sequences). Returns (TFLOP/s, seconds, sample description, threads)."""
    import oracle
    rng = np.random.default_rng([seed, 77])
    rows = np.sort(rng.choice(w.rows, size=n_rows, replace=False)).astype(np.int64)
    cu = w.cu_seqlens
    q, k, v = qkv64
    t0 = time.perf_counter()
    ref_o, _ = oracle.attn_fwd(q, k, v, cu, qrows=rows, rope=w.rope_desc())
    dt = time.perf_counter() - t0
    cpu_oracle_attention.last = (rows, ref_o)  # kept for the parity figures of the GPU arm
    seq_of = np.searchsorted(cu, rows, side="right") - 1
    flops = float(sum(4.0 * (cu[s + 1] - cu[s]) * w.head_dim * w.heads for s in seq_of))
    threads = oracle.threads()
    sample = (f"{n_rows} query rows x {w.heads} heads of {w.name}, all keys of their sequence; "
              f"the oracle's 3D-RoPE of the full q and k is inside the timed call (fp64, OpenMP)")
    return flops / dt / 1e12, dt, sample, threads


def cpu_oracle_memory_steps(w, x_bits, seed: int = 0, n_rows: int = 4096):
    """The oracle's adaLN modulation and gated residual on the first `n_rows` rows of
    x (one parameter group; the residual's branch input y is the next `n_rows` rows of
    x), on all its threads. Rates are in the bf16 algorithmic bytes of the GPU kernels
    (4 and 6 bytes per element), so that they compare with the GPU figures."""
    import oracle
    from diffusion_transformer_video_b200 import workloads as wl
    n = min(n_rows, w.rows // 2)
    D = w.d_model
    x = wl.bf16_bits_to_f64(x_bits[:n])
    y = wl.bf16_bits_to_f64(x_bits[n:2 * n])
    prm = wl.make_inputs(w, seed, which=("gamma", "beta", "alpha"))
    g, b, a = (wl.bf16_bits_to_f64(prm[k][:1]) for k in ("gamma", "beta", "alpha"))
    out = {}
    for name, call, per_elem in (("adaln_modulate", lambda: oracle.adaln_modulate(x, g, b, n), 4),
                                 ("gated_residual", lambda: oracle.gated_residual(x, y, a, n), 6)):
        t0 = time.perf_counter()
        call()
        dt = time.perf_counter() - t0
        out[name] = {"GB/s": per_elem * n * D / dt / 1e9, "seconds": dt, "rows": n}
    out["sample"] = (f"the first {n} rows x {D} of {w.name}'s x (the residual's y: the next "
                     f"{n}), one parameter group, fp64, {oracle.threads()} threads")
    return out


def cpu_oracle_attention_one_thread(w, qkv64, n_rows: int, seed: int = 0):
    """The oracle's attention on one host thread, over operands it rotated beforehand
    on all threads (its fp64 3D-RoPE of the whole q and k would dominate a one-thread
    sample): TFLOP/s, seconds and the sample, for `n_rows` sampled query rows."""
    import oracle
    rng = np.random.default_rng([seed, 78])
    rows = np.sort(rng.choice(w.rows, size=n_rows, replace=False)).astype(np.int64)
    cu = w.cu_seqlens
    q, k, v = qkv64
    r = w.rope_desc()
    qr = oracle.rope3d(q, cu, r["grid_h"], r["grid_w"], r["bands"], r["base"], r["offsets"])
    kr = oracle.rope3d(k, cu, r["grid_h"], r["grid_w"], r["bands"], r["base"], r["offsets"])
    before = oracle.threads()
    oracle.set_threads(1)
    try:
        t0 = time.perf_counter()
        oracle.attn_fwd(qr, kr, v, cu, qrows=rows)
        dt = time.perf_counter() - t0
    finally:
        oracle.set_threads(before)
    seq_of = np.searchsorted(cu, rows, side="right") - 1
    flops = float(sum(4.0 * (cu[s + 1] - cu[s]) * w.head_dim * w.heads for s in seq_of))
    sample = (f"{n_rows} query rows x {w.heads} heads of {w.name}, all keys of their sequence, "
              f"q and k rotated before the timed call (fp64, 1 thread)")
    return flops / dt / 1e12, dt, sample


L2_BYTES = 126e6                    # B200 L2
L2_FLUSH_BYTES = 256 << 20          # a write this large evicts every line of it


def l2_resident_free(w) -> bool:
    """True when one input tensor alone is larger than L2 (no flush needed)."""
    return w.rows * w.d_model * 2 > L2_BYTES


def resolve_workload(args):
    """The workload of this run (with --heads applied)."""
    from diffusion_transformer_video_b200 import workloads as wl
    w = wl.get_workload(args.workload, args.seed)
    if args.heads:
        import dataclasses
        w = dataclasses.replace(w, name=f"{w.name}-h{args.heads}", heads=args.heads)
    return w


def workload_config(w, world: int) -> dict:
    """The `config` object of the JSON line, the same for both arms."""
    rows, D = w.rows, w.d_model
    return {"workload": w.name, "batch": w.n_seq, "seq_len": w.max_seqlen,
            "rows": rows, "heads": w.heads, "head_dim": w.head_dim, "d_model": D,
            "rope_bands": list(w.bands), "grid": [w.grid_h, w.grid_w],
            "parallelism": f"dp{world} (independent batches)",
            "l2": "inputs larger than L2 (x, q, k, v are %.0f MB each)" % (rows * D * 2 / 1e6)
            if l2_resident_free(w) else
            "L2 flushed between steps (%d MB write outside the step events)" % (L2_FLUSH_BYTES >> 20),
            "note": w.note}


def run_reference(args, rank, world):
    from diffusion_transformer_video_b200 import workloads as wl
    if rank != 0:
        return
    w = resolve_workload(args)
    inp = wl.make_inputs(w, args.seed, which=("q", "k", "v"))
    qkv64 = widen_qkv(inp)
    n_rows = args.ref_rows
    vals = []
    for i in range(args.warmup + args.steps):
        tf, dt, sample, threads = cpu_oracle_attention(w, qkv64, n_rows, seed=args.seed + i)
        if i >= args.warmup:
            vals.append((tf, dt))
    value = statistics.mean(v for v, _ in vals)
    ms = 1e3 * statistics.mean(d for _, d in vals)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded bf16 N(0,1) inputs widened to fp64)",
            "config": workload_config(w, world),
            "cpu_baseline": {"kind": "oracle", "value": value, "unit": UNIT, "cores": threads,
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def rank_seed(seed: int, rank: int) -> int:
    """Every rank draws its own batch of the workload."""
    return seed + 1000 * rank


def max_over_ranks(values, dist=None, device="cpu"):
    """Elementwise max of per-rank timings (the slowest rank sets the job's time)."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return [float(v) for v in values]
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def job_throughput(flops_per_rank: float, world: int, ms_per_step: float) -> float:
    """Whole-job TFLOP/s: the units all ranks processed / the max-over-ranks step time."""
    return flops_per_rank * world / (ms_per_step * 1e-3) / 1e12


STEP_INPUTS = ("x", "q", "k", "v", "gamma", "beta", "alpha")


def param_sets_on_device(w, seed, torch):
    """The workload's adaLN parameter sets (two for the 720P expert pair) on the device."""
    from diffusion_transformer_video_b200 import workloads as wl
    sets = []
    for ps in range(w.param_sets):
        prm = wl.make_inputs(w, seed, which=("gamma", "beta", "alpha"), param_set=ps)
        sets.append({k: torch.from_numpy(v.view(np.int16)).view(torch.bfloat16).cuda()
                     for k, v in prm.items()})
    return sets


class StepRunner:
    """One workload's step on the device: modulate -> RoPE pass -> attention -> residual,
    with CUDA events around each call. Step i uses adaLN parameter set i % param_sets
    (the 720P workload alternates its high- and low-noise experts)."""

    def __init__(self, w, seed, args, torch, dit3d, host=None):
        from diffusion_transformer_video_b200 import workloads as wl
        self.w, self.args, self.torch, self.dit3d = w, args, torch, dit3d
        if host is None:
            inp = wl.make_inputs(w, seed, which=("x", "q", "k", "v"))
            host = {k: torch.from_numpy(v.view(np.int16)).view(torch.bfloat16)
                    for k, v in inp.items()}
        self.dev = {k: v.to("cuda", non_blocking=True) for k, v in host.items()}
        self.params = param_sets_on_device(w, seed, torch)
        rows, D, H, d = w.rows, w.d_model, w.heads, w.head_dim
        self.desc = dit3d.rope_desc(w.grid_h, w.grid_w, w.bands, w.base)
        self.cu = None
        if w.varlen:
            cu_host = torch.from_numpy(w.cu_seqlens)
            self.cu = (cu_host.cuda(), cu_host)
        self.u = torch.empty(rows, D, dtype=torch.bfloat16, device="cuda")
        self.o = torch.empty(rows, H, d, dtype=torch.bfloat16, device="cuda")
        self.out = torch.empty(rows, D, dtype=torch.bfloat16, device="cuda")
        self.q_rot = self.k_rot = None
        if args.rope_mode == "prepass":
            self.q_rot, self.k_rot = torch.empty_like(self.dev["q"]), torch.empty_like(self.dev["k"])
        self.stream = torch.cuda.current_stream()

    def step(self, b=None, i=0, ev=None, out_t=None):
        """One pass of the path over the batch `b` (default: this workload's inputs)."""
        w, dit3d, args = self.w, self.dit3d, self.args
        b = self.dev if b is None else b
        prm = b.get("params", self.params)[i % w.param_sets]
        out_t = self.out if out_t is None else out_t
        rec = (lambda k: ev[k].record(self.stream)) if ev is not None else (lambda k: None)
        rec(0)
        dit3d.dit_adaln_modulate(b["x"], prm["gamma"], prm["beta"], w.rows_per_group, out=self.u)
        rec(1)
        if args.rope_mode == "prepass":
            dit3d.dit_rope3d_qk(b["q"], b["k"], self.desc, n_seq=w.n_seq, cu_seqlens=self.cu,
                                q_out=self.q_rot, k_out=self.k_rot)
            qa, ka = self.q_rot, self.k_rot
        else:
            qa, ka = b["q"], b["k"]
        rec(2)
        dit3d.dit_attn_fwd(qa, ka, b["v"], n_seq=w.n_seq, cu_seqlens=self.cu, out=self.o,
                           rope=self.desc if args.rope_mode == "fused" else None)
        rec(3)
        dit3d.dit_gated_residual(b["x"], self.o.view(w.rows, w.d_model), prm["alpha"],
                                 w.rows_per_group, out=out_t)
        rec(4)

    def timed(self, steps, warmup, barrier=lambda: None, local_rank=0):
        """W untimed steps, then `steps` timed ones (L2 flushed between steps when one
        input tensor fits in L2). Returns per-call mean times, the timed region's length
        and the clocks sampled during it."""
        torch = self.torch
        for i in range(warmup):
            self.step(i=i)
        torch.cuda.synchronize()
        self.dit3d.dit_check_device()
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(steps)]
        flush = None if l2_resident_free(self.w) else torch.empty(L2_FLUSH_BYTES // 4,
                                                                  dtype=torch.float32,
                                                                  device="cuda")
        barrier()
        torch.cuda.synchronize()
        with ClockSampler(local_rank) as clk:
            t_start = torch.cuda.Event(enable_timing=True)
            t_end = torch.cuda.Event(enable_timing=True)
            t_start.record(self.stream)
            for i in range(steps):
                if flush is not None:
                    flush.fill_(float(i))
                self.step(i=i, ev=evs[i])
            t_end.record(self.stream)
            torch.cuda.synchronize()
        barrier()
        self.dit3d.dit_check_device()
        elapsed = (t_start.elapsed_time(t_end) if flush is None
                   else sum(e[0].elapsed_time(e[4]) for e in evs))
        mean = lambda a, b: statistics.mean(e[a].elapsed_time(e[b]) for e in evs)
        return {"elapsed_ms": elapsed, "mod": mean(0, 1), "rope": mean(1, 2), "attn": mean(2, 3),
                "res": mean(3, 4), "clocks": clk.summary()}

    def free(self):
        for name in ("dev", "params", "u", "o", "out", "q_rot", "k_rot", "cu"):
            setattr(self, name, None)
        self.torch.cuda.empty_cache()


def workload_figures(w, t, pk, rope_mode) -> dict:
    """Throughput and roofline fractions of one workload's timed steps: attention TFLOP/s
    against the burst bf16 peak (and the sustained one), memory-bound calls in GB/s
    against the HBM copy bandwidth."""
    rows, D = w.rows, w.d_model
    flops = w.attn_flops()
    att = flops / (t["attn"] * 1e-3) / 1e12
    def mem(ms, nbytes):
        gbs = nbytes / (ms * 1e-3) / 1e9
        return {"ms": ms, "GB/s": gbs, "frac_hbm": gbs / pk["hbm_gbs"], "bytes": nbytes}
    out = {
        "attn_fwd": {"ms": t["attn"], "TFLOP/s": att, "frac": att / pk["bf16_tflops"],
                     "frac_sustained": att / pk["bf16_tflops_sustained"], "flops": flops},
        "adaln_modulate": mem(t["mod"], 4.0 * rows * D),
        "rope3d_qk": mem(t["rope"], 8.0 * rows * D) if rope_mode == "prepass" else None,
        "gated_residual": mem(t["res"], 6.0 * rows * D),
        "step_ms": t["step_ms"], "step_TFLOP/s": flops / (t["step_ms"] * 1e-3) / 1e12,
        "rows": rows, "sequences": w.n_seq, "heads": w.heads, "d_model": D,
        "clocks_sm_mhz": t["clocks"]["sm_mhz"], "clock_reasons": t["clocks"]["reasons"],
    }
    if w.param_sets > 1:
        out["param_sets"] = f"{w.param_sets} adaLN parameter sets, alternated step by step"
    if w.varlen:
        out["frames"] = list(w.frames)
        out["seqlens"] = list(w.seqlens)
    if w.name.startswith("tiny"):
        out["note"] = "latency-bound (64 tokens): reported, not held to the roofline targets"
    return out


def run_ulysses(args, rank, world, local_rank):
    """Ulysses sequence parallelism over the job's ranks: ONE batch of the workload,
    each sequence split over the ranks by tokens (strong scaling), head chunks whose
    all-to-all overlaps the previous chunk's RoPE pass and attention. A step is one
    ulysses_attention call (exchange, RoPE, attention, exchange back)."""
    import datetime
    import torch
    import torch.distributed as dist
    from diffusion_transformer_video_b200 import dit3d, ulysses, workloads as wl

    torch.cuda.set_device(local_rank)
    if world == 1 and "MASTER_PORT" not in os.environ:   # a plain single-process run
        import socket
        with socket.socket() as sk:
            sk.bind(("127.0.0.1", 0))
            os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(sk.getsockname()[1]))
    dist.init_process_group("nccl", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120),
                            device_id=torch.device("cuda", local_rank))
    try:
        w = resolve_workload(args)
        layout = ulysses.UlyssesLayout(w.cu_seqlens, world)
        mine = layout.local_rows(rank).numpy()
        inp = wl.make_inputs(w, args.seed, which=("q", "k", "v"))
        loc = {k: torch.from_numpy(np.ascontiguousarray(v[mine]).view(np.int16))
               .view(torch.bfloat16).cuda() for k, v in inp.items()}
        del inp
        desc = dit3d.rope_desc(w.grid_h, w.grid_w, w.bands, w.base)
        h_loc = w.heads // world
        chunks = args.head_chunks if args.head_chunks else max(
            c for c in range(1, h_loc + 1) if h_loc % c == 0 and c <= 4)
        run = lambda: ulysses.ulysses_attention(loc["q"], loc["k"], loc["v"], rope=desc,
                                                cu_seqlens=w.cu_seqlens, head_chunks=chunks)
        for _ in range(args.warmup):
            run()
        torch.cuda.synchronize()
        dit3d.dit_check_device()
        dist.barrier()
        torch.cuda.synchronize()
        stream = torch.cuda.current_stream()
        with ClockSampler(local_rank) as clk:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(args.steps):
                run()
            e1.record(stream)
            torch.cuda.synchronize()
        dist.barrier()
        dit3d.dit_check_device()
        ms = max_over_ranks([e0.elapsed_time(e1) / args.steps], dist, "cuda")[0]
        clocks = clk.summary()
        flops = w.attn_flops()
        if rank == 0:
            pk = _peaks()
            value = flops / (ms * 1e-3) / 1e12
            line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
                    "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
                    "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
                    "dtype": "bf16", "data": "synthetic (seeded bf16 N(0,1) q/k/v)",
                    "config": dict(workload_config(w, world),
                                   parallelism=f"ulysses{world} (tokens split over ranks, "
                                               f"{chunks} head chunks per rank)"),
                    "gpu_launches": None,
                    "roofline": {"bound": "tensor", "achieved": value / world,
                                 "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                                 "frac": value / world / pk["bf16_tflops"], "traffic": None,
                                 "kernel": "whole Ulysses step per GPU (exchanges included)"},
                    "clocks": clocks, "e2e": None, "cpu_baseline": None}
            print(json.dumps(line), flush=True)
    finally:
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="480p")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=8)
    ap.add_argument("--ref-rows", type=int, default=24, help="oracle sample rows per step")
    ap.add_argument("--cpu-rows", type=int, default=64, help="oracle rows for cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-linear", action="store_true",
                    help="skip timing the block's linear layers (separate components)")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the other four workloads (the `workloads` object)")
    ap.add_argument("--workload-steps", type=int, default=10,
                    help="timed steps per workload in the `workloads` object")
    ap.add_argument("--rope-mode", default="prepass", choices=["prepass", "fused", "none"],
                    help="prepass: dit_rope3d_qk into scratch, then attention (the product "
                         "path, fastest); fused: RoPE inside the attention kernel (no scratch); "
                         "none: attention alone (not the workload, a kernel-speed reference)")
    ap.add_argument("--attn-variant", type=int, default=0, choices=[0, 1],
                    help="0: single-CTA attention kernel; 1: CTA-pair (cta_group::2) kernel")
    ap.add_argument("--heads", type=int, default=0,
                    help="override the workload's head count (smaller cases for profiling)")
    ap.add_argument("--ulysses", action="store_true",
                    help="Ulysses sequence parallelism: one batch split over the ranks by "
                         "tokens (strong scaling) instead of one batch per rank")
    ap.add_argument("--head-chunks", type=int, default=0,
                    help="Ulysses: head chunks per rank (default: up to 4)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if args.ulysses:
        run_ulysses(args, rank, world, local_rank)
        return

    import torch
    import torch.distributed as dist
    from diffusion_transformer_video_b200 import dit3d, workloads as wl

    torch.cuda.set_device(local_rank)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))

    def barrier():
        if world > 1:
            dist.barrier()

    dit3d.dit_set_attn_variant(args.attn_variant)
    pk = _peaks()
    w = resolve_workload(args)
    # every rank runs its own batch of the workload (seeded per rank)
    seed = rank_seed(args.seed, rank)
    inp = wl.make_inputs(w, seed, which=("x", "q", "k", "v"))
    host = {k: torch.from_numpy(v.view(np.int16)).view(torch.bfloat16).pin_memory()
            for k, v in inp.items()}
    run = StepRunner(w, seed, args, torch, dit3d, host=host)
    host.update({f"{k}{ps}": v.cpu().pin_memory() for ps, prm in enumerate(run.params)
                 for k, v in prm.items()})
    dev, stream = run.dev, run.stream
    rows, D, H, d = w.rows, w.d_model, w.heads, w.head_dim
    rpg = w.rows_per_group
    cu = run.cu
    o, u = run.o, run.u

    K = args.steps
    t = run.timed(K, args.warmup, barrier, local_rank)
    elapsed_ms = t["elapsed_ms"]
    t_mod, t_rope, t_att, t_res = t["mod"], t["rope"], t["attn"], t["res"]
    clocks = t["clocks"]
    q_rot = run.q_rot

    # the sampler's Euler step (x += dt_frame * u), timed on its own: not part of the step
    frame = w.grid_h * w.grid_w
    dt_dev = torch.from_numpy(
        np.random.default_rng([args.seed, 99]).uniform(0.0, 0.1, rows // frame).astype(np.float32)).cuda()
    x_next = torch.empty_like(dev["x"])
    u_vel = o.view(rows, D)
    for _ in range(3):
        dit3d.dit_flow_euler_step(dev["x"], u_vel, dt_dev, frame, out=x_next)
    ee = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    for a, b in ee:
        a.record(stream)
        dit3d.dit_flow_euler_step(dev["x"], u_vel, dt_dev, frame, out=x_next)
        b.record(stream)
    torch.cuda.synchronize()
    dit3d.dit_check_device()
    t_euler = statistics.mean(a.elapsed_time(b) for a, b in ee)

    # FP8 (E4M3) Q K^T: quantise the rotated q and k (power-of-two scale 1/64, exact
    # products), then attention with the E4M3 product; timed on its own, not in the step
    fp8 = None
    if d == 128 and args.rope_mode == "prepass":
        k_rot = run.k_rot
        q8 = torch.empty(rows, H, d, dtype=torch.uint8, device="cuda")
        k8 = torch.empty_like(q8)
        o8 = torch.empty_like(o)

        def fp8_attention():
            dit3d.dit_quantize_e4m3(q_rot, 64.0, out=q8)
            dit3d.dit_quantize_e4m3(k_rot, 64.0, out=k8)
            dit3d.dit_attn_fwd_qk8(q8, k8, dev["v"], 1 / 64, 1 / 64, n_seq=w.n_seq,
                                   cu_seqlens=cu, out=o8)
        for _ in range(2):
            fp8_attention()
        ev3 = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(max(K, 3))]
        for e in ev3:
            e[0].record(stream)
            dit3d.dit_quantize_e4m3(q_rot, 64.0, out=q8)
            dit3d.dit_quantize_e4m3(k_rot, 64.0, out=k8)
            e[1].record(stream)
            dit3d.dit_attn_fwd_qk8(q8, k8, dev["v"], 1 / 64, 1 / 64, n_seq=w.n_seq,
                                   cu_seqlens=cu, out=o8)
            e[2].record(stream)
        torch.cuda.synchronize()
        dit3d.dit_check_device()
        t_q8 = statistics.mean(e[0].elapsed_time(e[1]) for e in ev3)
        t_a8 = statistics.mean(e[1].elapsed_time(e[2]) for e in ev3)
        # the E4M3 operands straight from the unrotated q, k: RoPE and quantisation in
        # one pass, against the bf16 RoPE pass followed by the two quantisations
        q8f = torch.empty_like(q8)
        k8f = torch.empty_like(k8)

        def rope_e4m3():
            dit3d.dit_rope3d_qk_e4m3(dev["q"], dev["k"], run.desc, 64.0, 64.0, n_seq=w.n_seq,
                                     cu_seqlens=cu, q8_out=q8f, k8_out=k8f)
        for _ in range(3):
            rope_e4m3()
        ev5 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(max(K, 3))]
        for a, b in ev5:
            a.record(stream)
            rope_e4m3()
            b.record(stream)
        torch.cuda.synchronize()
        dit3d.dit_check_device()
        t_rq8 = statistics.mean(a.elapsed_time(b) for a, b in ev5)
        rq8_bytes = 3.0 * rows * H * d * 2  # bf16 q, k read; E4M3 q, k written
        fp8 = {"ms": t_a8, "TFLOP/s": w.attn_flops() / (t_a8 * 1e-3) / 1e12,
               "quantize_ms": t_q8, "max_abs_vs_bf16_attention": float((o8.float() - o.float()).abs().max()),
               "rope_e4m3": {"ms": t_rq8, "GB/s": rq8_bytes / (t_rq8 * 1e-3) / 1e9,
                             "two_pass_ms": t["rope"] + t_q8,
                             "bytes_equal_two_pass": bool(torch.equal(q8f, q8) and torch.equal(k8f, k8)),
                             "kernel": "dit_rope3d_qk_e4m3 (RoPE and E4M3 in one pass)"},
               "in_step": False, "note": "E4M3 q, k (scale 1/64), bf16 P and V"}
        # all of q, k, v (and P) in E4M3
        v8 = dit3d.dit_quantize_e4m3(dev["v"], 64.0)
        for _ in range(2):
            dit3d.dit_attn_fwd_fp8(q8, k8, v8, 1 / 64, 1 / 64, 1 / 64, n_seq=w.n_seq,
                                   cu_seqlens=cu, out=o8)
        ev4 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(max(K, 3))]
        for a, b in ev4:
            a.record(stream)
            dit3d.dit_attn_fwd_fp8(q8, k8, v8, 1 / 64, 1 / 64, 1 / 64, n_seq=w.n_seq,
                                   cu_seqlens=cu, out=o8)
            b.record(stream)
        torch.cuda.synchronize()
        dit3d.dit_check_device()
        t_f8 = statistics.mean(a.elapsed_time(b) for a, b in ev4)
        fp8["all_fp8"] = {"ms": t_f8, "TFLOP/s": w.attn_flops() / (t_f8 * 1e-3) / 1e12,
                          "max_abs_vs_bf16_attention": float((o8.float() - o.float()).abs().max()),
                          "note": "E4M3 q, k, v and P"}

        # the block's step with E4M3 attention operands, timed on its own: modulate ->
        # RoPE with E4M3 output -> attention (E4M3 Q K^T; or all E4M3, v quantised in the
        # step) -> gated residual
        prm0 = run.params[0]
        x_out = torch.empty_like(dev["x"])

        def fp8_step(all8):
            dit3d.dit_adaln_modulate(dev["x"], prm0["gamma"], prm0["beta"], rpg, out=u)
            dit3d.dit_rope3d_qk_e4m3(dev["q"], dev["k"], run.desc, 64.0, 64.0, n_seq=w.n_seq,
                                     cu_seqlens=cu, q8_out=q8f, k8_out=k8f)
            if all8:
                dit3d.dit_quantize_e4m3(dev["v"], 64.0, out=v8)
                dit3d.dit_attn_fwd_fp8(q8f, k8f, v8, 1 / 64, 1 / 64, 1 / 64, n_seq=w.n_seq,
                                       cu_seqlens=cu, out=o8)
            else:
                dit3d.dit_attn_fwd_qk8(q8f, k8f, dev["v"], 1 / 64, 1 / 64, n_seq=w.n_seq,
                                       cu_seqlens=cu, out=o8)
            dit3d.dit_gated_residual(dev["x"], o8.view(rows, D), prm0["alpha"], rpg, out=x_out)

        for all8, key in ((False, "step_qk8"), (True, "step_all_fp8")):
            for _ in range(3):
                fp8_step(all8)
            ev6 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(max(K, 3))]
            for a, b in ev6:
                a.record(stream)
                fp8_step(all8)
                b.record(stream)
            torch.cuda.synchronize()
            dit3d.dit_check_device()
            t_s = statistics.mean(a.elapsed_time(b) for a, b in ev6)
            fp8[key] = {"ms": t_s, "TFLOP/s": w.attn_flops() / (t_s * 1e-3) / 1e12,
                        "calls": "dit_adaln_modulate, dit_rope3d_qk_e4m3, "
                                 + ("dit_quantize_e4m3 (v), dit_attn_fwd_fp8" if all8
                                    else "dit_attn_fwd_qk8") + ", dit_gated_residual"}
        del q8, k8, v8, o8, q8f, k8f, x_out

    # the block's linear layers (projections with the fused adaLN-Zero gate, MLP up with
    # GELU), timed on their own: not part of the step; cuBLAS on the same shapes for context
    lin = {}
    if not args.no_linear:
        gen = torch.Generator(device="cuda").manual_seed(args.seed + 7)
        hidden = 4 * D
        shapes = {"linear_qkv": (3 * D, D, False, False), "linear_out_gated": (D, D, False, True),
                  "linear_mlp_up_gelu": (hidden, D, True, False),
                  "linear_mlp_down_gated": (D, hidden, False, True)}
        h_act = None
        alpha_g = (torch.randn(rows // rpg, D, device="cuda", generator=gen) * 0.1).to(torch.bfloat16)
        for name, (n_out, k_in, gelu, gated) in shapes.items():
            wt = (torch.randn(n_out, k_in, device="cuda", generator=gen) * k_in ** -0.5).to(torch.bfloat16)
            xin = u if k_in == D else h_act
            y = torch.empty(rows, n_out, dtype=torch.bfloat16, device="cuda")
            kw = dict(gelu=gelu, out=y)
            if gated:
                kw.update(residual=dev["x"], alpha=alpha_g, rows_per_group=rpg, out=x_next)
            run_lin = lambda: dit3d.dit_linear(xin, wt, **kw)
            run_cublas = lambda: torch.matmul(xin, wt.t())  # same product, no epilogue
            for _ in range(2):
                run_lin()
                run_cublas()

            def per_call(fn):
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                for _ in range(5):
                    fn()
                b.record(stream)
                torch.cuda.synchronize()
                return a.elapsed_time(b) / 5

            # ours and cuBLAS interleaved over three rounds (clocks drift under the power
            # cap), median per call of each
            t_ours, t_cublas = [], []
            for _ in range(3):
                t_ours.append(per_call(run_lin))
                t_cublas.append(per_call(run_cublas))
            dit3d.dit_check_device()
            ms, ms_cublas = statistics.median(t_ours), statistics.median(t_cublas)
            fl = 2.0 * rows * n_out * k_in
            lin[name] = {"ms": ms, "TFLOP/s": fl / (ms * 1e-3) / 1e12, "shape": [rows, n_out, k_in],
                         "frac_burst": fl / (ms * 1e-3) / 1e12 / pk["bf16_tflops"],
                         "cublas_ms": ms_cublas, "timing": "median of 3 rounds of 5 calls, "
                         "interleaved with cuBLAS", "in_step": False}
            if name == "linear_qkv":
                # the same projection on E4M3 activations and weights (scales 1/16, 1/256)
                x8 = dit3d.dit_quantize_e4m3(xin, 16.0)
                w8 = dit3d.dit_quantize_e4m3(wt, 256.0)
                run8 = lambda: dit3d.dit_linear_fp8(x8, w8, 1 / 16, 1 / 256, out=y)
                for _ in range(2):
                    run8()
                q0, q1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                q0.record(stream)
                for _ in range(5):
                    run8()
                q1.record(stream)
                torch.cuda.synchronize()
                dit3d.dit_check_device()
                ms8 = q0.elapsed_time(q1) / 5
                lin["linear_qkv_fp8"] = {"ms": ms8, "TFLOP/s": fl / (ms8 * 1e-3) / 1e12,
                                         "shape": [rows, n_out, k_in], "in_step": False,
                                         "note": "E4M3 x and w, fp32 accumulation, bf16 out"}
                del x8, w8
            if name == "linear_mlp_up_gelu":
                h_act = y  # the MLP's hidden activations feed the down projection
            del wt, y

    # end to end: every step copies its inputs (x, q, k, v and the step's adaLN
    # parameters) from pinned host memory and its result back, through the same calls.
    # Two device buffer sets and one upload and one download stream pipeline the steps:
    # step i+1's inputs upload and step i-1's result downloads while step i computes (a
    # set is reused only after the step that read it has finished, an output buffer only
    # after its download).
    data_keys = ("x", "q", "k", "v")
    prm_keys = ("gamma", "beta", "alpha")
    sets = [dict({k: torch.empty_like(dev[k]) for k in data_keys},
                 params=[{k: torch.empty_like(run.params[0][k]) for k in prm_keys}] * 1)
            for _ in range(2)]
    outs = [torch.empty(rows, D, dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    res_host = [torch.empty(rows, D, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    h2d = (sum(host[k].numel() * 2 for k in data_keys)
           + sum(run.params[0][k].numel() * 2 for k in prm_keys))
    d2h = res_host[0].numel() * 2
    up_stream, down_stream = torch.cuda.Stream(), torch.cuda.Stream()
    loaded = [torch.cuda.Event() for _ in range(2)]
    computed = [torch.cuda.Event() for _ in range(2)]
    drained = [torch.cuda.Event() for _ in range(2)]
    n_e2e = max(args.e2e_steps, 1)

    def upload(i):
        bset = i % 2
        with torch.cuda.stream(up_stream):
            if i >= 2:
                up_stream.wait_event(computed[bset])     # step i-2 has read this set
            for k in data_keys:
                sets[bset][k].copy_(host[k], non_blocking=True)
            ps = i % w.param_sets                        # this step's parameter set
            for k in prm_keys:
                sets[bset]["params"][0][k].copy_(host[f"{k}{ps}"], non_blocking=True)
            loaded[bset].record(up_stream)

    barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    up_stream.wait_event(e0)
    upload(0)
    for i in range(n_e2e):
        bset = i % 2
        if i + 1 < n_e2e:
            upload(i + 1)
        stream.wait_event(loaded[bset])
        if i >= 2:
            stream.wait_event(drained[bset])             # step i-2's result has left outs[bset]
        run.step(sets[bset], i=0, out_t=outs[bset])
        computed[bset].record(stream)
        with torch.cuda.stream(down_stream):
            down_stream.wait_event(computed[bset])
            res_host[bset].copy_(outs[bset], non_blocking=True)
            drained[bset].record(down_stream)
    stream.wait_stream(up_stream)
    stream.wait_stream(down_stream)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / n_e2e
    # the last downloaded result must be the device step's result (same inputs, same set)
    run.step(i=n_e2e - 1)
    torch.cuda.synchronize()
    e2e_same = bool(torch.equal(res_host[(n_e2e - 1) % 2].cuda(), run.out))
    del sets, outs

    flops = w.attn_flops()
    ms_step = elapsed_ms / K
    ms_step, e2e_ms = max_over_ranks([ms_step, e2e_ms], dist if world > 1 else None, "cuda")
    value = job_throughput(flops, world, ms_step)
    e2e_value = job_throughput(flops, world, e2e_ms)

    att_tflops = flops / (t_att * 1e-3) / 1e12
    per_head = ATTN_DRAM_BYTES_PER_HEAD_480P.get(args.rope_mode) if w.name == "480p" else None
    traffic = per_head * H if per_head is not None and args.attn_variant == 0 else None
    t["step_ms"] = elapsed_ms / K
    head_fig = workload_figures(w, t, pk, args.rope_mode)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        qkv64 = widen_qkv(inp)
        tf, dt, sample, threads = cpu_oracle_attention(w, qkv64, args.cpu_rows, args.seed)
        cpu = {"value": tf, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample,
               "seconds": dt}
        tf1, dt1, sample1 = cpu_oracle_attention_one_thread(w, qkv64, max(4, args.cpu_rows // 8),
                                                            args.seed)
        del qkv64
        cpu["one_thread"] = {"value": tf1, "unit": UNIT, "cores": 1, "seconds": dt1,
                             "sample": sample1}
        cpu["memory_steps"] = cpu_oracle_memory_steps(w, inp["x"], args.seed)
        # the step's attention output on the same sampled rows, against the oracle
        run.step(i=0)
        s_rows, ref_o = cpu_oracle_attention.last
        got = o[torch.from_numpy(s_rows).cuda()].float().cpu().double().numpy()
        err = np.abs(got - ref_o)
        cpu["parity"] = {"rows": int(len(s_rows)), "max_abs": float(err.max()),
                         "mean_abs": float(err.mean()), "tolerance_max_mean": [2e-2, 2e-3]}
    del inp
    run.free()
    del run, dev, o, u, x_next, u_vel, q_rot, host
    torch.cuda.empty_cache()

    # the other workloads, each on its own seeded inputs, timed the same way (fewer steps)
    workloads = {w.name: dict(head_fig, headline=True)}
    if not args.no_workloads and not args.heads:
        for name in wl.WORKLOADS:
            if name == w.name:
                continue
            ww = wl.get_workload(name, args.seed)
            r2 = StepRunner(ww, seed, args, torch, dit3d)
            t2 = r2.timed(max(args.workload_steps, 1), args.warmup, barrier, local_rank)
            t2["step_ms"] = t2["elapsed_ms"] / max(args.workload_steps, 1)
            workloads[name] = workload_figures(ww, t2, pk, args.rope_mode)
            workloads[name]["steps"] = max(args.workload_steps, 1)
            r2.free()
            del r2

    if rank == 0:
        launches_per_step = 4 if args.rope_mode == "prepass" else 3
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded bf16 N(0,1) x/q/k/v, N(0,0.1) adaLN params)",
            "config": workload_config(w, world),
            "gpu_launches": launches_per_step * K,
            "roofline": {"bound": "tensor", "achieved": att_tflops,
                         "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": att_tflops / pk["bf16_tflops"],
                         "frac_sustained": att_tflops / pk["bf16_tflops_sustained"],
                         "traffic": traffic,
                         "kernel": {"prepass": "dit_attn_fwd (operands rotated by dit_rope3d_qk)",
                                    "fused": "dit_attn_fwd (fused 3D-RoPE)",
                                    "none": "dit_attn_fwd without RoPE"}[args.rope_mode],
                         "attn_variant": ["single CTA", "CTA pair (cta_group::2)"][args.attn_variant],
                         "peak_source": f"{pk['source']} burst bf16 {pk['bf16_tflops']} TFLOP/s "
                                        f"(sustained {pk['bf16_tflops_sustained']}: frac_sustained)"},
            "components": {
                "adaln_modulate": head_fig["adaln_modulate"],
                "rope3d_qk": head_fig["rope3d_qk"],
                "attn_fwd": head_fig["attn_fwd"],
                "gated_residual": head_fig["gated_residual"],
                "flow_euler_step": {"ms": t_euler, "GB/s": 6.0 * rows * D / (t_euler * 1e-3) / 1e9,
                                    "frac_hbm": 6.0 * rows * D / (t_euler * 1e-3) / 1e9 / pk["hbm_gbs"],
                                    "bytes": 6.0 * rows * D, "in_step": False,
                                    "note": "sampler update x += dt_frame * u, timed separately"},
                "attn_fwd_qk8": fp8,
                **lin,
            },
            "workloads": workloads,
            "clocks": clocks,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "pipelined": "2 buffer sets; uploads and downloads overlap neighbouring steps",
                    "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                    "result_matches_device_step": e2e_same},
            "cpu_baseline": cpu,
            "peaks": {k: pk[k] for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained", "source")},
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
