#!/usr/bin/env python3
"""Throughput of the S^2-Attn hot path on B200: useful causal-within-group TFLOP/s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one pass of the whole hot path over one batch of the synthetic
LLaMA2-7B layer at N=32768 (B=1, H=32 with 16 shifted heads, D=128, G=8192):
rope_pi_apply(q, k) -> s2attn_fwd -> s2attn_bwd (preprocess, main, dQ convert).
Useful FLOPs per step = 3.5 * 4 * D * (causal in-group pairs) (forward 4*D per pair,
backward 2.5x the forward).  Inputs are resident in HBM and larger than L2.

Multi-GPU (torchrun, one process per GPU): the path does not shard across GPUs
here, so every rank runs an independent replica of the workload; value counts the
work of all ranks over the slowest rank's time ("scaling": "weak").

--impl reference times the fp64 CPU oracle (the method's plain definition) on a
bounded sample of the same workload, on this machine's host cores, rank 0 only.

--mode sequence splits the workload's sequence across the ranks (whole groups per rank,
the shifted heads' G/2 halo exchanged); --mode lora times the layer's LoRA-adapted
projections (q/k/v with fused RoPE-PI, and o) alone.  The default run also reports the
projections, the decoding step and full causal attention, outside the timed region.
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from shifted_sparse_attention_s2attn_b200.synthetic import WORKLOADS, make_tensor  # noqa: E402

METRIC = "S²-Attn fwd+bwd useful TFLOP/s at LLaMA2-7B shape N=32k (% of bf16 peak)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
LAUNCHES_PER_STEP = 5  # rope, fwd, bwd preprocess, bwd main, dQ convert


def useful_pairs(w):
    return w.B * w.H * (w.N // w.G) * w.G * (w.G + 1) // 2


def step_flops(w):
    return 3.5 * 4 * w.D * useful_pairs(w)


def max_over_ranks(ms, device=None):
    """Slowest rank's time: every rank contributes its own CUDA-event time (replicas)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(flops_per_step, steps, world, ms_max):
    """Work of all ranks (world replicas x steps x FLOPs per step) over the slowest rank's time."""
    return world * flops_per_step * steps / (ms_max / 1e3) / 1e12


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


# ---------------------------------------------------------------------------------
# clocks sampled during the timed region
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_indices):
        self.gpus = set(gpu_indices)
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in out.splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                idx = int(parts[0])
            except ValueError:
                continue
            if idx not in self.gpus:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                pass
            for name, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------------
# the oracle on a bounded sample (CPU baseline and the reference arm)
def oracle_sample_flops(w, R):
    """Useful FLOPs of the oracle sample: the last R query rows and the last R key rows of
    one group, i.e. forward + dQ for every pair whose query is among the R rows
    (10*D FLOPs per pair) and dK + dV for the pairs inside the R x R triangle (4*D)."""
    G, D = w.G, w.D
    q_pairs = sum(range(G - R + 1, G + 1))
    return 10 * D * q_pairs + 4 * D * R * (R + 1) // 2


def run_oracle_sample(w, inputs, R, unit):
    import oracle
    b, h, j = unit
    rows = list(range(w.G - R, w.G))
    t0 = time.perf_counter()
    oracle.s2attn_unit(inputs["q"], inputs["k"], inputs["v"], w.G, w.shift_heads, b, h, j, qrows=rows, krows=rows,
                       dout=inputs["dout"])
    return time.perf_counter() - t0


def oracle_inputs(w):
    import oracle
    inp = {n: make_tensor(w, n) for n in ("q", "k", "v", "dout")}
    inp["q"] = oracle.rope_pi_bf16(inp["q"], w.pos_scale, w.base)
    inp["k"] = oracle.rope_pi_bf16(inp["k"], w.pos_scale, w.base)
    return inp


def cpu_baseline(w, min_seconds=10.0, max_units=16):
    """Whole groups (fwd+bwd, every row) of the shifted heads' wrap-around group, until >= min_seconds."""
    inp = oracle_inputs(w)
    units = [(0, h, w.groups - 1) for h in range(w.H - 1, -1, -1)]
    elapsed, flops, n = 0.0, 0.0, 0
    while n < max_units and (elapsed < min_seconds or n == 0):
        elapsed += run_oracle_sample(w, inp, w.G, units[n % len(units)])
        flops += oracle_sample_flops(w, w.G)
        n += 1
    return {"value": flops / elapsed / 1e12, "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle",
            "sample": f"{n} whole group(s) (G={w.G}, all rows, fwd+bwd) of the {w.name} workload, heads from "
                      f"H-1 down, last group; fp64 C oracle with OpenMP; {elapsed:.1f} s"}


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    inp = oracle_inputs(w)
    unit = (0, w.H - 1, w.groups - 1)
    # size the per-step sample so that warmup + steps take about two minutes
    R = 256
    t = run_oracle_sample(w, inp, R, unit)
    budget = 120.0 / max(1, args.steps + args.warmup)
    while R < w.G and t < budget / 3:
        R = min(w.G, R * 2)
        t = run_oracle_sample(w, inp, R, unit)
    for _ in range(args.warmup):
        run_oracle_sample(w, inp, R, unit)
    total = 0.0
    for _ in range(args.steps):
        total += run_oracle_sample(w, inp, R, unit)
    value = oracle_sample_flops(w, R) * args.steps / total / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle",
                         "sample": f"per step: the last {R} query rows and {R} key rows (fwd+bwd) of group "
                                   f"{unit[2]} of head {unit[1]} (shifted, wraps around the sequence end)"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(w):
    return {"workload": w.name, "B": w.B, "N": w.N, "H": w.H, "D": w.D, "G": w.G, "shift_heads": w.shift_heads,
            "rope_pos_scale": w.pos_scale, "step": "rope_pi_apply + s2attn_fwd + s2attn_bwd",
            "l2": "inputs larger than L2 (q,k,v,dO = %.2f GB)" % (4 * w.B * w.N * w.H * w.D * 2 / 1e9),
            "parallelism": "replicas"}


def traffic_record(kernel_file, kernel):
    """DRAM bytes per launch from a committed ncu summary, if the kernel source is unchanged."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        recs = json.load(f)
    src = os.path.join(ROOT, "shifted_sparse_attention_s2attn_b200", "csrc", kernel_file)
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()
    rec = recs.get(kernel)
    if not rec or rec.get("source_sha256") != sha:
        return None
    return rec.get("dram_bytes_per_launch")


# ---------------------------------------------------------------------------------
def time_workload(w, dev, stream, reps=5, warmup=3):
    """fwd and fwd+bwd of one workload's step (RoPE-PI, forward, backward), timed with CUDA
    events on `stream` over `reps` steps after `warmup`.  The inputs are drawn on the device
    (a seeded torch generator, N(0,1) in bf16; the K outlier rows of the 100k workload are
    scaled x8 at the recipe's rows): the timing does not depend on the values, and drawing
    GBs on the host would dominate the run.  Every workload's inputs are larger than L2."""
    import torch

    import shifted_sparse_attention_s2attn_b200 as s2
    from shifted_sparse_attention_s2attn_b200.synthetic import outlier_rows

    B, N, H, D, G, SH = w.B, w.N, w.H, w.D, w.G, w.shift_heads
    gen = torch.Generator(device=dev)
    gen.manual_seed(1000 * w.index)
    t = {n: torch.randn((B, N, H, D), generator=gen, device=dev).to(torch.bfloat16) for n in ("q", "k", "v", "dout")}
    if w.k_outlier_frac > 0:
        for b, rows in enumerate(outlier_rows(w)):
            flat = t["k"][b].view(N * H, D)
            idx = torch.from_numpy(rows).to(dev)
            flat[idx] = flat[idx] * 8
    o, dq, dk, dv = (torch.empty_like(t["q"]) for _ in range(4))
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    ws = torch.empty(s2.s2attn_bwd_workspace_bytes(B, N, H, D), dtype=torch.uint8, device=dev)
    dq_acc = ws[: B * N * H * D * 4].view(torch.float32)
    delta_off = ((B * N * H * D * 4 + 255) // 256) * 256
    delta = ws[delta_off: delta_off + B * H * N * 4].view(torch.float32)
    s2.rope_pi_apply(t["q"], t["k"], w.pos_scale, w.base, stream)

    def one(ev=None):
        if ev is not None:
            ev[0].record(stream)
        s2.s2attn_fwd(t["q"], t["k"], t["v"], o, lse, G, SH, stream)
        if ev is not None:
            ev[1].record(stream)
        s2.s2attn_bwd_preprocess(o, t["dout"], delta, dq_acc, stream)
        s2.s2attn_bwd_main(t["q"], t["k"], t["v"], t["dout"], lse, delta, dq_acc, dk, dv, G, SH, stream)
        s2.s2attn_bwd_dq_convert(dq_acc, dq, stream)
        if ev is not None:
            ev[2].record(stream)

    for _ in range(warmup):
        one()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(reps)]
    for i in range(reps):
        one(evs[i])
    torch.cuda.synchronize(dev)
    fwd_ms = statistics.median(e[0].elapsed_time(e[1]) for e in evs)
    step_ms = statistics.median(e[0].elapsed_time(e[2]) for e in evs)
    peaks, peak_src = load_peaks()
    peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    pairs = useful_pairs(w)
    fwd_tf = 4 * D * pairs / (fwd_ms / 1e3) / 1e12
    step_tf = 14 * D * pairs / (step_ms / 1e3) / 1e12
    del t, o, dq, dk, dv, lse, ws
    return {"B": B, "N": N, "H": H, "G": G, "shift_heads": SH, "fwd_ms": fwd_ms, "fwd_tflops": fwd_tf,
            "fwd_frac": fwd_tf / peak, "fwd_bwd_ms": step_ms, "fwd_bwd_tflops": step_tf, "fwd_bwd_frac": step_tf / peak,
            "peak": peak, "peak_source": f"{peak_src} bf16_tflops (burst)", "reps": reps,
            "timing": "median of the per-step CUDA-event times; fwd+bwd = s2attn_fwd + s2attn_bwd (3 launches)"}


def run_ours(args, w):
    import torch
    import torch.distributed as dist

    import shifted_sparse_attention_s2attn_b200 as s2

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=180), device_id=dev)

    B, N, H, D, G, SH = w.B, w.N, w.H, w.D, w.G, w.shift_heads

    def to_dev(bits):
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(dev)

    host = {n: make_tensor(w, n) for n in ("q", "k", "v", "dout")}

    def buffer_set(inputs=None):
        """Device tensors of one step: inputs (q, k, v, dout), outputs (o, dq, dk, dv), lse and
        the backward workspace (fp32 dQ accumulator, delta)."""
        bs = dict(inputs) if inputs else {n: torch.empty((B, N, H, D), dtype=torch.bfloat16, device=dev)
                                          for n in ("q", "k", "v", "dout")}
        for n in ("o", "dq", "dk", "dv"):
            bs[n] = torch.empty((B, N, H, D), dtype=torch.bfloat16, device=dev)
        bs["lse"] = torch.empty((B, H, N), dtype=torch.float32, device=dev)
        ws = torch.empty(s2.s2attn_bwd_workspace_bytes(B, N, H, D), dtype=torch.uint8, device=dev)
        bs["dq_acc"] = ws[: B * N * H * D * 4].view(torch.float32)
        delta_off = ((B * N * H * D * 4 + 255) // 256) * 256
        bs["delta"] = ws[delta_off: delta_off + B * H * N * 4].view(torch.float32)
        return bs

    main_set = buffer_set({n: to_dev(host[n]) for n in ("q", "k", "v", "dout")})
    q, k, v = main_set["q"], main_set["k"], main_set["v"]
    stream = torch.cuda.current_stream(dev)

    def step(ev=None, bs=main_set, st=stream):
        s2.rope_pi_apply(bs["q"], bs["k"], w.pos_scale, w.base, st)
        if ev is not None:
            ev[0].record(st)
        s2.s2attn_fwd(bs["q"], bs["k"], bs["v"], bs["o"], bs["lse"], G, SH, st)
        if ev is not None:
            ev[1].record(st)
        s2.s2attn_bwd_preprocess(bs["o"], bs["dout"], bs["delta"], bs["dq_acc"], st)
        if ev is not None:
            ev[2].record(st)
        s2.s2attn_bwd_main(bs["q"], bs["k"], bs["v"], bs["dout"], bs["lse"], bs["delta"], bs["dq_acc"], bs["dk"],
                           bs["dv"], G, SH, st)
        if ev is not None:
            ev[3].record(st)
        s2.s2attn_bwd_dq_convert(bs["dq_acc"], bs["dq"], st)

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local])

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    s2.clear_device_error()

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(range(world)) if rank == 0 else None
    barrier()
    torch.cuda.synchronize(dev)
    if sampler:
        sampler.start()
        time.sleep(0.3)
    start.record(stream)
    for i in range(args.steps):
        step(evs[i])
    end.record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop() if sampler else None
    barrier()
    ms = start.elapsed_time(end)
    fwd_ms = [e[0].elapsed_time(e[1]) for e in evs]
    bwd_ms = [e[2].elapsed_time(e[3]) for e in evs]
    rc, detail = s2.get_device_error()
    if rc != 0:
        raise SystemExit(f"device error word set during the timed region: {detail:#x}")

    ms_max = max_over_ranks(ms, dev)
    if args.step_only:
        # profiling runs: the timed step loop and nothing after it
        if world > 1:
            dist.destroy_process_group()
        if rank == 0:
            print(json.dumps({"metric": METRIC, "value": whole_job_tflops(step_flops(w), args.steps, world, ms_max),
                              "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                              "ms_per_step": ms_max / args.steps, "step_only": True,
                              "config": workload_config(w)}), flush=True)
        return 0

    # ---- full causal attention (inference case: one group, no shift), forward only ----
    pairs_full = B * H * N * (N + 1) // 2
    fc_lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    fc_o = torch.empty_like(q)
    for _ in range(2):
        s2.s2attn_fwd(q, k, v, fc_o, fc_lse, N, 0, stream)
    fc0, fc1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    fc_reps = 5
    fc0.record(stream)
    for _ in range(fc_reps):
        s2.s2attn_fwd(q, k, v, fc_o, fc_lse, N, 0, stream)
    fc1.record(stream)
    torch.cuda.synchronize(dev)
    fc_ms = fc0.elapsed_time(fc1) / fc_reps
    del fc_o, fc_lse

    # ---- decoding step (inference, full causal attention of the last M positions) ----
    # The queries are the last M rows of q; K and V (0.54 GB, larger than L2) are read
    # once per call, which makes the step HBM-bound.
    decode = {}
    for M in (1, 16, 128):
        dq_ = q[:, N - M:].contiguous()
        d_o = torch.empty_like(dq_)
        d_lse = torch.empty((B, H, M), dtype=torch.float32, device=dev)
        d_ws = torch.empty(s2.s2attn_decode_workspace_bytes(B, M, N, H, D), dtype=torch.uint8, device=dev)
        for _ in range(3):
            s2.s2attn_decode(dq_, k, v, d_o, d_lse, d_ws, stream)
        d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        d_reps = 20
        d0.record(stream)
        for _ in range(d_reps):
            s2.s2attn_decode(dq_, k, v, d_o, d_lse, d_ws, stream)
        d1.record(stream)
        torch.cuda.synchronize(dev)
        d_ms = d0.elapsed_time(d1) / d_reps
        kv_bytes = 2 * B * N * H * D * 2
        decode[f"M{M}"] = {"ms": d_ms, "kv_bytes": kv_bytes, "gbs": kv_bytes / (d_ms / 1e3) / 1e9,
                           "tokens_per_s": B * M / (d_ms / 1e3)}
        del dq_, d_o, d_lse, d_ws

    # ---- the other LLaMA2 workloads: fwd and fwd+bwd of the same step, outside the timed region ----
    per_workload = {}
    for wname in ("llama2_7b_8k", "llama2_13b_64k", "llama2_7b_100k"):
        per_workload[wname] = time_workload(WORKLOADS[wname], dev, stream, reps=5)
    rc, detail = s2.get_device_error()
    if rc != 0:
        raise SystemExit(f"device error word set during the per-workload runs: {detail:#x}")

    # ---- LoRA-adapted projections on either side of the attention (LLaMA2-7B layer) ----
    # q, k, v stacked (3 x 4096 outputs, rank 8, scaling 2, RoPE-PI fused on q and k) and o
    # (4096 outputs, rank 8) over the B*N tokens; the plain q, k, v projection (no adapter,
    # no RoPE) is timed too, to show what the adapter and the rotation add.
    lora = {}
    T_l, K_l, n_l, r_l = B * N, H * D, H * D, 8
    gen = torch.Generator(device=dev)
    gen.manual_seed(20)
    lx = torch.randn((T_l, K_l), generator=gen, device=dev).to(torch.bfloat16)
    for name, parts, r_, rope_parts in (("qkv_lora_rope", 3, r_l, 2), ("qkv_plain", 3, 0, 0), ("o_lora", 1, r_l, 0)):
        lw = (torch.randn((parts * n_l, K_l), generator=gen, device=dev) / K_l ** 0.5).to(torch.bfloat16)
        la = (torch.randn((parts * r_, K_l), generator=gen, device=dev) / K_l ** 0.5).to(torch.bfloat16) if r_ else None
        lb = (0.05 * torch.randn((parts * n_l, r_), generator=gen, device=dev)).to(torch.bfloat16) if r_ else None
        ly = torch.empty((parts, T_l, n_l), dtype=torch.bfloat16, device=dev)
        lws = torch.empty(max(256, s2.lora_proj_workspace_bytes(T_l, K_l, n_l, parts, r_)), dtype=torch.uint8,
                          device=dev)
        call = lambda: s2.lora_proj_fwd(lx, lw, la, lb, ly, parts, 2.0, rope_parts=rope_parts, head_dim=D,  # noqa: E731
                                        seq_len=N, pos_scale=w.pos_scale, workspace=lws, stream=stream)
        for _ in range(3):
            call()
        l0, l1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        l_reps = 10
        l0.record(stream)
        for _ in range(l_reps):
            call()
        l1.record(stream)
        torch.cuda.synchronize(dev)
        l_ms = l0.elapsed_time(l1) / l_reps
        flops = 2 * T_l * K_l * parts * n_l + 2 * T_l * K_l * parts * r_ + 2 * T_l * r_ * parts * n_l
        lora[name] = {"ms": l_ms, "parts": parts, "r": r_, "rope_parts": rope_parts, "flops": flops,
                      "tflops": flops / (l_ms / 1e3) / 1e12}
        del lw, la, lb, ly, lws
    del lx
    rc, detail = s2.get_device_error()
    if rc != 0:
        raise SystemExit(f"device error word set during the projection runs: {detail:#x}")

    # ---- end to end: host buffers in, results out, through the same public calls ----
    # Each step copies its inputs from pinned host memory and its results back.  Steps are
    # pipelined over three streams with two device buffer sets: the host->device copy of
    # step i+1 and the device->host copy of step i-1 overlap the compute of step i.
    e2e_steps = max(3, min(args.steps, 200))  # the device-timed loop's step count (~22 ms each, PCIe-bound)
    pinned = {n: torch.from_numpy(host[n].view(np.int16)).view(torch.bfloat16).pin_memory() for n in host}
    sets = [main_set, buffer_set()]
    outs = [{n: torch.empty((B, N, H, D), dtype=torch.bfloat16).pin_memory() for n in ("o", "dq", "dk", "dv")}
            for _ in sets]
    h2d = sum(x.numel() * x.element_size() for x in pinned.values())
    d2h = sum(x.numel() * x.element_size() for x in outs[0].values())
    s_h2d, s_d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def e2e_run(nsteps, e_start=None, e_end=None):
        ev = lambda: torch.cuda.Event()  # noqa: E731
        h2d_done, cmp_done, d2h_done = [None, None], [None, None], [None, None]
        if e_start is not None:
            e_start.record(stream)
            s_h2d.wait_event(e_start)
            s_d2h.wait_event(e_start)
        for i in range(nsteps):
            slot = i % 2
            bs = sets[slot]
            with torch.cuda.stream(s_h2d):  # inputs of step i, once step i-2 stopped reading them
                if cmp_done[slot] is not None:
                    s_h2d.wait_event(cmp_done[slot])
                for n in pinned:
                    bs[n].copy_(pinned[n], non_blocking=True)
                h2d_done[slot] = ev()
                h2d_done[slot].record(s_h2d)
            stream.wait_event(h2d_done[slot])
            if d2h_done[slot] is not None:  # outputs of step i-2 copied out
                stream.wait_event(d2h_done[slot])
            step(bs=bs, st=stream)
            cmp_done[slot] = ev()
            cmp_done[slot].record(stream)
            with torch.cuda.stream(s_d2h):
                s_d2h.wait_event(cmp_done[slot])
                for n in outs[slot]:
                    outs[slot][n].copy_(bs[n], non_blocking=True)
                d2h_done[slot] = ev()
                d2h_done[slot].record(s_d2h)
        if e_end is not None:
            for e in h2d_done + d2h_done:
                if e is not None:
                    stream.wait_event(e)
            e_end.record(stream)

    e2e_run(2)
    torch.cuda.synchronize(dev)
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_run(e2e_steps, e0, e1)
    torch.cuda.synchronize(dev)
    barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dev)
    rc, detail = s2.get_device_error()
    if rc != 0:
        raise SystemExit(f"device error word set during the end-to-end run: {detail:#x}")
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return 0

    flops = step_flops(w)
    value = whole_job_tflops(flops, args.steps, world, ms_max)
    peaks, peak_src = load_peaks()
    fwd_flops, bwd_flops = 4 * D * useful_pairs(w), 10 * D * useful_pairs(w)
    bwd_avg = statistics.mean(bwd_ms) / 1e3
    fwd_avg = statistics.mean(fwd_ms) / 1e3
    # The timed region is short (0.2 s at 20 steps, about 1 s at 100), so the denominator is the
    # measured burst bf16 peak (cuBLAS at full clocks), not the sustained one of a seconds-long
    # power-capped loop; when the clocks record shows the cap lowering the SM clock, the burst peak
    # is the stricter of the two.
    peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    achieved = bwd_flops / bwd_avg / 1e12
    traffic = traffic_record("s2attn_bwd_sm100.cu", "s2attn_bwd_kernel")
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": workload_config(w),
        "pct_of_peak": 100.0 * value / world / peak,
        "peak_used": {"bf16_tflops": peak, "source": peak_src,
                      "why": ("burst: the timed region lasts a second or less; under sw_power_cap (see clocks) "
                              "the burst peak is the stricter denominator")},
        "fwd": {"ms": 1e3 * fwd_avg, "tflops": fwd_flops / fwd_avg / 1e12},
        "bwd_main": {"ms": 1e3 * bwd_avg, "tflops": achieved},
        "roofline": {"kernel": "s2attn_bwd_kernel", "bound": "tensor", "achieved": achieved, "peak": peak,
                     "unit": "TFLOP/s", "frac": achieved / peak, "traffic": traffic,
                     "peak_source": f"{peak_src} bf16_tflops (burst; the timed region is short)"},
        "roofline_fwd": {"kernel": "s2attn_fwd_kernel", "bound": "tensor",
                         "achieved": fwd_flops / fwd_avg / 1e12, "peak": peak, "unit": "TFLOP/s",
                         "frac": fwd_flops / fwd_avg / 1e12 / peak,
                         "traffic": traffic_record("s2attn_fwd_sm100.cu", "s2attn_fwd_kernel")},
        "e2e": {"value": whole_job_tflops(flops, e2e_steps, world, e2e_ms), "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "overlap": ("H2D of step i+1 and D2H of step i-1 run on their own streams during step i; the "
                            "timed region also holds the first step's H2D and the last step's D2H, which "
                            "overlap nothing")},
        "per_workload": per_workload,
        "full_causal_fwd": {"workload": f"{w.name} with G=N={N}, shift_heads=0 (inference: full causal attention)",
                            "ms": fc_ms, "tflops": 4 * D * pairs_full / (fc_ms / 1e3) / 1e12},
        "decode": {"workload": f"{w.name}: the last M rows of q as decoding queries (query m at position "
                               f"N-M+m) against all N={N} positions of k, v; full causal attention",
                   "bound": "hbm", "peak_gbs": peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]),
                   **{k_: dict(v_, frac=v_["gbs"] / peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
                      for k_, v_ in decode.items()}},
        "lora_proj": {"workload": f"LLaMA2-7B layer projections over T=B*N={B * N} tokens, K={H * D}: q,k,v "
                                  f"stacked (3x{H * D} outputs) and o ({H * D}); LoRA rank 8, scaling 2; RoPE-PI "
                                  f"(pos_scale {w.pos_scale}) fused on q and k; flops = 2*T*K*outputs + adapter",
                      "bound": "tensor", "peak": peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]),
                      "peak_source": f"{peak_src} bf16_tflops (burst: each call timed alone, 10 calls)",
                      **{k_: dict(v_, frac=v_["tflops"] / peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
                         for k_, v_ in lora.items()}},
        "gpu_launches": LAUNCHES_PER_STEP * args.steps,
        "clocks": clocks,
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w)
    print(json.dumps(line), flush=True)
    return 0


def run_sequence_sharded(args, w):
    """--mode sequence: one sequence split across the ranks (whole groups per rank, the
    shifted heads' G/2 halo exchanged between neighbours).  A step = RoPE-PI of the rank's
    rows at their positions + sharded forward + sharded backward; the total work is fixed,
    so "scaling" is "strong".  With one GPU the halo is the rank's own first rows, and the
    number measures the cost of the local layout against the direct path."""
    import torch
    import torch.distributed as dist

    import shifted_sparse_attention_s2attn_b200 as s2
    from shifted_sparse_attention_s2attn_b200.sharded import shard_range, sharded_bwd, sharded_fwd

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=180), device_id=dev)
    t0, t1 = shard_range(w.N, w.G, world, rank)
    host = {n: make_tensor(w, n)[:, t0:t1] for n in ("q", "k", "v", "dout")}
    dv_ = {n: torch.from_numpy(np.ascontiguousarray(host[n]).view(np.int16)).view(torch.bfloat16).to(dev)
           for n in host}
    q, k = dv_["q"], dv_["k"]
    stream = torch.cuda.current_stream(dev)

    def step():
        # in place every step, as in the replicas mode (the timing does not depend on the values)
        s2.rope_pi_apply_offset(q, k, t0, w.pos_scale, w.base, stream)
        o, lse = sharded_fwd(q, k, dv_["v"], w.G, w.shift_heads)
        return sharded_bwd(q, k, dv_["v"], o, dv_["dout"], lse, w.G, w.shift_heads)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    s2.clear_device_error()
    if world > 1:
        dist.barrier(device_ids=[local])
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier(device_ids=[local])
    rc, detail = s2.get_device_error()
    if rc != 0:
        raise SystemExit(f"device error word set during the timed region: {detail:#x}")
    ms_max = max_over_ranks(e0.elapsed_time(e1), dev)
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return 0
    value = step_flops(w) * args.steps / (ms_max / 1e3) / 1e12   # the whole sequence's work, all ranks
    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
            "scaling": "strong", "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "mode": "sequence",
            "config": dict(workload_config(w), parallelism=f"sequence x{world}",
                           step="rope_pi_apply_offset + sharded fwd + sharded bwd (G/2 halo of the shifted heads)")}
    print(json.dumps(line), flush=True)
    return 0


def run_lora_projections(args, w):
    """--mode lora: the LoRA-adapted projections of the workload's layer alone (one GPU; with
    several ranks each runs the same calls and rank 0 reports), so that a profiler can capture
    exactly these launches.  Five calls of lora_proj_fwd over T = B*N tokens, K = H*D: q, k, v
    stacked with a rank-8 adapter and RoPE-PI fused on q and k; the same without RoPE; without
    adapter or RoPE; o with the adapter; o without.  Each: `warmup` calls, then `steps` calls
    timed with CUDA events.  value = the first one's TFLOP/s (2*T*K*outputs + adapter flops)."""
    import torch

    import shifted_sparse_attention_s2attn_b200 as s2

    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    T, K, n, D = w.B * w.N, w.H * w.D, w.H * w.D, w.D
    gen = torch.Generator(device=dev)
    gen.manual_seed(20)
    x = torch.randn((T, K), generator=gen, device=dev).to(torch.bfloat16)
    s2.clear_device_error()
    out = {}
    for name, parts, r, rope_parts in (("qkv_lora_rope", 3, 8, 2), ("qkv_lora", 3, 8, 0), ("qkv_plain", 3, 0, 0),
                                       ("o_lora", 1, 8, 0), ("o_plain", 1, 0, 0)):
        wt = (torch.randn((parts * n, K), generator=gen, device=dev) / K ** 0.5).to(torch.bfloat16)
        a = (torch.randn((parts * r, K), generator=gen, device=dev) / K ** 0.5).to(torch.bfloat16) if r else None
        b = (0.05 * torch.randn((parts * n, r), generator=gen, device=dev)).to(torch.bfloat16) if r else None
        y = torch.empty((parts, T, n), dtype=torch.bfloat16, device=dev)
        ws = torch.empty(max(256, s2.lora_proj_workspace_bytes(T, K, n, parts, r)), dtype=torch.uint8, device=dev)

        def call():
            s2.lora_proj_fwd(x, wt, a, b, y, parts, 2.0, rope_parts=rope_parts, head_dim=D, seq_len=w.N,
                             pos_scale=w.pos_scale, workspace=ws, stream=stream)
        for _ in range(args.warmup):
            call()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            call()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        ms = e0.elapsed_time(e1) / args.steps
        flops = 2 * T * K * parts * n + 2 * T * K * parts * r + 2 * T * r * parts * n
        out[name] = {"ms": ms, "tflops": flops / (ms / 1e3) / 1e12, "parts": parts, "r": r,
                     "rope_parts": rope_parts}
        del wt, a, b, y, ws
    rc, detail = s2.get_device_error()
    if rc != 0:
        raise SystemExit(f"device error word set during the projection runs: {detail:#x}")
    if rank != 0:
        return 0
    peaks, peak_src = load_peaks()
    peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    line = {"metric": "LoRA-adapted q/k/v projection with fused RoPE-PI, TFLOP/s", "value": out["qkv_lora_rope"]["tflops"],
            "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": out["qkv_lora_rope"]["ms"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "mode": "lora",
            "config": {"workload": f"{w.name} layer projections: T={T} tokens, K={K}, q/k/v 3x{n} and o {n} "
                                   f"outputs, LoRA rank 8, scaling 2, RoPE-PI pos_scale {w.pos_scale}"},
            "roofline": {"kernel": "lora_gemm_kernel<256,true>", "bound": "tensor",
                         "achieved": out["qkv_lora_rope"]["tflops"], "peak": peak, "unit": "TFLOP/s",
                         "frac": out["qkv_lora_rope"]["tflops"] / peak, "traffic": None,
                         "peak_source": f"{peak_src} bf16_tflops (burst)",
                         "note": "achieved covers the call's three kernels (pad, down projection, projection)"},
            "calls": {k_: dict(v_, frac=v_["tflops"] / peak) for k_, v_ in out.items()},
            "gpu_launches": sum(args.steps * (3 if v_["r"] else 1) for v_ in out.values())}
    print(json.dumps(line), flush=True)
    return 0


def run_layer(args, w):
    """--mode layer: one LongLoRA attention layer training step of the workload's shape (one GPU):
    the LoRA-adapted q/k/v projection with RoPE-PI fused in its epilogue (no separate rotation
    pass), S^2-Attn forward, the o projection; then their backward (W frozen; the RoPE backward is
    rope_pi_apply with -pos_scale on dq, dk).  Adapter rank 8, scaling 2.  Every launch is one of
    this library's kernels.  value = the step's useful TFLOP/s: projections 2*T*K*outputs per
    direction (dx only, W frozen) plus the adapters, attention as in the default mode."""
    import torch

    import shifted_sparse_attention_s2attn_b200 as s2
    from shifted_sparse_attention_s2attn_b200.layer import LayerBuffers, LayerShape, LayerWeights, layer_bwd, layer_fwd

    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    r = 8
    s = LayerShape(B=w.B, N=w.N, H=w.H, D=w.D, G=w.G, shift_heads=w.shift_heads, r=r, scaling=2.0,
                   pos_scale=w.pos_scale, base=w.base)
    T, n = s.T, s.width
    gen = torch.Generator(device=dev)
    gen.manual_seed(30)
    bf = torch.bfloat16

    def rnd(shape, std):
        return (std * torch.randn(shape, generator=gen, device=dev)).to(bf)
    x, dy = rnd((T, n), 1.0), rnd((1, T, n), 1.0)
    wts = LayerWeights(rnd((3 * n, n), n ** -0.5), rnd((n, n), n ** -0.5), rnd((3 * r, n), n ** -0.5),
                       rnd((3 * n, r), 0.05), rnd((r, n), n ** -0.5), rnd((n, r), 0.05))
    buf = LayerBuffers(s, dev)
    s2.clear_device_error()

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        layer_fwd(s, wts, x, buf, stream)
        if ev is not None:
            ev[1].record(stream)
        layer_bwd(s, wts, x, dy, buf, stream)
        if ev is not None:
            ev[2].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(args.steps):
        step(evs[i])
    e1.record(stream)
    torch.cuda.synchronize(dev)
    rc, detail = s2.get_device_error()
    if rc != 0:
        raise SystemExit(f"device error word set during the layer steps: {detail:#x}")
    if rank != 0:
        return 0
    ms = e0.elapsed_time(e1) / args.steps
    fwd_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    bwd_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    attn = step_flops(w)
    proj_fwd = 2 * T * n * 4 * n + 2 * T * n * 4 * r + 2 * T * r * 4 * n
    proj_bwd = 2 * T * n * 4 * n + 3 * (2 * T * n * 4 * r)   # dx (+ adapter terms) and dA, dB
    flops = attn + proj_fwd + proj_bwd
    peaks, peak_src = load_peaks()
    peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    value = flops / (ms / 1e3) / 1e12
    line = {"metric": "LongLoRA attention layer training step (LoRA q/k/v + RoPE-PI fused, S2-Attn, LoRA o; fwd+bwd) "
                      "useful TFLOP/s",
            "value": value, "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "mode": "layer",
            "config": {"workload": f"{w.name} layer: T={T} tokens, width {n}, H={w.H}, D={w.D}, G={w.G}, "
                                   f"{w.shift_heads} shifted heads, LoRA rank {r} on q/k/v and o, scaling 2"},
            "fwd_ms": fwd_ms, "bwd_ms": bwd_ms, "flops_per_step": flops, "frac_of_peak": value / peak,
            "peak_source": f"{peak_src} bf16_tflops (burst)",
            "launches": "fwd: pad, down, projection (q/k/v, RoPE fused), s2attn_fwd, pad, down, projection (o); "
                        "bwd: the o projection's backward, s2attn_bwd (3 kernels), rope_pi_apply(-pos_scale), the "
                        "q/k/v projection's backward"}
    print(json.dumps(line), flush=True)
    return 0


def run_decode(args, w):
    """--mode decode: the decoding step of full causal attention alone (one GPU): the last M rows of q
    as queries against all N positions of k and v at the workload's shape, M = 1, 16, 128; `warmup`
    calls, then `steps` calls timed with CUDA events.  HBM-bound: K and V are read once per call
    (0.54 GB at 32k, larger than L2).  value = the M = 16 call's K/V read bandwidth in GB/s."""
    import torch

    import shifted_sparse_attention_s2attn_b200 as s2

    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    B, N, H, D = w.B, w.N, w.H, w.D
    gen = torch.Generator(device=dev)
    gen.manual_seed(40)
    k, v = (torch.randn((B, N, H, D), generator=gen, device=dev).to(torch.bfloat16) for _ in range(2))
    peaks, peak_src = load_peaks()
    peak = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    s2.clear_device_error()
    out = {}
    for M in (1, 16, 128):
        q = torch.randn((B, M, H, D), generator=gen, device=dev).to(torch.bfloat16)
        o = torch.empty_like(q)
        lse = torch.empty((B, H, M), dtype=torch.float32, device=dev)
        ws = torch.empty(s2.s2attn_decode_workspace_bytes(B, M, N, H, D), dtype=torch.uint8, device=dev)
        for _ in range(args.warmup):
            s2.s2attn_decode(q, k, v, o, lse, ws, stream)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            s2.s2attn_decode(q, k, v, o, lse, ws, stream)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        ms = e0.elapsed_time(e1) / args.steps
        kv_bytes = 2 * B * N * H * D * 2
        out[f"M{M}"] = {"ms": ms, "gbs": kv_bytes / (ms / 1e3) / 1e9, "frac": kv_bytes / (ms / 1e3) / 1e9 / peak}
        del q, o, lse, ws
    rc, detail = s2.get_device_error()
    if rc != 0:
        raise SystemExit(f"device error word set during the decoding steps: {detail:#x}")
    if rank != 0:
        return 0
    line = {"metric": "decoding step K/V read bandwidth, GB/s (M = 16 queries)", "value": out["M16"]["gbs"],
            "unit": "GB/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": out["M16"]["ms"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "mode": "decode",
            "config": {"workload": f"{w.name}: the last M rows of a query tensor against all N={N} positions of k, v "
                                   f"(H={H}, D={D}); full causal attention"},
            "roofline": {"bound": "hbm", "peak": peak, "unit": "GB/s", "peak_source": f"{peak_src} hbm_gbs"},
            "calls": out}
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="llama2_7b_32k", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--step-only", action="store_true",
                    help="time the step loop and stop (no other sections, no CPU baseline): for profiler captures")
    ap.add_argument("--mode", default="replicas", choices=["replicas", "sequence", "lora", "layer", "decode"],
                    help="replicas: every rank runs the whole workload (default); sequence: the "
                         "workload's sequence is split across the ranks; lora: the layer's LoRA-adapted "
                         "projections alone; layer: one LongLoRA attention layer training step; decode: the "
                         "decoding step of full causal attention alone")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        raise SystemExit("--warmup must be >= 3")
    w = WORKLOADS[args.workload]
    if w.dtype != "bf16":
        raise SystemExit("the bench times the bf16 tensor-core path")
    if args.impl == "reference":
        return run_reference(args, w)
    if args.mode == "sequence":
        return run_sequence_sharded(args, w)
    if args.mode == "lora":
        return run_lora_projections(args, w)
    if args.mode == "layer":
        return run_layer(args, w)
    if args.mode == "decode":
        return run_decode(args, w)
    return run_ours(args, w)


if __name__ == "__main__":
    sys.exit(main())
