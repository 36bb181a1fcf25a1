"""Benchmark of the per-frame decode step (and the reference arm: the CPU oracle).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl vc|reference]

Default workload: the Nemotron-Nano-9B-v2-shaped backbone with W4 group-64 weights (bf16 heads),
batch 1, steady state decode at a context of 2000 frames (KV cache and SSM state pre-filled from
N(0,1)), synthetic seeded weights N(0, 0.02) and inputs N(0, 1).  One "step" is one frame through
all 56 layers and both vocabulary heads.  The same run then measures the bf16-weight backbone
(nano_bf16) for up to 300 steps and reports it under "also"; on one GPU it then runs W3 at batch
1, W8 g128 with 16 ragged sessions and the 4096-frame prefill, each as a short bench.py process of
its own, and adds their numbers under "also" too (--no-second skips all of these).  Other
workloads: --config nano_bf16 | nano_w3 | nano_w4_qheads | nano_w8_b16 | tiny_w8 (see
synth.CONFIGS), and nano_prefill: one step is then one prefill of the 4096-frame opening context
(tensor-core GEMMs, chunked SSD, causal attention).

With N > 1 (torchrun) every rank serves its own independent sessions with a full replica of
the weights (no collective on the data path); the reported value is the sum over ranks of
frames / max-over-ranks time.  Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "backbone frame-steps/s & ms/frame at batch 1 and 16; achieved HBM GB/s vs 8 TB/s"
DEFAULT_CONFIG = "nano_w4"   # the batch-1 W4 backbone (the configuration the HBM-roofline target names)


# ------------------------------------------------------------------------------------------------
# algorithmic bytes (layout independent: what the method must read per frame)
# ------------------------------------------------------------------------------------------------

def weight_bits(fmt):
    return {synth.FMT_BF16: 16, synth.FMT_W8: 8, synth.FMT_W4: 4, synth.FMT_W3: 3}[fmt]


def matrix_bytes(fmt, group, N, K):
    if fmt == synth.FMT_BF16:
        return N * K * 2
    ng = (K + group - 1) // group
    zero_bits = 0 if fmt == synth.FMT_W8 else weight_bits(fmt)
    return N * K * weight_bits(fmt) / 8 + N * ng * (2 + zero_bits / 8)


def step_bytes(cfg, B, ctx_mean):
    """bytes read per frame-step for B sessions: weights once, per-session SSM state, conv rows,
    KV cache (ctx+1 keys), small vectors; and bytes written (state, conv row, KV append)."""
    w = 0.0
    for l in range(cfg.n_layers):
        for _, N, K in synth.linear_shapes(cfg, l):
            w += matrix_bytes(cfg.wfmt, cfg.group_size, N, K)
        w += cfg.d_model * 4
        if cfg.pattern[l] == "M":
            w += (cfg.conv_dim * (cfg.conv_width + 1) + 3 * cfg.ssm_heads + cfg.d_inner) * 4
    heads = matrix_bytes(cfg.head_fmt, cfg.group_size, cfg.vocab_text, cfg.d_model) + \
        matrix_bytes(cfg.head_fmt, cfg.group_size, cfg.vocab_func, cfg.d_model)
    ssm = cfg.n_mamba * cfg.ssm_heads * cfg.ssm_head_dim * cfg.ssm_state * 4
    conv = cfg.n_mamba * (cfg.conv_width - 1) * cfg.conv_dim * 2
    kv_frame = cfg.n_attn * 2 * cfg.attn_kv_heads * cfg.attn_head_dim * 2
    read = w + heads + B * (ssm + conv + kv_frame * (ctx_mean + 1))
    write = B * (ssm + cfg.n_mamba * cfg.conv_dim * 2 + kv_frame)
    return read, write, w + heads


def launches_per_step(cfg):
    n = 1 + 1   # step input + heads
    for k in cfg.pattern:
        n += 3 if k in "M*" else 2
    return n


# DRAM bytes (read + write) per launch of the roofline kernel, from one ncu capture of the same
# kernel and shape (profiles/gemv_mlp_shapes_bf16_w4.md, profiles/gemm_tc_prefill_4096x15680x4480.md);
# None where no capture of the current kernel exists.
TRAFFIC = {
    "nano_bf16": 141.126400e6 + 4.253184e6,      # gemv bf16 15680 x 4480, B = 1
    "nano_w4": 38.456576e6 + 0.0,                # gemv W4 g64 15680 x 4480, B = 1
    "nano_prefill": 241.034496e6 + 236.244736e6,  # tcgen05 GEMM 4096 x 15680 x 4480
}


# DRAM bytes (read + write) per frame-kernel launch, from one ncu capture of the same workload;
# None where no capture of the current kernel exists
FRAME_TRAFFIC = {}


def max_over_ranks(value: float, world: int) -> float:
    """the largest of every rank's value (device timings are taken as the max over ranks);
    the tensor lives where the process group's backend wants it (CUDA for NCCL, CPU for gloo)"""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_rate(units_per_rank: float, world: int, seconds: float) -> float:
    """whole-job throughput of `world` independent replicas that each processed
    units_per_rank units in at most `seconds` (the max over ranks)"""
    return world * units_per_rank / seconds


def latency_ms(durations_s):
    """mean, median and 95th percentile (ms) of per-step wall times in seconds, as the pages report a
    frame's latency (mean and p95)"""
    d = np.asarray(durations_s, np.float64) * 1000.0
    if d.size == 0:
        return {"mean_ms": None, "p50_ms": None, "p95_ms": None}
    return {"mean_ms": float(d.mean()), "p50_ms": float(np.percentile(d, 50)), "p95_ms": float(np.percentile(d, 95))}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms while running"""

    def __init__(self, index=0):
        self.index = index
        self.samples = []
        self._stop = threading.Event()
        self._t = None

    def _run(self):
        q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
             "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
             "clocks_event_reasons.sw_power_cap")
        while not self._stop.is_set():
            try:
                out = subprocess.run(["nvidia-smi", f"--id={self.index}", f"--query-gpu={q}",
                                      "--format=csv,noheader,nounits"], capture_output=True, text=True, timeout=5)
                f = [x.strip() for x in out.stdout.strip().split(",")]
                if len(f) >= 7:
                    self.samples.append(f)
            except Exception:
                pass
            self._stop.wait(0.2)

    def start(self):
        self._t = threading.Thread(target=self._run, daemon=True)
        self._t.start()

    def stop(self):
        self._stop.set()
        if self._t:
            self._t.join(timeout=10)
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(s[0]) for s in self.samples if s[0].replace(".", "").isdigit()]
        mx = [float(s[1]) for s in self.samples if s[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for s in self.samples for i in range(4) if s[3 + i].lower() == "active"})
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(self.samples)}


# ------------------------------------------------------------------------------------------------
# CPU oracle (cpu_baseline leg and --impl reference)
# ------------------------------------------------------------------------------------------------

def oracle_run(cfg, max_steps, seed=0, warmup=0, budget_s=None):
    """time up to max_steps frame-steps of the oracle on this host (all cores) from the same
    pre-filled state, after `warmup` untimed ones; with a budget, the timing stops after the step
    that crosses it.  Returns (frame-steps/s, seconds timed, steps timed)."""
    import oracle
    B = cfg.batch
    model = oracle.Model(cfg, seed)
    st = model.new_state(B, cfg.kv_capacity)
    if cfg.random_state:
        st.fill_random(seed, synth.context_lengths(cfg, seed, B))
    for s in range(warmup):
        model.step(st, synth.frame_inputs(cfg, seed, s, B), oracle.MIRROR)
    n = 0
    t0 = time.perf_counter()
    while n < max_steps:
        model.step(st, synth.frame_inputs(cfg, seed, warmup + n, B), oracle.MIRROR)
        n += 1
        if budget_s is not None and time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    return B * n / dt, dt, n


def cpu_threads():
    """threads the oracle actually runs on (its OpenMP team size)"""
    import oracle
    return oracle.threads()


REF_BUDGET_S = 30.0   # seconds of oracle work the reference arm times, so that its run ends in minutes
REF_PREFILL_FRAMES = 16


def run_reference(args, cfg, rank):
    """The reference arm: the oracle on this host's cores, on this workload.  At most one untimed
    warm-up step, then up to --steps timed steps, each a bounded sample of the workload (decode: one
    frame-step of the whole batch, continuing from the same pre-filled state; prefill: the oracle's
    prefill of the context's first 16 frames into an empty slot); the timing stops after the step
    that crosses REF_BUDGET_S, and the line reports the steps it timed."""
    if rank != 0:
        return
    warm = min(args.warmup, 1)
    if cfg.prefill_T:
        Ts = REF_PREFILL_FRAMES
        value, dt, n = prefill_oracle_run(cfg, Ts, args.steps, warmup=warm, budget_s=REF_BUDGET_S)
        sample = (f"each step: the oracle's prefill of the first {Ts} frames of the {cfg.prefill_T}-frame "
                  f"context; {n} step(s) timed, {dt:.1f} s")
        line = {"impl": "reference", "metric": PREFILL_METRIC, "value": value, "unit": "frames/s",
                "n_gpus": args.gpus, "steps": n, "steps_requested": args.steps, "warmup": warm,
                "ms_per_step": 1000.0 * dt / n, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "f64", "data": "synthetic", "config": {"workload": cfg.name, "frames": cfg.prefill_T,
                                                                "batch": 1, "layers": cfg.n_layers,
                                                                "ssd_chunk": 256},
                "cpu_baseline": {"value": value, "unit": "frames/s", "cores": cpu_threads(), "kind": "oracle",
                                 "sample": sample},
                "e2e": {"value": value, "unit": "frames/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return
    ctx0 = synth.context_lengths(cfg, 0, cfg.batch)
    room = cfg.kv_capacity - int(ctx0.max()) - warm   # frames the cache holds
    value, dt, n = oracle_run(cfg, max(1, min(args.steps, room)), warmup=warm, budget_s=REF_BUDGET_S)
    sample = (f"each step: one frame-step of the batch of {cfg.batch} of {cfg.name}, continuing from the workload's starting "
              f"state; {n} step(s) timed, {dt:.1f} s")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "frame-steps/s", "n_gpus": args.gpus,
            "steps": n, "steps_requested": args.steps, "warmup": warm, "ms_per_step": 1000.0 * dt / n,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": cfg.name, "batch": cfg.batch,
                       "ctx_start": int(ctx0.max()) if cfg.batch == 1 else [int(ctx0.min()), int(ctx0.max())],
                       "layers": cfg.n_layers, "weights": synth.FMT_NAMES[cfg.wfmt], "group": cfg.group_size,
                       "heads": synth.FMT_NAMES[cfg.head_fmt]},
            "cpu_baseline": {"value": value, "unit": "frame-steps/s", "cores": cpu_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "frame-steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------------------------------
# prefill workload (--config nano_prefill): one step = one vc_prefill of the opening context
# ------------------------------------------------------------------------------------------------

PREFILL_METRIC = "prefill frames/s & ms per opening context (T frames, batch 1); tensor-pipe TFLOP/s"


def prefill_flops(cfg, T):
    """algorithmic FLOPs of one prefill of T frames: the projections (2 T N K each), the causal
    attention (QK^T and PV over the T(T+1)/2 visible pairs per q head) and the chunked SSD
    (intra-chunk C.B^T and its product with x, chunk states, off-diagonal readout), chunk 256."""
    proj = sum(2.0 * T * N * K for l in range(cfg.n_layers) for _, N, K in synth.linear_shapes(cfg, l))
    attn = cfg.n_attn * cfg.attn_q_heads * 2 * 2.0 * cfg.attn_head_dim * T * (T + 1) / 2
    Q = 256
    H, P, N, G = cfg.ssm_heads, cfg.ssm_head_dim, cfg.ssm_state, cfg.ssm_groups
    nch = (T + Q - 1) // Q
    per_chunk = (G * 2.0 * Q * Q * N / 2       # C.B^T, lower triangle, per group
                 + H * 2.0 * Q * Q * P / 2     # weighted sum over j <= i, per head
                 + H * 2.0 * Q * P * N         # chunk state
                 + H * 2.0 * Q * P * N)        # off-diagonal readout C.S_in
    ssd = cfg.n_mamba * nch * per_chunk
    return proj, attn, ssd


def prefill_oracle_run(cfg, T, max_runs, seed=0, warmup=0, budget_s=None):
    """time up to max_runs oracle prefills of the context's first T frames, each into an empty
    slot, after `warmup` untimed ones; with a budget, the timing stops after the run that crosses
    it.  Returns (frames/s, seconds timed, runs timed)."""
    import oracle
    model = oracle.Model(cfg, seed)
    x = synth.prefill_inputs(cfg, seed, T)
    for _ in range(warmup):
        model.prefill(model.new_state(1, max(T, 1) + 8), 0, x, oracle.MIRROR, ssd_chunk=256)
    n, dt = 0, 0.0
    while n < max_runs:
        st = model.new_state(1, max(T, 1) + 8)
        t0 = time.perf_counter()
        model.prefill(st, 0, x, oracle.MIRROR, ssd_chunk=256)
        dt += time.perf_counter() - t0
        n += 1
        if budget_s is not None and dt >= budget_s:
            break
    return T * n / dt, dt, n


def prefill_oracle_rate(cfg, T, seed=0):
    rate, dt, _ = prefill_oracle_run(cfg, T, 1, seed)
    return rate, dt


def run_prefill_bench(args, cfg, world, rank, local):
    import torch
    import torch.distributed as dist
    import attention_frame_decode_b200 as vc
    from attention_frame_decode_b200.synthetic import build_model
    T = cfg.prefill_T
    seed = 0
    dm = build_model(cfg, seed)
    cap = cfg.kv_capacity
    bb = dm.backbone(1, cap, 1)
    st = dm.new_state(1, cap)
    x = torch.from_numpy(synth.prefill_inputs(cfg, seed + 1000 * rank, T)).cuda().view(torch.bfloat16)
    for _ in range(args.warmup):
        bb.prefill(x, 0, st)
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        bb.prefill(x, 0, st)
    e1.record()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    ms = e0.elapsed_time(e1)
    ms = max_over_ranks(ms, world)
    ms_step = ms / args.steps
    value = replica_rate(T * args.steps, world, ms / 1000.0)
    proj, attn, ssd = prefill_flops(cfg, T)
    step_tflops = (proj + attn + ssd) / (ms_step / 1000.0) / 1e12

    # ---- roofline of the dominant kernel: the tcgen05 GEMM on the MLP up projection shape ----
    pk = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json"))) if os.path.exists(
        os.path.join(ROOT, "MEASURED_PEAKS.json")) else None
    peak = float(pk["bf16_tflops"]) if pk else 1590.0
    M, N, K = T, cfg.mlp_hidden, cfg.d_model
    A = torch.randn((M, K), device="cuda").to(torch.bfloat16)
    W = (0.02 * torch.randn((N, K), device="cuda")).to(torch.bfloat16)
    out = torch.empty((M, N), dtype=torch.float32, device="cuda")
    status = torch.zeros((1,), dtype=torch.int32, device="cuda")
    for _ in range(3):
        vc.debug_gemm(A, W, status, out=out)
    reps = 20
    g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    g0.record()
    for _ in range(reps):
        vc.debug_gemm(A, W, status, out=out)
    g1.record()
    torch.cuda.synchronize()
    gemm_ms = g0.elapsed_time(g1) / reps
    gemm_tf = 2.0 * M * N * K / (gemm_ms / 1000.0) / 1e12

    # ---- end to end: the context from pinned host memory, the slot's ctx_len back to the host ----
    xh = torch.from_numpy(synth.prefill_inputs(cfg, seed + 1000 * rank, T)).view(torch.bfloat16).pin_memory()
    ch = torch.empty((1,), dtype=torch.int32).pin_memory()
    xd = torch.empty_like(x)
    stream = torch.cuda.current_stream()
    ne = max(2, min(args.steps, 10))
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    lat = []
    for _ in range(ne):
        t1 = time.perf_counter()
        xd.copy_(xh, non_blocking=True)
        bb.prefill(xd, 0, st)
        ch.copy_(st.ctx_len[:1], non_blocking=True)
        stream.synchronize()
        lat.append(time.perf_counter() - t1)
    e2e_s = time.perf_counter() - t0
    assert int(ch[0]) == T
    e2e_value = world * T * ne / e2e_s

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        Ts = 16
        v, dt = prefill_oracle_rate(cfg, Ts)
        cpu = {"value": v, "unit": "frames/s", "cores": cpu_threads(), "kind": "oracle",
               "sample": f"prefill of the first {Ts} frames of the same context on the same model, {dt:.1f} s"}
    if rank == 0:
        # per layer: pre-norm, two unpacks (side stream) and two GEMMs, plus conv, dt, chunk
        # states, scan, SSD outputs and gated norm (Mamba-2) or flash attention; one final kernel
        n_launch = 1 + sum({"M": 11, "*": 6, "-": 5}[k] for k in cfg.pattern)
        line = {
            "metric": PREFILL_METRIC, "value": value, "unit": "frames/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16-operands/fp32-accum", "data": "synthetic (seeded)",
            "config": {"workload": cfg.name, "frames": T, "batch": 1, "layers": cfg.n_layers, "ssd_chunk": 256,
                       "l2": "no flush: 15.4 GB of weights per prefill >> 126 MB L2",
                       "parallelism": f"replicas x{world}"},
            "step_tflops": step_tflops, "flops_per_step": {"projections": proj, "attention": attn, "ssd": ssd},
            "roofline": {"bound": "tensor", "kernel": "tcgen05 GEMM (MLP up projection shape)", "achieved": gemm_tf,
                         "peak": peak, "peak_kind": "measured burst" if pk else "fallback", "unit": "TFLOP/s",
                         "frac": gemm_tf / peak, "traffic": TRAFFIC.get(cfg.name), "launch_ms": gemm_ms,
                         "flops_per_launch": 2.0 * M * N * K},
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": "frames/s", "h2d_bytes_per_step": T * cfg.d_model * 2,
                    "d2h_bytes_per_step": 4, "steps": ne, "prefill_latency": latency_ms(lat)},
            "gpu_launches": n_launch * args.steps, "clocks": clk, "device_status": int(st.status.cpu()[0]),
        }
        print(json.dumps(line), flush=True)
    bb.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_decode(args, cfg, world, rank, local, steps, e2e_steps, cpu_baseline):
    """one decode measurement of workload cfg: `steps` timed frame-steps after args.warmup, the GEMV
    roofline launch and the end-to-end host run; returns the JSON line on rank 0 (else None)"""
    import torch
    import torch.distributed as dist
    import attention_frame_decode_b200 as vc
    from attention_frame_decode_b200.synthetic import build_model, fill_state

    B = cfg.batch
    seed = 0
    dm = build_model(cfg, seed)
    ctx0 = synth.context_lengths(cfg, seed, B)
    total = args.warmup + steps
    # the workload's cache capacity, grown when the run itself needs more frames than it holds
    cap = max(cfg.kv_capacity, int(ctx0.max()) + total + e2e_steps + 8)
    bb = dm.backbone(B, cap, B)
    if args.no_graph:
        bb.set_option(vc.OPT_GRAPH, 0)
    if args.per_kernel:
        bb.set_option(vc.OPT_FRAME, 0)
    if args.frame:
        bb.set_option(vc.OPT_FRAME, 1)
    if args.gemv_shape is not None:
        bb.set_option(vc.OPT_GEMV_SHAPE, args.gemv_shape)
    frame = bb.uses_frame_kernel(B)
    st = dm.new_state(B, cap)
    if cfg.random_state:
        fill_state(st, cfg, seed + rank, ctx0, cap)
    # every frame input of the run, resident in HBM before timing (rank r serves its own sessions)
    xs = torch.empty((total, B, cfg.d_model), dtype=torch.bfloat16, device="cuda")
    for s in range(total):
        xs[s] = torch.from_numpy(synth.frame_inputs(cfg, seed + 1000 * rank, s, B)).view(torch.bfloat16)
    tt = torch.zeros((B,), dtype=torch.int32, device="cuda")
    tf = torch.zeros((B,), dtype=torch.int32, device="cuda")
    if int(cap - ctx0.max()) < total + e2e_steps + 8:
        raise SystemExit(f"kv capacity {cap} too small for {total + e2e_steps} steps")

    for s in range(args.warmup):
        bb.step(xs[s], st, tt, tf)
    torch.cuda.synchronize()

    clocks = ClockSampler(local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for s in range(args.warmup, total):
        bb.step(xs[s], st, tt, tf)
    e1.record()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    ms = e0.elapsed_time(e1)
    ms = max_over_ranks(ms, world)
    status = int(st.status.cpu()[0])
    ms_step = ms / steps
    value = replica_rate(B * steps, world, ms / 1000.0)
    ctx_mean = float(ctx0.mean()) + args.warmup + steps / 2.0
    rbytes, wbytes, weight_total = step_bytes(cfg, B, ctx_mean)
    step_gbs = rbytes / (ms_step / 1000.0) / 1e9

    # ---- roofline of the dominant kernel: the streaming GEMV on the layer MLP up projection ----
    peak, peak_kind = load_peaks()
    mlp = cfg.pattern.index("-")
    up = dm.layers[mlp].up
    K_up = cfg.d_model
    act_ld = (K_up + 127) // 128 * 128
    act = torch.zeros((B, act_ld), dtype=torch.bfloat16 if cfg.wfmt == synth.FMT_BF16 else torch.float16,
                      device="cuda")
    act[:, :K_up] = torch.randn((B, K_up), device="cuda").to(act.dtype)
    scratch = vc.gemv_scratch()
    ybuf = torch.empty((B, up.N), dtype=torch.float32, device="cuda")
    wbuf = next(t for t in dm.keep if t.data_ptr() == up.data)
    for _ in range(5):
        vc.debug_gemv(wbuf, cfg.wfmt, cfg.group_size, up.N, up.K, act, scratch, out=ybuf)
    reps = 50
    g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    g0.record()
    for _ in range(reps):
        vc.debug_gemv(wbuf, cfg.wfmt, cfg.group_size, up.N, up.K, act, scratch, out=ybuf)
    g1.record()
    torch.cuda.synchronize()
    gemv_ms = g0.elapsed_time(g1) / reps
    gemv_bytes = matrix_bytes(cfg.wfmt, cfg.group_size, up.N, up.K) + B * K_up * 2 + B * up.N * 4
    gemv_gbs = gemv_bytes / (gemv_ms / 1000.0) / 1e9

    # ---- end to end through the C ABI with host buffers (pinned x in, tokens out, every step) ----
    ne = max(1, e2e_steps)
    xh = torch.empty((ne, B, cfg.d_model), dtype=torch.bfloat16).pin_memory()
    for s in range(ne):
        xh[s] = torch.from_numpy(synth.frame_inputs(cfg, seed + 1000 * rank, total + s, B)).view(torch.bfloat16)
    th = torch.empty((B,), dtype=torch.int32).pin_memory()
    fh = torch.empty((B,), dtype=torch.int32).pin_memory()
    stream = torch.cuda.current_stream()
    bb.step_host(xh[0], st, th, fh)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    t0 = time.perf_counter()
    lat = []
    for s in range(1, ne):
        t1 = time.perf_counter()
        bb.step_host(xh[s], st, th, fh)
        stream.synchronize()   # the frame's tokens are on the host before the next frame
        lat.append(time.perf_counter() - t1)
    e2e_s = time.perf_counter() - t0
    e2e_s = max_over_ranks(e2e_s, world)
    e2e_value = world * B * (ne - 1) / e2e_s

    cpu = None
    if rank == 0 and world == 1 and cpu_baseline:
        # a bounded sample: frame-steps from the same pre-filled state until 15 s of work, 64 at most
        v, dt, n_or = oracle_run(cfg, 64, budget_s=15.0)
        cpu = {"value": v, "unit": "frame-steps/s", "cores": cpu_threads(), "kind": "oracle",
               "sample": f"{n_or} frame-step(s) of the same workload (batch {B}) from the same pre-filled state, "
                         f"{dt:.1f} s"}

    gemv_line = {"kernel": "gemv (mlp up projection, streaming weights)", "achieved": gemv_gbs, "peak": peak,
                 "peak_kind": peak_kind, "unit": "GB/s", "frac": gemv_gbs / peak, "launch_ms": gemv_ms,
                 "bytes_per_launch": gemv_bytes}
    if frame:
        # the frame kernel is the whole step: one launch per frame, timed above on its stream
        roofline = {"bound": "hbm", "kernel": "frame kernel (one launch per frame: all layers and both heads)",
                    "achieved": step_gbs, "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                    "frac": step_gbs / peak, "traffic": FRAME_TRAFFIC.get(cfg.name), "launch_ms": ms_step,
                    "bytes_per_launch": rbytes}
        launch = "frame kernel"
        n_launches = steps
    else:
        roofline = dict(gemv_line, bound="hbm", traffic=TRAFFIC.get(cfg.name))
        launch = "direct" if args.no_graph else "cuda graph"
        n_launches = launches_per_step(cfg) * steps
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "frame-steps/s", "n_gpus": world, "steps": steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None,
            "dtype": {synth.FMT_BF16: "bf16", synth.FMT_W8: "w8-fp16", synth.FMT_W4: "w4-fp16",
                      synth.FMT_W3: "w3-fp16"}[cfg.wfmt] + "-weights/fp32-accum",
            "data": "synthetic (seeded N(0,0.02) weights, N(0,1) inputs and pre-filled state)",
            "config": {"workload": cfg.name, "batch": B, "ctx_start": int(ctx0.max()) if B == 1 else
                       [int(ctx0.min()), int(ctx0.max())], "layers": cfg.n_layers, "weights": synth.FMT_NAMES[cfg.wfmt],
                       "group": cfg.group_size, "heads": synth.FMT_NAMES[cfg.head_fmt],
                       "l2": f"no flush: {weight_total / 1e9:.2f} GB of weights per step >> 126 MB L2",
                       "parallelism": f"replicas x{world}", "launch": launch,
                       **({"gemv_shape": args.gemv_shape} if args.gemv_shape is not None else {})},
            "achieved_step_gbs": step_gbs, "step_bytes_read": rbytes, "step_bytes_written": wbytes,
            "step_frac_of_peak": step_gbs / peak,
            "roofline": roofline, "gemv_kernel_alone": gemv_line,
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": "frame-steps/s", "h2d_bytes_per_step": B * cfg.d_model * 2,
                    "d2h_bytes_per_step": 2 * B * 4, "steps": ne - 1, "frame_latency": latency_ms(lat)},
            "gpu_launches": n_launches,
            "clocks": clk, "device_status": status,
        }
    bb.close()
    return line if rank == 0 else None


# the other configurations of the metric, measured after the default workload in the same
# single-GPU run: W3 at batch 1, W8 g128 with 16 ragged sessions, and the opening-context prefill
EXTRA_CONFIGS = ("nano_w3", "nano_w8_b16", "nano_prefill")
EXTRA_KEYS = ("value", "unit", "ms_per_step", "steps", "warmup", "achieved_step_gbs", "step_frac_of_peak",
              "step_tflops", "e2e", "clocks", "device_status")


def extra_command(name, steps, warmup):
    """the bench.py command line of one further configuration (a short run of its own)"""
    cfg = synth.CONFIGS[name]
    n = 3 if cfg.prefill_T else max(1, min(steps, 300))
    return [sys.executable, os.path.join(ROOT, "bench.py"), "--config", name, "--steps", str(n),
            "--warmup", str(max(3, min(warmup, 10))), "--no-cpu-baseline", "--e2e-steps", "20"]


def extra_summary(line):
    """the numbers of a further configuration's JSON line that go under "also\" """
    out = {k: line[k] for k in EXTRA_KEYS if k in line}
    out["roofline_frac"] = line["roofline"]["frac"]
    out["config"] = line["config"]
    return out


def run_extras(args, budget_s=300.0, run=subprocess.run):
    """each further configuration as its own process on the same GPU (so that a failure there
    leaves the default workload's line intact); a configuration that fails or would start after
    `budget_s` seconds is recorded with the reason instead of numbers"""
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "LOCAL_RANK", "WORLD_SIZE", "LOCAL_WORLD_SIZE",
                                                              "MASTER_ADDR", "MASTER_PORT")}
    out = {}
    t0 = time.perf_counter()
    for name in EXTRA_CONFIGS:
        if time.perf_counter() - t0 > budget_s:
            out[name] = {"skipped": f"time budget of {budget_s:.0f} s for the further configurations spent"}
            continue
        try:
            r = run(extra_command(name, args.steps, args.warmup), capture_output=True, text=True, timeout=240,
                    env=env, cwd=ROOT)
            lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
            if r.returncode != 0 or not lines:
                tail = (r.stderr or r.stdout).strip().splitlines()[-1:] or [""]
                out[name] = {"error": f"exit {r.returncode}: {tail[0][:300]}"}
            else:
                out[name] = extra_summary(json.loads(lines[-1]))
        except Exception as e:   # a timeout or an unreadable line: recorded, the default line stands
            out[name] = {"error": f"{type(e).__name__}: {str(e)[:300]}"}
    return out


# ------------------------------------------------------------------------------------------------
# GPU arm
# ------------------------------------------------------------------------------------------------

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--config", default=DEFAULT_CONFIG, choices=sorted(synth.CONFIGS))
    ap.add_argument("--impl", default="vc", choices=["vc", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-second", action="store_true",
                    help="default workload only: skip the second, bf16-weight measurement")
    ap.add_argument("--e2e-steps", type=int, default=200)
    ap.add_argument("--no-graph", action="store_true",
                    help="per-kernel path: launch each step's kernels directly instead of replaying a CUDA graph "
                         "(for profilers that cannot replay graph kernel nodes with programmatic dependencies)")
    ap.add_argument("--per-kernel", action="store_true",
                    help="run each frame as one kernel per operation")
    ap.add_argument("--frame", action="store_true",
                    help="run each frame as one launch of the frame kernel")
    ap.add_argument("--gemv-shape", type=int, default=None, choices=[0, 1, 2],
                    help="per-kernel path, up to 8 rows: SM occupancy of the streaming GEMV (VC_OPT_GEMV_SHAPE)")
    args = ap.parse_args()
    assert args.warmup >= 3, "at least 3 warm-up steps"
    cfg = synth.CONFIGS[args.config]

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        run_reference(args, cfg, rank)
        return

    import torch
    import torch.distributed as dist
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300))

    if cfg.prefill_T:
        run_prefill_bench(args, cfg, world, rank, local)
        return

    line = run_decode(args, cfg, world, rank, local, steps=args.steps, e2e_steps=args.e2e_steps,
                      cpu_baseline=not args.no_cpu_baseline)
    if cfg.name == DEFAULT_CONFIG and not args.no_second:
        # the bf16-weight backbone (the pages' unquantized model) as a second, shorter measurement
        torch.cuda.empty_cache()
        second = run_decode(args, synth.CONFIGS["nano_bf16"], world, rank, local, steps=min(args.steps, 300),
                            e2e_steps=min(args.e2e_steps, 20), cpu_baseline=False)
        if rank == 0:
            line["also"] = {"nano_bf16": {k: second[k] for k in ("value", "unit", "ms_per_step", "steps",
                                                                  "achieved_step_gbs", "step_frac_of_peak",
                                                                  "e2e", "clocks")}}
            line["also"]["nano_bf16"]["roofline_frac"] = second["roofline"]["frac"]
            line["gpu_launches"] += second["gpu_launches"]
        if world == 1:
            # the further configurations, after this run's own timed regions (not counted in its
            # gpu_launches)
            import gc
            del second
            gc.collect()
            torch.cuda.empty_cache()
            line["also"].update(run_extras(args))
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
