"""Small, self-contained launches of single kernels, for profilers (ncu) and quick timing.

    python -m attention_frame_decode_b200.kernel_cases gemv --fmt w4 --n 15680 --k 4480
    python -m attention_frame_decode_b200.kernel_cases gemm --m 4096 --n 15680 --k 4480
    python -m attention_frame_decode_b200.kernel_cases ssd --frames 1024
    python -m attention_frame_decode_b200.kernel_cases attn --batch 16

Each case builds its inputs on the device from the seeded generators, runs the kernel a few
times, and prints the mean time of `--reps` further launches measured with CUDA events.  The
inputs are larger than the 126 MB L2 where the kernel is bandwidth-bound (weights of the Nano
projections), and small enough (a few GB at most) for a profiler to save and restore.
"""
from __future__ import annotations

import argparse
import sys

FMTS = {"bf16": 0, "w8": 1, "w4": 2, "w3": 3}


def _time(fn, reps):
    import torch
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record()
    for _ in range(reps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / max(reps, 1) * 1000.0


def case_gemv(a):
    import torch
    import attention_frame_decode_b200 as vc
    import synth
    fmt = FMTS[a.fmt]
    N, K, B = a.n, a.k, a.batch
    w = torch.from_numpy(synth.normal_f32(1, 1, (N, K), 0.0, 0.02)).cuda()
    buf = vc.pack_bf16_weight(w.to(torch.bfloat16).contiguous()) if fmt == 0 else vc.quantize_weight(w, fmt, a.group)
    del w
    ld = (K + 127) // 128 * 128
    act = torch.zeros((B, ld), dtype=torch.bfloat16 if fmt == 0 else torch.float16, device="cuda")
    act[:, :K] = torch.from_numpy(synth.bf16_to_f32(synth.normal_bf16(1, 2, (B, K)))).cuda().to(act.dtype)
    scratch = vc.gemv_scratch()
    out = torch.empty((B, N), dtype=torch.float32, device="cuda")
    run = lambda: vc.debug_gemv(buf, fmt, a.group, N, K, act, scratch, out=out)
    for _ in range(a.warmup):
        run()
    us = _time(run, a.reps)
    print(f"gemv {a.fmt} g{a.group} N={N} K={K} B={B}: {us:.2f} us/launch")


def case_gemm(a):
    import torch
    import attention_frame_decode_b200 as vc
    import synth
    M, N, K = a.m, a.n, a.k
    A = torch.from_numpy(synth.bf16_to_f32(synth.normal_bf16(2, 1, (M, K)))).cuda().to(torch.bfloat16)
    W = torch.from_numpy(synth.bf16_to_f32(synth.normal_bf16(2, 2, (N, K), 0.0, 0.02))).cuda().to(torch.bfloat16)
    out = torch.empty((M, N), dtype=torch.float32, device="cuda")
    status = torch.zeros((1,), dtype=torch.int32, device="cuda")
    run = lambda: vc.debug_gemm(A, W, status, out=out)
    for _ in range(a.warmup):
        run()
    us = _time(run, a.reps)
    print(f"gemm M={M} N={N} K={K}: {us:.1f} us/launch, {2.0 * M * N * K / us / 1e6:.1f} TFLOP/s, "
          f"status {int(status.item())}")


def case_ssd(a):
    import torch
    import attention_frame_decode_b200 as vc
    import synth
    from attention_frame_decode_b200.model import DeviceModel
    cfg = synth.nano_config(name="nano_mixer", pattern="M", vocab_text=2048, vocab_func=2048)
    dm = DeviceModel(cfg)
    for k, v in synth.small_params(cfg, 5, 0).items():
        dm.set_small(0, k, v)
    T = a.frames
    c = vc.make_config(cfg, 1, T, 1)
    zx = torch.from_numpy(synth.normal_bf16(5, 600, (T, cfg.in_proj_rows))).cuda().view(torch.bfloat16)
    ssm = torch.zeros((cfg.ssm_heads, cfg.ssm_head_dim, cfg.ssm_state), device="cuda")
    conv = torch.zeros((cfg.conv_width, cfg.conv_dim), dtype=torch.bfloat16, device="cuda")
    y = torch.zeros((T, cfg.d_inner), device="cuda")
    act = torch.zeros((T, cfg.d_inner), dtype=torch.bfloat16, device="cuda")
    run = lambda: vc.debug_mamba_prefill(c, dm.layers[0], zx, ssm, conv, y, act)
    for _ in range(a.warmup):
        run()
    us = _time(run, a.reps)
    print(f"prefill mixer (conv + chunked SSD + gated norm), Nano widths, T={T}: {us:.1f} us/call")


def case_mamba(a):
    """decode frames of one Nano Mamba-2 layer (W8 g128 projections) for `batch` sessions with
    random state, launched kernel by kernel: its Mamba-2 step is the kernel of interest"""
    import numpy as np
    import torch
    import attention_frame_decode_b200 as vc
    import synth
    from attention_frame_decode_b200.synthetic import build_model, fill_state
    B = a.batch
    cfg = synth.nano_config(name="nano_mamba_layer", pattern="M", wfmt=synth.FMT_W8, group_size=128,
                            vocab_text=4096, vocab_func=2048)
    dm = build_model(cfg, 0)
    cap = 64
    bb = dm.backbone(B, cap, B)
    bb.set_option(vc.OPT_GRAPH, 0)
    st = dm.new_state(B, cap)
    fill_state(st, cfg, 0, np.full(B, 8), cap)
    tt = torch.zeros((B,), dtype=torch.int32, device="cuda")
    tf = torch.zeros_like(tt)
    x = torch.from_numpy(synth.frame_inputs(cfg, 0, 0, B)).cuda().view(torch.bfloat16)
    run = lambda: bb.step(x, st, tt, tf)
    for _ in range(a.warmup):
        run()
    us = _time(run, a.reps)
    print(f"one Nano Mamba-2 layer + heads, {B} sessions: {us:.1f} us/step, status {int(st.status.cpu()[0])}")
    bb.close()


def case_attn(a):
    """decode frames of one Nano attention layer (W8 g128 projections) for `batch` sessions whose
    K/V caches hold contexts drawn U(500, 6000) (a fixed 2000 for one session), launched kernel by
    kernel: its split-K decode attention is the kernel of interest"""
    import numpy as np
    import torch
    import attention_frame_decode_b200 as vc
    import synth
    from attention_frame_decode_b200.synthetic import build_model, fill_state
    B = a.batch
    cfg = synth.nano_config(name="nano_attn_layer", pattern="*", wfmt=synth.FMT_W8, group_size=128,
                            vocab_text=4096, vocab_func=2048, batch=B,
                            ctx_range=None if B == 1 else (500, 6000), kv_capacity=7000)
    ctx = synth.context_lengths(cfg, 0, B)
    cap = int(ctx.max()) + a.warmup + a.reps + 8
    dm = build_model(cfg, 0)
    bb = dm.backbone(B, cap, B)
    bb.set_option(vc.OPT_GRAPH, 0)
    st = dm.new_state(B, cap)
    fill_state(st, cfg, 0, ctx, cap)
    tt = torch.zeros((B,), dtype=torch.int32, device="cuda")
    tf = torch.zeros_like(tt)
    x = torch.from_numpy(synth.frame_inputs(cfg, 0, 0, B)).cuda().view(torch.bfloat16)
    run = lambda: bb.step(x, st, tt, tf)
    for _ in range(a.warmup):
        run()
    us = _time(run, a.reps)
    print(f"one Nano attention layer + heads, {B} sessions, contexts {int(ctx.min())}..{int(ctx.max())}: "
          f"{us:.1f} us/step, status {int(st.status.cpu()[0])}")
    bb.close()


def main(argv=None):
    ap = argparse.ArgumentParser()
    sub = ap.add_subparsers(dest="case", required=True)
    g = sub.add_parser("gemv")
    g.add_argument("--fmt", default="w4", choices=sorted(FMTS))
    g.add_argument("--group", type=int, default=64)
    g.add_argument("--n", type=int, default=15680)
    g.add_argument("--k", type=int, default=4480)
    g.add_argument("--batch", type=int, default=1)
    m = sub.add_parser("gemm")
    m.add_argument("--m", type=int, default=4096)
    m.add_argument("--n", type=int, default=15680)
    m.add_argument("--k", type=int, default=4480)
    s = sub.add_parser("ssd")
    s.add_argument("--frames", type=int, default=1024)
    mb = sub.add_parser("mamba")
    mb.add_argument("--batch", type=int, default=16)
    at = sub.add_parser("attn")
    at.add_argument("--batch", type=int, default=16)
    for p in (g, m, s, mb, at):
        p.add_argument("--warmup", type=int, default=3)
        p.add_argument("--reps", type=int, default=20)
    a = ap.parse_args(argv)
    {"gemv": case_gemv, "gemm": case_gemm, "ssd": case_ssd, "mamba": case_mamba, "attn": case_attn}[a.case](a)


if __name__ == "__main__":
    sys.exit(main())
