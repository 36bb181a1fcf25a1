"""The algorithmic byte and FLOP counts bench.py divides by (the roofline's numerator), checked
against the per-step totals computed by hand from the layer shapes (d 4480; 27 Mamba-2 layers with
in_proj 22656 x 4480 and out_proj 4480 x 10240; 4 attention layers with qkv 7168 x 4480 and
o 4480 x 5120; 25 MLP layers 15680 x 4480 and back; two bf16 heads 131072 x 4480).  Also the
reference arm's JSON line, run on the host for the tiny workload (alone and under torchrun with two
ranks), and the summary of the clock record."""
import pytest

import bench
import synth


def test_linear_weight_count():
    cfg = synth.CONFIGS["nano_bf16"]
    n = sum(N * K for l in range(cfg.n_layers) for _, N, K in synth.linear_shapes(cfg, l))
    assert n == 27 * (22656 * 4480 + 4480 * 10240) + 4 * (7168 * 4480 + 4480 * 5120) + 25 * 2 * 15680 * 4480


@pytest.mark.parametrize("name,gb", [("nano_bf16", 17.95), ("nano_w4", 6.69), ("nano_w3", 5.71)])
def test_step_bytes_batch1_ctx2000(name, gb):
    cfg = synth.CONFIGS[name]
    read, write, weights = bench.step_bytes(cfg, 1, 2000)
    assert abs(read / 1e9 - gb) < 0.02, read
    # what the step writes: the SSM state, one conv row per Mamba layer, one KV row per attention layer
    assert write == 27 * 128 * 80 * 128 * 4 + 27 * 12288 * 2 + 4 * 2 * 8 * 128 * 2


def test_quantized_matrix_bytes():
    # W4 g64: 4 bits per weight, then per 64 weights an fp16 scale and a 4-bit zero
    assert bench.matrix_bytes(synth.FMT_W4, 64, 16, 128) == 16 * 128 / 2 + 16 * 2 * (2 + 0.5)
    # W8: 8 bits per weight, an fp16 scale per group, no zero
    assert bench.matrix_bytes(synth.FMT_W8, 128, 16, 256) == 16 * 256 + 16 * 2 * 2
    assert bench.matrix_bytes(synth.FMT_BF16, 64, 16, 128) == 16 * 128 * 2


def test_prefill_flops_4096():
    proj, attn, ssd = bench.prefill_flops(synth.CONFIGS["nano_prefill"], 4096)
    assert abs(proj / 1e12 - 63.17) < 0.01
    # causal attention: QK^T and PV over T(T+1)/2 pairs, 40 q heads of 128, 4 layers
    assert attn == 4 * 40 * 2 * 2.0 * 128 * 4096 * 4097 / 2
    assert 0 < ssd < 0.05 * proj


def test_reference_arm_line_on_the_tiny_workload():
    """`bench.py --impl reference` times the oracle on the host (no GPU, no torch.cuda) and prints
    one JSON line with the base keys, the steps it timed and its own cpu_baseline and e2e."""
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--config", "tiny_w8", "--steps", "5",
                          "--warmup", "3"], cwd=root, capture_output=True, text=True, timeout=300, check=True)
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "frame-steps/s" and d["higher_is_better"] is True
    assert d["steps"] == 5 and d["steps_requested"] == 5 and d["warmup"] == 1
    assert d["value"] > 0 and abs(d["ms_per_step"] - 1000.0 / d["value"]) < 1e-6 * d["ms_per_step"]
    assert d["config"]["workload"] == "tiny"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "frame-steps/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_reference_arm_under_torchrun_prints_once():
    """launched as N > 1 runs are (torchrun, two local ranks on 127.0.0.1), only rank 0
    runs the oracle and prints; the other rank exits 0 without work"""
    import json
    import os
    import subprocess
    import sys
    import socket
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    with socket.socket() as sock:
        sock.bind(("127.0.0.1", 0))
        port = sock.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--gpus", "2", "--impl",
           "reference", "--config", "tiny_w8", "--steps", "4", "--warmup", "3"]
    out = subprocess.run(cmd, cwd=root, capture_output=True, text=True, timeout=600, check=True)
    lines = [l for l in out.stdout.splitlines() if l.lstrip().startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["steps"] == 4


def test_clock_record_summary():
    """the clocks object of the JSON line: median SM clock, the highest max clock seen, and every
    throttle reason that was active in any sample"""
    s = bench.ClockSampler()
    s.samples = [["1965", "1965", "700.1", "Not Active", "Not Active", "Not Active", "Not Active"],
                 ["1800", "1965", "990.0", "Not Active", "Not Active", "Not Active", "Active"],
                 ["1900", "1965", "980.5", "Not Active", "Not Active", "Not Active", "Not Active"],
                 ["[N/A]", "1965", "[N/A]", "Not Active", "Not Active", "Not Active", "Not Active"]]
    c = s.stop()
    assert c["sm_mhz"] == 1900.0 and c["sm_max_mhz"] == 1965.0
    assert c["reasons"] == ["sw_power_cap"] and c["samples"] == 4
    s2 = bench.ClockSampler()
    assert s2.stop()["reasons"] == ["no samples"]


def test_decode_launch_count():
    """kernels per decode step: the input kernel, in_proj GEMV + Mamba-2 step + out_proj GEMV per
    Mamba-2 layer (27), QKV GEMV + attention + o_proj GEMV per attention layer (4), up and down
    GEMVs per MLP layer (25), and the heads: 1 + 81 + 12 + 50 + 1 (the same counts per kernel as
    the ncu launch lists of the step)"""
    assert bench.launches_per_step(synth.CONFIGS["nano_bf16"]) == 145
    assert bench.launches_per_step(synth.CONFIGS["tiny_w8"]) == 1 + 3 + 2 + 3 + 2 + 1


def test_further_configurations_of_the_default_run():
    """the default run measures W3, 16 sessions and the prefill as short runs of their own (one
    process each): their command lines, the summary kept under "also", and that a failing or late
    configuration is recorded without numbers while the others still report"""
    import json
    import subprocess
    from types import SimpleNamespace

    cmd = bench.extra_command("nano_w3", 20, 5)
    assert cmd[cmd.index("--steps") + 1] == "20" and cmd[cmd.index("--warmup") + 1] == "5"
    assert "--no-cpu-baseline" in cmd and cmd[cmd.index("--config") + 1] == "nano_w3"
    cmd = bench.extra_command("nano_prefill", 1000, 20)
    assert cmd[cmd.index("--steps") + 1] == "3" and cmd[cmd.index("--warmup") + 1] == "10"
    assert bench.extra_command("nano_w8_b16", 1000, 1)[4:8] == ["--steps", "300", "--warmup", "3"]

    calls = []

    def fake_run(cmd, **kw):
        name = cmd[cmd.index("--config") + 1]
        calls.append((name, kw.get("env", {})))
        if name == "nano_w8_b16":
            return subprocess.CompletedProcess(cmd, 1, "", "Traceback ...\nRuntimeError: out of memory\n")
        line = {"value": 12.5, "unit": "u", "ms_per_step": 3.0, "steps": 20, "roofline": {"frac": 0.25},
                "config": {"workload": name}, "e2e": {"value": 12.0}, "clocks": {"sm_mhz": 1965.0}}
        return subprocess.CompletedProcess(cmd, 0, "noise\n" + json.dumps(line) + "\n", "")

    out = bench.run_extras(SimpleNamespace(steps=20, warmup=5), run=fake_run)
    assert [c[0] for c in calls] == list(bench.EXTRA_CONFIGS)
    assert all("RANK" not in env and "WORLD_SIZE" not in env for _, env in calls)
    assert out["nano_w3"]["roofline_frac"] == 0.25 and out["nano_w3"]["value"] == 12.5
    assert out["nano_w3"]["config"] == {"workload": "nano_w3"}
    assert out["nano_w8_b16"] == {"error": "exit 1: RuntimeError: out of memory"}
    assert out["nano_prefill"]["ms_per_step"] == 3.0
    late = bench.run_extras(SimpleNamespace(steps=20, warmup=5), budget_s=-1.0, run=fake_run)
    assert all("skipped" in late[n] for n in bench.EXTRA_CONFIGS)


def test_default_run_assembles_one_line(monkeypatch, capsys):
    """main() of the default run on one GPU, with the measurements faked on the host: one JSON line
    whose "also" holds the bf16 backbone and the further configurations, and whose gpu_launches
    counts the two timed decode runs only"""
    import json
    import sys
    import torch

    def fake_decode(args, cfg, world, rank, local, steps, e2e_steps, cpu_baseline):
        return {"metric": bench.METRIC, "value": 1.0 if cfg.name == bench.DEFAULT_CONFIG else 2.0,
                "unit": "frame-steps/s", "ms_per_step": 3.0, "steps": steps, "achieved_step_gbs": 1.0,
                "step_frac_of_peak": 0.5, "e2e": {"value": 1.0}, "clocks": {}, "roofline": {"frac": 0.4},
                "gpu_launches": 100 if cfg.name == bench.DEFAULT_CONFIG else 7, "config": {"workload": cfg.name}}

    monkeypatch.setattr(bench, "run_decode", fake_decode)
    monkeypatch.setattr(bench, "run_extras", lambda args: {n: {"value": 3.0} for n in bench.EXTRA_CONFIGS})
    monkeypatch.setattr(torch.cuda, "set_device", lambda *a: None)
    monkeypatch.setattr(torch.cuda, "empty_cache", lambda *a: None)
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    monkeypatch.setattr(sys, "argv", ["bench.py", "--steps", "20", "--warmup", "5"])
    bench.main()
    lines = [l for l in capsys.readouterr().out.splitlines() if l.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["config"]["workload"] == bench.DEFAULT_CONFIG and line["value"] == 1.0
    assert set(line["also"]) == {"nano_bf16", *bench.EXTRA_CONFIGS}
    assert line["also"]["nano_bf16"]["value"] == 2.0 and line["also"]["nano_bf16"]["roofline_frac"] == 0.4
    assert line["gpu_launches"] == 107


def test_latency_summary():
    """per-step wall times (s) -> mean, median and 95th percentile in ms (linear interpolation
    between order statistics, numpy's default)"""
    d = [0.001 * i for i in range(1, 101)]          # 1 .. 100 ms
    r = bench.latency_ms(d)
    assert abs(r["mean_ms"] - 50.5) < 1e-9
    assert abs(r["p50_ms"] - 50.5) < 1e-9
    assert abs(r["p95_ms"] - 95.05) < 1e-9
    assert bench.latency_ms([]) == {"mean_ms": None, "p50_ms": None, "p95_ms": None}
