"""The streaming GEMV's stream-K partition, checked on the host (no GPU): the partition helpers of
attention_frame_decode_b200/csrc/gemv_core.cuh (part_begin, part_owner, warp_range; host and
device functions) are compiled by nvcc into tests/host/partition_check.cu and run on the CPU for
every projection shape of the Nano and tiny stacks, every weight format and group size, and the
grids the launches use (one or two 8-warp CTAs per SM on 148 or 132 SMs, and the no-allocation
entry's 32 SMs).  The harness checks that the workers' block ranges tile each matrix, that the
32-bit quotients equal the 64-bit ones, that part_owner names exactly the workers that touch each
row unit (the last contributor counts on it), that a split unit is the first or last unit of each
contributor's range (two partial-sum slots per worker), and that every scratch index stays in
bounds."""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


@pytest.mark.skipif(not (os.path.exists(NVCC) or shutil.which("nvcc")), reason="needs nvcc")
def test_stream_k_partition_covers_and_names_contributors(tmp_path):
    exe = str(tmp_path / "partition_check")
    nvcc = NVCC if os.path.exists(NVCC) else shutil.which("nvcc")
    r = subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O2", "-std=c++17",
                        "--expt-relaxed-constexpr", "-I" + os.path.join(ROOT, "include"), "-o", exe,
                        os.path.join(HERE, "host", "partition_check.cu")], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    out = subprocess.run([exe], capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stdout
    lines = out.stdout.splitlines()
    assert lines[-1] == "ok"
    assert lines[-2] == "490 launch geometries"
