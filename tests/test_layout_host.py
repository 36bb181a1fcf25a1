"""The device weight layout of the streaming GEMV, checked on the host (no GPU): the header that
defines it (attention_frame_decode_b200/csrc/layout.cuh) is compiled by the host compiler into
tests/host/layout_check.cpp, which walks every code of padded matrices in every format and group
size and checks that codes stay inside their block's tiles, share no bit and fill the tiles, and
that each slab's metadata record sits after the tiles inside its block.  The stored bits per weight
it reports are the layout's cost (not the roofline's algorithmic bytes, which count a 3-bit zero as
3 bits where the layout keeps 4)."""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs a host C++ compiler")
def test_layout_is_in_bounds_injective_and_packed(tmp_path):
    exe = str(tmp_path / "layout_check")
    subprocess.run(["g++", "-O2", "-std=c++17", "-o", exe, os.path.join(HERE, "host", "layout_check.cpp")],
                   check=True, capture_output=True, timeout=300)
    out = subprocess.run([exe], capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stdout
    lines = out.stdout.splitlines()
    assert lines[-1] == "ok"
    per_weight = {}
    for l in lines[:-1]:
        head, tail = l.split(":")
        per_weight[head.strip()] = int(tail.split("/")[0])
    assert per_weight["fmt 0 g 64"] == 16 * 64          # bf16
    assert per_weight["fmt 1 g 64"] == 8 * 64 + 16      # W8: one fp16 scale per 64 weights
    assert per_weight["fmt 1 g 128"] == 8 * 64 + 8
    assert per_weight["fmt 2 g 64"] == 4 * 64 + 20      # W4: fp16 scale + 4-bit zero per 64
    assert per_weight["fmt 3 g 64"] == 3 * 64 + 20      # W3: fp16 scale + zero kept in 4 bits
