"""Host logic of the streaming gate: the per-CTA tile ranges cut on the host cover every query tile
exactly once when walked the way the kernel walks them (CPU only; compiles a small C++ driver
against csrc/gate_stream.cu with nvcc, whose device code is never launched)."""
import os
import shutil
import subprocess

import pytest

from block_sparse_long_moba_b200 import build

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


def test_gate_schedule_covers_every_tile_once(tmp_path):
    try:
        nvcc = build.nvcc()
    except RuntimeError:
        pytest.skip("nvcc not available")
    exe = str(tmp_path / "gate_schedule_check")
    cmd = [nvcc, *build.ARCH, "-O1", "-std=c++17", "--expt-relaxed-constexpr",
           "-I", os.path.join(ROOT, "include"),
           os.path.join(HERE, "host", "gate_schedule_check.cu"),
           os.path.join(ROOT, "block_sparse_long_moba_b200", "csrc", "gate_stream.cu"),
           "-o", exe, "-lcuda"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    out = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stdout + out.stderr
    assert out.stdout.count(": ok") == 11, out.stdout
