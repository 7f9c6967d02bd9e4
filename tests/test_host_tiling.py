"""The kernels' host-side tiling rules (router tile height and stage ring, TMEM columns,
the combine's row split, the GEMM ring), swept exhaustively by a small host-only program
compiled with nvcc from the same headers (CPU only: it makes no CUDA call)."""
import os
import subprocess

from mixture_experts_layer_65_b200 import build

HERE = os.path.dirname(os.path.abspath(__file__))


def test_tiling_rules_hold_for_every_shape(tmp_path):
    exe = str(tmp_path / "host_tiling_check")
    cmd = [build.nvcc_path(), "-gencode", build.GENCODE, "-O2", "-std=c++17",
           "--expt-relaxed-constexpr", "-I", build.INCLUDE, "-I", build.CSRC,
           "-o", exe, os.path.join(HERE, "host_tiling_check.cu")]
    comp = subprocess.run(cmd, capture_output=True, text=True)
    assert comp.returncode == 0, comp.stdout + comp.stderr
    run = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0, run.stdout + run.stderr
    assert "all tiling rules hold" in run.stdout
