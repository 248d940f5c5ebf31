"""The GEMMs' raster order, checked on the host: tile_coords (csrc/ptx.cuh)
with raster_group's group size (csrc/internal.cuh) is a bijection onto the
(token tile, weight tile) grid, keeps each group's activations within its
budget, and keeps the token tiles of a weight tile consecutive. Compiled
with nvcc as host code (no GPU needed)."""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
NVCC = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"


@pytest.mark.skipif(not os.path.exists(NVCC), reason="needs nvcc")
def test_raster_order_is_a_bijection_with_bounded_groups(tmp_path):
    exe = tmp_path / "raster_check"
    csrc = os.path.join(ROOT, "block_scaled_fp8_fp8blk_b200", "csrc")
    subprocess.run([NVCC, "-std=c++17", "-O1", "-gencode", "arch=compute_100a,code=sm_100a",
                    "-I", csrc, "-I", os.path.join(ROOT, "include"), "-o", str(exe),
                    os.path.join(HERE, "native", "raster_check.cu")], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert out.returncode == 0 and out.stdout.startswith("ok"), out.stdout
