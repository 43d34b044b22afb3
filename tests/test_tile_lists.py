"""The symmetric-product tiling of the tensor-core path, checked on the host:
the real header functions (for_each_sym_tile, for_each_full_tile, split_n, sym_block_mode), compiled with
g++ against csrc/muon_internal.cuh (no GPU), walked the way the epilogue
walks a tile.  See tests/host/sym_tiles_check.cpp for the properties."""

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA_INC = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "include")


@pytest.mark.skipif(shutil.which("g++") is None or not os.path.isdir(CUDA_INC), reason="needs g++ and CUDA headers")
def test_sym_tile_list_covers_the_lower_triangle_once(tmp_path):
    exe = tmp_path / "sym_tiles_check"
    cmd = ["g++", "-std=c++17", "-O2", "-I", os.path.join(ROOT, "include"),
           "-I", os.path.join(ROOT, "matrix_orthogonalizing_optimizer_muon_b200", "csrc"), "-I", CUDA_INC,
           os.path.join(ROOT, "tests", "host", "sym_tiles_check.cpp"), "-o", str(exe)]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stdout
    # 1408 = 11 blocks of 128 rows: 10 + 5 + 3 tiles; 2048 = 16 blocks: 28 + 8 tiles;
    # split along N once every 256-column tile becomes two, twice four
    assert out.stdout.strip().splitlines() == ["ok 18 36", "split 1 36 72", "split 2 72 144", "full ok"]
