"""Host-only native checks (no GPU): the tcgen05 descriptor bit packing used
by the scoring kernel equals CUTLASS/CuTe's bitfield definitions."""

import glob
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _cutlass_include():
    for pat in ("/opt/prime-rl/.venv/lib/python3*/site-packages/flashinfer/data/cutlass/include",
                "/opt/prime-rl/.venv/lib/python3*/site-packages/tilelang/3rdparty/cutlass/include"):
        for d in glob.glob(pat):
            if os.path.exists(os.path.join(d, "cute", "arch", "mma_sm100_desc.hpp")):
                return d
    return None


def test_umma_descriptors_match_cute(tmp_path):
    inc = _cutlass_include()
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if inc is None or not os.path.exists(nvcc):
        pytest.skip("CUTLASS headers or nvcc not available")
    exe = tmp_path / "umma_check"
    subprocess.run([nvcc, "-std=c++17", "-Wno-deprecated-gpu-targets", f"-I{inc}",
                    "-I" + os.path.join(ROOT, "block_sparse_decode_b200", "csrc"),
                    os.path.join(ROOT, "tests", "native", "umma_desc_check.cu"), "-o", str(exe)],
                   check=True, capture_output=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0 and "OK" in r.stdout, r.stdout
