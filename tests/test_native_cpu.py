"""Host-only native checks (no GPU): the tcgen05 descriptor bit packing used
by the scoring kernel equals CUTLASS/CuTe's bitfield definitions."""

import importlib.util
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _cutlass_include():
    """CUTLASS/CuTe headers: $CUTLASS_INCLUDE, else a copy vendored inside an
    installed Python package (found through the import system, not a path)."""
    cands = [os.environ.get("CUTLASS_INCLUDE", "")]
    for pkg, sub in (("flashinfer", ("data", "cutlass", "include")),
                     ("tilelang", ("3rdparty", "cutlass", "include"))):
        spec = importlib.util.find_spec(pkg)
        if spec is not None and spec.submodule_search_locations:
            for loc in spec.submodule_search_locations:
                cands.append(os.path.join(loc, *sub))
    for d in cands:
        if d and os.path.exists(os.path.join(d, "cute", "arch", "mma_sm100_desc.hpp")):
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
