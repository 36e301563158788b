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


def test_nvtx_ranges_build(tmp_path):
    # the tracing build (-DQSA_NVTX) compiles and names the C-ABI calls as
    # NVTX ranges; the default build has none
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not available")
    src = os.path.join(ROOT, "block_sparse_decode_b200", "csrc", "abi.cu")
    objs = {}
    for name, extra in (("plain", []), ("nvtx", ["-DQSA_NVTX"])):
        obj = tmp_path / f"abi_{name}.o"
        subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-std=c++17",
                        "-Xcompiler", "-fPIC", "-I" + os.path.join(ROOT, "include"), *extra,
                        "-c", src, "-o", str(obj)], check=True, capture_output=True)
        objs[name] = subprocess.run(["strings", str(obj)], capture_output=True,
                                    text=True).stdout
    assert "qsa_decode_step" in objs["nvtx"] and "nvtx" in objs["nvtx"].lower()
    assert "nvtx" not in objs["plain"].lower()
