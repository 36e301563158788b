"""The C-ABI library loads, exports every symbol include/qsa.h declares, and
rejects bad arguments on the host (no GPU needed: none of these calls reaches
a CUDA call)."""

import ctypes
import os
import re

import pytest

from block_sparse_decode_b200 import build, qsa

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                      "include", "qsa.h")


@pytest.fixture(scope="module")
def L():
    build.build()
    return qsa.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(qsa_\w+)\s*\(", text)))


def test_header_declares_the_binding_exports():
    assert declared_functions() == sorted(qsa.EXPORTS)


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name
    out = os.popen(f"nm -D --defined-only {qsa.LIB_PATH}").read()
    for name in declared_functions():
        assert re.search(rf"\bT {name}\b", out), f"{name} not exported"


def test_version_and_workspace_sizes(L):
    assert qsa.qsa_version() == 100
    assert qsa.qsa_topk_workspace_size(8, 65536, 512) == 0
    d = qsa.QsaDims(32, 4, 128, 16, 128, 64, 0.088)
    # records of shared slices: 296 CTA slots / B sequences CTAs per sequence
    # (at most one per tile, at least ceil((k/4 + R - 1) / 256) for the page
    # table), keyed by CTA + slice, each 32 heads x (128 + 1) floats; plus one
    # (c_lo, c_hi) pair per (sequence, slice) and one arrival counter per
    # (sequence, group of 8 query heads) for the decode step's fused merge;
    # then, 16-byte aligned, the R + 1 slice starts per sequence that the
    # decode step's top-k hands to its decode kernel
    for B, k, R, ncb in ((8, 512, 4, 37), (512, 512, 4, 1), (512, 4096, 4, 5),
                         (2, 512, 2, 129), (1, 1, 1, 1)):
        used = B * (ncb + R - 1) * 32 * 129 * 4 + B * R * 8 + B * 4 * 4
        assert qsa.qsa_sparse_decode_workspace_size(d, B, k, R) == \
            (used + 15) // 16 * 16 + B * (R + 1) * 4, (B, k, R)


def test_prefill_workspace_sizes(L):
    # plan scratch: 16-byte header, each row's sequence, the groups' tile
    # prefix and their {sequence, first row, rows, blocks} (16 bytes), for at
    # most S + ceil(Nq / QG) groups of QG = 256 / Hi rows
    def r16(x):
        return (x + 15) // 16 * 16
    for Hi, di in ((16, 128), (4, 64), (8, 128), (32, 64)):
        d = qsa.QsaDims(32, 4, 128, Hi, di, 64, 0.088)
        QG = 256 // Hi
        for S, Nq in ((8, 256), (2, 73), (1, 1), (3, 130)):
            gmax = S + (Nq + QG - 1) // QG
            plan = 16 + r16(4 * Nq) + r16(4 * (gmax + 1)) + 16 * gmax
            assert qsa.qsa_prefill_index_score_workspace_size(d, S, Nq) == plan, (Hi, S, Nq)
            for k, R in ((512, 4), (64, 1)):
                total = (plan + 255) // 256 * 256 + \
                    qsa.qsa_sparse_decode_workspace_size(d, Nq, k, R)
                assert qsa.qsa_sparse_prefill_workspace_size(d, S, Nq, k, R) == total
    # indexer heads that do not tile the 256-column MMA are not supported
    assert qsa.qsa_prefill_index_score_workspace_size(qsa.QsaDims(32, 4, 128, 12, 128, 64,
                                                                  0.1), 1, 8) == 0
    assert qsa.qsa_sparse_prefill_workspace_size(qsa.QsaDims(32, 4, 128, 16, 128, 48, 0.1),
                                                 1, 8, 64, 1) == 0


def _status(fn, *args):
    return fn(*args)


def test_host_side_argument_checks(L):
    D = qsa._Dims
    bad = [
        D(32, 4, 64, 16, 128, 64, 0.1),    # D != 128
        D(32, 5, 128, 16, 128, 64, 0.1),   # Hq % Hkv
        D(32, 4, 128, 16, 96, 64, 0.1),    # di
        D(32, 4, 128, 33, 128, 64, 0.1),   # Hi > 32
        D(32, 2, 128, 16, 128, 64, 0.1),   # G = 16 > 8
        D(32, 4, 128, 16, 128, 62, 0.1),   # P % 4
    ]
    c = qsa._Cache(16, 16, 16, 16, 16, 1, 1, 1)
    for d in bad:
        st = L.qsa_index_score(ctypes.byref(d), ctypes.byref(c), 1, 16, 16, 16, 16, 4, None)
        assert st in (qsa.QSA_ERR_UNSUPPORTED, qsa.QSA_ERR_INVALID_ARG)
        assert L.qsa_last_error().decode()
    ok = D(32, 4, 128, 16, 128, 64, 0.1)
    assert L.qsa_index_score(None, ctypes.byref(c), 1, 16, 16, 16, 16, 4, None) == \
        qsa.QSA_ERR_INVALID_ARG
    assert L.qsa_topk_select(1, 16, 16, 100, 0, 16, None, 0, None) == qsa.QSA_ERR_UNSUPPORTED
    assert L.qsa_topk_select(1, 16, 16, 1 << 30, 8, 16, None, 0, None) == \
        qsa.QSA_ERR_UNSUPPORTED
    assert L.qsa_merge(0, 1, 1, 128, 16, 16, 16, 1, None, None) == qsa.QSA_ERR_UNSUPPORTED
    assert L.qsa_merge(2, 1, 1, 126, 16, 16, 16, 1, None, None) == qsa.QSA_ERR_INVALID_ARG
    assert L.qsa_sparse_decode(ctypes.byref(ok), ctypes.byref(c), 1, 16, 16, 16, 8, 0, 16, 16,
                               16, 1 << 20, None) == qsa.QSA_ERR_UNSUPPORTED
    assert L.qsa_append(ctypes.byref(ok), ctypes.byref(c), -1, 16, 16, 16, 16, 16, None) == \
        qsa.QSA_ERR_INVALID_ARG
    unaligned = qsa._Cache(17, 16, 16, 16, 16, 1, 1, 1)
    assert L.qsa_append(ctypes.byref(ok), ctypes.byref(unaligned), 1, 16, 16, 16, 16, 16,
                        None) == qsa.QSA_ERR_INVALID_ARG


def test_missing_library_fails_loudly(tmp_path):
    # no fallback: without libqsa.so every call raises instead of computing
    # anything on the host
    import subprocess
    import sys
    code = (
        "import sys; sys.path.insert(0, %r)\n"
        "from block_sparse_decode_b200 import qsa\n"
        "qsa.LIB_PATH = %r\n"
        "try:\n"
        "    qsa.qsa_version()\n"
        "except ImportError as e:\n"
        "    print('raised', 'missing' in str(e))\n"
    ) % (os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
         str(tmp_path / "libqsa.so"))
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == "raised True"
