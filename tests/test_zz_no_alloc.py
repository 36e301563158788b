"""qsa_sparse_decode_static: the decode call for callers that cannot
allocate device memory (a plain C host holding only the buffers it was
handed, a process whose device memory belongs to another allocator's pool, a
latency-critical loop where cudaMalloc / cudaFree may synchronise the
device). Its scratch is a fixed array inside the library, so it takes no
workspace argument. This checks, through the C ABI, that two calls in a row
give the same partial outputs as qsa_sparse_decode with a caller workspace:
the same kernels on the same inputs, so the same bits (which is inside the
attention tolerance of the other parity tests).

The file name makes pytest collect it last, so a run that stops at the first
failure has already run every other test.
"""

import numpy as np
import pytest
import torch

from block_sparse_decode_b200 import qsa
from synth import make_custom
from synth.workloads import DIMS_FULL
from tests.gpu_harness import CudaRun
from tests.helpers import check_attention

pytestmark = pytest.mark.gpu


def _workspace_decode(run, wl):
    """The regular entry point with a caller workspace, on the step's selection."""
    o = torch.full_like(run.buf.o_part, float("nan"))
    l = torch.full_like(run.buf.lse_part, float("nan"))
    qsa.qsa_sparse_decode(run.dims, run.cache, run.seq_lens, wl.q, run.buf.sel, wl.k, wl.R, o, l,
                          run.buf.ws)
    assert qsa.qsa_check_device_errors() == 0
    return o, l


def _same(o, l, ref_o, ref_l, what):
    assert torch.equal(o, ref_o), f"{what}: partial outputs differ from the workspace call"
    assert torch.equal(l, ref_l), f"{what}: LSEs differ from the workspace call"
    for b in range(o.shape[1]):  # and so inside the parity bar
        check_attention(o[:, b].cpu().numpy(), l[:, b].cpu().numpy(),
                        ref_o[:, b].cpu().numpy(), ref_l[:, b].cpu().numpy(), what=f"{what} b={b}")


def test_static_scratch_decode_matches_workspace_decode():
    lens = [5000, 20001, 3, 2051, 40000, 777]
    wl = make_custom(DIMS_FULL, lens, k=512, R=4, seed=201, device="cuda", paged=True)
    run = CudaRun(wl)
    run.step()  # cache complete, selection in run.buf.sel
    need = qsa.qsa_sparse_decode_workspace_size(run.dims, wl.B, wl.k, wl.R)
    assert need <= (32 << 20)
    ref_o, ref_l = _workspace_decode(run, wl)
    for _ in range(2):  # two calls in a row share the one static array
        o = torch.full_like(ref_o, float("nan"))
        l = torch.full_like(ref_l, float("nan"))
        qsa.qsa_sparse_decode_static(run.dims, run.cache, run.seq_lens, wl.q, run.buf.sel, wl.k,
                                     wl.R, o, l)
        assert qsa.qsa_check_device_errors() == 0
        _same(o, l, ref_o, ref_l, "static scratch")


def test_static_scratch_serves_the_largest_k_and_R():
    # k = 4096 and R = 64, the largest the call accepts, at a small batch: the
    # scratch need fits the static array, and the result equals the regular
    # entry point's
    d = qsa.QsaDims.of(DIMS_FULL)
    need = qsa.qsa_sparse_decode_workspace_size(d, 2, 4096, 64)
    assert need <= (32 << 20)
    wl = make_custom(DIMS_FULL, [20000, 16390], k=4096, R=64, seed=202, device="cuda",
                     paged=True)
    run = CudaRun(wl)
    run.step()
    ref_o, ref_l = _workspace_decode(run, wl)
    for _ in range(2):
        o = torch.full_like(ref_o, float("nan"))
        l = torch.full_like(ref_l, float("nan"))
        qsa.qsa_sparse_decode_static(run.dims, run.cache, run.seq_lens, wl.q, run.buf.sel, wl.k,
                                     wl.R, o, l)
        assert qsa.qsa_check_device_errors() == 0
        _same(o, l, ref_o, ref_l, "static scratch k=4096 R=64")


def test_static_scratch_rejects_oversized_calls():
    # B = 4096 sequences at k = 4096, R = 64 needs far more than the static array
    need = qsa.qsa_sparse_decode_workspace_size(qsa.QsaDims.of(DIMS_FULL), 4096, 4096, 64)
    assert need > (32 << 20)
    d = qsa.QsaDims.of(DIMS_FULL)
    bt = torch.zeros((4096, 1), dtype=torch.int32, device="cuda")
    cache = qsa.alloc_cache(d, 1, bt, device="cuda")
    sl = torch.ones(4096, dtype=torch.int32, device="cuda")
    q = torch.zeros((4096, d.Hq, d.D), dtype=torch.bfloat16, device="cuda")
    sel = torch.zeros((4096, 4096), dtype=torch.int32, device="cuda")
    o = torch.empty((1,), dtype=torch.float32, device="cuda")
    with pytest.raises(qsa.QsaError) as ei:
        qsa.qsa_sparse_decode_static(d, cache, sl, q, sel, 4096, 64, o, o)
    assert ei.value.status == qsa.QSA_ERR_UNSUPPORTED
    assert "static scratch" in str(ei.value)
