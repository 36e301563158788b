"""Failure detection on the GPU without a fault: a bounded wait that runs out.

The decode scoring kernel's roles wait on mbarriers with an iteration limit;
when a wait gives up, the kernel sets the TIMEOUT bit of the device error
word, stops every role, waits (bounded) for the copies and tensor-core work
it already issued and frees its tensor memory, so the context stays usable.
The environment variable QSA_DEBUG_STALL_SCORE=1 makes the producers issue
nothing, so the first data wait can never complete and gives up after a short
limit (a barrier nothing completes; no trap, assert or bad address). The test
checks that qsa_check_device_errors reports QSA_ERR_TIMEOUT and that a normal
decode step on the same context afterwards passes parity with the oracle.
"""

import pytest

from block_sparse_decode_b200 import qsa
from synth import make_custom
from synth.workloads import DIMS_FULL
from tests.gpu_harness import CudaRun
from tests.test_gpu_parity import _check_seq

pytestmark = pytest.mark.gpu


def test_scoring_wait_that_runs_out_is_reported_and_the_context_survives(monkeypatch):
    wl = make_custom(DIMS_FULL, [20000, 9001, 517], k=512, R=2, seed=404, device="cuda",
                     paged=True)
    run = CudaRun(wl)
    run.step()  # cache complete, a healthy context
    monkeypatch.setenv("QSA_DEBUG_STALL_SCORE", "1")
    qsa.qsa_index_score(run.dims, run.cache, run.seq_lens, wl.q_idx, wl.w, run.buf.scores)
    with pytest.raises(qsa.QsaError) as ei:
        qsa.qsa_check_device_errors()
    assert ei.value.status == qsa.QSA_ERR_TIMEOUT
    assert qsa.qsa_check_device_errors() == 0  # the flag was read and cleared
    monkeypatch.delenv("QSA_DEBUG_STALL_SCORE")
    run.step(append=False)  # the same context still runs the whole step
    for b in range(wl.B):
        _check_seq(run, b)


def test_stalled_scoring_inside_a_decode_step(monkeypatch):
    """The same failure inside qsa_decode_step (append, then the stalled
    scoring chained to it): every role gives up, the kernel drains and frees
    TMEM, the later kernels of the step run on whatever the scores hold (no
    fault), TIMEOUT is reported, and the next step passes parity."""
    wl = make_custom(DIMS_FULL, [70001, 9001, 517, 40000], k=512, R=2, seed=405,
                     device="cuda", paged=True)
    run = CudaRun(wl)
    monkeypatch.setenv("QSA_DEBUG_STALL_SCORE", "1")
    qsa.decode_step(run.dims, run.cache, run.seq_lens, wl.q, wl.q_idx, wl.w, run.k, run.R,
                    run.buf, append=run.current_tokens())
    with pytest.raises(qsa.QsaError) as ei:
        qsa.qsa_check_device_errors()
    assert ei.value.status == qsa.QSA_ERR_TIMEOUT
    monkeypatch.delenv("QSA_DEBUG_STALL_SCORE")
    run.step()
    for b in range(wl.B):
        _check_seq(run, b)
