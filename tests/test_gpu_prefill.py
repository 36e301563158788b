"""Sparse prefill on the GPU (through the C ABI) against the CPU oracle.

Every row of an appended chunk is the decode step of its sequence cut right
after the row's token: scores over that prefix, its own top-k, split
attention and merge. Each row is compared with the oracle's decode of the
cut sequence: scores within the fp32 bound, the selection set up to the
near-tie band, partials and merged output over the GPU's own selection.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from block_sparse_decode_b200 import qsa
from synth import make_custom, prefill_queries
from synth.workloads import DIMS_FULL, DIMS_TINY, Dims
from tests.gpu_harness import CudaRun
from tests.helpers import bits, check_attention, check_selection

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


def _row_score_tolerance(X, L, q_idx_row, w_row):
    kc = oracle.block_keys(bits(X), L)
    q = oracle.bf16_to_f32(bits(q_idx_row)).astype(np.float64)
    ww = w_row.detach().cpu().numpy().astype(np.float64)
    return (np.abs(kc) @ np.abs(q).T) @ np.abs(ww) * 2.0 ** -12 + 1e-30


def _check_rows(wl, chunks, rows_to_check, row_start, q, q_idx, w, buf, k, R):
    d = wl.dims
    row_seq, row_len = oracle.prefill_rows(wl.seq_lens, row_start.cpu().tolist())
    assert np.array_equal(buf.row_len.cpu().numpy(), row_len)
    scores = buf.scores.cpu().numpy()
    sel = buf.sel.cpu().numpy()
    o_part, lse_part = buf.o_part.cpu().numpy(), buf.lse_part.cpu().numpy()
    out, lse = buf.out.float().cpu().numpy(), buf.lse.cpu().numpy()
    for r in rows_to_check:
        s, ell = int(row_seq[r]), int(row_len[r])
        K, V, X = wl.seq_tokens(s, ell)
        ref = oracle.decode_sequence(bits(X), bits(K), bits(V), bits(q[r]), bits(q_idx[r]),
                                     w[r].cpu().numpy(), ell, k, R, d.scale, sel=sel[r])
        nb = (ell + 3) // 4
        tol = _row_score_tolerance(X, ell, q_idx[r], w[r])
        err = np.abs(scores[r, :nb] - ref["scores"])
        assert np.all(err <= tol), f"row {r}: score error {err.max():.3e} at {int(err.argmax())}"
        check_selection(sel[r], ref["sel"], ref["scores"], k, what=f"row {r}")
        check_attention(o_part[:, r], lse_part[:, r], ref["O_part"], ref["LSE_part"],
                        what=f"row {r} partials")
        # the merged bf16 output is held to the same bar as every other output
        check_attention(out[r], lse[r], ref["O"], ref["LSE"], what=f"row {r} merged")


@pytest.mark.parametrize("dims,lens,chunks,k,R", [
    # tiny heads (Hi = 4: 64 rows per group): a chunk of 70 rows spans two
    # groups, a sequence with no rows, a chunk that is the whole context
    # (rows of 1, 2, 3 tokens: only a partial block), k above some rows' blocks
    (DIMS_TINY, [1500, 777, 130], [70, 0, 130], 64, 2),
    # full heads (16 rows per group), ragged chunks, R = 4
    (DIMS_FULL, [9001, 2050, 40003], [37, 16, 20], 256, 4),
    # one row per sequence: the decode step itself
    (DIMS_FULL, [5000, 123, 65536], [1, 1, 1], 512, 1),
])
def test_sparse_prefill_matches_oracle(dims, lens, chunks, k, R):
    wl = make_custom(dims, lens, k=k, R=R, seed=500 + sum(chunks), device=DEV)
    run = CudaRun(wl, prefill=lens)  # every token, chunks included, appended
    d = run.dims
    row_start, q, q_idx, w = prefill_queries(wl, chunks)
    Nq = int(row_start[-1])
    buf = qsa.alloc_prefill(d, wl.B, Nq, qsa.ld_for(lens), k, R, device=DEV)
    for t in (buf.scores, buf.o_part, buf.lse_part):
        t.fill_(float("nan"))
    qsa.sparse_prefill(d, run.cache, run.seq_lens, row_start, q, q_idx, w, k, R, buf)
    assert qsa.qsa_check_device_errors() == 0
    _check_rows(wl, chunks, range(Nq), row_start, q, q_idx, w, buf, k, R)


def test_prefill_calls_one_by_one_equal_the_single_call():
    lens, chunks, k, R = [3001, 999], [40, 33], 128, 3
    wl = make_custom(DIMS_FULL, lens, k=k, R=R, seed=77, device=DEV)
    run = CudaRun(wl, prefill=lens)
    d = run.dims
    row_start, q, q_idx, w = prefill_queries(wl, chunks)
    Nq, S, ld = int(row_start[-1]), wl.B, qsa.ld_for(lens)
    buf = qsa.alloc_prefill(d, S, Nq, ld, k, R, device=DEV)
    qsa.sparse_prefill(d, run.cache, run.seq_lens, row_start, q, q_idx, w, k, R, buf)
    scores = torch.full((Nq, ld), float("nan"), device=DEV)
    row_len = torch.empty(Nq, dtype=torch.int32, device=DEV)
    ws1 = torch.empty(qsa.qsa_prefill_index_score_workspace_size(d, S, Nq), dtype=torch.uint8,
                      device=DEV)
    qsa.qsa_prefill_index_score(d, run.cache, run.seq_lens, row_start, q_idx, w, scores,
                                row_len, ws1)
    sel = torch.empty((Nq, k), dtype=torch.int32, device=DEV)
    qsa.qsa_topk_select(row_len, scores, k, sel)
    o = torch.empty((R, Nq, d.Hq, d.D), device=DEV)
    lse = torch.empty((R, Nq, d.Hq), device=DEV)
    ws2 = torch.empty(qsa.qsa_sparse_decode_workspace_size(d, Nq, k, R), dtype=torch.uint8,
                      device=DEV)
    qsa.qsa_prefill_sparse_decode(d, run.cache, run.seq_lens, row_start, q, sel, k, R, o, lse,
                                  ws2)
    assert qsa.qsa_check_device_errors() == 0
    assert torch.equal(row_len, buf.row_len)
    for r in range(Nq):  # the blocks each row owns are bitwise the same
        nb = (int(row_len[r]) + 3) // 4
        assert torch.equal(scores[r, :nb], buf.scores[r, :nb]), r
    assert torch.equal(sel, buf.sel)
    assert torch.equal(o, buf.o_part) and torch.equal(lse, buf.lse_part)


def test_prefill_last_rows_equal_the_decode_step():
    # a row at a sequence's last position is that sequence's decode step:
    # same bytes in, the decode kernels' scores, selection and output out
    lens, chunks, k, R = [20000, 4097, 333], [17, 3, 5], 512, 4
    wl = make_custom(DIMS_FULL, lens, k=k, R=R, seed=12, device=DEV)
    run = CudaRun(wl, prefill=lens)
    d = run.dims
    row_start, q, q_idx, w = prefill_queries(wl, chunks)
    Nq = int(row_start[-1])
    buf = qsa.alloc_prefill(d, wl.B, Nq, run.ld, k, R, device=DEV)
    qsa.sparse_prefill(d, run.cache, run.seq_lens, row_start, q, q_idx, w, k, R, buf)
    last = (row_start[1:] - 1).long()
    run.step(q=q[last].contiguous(), q_idx=q_idx[last].contiguous(), w=w[last].contiguous(),
             append=False)
    for b, L in enumerate(lens):
        nb = (L + 3) // 4
        r = int(last[b])
        # same MMA per (block, head) column and the same head order: same bits
        assert torch.equal(buf.scores[r, :nb], run.buf.scores[b, :nb]), b
        assert torch.equal(buf.sel[r], run.buf.sel[b]), b
        # the CTAs split a row's tiles differently from the decode's (other
        # running maxima, so other bf16 roundings of the probabilities before
        # the PV product): the two agree to the parity bar, not bitwise
        check_attention(buf.o_part[:, r].cpu().numpy(), buf.lse_part[:, r].cpu().numpy(),
                        run.buf.o_part[:, b].cpu().numpy(), run.buf.lse_part[:, b].cpu().numpy(),
                        what=f"sequence {b}")


def test_prefill_bad_layout_is_flagged_and_rows_left_empty():
    lens = [300, 200]
    wl = make_custom(DIMS_FULL, lens, k=64, R=1, seed=3, device=DEV)
    run = CudaRun(wl, prefill=lens)
    d = run.dims
    _, q, q_idx, w = prefill_queries(wl, [10, 5])
    # sequence 1's chunk claims 250 rows, more than its 200 tokens
    row_start = torch.tensor([0, 10, 260], dtype=torch.int32, device=DEV)
    Nq = 15
    scores = torch.zeros((Nq, run.ld), device=DEV)
    row_len = torch.full((Nq,), -5, dtype=torch.int32, device=DEV)
    ws = torch.empty(qsa.qsa_prefill_index_score_workspace_size(d, 2, Nq), dtype=torch.uint8,
                     device=DEV)
    qsa.qsa_prefill_index_score(d, run.cache, run.seq_lens, row_start, q_idx[:Nq], w[:Nq],
                                scores, row_len, ws)
    flags = 0
    try:
        qsa.qsa_check_device_errors()
    except qsa.QsaError as e:
        flags = int(str(e).split("flags=")[1].rstrip("]"))
    assert flags & 16
    rl = row_len.cpu().numpy()
    assert np.array_equal(rl[:10], 300 - 10 + np.arange(10) + 1)  # sequence 0 is fine
    assert np.all(rl[10:] == 0)                                  # rows of the bad chunk


def test_prefill_rejects_unsupported_and_bad_arguments():
    d4 = qsa.QsaDims(Hq=8, Hkv=2, D=128, Hi=12, di=64, P=64, scale=0.1)
    assert qsa.qsa_prefill_index_score_workspace_size(d4, 1, 8) == 0
    lens = [64]
    wl = make_custom(Dims(Hq=8, Hkv=2, D=128, Hi=12, di=64, P=64, scale=0.1), lens, k=8, R=1,
                     seed=1, device=DEV)
    run = CudaRun(wl, prefill=lens)
    row_start, q, q_idx, w = prefill_queries(wl, [4])
    scores = torch.empty((4, run.ld), device=DEV)
    row_len = torch.empty(4, dtype=torch.int32, device=DEV)
    ws = torch.empty(1024, dtype=torch.uint8, device=DEV)
    with pytest.raises(qsa.QsaError) as e:
        qsa.qsa_prefill_index_score(run.dims, run.cache, run.seq_lens, row_start, q_idx, w,
                                    scores, row_len, ws)
    assert e.value.status == qsa.QSA_ERR_UNSUPPORTED
    # a workspace below the stated size is refused on the host
    wl2 = make_custom(DIMS_FULL, [100], k=8, R=1, seed=2, device=DEV)
    run2 = CudaRun(wl2, prefill=[100])
    row_start, q, q_idx, w = prefill_queries(wl2, [4])
    need = qsa.qsa_prefill_index_score_workspace_size(run2.dims, 1, 4)
    small = torch.empty(need - 16, dtype=torch.uint8, device=DEV)
    with pytest.raises(qsa.QsaError) as e:
        qsa.qsa_prefill_index_score(run2.dims, run2.cache, run2.seq_lens, row_start, q_idx, w,
                                    torch.empty((4, run2.ld), device=DEV),
                                    torch.empty(4, dtype=torch.int32, device=DEV), small)
    assert e.value.status == qsa.QSA_ERR_INVALID_ARG


def test_prefill_256k_chunks_sampled_rows():
    # two 262,144-token sequences with a 128-row chunk each (the prefill
    # benchmark's shape): every row's length and, for sampled rows, scores,
    # selection and output against the oracle
    lens, chunks, k, R = [262144, 262144], [128, 128], 512, 4
    wl = make_custom(DIMS_FULL, lens, k=k, R=R, seed=2026, device=DEV, mixture=True)
    run = CudaRun(wl, prefill=lens)
    d = run.dims
    row_start, q, q_idx, w = prefill_queries(wl, chunks)
    Nq = int(row_start[-1])
    buf = qsa.alloc_prefill(d, wl.B, Nq, run.ld, k, R, device=DEV)
    qsa.sparse_prefill(d, run.cache, run.seq_lens, row_start, q, q_idx, w, k, R, buf)
    assert qsa.qsa_check_device_errors() == 0
    _check_rows(wl, chunks, [0, 15, 16, 127, 128, 200, 255], row_start, q, q_idx, w, buf, k, R)
