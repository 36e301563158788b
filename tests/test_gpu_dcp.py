"""Decode context parallelism end to end: dcp.dcp_decode_step on two ranks.

Two spawned processes share cuda:0 and form a gloo group (the exchange goes
through host memory; no kernel of one rank waits on the other). Each rank
scores and selects on the replicated side cache, keeps the selected blocks of
the pages it holds (page p on rank p mod 2), reads them through a K/V cache
that holds only its own pages (the others unmapped), gathers both partials
and merges them. Every rank's merged output must equal the oracle's attention
over the whole selection, within the parity bar, and the two ranks' outputs
must be the same bits. The step runs on a non-default stream, so the
collective's ordering against the library's launches is exercised.
"""

import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu

LENS = [5000, 20001, 3001, 777]
K_SEL = 256


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _own_kv_cache(qsa, dims, cache, W, r):
    """A cache whose K/V pools hold only rank r's pages (page column j of a
    sequence on rank j mod W), packed; other columns map to -1."""
    bt = cache.block_table.cpu()
    B, maxp = bt.shape
    bt_kv = torch.full_like(bt, -1)
    src = []
    for b in range(B):
        for j in range(r, maxp, W):
            if bt[b, j] >= 0:
                bt_kv[b, j] = len(src)
                src.append(int(bt[b, j]))
    idx = torch.tensor(src, dtype=torch.long, device=cache.k_pool.device)
    return qsa.QsaCache(k_pool=cache.k_pool[idx].contiguous(),
                        v_pool=cache.v_pool[idx].contiguous(),
                        kidx_pool=cache.kidx_pool[:1], side_pool=cache.side_pool[:1],
                        block_table=bt_kv.to(cache.k_pool.device))


def _worker(rank, world, port, out_q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch.distributed as dist
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        from block_sparse_decode_b200 import dcp, qsa
        from synth import make_custom
        from synth.workloads import DIMS_FULL
        from tests.gpu_harness import CudaRun, oracle_sequence
        from tests.helpers import check_attention, check_selection

        wl = make_custom(DIMS_FULL, LENS, k=K_SEL, R=1, seed=303, device="cuda", paged=True)
        run = CudaRun(wl, prefill=list(wl.seq_lens))  # every token already appended
        kv = _own_kv_cache(qsa, run.dims, run.cache, world, rank)
        buf = dcp.alloc_dcp(run.dims, wl.B, run.ld, K_SEL, device="cuda")
        stream = torch.cuda.Stream()
        dcp.dcp_decode_step(run.dims, run.cache, run.seq_lens, wl.q, wl.q_idx, wl.w, K_SEL, buf,
                            stream=stream, kv_cache=kv)
        stream.synchronize()
        flags = qsa.qsa_check_device_errors(stream)
        sel = buf.step.sel.cpu().numpy()
        out = buf.step.out.float().cpu().numpy()
        lse = buf.step.lse.cpu().numpy()
        worst = []
        for b in range(wl.B):
            ref_sel = oracle_sequence(wl, b, k=K_SEL, R=1)
            check_selection(sel[b], ref_sel["sel"], ref_sel["scores"], K_SEL, what=f"sel b={b}")
            ref = oracle_sequence(wl, b, k=K_SEL, R=1, sel=sel[b])
            worst.append(check_attention(out[b], lse[b], ref["O"], ref["LSE"],
                                         what=f"rank {rank} b={b}"))
        out_q.put((rank, flags, worst, out, lse, None))
    except Exception as e:  # reported to the parent, which fails the test
        out_q.put((rank, -1, None, None, None, repr(e)))
    finally:
        dist.destroy_process_group()


def test_dcp_step_two_ranks_matches_oracle():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    try:
        results = sorted((q.get(timeout=600) for _ in range(world)), key=lambda x: x[0])
    finally:
        for p in procs:
            p.join(timeout=120)
            if p.exitcode is None:
                p.kill()
    for rank, flags, worst, out, lse, err in results:
        assert err is None, f"rank {rank}: {err}"
        assert flags == 0, (rank, flags)
    # both ranks merged the same gathered partials with the same kernel
    assert np.array_equal(results[0][3], results[1][3])
    assert np.array_equal(results[0][4], results[1][4])
    for p in procs:
        assert p.exitcode == 0
