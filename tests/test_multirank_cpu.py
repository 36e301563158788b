"""Host logic of bench.py's multi-GPU (replica) mode, on CPU with gloo.

The decode step shards by sequence with no exchange: each rank runs its own
replica and the only collective is the max of the timed totals. These tests
run two gloo ranks on CPU and check that every rank sees the slowest rank's
time, that the replicas draw different batches, that the reported rate counts
the work of all ranks, and that the reference arm runs on rank 0 alone.
"""

import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        # rank r "took" 10 + 5r ms in total; everyone must see the slowest
        slowest = bench.max_over_ranks(10.0 + 5.0 * rank, torch.device("cpu"))
        seed = bench.replica_seed("b8x256k", rank)
        seeds = [None] * world
        dist.all_gather_object(seeds, seed)
        out_q.put((rank, slowest, seeds))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_and_draw_distinct_batches():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, slowest, seeds in results:
        assert slowest == 10.0 + 5.0 * (world - 1)
        assert len(set(seeds)) == world  # each replica its own batch


def _dcp_worker(rank, world, port, out_q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        import numpy as np
        import oracle
        from block_sparse_decode_b200 import dcp
        from synth import make_custom
        from synth.workloads import Dims
        from tests.helpers import bits
        d = Dims(Hq=8, Hkv=2, D=32, Hi=4, di=32, P=16, scale=0.2)
        wl = make_custom(d, [2001, 517], k=48, R=1, seed=77, paged=False)
        O_r, L_r, full = [], [], []
        for b, L in enumerate(wl.seq_lens):
            K, V, X = wl.seq_tokens(b)
            sel = oracle.topk_blocks(oracle.index_scores(oracle.block_keys(bits(X), L),
                                                         bits(wl.q_idx[b]), wl.w[b].numpy()), 48)
            args = (bits(wl.q[b]), bits(K), bits(V))
            o, l = oracle.attend_slices(*args, oracle.owned_blocks(sel, d.P, world, rank), L,
                                        d.scale, 1)
            O_r.append(o[0])
            L_r.append(l[0])
            full.append(oracle.attend_slices(*args, sel, L, d.scale, 1))
        # the product's exchange step, on CPU tensors over gloo
        O, Ls = dcp.exchange_partials(torch.from_numpy(np.stack(O_r)),
                                      torch.from_numpy(np.stack(L_r)))
        worst = 0.0
        for b in range(len(wl.seq_lens)):
            Om, Lm = oracle.merge_partials(O[:, b].numpy(), Ls[:, b].numpy())
            worst = max(worst, float(np.abs(Om - full[b][0][0]).max()),
                        float(np.abs(Lm - full[b][1][0]).max()))
        out_q.put((rank, tuple(O.shape), worst))
    finally:
        dist.destroy_process_group()


def test_context_parallel_exchange_over_two_gloo_ranks():
    # each rank holds the partial over its own pages' share of the selection;
    # the gathered, merged partials equal the attention over the whole
    # selection on every rank
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_dcp_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=180) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, shape, worst in results:
        assert shape == (world, 2, 8, 32)
        assert worst <= 1e-12, (rank, worst)


def test_single_process_max_is_identity():
    assert not dist.is_initialized()
    assert bench.max_over_ranks(3.25, torch.device("cpu")) == 3.25


def test_job_rate_counts_all_ranks():
    # 8 sequences per rank, 0.1 ms per step, 4 ranks -> 320,000 seqs/s
    assert bench.job_rate(4, 8, 0.1) == pytest.approx(320000.0)
    assert bench.job_rate(1, 8, 0.1) == pytest.approx(80000.0)


def _run_reference_arm(rank, world):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
               OMP_NUM_THREADS="2")
    return subprocess.run(
        [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
         "--workload", "b32x32k", "--steps", "1", "--warmup", "0"],
        env=env, capture_output=True, text=True, timeout=300)


def test_reference_arm_other_ranks_exit_quietly():
    r = _run_reference_arm(1, 2)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


@pytest.mark.slow
def test_reference_arm_rank0_prints_one_line():
    r = _run_reference_arm(0, 2)
    assert r.returncode == 0, r.stderr
    lines = [x for x in r.stdout.splitlines() if x.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["value"] > 0
