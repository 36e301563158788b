#!/usr/bin/env python
"""Benchmark of the QSA decode step on B200.

One step = the whole hot path on one batch: qsa_append (the current token of
every sequence) -> qsa_index_score -> qsa_topk_select -> qsa_sparse_decode
(R-way split) -> qsa_merge, on seeded synthetic inputs already resident in
HBM. Default workload: B=8 sequences x 262,144 tokens, 32 query / 4 KV heads,
head dim 128, indexer 16 x 128, top-512 blocks, R=4, paged (P=64, shuffled).

The step is captured once in a CUDA graph and replayed; L2 is flushed (a
write larger than L2) before every timed step, outside the step's events.
Prints one JSON line (rank 0). ``--impl reference`` times the CPU oracle on
the same workload instead (a bounded sample per step).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload b8x256k]
    torchrun --nproc-per-node N bench.py --gpus N ...   (replicas, weak scaling)
"""

from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "QSA decode seqs/s & attended tokens/s at 256K ctx; HBM GB/s as % of roofline"
L2_FLUSH_BYTES = 512 << 20
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="b8x256k",
                    choices=["b32x32k", "b8x256k", "ragged64", "steady128x64k"])
    ap.add_argument("--batch", type=int, default=None,
                    help="override the batch size (smaller profiling case)")
    ap.add_argument("--k", type=int, default=None)
    ap.add_argument("--R", type=int, default=None)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the other workloads (b32x32k, steady128x64k k-sweep, "
                         "ragged64 R-sweep) timed after the headline step")
    ap.add_argument("--dcp-world", type=int, default=0,
                    help="also time, on this GPU, rank 0's share of a decode-context-parallel "
                         "step over this many ranks (page p on rank p mod W)")
    ap.add_argument("--prefill-rows", type=int, default=32,
                    help="also time a sparse prefill of each sequence's this many newest "
                         "tokens (one query row per token) on the step's cache; 0: skip")
    ap.add_argument("--queries", type=int, default=1,
                    help="decode queries per sequence (multi-query decode: each step appends "
                         "this many tokens per sequence and decodes all of them)")
    return ap.parse_args()


# ----------------------------------------------------------------- helpers

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def load_tensor_peak():
    """Dense bf16 TFLOP/s (burst: a kernel timed alone) and its source."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        if "bf16_tflops" in d:
            return float(d["bf16_tflops"]), "measured"
    return FALLBACK_BF16_TFLOPS, "fallback"


def profile_traffic(kernel_src: str, summary: str):
    """Per-launch DRAM bytes of a kernel from a committed ncu summary, if the
    summary was taken on the current source of that kernel (else None)."""
    path = os.path.join(ROOT, "profiles", summary)
    src = os.path.join(ROOT, "block_sparse_decode_b200", "csrc", kernel_src)
    if not (os.path.exists(path) and os.path.exists(src)):
        return None
    text = open(path).read()
    m_sha = re.search(r"source_sha256:\s*([0-9a-f]{64})", text)
    m_b = re.search(r"dram_bytes_per_full_launch:\s*([0-9.eE+]+)", text)
    if not (m_sha and m_b):
        return None
    if hashlib.sha256(open(src, "rb").read()).hexdigest() != m_sha.group(1):
        return None
    return float(m_b.group(1))


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled while running."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.out = ""
        if self.proc is not None:
            time.sleep(0.06)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self):
        rows = []
        for line in (self.out or "").strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                rows.append((float(parts[0]), float(parts[1]), parts[4:8]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({n for _, _, flags in rows for n, f in zip(names, flags)
                          if f.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows),
                "sm_max_mhz": max(r[1] for r in rows), "reasons": reasons,
                "samples": len(rows)}


def replica_seed(preset: str, rank: int) -> int:
    """Seed of the replica on ``rank``: every GPU draws its own batch."""
    from synth import seed_for
    return seed_for(preset) + 7919 * rank


def max_over_ranks(x: float, device) -> float:
    """The largest ``x`` over all ranks (the job is as slow as its slowest
    replica); the identity on a single process."""
    t = torch.tensor([x], dtype=torch.float64, device=device)
    if torch.distributed.is_initialized() and torch.distributed.get_world_size() > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_rate(world: int, units_per_rank: int, ms_per_step: float) -> float:
    """Whole-job throughput: units processed by all ranks per second."""
    return world * units_per_rank / (ms_per_step / 1e3)


def algorithmic_bytes(seq_lens, dims, k):
    side = sum(((L + 3) // 4) * dims.di * 2 for L in seq_lens)
    kv = sum(min(4 * k, L) * dims.Hkv * dims.D * 2 * 2 for L in seq_lens)
    return side, kv


def kernel_nodes(graph) -> int | None:
    """Kernel nodes of a captured CUDA graph (None if the graph is not kept)."""
    try:
        import cuda.bindings.runtime as rt
        raw = graph.raw_cuda_graph()
        err, _, n = rt.cudaGraphGetNodes(raw, 0)
        err, nodes, n = rt.cudaGraphGetNodes(raw, n)
        if int(err) != 0:
            return None
        kern = 0
        for nd in nodes:
            e, t = rt.cudaGraphNodeGetType(nd)
            if int(e) == 0 and t == rt.cudaGraphNodeType.cudaGraphNodeTypeKernel:
                kern += 1
        return kern
    except Exception:
        return None


class GraphTimer:
    """CUDA graphs of library calls, replayed after an L2 flush and timed with
    CUDA events on the launching stream."""

    def __init__(self, dev, stream):
        self.dev, self.stream = dev, stream
        # write a buffer larger than L2, then read another one: the timed
        # launch starts with a cold L2 that holds no dirty lines (otherwise the
        # flush's own write-backs would be billed to the first kernels)
        self.flush_w = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
        self.flush_r = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
        self.flush_o = torch.empty((), dtype=torch.float32, device=dev)
        self.e0 = torch.cuda.Event(enable_timing=True)
        self.e1 = torch.cuda.Event(enable_timing=True)

    def capture(self, fn):
        try:
            g = torch.cuda.CUDAGraph(keep_graph=True)
        except TypeError:
            g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=self.stream):
            fn()
        return g

    def flush(self):
        self.flush_w.zero_()
        torch.sum(self.flush_r, dim=0, out=self.flush_o)

    def timed(self, g) -> float:
        with torch.cuda.stream(self.stream):
            self.flush()
            self.e0.record()
            g.replay()
            self.e1.record()
        self.e1.synchronize()
        return self.e0.elapsed_time(self.e1)

    def mean_ms(self, g, n: int, warm: int = 3) -> float:
        for _ in range(warm):
            self.timed(g)
        return statistics.mean(self.timed(g) for _ in range(n))


def prepare_batch(qsa, dims_spec, lens, k, R, seed, dev, spec, name, Qn=1):
    """Draw a workload, fill its paged cache with every token but the step's
    Qn newest (one bulk qsa_append) and allocate the step's buffers. Returns
    (wl, dims, cache, step inputs, buffers)."""
    from synth import make_custom
    wl = make_custom(dims_spec, lens, k=k, R=R, seed=seed, device=dev, paged=spec["paged"],
                     needles=spec["needles"], mixture=spec["mixture"], name=name)
    dims = qsa.QsaDims.of(wl.dims)
    B = wl.B
    cache = qsa.alloc_cache(dims, wl.num_pages, wl.block_table, device=dev)
    T = sum(wl.cap_lens)
    tok_seq = torch.empty(T, dtype=torch.int32, device=dev)
    tok_pos = torch.empty(T, dtype=torch.int32, device=dev)
    for b, L in enumerate(wl.cap_lens):
        o = wl.tok_off[b]
        tok_seq[o:o + L] = b
        tok_pos[o:o + L] = torch.arange(L, dtype=torch.int32, device=dev)
        tok_seq[o + wl.seq_lens[b] - Qn:o + L] = -1
    qsa.qsa_append(dims, cache, tok_seq, tok_pos, wl.k_tok, wl.v_tok, wl.kidx_tok)
    del tok_seq, tok_pos
    rows = torch.tensor([wl.tok_off[b] + L - Qn + j for b, L in enumerate(wl.seq_lens)
                         for j in range(Qn)], device=dev)
    if Qn == 1:
        q_step = wl.q.contiguous()
    else:  # one decode query per new token
        gq = torch.Generator(device=dev).manual_seed(seed + 17)
        q_step = torch.randn((B, Qn, wl.dims.Hq, wl.dims.D), generator=gq,
                             device=dev).to(torch.bfloat16)
    step_in = dict(
        tok_seq=torch.arange(B, dtype=torch.int32, device=dev).repeat_interleave(Qn),
        tok_pos=torch.tensor([L - Qn + j for L in wl.seq_lens for j in range(Qn)],
                             dtype=torch.int32, device=dev),
        k_new=wl.k_tok[rows].contiguous(), v_new=wl.v_tok[rows].contiguous(),
        kidx_new=wl.kidx_tok[rows].contiguous(),
        seq_lens=torch.tensor(wl.seq_lens, dtype=torch.int32, device=dev),
        q=q_step, q_idx=wl.q_idx.contiguous(), w=wl.w.contiguous())
    buf = qsa.alloc_step(dims, B, qsa.ld_for(wl.seq_lens), k, R, device=dev)
    return wl, dims, cache, step_in, buf


def time_batch(qsa, timer, dims, cache, si, buf, k, R, n_rep):
    """The one-call step and the calls of the step, each in its own graph;
    also index score + sparse decode back to back in one graph. Returns
    ({name: mean us}, kernel nodes of the step graph)."""
    app = (si["tok_seq"], si["tok_pos"], si["k_new"], si["v_new"], si["kidx_new"])
    step_buf = qsa.StepBuffers(scores=buf.scores, sel=buf.sel, o_part=buf.o_part,
                               lse_part=buf.lse_part, out=buf.out, lse=buf.lse, ws=buf.ws)

    def step():
        qsa.decode_step(dims, cache, si["seq_lens"], si["q"], si["q_idx"], si["w"], k, R,
                        step_buf, append=app)

    def score():
        qsa.qsa_index_score(dims, cache, si["seq_lens"], si["q_idx"], si["w"], buf.scores)

    def decode():
        qsa.qsa_sparse_decode(dims, cache, si["seq_lens"], si["q"], buf.sel, k, R, buf.o_part,
                              buf.lse_part, buf.ws)

    calls = {"step": step, "index_score": score,
             "topk_select": lambda: qsa.qsa_topk_select(si["seq_lens"], buf.scores, k, buf.sel),
             "sparse_decode": decode,
             "score_then_decode": lambda: (score(), decode())}
    with torch.cuda.stream(timer.stream):
        for _ in range(2):
            step()
    torch.cuda.synchronize(timer.dev)
    qsa.qsa_check_device_errors()
    graphs = {n: timer.capture(fn) for n, fn in calls.items()}
    nodes = kernel_nodes(graphs["step"])
    us = {n: 1e3 * timer.mean_ms(g, n_rep) for n, g in graphs.items()}
    qsa.qsa_check_device_errors()
    for g in graphs.values():
        g.reset()
    return us, nodes


def config_line(name, lens, dims, k, R, us, peak):
    side_b, kv_b = algorithmic_bytes(lens, dims, k)
    pair = us["index_score"] + us["sparse_decode"]
    return {
        "workload": name, "batch": len(lens), "k": k, "R": R,
        "step_us": us["step"], "seqs_per_s": len(lens) / (us["step"] * 1e-6),
        "attended_tokens_per_s": sum(min(4 * k, L) for L in lens) / (us["step"] * 1e-6),
        "kernels_us": {n: us[n] for n in ("index_score", "topk_select", "sparse_decode")},
        "bytes": {"side_cache": side_b, "selected_kv": kv_b},
        "index_score_frac": side_b / (us["index_score"] * 1e-6) / 1e9 / peak,
        "sparse_decode_frac": kv_b / (us["sparse_decode"] * 1e-6) / 1e9 / peak,
        "score_plus_decode_frac": (side_b + kv_b) / (pair * 1e-6) / 1e9 / peak,
        "score_then_decode_one_graph_us": us["score_then_decode"],
        "score_then_decode_one_graph_frac":
            (side_b + kv_b) / (us["score_then_decode"] * 1e-6) / 1e9 / peak,
        "step_frac": (side_b + kv_b) / (us["step"] * 1e-6) / 1e9 / peak,
    }


def time_configs(args, qsa, timer, dev, peak):
    """The other workloads of the scope, each at its full size: b32x32k,
    steady128x64k (one step at L = 65,537, k in {256, 512, 1024}) and ragged64
    (R in {1, 2, 4, 8}); same graphs, flush and events as the headline."""
    from synth import preset_spec, seed_for
    out = {}
    n_rep = max(10, min(args.steps, 50))
    plan = [("b32x32k", None, [(512, 1)]),
            ("steady128x64k", [65537] * 128, [(256, 4), (512, 4), (1024, 4)]),
            ("ragged64", None, [(512, 1), (512, 2), (512, 4), (512, 8)])]
    for name, lens, kr in plan:
        spec = preset_spec(name)
        lens = lens or list(spec["seq_lens"])
        k0, R0 = kr[0]
        wl, dims, cache, si, buf = prepare_batch(qsa, spec["dims"], lens, k0, R0,
                                                 seed_for(name), dev, spec, name)
        del wl.k_tok, wl.v_tok, wl.kidx_tok
        for k, R in kr:
            buf = qsa.alloc_step(dims, len(lens), qsa.ld_for(lens), k, R, device=dev)
            us, _ = time_batch(qsa, timer, dims, cache, si, buf, k, R, n_rep)
            out[f"{name}_k{k}_R{R}"] = config_line(name, lens, dims, k, R, us, peak)
            del buf
        del wl, cache, si
        torch.cuda.empty_cache()
    return out


# ------------------------------------------------------------ our arm

def run_ours(args, rank, world, local_rank):
    from block_sparse_decode_b200 import qsa
    from synth import make_custom, preset_spec, seed_for

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    spec = preset_spec(args.workload)
    k = args.k or spec["k"]
    R = args.R or spec["R"]
    lens = list(spec["seq_lens"])
    if args.batch:
        lens = (lens * ((args.batch + len(lens) - 1) // len(lens)))[:args.batch]
    if args.workload == "steady128x64k":
        lens = [spec["prefill"] + 1] * len(lens)
    seed = replica_seed(args.workload, rank)
    wl = make_custom(spec["dims"], lens, k=k, R=R, seed=seed, device=dev,
                     paged=spec["paged"], needles=spec["needles"], mixture=spec["mixture"],
                     name=args.workload)
    dims = qsa.QsaDims.of(wl.dims)
    B = wl.B

    Qn = args.queries
    # cache: prefill L - Qn tokens in bulk; the step appends tokens L - Qn .. L - 1
    cache = qsa.alloc_cache(dims, wl.num_pages, wl.block_table, device=dev)
    T = sum(wl.cap_lens)
    tok_seq = torch.empty(T, dtype=torch.int32, device=dev)
    tok_pos = torch.empty(T, dtype=torch.int32, device=dev)
    for b, L in enumerate(wl.cap_lens):
        o = wl.tok_off[b]
        tok_seq[o:o + L] = b
        tok_pos[o:o + L] = torch.arange(L, dtype=torch.int32, device=dev)
        tok_seq[o + wl.seq_lens[b] - Qn:o + L] = -1
    qsa.qsa_append(dims, cache, tok_seq, tok_pos, wl.k_tok, wl.v_tok, wl.kidx_tok)
    del tok_seq, tok_pos
    rows = torch.tensor([wl.tok_off[b] + L - Qn + j for b, L in enumerate(wl.seq_lens)
                         for j in range(Qn)], device=dev)
    if Qn == 1:
        q_step = wl.q.contiguous()
    else:  # one decode query per new token
        gq = torch.Generator(device=dev).manual_seed(seed + 17)
        q_step = torch.randn((B, Qn, wl.dims.Hq, wl.dims.D), generator=gq,
                             device=dev).to(torch.bfloat16)
    step_in = dict(
        tok_seq=torch.arange(B, dtype=torch.int32, device=dev).repeat_interleave(Qn),
        tok_pos=torch.tensor([L - Qn + j for L in wl.seq_lens for j in range(Qn)],
                             dtype=torch.int32, device=dev),
        k_new=wl.k_tok[rows].contiguous(), v_new=wl.v_tok[rows].contiguous(),
        kidx_new=wl.kidx_tok[rows].contiguous(),
        seq_lens=torch.tensor(wl.seq_lens, dtype=torch.int32, device=dev),
        q=q_step, q_idx=wl.q_idx.contiguous(), w=wl.w.contiguous())
    ld = qsa.ld_for(wl.seq_lens)
    buf = qsa.alloc_step(dims, B, ld, k, R, device=dev)
    if Qn > 1:  # partials, merged output and scratch with a query axis
        buf.o_part = torch.empty((R, B, Qn, dims.Hq, dims.D), dtype=torch.float32, device=dev)
        buf.lse_part = torch.empty((R, B, Qn, dims.Hq), dtype=torch.float32, device=dev)
        buf.out = torch.empty((B * Qn, dims.Hq, dims.D), dtype=torch.bfloat16, device=dev)
        buf.lse = torch.empty((B * Qn, dims.Hq), dtype=torch.float32, device=dev)
        buf.ws = torch.empty(max(16, qsa.qsa_sparse_decode_mq_workspace_size(dims, B, Qn, k, R)),
                             dtype=torch.uint8, device=dev)
    qsa.qsa_check_device_errors()

    # host-side copies for the oracle baseline (seq 0), then free the token arrays
    cpu_sample = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and Qn == 1:
        K0, V0, X0 = wl.seq_tokens(0)
        cpu_sample = dict(K=K0.cpu(), V=V0.cpu(), X=X0.cpu(), q=wl.q[0].cpu(),
                          q_idx=wl.q_idx[0].cpu(), w=wl.w[0].cpu(), L=wl.seq_lens[0])
    del wl.k_tok, wl.v_tok, wl.kidx_tok
    torch.cuda.empty_cache()

    stream = torch.cuda.Stream(device=dev)
    si = step_in
    calls = {
        "append": lambda: qsa.qsa_append(dims, cache, si["tok_seq"], si["tok_pos"], si["k_new"],
                                         si["v_new"], si["kidx_new"]),
        "index_score": lambda: qsa.qsa_index_score(dims, cache, si["seq_lens"], si["q_idx"],
                                                   si["w"], buf.scores),
        "topk_select": lambda: qsa.qsa_topk_select(si["seq_lens"], buf.scores, k, buf.sel),
        "sparse_decode": (lambda: qsa.qsa_sparse_decode(dims, cache, si["seq_lens"], si["q"],
                                                        buf.sel, k, R, buf.o_part, buf.lse_part,
                                                        buf.ws)) if Qn == 1 else
                         (lambda: qsa.qsa_sparse_decode_mq(dims, cache, si["seq_lens"], si["q"],
                                                           buf.sel, k, R, buf.o_part,
                                                           buf.lse_part, buf.ws)),
        "merge": lambda: qsa.qsa_merge(buf.o_part.view(R, B * Qn, dims.Hq, dims.D),
                                       buf.lse_part.view(R, B * Qn, dims.Hq), buf.out, buf.lse),
    }

    if Qn == 1:
        # the user's one-call step (append, score, top-k, decode with the
        # merge fused into its last kernel)
        step_buf = qsa.StepBuffers(scores=buf.scores, sel=buf.sel, o_part=buf.o_part,
                                   lse_part=buf.lse_part, out=buf.out, lse=buf.lse, ws=buf.ws)
        step_app = (si["tok_seq"], si["tok_pos"], si["k_new"], si["v_new"], si["kidx_new"])

        def step():
            qsa.decode_step(dims, cache, si["seq_lens"], si["q"], si["q_idx"], si["w"], k, R,
                            step_buf, append=step_app)
    else:
        def step():
            for fn in calls.values():
                fn()

    with torch.cuda.stream(stream):
        for _ in range(3):  # eager warm-up (module load, attributes)
            step()
    torch.cuda.synchronize(dev)
    qsa.qsa_check_device_errors()

    def capture(fn):
        try:  # keep the graph so that its kernel nodes can be counted
            g = torch.cuda.CUDAGraph(keep_graph=True)
        except TypeError:
            g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            fn()
        return g

    graph = capture(step)
    step_kernels = kernel_nodes(graph)
    kgraphs = {n: capture(fn) for n, fn in calls.items()}
    if Qn == 1:  # the two HBM-bound calls back to back, one launch of the pair
        kgraphs["score_then_decode"] = capture(lambda: (calls["index_score"](),
                                                        calls["sparse_decode"]()))
    # L2 flush: write a buffer larger than L2, then read another one, so the
    # timed step starts with a cold L2 that holds no dirty lines (otherwise
    # the flush's own write-backs would be billed to the first kernels)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flush_rd = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    flush_out = torch.empty((), dtype=torch.float32, device=dev)

    def do_flush():
        flush.zero_()
        torch.sum(flush_rd, dim=0, out=flush_out)

    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def timed(g):
        with torch.cuda.stream(stream):
            do_flush()
            s0.record()
            g.replay()
            s1.record()
        s1.synchronize()
        return s0.elapsed_time(s1)

    for _ in range(max(3, args.warmup)):
        timed(graph)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    step_ms = []
    with ClockSampler(local_rank) as clk:
        for _ in range(args.steps):
            step_ms.append(timed(graph))
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    qsa.qsa_check_device_errors()

    ms_per_step = max_over_ranks(sum(step_ms), dev) / args.steps

    # per-kernel durations: each call in its own graph, timed like the step
    # (L2 flushed before every launch, events on the launching stream)
    kern_ms = {}
    for n, g in kgraphs.items():
        for _ in range(3):
            timed(g)
        kern_ms[n] = statistics.mean(timed(g) for _ in range(args.steps))
    qsa.qsa_check_device_errors()

    # decode context parallelism, emulated on one GPU: rank 0 maps only its
    # pages (p = 0 mod W), filters the selection to them and decodes one slice
    dcp_res = None
    if args.dcp_world > 1 and Qn == 1:
        Wd = args.dcp_world
        bt0 = cache.block_table.clone()
        cols = torch.arange(bt0.shape[1], device=dev)
        bt0[:, (cols % Wd) != 0] = -1
        cache0 = qsa.QsaCache(cache.k_pool, cache.v_pool, cache.kidx_pool, cache.side_pool, bt0)
        sel0 = torch.empty_like(buf.sel)
        o0 = torch.empty((1, B, dims.Hq, dims.D), dtype=torch.float32, device=dev)
        l0 = torch.empty((1, B, dims.Hq), dtype=torch.float32, device=dev)
        ws0 = torch.empty(max(16, qsa.qsa_sparse_decode_workspace_size(dims, B, k, 1)),
                          dtype=torch.uint8, device=dev)

        def rank0():
            qsa.qsa_select_owned(buf.sel, dims.P, Wd, 0, sel0)
            qsa.qsa_sparse_decode(dims, cache0, si["seq_lens"], si["q"], sel0, k, 1, o0, l0, ws0)

        g0 = capture(rank0)
        for _ in range(3):
            timed(g0)
        r0_ms = statistics.mean(timed(g0) for _ in range(args.steps))
        qsa.qsa_check_device_errors()
        kept = int((sel0 >= 0).sum())
        dcp_res = {"world": Wd, "rank0_select_and_decode_us": 1e3 * r0_ms,
                   "rank0_selected_blocks": kept,
                   "rank0_kv_bytes": kept * 4 * dims.Hkv * dims.D * 2 * 2,
                   "exchange_bytes_per_rank": B * dims.Hq * (dims.D + 1) * 4,
                   "note": "one GPU: rank 0's filter + one-slice decode over its pages, in a "
                           "graph after an L2 flush; the all-gather and the merge of W "
                           "partials are not timed here"}
        g0.reset()

    # sparse prefill on the same cache: the chunk is each sequence's newest
    # prefill_rows tokens (appended by the step), one query row per token
    prefill_res = None
    if args.prefill_rows > 0 and Qn == 1:
        prefill_res = time_prefill(args, qsa, wl, dims, cache, si["seq_lens"], k, R, ld, dev,
                                   capture, timed)

    # the other workloads of the scope (their own caches; the headline's
    # buffers stay allocated, every config frees its own)
    configs = None
    if not args.no_configs and Qn == 1 and world == 1 and not args.batch:
        timer = GraphTimer(dev, stream)
        peak_c, _ = load_peaks()
        configs = time_configs(args, qsa, timer, dev, peak_c)
        del timer

    # e2e: host buffers in pinned memory, copies inside the timed region,
    # calls made eagerly through the binding (the user's API)
    e2e = None
    if not args.no_e2e and Qn == 1:
        # the step's inputs travel in one pinned staging buffer (one copy), the
        # merged output and its LSE in one device buffer (one copy back)
        def packed(tensors, device, pin):
            offs, o = {}, 0
            for n, t in tensors.items():
                offs[n] = o
                o += (t.numel() * t.element_size() + 255) // 256 * 256
            raw = torch.empty(o, dtype=torch.uint8, device=device)
            if pin:
                raw = raw.pin_memory()
            views = {n: raw[offs[n]:offs[n] + t.numel() * t.element_size()].view(t.dtype)
                     .view(t.shape) for n, t in tensors.items()}
            return raw, views
        host_raw, host_in = packed(step_in, "cpu", True)
        for n, t in step_in.items():
            host_in[n].copy_(t.cpu())
        dev_raw, dev_in = packed(step_in, dev, False)
        out_raw, outs = packed({"out": buf.out, "lse": buf.lse}, dev, False)
        host_out_raw = torch.empty_like(out_raw, device="cpu").pin_memory()
        ebuf = qsa.StepBuffers(scores=buf.scores, sel=buf.sel, o_part=buf.o_part,
                               lse_part=buf.lse_part, out=outs["out"], lse=outs["lse"], ws=buf.ws)
        h2d = host_raw.numel()
        d2h = host_out_raw.numel()
        app = (dev_in["tok_seq"], dev_in["tok_pos"], dev_in["k_new"], dev_in["v_new"],
               dev_in["kidx_new"])
        e_ms = []
        for i in range(max(3, args.warmup) + args.steps):
            with torch.cuda.stream(stream):
                do_flush()
                s0.record()
                dev_raw.copy_(host_raw, non_blocking=True)
                qsa.decode_step(dims, cache, dev_in["seq_lens"], dev_in["q"], dev_in["q_idx"],
                                dev_in["w"], k, R, ebuf, append=app)
                host_out_raw.copy_(out_raw, non_blocking=True)
                s1.record()
            s1.synchronize()
            if i >= max(3, args.warmup):
                e_ms.append(s0.elapsed_time(s1))
        e_step = max_over_ranks(sum(e_ms), dev) / args.steps
        e2e = {"value": job_rate(world, B, e_step), "unit": "seqs/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": e_step,
               "api": "qsa.decode_step (one qsa_decode_step C call per step); one pinned "
                      "H2D copy of the packed step inputs, one D2H copy of output + LSE"}

    side_b, kv_b = algorithmic_bytes(wl.seq_lens, dims, k)
    peak, peak_kind = load_peaks()
    score_ms = kern_ms["index_score"]
    dec_ms = kern_ms["sparse_decode"]
    achieved = side_b / (score_ms / 1e3) / 1e9
    traffic = profile_traffic("index_score.cu", "index_score_b8x256k.md")
    attended = Qn * sum(min(4 * k, L) for L in wl.seq_lens)
    # kernels per step: the kernel nodes of the captured step graph (every
    # node is one of the library's kernels: the step is library calls only)
    launches = step_kernels if step_kernels is not None else 0
    res = {
        "metric": METRIC,
        "value": job_rate(world, B, ms_per_step),
        "unit": "seqs/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": f"{args.workload}: B={B} x L={max(wl.seq_lens)} tokens, "
                               f"32q/4kv heads x 128, indexer 16x128, top-{k} blocks of 4, "
                               f"R={R}, paged P=64 (shuffled)"
                               + (f", {Qn} decode queries per sequence (multi-query)"
                                  if Qn > 1 else ""),
                   "batch": B, "context": max(wl.seq_lens), "k": k, "R": R, "queries": Qn,
                   "l2": "flushed before every timed step (512 MiB write, then 512 MiB read)",
                   "step": ("CUDA graph of one qsa_decode_step call (append, score, top-k, "
                            "decode with the merge fused into its combine kernel)"
                            if Qn == 1 else
                            "CUDA graph of append+score+topk+decode (per query pair)+merge"),
                   "parallelism": f"replicas x{world}"},
        "attended_tokens_per_s": job_rate(world, attended, ms_per_step),
        "query_tokens_per_s": job_rate(world, B * Qn, ms_per_step),
        "step_us_p10_p50_p90": [round(1e3 * float(np.percentile(step_ms, q)), 2)
                                for q in (10, 50, 90)],
        "roofline": {"bound": "hbm", "kernel": "qsa_index_score", "achieved": achieved,
                     "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "peak_source": peak_kind,
                     "traffic": None if traffic is None else traffic * B / 8.0,
                     "algorithmic_bytes": side_b},
        "kernels_us": {n: 1e3 * m for n, m in kern_ms.items()},
        "kernels_timing": "each call alone in a CUDA graph, L2 flushed before, CUDA events",
        "score_plus_decode": {
            "bytes": side_b + kv_b,
            "us": 1e3 * (score_ms + dec_ms),
            "gbs": (side_b + kv_b) / ((score_ms + dec_ms) / 1e3) / 1e9,
            "frac": (side_b + kv_b) / ((score_ms + dec_ms) / 1e3) / 1e9 / peak,
            "timing": "sum of the two calls, each alone in its own graph",
            **({"one_graph_us": 1e3 * kern_ms["score_then_decode"],
                "one_graph_frac": (side_b + kv_b) / (kern_ms["score_then_decode"] / 1e3)
                / 1e9 / peak,
                "one_graph_timing": "the two calls back to back in one graph (the decode "
                                    "reads the step's selection)"}
               if "score_then_decode" in kern_ms else {})},
        "sparse_decode_frac": kv_b / (dec_ms / 1e3) / 1e9 / peak,
        "step_roofline_frac": (side_b + kv_b) / (ms_per_step / 1e3) / 1e9 / peak,
        "gpu_launches": launches * args.steps,
        "kernels_per_step": launches,
        "clocks": clk.summary(),
        "e2e": e2e,
    }
    if dcp_res is not None:
        res["dcp_emulated"] = dcp_res
    if prefill_res is not None:
        res["prefill"] = prefill_res
    if configs is not None:
        res["configs"] = configs
    graph.reset()
    for g in kgraphs.values():
        g.reset()
    if cpu_sample is not None:
        res["cpu_baseline"] = cpu_baseline(cpu_sample, dims, k, R)
    return res


def time_prefill(args, qsa, wl, dims, cache, seq_lens, k, R, ld, dev, capture, timed):
    """Sparse prefill of every sequence's newest rows: the whole call and each
    of its four calls in their own graphs (L2 flushed before each launch)."""
    from synth import prefill_queries

    T = min(args.prefill_rows, min(wl.seq_lens))
    B = wl.B
    row_start, q, q_idx, w = prefill_queries(wl, [T] * B)
    Nq = B * T
    pb = qsa.alloc_prefill(dims, B, Nq, ld, k, R, device=dev)
    ws1 = torch.empty(max(16, qsa.qsa_prefill_index_score_workspace_size(dims, B, Nq)),
                      dtype=torch.uint8, device=dev)
    ws2 = torch.empty(max(16, qsa.qsa_sparse_decode_workspace_size(dims, Nq, k, R)),
                      dtype=torch.uint8, device=dev)
    calls = {
        "prefill_index_score": lambda: qsa.qsa_prefill_index_score(
            dims, cache, seq_lens, row_start, q_idx, w, pb.scores, pb.row_len, ws1),
        "topk_select": lambda: qsa.qsa_topk_select(pb.row_len, pb.scores, k, pb.sel),
        "prefill_sparse_decode": lambda: qsa.qsa_prefill_sparse_decode(
            dims, cache, seq_lens, row_start, q, pb.sel, k, R, pb.o_part, pb.lse_part, ws2),
        "merge": lambda: qsa.qsa_merge(pb.o_part, pb.lse_part, pb.out, pb.lse),
    }
    whole = capture(lambda: qsa.sparse_prefill(dims, cache, seq_lens, row_start, q, q_idx, w,
                                               k, R, pb))
    graphs = {n: capture(fn) for n, fn in calls.items()}
    n_rep = max(10, min(args.steps, 100))
    for _ in range(3):
        timed(whole)
    all_ms = statistics.mean(timed(whole) for _ in range(n_rep))
    us = {}
    for n, g in graphs.items():
        for _ in range(3):
            timed(g)
        us[n] = 1e3 * statistics.mean(timed(g) for _ in range(n_rep))
    qsa.qsa_check_device_errors()
    whole.reset()
    for g in graphs.values():
        g.reset()
    lens = [L - T + i + 1 for L in wl.seq_lens for i in range(T)]
    flops = 2.0 * dims.Hi * dims.di * sum(ell // 4 for ell in lens)
    kv_rows = sum(min(4 * k, ell) for ell in lens) * dims.Hkv * dims.D * 2 * 2
    # the rows of a sequence share most of their selected blocks: the bytes
    # that must come from HBM are the K/V of the union of its rows' selections
    sel = pb.sel.cpu().numpy()
    rs = row_start.cpu().tolist()
    union_tokens = 0
    for s_, L in enumerate(wl.seq_lens):
        blocks = np.unique(sel[rs[s_]:rs[s_ + 1]])
        blocks = blocks[blocks >= 0].astype(np.int64)
        union_tokens += int(np.minimum(4, L - 4 * blocks).sum())
    kv = union_tokens * dims.Hkv * dims.D * 2 * 2
    tpk, tpk_src = load_tensor_peak()
    hbm, hbm_src = load_peaks()
    s_tf = flops / (us["prefill_index_score"] * 1e-6) / 1e12
    d_gb = kv / (us["prefill_sparse_decode"] * 1e-6) / 1e9
    return {
        "workload": f"the decode cache; each of the {B} sequences' newest {T} tokens as "
                    f"query rows ({Nq} rows, context {min(wl.seq_lens) - T + 1}.."
                    f"{max(wl.seq_lens)}), top-{k}, R={R}",
        "rows": Nq,
        "rows_per_s": Nq / (all_ms / 1e3),
        "us": 1e3 * all_ms,
        "kernels_us": us,
        "timing": "qsa_sparse_prefill and each of its calls alone in a CUDA graph, L2 "
                  "flushed before every launch, CUDA events, mean of %d" % n_rep,
        "roofline": {
            "prefill_index_score": {"bound": "tensor", "achieved": s_tf, "peak": tpk,
                                    "unit": "TFLOP/s", "frac": s_tf / tpk,
                                    "peak_source": tpk_src, "flops": flops},
            "prefill_sparse_decode": {"bound": "hbm", "achieved": d_gb, "peak": hbm,
                                      "unit": "GB/s", "frac": d_gb / hbm,
                                      "peak_source": hbm_src, "algorithmic_bytes": kv,
                                      "bytes_definition": "K/V of the union of each "
                                                          "sequence's rows' selected blocks",
                                      "bytes_per_row_sum": kv_rows},
        },
    }


def _threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info()]
        return max(n) if n else 1
    except Exception:
        return 1


def _oracle_one(sample, dims, k, R):
    import oracle
    to_bits = lambda t: t.contiguous().view(torch.int16).numpy().view(np.uint16)
    return oracle.decode_sequence(to_bits(sample["X"]), to_bits(sample["K"]),
                                  to_bits(sample["V"]), to_bits(sample["q"]),
                                  to_bits(sample["q_idx"]), sample["w"].numpy(), sample["L"],
                                  k, R, dims.scale)


def _oracle_rate(sample, dims, k, R, budget_s):
    n, t0 = 0, time.perf_counter()
    while True:
        _oracle_one(sample, dims, k, R)
        n += 1
        el = time.perf_counter() - t0
        if el >= budget_s or n >= 20:
            return n, n / el


def cpu_baseline(sample, dims, k, R, budget_s=12.0, single_budget_s=8.0):
    """The oracle, as it stands, on whole sequences of the same workload: with
    the BLAS threads numpy brings (all host cores), and on one thread."""
    n, rate = _oracle_rate(sample, dims, k, R, budget_s)
    res = {"value": rate, "unit": "seqs/s", "cores": _threads(), "kind": "oracle",
           "sample": f"{n} full decode(s) of one {sample['L']}-token sequence of the same "
                     f"workload (score, top-{k}, R={R} attention, merge), numpy fp64"}
    try:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            n1, rate1 = _oracle_rate(sample, dims, k, R, single_budget_s)
        res["single_thread"] = {"value": rate1, "unit": "seqs/s", "cores": 1,
                                "sample": f"{n1} full decode(s), BLAS limited to one thread"}
    except Exception as e:  # threadpoolctl missing: report the multi-thread figure only
        res["single_thread"] = {"unavailable": str(e)[:120]}
    try:
        res["cpu_model"] = open("/proc/cpuinfo").read().split("model name")[1].split(
            "\n")[0].strip(" :\t")
    except Exception:
        pass
    return res


# ------------------------------------------------------------ reference arm

def run_reference(args):
    from synth import make_custom, preset_spec, seed_for
    from block_sparse_decode_b200.qsa import QsaDims

    spec = preset_spec(args.workload)
    k = args.k or spec["k"]
    R = args.R or spec["R"]
    L = (max(spec["seq_lens"]) if args.workload != "steady128x64k"
         else spec["prefill"] + 1)
    B = len(spec["seq_lens"]) if not args.batch else args.batch
    wl = make_custom(spec["dims"], [L], k=k, R=R, seed=seed_for(args.workload), device="cpu",
                     paged=spec["paged"], needles=spec["needles"], mixture=spec["mixture"])
    K, V, X = wl.seq_tokens(0)
    sample = dict(K=K, V=V, X=X, q=wl.q[0], q_idx=wl.q_idx[0], w=wl.w[0], L=L)
    dims = QsaDims.of(wl.dims)
    for _ in range(max(0, min(args.warmup, 3))):
        _oracle_one(sample, dims, k, R)
    t = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        _oracle_one(sample, dims, k, R)
        t.append(time.perf_counter() - t0)
    ms = 1e3 * statistics.mean(t)
    v = 1.0 / (ms / 1e3)
    return {"impl": "reference", "metric": METRIC, "value": v, "unit": "seqs/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": f"{args.workload}: one {L}-token sequence per step "
                                   f"(B={B} workload sampled), top-{k}, R={R}",
                       "batch": 1, "context": L, "k": k, "R": R},
            "cpu_baseline": {"value": v, "unit": "seqs/s", "cores": _threads(),
                             "kind": "oracle",
                             "sample": f"one sequence of {L} tokens per step"},
            "e2e": {"value": v, "unit": "seqs/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return
    if world > 1:
        torch.distributed.init_process_group(
            "nccl", timeout=datetime.timedelta(seconds=120),
            device_id=torch.device("cuda", local_rank))
    res = run_ours(args, rank, world, local_rank)
    if rank == 0:
        print(json.dumps(res), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
