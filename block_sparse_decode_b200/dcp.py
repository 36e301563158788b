"""Decode context parallelism (DCP) over the ranks of a torch.distributed group.

Page "Qwen 4 QSA gets decode context parallelism" (orcarouter.ai), section
"What the pull request actually changes": under DCP a rank reads just its
own part of the main KV cache, the indexer's selector state is copied on
every rank rather than split, and the partial attention results are merged
afterwards ("Questions worth answering directly"). Here a rank's slice is
the pages it holds: page p of every sequence on rank p mod W (see
qsa_select_owned in include/qsa.h).

One step on every rank, in the same order:

1. (optional) qsa_append of the step's new tokens;
2. qsa_index_score and qsa_topk_select on the replicated side cache (every
   rank derives the same selection);
3. qsa_select_owned keeps the selected blocks of the rank's pages;
4. qsa_sparse_decode (one slice) over them gives the rank's partial
   (O_r [B, Hq, D], LSE_r [B, Hq]);
5. all-gather of the W partials (the one exchange of the step: B * Hq *
   (D + 1) * 4 bytes per rank, NCCL over NVLink for CUDA tensors);
6. qsa_merge of the W partials (R = W).

The selector side is replicated: ``cache`` maps every page of the side pool
and the per-token indexer keys on every rank. The K/V read may use its own
``kv_cache`` whose block table maps only the rank's pages (the others -1)
and whose K/V pools hold only those pages: the decode touches only the pages
of the blocks step 3 keeps, so a rank's K/V memory shrinks W-fold (the
capacity gain the page reports for DCP).
"""

from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.distributed as dist

from . import qsa


def exchange_partials(o_r: torch.Tensor, lse_r: torch.Tensor, group=None):
    """All-gather this rank's partial. Returns (O [W, ...], LSE [W, ...]) in
    rank order, on the device of the inputs. CUDA tensors are gathered on the
    current CUDA stream (NCCL orders its work after what that stream already
    holds); over a gloo group they travel through host memory, after a
    synchronising copy on the current stream."""
    W = dist.get_world_size(group)
    dev = o_r.device
    staged = o_r.is_cuda and dist.get_backend(group) == "gloo"
    if staged:
        o_r, lse_r = o_r.cpu(), lse_r.cpu()
    O = torch.empty((W,) + tuple(o_r.shape), dtype=o_r.dtype, device=o_r.device)
    L = torch.empty((W,) + tuple(lse_r.shape), dtype=lse_r.dtype, device=lse_r.device)
    dist.all_gather(list(O.unbind(0)), o_r.contiguous(), group=group)
    dist.all_gather(list(L.unbind(0)), lse_r.contiguous(), group=group)
    if staged:
        O, L = O.to(dev), L.to(dev)
    return O, L


@dataclass
class DcpBuffers:
    """Per-rank buffers of a DCP step, on top of a qsa.StepBuffers."""

    step: qsa.StepBuffers      # scores, selection, merged output (o_part unused)
    sel_owned: torch.Tensor    # int32 [B, k]
    o_r: torch.Tensor          # fp32 [1, B, Hq, D]: this rank's partial
    lse_r: torch.Tensor        # fp32 [1, B, Hq]
    ws: torch.Tensor           # uint8 scratch of the one-slice decode


def alloc_dcp(dims: qsa.QsaDims, B: int, ld: int, k: int, device="cuda") -> DcpBuffers:
    step = qsa.alloc_step(dims, B, ld, k, 1, device=device)
    ws_bytes = max(16, qsa.qsa_sparse_decode_workspace_size(dims, B, k, 1))
    return DcpBuffers(step=step,
                      sel_owned=torch.empty((B, k), dtype=torch.int32, device=device),
                      o_r=torch.empty((1, B, dims.Hq, dims.D), dtype=torch.float32, device=device),
                      lse_r=torch.empty((1, B, dims.Hq), dtype=torch.float32, device=device),
                      ws=torch.empty((ws_bytes,), dtype=torch.uint8, device=device))


def dcp_decode_step(dims: qsa.QsaDims, cache: qsa.QsaCache, seq_lens, q, q_idx, w, k: int,
                    buf: DcpBuffers, group=None, append=None, stream=None, kv_cache=None):
    """One DCP decode step on this rank (steps 1-6 of the module docstring).
    The merged output lands in buf.step.out / buf.step.lse on every rank.
    ``kv_cache`` (default ``cache``) is the cache the K/V read goes through;
    ``append``, if given, writes into ``cache``.

    Every launch and the all-gather run on one stream: ``stream`` (a
    torch.cuda.Stream or a raw cudaStream_t handle) or, when it is None, the
    current stream. It is made the current stream for the whole step, so the
    collective, which torch issues on the current stream, is ordered after
    the decode that writes the rank's partial and before the merge."""
    rank, W = dist.get_rank(group), dist.get_world_size(group)
    sb = buf.step
    if stream is not None and not isinstance(stream, torch.cuda.Stream):
        stream = torch.cuda.ExternalStream(int(stream))
    with torch.cuda.stream(stream):
        st = torch.cuda.current_stream()
        if append is not None:
            qsa.qsa_append(dims, cache, *append, stream=st)
        qsa.qsa_index_score(dims, cache, seq_lens, q_idx, w, sb.scores, stream=st)
        qsa.qsa_topk_select(seq_lens, sb.scores, k, sb.sel, stream=st)
        qsa.qsa_select_owned(sb.sel, dims.P, W, rank, buf.sel_owned, stream=st)
        qsa.qsa_sparse_decode(dims, cache if kv_cache is None else kv_cache, seq_lens, q,
                              buf.sel_owned, k, 1, buf.o_r, buf.lse_r, buf.ws, stream=st)
        O, L = exchange_partials(buf.o_r[0], buf.lse_r[0], group)
        qsa.qsa_merge(O, L, sb.out, sb.lse, stream=st)
