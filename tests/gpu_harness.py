"""Runs seeded workloads through the CUDA library (via the C ABI binding) and
through the oracle, for the parity tests. Only test code imports this."""

from __future__ import annotations

import numpy as np
import torch

import oracle
from block_sparse_decode_b200 import qsa
from tests.helpers import bits


def token_index(wl, upto=None):
    """(tok_seq, tok_pos) of every drawn token row; rows at positions >=
    upto[b] are marked as padding (-1) so that they write nothing."""
    seq = np.empty(sum(wl.cap_lens), dtype=np.int32)
    pos = np.empty_like(seq)
    for b, n in enumerate(wl.cap_lens):
        o = wl.tok_off[b]
        seq[o:o + n] = b
        pos[o:o + n] = np.arange(n)
        if upto is not None:
            seq[o + upto[b]:o + n] = -1
    return seq, pos


class CudaRun:
    """The cache of a workload on the GPU plus the buffers of one decode step."""

    def __init__(self, wl, k=None, R=None, prefill=None, poison=True):
        self.wl = wl
        self.dims = qsa.QsaDims.of(wl.dims)
        self.k = wl.k if k is None else k
        self.R = wl.R if R is None else R
        dev = wl.k_tok.device
        assert dev.type == "cuda"
        self.cache = qsa.alloc_cache(self.dims, wl.num_pages, wl.block_table, device=dev)
        if poison:  # stale bytes, so reads of unwritten slots show up
            for t in (self.cache.k_pool, self.cache.v_pool, self.cache.kidx_pool,
                      self.cache.side_pool):
                t.view(torch.int16).random_(-32768, 32767)
        upto = [L - 1 for L in wl.seq_lens] if prefill is None else prefill
        seq, pos = token_index(wl, upto)
        qsa.qsa_append(self.dims, self.cache, torch.from_numpy(seq).to(dev),
                       torch.from_numpy(pos).to(dev), wl.k_tok, wl.v_tok, wl.kidx_tok)
        self.seq_lens = torch.tensor(wl.seq_lens, dtype=torch.int32, device=dev)
        self.ld = qsa.ld_for(wl.cap_lens)
        self.buf = qsa.alloc_step(self.dims, wl.B, self.ld, self.k, self.R, device=dev)

    def current_tokens(self, lens=None):
        """Append arguments that write token L_b - 1 of every sequence."""
        wl = self.wl
        lens = wl.seq_lens if lens is None else lens
        dev = wl.k_tok.device
        rows = torch.tensor([wl.tok_off[b] + L - 1 for b, L in enumerate(lens)], device=dev)
        return (torch.arange(wl.B, dtype=torch.int32, device=dev),
                torch.tensor([L - 1 for L in lens], dtype=torch.int32, device=dev),
                wl.k_tok[rows].contiguous(), wl.v_tok[rows].contiguous(),
                wl.kidx_tok[rows].contiguous())

    def step(self, q=None, q_idx=None, w=None, append=True, lens=None):
        wl = self.wl
        if lens is not None:
            self.seq_lens = torch.tensor(lens, dtype=torch.int32, device=wl.k_tok.device)
        qsa.decode_step(self.dims, self.cache, self.seq_lens,
                        wl.q if q is None else q, wl.q_idx if q_idx is None else q_idx,
                        wl.w if w is None else w, self.k, self.R, self.buf,
                        append=self.current_tokens(lens) if append else None)
        flags = qsa.qsa_check_device_errors()
        assert flags == 0, f"device error flags {flags}"

    def side_rows(self, b, L):
        """The side-cache rows of sequence b's complete blocks, in block order."""
        P = self.dims.P
        rpp = P // 4
        nfull = L // 4
        j = torch.arange(nfull, device=self.cache.side_pool.device)
        pages = self.cache.block_table[b].long()[j // rpp]
        return bits(self.cache.side_pool[pages, j % rpp])


def oracle_sequence(wl, b, L=None, q=None, q_idx=None, w=None, k=None, R=None, sel=None):
    """Oracle decode of sequence b on host copies of the workload's bytes."""
    L = wl.seq_lens[b] if L is None else L
    K, V, X = wl.seq_tokens(b, L)
    q = wl.q[b] if q is None else q
    q_idx = wl.q_idx[b] if q_idx is None else q_idx
    w = wl.w[b] if w is None else w
    return oracle.decode_sequence(bits(X), bits(K), bits(V), bits(q), bits(q_idx),
                                  w.detach().cpu().numpy(), L, wl.k if k is None else k,
                                  wl.R if R is None else R, wl.dims.scale, sel=sel)


def score_tolerance(wl, b, L, q_idx=None, w=None):
    """Per-block bound on |s_gpu - s_oracle|: 2^-12 of the absolute-value sum
    sum_h w_h sum_d |q_hd kc_d| (fp32 accumulation of exact bf16 products, then
    a 16-term fp32 head sum, stays far inside it)."""
    _, _, X = wl.seq_tokens(b, L)
    kc = oracle.block_keys(bits(X), L)
    q = oracle.bf16_to_f32(bits(wl.q_idx[b] if q_idx is None else q_idx)).astype(np.float64)
    ww = (wl.w[b] if w is None else w).detach().cpu().numpy().astype(np.float64)
    return (np.abs(kc) @ np.abs(q).T) @ np.abs(ww) * 2.0 ** -12 + 1e-30
