"""Thin Python binding of libqsa.so (ctypes).

Argument marshalling only: every call checks tensor dtypes, devices and
shapes, turns them into raw device pointers plus sizes, and calls the C
function of the same name (declared in include/qsa.h). Every step of the
decode path runs in the library's CUDA kernels; there is no other backend.
PyTorch provides the device memory and the current CUDA stream.
"""

from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqsa.so")

QSA_OK = 0
QSA_ERR_INVALID_ARG = 1
QSA_ERR_UNSUPPORTED = 2
QSA_ERR_CUDA = 3
QSA_ERR_BOUNDS = 4
QSA_ERR_TIMEOUT = 5

# Symbols declared in include/qsa.h (checked by the test suite).
EXPORTS = ("qsa_version", "qsa_last_error", "qsa_append", "qsa_index_score",
           "qsa_topk_workspace_size", "qsa_topk_select", "qsa_sparse_decode_workspace_size",
           "qsa_sparse_decode", "qsa_sparse_decode_static", "qsa_merge",
           "qsa_decode_step", "qsa_sparse_decode_mq_workspace_size", "qsa_sparse_decode_mq",
           "qsa_select_owned", "qsa_check_device_errors",
           "qsa_prefill_index_score_workspace_size", "qsa_prefill_index_score",
           "qsa_prefill_sparse_decode", "qsa_sparse_prefill_workspace_size",
           "qsa_sparse_prefill")


class QsaError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"qsa status {status}: {msg}")
        self.status = status


class _Dims(ctypes.Structure):
    _fields_ = [("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32), ("D", ctypes.c_int32),
                ("Hi", ctypes.c_int32), ("di", ctypes.c_int32), ("P", ctypes.c_int32),
                ("scale", ctypes.c_float)]


class _Cache(ctypes.Structure):
    _fields_ = [("k_pool", ctypes.c_void_p), ("v_pool", ctypes.c_void_p),
                ("kidx_pool", ctypes.c_void_p), ("side_pool", ctypes.c_void_p),
                ("block_table", ctypes.c_void_p), ("num_seqs", ctypes.c_int32),
                ("max_pages_per_seq", ctypes.c_int32), ("num_pages", ctypes.c_int32)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libqsa.so (raises if it was not built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m block_sparse_decode_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, I32, SZ, F = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t, ctypes.c_float
    DP, CP = ctypes.POINTER(_Dims), ctypes.POINTER(_Cache)
    sig = {
        "qsa_version": (I32, []),
        "qsa_last_error": (ctypes.c_char_p, []),
        "qsa_append": (I32, [DP, CP, I32, P, P, P, P, P, P]),
        "qsa_index_score": (I32, [DP, CP, I32, P, P, P, P, I32, P]),
        "qsa_topk_workspace_size": (SZ, [I32, I32, I32]),
        "qsa_topk_select": (I32, [I32, P, P, I32, I32, P, P, SZ, P]),
        "qsa_sparse_decode_workspace_size": (SZ, [DP, I32, I32, I32]),
        "qsa_sparse_decode": (I32, [DP, CP, I32, P, P, P, I32, I32, P, P, P, SZ, P]),
        "qsa_sparse_decode_static": (I32, [DP, CP, I32, P, P, P, I32, I32, P, P, P]),
        "qsa_sparse_decode_mq_workspace_size": (SZ, [DP, I32, I32, I32, I32]),
        "qsa_sparse_decode_mq": (I32, [DP, CP, I32, I32, P, P, P, I32, I32, P, P, P, SZ, P]),
        "qsa_select_owned": (I32, [I32, P, I32, I32, I32, I32, P, P]),
        "qsa_merge": (I32, [I32, I32, I32, I32, P, P, P, I32, P, P]),
        "qsa_decode_step": (I32, [DP, CP, I32, P, P, P, P, P, I32, P, P, P, P, I32, I32, P, I32,
                                  P, P, P, P, SZ, P, I32, P, P]),
        "qsa_check_device_errors": (I32, [P, ctypes.POINTER(I32)]),
        "qsa_prefill_index_score_workspace_size": (SZ, [DP, I32, I32]),
        "qsa_prefill_index_score": (I32, [DP, CP, I32, P, P, I32, P, P, P, I32, P, P, SZ, P]),
        "qsa_prefill_sparse_decode": (I32, [DP, CP, I32, P, P, I32, P, P, I32, I32, P, P, P, SZ,
                                            P]),
        "qsa_sparse_prefill_workspace_size": (SZ, [DP, I32, I32, I32, I32]),
        "qsa_sparse_prefill": (I32, [DP, CP, I32, P, P, I32, P, P, P, I32, I32, P, I32, P, P, P,
                                     P, P, SZ, P, I32, P, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _lib = L
    return L


def _check(status: int):
    if status != QSA_OK:
        raise QsaError(status, lib().qsa_last_error().decode())


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _nbytes(t: torch.Tensor | None) -> int:
    """Size in bytes of an optional scratch tensor (0 for None)."""
    return 0 if t is None else t.numel() * t.element_size()


def _ptr(t: torch.Tensor | None, dtype=None, name="tensor") -> int | None:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    return t.data_ptr()


# ------------------------------------------------------------------ structs

@dataclass(frozen=True)
class QsaDims:
    Hq: int
    Hkv: int
    D: int
    Hi: int
    di: int
    P: int
    scale: float

    @classmethod
    def of(cls, d) -> "QsaDims":
        return cls(int(d.Hq), int(d.Hkv), int(d.D), int(d.Hi), int(d.di), int(d.P),
                   float(d.scale))

    def c(self) -> _Dims:
        c = self.__dict__.get("_c")
        if c is None:  # built once (the dims are frozen)
            c = _Dims(self.Hq, self.Hkv, self.D, self.Hi, self.di, self.P, self.scale)
            object.__setattr__(self, "_c", c)
        return c


@dataclass
class QsaCache:
    """The paged pools plus the one block table that indexes all of them."""

    k_pool: torch.Tensor      # bf16 [num_pages, P, Hkv, D]
    v_pool: torch.Tensor      # bf16 [num_pages, P, Hkv, D]
    kidx_pool: torch.Tensor   # bf16 [num_pages, P, di]
    side_pool: torch.Tensor   # bf16 [num_pages, P/4, di]
    block_table: torch.Tensor  # int32 [num_seqs, max_pages_per_seq]

    def c(self) -> _Cache:
        # rebuilt only when a pool or the block table is replaced
        key = (self.k_pool.data_ptr(), self.v_pool.data_ptr(), self.kidx_pool.data_ptr(),
               self.side_pool.data_ptr(), self.block_table.data_ptr(),
               tuple(self.block_table.shape), int(self.k_pool.shape[0]))
        hit = self.__dict__.get("_c")
        if hit is not None and hit[0] == key:
            return hit[1]
        bf = torch.bfloat16
        c = _Cache(_ptr(self.k_pool, bf, "k_pool"), _ptr(self.v_pool, bf, "v_pool"),
                      _ptr(self.kidx_pool, bf, "kidx_pool"), _ptr(self.side_pool, bf, "side_pool"),
                      _ptr(self.block_table, torch.int32, "block_table"),
                      int(self.block_table.shape[0]), int(self.block_table.shape[1]),
                      int(self.k_pool.shape[0]))
        self.__dict__["_c"] = (key, c)
        return c


def alloc_cache(dims: QsaDims, num_pages: int, block_table: torch.Tensor,
                device="cuda") -> QsaCache:
    """Allocate the four pools (uninitialised) for ``num_pages`` pages."""
    d = dims
    bf = torch.bfloat16
    return QsaCache(
        k_pool=torch.empty((num_pages, d.P, d.Hkv, d.D), dtype=bf, device=device),
        v_pool=torch.empty((num_pages, d.P, d.Hkv, d.D), dtype=bf, device=device),
        kidx_pool=torch.empty((num_pages, d.P, d.di), dtype=bf, device=device),
        side_pool=torch.empty((num_pages, d.P // 4, d.di), dtype=bf, device=device),
        block_table=block_table.to(device=device, dtype=torch.int32).contiguous())


# ------------------------------------------------------------------ calls

def qsa_version() -> int:
    return int(lib().qsa_version())


def qsa_append(dims: QsaDims, cache: QsaCache, tok_seq, tok_pos, k_new, v_new, kidx_new,
               stream=None):
    N = int(tok_seq.shape[0])
    bf = torch.bfloat16
    _check(lib().qsa_append(ctypes.byref(dims.c()), ctypes.byref(cache.c()), N,
                            _ptr(tok_seq, torch.int32, "tok_seq"),
                            _ptr(tok_pos, torch.int32, "tok_pos"), _ptr(k_new, bf, "k_new"),
                            _ptr(v_new, bf, "v_new"), _ptr(kidx_new, bf, "kidx_new"),
                            _stream(stream)))


def qsa_index_score(dims: QsaDims, cache: QsaCache, seq_lens, q_idx, w, scores, stream=None):
    B = int(seq_lens.shape[0])
    _check(lib().qsa_index_score(ctypes.byref(dims.c()), ctypes.byref(cache.c()), B,
                                 _ptr(seq_lens, torch.int32, "seq_lens"),
                                 _ptr(q_idx, torch.bfloat16, "q_idx"),
                                 _ptr(w, torch.float32, "w"),
                                 _ptr(scores, torch.float32, "scores"),
                                 int(scores.shape[1]), _stream(stream)))


def qsa_topk_workspace_size(B: int, ld_scores: int, k: int) -> int:
    return int(lib().qsa_topk_workspace_size(B, ld_scores, k))


def qsa_topk_select(seq_lens, scores, k: int, sel, ws=None, stream=None):
    B = int(seq_lens.shape[0])
    _check(lib().qsa_topk_select(B, _ptr(seq_lens, torch.int32, "seq_lens"),
                                 _ptr(scores, torch.float32, "scores"), int(scores.shape[1]),
                                 int(k), _ptr(sel, torch.int32, "sel"),
                                 _ptr(ws, None, "ws"),
                                 0 if ws is None else ws.numel() * ws.element_size(),
                                 _stream(stream)))


def qsa_sparse_decode_workspace_size(dims: QsaDims, B: int, k: int, R: int) -> int:
    return int(lib().qsa_sparse_decode_workspace_size(ctypes.byref(dims.c()), B, k, R))


def qsa_sparse_decode(dims: QsaDims, cache: QsaCache, seq_lens, q, sel, k: int, R: int, o_part,
                      lse_part, ws, stream=None):
    B = int(seq_lens.shape[0])
    _check(lib().qsa_sparse_decode(ctypes.byref(dims.c()), ctypes.byref(cache.c()), B,
                                   _ptr(seq_lens, torch.int32, "seq_lens"),
                                   _ptr(q, torch.bfloat16, "q"), _ptr(sel, torch.int32, "sel"),
                                   int(k), int(R), _ptr(o_part, torch.float32, "o_part"),
                                   _ptr(lse_part, torch.float32, "lse_part"),
                                   _ptr(ws, None, "ws"), _nbytes(ws),
                                   _stream(stream)))


def qsa_sparse_decode_mq_workspace_size(dims: QsaDims, B: int, Qn: int, k: int, R: int) -> int:
    return int(lib().qsa_sparse_decode_mq_workspace_size(ctypes.byref(dims.c()), B, Qn, k, R))


def qsa_sparse_decode_mq(dims: QsaDims, cache: QsaCache, seq_lens, q, sel, k: int, R: int,
                         o_part, lse_part, ws, stream=None):
    """Multi-query decode: q [B, Qn, Hq, D] -> o_part [R, B, Qn, Hq, D]."""
    B, Qn = int(q.shape[0]), int(q.shape[1])
    _check(lib().qsa_sparse_decode_mq(ctypes.byref(dims.c()), ctypes.byref(cache.c()), B, Qn,
                                      _ptr(seq_lens, torch.int32, "seq_lens"),
                                      _ptr(q, torch.bfloat16, "q"), _ptr(sel, torch.int32, "sel"),
                                      int(k), int(R), _ptr(o_part, torch.float32, "o_part"),
                                      _ptr(lse_part, torch.float32, "lse_part"),
                                      _ptr(ws, None, "ws"), _nbytes(ws),
                                      _stream(stream)))


def qsa_sparse_decode_static(dims: QsaDims, cache: QsaCache, seq_lens, q, sel, k: int, R: int,
                             o_part, lse_part, stream=None):
    """qsa_sparse_decode with the library's static device scratch (no
    workspace, no allocation; see include/qsa.h for its limits)."""
    B = int(seq_lens.shape[0])
    _check(lib().qsa_sparse_decode_static(ctypes.byref(dims.c()), ctypes.byref(cache.c()), B,
                                          _ptr(seq_lens, torch.int32, "seq_lens"),
                                          _ptr(q, torch.bfloat16, "q"),
                                          _ptr(sel, torch.int32, "sel"), int(k), int(R),
                                          _ptr(o_part, torch.float32, "o_part"),
                                          _ptr(lse_part, torch.float32, "lse_part"),
                                          _stream(stream)))


def qsa_select_owned(sel, P: int, world: int, rank: int, sel_out, stream=None):
    """The selected blocks whose page rank ``rank`` of ``world`` holds (page p
    on rank p mod world), same order, -1 padded."""
    B, k = (int(x) for x in sel.shape)
    _check(lib().qsa_select_owned(B, _ptr(sel, torch.int32, "sel"), k, int(P), int(world),
                                  int(rank), _ptr(sel_out, torch.int32, "sel_out"),
                                  _stream(stream)))


def qsa_merge(o_part, lse_part, out, lse_out=None, stream=None):
    R, B, Hq, D = (int(x) for x in o_part.shape)
    if out.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("out must be bf16 or fp32")
    _check(lib().qsa_merge(R, B, Hq, D, _ptr(o_part, torch.float32, "o_part"),
                           _ptr(lse_part, torch.float32, "lse_part"), _ptr(out, None, "out"),
                           1 if out.dtype == torch.bfloat16 else 0,
                           _ptr(lse_out, torch.float32, "lse_out"), _stream(stream)))


def qsa_check_device_errors(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device error flags.
    Raises QsaError on QSA_ERR_BOUNDS / QSA_ERR_TIMEOUT."""
    flags = ctypes.c_int32(0)
    st = lib().qsa_check_device_errors(_stream(stream), ctypes.byref(flags))
    if st != QSA_OK:
        raise QsaError(st, lib().qsa_last_error().decode() + f" [flags={flags.value}]")
    return flags.value


# ------------------------------------------------------------ decode step

@dataclass
class StepBuffers:
    """Outputs and scratch of one decode step for a fixed (B, k, R, ld)."""

    scores: torch.Tensor     # fp32 [B, ld]
    sel: torch.Tensor        # int32 [B, k]
    o_part: torch.Tensor     # fp32 [R, B, Hq, D]
    lse_part: torch.Tensor   # fp32 [R, B, Hq]
    out: torch.Tensor        # bf16 [B, Hq, D]
    lse: torch.Tensor        # fp32 [B, Hq]
    ws: torch.Tensor         # uint8 scratch of qsa_sparse_decode


def alloc_step(dims: QsaDims, B: int, ld: int, k: int, R: int, device="cuda",
               out_dtype=torch.bfloat16) -> StepBuffers:
    ws_bytes = max(16, qsa_sparse_decode_workspace_size(dims, B, k, R))
    return StepBuffers(
        scores=torch.empty((B, ld), dtype=torch.float32, device=device),
        sel=torch.empty((B, k), dtype=torch.int32, device=device),
        o_part=torch.empty((R, B, dims.Hq, dims.D), dtype=torch.float32, device=device),
        lse_part=torch.empty((R, B, dims.Hq), dtype=torch.float32, device=device),
        out=torch.empty((B, dims.Hq, dims.D), dtype=out_dtype, device=device),
        lse=torch.empty((B, dims.Hq), dtype=torch.float32, device=device),
        ws=torch.empty((ws_bytes,), dtype=torch.uint8, device=device))


def decode_step(dims: QsaDims, cache: QsaCache, seq_lens, q, q_idx, w, k: int, R: int,
                buf: StepBuffers, stream=None, append=None):
    """One QSA decode step: [append] -> score -> top-k -> split attention -> merge,
    issued by the library's single qsa_decode_step call.

    ``append`` is an optional (tok_seq, tok_pos, k_new, v_new, kidx_new) tuple
    written first. Results land in ``buf``.
    """
    B = int(seq_lens.shape[0])
    if append is not None:
        tok_seq, tok_pos, k_new, v_new, kidx_new = append
        N = int(tok_seq.shape[0])
        app = (_ptr(tok_seq, torch.int32, "tok_seq"), _ptr(tok_pos, torch.int32, "tok_pos"),
               _ptr(k_new, torch.bfloat16, "k_new"), _ptr(v_new, torch.bfloat16, "v_new"),
               _ptr(kidx_new, torch.bfloat16, "kidx_new"))
    else:
        N, app = 0, (None,) * 5
    _check(lib().qsa_decode_step(
        ctypes.byref(dims.c()), ctypes.byref(cache.c()), N, *app, B,
        _ptr(seq_lens, torch.int32, "seq_lens"), _ptr(q, torch.bfloat16, "q"),
        _ptr(q_idx, torch.bfloat16, "q_idx"), _ptr(w, torch.float32, "w"), int(k), int(R),
        _ptr(buf.scores, torch.float32, "scores"), int(buf.scores.shape[1]),
        _ptr(buf.sel, torch.int32, "sel"), _ptr(buf.o_part, torch.float32, "o_part"),
        _ptr(buf.lse_part, torch.float32, "lse_part"), _ptr(buf.ws, None, "ws"),
        _nbytes(buf.ws), _ptr(buf.out, None, "out"),
        1 if buf.out.dtype == torch.bfloat16 else 0, _ptr(buf.lse, torch.float32, "lse"),
        _stream(stream)))


def ld_for(seq_lens) -> int:
    """Smallest score row length that holds every sequence's blocks."""
    return max(1, max(int(math.ceil(int(L) / 4)) for L in seq_lens))


# ------------------------------------------------------------ sparse prefill

def qsa_prefill_index_score_workspace_size(dims: QsaDims, S: int, Nq: int) -> int:
    return int(lib().qsa_prefill_index_score_workspace_size(ctypes.byref(dims.c()), S, Nq))


def qsa_prefill_index_score(dims: QsaDims, cache: QsaCache, seq_lens, row_start, q_idx, w,
                            scores, row_len, ws, stream=None):
    """Scores of every prefill row: q_idx [Nq, Hi, di] -> scores [Nq, ld], row_len [Nq]."""
    S, Nq = int(seq_lens.shape[0]), int(q_idx.shape[0])
    _check(lib().qsa_prefill_index_score(
        ctypes.byref(dims.c()), ctypes.byref(cache.c()), S,
        _ptr(seq_lens, torch.int32, "seq_lens"), _ptr(row_start, torch.int32, "row_start"), Nq,
        _ptr(q_idx, torch.bfloat16, "q_idx"), _ptr(w, torch.float32, "w"),
        _ptr(scores, torch.float32, "scores"), int(scores.shape[1]),
        _ptr(row_len, torch.int32, "row_len"), _ptr(ws, None, "ws"),
        _nbytes(ws), _stream(stream)))


def qsa_prefill_sparse_decode(dims: QsaDims, cache: QsaCache, seq_lens, row_start, q, sel,
                              k: int, R: int, o_part, lse_part, ws, stream=None):
    """Split attention of every prefill row: q [Nq, Hq, D] -> o_part [R, Nq, Hq, D]."""
    S, Nq = int(seq_lens.shape[0]), int(q.shape[0])
    _check(lib().qsa_prefill_sparse_decode(
        ctypes.byref(dims.c()), ctypes.byref(cache.c()), S,
        _ptr(seq_lens, torch.int32, "seq_lens"), _ptr(row_start, torch.int32, "row_start"), Nq,
        _ptr(q, torch.bfloat16, "q"), _ptr(sel, torch.int32, "sel"), int(k), int(R),
        _ptr(o_part, torch.float32, "o_part"), _ptr(lse_part, torch.float32, "lse_part"),
        _ptr(ws, None, "ws"), _nbytes(ws), _stream(stream)))


def qsa_sparse_prefill_workspace_size(dims: QsaDims, S: int, Nq: int, k: int, R: int) -> int:
    return int(lib().qsa_sparse_prefill_workspace_size(ctypes.byref(dims.c()), S, Nq, k, R))


@dataclass
class PrefillBuffers:
    """Outputs and scratch of one sparse prefill for fixed (S, Nq, k, R, ld)."""

    scores: torch.Tensor     # fp32 [Nq, ld]
    row_len: torch.Tensor    # int32 [Nq]
    sel: torch.Tensor        # int32 [Nq, k]
    o_part: torch.Tensor     # fp32 [R, Nq, Hq, D]
    lse_part: torch.Tensor   # fp32 [R, Nq, Hq]
    out: torch.Tensor        # bf16 [Nq, Hq, D]
    lse: torch.Tensor        # fp32 [Nq, Hq]
    ws: torch.Tensor         # uint8 scratch of qsa_sparse_prefill


def alloc_prefill(dims: QsaDims, S: int, Nq: int, ld: int, k: int, R: int, device="cuda",
                  out_dtype=torch.bfloat16) -> PrefillBuffers:
    ws_bytes = max(16, qsa_sparse_prefill_workspace_size(dims, S, Nq, k, R))
    return PrefillBuffers(
        scores=torch.empty((Nq, ld), dtype=torch.float32, device=device),
        row_len=torch.empty((Nq,), dtype=torch.int32, device=device),
        sel=torch.empty((Nq, k), dtype=torch.int32, device=device),
        o_part=torch.empty((R, Nq, dims.Hq, dims.D), dtype=torch.float32, device=device),
        lse_part=torch.empty((R, Nq, dims.Hq), dtype=torch.float32, device=device),
        out=torch.empty((Nq, dims.Hq, dims.D), dtype=out_dtype, device=device),
        lse=torch.empty((Nq, dims.Hq), dtype=torch.float32, device=device),
        ws=torch.empty((ws_bytes,), dtype=torch.uint8, device=device))


def sparse_prefill(dims: QsaDims, cache: QsaCache, seq_lens, row_start, q, q_idx, w, k: int,
                   R: int, buf: PrefillBuffers, stream=None):
    """Sparse prefill of the chunk rows (already appended): score -> top-k ->
    split attention -> merge per row, by the library's single qsa_sparse_prefill
    call. Results land in ``buf``."""
    S, Nq = int(seq_lens.shape[0]), int(q.shape[0])
    _check(lib().qsa_sparse_prefill(
        ctypes.byref(dims.c()), ctypes.byref(cache.c()), S,
        _ptr(seq_lens, torch.int32, "seq_lens"), _ptr(row_start, torch.int32, "row_start"), Nq,
        _ptr(q, torch.bfloat16, "q"), _ptr(q_idx, torch.bfloat16, "q_idx"),
        _ptr(w, torch.float32, "w"), int(k), int(R), _ptr(buf.scores, torch.float32, "scores"),
        int(buf.scores.shape[1]), _ptr(buf.row_len, torch.int32, "row_len"),
        _ptr(buf.sel, torch.int32, "sel"), _ptr(buf.o_part, torch.float32, "o_part"),
        _ptr(buf.lse_part, torch.float32, "lse_part"), _ptr(buf.ws, None, "ws"),
        _nbytes(buf.ws), _ptr(buf.out, None, "out"),
        1 if buf.out.dtype == torch.bfloat16 else 0, _ptr(buf.lse, torch.float32, "lse"),
        _stream(stream)))
