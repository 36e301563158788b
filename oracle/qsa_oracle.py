"""CPU oracle for the QSA sparse decode step.

TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT. Only the test suite, the smoke
check in ``__graft_entry__`` and the CPU-baseline / reference arm of
``bench.py`` may import or run this module. The CUDA library never calls it
and shares no code with it.

It is a plain, slow restatement of what the decode step computes, written
from the page "Qwen 4 QSA gets decode context parallelism: inside vLLM's
draft PR for Qwen3.8-Flash-Next" (orcarouter.ai):

* section "What the pull request actually changes", QSA paragraph: a small
  indexer shrinks the keys four to one into micro-blocks, ranks the blocks
  and retains the top 512 (near 2,048 tokens); exact attention (softmax and
  the weighted sum of V) then uses the full-precision K and V of those blocks;
* same section, first bullet and the DCP paragraph: each rank reads only its
  slice of the main KV cache, the selector stays replicated, and the partial
  attention results are combined after the split read (also the answer on
  DCP vs TP in "Questions worth answering directly");
* same section, third and fourth bullets: selector and main cache share one
  cache group; synthetic batches write nothing into the side caches.

The page gives no formulas. The readings this oracle fixes, and that the
CUDA library follows, are:

* micro-block key kc = bf16_rne(fp32 left-to-right sum of its n keys / n),
  n = 4 for complete blocks and n = L mod 4 for the trailing partial block;
* block score s_b = sum_h w_h * max(0, q_idx_h . kc_b), no other factor;
* top-k order: score descending, then block index ascending; the k_b =
  min(k, nb) winners are reported in ascending block order, padded with -1;
* slice r of R owns blocks [floor(r*nb/R), floor((r+1)*nb/R)); the one
  selection serves every slice;
* per slice: z_t = scale * q_h . K_t over the tokens t < L of its selected
  blocks, LSE_r = ln sum_t exp z_t, O_r = sum_t softmax(z)_t V_t, and an empty
  slice gives O_r = 0, LSE_r = -inf;
* merge: O = sum_r e^(LSE_r - m) O_r / sum_r e^(LSE_r - m), LSE = m +
  ln sum_r e^(LSE_r - m), m = max_r LSE_r;
* sparse prefill (listed on the page beside the decode path, with no steps
  given): every token of an appended chunk queries like a decode step over
  its own causal prefix, i.e. the decode step of the sequence cut right
  after that token.

Floating point: fp64 for every dot product, softmax and merge; exact fp32
(IEEE round-to-nearest adds and division) plus round-to-nearest-even to bf16
where the reading fixes bits (the compressed keys). bf16 tensors are handled
as their uint16 bit patterns. Every function here is pinned by a CPU test
against something other than itself (hand-worked fixtures, closed forms,
brute force, an independent dense attention, torch's bf16 conversion).
"""

from __future__ import annotations

import numpy as np

NEG_INF = float("-inf")


# ---------------------------------------------------------------- bf16 bits

def bf16_to_f32(bits) -> np.ndarray:
    """uint16 bf16 bit patterns -> float32 (exact)."""
    b = np.asarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def f32_to_bf16(x) -> np.ndarray:
    """float32 -> bf16 bits, IEEE round-to-nearest-even (NaN stays NaN)."""
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    u = x.view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    rounded = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    nan = (u & np.uint32(0x7FFFFFFF)) > np.uint32(0x7F800000)
    out = np.where(nan, (u >> np.uint32(16)) | np.uint32(0x0040), rounded)
    return out.astype(np.uint16)


# ------------------------------------------------------ micro-block keys

def compress_keys(keys_bits) -> np.ndarray:
    """Compressed key of micro-blocks from their n (1..4) indexer keys.

    keys_bits [..., n, di]: fp32 sum in token order ((k0 + k1) + k2) + k3,
    divided by n in fp32, rounded to bf16. Returns bf16 bits [..., di].
    """
    k = bf16_to_f32(keys_bits)
    n = k.shape[-2]
    assert 1 <= n <= 4
    acc = k[..., 0, :].copy()
    for i in range(1, n):
        acc = (acc + k[..., i, :]).astype(np.float32)
    mean = (acc / np.float32(n)).astype(np.float32)
    return f32_to_bf16(mean)


def side_cache(kidx_bits, L: int) -> np.ndarray:
    """One-shot side cache of a sequence: compressed keys of its L // 4 complete
    blocks, bf16 bits [L // 4, di]."""
    kidx_bits = np.asarray(kidx_bits, dtype=np.uint16)
    nfull = L // 4
    di = kidx_bits.shape[1]
    return compress_keys(kidx_bits[:4 * nfull].reshape(nfull, 4, di))


def block_keys(kidx_bits, L: int) -> np.ndarray:
    """Keys of all nb = ceil(L/4) micro-blocks as float64 [nb, di]: the side
    cache for complete blocks, plus the trailing partial block's key built the
    same way from its L mod 4 tokens."""
    kidx_bits = np.asarray(kidx_bits, dtype=np.uint16)
    keys = [side_cache(kidx_bits, L)]
    if L % 4:
        j = L // 4
        keys.append(compress_keys(kidx_bits[4 * j:L])[None, :])
    return bf16_to_f32(np.concatenate(keys, axis=0)).astype(np.float64)


# ------------------------------------------------------------- scoring

def index_scores(kc64, q_idx_bits, w) -> np.ndarray:
    """s_b = sum_h w_h * max(0, q_idx_h . kc_b) in float64, for every block."""
    q = bf16_to_f32(q_idx_bits).astype(np.float64)          # [Hi, di]
    w64 = np.asarray(w, dtype=np.float32).astype(np.float64)  # [Hi]
    dots = np.asarray(kc64, dtype=np.float64) @ q.T           # [nb, Hi]
    return np.maximum(dots, 0.0) @ w64


# ----------------------------------------------------------- selection

def topk_blocks(scores, k: int) -> np.ndarray:
    """The k_b = min(k, nb) best blocks by (score desc, index asc), returned in
    ascending block order and padded with -1 to length k. -0.0 ranks as 0.0."""
    s = np.asarray(scores, dtype=np.float64) + 0.0
    nb = s.shape[0]
    idx = np.arange(nb)
    order = np.lexsort((idx, -s))   # primary: -score ascending; secondary: index
    kb = min(k, nb)
    chosen = np.sort(order[:kb])
    out = np.full(k, -1, dtype=np.int64)
    out[:kb] = chosen
    return out


# ----------------------------------------------------------- attention

def slice_bounds(nb: int, R: int):
    """Block range [lo, hi) owned by each of the R context slices."""
    return [((r * nb) // R, ((r + 1) * nb) // R) for r in range(R)]


def attend_slices(q_bits, k_bits, v_bits, sel, L: int, scale: float, R: int, visible=None):
    """Per-slice partial attention over the selected blocks.

    q_bits [Hq, D]; k_bits, v_bits [>=L, Hkv, D]; sel: selected block indices
    (ascending, -1 padding ignored). Query head h reads KV head h // (Hq/Hkv).
    The slices are those of the nb = ceil(L/4) blocks; the query sees tokens
    t < L, or t < `visible` when given (a query placed before the end).
    Returns O [R, Hq, D] float64 and LSE [R, Hq] float64 (natural log,
    including the softmax scale).
    """
    q = bf16_to_f32(q_bits).astype(np.float64)
    Kf = bf16_to_f32(np.asarray(k_bits)[:L]).astype(np.float64)
    Vf = bf16_to_f32(np.asarray(v_bits)[:L]).astype(np.float64)
    Hq, D = q.shape
    Hkv = Kf.shape[1]
    G = Hq // Hkv
    nb = (L + 3) // 4
    blocks = [int(j) for j in np.asarray(sel).ravel() if j >= 0]
    O = np.zeros((R, Hq, D), dtype=np.float64)
    LSE = np.full((R, Hq), NEG_INF, dtype=np.float64)
    for r, (lo, hi) in enumerate(slice_bounds(nb, R)):
        lim = L if visible is None else min(L, visible)
        toks = [t for j in blocks if lo <= j < hi for t in range(4 * j, 4 * j + 4) if t < lim]
        if not toks:
            continue
        toks = np.asarray(toks)
        for h in range(Hq):
            g = h // G
            z = scale * (Kf[toks, g, :] @ q[h])
            m = z.max()
            lse = m + np.log(np.exp(z - m).sum())
            p = np.exp(z - lse)
            O[r, h] = p @ Vf[toks, g, :]
            LSE[r, h] = lse
    return O, LSE


def attend_slices_mq(q_bits, k_bits, v_bits, sel, L: int, scale: float, R: int):
    """Several decode queries per sequence sharing one selection (multi-query
    decode, e.g. draft tokens of multi-token prediction): q_bits [Q, Hq, D],
    query j sits at position L - Q + j and sees the selected tokens
    t <= L - Q + j. Returns O [R, Q, Hq, D] and LSE [R, Q, Hq] (float64)."""
    q_all = np.asarray(q_bits)
    Q = q_all.shape[0]
    parts = [attend_slices(q_all[j], k_bits, v_bits, sel, L, scale, R, visible=L - Q + j + 1)
             for j in range(Q)]
    return (np.stack([o for o, _ in parts], axis=1), np.stack([l for _, l in parts], axis=1))


def owned_blocks(sel, P: int, W: int, r: int) -> np.ndarray:
    """Decode context parallelism over W ranks: the selected blocks whose page
    (block j lies on page 4j // P of its sequence) belongs to rank r, page p
    belonging to rank p mod W. Same order as `sel`, -1 padded to len(sel)."""
    sel = np.asarray(sel)
    own = [int(j) for j in sel if j >= 0 and ((4 * int(j)) // P) % W == r]
    return np.array(own + [-1] * (len(sel) - len(own)), dtype=np.int64)


def merge_partials(O, LSE):
    """LSE-weighted combine of R partials: O [R, H, D], LSE [R, H] -> O [H, D], LSE [H].
    Slices with LSE = -inf contribute nothing."""
    O = np.asarray(O, dtype=np.float64)
    LSE = np.asarray(LSE, dtype=np.float64)
    R, H, D = O.shape
    out = np.zeros((H, D), dtype=np.float64)
    lse_out = np.full(H, NEG_INF, dtype=np.float64)
    for h in range(H):
        live = [r for r in range(R) if LSE[r, h] != NEG_INF]
        if not live:
            continue
        m = max(LSE[r, h] for r in live)
        wts = np.array([np.exp(LSE[r, h] - m) for r in live])
        out[h] = sum(wt * O[r, h] for wt, r in zip(wts, live)) / wts.sum()
        lse_out[h] = m + np.log(wts.sum())
    return out, lse_out


# ------------------------------------------------- the whole decode step

def decode_sequence(kidx_bits, k_bits, v_bits, q_bits, q_idx_bits, w, L: int, k: int,
                    R: int, scale: float, sel=None):
    """Score -> top-k -> R-way split attention -> merge for one sequence.

    If ``sel`` is given, attention runs over that selection instead of the
    oracle's own (used to recompute attention over another selection).
    """
    kc = block_keys(kidx_bits, L)
    scores = index_scores(kc, q_idx_bits, w)
    own_sel = topk_blocks(scores, k)
    use_sel = own_sel if sel is None else np.asarray(sel)
    O_part, LSE_part = attend_slices(q_bits, k_bits, v_bits, use_sel, L, scale, R)
    O, LSE = merge_partials(O_part, LSE_part)
    return dict(scores=scores, sel=own_sel, O_part=O_part, LSE_part=LSE_part, O=O, LSE=LSE)


# -------------------------------------------------------- sparse prefill

def prefill_rows(seq_lens, row_start):
    """Query rows of a chunked prefill (this library's reading of the sparse
    prefill the page lists beside the decode path; the page describes no
    step of it). Sequence s holds rows [row_start[s], row_start[s+1]): its
    T_s newest tokens, already appended, so L_s = seq_lens[s] counts them.
    Row i of sequence s is the token at position L_s - T_s + i; it queries
    like a decode step of a sequence of length row_len = L_s - T_s + i + 1.
    Returns (row_seq, row_len) as int64 arrays over all rows."""
    seq_lens = [int(x) for x in seq_lens]
    row_start = [int(x) for x in row_start]
    assert len(row_start) == len(seq_lens) + 1 and row_start[0] == 0
    row_seq, row_len = [], []
    for s, L in enumerate(seq_lens):
        T = row_start[s + 1] - row_start[s]
        assert 0 <= T <= L
        for i in range(T):
            row_seq.append(s)
            row_len.append(L - T + i + 1)
    return np.asarray(row_seq, dtype=np.int64), np.asarray(row_len, dtype=np.int64)


def prefill_sequence(kidx_bits, k_bits, v_bits, q_bits, q_idx_bits, w, L: int, T: int, k: int,
                     R: int, scale: float, sels=None):
    """The T chunk rows of one sequence of length L (after the chunk): row i is
    the decode step (score -> top-k -> R-way split attention -> merge) of the
    sequence cut to its first L - T + i + 1 tokens, with the row's own
    q [Hq, D], q_idx [Hi, di] and w [Hi] (q_bits [T, Hq, D], q_idx_bits
    [T, Hi, di], w [T, Hi]). ``sels`` [T, k], when given, replaces each row's
    own selection in the attention. Returns one decode_sequence dict per row."""
    out = []
    for i in range(T):
        ell = L - T + i + 1
        out.append(decode_sequence(kidx_bits, k_bits, v_bits, np.asarray(q_bits)[i],
                                   np.asarray(q_idx_bits)[i], np.asarray(w)[i], ell, k, R, scale,
                                   sel=None if sels is None else np.asarray(sels)[i]))
    return out


# ------------------------------------------------------ paged cache append

def append_paged(k_pool, v_pool, kidx_pool, side_pool, block_table, P: int,
                 tok_seq, tok_pos, k_new, v_new, kidx_new):
    """Write a batch of new tokens into the paged pools (all uint16 bf16 bits).

    k_pool, v_pool [pages, P, Hkv, D]; kidx_pool [pages, P, di];
    side_pool [pages, P/4, di]; block_table [B, max_pages].
    Token i goes to page block_table[seq, pos // P], slot pos % P. Entries with
    seq < 0 or pos < 0 write nothing. After every token is written, each token
    whose position closes a micro-block (pos % 4 == 3) stores the compressed
    key of its block, read back from the indexer-key pool, at side slot
    (pos % P) // 4 of the same page. Pools are modified in place.
    """
    tok_seq = np.asarray(tok_seq)
    tok_pos = np.asarray(tok_pos)
    for i in range(tok_seq.shape[0]):
        s, p = int(tok_seq[i]), int(tok_pos[i])
        if s < 0 or p < 0:
            continue
        page = int(block_table[s, p // P])
        k_pool[page, p % P] = k_new[i]
        v_pool[page, p % P] = v_new[i]
        kidx_pool[page, p % P] = kidx_new[i]
    for i in range(tok_seq.shape[0]):
        s, p = int(tok_seq[i]), int(tok_pos[i])
        if s < 0 or p < 0 or p % 4 != 3:
            continue
        page = int(block_table[s, p // P])
        first = p % P - 3
        side_pool[page, (p % P) // 4] = compress_keys(kidx_pool[page, first:first + 4])
