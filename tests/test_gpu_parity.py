"""Parity of the CUDA library (through its C ABI) with the CPU oracle.

Bars: side cache, pool bytes and top-k indices bit-exact (top-k compared on
the GPU's own fp32 scores, so both sides decide in the same precision);
scores within the bound of tests/gpu_harness.score_tolerance; selection equal
to the oracle's up to the near-tie band; attention, recomputed by the oracle
over the GPU's own selection, within max abs 1e-2 and rel-L2 5e-3, LSE within
1e-3.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from block_sparse_decode_b200 import qsa
from synth import make_custom, make_workload, step_queries
from synth.workloads import DIMS_FULL, Dims
from tests.gpu_harness import CudaRun, oracle_sequence, score_tolerance, token_index
from tests.helpers import bf16_same, bits, check_attention, check_selection

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _check_seq(run, b, L=None, q=None, q_idx=None, w=None, full=True):
    wl, k, R = run.wl, run.k, run.R
    L = wl.seq_lens[b] if L is None else L
    nb = (L + 3) // 4
    ref = oracle_sequence(wl, b, L, q, q_idx, w, k=k, R=R)
    K, V, X = wl.seq_tokens(b, L)
    # side cache: bit-exact against the one-shot build
    assert np.array_equal(run.side_rows(b, L), oracle.side_cache(bits(X), L)), f"side b={b}"
    # scores
    s_gpu = run.buf.scores[b, :nb].double().cpu().numpy()
    tol = score_tolerance(wl, b, L, q_idx, w)
    err = np.abs(s_gpu - ref["scores"])
    assert np.all(err <= tol), f"scores b={b}: worst {err.max():.3e} at {int(err.argmax())}"
    # top-k: exact on the GPU's scores; oracle's own selection up to ties
    sel_gpu = run.buf.sel[b].cpu().numpy()
    assert np.array_equal(sel_gpu, oracle.topk_blocks(s_gpu, k)), f"top-k b={b}"
    check_selection(sel_gpu, ref["sel"], ref["scores"], k, what=f"sel b={b}")
    if not full:
        return
    # attention over the GPU's own selection
    ref2 = oracle_sequence(wl, b, L, q, q_idx, w, k=k, R=R, sel=sel_gpu)
    check_attention(run.buf.o_part[:, b].cpu().numpy(), run.buf.lse_part[:, b].cpu().numpy(),
                    ref2["O_part"], ref2["LSE_part"], what=f"partials b={b}")
    check_attention(run.buf.out[b].float().cpu().numpy(), run.buf.lse[b].cpu().numpy(),
                    ref2["O"], ref2["LSE"], what=f"merged b={b}")


# ------------------------------------------------------------ small cases

@pytest.mark.parametrize("R", [2, 1, 3, 8])
def test_tiny_preset_end_to_end(R):
    wl = make_workload("tiny", device=DEV)
    run = CudaRun(wl, R=R)
    run.step()
    for b in range(wl.B):
        _check_seq(run, b)
        assert set(wl.needles[b]) <= set(run.buf.sel[b].tolist())


@pytest.mark.parametrize("R", [1, 2, 4, 8])
def test_ragged_paged_full_heads(R):
    lens = [1, 2, 3, 4, 5, 63, 64, 65, 2047, 2048, 2049, 2051, 4099, 9001, 20000]
    wl = make_custom(DIMS_FULL, lens, k=512, R=R, seed=101, device=DEV, paged=True)
    run = CudaRun(wl)
    run.step()
    for b in range(wl.B):
        _check_seq(run, b)


@pytest.mark.parametrize("dims,lens,k", [
    (Dims(Hq=4, Hkv=4, D=128, Hi=5, di=64, P=32, scale=0.11), [77, 1030, 3], 40),
    (Dims(Hq=12, Hkv=2, D=128, Hi=24, di=128, P=128, scale=0.09), [4096, 515, 6000], 100),
    (Dims(Hq=2, Hkv=1, D=128, Hi=1, di=128, P=1024, scale=0.2), [33, 2570], 7),
    (Dims(Hq=16, Hkv=2, D=128, Hi=32, di=64, P=64, scale=0.088), [1500, 2600], 1),
    # page sizes that are not powers of two: P = 96 (a multiple of 32, the
    # tensor-core kernel with 8-row page pieces), P = 16 and 48 (the
    # warp-level kernel that gathers side-cache rows one by one), and P = 4
    # (one micro-block per page)
    (Dims(Hq=32, Hkv=4, D=128, Hi=16, di=128, P=96, scale=0.088), [9001, 300, 40003], 512),
    (Dims(Hq=32, Hkv=4, D=128, Hi=16, di=128, P=16, scale=0.088), [9001, 301, 2], 512),
    (Dims(Hq=8, Hkv=2, D=128, Hi=5, di=64, P=48, scale=0.11), [4099, 1500, 7], 64),
    (Dims(Hq=8, Hkv=8, D=128, Hi=32, di=128, P=4, scale=0.1), [517, 2049], 100),
])
def test_other_dims(dims, lens, k):
    for R in (1, 3):
        wl = make_custom(dims, lens, k=k, R=R, seed=102, device=DEV, paged=True)
        run = CudaRun(wl)
        run.step()
        for b in range(wl.B):
            _check_seq(run, b)


@pytest.mark.parametrize("P", [32, 64])
def test_index_score_long_rows_refill_the_page_table(P):
    """Score rows so long that each scoring CTA's tiles overflow its shared
    page table (two halves of 1,024 page ids: 64 tiles at P = 32, 128 tiles
    at P = 64) more than once, so both halves are refilled while the
    producers run: 4 sequences of 2,600,000 tokens at P = 32 (137 tiles per
    CTA), of 5,200,000 at P = 64. Scoring reads only the side cache here
    (every length a multiple of 4: no partial block), filled with random
    bf16 rows through a shuffled block table; sampled blocks of every
    sequence (both ends, tile and page boundaries, random ones) are checked
    against the oracle's score formula within the scores' fp32 bound."""
    g = torch.Generator(device=DEV).manual_seed(4200 + P)
    di, Hi, B = 128, 16, 4
    L = 2_600_000 * (P // 32)
    dims = qsa.QsaDims(Hq=8, Hkv=1, D=128, Hi=Hi, di=di, P=P, scale=0.088)
    npp = L // P                                 # pages per sequence
    num_pages = B * npp
    perm = torch.randperm(num_pages, generator=g, device=DEV).to(torch.int32)
    bt = perm.view(B, npp).contiguous()
    side = torch.randn((num_pages, P // 4, di), generator=g, device=DEV).to(torch.bfloat16)
    small = torch.zeros((num_pages, 1, 1, 8), dtype=torch.bfloat16, device=DEV)  # never read
    cache = qsa.QsaCache(k_pool=small, v_pool=small, kidx_pool=small, side_pool=side,
                         block_table=bt)
    q_idx = torch.randn((B, Hi, di), generator=g, device=DEV).to(torch.bfloat16)
    w = torch.rand((B, Hi), generator=g, device=DEV)
    lens = torch.full((B,), L, dtype=torch.int32, device=DEV)
    nb = L // 4
    scores = torch.full((B, nb), float("nan"), device=DEV)
    qsa.qsa_index_score(dims, cache, lens, q_idx, w, scores)
    assert qsa.qsa_check_device_errors() == 0
    assert not torch.isnan(scores).any()
    rng = np.random.default_rng(P)
    picks = np.unique(np.concatenate([
        np.arange(0, 300), np.arange(nb - 300, nb),
        np.arange(127, nb, 128 * 997), np.arange(128, nb, 128 * 997),
        np.arange(P // 4 - 1, nb, (P // 4) * 4999), rng.integers(0, nb, 3000)]))
    rpp = P // 4
    for b in range(B):
        j = torch.from_numpy(picks).to(DEV)
        rows = side[bt[b].long()[j // rpp], j % rpp]                   # [n, di] bf16
        kc = oracle.bf16_to_f32(bits(rows)).astype(np.float64)
        qb = bits(q_idx[b])
        wb = w[b].cpu().numpy()
        ref = oracle.index_scores(kc, qb, wb)
        q64 = oracle.bf16_to_f32(qb).astype(np.float64)
        tol = (np.abs(kc) @ np.abs(q64).T) @ np.abs(wb.astype(np.float64)) * 2.0 ** -12 + 1e-30
        got = scores[b, j].double().cpu().numpy()
        err = np.abs(got - ref)
        assert np.all(err <= tol), (b, int(picks[err.argmax()]), float(err.max()))


def test_clustered_selection_leaves_empty_slices():
    # needles + k small: the selection sits in a few slices, most slices empty
    d = DIMS_FULL
    wl = make_custom(d, [8192, 3000], k=4, R=16, seed=103, device=DEV, needles=4)
    run = CudaRun(wl)
    run.step()
    for b in range(wl.B):
        _check_seq(run, b)
        assert np.isneginf(run.buf.lse_part[:, b].cpu().numpy()).any()


# ------------------------------------------------------------ top-k alone

def _topk_gpu(scores_np, k, lens=None):
    B, ld = scores_np.shape
    lens = [4 * ld] * B if lens is None else lens
    sl = torch.tensor(lens, dtype=torch.int32, device=DEV)
    sc = torch.from_numpy(np.ascontiguousarray(scores_np, dtype=np.float32)).to(DEV)
    sel = torch.full((B, k), -7, dtype=torch.int32, device=DEV)
    qsa.qsa_topk_select(sl, sc, k, sel)
    assert qsa.qsa_check_device_errors() == 0
    return sel.cpu().numpy()


# clusters of 8 CTAs per row (6 rows), of 4 (66 rows), one CTA per row (300)
@pytest.mark.parametrize("rows", [6, 66, 300])
@pytest.mark.parametrize("case", ["random", "ties", "allzero", "negzero", "negative", "few",
                                  "heavy", "bucket900", "bucket1100"])
def test_topk_exact(case, rows):
    g = np.random.default_rng(sum(map(ord, case)))
    # one CTA per row takes rows of at most 65,536 blocks
    B, ld, k = 6, (70001 if rows <= 6 else 65536), 512
    if case == "random":
        s = g.standard_normal((B, ld)).astype(np.float32) ** 2
    elif case == "ties":
        s = g.integers(0, 40, (B, ld)).astype(np.float32)
    elif case == "allzero":
        s = np.zeros((B, ld), np.float32)
    elif case == "negzero":
        s = np.where(g.random((B, ld)) < 0.5, -0.0, 0.0).astype(np.float32)
        s[:, ::97] = 1.0
    elif case == "negative":
        s = g.standard_normal((B, ld)).astype(np.float32)
    elif case == "few":
        s = g.standard_normal((B, ld)).astype(np.float32)
    elif case == "heavy":  # heavy tail with a block of exact ties at the threshold
        s = np.exp(3 * g.standard_normal((B, ld))).astype(np.float32)
        s[:, 1000:3000] = np.float32(np.sort(s[0])[-400])
    else:
        # 400 clear winners, then n keys in [1, 1 + 2^-7): one bucket of the
        # upper 16 key bits holding the k-th key, their low bits drawn from
        # 300 values (many exact duplicates, ranked by index), the rest far
        # below. n = 900 is resolved as one tie list in the cluster kernel,
        # n = 1100 takes its two further digit passes.
        n = int(case[len("bucket"):])
        s = (0.25 * g.random((B, ld))).astype(np.float32)
        for b in range(B):
            pos = g.permutation(ld)
            s[b, pos[:400]] = (2.0 + g.random(400)).astype(np.float32)
            low = g.integers(0, 300, n).astype(np.uint32)
            s[b, pos[400:400 + n]] = (np.uint32(0x3F800000) + low).view(np.float32)
    lens = [4 * ld - 3, 4 * ld, 2049, 2048, 4 * 513, 1]
    if case == "few":
        lens = [5, 4 * 511 + 1, 4 * 512, 4 * 512 + 1, 4 * 65536, 4 * 70001]
    lens = [min(x, 4 * ld) for x in lens]
    if rows > B:  # the same rows again, each with a shifted copy of its scores
        s = np.concatenate([np.roll(s, 7 * r, axis=1) for r in range(rows // B)], axis=0)
        lens = lens * (rows // B)
        B = rows
    got = _topk_gpu(s, k, lens)
    for b in range(B):
        nb = (lens[b] + 3) // 4
        ref = oracle.topk_blocks(s[b, :nb].astype(np.float64), k)
        assert np.array_equal(got[b], ref), f"{case} b={b} nb={nb}"


@pytest.mark.parametrize("rows", [3, 66, 300])  # clusters of 8, 4 CTAs; one CTA per row
@pytest.mark.parametrize("k", [1, 2, 255, 256, 1024, 4096])
def test_topk_k_sweep(k, rows):
    g = np.random.default_rng(k)
    s = (g.integers(0, 1000, (rows, 30000)) * 0.25).astype(np.float32)
    lens = ([4 * 30000, 4 * 4097 - 2, 4 * k + 4] * rows)[:rows]
    got = _topk_gpu(s, k, lens)
    for b in range(rows):
        nb = (lens[b] + 3) // 4
        assert np.array_equal(got[b], oracle.topk_blocks(s[b, :nb].astype(np.float64), k))


def test_topk_many_rows_long_score_rows_use_clusters():
    # rows longer than the one-CTA kernel's shared-memory key array
    g = np.random.default_rng(5)
    B, ld, k = 64, 100003, 512
    s = g.standard_normal((B, ld)).astype(np.float32) ** 2
    lens = [4 * ld - 1 - 4 * b for b in range(B)]
    got = _topk_gpu(s, k, lens)
    for b in range(0, B, 9):
        nb = (lens[b] + 3) // 4
        assert np.array_equal(got[b], oracle.topk_blocks(s[b, :nb].astype(np.float64), k)), b


# ------------------------------------------------------------ merge alone

@pytest.mark.parametrize("R,out_bf16,D", [(1, True, 128), (2, False, 128), (5, True, 128),
                                          (64, False, 128),
                                          # head dims that are not a multiple of 128: some
                                          # lanes of the row's warp own no dims in a pass
                                          (3, True, 64), (9, False, 192), (2, False, 4),
                                          (33, True, 260)])
def test_merge_matches_oracle(R, out_bf16, D):
    g = np.random.default_rng(R * 1000 + D)
    B, Hq = 3, 32
    O = g.standard_normal((R, B, Hq, D)).astype(np.float32)
    LSE = (3 * g.standard_normal((R, B, Hq))).astype(np.float32)
    LSE[R // 2, 1, :5] = -np.inf
    if R > 1:
        LSE[:, 2, 7] = -np.inf  # a row with every slice empty
    o_t, l_t = torch.from_numpy(O).to(DEV), torch.from_numpy(LSE).to(DEV)
    out = torch.empty((B, Hq, D), dtype=torch.bfloat16 if out_bf16 else torch.float32,
                      device=DEV)
    lse = torch.empty((B, Hq), dtype=torch.float32, device=DEV)
    qsa.qsa_merge(o_t, l_t, out, lse)
    out_np, lse_np = out.float().cpu().numpy(), lse.cpu().numpy()
    for b in range(B):
        Om, Lm = oracle.merge_partials(O[:, b].astype(np.float64), LSE[:, b].astype(np.float64))
        check_attention(out_np[b], lse_np[b], Om, Lm, what=f"merge b={b}")


# ------------------------------------------------------------ append alone

@pytest.mark.parametrize("lens", [[259, 64, 3, 100], [13, 7, 30, 40], [4, 1]])
def test_append_pools_bit_exact(lens):
    d = Dims(Hq=8, Hkv=4, D=128, Hi=4, di=128, P=16, scale=0.1)
    wl = make_custom(d, lens, k=8, R=1, seed=104, device=DEV, paged=True, pool_slack_pages=3)
    cache = qsa.alloc_cache(qsa.QsaDims.of(d), wl.num_pages, wl.block_table, device=DEV)
    for t in (cache.k_pool, cache.v_pool, cache.kidx_pool, cache.side_pool):
        t.view(torch.int16).random_(-32768, 32767)
    host = [bits(t).copy() for t in (cache.k_pool, cache.v_pool, cache.kidx_pool,
                                     cache.side_pool)]
    seq, pos = token_index(wl)
    perm = np.random.default_rng(0).permutation(len(seq))
    seq, pos = seq[perm], pos[perm]
    pos[::17] = -1  # padding entries
    seq[5::23] = -1
    rows = torch.from_numpy(perm).to(DEV)
    kn, vn, xn = wl.k_tok[rows].contiguous(), wl.v_tok[rows].contiguous(), \
        wl.kidx_tok[rows].contiguous()
    qsa.qsa_append(qsa.QsaDims.of(d), cache, torch.from_numpy(seq).to(DEV),
                   torch.from_numpy(pos).to(DEV), kn, vn, xn)
    assert qsa.qsa_check_device_errors() == 0
    oracle.append_paged(*host, wl.block_table.cpu().numpy(), d.P, seq, pos, bits(kn), bits(vn),
                        bits(xn))
    for got, want, name in zip((cache.k_pool, cache.v_pool, cache.kidx_pool, cache.side_pool),
                               host, ("k", "v", "kidx", "side")):
        # the poisoned pools hold NaN patterns; sums over them give NaN whose
        # payload is hardware-specific
        assert bf16_same(bits(got), want), f"{name} pool differs"


def test_append_incremental_equals_bulk_side_cache():
    d = DIMS_FULL
    lens = [515, 64, 7]
    wl = make_custom(d, lens, k=8, R=1, seed=105, device=DEV, paged=True)
    run = CudaRun(wl, prefill=[0] * 3)  # nothing written in bulk
    for t in range(max(lens)):
        live = [b for b in range(3) if t < lens[b]]
        rows = torch.tensor([wl.tok_off[b] + t for b in live], device=DEV)
        qsa.qsa_append(run.dims, run.cache, torch.tensor(live, dtype=torch.int32, device=DEV),
                       torch.full((len(live),), t, dtype=torch.int32, device=DEV),
                       wl.k_tok[rows].contiguous(), wl.v_tok[rows].contiguous(),
                       wl.kidx_tok[rows].contiguous())
    assert qsa.qsa_check_device_errors() == 0
    for b, L in enumerate(lens):
        _, _, X = wl.seq_tokens(b, L)
        assert np.array_equal(run.side_rows(b, L), oracle.side_cache(bits(X), L))


# ------------------------------------------------------------ error paths

def test_bad_page_ids_are_flagged_not_faulted():
    wl = make_custom(DIMS_FULL, [3000, 900], k=64, R=2, seed=106, device=DEV)
    run = CudaRun(wl)
    bad = run.cache.block_table.clone()
    run.cache.block_table[0, 3] = wl.num_pages + 1000   # out-of-range page id
    run.cache.block_table[1, 1] = -5
    with pytest.raises(qsa.QsaError) as ei:
        run.step(append=False)
    assert ei.value.status == qsa.QSA_ERR_BOUNDS
    run.cache.block_table.copy_(bad)
    run.step()  # the context is still healthy
    _check_seq(run, 0)


def test_seq_len_beyond_score_row_is_flagged():
    wl = make_custom(DIMS_FULL, [3000, 900], k=64, R=1, seed=107, device=DEV)
    run = CudaRun(wl)
    sc = torch.zeros((2, 100), dtype=torch.float32, device=DEV)  # ld too short for seq 0
    qsa.qsa_index_score(run.dims, run.cache, run.seq_lens, wl.q_idx, wl.w, sc)
    with pytest.raises(qsa.QsaError) as ei:
        qsa.qsa_check_device_errors()
    assert ei.value.status == qsa.QSA_ERR_BOUNDS


def test_invalid_arguments_rejected_on_host():
    wl = make_custom(DIMS_FULL, [100], k=8, R=1, seed=108, device=DEV)
    run = CudaRun(wl)
    with pytest.raises(qsa.QsaError) as ei:
        qsa.qsa_sparse_decode(run.dims, run.cache, run.seq_lens, wl.q, run.buf.sel, 8, 65,
                              run.buf.o_part, run.buf.lse_part, run.buf.ws)
    assert ei.value.status == qsa.QSA_ERR_UNSUPPORTED
    o_mis = torch.empty(run.buf.o_part.numel() + 1, dtype=torch.float32, device=DEV)[1:]
    with pytest.raises(qsa.QsaError) as ei:  # o_part not 16-byte aligned
        qsa.qsa_sparse_decode(run.dims, run.cache, run.seq_lens, wl.q, run.buf.sel, 8, 1,
                              o_mis.view_as(run.buf.o_part), run.buf.lse_part, run.buf.ws)
    assert ei.value.status == qsa.QSA_ERR_INVALID_ARG
    small_ws = torch.empty(16, dtype=torch.uint8, device=DEV)
    for ws in (small_ws, None):
        with pytest.raises(qsa.QsaError) as ei:
            qsa.qsa_sparse_decode(run.dims, run.cache, run.seq_lens, wl.q, run.buf.sel, 8, 1,
                                  run.buf.o_part, run.buf.lse_part, ws)
        assert ei.value.status == qsa.QSA_ERR_INVALID_ARG


def test_decode_shapes_back_to_back():
    # calls of different B, k and R in a row (different CTA splits and slice
    # layouts) sharing one scratch buffer, each checked against the oracle
    wl = make_custom(DIMS_FULL, [9000, 3001, 17, 40000], k=512, R=4, seed=109, device=DEV)
    run = CudaRun(wl)
    run.step()
    sel = run.buf.sel
    ws = torch.empty(max(qsa.qsa_sparse_decode_workspace_size(run.dims, B, k, R)
                         for B, k, R in ((4, 512, 4), (2, 512, 7), (4, 128, 1))),
                     dtype=torch.uint8, device=DEV)
    for B, k, R in ((4, 512, 4), (2, 512, 7), (4, 128, 1), (4, 512, 4), (2, 512, 7)):
        o = torch.full((R, B, run.dims.Hq, run.dims.D), float("nan"), device=DEV)
        lse = torch.full((R, B, run.dims.Hq), float("nan"), device=DEV)
        sl = run.seq_lens[:B]
        if k == 512:
            s_ = sel[:B]
        else:  # a smaller selection: the first k of every row, still ascending
            nb = [(L + 3) // 4 for L in wl.seq_lens[:B]]
            s_ = torch.stack([torch.arange(k, device=DEV, dtype=torch.int32) * max(1, n // k)
                              for n in nb]).contiguous()
            for b, n in enumerate(nb):
                if n < k:
                    s_[b, n:] = -1
                    s_[b, :n] = torch.arange(n, device=DEV, dtype=torch.int32)
        qsa.qsa_sparse_decode(run.dims, run.cache, sl, wl.q[:B].contiguous(), s_, k, R, o, lse,
                              ws)
        assert qsa.qsa_check_device_errors() == 0
        for b in range(B):
            ref = oracle_sequence(wl, b, k=k, R=R, sel=s_[b].cpu().numpy())
            check_attention(o[:, b].cpu().numpy(), lse[:, b].cpu().numpy(), ref["O_part"],
                            ref["LSE_part"], what=f"B={B} k={k} R={R} b={b}")


def test_empty_batch_is_a_no_op():
    d = qsa.QsaDims.of(DIMS_FULL)
    bt = torch.zeros((1, 1), dtype=torch.int32, device=DEV)
    cache = qsa.alloc_cache(d, 1, bt, device=DEV)
    buf = qsa.alloc_step(d, 1, 4, 8, 1, device=DEV)
    e = torch.empty(0, dtype=torch.int32, device=DEV)
    qsa.qsa_index_score(d, cache, e, buf.out[:0], buf.lse[:0], buf.scores[:0])
    qsa.qsa_topk_select(e, buf.scores[:0], 8, buf.sel[:0])
    qsa.qsa_merge(buf.o_part[:, :0], buf.lse_part[:, :0], buf.out[:0], buf.lse[:0])
    assert qsa.qsa_check_device_errors() == 0


# ------------------------------------------------------------ full-size presets

def _sampled(wl, n):
    B = wl.B
    idx = sorted({0, B - 1, *np.random.default_rng(wl.seed).choice(B, size=min(n, B),
                                                                   replace=False).tolist()})
    return idx


def test_b32x32k_full_size():
    wl = make_workload("b32x32k", device=DEV)
    run = CudaRun(wl)
    run.step()
    for b in _sampled(wl, 3):
        _check_seq(run, b)
    del run, wl
    torch.cuda.empty_cache()


def test_b8x256k_split_equals_unsplit():
    wl = make_workload("b8x256k", device=DEV)
    run = CudaRun(wl)
    run.step()
    for b in _sampled(wl, 2):
        _check_seq(run, b)
        assert set(wl.needles[b]) <= set(run.buf.sel[b].tolist())
    out4, lse4 = run.buf.out.float().clone(), run.buf.lse.clone()
    sel4 = run.buf.sel.clone()
    run.R = 1
    run.buf = qsa.alloc_step(run.dims, wl.B, run.ld, run.k, 1, device=DEV)
    run.step(append=False)
    assert torch.equal(run.buf.sel, sel4)
    d = (run.buf.out.float() - out4).abs().max().item()
    assert d <= 1e-2 and (run.buf.lse - lse4).abs().max().item() <= 1e-3
    del run, wl
    torch.cuda.empty_cache()


@pytest.mark.parametrize("R", [1, 2, 4, 8])
def test_ragged64_full_size(R):
    wl = make_workload("ragged64", device=DEV)
    run = CudaRun(wl, R=R)
    run.step()
    lens = np.array(wl.seq_lens)
    pick = {int(lens.argmin()), int(lens.argmax())}
    for res in (1, 2, 3):
        pick.add(int(np.nonzero(lens % 4 == res)[0][0]))
    pick.add(int(np.nonzero(lens < 2048)[0][0]))
    for b in sorted(pick):
        _check_seq(run, b, full=(R in (1, 8)) or b == min(pick))
    del run, wl
    torch.cuda.empty_cache()


def test_steady128x64k_append_steps():
    wl = make_workload("steady128x64k", device=DEV)
    spec_prefill, steps = wl.extra["prefill"], wl.extra["steps"]
    for k in (256, 512, 1024):
        run = CudaRun(wl, k=k, prefill=[spec_prefill] * wl.B)
        for t in range(steps):
            lens = [spec_prefill + t + 1] * wl.B
            q, q_idx, w = step_queries(wl, t)
            run.step(q=q, q_idx=q_idx, w=w, lens=lens)
            if t in (0, 3, steps - 1):
                for b in (0, 77):
                    _check_seq(run, b, L=lens[0], q=q[b], q_idx=q_idx[b], w=w[b],
                               full=(k == 512 or t == steps - 1))
        if k != 1024:
            del run
            torch.cuda.empty_cache()
    # after the 64 incremental steps, every sequence's side cache equals the
    # oracle's one-shot rebuild from its tokens
    L = spec_prefill + steps
    for b in range(wl.B):
        _, _, X = wl.seq_tokens(b, L)
        assert np.array_equal(run.side_rows(b, L), oracle.side_cache(bits(X), L)), b


@pytest.mark.parametrize("lens,R", [
    # sequences split over CTAs: the merge is fused into the combine; with
    # 2 <= R <= 8 and few sequences one CTA holds every slice of its heads
    # and merges them in shared memory (a 9-token sequence, whose one tile
    # lies in one decode CTA, has its partial from the decode kernel) ...
    ([30001, 5000, 77, 12345, 2048], 4),
    ([30001, 5000, 9, 12345, 2048], 3),
    ([30001, 5000, 77, 12345, 2048], 8),
    # ... with R = 1 every combine warp merges its own row ...
    ([70001, 9001, 9, 517], 1),
    # ... and beyond 8 slices, or with more combine CTAs than fit the GPU at
    # once, the CTA completing a row group's slices merges
    ([30001, 5000, 77, 12345, 2048], 16),
    ([30001, 5000, 77, 12345, 2048] * 16, 4),
    ([3000] * 300, 2),                     # one CTA per sequence: the merge kernel
])
def test_decode_step_fused_merge_equals_qsa_merge(lens, R):
    wl = make_custom(DIMS_FULL, lens, k=512, R=R, seed=len(lens) + R, device=DEV)
    run = CudaRun(wl)
    for out_dtype in (torch.bfloat16, torch.float32):
        run.buf.out = torch.full((wl.B, run.dims.Hq, run.dims.D), float("nan"), device=DEV,
                                 dtype=out_dtype)
        run.step()
        out2 = torch.full_like(run.buf.out, float("nan"))
        lse2 = torch.full_like(run.buf.lse, float("nan"))
        qsa.qsa_merge(run.buf.o_part, run.buf.lse_part, out2, lse2)
        assert qsa.qsa_check_device_errors() == 0
        assert torch.equal(run.buf.out.view(torch.int16 if out_dtype == torch.bfloat16
                                            else torch.int32),
                           out2.view(torch.int16 if out_dtype == torch.bfloat16 else torch.int32))
        assert torch.equal(run.buf.lse.view(torch.int32), lse2.view(torch.int32))
    for b in (0, 2, wl.B - 1):
        _check_seq(run, b)


@pytest.mark.parametrize("lens,R", [
    ([30001, 5000, 77, 12345, 2048, 262144], 4),  # clusters of 8 per selection
    ([9000, 2049, 40003, 3] * 10, 3),              # 40 rows: clusters of 4
    ([700, 3000, 1] * 2, 64),                      # more slices than some rows have blocks
])
def test_decode_step_slice_starts_equal_the_decode_kernels_own(lens, R):
    """Inside qsa_decode_step the top-k kernel hands each selection's slice
    starts to the decode kernel; a standalone qsa_sparse_decode finds them by
    binary search in the selection. Same starts mean the same tiles and
    slices, so the partials must be the same bits."""
    wl = make_custom(DIMS_FULL, lens, k=512, R=R, seed=len(lens) + 7 * R, device=DEV)
    run = CudaRun(wl)
    run.step()
    o2 = torch.full_like(run.buf.o_part, float("nan"))
    l2 = torch.full_like(run.buf.lse_part, float("nan"))
    qsa.qsa_sparse_decode(run.dims, run.cache, run.seq_lens, wl.q, run.buf.sel, run.k, run.R,
                          o2, l2, run.buf.ws)
    assert qsa.qsa_check_device_errors() == 0
    assert torch.equal(run.buf.o_part.view(torch.int32), o2.view(torch.int32))
    assert torch.equal(run.buf.lse_part.view(torch.int32), l2.view(torch.int32))
    for b in (0, len(lens) - 1):
        _check_seq(run, b)


# ------------------------------------------------------------ multi-query decode

@pytest.mark.parametrize("Qn,R", [(1, 4), (2, 1), (2, 4), (3, 8), (5, 2)])
def test_multi_query_decode_matches_oracle(Qn, R):
    # the Qn queries are the sequence's last Qn positions (all appended); each
    # sees the shared selection's tokens up to its own position. Lengths below
    # Qn leave the first queries with nothing to see (zeros, LSE = -inf).
    lens = [9001, 2050, 3, 40003, 1026, 13]
    wl = make_custom(DIMS_FULL, lens, k=256, R=R, seed=300 + 10 * Qn + R, device=DEV)
    run = CudaRun(wl)
    run.step()  # cache complete, selection of every sequence in run.buf.sel
    d = run.dims
    g = torch.Generator(device=DEV).manual_seed(Qn)
    q = torch.randn((wl.B, Qn, d.Hq, d.D), generator=g, device=DEV).to(torch.bfloat16)
    o = torch.full((R, wl.B, Qn, d.Hq, d.D), float("nan"), device=DEV)
    lse = torch.full((R, wl.B, Qn, d.Hq), float("nan"), device=DEV)
    ws = torch.empty(max(16, qsa.qsa_sparse_decode_mq_workspace_size(d, wl.B, Qn, wl.k, R)),
                     dtype=torch.uint8, device=DEV)
    qsa.qsa_sparse_decode_mq(d, run.cache, run.seq_lens, q, run.buf.sel, wl.k, R, o, lse, ws)
    out = torch.empty((wl.B * Qn, d.Hq, d.D), dtype=torch.float32, device=DEV)
    lse_m = torch.empty((wl.B * Qn, d.Hq), dtype=torch.float32, device=DEV)
    qsa.qsa_merge(o.view(R, wl.B * Qn, d.Hq, d.D), lse.view(R, wl.B * Qn, d.Hq), out, lse_m)
    assert qsa.qsa_check_device_errors() == 0
    o_np, l_np = o.cpu().numpy(), lse.cpu().numpy()
    om_np, lm_np = out.view(wl.B, Qn, d.Hq, d.D).cpu().numpy(), lse_m.view(wl.B, Qn, d.Hq).cpu().numpy()
    for b, L in enumerate(lens):
        K, V, _ = wl.seq_tokens(b)
        sel = run.buf.sel[b].cpu().numpy()
        O_ref, L_ref = oracle.attend_slices_mq(bits(q[b]), bits(K), bits(V), sel, L,
                                               wl.dims.scale, R)
        for j in range(Qn):
            check_attention(o_np[:, b, j], l_np[:, b, j], O_ref[:, j], L_ref[:, j],
                            what=f"Qn={Qn} R={R} b={b} query {j}")
            Om, Lm = oracle.merge_partials(O_ref[:, j], L_ref[:, j])
            check_attention(om_np[b, j], lm_np[b, j], Om, Lm,
                            what=f"merged Qn={Qn} R={R} b={b} query {j}")


# ------------------------------------------------------------ context parallel

@pytest.mark.parametrize("W", [2, 4])
def test_context_parallel_ranks_merge_to_full_attention(W):
    # one process emulates W ranks: rank r maps only the pages p = r mod W of
    # every sequence (the others -1), filters the shared selection to them,
    # decodes one slice over its own pages; the merge of the W partials is the
    # attention over the whole selection
    lens = [30001, 5000, 77, 12345, 2048]
    wl = make_custom(DIMS_FULL, lens, k=512, R=1, seed=400 + W, device=DEV)
    run = CudaRun(wl)
    run.step()
    d, B = run.dims, wl.B
    sel = run.buf.sel
    cols = torch.arange(run.cache.block_table.shape[1], device=DEV)
    O, L = [], []
    for r in range(W):
        bt = run.cache.block_table.clone()
        bt[:, (cols % W) != r] = -1
        cache_r = qsa.QsaCache(run.cache.k_pool, run.cache.v_pool, run.cache.kidx_pool,
                               run.cache.side_pool, bt)
        sel_r = torch.full_like(sel, -7)
        qsa.qsa_select_owned(sel, d.P, W, r, sel_r)
        for b in range(B):
            assert np.array_equal(sel_r[b].cpu().numpy(),
                                  oracle.owned_blocks(sel[b].cpu().numpy(), d.P, W, r)), (r, b)
        o_r = torch.empty((1, B, d.Hq, d.D), dtype=torch.float32, device=DEV)
        l_r = torch.empty((1, B, d.Hq), dtype=torch.float32, device=DEV)
        ws = torch.empty(max(16, qsa.qsa_sparse_decode_workspace_size(d, B, wl.k, 1)),
                         dtype=torch.uint8, device=DEV)
        qsa.qsa_sparse_decode(d, cache_r, run.seq_lens, wl.q, sel_r, wl.k, 1, o_r, l_r, ws)
        assert qsa.qsa_check_device_errors() == 0  # no page outside the rank's share was read
        O.append(o_r[0])
        L.append(l_r[0])
    out = torch.empty((B, d.Hq, d.D), dtype=torch.float32, device=DEV)
    lse = torch.empty((B, d.Hq), dtype=torch.float32, device=DEV)
    qsa.qsa_merge(torch.stack(O), torch.stack(L), out, lse)
    for b, Lb in enumerate(lens):
        K, V, _ = wl.seq_tokens(b)
        ref_o, ref_l = oracle.attend_slices(bits(wl.q[b]), bits(K), bits(V),
                                            sel[b].cpu().numpy(), Lb, wl.dims.scale, 1)
        check_attention(out[b].cpu().numpy(), lse[b].cpu().numpy(), ref_o[0], ref_l[0],
                        what=f"DCP W={W} b={b}")
