"""Pins of the CPU oracle against things other than itself.

Hand-worked fixtures, closed forms, brute force on tiny inputs, an
independently written dense attention (plus torch's SDPA in fp64), torch's
bf16 conversion, and the structural invariants the page implies (split read
plus combine equals the unsplit read; replicated selector; one cache group;
synthetic tokens write nothing).
"""

import itertools
import math

import numpy as np
import pytest
import torch

import oracle
from synth import make_custom, make_workload
from synth.workloads import Dims
from tests.helpers import bits, exact_bf16, golden

pytestmark = pytest.mark.filterwarnings("ignore")


# ------------------------------------------------------------ bf16 helpers

def test_bf16_rounding_matches_torch():
    g = torch.Generator().manual_seed(7)
    x = torch.randn(200000, generator=g) * torch.exp(torch.randn(200000, generator=g) * 8)
    special = torch.tensor([0.0, -0.0, 1.0, -1.0, 1.00390625, 1.01171875, 3.3895314e38,
                            float("inf"), float("-inf"), 1e-40, -1e-40, 65504.0],
                           dtype=torch.float32)
    x = torch.cat([x, special])
    ref = bits(x.to(torch.bfloat16))
    got = oracle.f32_to_bf16(x.numpy())
    assert np.array_equal(got, ref)
    back = oracle.bf16_to_f32(ref)
    assert np.array_equal(back, x.to(torch.bfloat16).to(torch.float32).numpy())


# ---------------------------------------------------- micro-block keys

def test_compress_hand_cases():
    d = golden("compress_rounding_hand.json")
    for case in d["cases"] + d["partial_cases"]:
        keys = exact_bf16(case["keys"]).reshape(len(case["keys"]), 1)
        got = int(oracle.compress_keys(keys)[0])
        assert got == int(case["bf16"], 16), case["derivation"]


def test_compress_within_one_ulp_of_exact_mean():
    g = np.random.default_rng(3)
    keys = oracle.f32_to_bf16(g.standard_normal((4096, 4, 64)).astype(np.float32))
    kc = oracle.bf16_to_f32(oracle.compress_keys(keys)).astype(np.float64)
    exact = oracle.bf16_to_f32(keys).astype(np.float64).mean(axis=1)
    ulp = np.ldexp(1.0, np.floor(np.log2(np.maximum(np.abs(exact), 1e-30))).astype(int) - 7)
    assert np.all(np.abs(kc - exact) <= ulp)


def test_side_cache_equals_blockwise_compress():
    g = np.random.default_rng(4)
    kidx = oracle.f32_to_bf16(g.standard_normal((403, 16)).astype(np.float32))
    side = oracle.side_cache(kidx, 403)
    assert side.shape == (100, 16)
    for j in (0, 1, 57, 99):
        assert np.array_equal(side[j], oracle.compress_keys(kidx[4 * j:4 * j + 4]))
    kc = oracle.block_keys(kidx, 403)
    assert kc.shape == (101, 16)
    tail = oracle.bf16_to_f32(oracle.compress_keys(kidx[400:403]))
    assert np.array_equal(kc[100], tail.astype(np.float64))


# ------------------------------------------------------------- scoring

def test_score_and_topk_hand():
    d = golden("score_topk_hand.json")
    kidx = exact_bf16(d["kidx"])
    q = exact_bf16(d["q_idx"])
    w = np.asarray(d["w"], dtype=np.float32)
    kc = oracle.block_keys(kidx, d["L"])
    assert np.array_equal(kc, np.asarray(d["kc"], dtype=np.float64))
    s = oracle.index_scores(kc, q, w)
    assert np.array_equal(s, np.asarray(d["scores"]))
    for k, sel in d["topk"].items():
        assert oracle.topk_blocks(s, int(k)).tolist() == sel
    full = oracle.decode_sequence(kidx, np.zeros((10, 1, 4), np.uint16),
                                  np.zeros((10, 1, 4), np.uint16), np.zeros((1, 4), np.uint16),
                                  q, w, d["L"], 2, 1, 1.0)
    assert full["sel"].tolist() == d["topk"]["2"]


def test_score_closed_form_single_head():
    # One head, w = 1: s_b = max(0, q . kc_b), checked with scalar loops.
    g = np.random.default_rng(5)
    kidx = oracle.f32_to_bf16(g.standard_normal((64, 8)).astype(np.float32))
    q = oracle.f32_to_bf16(g.standard_normal((1, 8)).astype(np.float32))
    kc = oracle.block_keys(kidx, 64)
    s = oracle.index_scores(kc, q, np.ones(1, np.float32))
    qf = oracle.bf16_to_f32(q)[0].astype(np.float64)
    for b in range(16):
        dot = sum(float(qf[i]) * float(kc[b, i]) for i in range(8))
        assert abs(s[b] - max(0.0, dot)) <= 1e-12 * (1 + abs(dot))


# ----------------------------------------------------------- selection

def _topk_by_beat_count(scores, k):
    """Brute force: block i is kept iff fewer than k blocks beat it, where j
    beats i if s_j > s_i, or s_j == s_i and j < i."""
    n = len(scores)
    keep = [i for i in range(n)
            if sum(1 for j in range(n) if scores[j] > scores[i]
                   or (scores[j] == scores[i] and j < i)) < k]
    return keep + [-1] * (k - len(keep))


def test_topk_ties_hand():
    for case in golden("topk_ties_hand.json")["cases"]:
        got = oracle.topk_blocks(np.asarray(case["scores"], dtype=np.float64), case["k"])
        assert got.tolist() == case["sel"], case["derivation"]


def test_topk_exhaustive_tiny():
    for nb in range(1, 8):
        for combo in itertools.product((0.0, 1.0, 2.0), repeat=nb):
            for k in range(1, nb + 2):
                assert oracle.topk_blocks(np.asarray(combo), k).tolist() == \
                    _topk_by_beat_count(list(combo), k)


def test_topk_random_with_ties():
    g = np.random.default_rng(6)
    for _ in range(300):
        nb = int(g.integers(1, 60))
        s = g.integers(0, 6, nb).astype(np.float64) * 0.5
        k = int(g.integers(1, 70))
        assert oracle.topk_blocks(s, k).tolist() == _topk_by_beat_count(s.tolist(), k)


def test_all_zero_index_keys_select_first_blocks():
    kidx = np.zeros((4099, 64), dtype=np.uint16)
    q = oracle.f32_to_bf16(np.random.default_rng(1).standard_normal((4, 64)).astype(np.float32))
    s = oracle.index_scores(oracle.block_keys(kidx, 4099), q, np.ones(4, np.float32))
    assert np.all(s == 0.0)
    assert oracle.topk_blocks(s, 512).tolist() == list(range(512))


def test_planted_needles_always_selected_tiny_preset():
    wl = make_workload("tiny", device="cpu")
    for b in range(wl.B):
        K, V, X = wl.seq_tokens(b)
        res = oracle.decode_sequence(bits(X), bits(K), bits(V), bits(wl.q[b]), bits(wl.q_idx[b]),
                                     wl.w[b].numpy(), wl.seq_lens[b], wl.k, wl.R, wl.dims.scale)
        sel = set(res["sel"].tolist())
        assert set(wl.needles[b]) <= sel
        s = res["scores"]
        assert min(s[j] for j in wl.needles[b]) > np.sort(s)[::-1][min(wl.k, len(s)) - 1]


def test_planted_needles_always_selected_mixture():
    d = Dims(Hq=8, Hkv=1, D=32, Hi=16, di=128, P=64, scale=1 / math.sqrt(32))
    wl = make_custom(d, [16384], k=512, R=4, seed=11, needles=8, mixture=True)
    K, V, X = wl.seq_tokens(0)
    kc = oracle.block_keys(bits(X), 16384)
    s = oracle.index_scores(kc, bits(wl.q_idx[0]), wl.w[0].numpy())
    sel = set(oracle.topk_blocks(s, 512).tolist())
    assert set(wl.needles[0]) <= sel


# ----------------------------------------------------------- attention

def _expr(e):
    return float(eval(e, {"e": math.e, "ln": math.log}))


def test_attention_hand():
    d = golden("attention_hand.json")
    q = exact_bf16(d["q"])
    K = exact_bf16(d["K"])
    V = exact_bf16(d["V"])
    sel = np.array([0, 1, -1])
    O1, L1 = oracle.attend_slices(q, K, V, sel, d["L"], d["scale"], 1)
    for h in range(2):
        assert abs(L1[0, h] - _expr(d["expr"]["R1"]["LSE"][h])) < 1e-12
        for c in range(2):
            assert abs(O1[0, h, c] - _expr(d["expr"]["R1"]["O"][h][c])) < 1e-12
    O2, L2 = oracle.attend_slices(q, K, V, sel, d["L"], d["scale"], 2)
    for r in range(2):
        for h in range(2):
            assert abs(L2[r, h] - _expr(d["expr"]["R2"]["LSE"][r][h])) < 1e-12
            for c in range(2):
                assert abs(O2[r, h, c] - _expr(d["expr"]["R2"]["O"][r][h][c])) < 1e-12
    Om, Lm = oracle.merge_partials(O2, L2)
    assert np.allclose(Om, O1[0], atol=1e-12) and np.allclose(Lm, L1[0], atol=1e-12)
    # selecting only the partial block: one token, LSE = z_4
    O3, L3 = oracle.attend_slices(q, K, V, np.array([1]), d["L"], d["scale"], 1)
    assert L3[0].tolist() == [2.0, 0.0] and O3[0].tolist() == [[4.0, -4.0], [4.0, -4.0]]


def _dense_loops(q, K, V, L, scale, G):
    """Textbook softmax attention with scalar loops (independent of the oracle)."""
    Hq, D = len(q), len(q[0])
    out, lses = [], []
    for h in range(Hq):
        g = h // G
        z = [scale * sum(q[h][d] * K[t][g][d] for d in range(D)) for t in range(L)]
        m = max(z)
        ex = [math.exp(v - m) for v in z]
        s = sum(ex)
        out.append([sum(ex[t] * V[t][g][d] for t in range(L)) / s for d in range(D)])
        lses.append(m + math.log(s))
    return np.array(out), np.array(lses)


def test_full_selection_equals_dense_attention_loops():
    d = Dims(Hq=4, Hkv=2, D=8, Hi=2, di=8, P=8, scale=0.35)
    wl = make_custom(d, [37], k=16, R=3, seed=12, paged=False)
    K, V, X = wl.seq_tokens(0)
    res = oracle.decode_sequence(bits(X), bits(K), bits(V), bits(wl.q[0]), bits(wl.q_idx[0]),
                                 wl.w[0].numpy(), 37, 16, 3, d.scale)
    assert res["sel"][:10].tolist() == list(range(10)) and np.all(res["sel"][10:] == -1)
    f = lambda t: t.to(torch.float64).tolist()
    O, LSE = _dense_loops(f(wl.q[0]), f(K), f(V), 37, d.scale, d.G)
    assert np.allclose(res["O"], O, atol=1e-12, rtol=0)
    assert np.allclose(res["LSE"], LSE, atol=1e-12, rtol=0)


def test_full_selection_equals_sdpa_fp64():
    # the tiny preset's 1500-token sequence has 375 < 512 blocks: all selected
    wl = make_workload("tiny", device="cpu")
    b, L = 1, wl.seq_lens[1]
    K, V, X = wl.seq_tokens(b)
    res = oracle.decode_sequence(bits(X), bits(K), bits(V), bits(wl.q[b]), bits(wl.q_idx[b]),
                                 wl.w[b].numpy(), L, wl.k, wl.R, wl.dims.scale)
    assert res["sel"][:375].tolist() == list(range(375))
    G = wl.dims.G
    qh = wl.q[b].to(torch.float64)[None, :, None, :]                   # [1, Hq, 1, D]
    Kh = K.to(torch.float64).repeat_interleave(G, dim=1).permute(1, 0, 2)[None]
    Vh = V.to(torch.float64).repeat_interleave(G, dim=1).permute(1, 0, 2)[None]
    ref = torch.nn.functional.scaled_dot_product_attention(qh, Kh, Vh, scale=wl.dims.scale)
    assert np.allclose(res["O"], ref[0, :, 0].numpy(), atol=1e-10, rtol=0)
    z = (qh @ Kh.transpose(-1, -2))[0, :, 0] * wl.dims.scale
    assert np.allclose(res["LSE"], torch.logsumexp(z, dim=-1).numpy(), atol=1e-10, rtol=0)


def test_split_merge_equals_unsplit():
    d = Dims(Hq=8, Hkv=2, D=32, Hi=4, di=32, P=16, scale=0.2)
    wl = make_custom(d, [997], k=40, R=1, seed=13, paged=False)
    K, V, X = wl.seq_tokens(0)
    args = (bits(wl.q[0]), bits(K), bits(V))
    sel = oracle.topk_blocks(oracle.index_scores(oracle.block_keys(bits(X), 997),
                                                 bits(wl.q_idx[0]), wl.w[0].numpy()), 40)
    O1, L1 = oracle.attend_slices(*args, sel, 997, d.scale, 1)
    for R in (2, 3, 4, 7, 8, 64):
        O, Ls = oracle.attend_slices(*args, sel, 997, d.scale, R)
        Om, Lm = oracle.merge_partials(O, Ls)
        assert np.abs(Om - O1[0]).max() <= 1e-12 and np.abs(Lm - L1[0]).max() <= 1e-12


def test_slice_bounds_hand():
    assert oracle.slice_bounds(10, 4) == [(0, 2), (2, 5), (5, 7), (7, 10)]
    assert oracle.slice_bounds(3, 4) == [(0, 0), (0, 1), (1, 2), (2, 3)]
    assert oracle.slice_bounds(7, 1) == [(0, 7)]


def test_q_zero_closed_form_per_slice():
    # q = 0: every z_t = 0, so LSE_r = ln(#valid tokens of slice r) and O_r is the
    # plain mean of those V rows. L = 41 -> nb = 11, R = 4 -> slices
    # [0,2) [2,5) [5,8) [8,11); block 10 holds only token 40.
    d = Dims(Hq=4, Hkv=2, D=16, Hi=2, di=16, P=16, scale=0.3)
    wl = make_custom(d, [41], k=11, R=4, seed=14, paged=False)
    K, V, _ = wl.seq_tokens(0)
    q0 = np.zeros((4, 16), np.uint16)
    sel = np.array([0, 3, 4, 5, 9, 10, -1])
    O, LSE = oracle.attend_slices(q0, bits(K), bits(V), sel, 41, d.scale, 4)
    counts = [4, 8, 4, 5]             # slice 0: block 0; 1: 3,4; 2: 5; 3: 9 + token 40
    toks = [[0, 1, 2, 3], list(range(12, 20)), list(range(20, 24)), [36, 37, 38, 39, 40]]
    Vf = V.to(torch.float64).numpy()
    for r in range(4):
        for h in range(4):
            assert abs(LSE[r, h] - math.log(counts[r])) < 1e-12
            assert np.allclose(O[r, h], Vf[toks[r], h // 2].mean(axis=0), atol=1e-12)


def test_constant_v_per_kv_head_gives_that_constant():
    d = Dims(Hq=8, Hkv=4, D=16, Hi=2, di=16, P=16, scale=0.3)
    wl = make_custom(d, [50], k=13, R=2, seed=15, paged=False)
    K, _, _ = wl.seq_tokens(0)
    consts = [1.5, -2.0, 0.25, 3.0]
    Vc = np.stack([exact_bf16([[c] * 16 for c in consts])] * 50)   # [50, Hkv, D]
    O, LSE = oracle.attend_slices(bits(wl.q[0]), bits(K), Vc, np.arange(13), 50, d.scale, 1)
    for h in range(8):
        assert np.allclose(O[0, h], consts[h // 2], atol=1e-12)


def test_single_token_closed_form():
    d = Dims(Hq=4, Hkv=1, D=16, Hi=2, di=16, P=16, scale=0.25)
    wl = make_custom(d, [1], k=4, R=2, seed=16, paged=False)
    K, V, X = wl.seq_tokens(0)
    res = oracle.decode_sequence(bits(X), bits(K), bits(V), bits(wl.q[0]), bits(wl.q_idx[0]),
                                 wl.w[0].numpy(), 1, 4, 2, d.scale)
    assert res["sel"].tolist() == [0, -1, -1, -1]
    q = wl.q[0].to(torch.float64).numpy()
    k0 = K[0, 0].to(torch.float64).numpy()
    for h in range(4):
        assert abs(res["LSE"][h] - d.scale * float(q[h] @ k0)) < 1e-12
        assert np.allclose(res["O"][h], V[0, 0].to(torch.float64).numpy(), atol=1e-12)
    # nb = 1 with R = 2: slice 0 owns no block, slice 1 owns block 0
    assert np.all(np.isneginf(res["LSE_part"][0])) and np.all(res["O_part"][0] == 0)


def test_merge_ignores_empty_slices():
    g = np.random.default_rng(8)
    O = g.standard_normal((3, 5, 4))
    LSE = g.standard_normal((3, 5))
    LSE[1, :] = -np.inf
    O[1] = 123.0
    Om, Lm = oracle.merge_partials(O, LSE)
    Om2, Lm2 = oracle.merge_partials(O[[0, 2]], LSE[[0, 2]])
    assert np.allclose(Om, Om2, atol=1e-14) and np.allclose(Lm, Lm2, atol=1e-14)
    Os, Ls = oracle.merge_partials(O[:1], LSE[:1])
    assert np.allclose(Os, O[0]) and np.allclose(Ls, LSE[0])
    # two equal-weight slices average; LSE grows by ln 2
    Oe, Le = oracle.merge_partials(np.stack([O[0], O[2]]), np.stack([LSE[0], LSE[0]]))
    assert np.allclose(Oe, (O[0] + O[2]) / 2) and np.allclose(Le, LSE[0] + math.log(2))


# ------------------------------------------------------------ paged append

def _pools(wl):
    d = wl.dims
    n = wl.num_pages
    rng = np.random.default_rng(99)   # stale garbage, so untouched bytes are visible
    mk = lambda *s: rng.integers(0, 1 << 16, size=s, dtype=np.uint16)
    return (mk(n, d.P, d.Hkv, d.D), mk(n, d.P, d.Hkv, d.D), mk(n, d.P, d.di),
            mk(n, d.P // 4, d.di))


def test_append_token_by_token_equals_one_shot():
    d = Dims(Hq=4, Hkv=2, D=8, Hi=2, di=8, P=16, scale=0.3)
    lens = [259, 64, 3, 100]
    wl = make_custom(d, lens, k=8, R=1, seed=17, paged=True)
    bt = wl.block_table.numpy()
    kp, vp, xp, sp = _pools(wl)
    kp2, vp2, xp2, sp2 = (a.copy() for a in (kp, vp, xp, sp))
    Kb, Vb, Xb = bits(wl.k_tok), bits(wl.v_tok), bits(wl.kidx_tok)
    # incremental: one call per decode step, one token per sequence
    for t in range(max(lens)):
        seqs = [b for b in range(4) if t < lens[b]]
        rows = [wl.tok_off[b] + t for b in seqs]
        oracle.append_paged(kp, vp, xp, sp, bt, d.P, seqs, [t] * len(seqs),
                            Kb[rows], Vb[rows], Xb[rows])
    # bulk: every token in one call, in a shuffled order
    order = np.random.default_rng(5).permutation(sum(lens))
    seq_of = np.concatenate([[b] * n for b, n in enumerate(lens)])
    pos_of = np.concatenate([np.arange(n) for n in lens])
    oracle.append_paged(kp2, vp2, xp2, sp2, bt, d.P, seq_of[order], pos_of[order],
                        Kb[order], Vb[order], Xb[order])
    for a, b in zip((kp, vp, xp, sp), (kp2, vp2, xp2, sp2)):
        assert np.array_equal(a, b)
    # side slots of every complete block equal the one-shot side cache
    for b, L in enumerate(lens):
        one_shot = oracle.side_cache(Xb[wl.tok_off[b]:wl.tok_off[b] + L], L)
        for j in range(L // 4):
            page = bt[b, (4 * j) // d.P]
            assert np.array_equal(sp[page, (4 * j % d.P) // 4], one_shot[j])
            assert np.array_equal(kp[page, 4 * j % d.P], Kb[wl.tok_off[b] + 4 * j])


def test_append_placement_by_hand():
    d = Dims(Hq=2, Hkv=1, D=8, Hi=1, di=8, P=8, scale=1.0)
    bt = np.array([[5, 2, -1], [0, 4, 1]])
    n = 6
    kp = np.zeros((n, 8, 1, 8), np.uint16)
    vp, xp, sp = kp.copy(), np.zeros((n, 8, 8), np.uint16), np.zeros((n, 2, 8), np.uint16)
    kv = np.arange(8, dtype=np.uint16).reshape(1, 1, 8) + 1
    # seq 1, position 13 -> page bt[1][1] = 4, slot 5
    oracle.append_paged(kp, vp, xp, sp, bt, d.P, [1], [13], kv, kv, kv[0])
    assert np.array_equal(kp[4, 5], kv[0]) and kp.sum() == kv.sum()
    # positions 4..7 of seq 0 close block 1 -> side page 5, slot 1
    x = exact_bf16([[1.0] * 8, [2.0] * 8, [2.0] * 8, [3.0] * 8])
    oracle.append_paged(kp, vp, xp, sp, bt, d.P, [0] * 4, [4, 5, 6, 7],
                        np.zeros((4, 1, 8), np.uint16), np.zeros((4, 1, 8), np.uint16), x)
    assert np.all(sp[5, 1] == 0x4000) and sp.sum() == 8 * 0x4000   # mean 2.0


def test_padding_tokens_write_nothing():
    d = Dims(Hq=4, Hkv=2, D=8, Hi=2, di=8, P=16, scale=0.3)
    wl = make_custom(d, [40, 40], k=8, R=1, seed=18, paged=True)
    bt = wl.block_table.numpy()
    pools = _pools(wl)
    before = [a.copy() for a in pools]
    K, V, X = bits(wl.k_tok[:4]), bits(wl.v_tok[:4]), bits(wl.kidx_tok[:4])
    oracle.append_paged(*pools, bt, d.P, [-1, 0, -1, 1], [3, -1, 7, -5], K, V, X)
    for a, b in zip(pools, before):
        assert np.array_equal(a, b)


# ------------------------------------------------------------ multi-query decode

def _mq_case(L, Q, seed, D=32, Hq=8, Hkv=2):
    g = torch.Generator().manual_seed(seed)
    K = torch.randn(L, Hkv, D, generator=g).to(torch.bfloat16)
    V = torch.randn(L, Hkv, D, generator=g).to(torch.bfloat16)
    q = torch.randn(Q, Hq, D, generator=g).to(torch.bfloat16)
    return q, K, V


@pytest.mark.parametrize("L,Q", [(37, 1), (37, 2), (40, 3), (5, 4), (1000, 2)])
def test_multi_query_full_selection_equals_masked_sdpa_fp64(L, Q):
    # every block selected, one slice: query j is dense attention over the
    # tokens t <= L - Q + j (a bottom-right causal mask), by torch's SDPA
    q, K, V = _mq_case(L, Q, seed=L * 10 + Q)
    nb = (L + 3) // 4
    scale = 0.17
    O, LSE = oracle.attend_slices_mq(bits(q), bits(K), bits(V), np.arange(nb), L, scale, 1)
    Hq, G = q.shape[1], q.shape[1] // K.shape[1]
    qh = q.to(torch.float64).permute(1, 0, 2)[None]                          # [1, Hq, Q, D]
    Kh = K.to(torch.float64).repeat_interleave(G, dim=1).permute(1, 0, 2)[None]
    Vh = V.to(torch.float64).repeat_interleave(G, dim=1).permute(1, 0, 2)[None]
    mask = torch.arange(L)[None, :] <= (L - Q + torch.arange(Q))[:, None]   # [Q, L]
    ref = torch.nn.functional.scaled_dot_product_attention(qh, Kh, Vh, attn_mask=mask,
                                                           scale=scale)
    assert np.allclose(O[0], ref[0].permute(1, 0, 2).numpy(), atol=1e-10, rtol=0)
    z = (qh @ Kh.transpose(-1, -2)) * scale
    z = z.masked_fill(~mask, float("-inf"))
    assert np.allclose(LSE[0], torch.logsumexp(z, dim=-1)[0].T.numpy(), atol=1e-10, rtol=0)


def test_multi_query_split_merge_equals_unsplit_and_hides_future_blocks():
    L, Q = 203, 3
    q, K, V = _mq_case(L, Q, seed=5)
    nb = (L + 3) // 4
    sel = np.array([0, 3, 7, 20, 33, 49, nb - 1])  # the last block holds the queries' tokens
    O1, L1 = oracle.attend_slices_mq(bits(q), bits(K), bits(V), sel, L, 0.2, 1)
    for R in (2, 5, 51):
        O, Ls = oracle.attend_slices_mq(bits(q), bits(K), bits(V), sel, L, 0.2, R)
        for j in range(Q):
            Om, Lm = oracle.merge_partials(O[:, j], Ls[:, j])
            assert np.abs(Om - O1[0, j]).max() <= 1e-12
            assert np.abs(Lm - L1[0, j]).max() <= 1e-12
    # R = nb: the last slice is exactly the last block {200, 201, 202}: query 0
    # (position 200) sees one token of it, query 2 all three; a slice holding
    # only tokens after a query is empty for that query
    O, Ls = oracle.attend_slices_mq(bits(q), bits(K), bits(V), np.array([nb - 1]), L, 0.2, nb)
    assert np.all(Ls[: nb - 1] == -np.inf)
    assert np.all(np.isfinite(Ls[nb - 1]))
    Lq, Kq = 201, K[:201]
    O0, L0 = oracle.attend_slices(bits(q[0]), bits(Kq), bits(V[:201]), np.array([50]), Lq, 0.2, 1)
    assert np.abs(O[nb - 1, 0] - O0[0]).max() <= 1e-12   # query 0 = single query over t < 201


# ------------------------------------------------------------ context parallel

@pytest.mark.parametrize("W,P", [(2, 64), (4, 64), (3, 32), (8, 16)])
def test_owned_blocks_partition_the_selection(W, P):
    g = np.random.default_rng(W * 100 + P)
    sel = np.sort(g.choice(5000, size=300, replace=False))
    sel = np.concatenate([sel, -np.ones(20, dtype=np.int64)])
    parts = [oracle.owned_blocks(sel, P, W, r) for r in range(W)]
    got = np.sort(np.concatenate([p[p >= 0] for p in parts]))
    assert np.array_equal(got, sel[sel >= 0])          # every block on exactly one rank
    for r, p in enumerate(parts):
        live = p[p >= 0]
        assert np.all(np.diff(live) > 0) and np.all(p[len(live):] == -1)
        assert np.all(((4 * live) // P) % W == r)      # by its page


def test_owned_blocks_hand():
    for case in golden("owned_blocks_hand.json")["cases"]:
        sel = np.asarray(case["sel"], dtype=np.int64)
        for r in range(case["W"]):
            got = oracle.owned_blocks(sel, case["P"], case["W"], r)
            assert got.tolist() == case["owned"][r], (case["derivation"], r)


def test_owned_blocks_fixture_catches_plausible_mistakes():
    # the hand fixture would reject an owner rule that ranks by block index,
    # or that forgets the 4 tokens per block when finding the page
    wrong_rules = [lambda j, P, W: j % W,
                   lambda j, P, W: (j // P) % W,
                   lambda j, P, W: ((4 * j) // P) % (W + 1)]
    for rule in wrong_rules:
        caught = False
        for case in golden("owned_blocks_hand.json")["cases"]:
            P, W = case["P"], case["W"]
            for r in range(W):
                own = [j for j in case["sel"] if j >= 0 and rule(j, P, W) == r]
                if own + [-1] * (len(case["sel"]) - len(own)) != case["owned"][r]:
                    caught = True
        assert caught


def test_context_parallel_merge_equals_single_rank_attention():
    # each rank attends over its own pages' share of the one selection; the
    # LSE-weighted merge of the W partials is the attention over all of it
    d = Dims(Hq=8, Hkv=2, D=32, Hi=4, di=32, P=16, scale=0.2)
    wl = make_custom(d, [1501], k=64, R=1, seed=21, paged=False)
    K, V, X = wl.seq_tokens(0)
    args = (bits(wl.q[0]), bits(K), bits(V))
    sel = oracle.topk_blocks(oracle.index_scores(oracle.block_keys(bits(X), 1501),
                                                 bits(wl.q_idx[0]), wl.w[0].numpy()), 64)
    O1, L1 = oracle.attend_slices(*args, sel, 1501, d.scale, 1)
    for W in (2, 3, 4):
        parts = [oracle.attend_slices(*args, oracle.owned_blocks(sel, d.P, W, r), 1501,
                                      d.scale, 1) for r in range(W)]
        Om, Lm = oracle.merge_partials(np.stack([o[0] for o, _ in parts]),
                                       np.stack([l[0] for _, l in parts]))
        assert np.abs(Om - O1[0]).max() <= 1e-12 and np.abs(Lm - L1[0]).max() <= 1e-12


# ------------------------------------------------------------ sparse prefill

def test_prefill_rows_hand():
    # sequence 0: L=10, 3 chunk rows at positions 7, 8, 9; sequence 1: L=7,
    # rows at 5, 6; sequence 2: no rows; sequence 3: the whole context is the chunk
    row_seq, row_len = oracle.prefill_rows([10, 7, 3, 3], [0, 3, 5, 5, 8])
    assert row_seq.tolist() == [0, 0, 0, 1, 1, 3, 3, 3]
    assert row_len.tolist() == [8, 9, 10, 6, 7, 1, 2, 3]


def _prefill_case(L, T, seed, D=32, Hq=8, Hkv=2, Hi=3, di=16):
    g = torch.Generator().manual_seed(seed)
    K = torch.randn(L, Hkv, D, generator=g).to(torch.bfloat16)
    V = torch.randn(L, Hkv, D, generator=g).to(torch.bfloat16)
    X = torch.randn(L, di, generator=g).to(torch.bfloat16)
    q = torch.randn(T, Hq, D, generator=g).to(torch.bfloat16)
    qi = torch.randn(T, Hi, di, generator=g).to(torch.bfloat16)
    w = torch.rand(T, Hi, generator=g)
    return K, V, X, q, qi, w


@pytest.mark.parametrize("L,T", [(45, 9), (13, 13), (40, 1), (7, 3)])
def test_prefill_dense_when_k_covers_the_context(L, T):
    # k >= every row's block count: each row attends densely over its own
    # causal prefix, i.e. a bottom-right causal mask over the chunk, by SDPA
    K, V, X, q, qi, w = _prefill_case(L, T, seed=L * 100 + T)
    scale = 0.21
    rows = oracle.prefill_sequence(bits(X), bits(K), bits(V), bits(q), bits(qi), w.numpy(), L, T,
                                   k=64, R=1, scale=scale)
    G = q.shape[1] // K.shape[1]
    qh = q.to(torch.float64).permute(1, 0, 2)[None]                          # [1, Hq, T, D]
    Kh = K.to(torch.float64).repeat_interleave(G, dim=1).permute(1, 0, 2)[None]
    Vh = V.to(torch.float64).repeat_interleave(G, dim=1).permute(1, 0, 2)[None]
    mask = torch.arange(L)[None, :] <= (L - T + torch.arange(T))[:, None]   # [T, L]
    ref = torch.nn.functional.scaled_dot_product_attention(qh, Kh, Vh, attn_mask=mask, scale=scale)
    z = ((qh @ Kh.transpose(-1, -2)) * scale).masked_fill(~mask, float("-inf"))
    lse = torch.logsumexp(z, dim=-1)[0].T.numpy()                           # [T, Hq]
    for i, r in enumerate(rows):
        assert np.allclose(r["O"], ref[0, :, i].numpy(), atol=1e-10, rtol=0)
        assert np.allclose(r["LSE"], lse[i], atol=1e-10, rtol=0)
        assert r["sel"][r["sel"] >= 0].tolist() == list(range((L - T + i + 1 + 3) // 4))


def _brute_row_scores(X, qi_row, w_row, ell):
    # the score definition written out with loops: block b holds tokens
    # 4b..4b+3 that are < ell; its key is the bf16 rounding of the fp32
    # left-to-right sum of those keys divided by their count
    Xf = X.to(torch.float32)
    out = []
    for b in range((ell + 3) // 4):
        toks = [t for t in range(4 * b, 4 * b + 4) if t < ell]
        acc = Xf[toks[0]].clone()
        for t in toks[1:]:
            acc = acc + Xf[t]
        kc = (acc / float(len(toks))).to(torch.bfloat16).to(torch.float64)
        s = 0.0
        for h in range(qi_row.shape[0]):
            dot = float((qi_row[h].to(torch.float64) * kc).sum())
            s += float(w_row[h]) * max(0.0, dot)
        out.append(s)
    return np.array(out)


def test_prefill_row_scores_by_brute_force():
    L, T = 23, 6   # rows see 18..23 tokens: partial blocks of every size
    K, V, X, q, qi, w = _prefill_case(L, T, seed=99)
    rows = oracle.prefill_sequence(bits(X), bits(K), bits(V), bits(q), bits(qi), w.numpy(), L, T,
                                   k=3, R=2, scale=0.3)
    for i, r in enumerate(rows):
        ref = _brute_row_scores(X, qi[i], w[i], L - T + i + 1)
        assert r["scores"].shape == ref.shape
        assert np.allclose(r["scores"], ref, rtol=1e-12, atol=1e-12)


def test_prefill_rows_ignore_later_tokens():
    L, T = 61, 5
    K, V, X, q, qi, w = _prefill_case(L, T, seed=7)
    args = dict(L=L, T=T, k=4, R=3, scale=0.25)
    base = oracle.prefill_sequence(bits(X), bits(K), bits(V), bits(q), bits(qi), w.numpy(), **args)
    for i in range(T):
        pos = L - T + i
        K2, V2, X2 = K.clone(), V.clone(), X.clone()
        K2[pos + 1:] = -K2[pos + 1:] * 3
        V2[pos + 1:] = V2[pos + 1:] + 5
        X2[pos + 1:] = -X2[pos + 1:]
        got = oracle.prefill_sequence(bits(X2), bits(K2), bits(V2), bits(q), bits(qi), w.numpy(),
                                      **args)
        assert np.array_equal(got[i]["sel"], base[i]["sel"])
        assert np.array_equal(got[i]["scores"], base[i]["scores"])
        assert np.array_equal(got[i]["O"], base[i]["O"])
        if i + 1 < T:   # a later row sees the change
            assert not np.array_equal(got[T - 1]["O"], base[T - 1]["O"])


def test_prefill_rows_split_merge_equals_unsplit():
    # each row's R partials merged equal its one-slice result (fp64 rounding)
    L, T = 97, 7
    K, V, X, q, qi, w = _prefill_case(L, T, seed=31)
    one = oracle.prefill_sequence(bits(X), bits(K), bits(V), bits(q), bits(qi), w.numpy(), L, T,
                                  k=9, R=1, scale=0.3)
    for R in (2, 3, 8):
        rows = oracle.prefill_sequence(bits(X), bits(K), bits(V), bits(q), bits(qi), w.numpy(), L,
                                       T, k=9, R=R, scale=0.3)
        for a, b in zip(rows, one):
            assert np.array_equal(a["sel"], b["sel"])
            Om, Lm = oracle.merge_partials(a["O_part"], a["LSE_part"])
            assert np.abs(Om - b["O"]).max() <= 1e-12
            assert np.abs(Lm - b["LSE"]).max() <= 1e-12
