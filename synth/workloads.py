"""Seeded, synthetic QSA decode workloads.

Shapes follow the long-context serving setting described on the page
"Qwen 4 QSA gets decode context parallelism: inside vLLM's draft PR for
Qwen3.8-Flash-Next" (orcarouter.ai), sections "What the pull request actually
changes" (micro-blocks of 4 keys, best 512 blocks) and "Why a serving PR ... is
still worth your time" (262,144-token native context). The page fixes no head
counts or value distributions; the five presets below are this library's
test and benchmark workloads:

  tiny           B=2, L = 4099 and 1500, 8 q / 2 kv heads, indexer 4 x 64,
                 contiguous cache, 3 planted needle blocks per sequence,
                 k=512, R=2
  b32x32k        B=32 x 32,768 tokens, 32 q / 4 kv heads, indexer 16 x 128,
                 paged (P=64, shuffled pages), k=512, R=1
  b8x256k        B=8 x 262,144 tokens, heads as b32x32k, indexer keys and K
                 drawn from a 90/10 mixture (N(0,I), N(0,I) + 3u), 8 planted
                 needles, k=512, R=4
  ragged64       B=64 ragged, L log-uniform in [1,024, 262,144], k=512,
                 R in {1,2,4,8}
  steady128x64k  B=128, 65,536-token prefill then 64 decode steps,
                 k in {256,512,1024}, R=4

Everything is drawn in fp32 from one ``torch.Generator`` per tensor stream and
rounded to bf16 by torch's round-to-nearest-even conversion. Nothing in this
module computes any part of the decode step itself.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

PRESETS = ("tiny", "b32x32k", "b8x256k", "ragged64", "steady128x64k")
BASE_SEED = 20261202

# RNG stream ids, in the fixed order the tensors are drawn.
_S_LENS, _S_K, _S_V, _S_KIDX, _S_Q, _S_QIDX, _S_W, _S_PAGES, _S_NEEDLE, _S_MIX = range(10)
_S_STEP = 100  # + step index: per-step queries of the append workload
_S_PREFILL = 90  # query rows of a prefill chunk


def seed_for(preset: str) -> int:
    """Base seed of a preset (fixed, so every run draws the same bytes)."""
    return BASE_SEED + 1 + PRESETS.index(preset)


@dataclass(frozen=True)
class Dims:
    """Head geometry. Hq query heads share Hkv KV heads (GQA group G = Hq/Hkv);
    the indexer has Hi heads of width di; P tokens per cache page."""

    Hq: int
    Hkv: int
    D: int
    Hi: int
    di: int
    P: int
    scale: float

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv


DIMS_TINY = Dims(Hq=8, Hkv=2, D=128, Hi=4, di=64, P=64, scale=1.0 / math.sqrt(128.0))
DIMS_FULL = Dims(Hq=32, Hkv=4, D=128, Hi=16, di=128, P=64, scale=1.0 / math.sqrt(128.0))


@dataclass
class Workload:
    """One decode batch plus the token history behind it.

    Token t of sequence b lives at row ``tok_off[b] + t`` of the flattened
    per-token arrays. ``seq_lens[b]`` is the context length L_b *after* the
    current token (position L_b - 1) is appended; ``cap_lens[b] >= seq_lens[b]``
    tokens are drawn (the append workload draws its future tokens up front).
    ``block_table[b, j]`` is the physical page holding tokens
    [j*P, (j+1)*P) of sequence b; unused entries are -1.
    """

    name: str
    seed: int
    dims: Dims
    seq_lens: list
    cap_lens: list
    k: int
    R: int
    tok_off: list
    k_tok: torch.Tensor
    v_tok: torch.Tensor
    kidx_tok: torch.Tensor
    q: torch.Tensor
    q_idx: torch.Tensor
    w: torch.Tensor
    block_table: torch.Tensor
    num_pages: int
    needles: list = field(default_factory=list)
    extra: dict = field(default_factory=dict)

    @property
    def B(self) -> int:
        return len(self.seq_lens)

    @property
    def max_pages(self) -> int:
        return int(self.block_table.shape[1])

    def seq_tokens(self, b: int, n: int | None = None):
        """(K, V, kidx) rows of sequence b, first n tokens (default L_b)."""
        n = self.seq_lens[b] if n is None else n
        o = self.tok_off[b]
        return self.k_tok[o:o + n], self.v_tok[o:o + n], self.kidx_tok[o:o + n]


def _gen(device, seed: int, stream: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed * 1009 + stream)
    return g


def _randn_bf16(shape, gen, device, chunk_rows=1 << 20):
    """N(0,1) in fp32, rounded to bf16, drawn in row chunks to bound temporaries."""
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    rows = shape[0]
    for r0 in range(0, rows, chunk_rows):
        r1 = min(rows, r0 + chunk_rows)
        out[r0:r1] = torch.randn((r1 - r0,) + tuple(shape[1:]), generator=gen,
                                 device=device, dtype=torch.float32).to(torch.bfloat16)
    return out


def _mixture_bf16(shape, gen, device, p=0.1, amp=3.0, chunk_rows=1 << 20):
    """Per row: N(0,I) with prob 1-p, N(0,I) + amp*u with prob p, where u is one
    unit vector (over the last dimension) fixed for the whole tensor."""
    last = shape[-1]
    u = torch.randn(last, generator=gen, device=device, dtype=torch.float32)
    u = u / u.norm()
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    rows = shape[0]
    for r0 in range(0, rows, chunk_rows):
        r1 = min(rows, r0 + chunk_rows)
        x = torch.randn((r1 - r0,) + tuple(shape[1:]), generator=gen, device=device,
                        dtype=torch.float32)
        pick = torch.rand((r1 - r0,), generator=gen, device=device) < p
        pick = pick.view((r1 - r0,) + (1,) * (len(shape) - 1)).to(torch.float32)
        out[r0:r1] = (x + amp * pick * u).to(torch.bfloat16)
    return out


def _page_table(cap_lens, P, gen, device, shuffle: bool):
    pages = [(c + P - 1) // P for c in cap_lens]
    total = sum(pages)
    if shuffle:
        perm = torch.randperm(total, generator=gen, device=device).to(torch.int32)
    else:
        perm = torch.arange(total, device=device, dtype=torch.int32)
    width = max(pages)
    bt = torch.full((len(cap_lens), width), -1, dtype=torch.int32, device=device)
    c = 0
    for b, n in enumerate(pages):
        bt[b, :n] = perm[c:c + n]
        c += n
    return bt, total


def _plant_needles(wl: Workload, n_needles: int, gen_device):
    """Overwrite the indexer keys of n_needles complete blocks per sequence with
    bf16(4 * mean over indexer heads of that sequence's indexer query)."""
    g = _gen(gen_device, wl.seed, _S_NEEDLE)
    needles = []
    for b, L in enumerate(wl.seq_lens):
        n_complete = L // 4
        hi = max(1, n_complete - 1)  # keep clear of the block holding the newest tokens
        cand = torch.randperm(hi, generator=g, device=gen_device)[:n_needles].tolist()
        cand = sorted(int(j) for j in cand)
        key = (4.0 * wl.q_idx[b].to(torch.float32).mean(dim=0)).to(torch.bfloat16)
        o = wl.tok_off[b]
        for j in cand:
            wl.kidx_tok[o + 4 * j:o + 4 * j + 4] = key
        needles.append(cand)
    wl.needles = needles


def _lens_ragged64(seed):
    g = _gen("cpu", seed, _S_LENS)
    u = torch.rand(64, generator=g, dtype=torch.float64)
    lo, hi = math.log(1024.0), math.log(262144.0)
    lens = [int(round(math.exp(lo + (hi - lo) * float(x)))) for x in u]
    lens = [min(262144, max(1024, x)) for x in lens]
    for i, res in ((0, 1), (1, 2), (2, 3)):
        if not any(x % 4 == res for x in lens):
            x = lens[i] - (lens[i] % 4) + res
            lens[i] = x if x <= 262144 else x - 4
    if not any(x < 2048 for x in lens):
        u2 = float(torch.rand(1, generator=g, dtype=torch.float64))
        x = int(round(math.exp(lo + (math.log(2048.0) - lo) * u2)))
        x = min(2047, max(1024, x))
        if x % 4 == 0:
            x += 1
        lens[3] = x
    return lens


def preset_spec(preset: str) -> dict:
    """Sizes of a preset, without drawing anything."""
    if preset == "tiny":
        return dict(dims=DIMS_TINY, seq_lens=[4099, 1500], k=512, R=2, paged=False,
                    needles=3, mixture=False)
    if preset == "b32x32k":
        return dict(dims=DIMS_FULL, seq_lens=[32768] * 32, k=512, R=1, paged=True,
                    needles=0, mixture=False)
    if preset == "b8x256k":
        return dict(dims=DIMS_FULL, seq_lens=[262144] * 8, k=512, R=4, paged=True,
                    needles=8, mixture=True)
    if preset == "ragged64":
        return dict(dims=DIMS_FULL, seq_lens=_lens_ragged64(seed_for(preset)), k=512, R=4,
                    paged=True, needles=0, mixture=False, R_sweep=(1, 2, 4, 8))
    if preset == "steady128x64k":
        return dict(dims=DIMS_FULL, seq_lens=[65537] * 128, cap_lens=[65536 + 64] * 128,
                    k=512, R=4, paged=True, needles=0, mixture=False,
                    k_sweep=(256, 512, 1024), prefill=65536, steps=64)
    raise ValueError(f"unknown preset {preset!r}; known: {', '.join(PRESETS)}")


def make_custom(dims: Dims, seq_lens, k: int, R: int, seed: int, device="cpu",
                paged: bool = True, needles: int = 0, mixture: bool = False,
                cap_lens=None, name: str = "custom", pool_slack_pages: int = 0) -> Workload:
    """Draw a workload of arbitrary size (used by the presets and by small tests)."""
    device = torch.device(device)
    seq_lens = [int(x) for x in seq_lens]
    cap_lens = [int(x) for x in (cap_lens or seq_lens)]
    assert all(c >= L >= 1 for c, L in zip(cap_lens, seq_lens))
    B = len(seq_lens)
    tok_off, c = [], 0
    for n in cap_lens:
        tok_off.append(c)
        c += n
    T = c
    gk, gv, gx = _gen(device, seed, _S_K), _gen(device, seed, _S_V), _gen(device, seed, _S_KIDX)
    if mixture:
        k_tok = _mixture_bf16((T, dims.Hkv, dims.D), gk, device)
        kidx_tok = _mixture_bf16((T, dims.di), gx, device)
    else:
        k_tok = _randn_bf16((T, dims.Hkv, dims.D), gk, device)
        kidx_tok = _randn_bf16((T, dims.di), gx, device)
    v_tok = _randn_bf16((T, dims.Hkv, dims.D), gv, device)
    q = torch.randn((B, dims.Hq, dims.D), generator=_gen(device, seed, _S_Q), device=device,
                    dtype=torch.float32).to(torch.bfloat16)
    q_idx = torch.randn((B, dims.Hi, dims.di), generator=_gen(device, seed, _S_QIDX),
                        device=device, dtype=torch.float32).to(torch.bfloat16)
    w = torch.rand((B, dims.Hi), generator=_gen(device, seed, _S_W), device=device,
                   dtype=torch.float32)
    bt, num_pages = _page_table(cap_lens, dims.P, _gen(device, seed, _S_PAGES), device, paged)
    wl = Workload(name=name, seed=seed, dims=dims, seq_lens=seq_lens,
                  cap_lens=cap_lens, k=k, R=R, tok_off=tok_off, k_tok=k_tok, v_tok=v_tok,
                  kidx_tok=kidx_tok, q=q, q_idx=q_idx, w=w, block_table=bt,
                  num_pages=num_pages + pool_slack_pages)
    if needles:
        _plant_needles(wl, needles, device)
    return wl


def make_workload(preset: str, device="cpu", seed: int | None = None) -> Workload:
    """Draw one of ``PRESETS`` on ``device``."""
    spec = preset_spec(preset)
    seed = seed_for(preset) if seed is None else seed
    wl = make_custom(spec["dims"], spec["seq_lens"], spec["k"], spec["R"], seed, device,
                     paged=spec["paged"], needles=spec["needles"], mixture=spec["mixture"],
                     cap_lens=spec.get("cap_lens"), name=preset)
    wl.extra = {k: v for k, v in spec.items()
                if k in ("R_sweep", "k_sweep", "prefill", "steps")}
    return wl


def step_queries(wl: Workload, t: int):
    """(q, q_idx, w) for decode step t of an append workload, one draw per step."""
    d, dev, B = wl.dims, wl.q.device, wl.B
    g = _gen(dev, wl.seed, _S_STEP + t)
    q = torch.randn((B, d.Hq, d.D), generator=g, device=dev).to(torch.bfloat16)
    q_idx = torch.randn((B, d.Hi, d.di), generator=g, device=dev).to(torch.bfloat16)
    w = torch.rand((B, d.Hi), generator=g, device=dev)
    return q, q_idx, w


def prefill_queries(wl: Workload, chunk_lens, seed: int | None = None):
    """Query rows of a sparse prefill whose chunks are the chunk_lens[s]
    newest tokens of each sequence (already part of seq_lens[s]): returns
    (row_start int32 [S + 1], q [Nq, Hq, D], q_idx [Nq, Hi, di], w [Nq, Hi]),
    rows in chunk order, one draw per tensor (N(0, 1) rounded to bf16, w from
    U(0, 1) as for decode queries)."""
    d, dev = wl.dims, wl.q.device
    chunk_lens = [int(x) for x in chunk_lens]
    assert len(chunk_lens) == wl.B
    assert all(0 <= T <= L for T, L in zip(chunk_lens, wl.seq_lens))
    row_start = [0]
    for T in chunk_lens:
        row_start.append(row_start[-1] + T)
    Nq = row_start[-1]
    g = _gen(dev, wl.seed if seed is None else seed, _S_PREFILL)
    q = torch.randn((Nq, d.Hq, d.D), generator=g, device=dev).to(torch.bfloat16)
    q_idx = torch.randn((Nq, d.Hi, d.di), generator=g, device=dev).to(torch.bfloat16)
    w = torch.rand((Nq, d.Hi), generator=g, device=dev)
    return torch.tensor(row_start, dtype=torch.int32, device=dev), q, q_idx, w
