"""Test-harness helpers: tensor <-> bit-pattern conversion and comparisons.

Nothing here computes any part of the decode step; the comparisons only
decide whether two results agree within the stated tolerances.
"""

from __future__ import annotations

import json
import os

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")

# Parity bar for floating-point outputs (bf16 inputs, fp32 accumulation).
ATTN_MAX_ABS = 1e-2
ATTN_REL_L2 = 5e-3
LSE_MAX_ABS = 1e-3
# Near-tie band for selection: a set difference is allowed only for blocks whose
# oracle score lies within this relative distance of the k-th best score.
SEL_TIE_REL = 1e-3


def golden(name: str) -> dict:
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> numpy uint16 bit patterns (host copy)."""
    assert t.dtype == torch.bfloat16
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def from_bits(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)


def exact_bf16(values) -> np.ndarray:
    """Bit patterns of values that bf16 represents exactly (asserted)."""
    x = torch.tensor(values, dtype=torch.float64)
    b = x.to(torch.bfloat16)
    assert torch.equal(b.to(torch.float64), x), "fixture value not exact in bf16"
    return bits(b)


def bf16_same(a, b) -> bool:
    """Bit-equal bf16 arrays, except that any two NaNs count as equal (a NaN's
    payload depends on the hardware's NaN propagation, not on the method)."""
    a = np.asarray(a, dtype=np.uint16)
    b = np.asarray(b, dtype=np.uint16)
    nan_a = (a & 0x7FFF) > 0x7F80
    nan_b = (b & 0x7FFF) > 0x7F80
    return bool(np.array_equal(nan_a, nan_b) and np.array_equal(a[~nan_a], b[~nan_b]))


def rel_l2(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    den = np.linalg.norm(b.ravel())
    return float(np.linalg.norm((a - b).ravel()) / max(den, 1e-300))


def check_attention(o_gpu, lse_gpu, o_ref, lse_ref, what=""):
    """Assert the attention parity bar; returns (max_abs, rel_l2, lse_abs)."""
    o_gpu = np.asarray(o_gpu, dtype=np.float64)
    o_ref = np.asarray(o_ref, dtype=np.float64)
    lse_gpu = np.asarray(lse_gpu, dtype=np.float64)
    lse_ref = np.asarray(lse_ref, dtype=np.float64)
    fin = np.isfinite(lse_ref)
    assert np.array_equal(fin, np.isfinite(lse_gpu)), f"{what}: -inf pattern of LSE differs"
    max_abs = float(np.abs(o_gpu - o_ref).max()) if o_ref.size else 0.0
    rl2 = rel_l2(o_gpu, o_ref) if np.any(o_ref) else float(np.abs(o_gpu).max(initial=0.0))
    lse_abs = float(np.abs(lse_gpu[fin] - lse_ref[fin]).max()) if fin.any() else 0.0
    assert max_abs <= ATTN_MAX_ABS, f"{what}: max abs {max_abs:.3e}"
    assert rl2 <= ATTN_REL_L2, f"{what}: rel L2 {rl2:.3e}"
    assert lse_abs <= LSE_MAX_ABS, f"{what}: LSE abs {lse_abs:.3e}"
    return max_abs, rl2, lse_abs


def check_selection(sel_gpu, sel_ref, scores_ref, k: int, what=""):
    """Selection parity: equal sets, except blocks whose oracle score is within
    SEL_TIE_REL (relative) of the k-th best oracle score. Also checks the GPU
    list is ascending, duplicate-free and -1 padded to k."""
    sel_gpu = np.asarray(sel_gpu).astype(np.int64)
    sel_ref = np.asarray(sel_ref).astype(np.int64)
    nb = len(scores_ref)
    kb = min(k, nb)
    g = sel_gpu[:kb]
    assert np.all(sel_gpu[kb:] == -1), f"{what}: padding is not -1"
    assert np.all(g >= 0) and np.all(g < nb), f"{what}: index out of range"
    assert np.all(np.diff(g) > 0), f"{what}: not strictly ascending"
    a, b = set(g.tolist()), set(sel_ref[:kb].tolist())
    diff = a ^ b
    if diff:
        s = np.asarray(scores_ref, dtype=np.float64)
        kth = np.sort(s)[::-1][kb - 1]
        band = SEL_TIE_REL * abs(kth)
        bad = [j for j in diff if abs(s[j] - kth) > band]
        assert not bad, f"{what}: selection differs outside the tie band at {bad[:8]}"
    return len(diff)
