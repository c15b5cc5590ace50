"""Helpers shared by the GPU parity tests: row-wise oracle evaluation on
slices of the inputs, and the selection / output comparison rules.

Selection rule: selected block sets must be equal, except for swaps at the
k-th boundary where the oracle's two block scores differ by at most
1e-4*|score| + 1e-4.  Output rule: against the oracle attending over the
(validated) GPU selection, max-abs error <= 2e-2 and mean-abs <= 2e-3.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle.msa_oracle as O

SWAP_RTOL = 1e-4
SWAP_ATOL = 1e-4
OUT_MAX_ABS = 2e-2
OUT_MEAN_ABS = 2e-3


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def sel_set(row) -> list[int]:
    return sorted(int(x) for x in np.asarray(row).tolist() if x >= 0)


def check_selection_row(gpu_row, ref_row, bscores: np.ndarray, t: int, top_k: int,
                        block: int = 128) -> bool:
    """True if identical; False if it differs only by allowed boundary swaps;
    raises AssertionError otherwise.  bscores: oracle fp64 block scores of
    this (query, group) row."""
    g = sel_set(gpu_row)
    r = sel_set(ref_row)
    bt = t // block
    assert len(g) == len(r) == min(top_k, bt + 1), (t, g, r)
    assert bt in g, (t, g)
    assert len(set(g)) == len(g), (t, g)
    assert list(np.asarray(gpu_row)[: len(g)]) == g, ("not sorted ascending / padded", gpu_row)
    assert all(int(x) == -1 for x in np.asarray(gpu_row)[len(g):]), gpu_row
    if g == r:
        return True
    only_g = sorted(set(g) - set(r), key=lambda j: (-bscores[j], j))
    only_r = sorted(set(r) - set(g), key=lambda j: (-bscores[j], j))
    assert len(only_g) == len(only_r)
    for a, b in zip(only_g, only_r):
        sa, sb = bscores[a], bscores[b]
        assert abs(sa - sb) <= SWAP_RTOL * abs(sb) + SWAP_ATOL, (
            f"t={t}: gpu picked {a} ({sa}) instead of {b} ({sb})")
    return False


def oracle_rows(q, k, v, q_idx, k_idx, rows, top_k, scale=None, block=128, sel_override=None):
    """Evaluate the oracle on selected (b, t) rows from torch bf16 tensors,
    converting only what each row needs.  Returns dict keyed by (b, t, g):
    (bscores, sel list, out [r,d], lse [r])."""
    B, L, H, d = q.shape
    G = k.shape[2]
    r = H // G
    sc = (1.0 / math.sqrt(d)) if not scale else scale
    k_idx64 = {b: f64(k_idx[b]) for b in {b for b, _ in rows}}
    res = {}
    for (b, t) in rows:
        for g in range(G):
            bs = O.block_scores_row(f64(q_idx[b, t, g]), k_idx64[b], t, block)
            if sel_override is not None:
                blocks = sel_set(sel_override[b, g, t])
            else:
                blocks = O.select_blocks_row(bs, t, block, top_k)
            tok = O.selected_tokens(blocks, t, block)
            tok_t = torch.from_numpy(tok)
            o, lse, _ = O.attend_rows(f64(q[b, t, g * r:(g + 1) * r]), f64(k[b, tok_t, g]),
                                      f64(v[b, tok_t, g]), sc)
            res[(b, t, g)] = (bs, blocks, o, lse)
    return res


def out_errors(gpu: np.ndarray, ref: np.ndarray):
    e = np.abs(gpu.astype(np.float64) - ref)
    return float(e.max()), float(e.mean())
