"""The benchmark's roofline numerators (algorithmic flops and bytes) against
explicit counts over the oracle's own definitions: the selection of each
(query, group) row and the token set it attends (selected_tokens).  The
formulas in bench.py use closed forms; these loops count the same work
row by row on small problems, so a wrong closed form (an off-by-one in the
causal triangle, the local block miscounted) fails here."""
import math

import numpy as np
import pytest

import bench
import oracle.msa_oracle as O
from block_sparse_long_08_b200 import inputs as I

BLK = 128


def _sel(L, G, top_k, seed, blk=BLK):
    """Selections of an N(0,1) problem, from the oracle (rows of every
    (query, group))."""
    x = I.prefill_inputs_small(1, L, G, G, 8, 8, seed)
    qi, ki = O.as_f64(x["q_idx"]), O.as_f64(x["k_idx"])
    sel = []
    for t in range(L):
        for g in range(G):
            bs = O.block_scores_row(qi[0, t, g], ki[0], t, blk)
            sel.append((t, g, O.select_blocks_row(bs, t, blk, top_k)))
    return sel


@pytest.mark.parametrize("L,G,H,top_k,blk", [(1024, 2, 8, 4, 128), (2048, 1, 4, 16, 128),
                                             (1280, 2, 2, 3, 128), (1024, 2, 8, 8, 64),
                                             (1000, 1, 4, 5, 64), (1100, 2, 4, 3, 128)])
def test_prefill_formulas_match_row_counts(L, G, H, top_k, blk):
    d, d_idx = 128, 64
    r = H // G
    sel = _sel(L, G, top_k, seed=L + top_k, blk=blk)
    n_tok = {(t, g): len(O.selected_tokens(b, t, blk)) for (t, g, b) in sel}
    entries = sum(len(b) for (_, _, b) in sel)
    # main branch: 2 products of 2d flops per (query, head, attended token)
    main = sum(H // G * 4.0 * d * n for n in n_tok.values())
    assert bench.prefill_main_flops(1, L, H, d, top_k, blk) == pytest.approx(main, rel=1e-12)
    # forward attention bytes: per (query, group, block) entry, R q rows
    # gathered and R bf16 partial rows written and read back (+ fp32 lse
    # written and read); the merged output written once
    att = entries * r * (3 * d * 2 + 2 * 4) + L * H * d * 2
    assert bench.prefill_attn_bytes(1, L, H, G, d, top_k, blk) == pytest.approx(att, rel=1e-12)
    # index: every (query, group) row that chooses among its earlier blocks
    # (b_t >= top_k) scores every token of those blocks, one d_idx dot
    # product each (counted from the oracle's token scores of the row)
    x = I.prefill_inputs_small(1, L, G, G, 8, 8, L + top_k)
    scored = 0
    for t in range(L):
        bt = t // blk
        if bt >= top_k:
            scored += len(O.token_index_scores(O.as_f64(x["q_idx"][0, t, 0]),
                                               O.as_f64(x["k_idx"][0, :bt * blk])))
    assert bench.prefill_index_flops(1, L, G, d_idx, top_k, blk) == \
        pytest.approx(G * 2.0 * d_idx * scored, rel=1e-12)
    if blk == 128:
        # the same count as 128 x 128 tiles: every 128-query tile whose rows
        # need scores times every earlier key tile
        nb = L // BLK
        tiles = sum(1 for i in range(nb) for j in range(i) if i >= top_k)
        full = (L % BLK == 0)
        if full:
            idx = G * tiles * 2.0 * d_idx * BLK * BLK
            assert bench.prefill_index_flops(1, L, G, d_idx, top_k) == pytest.approx(idx, rel=1e-12)
        # backward: 5 products per (query, head, attended token)
        assert bench.prefill_bwd_flops(1, L, H, d, top_k) == pytest.approx(main * 2.5, rel=1e-12)
        # backward bytes: q and do gathered, bf16 dq partial written and
        # read back, lse and D read, per entry row; o, do read and dq written
        # per token; k, v read and dk, dv written once
        bwd = entries * r * (2 * d * 2 + 2 * d * 2 + 8) + 3 * L * H * d * 2 + 4 * L * G * d * 2
        assert bench.prefill_bwd_bytes(1, L, H, G, d, top_k) == pytest.approx(bwd, rel=1e-12)


def test_decode_bytes_match_token_counts():
    """Decode bytes: the whole index-key scan plus the K/V of each
    sequence's attended tokens (one row per token per group), in bf16 or
    E4M3 (+ fp32 scales), plus the per-step q, q_idx and out."""
    lens = np.array([1, 127, 128, 129, 700, 2048])
    G, H, d, d_idx, top_k = 2, 8, 128, 64, 4
    n_att = np.array([len(O.selected_tokens(list(range(max(0, (n - 1) // BLK - top_k + 1),
                                                            (n - 1) // BLK + 1)), n - 1, BLK))
                      for n in lens])
    small = len(lens) * (H * d * 2 * 2 + G * d_idx * 2)
    bf16 = float((lens * d_idx * 2 + G * 2 * d * 2 * n_att).sum() + small)
    assert bench.decode_bytes(lens, H, G, d, d_idx, top_k) == pytest.approx(bf16, rel=1e-12)
    f8i = float((lens * (d_idx + 4) + G * 2 * d * 2 * n_att).sum() + small)
    assert bench.decode_bytes(lens, H, G, d, d_idx, top_k, fp8_index=True) == pytest.approx(f8i, rel=1e-12)
    f8 = float((lens * (d_idx + 4) + G * 2 * (d + 4) * n_att).sum() + small)
    assert bench.decode_bytes(lens, H, G, d, d_idx, top_k, fp8_index=True, fp8_kv=True) == \
        pytest.approx(f8, rel=1e-12)
    assert math.isfinite(bf16)
