"""Pins for the fp64 oracle: each check ties it to something other than
itself -- a hand-worked example, a library routine (torch's
scaled_dot_product_attention in fp64), brute-force enumeration, closed forms
and invariants.  The mutation tests at the end plant plausible mistakes in
the oracle and confirm that some pin catches each one.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle.msa_oracle as O
from block_sparse_long_08_b200 import inputs as I

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_worked_msa.json")


def _lnval(x):
    if isinstance(x, str) and x.startswith("ln"):
        return math.log(float(x[2:]))
    return float(x)


# ---------------------------------------------------------------------------
# checks (plain functions so the mutation tests can re-run them)
# ---------------------------------------------------------------------------

def check_golden():
    g = json.load(open(GOLDEN))
    s = g["shape"]
    B, L, H, G, d, di, blk, k = (s[x] for x in ("B", "L", "H", "G", "d", "d_idx", "block", "top_k"))
    k_idx = np.array(g["k_idx"], float)[None]
    q_idx = np.array(g["q_idx"], float)[None, :, None, :]
    kk = np.array(g["k"], float)[None, :, None, :]
    vv = np.array(g["v"], float)[None, :, None, :]
    q = np.zeros((B, L, H, d))
    q[0, :, 0] = g["q_head0"]
    q[0, :, 1] = g["q_head1"]
    sc = math.log(2.0)
    ex = g["expected"]
    np.testing.assert_array_equal(O.block_scores_row(q_idx[0, 4, 0], k_idx[0], 4, blk), ex["block_scores_t4"])
    np.testing.assert_array_equal(O.block_scores_row(q_idx[0, 5, 0], k_idx[0], 5, blk), ex["block_scores_t5"])
    res = O.prefill(q, kk, vv, q_idx, k_idx, top_k=k, block=blk, scale=sc)
    np.testing.assert_array_equal(res["sel"][0, 0], np.array(ex["sel"]))
    for t, rows in ex["out"].items():
        np.testing.assert_allclose(res["out"][0, int(t)], np.array(rows), rtol=0, atol=1e-14)
    for t, vals in ex["lse"].items():
        np.testing.assert_allclose(res["lse"][0, int(t)], [_lnval(x) for x in vals], rtol=0, atol=1e-14)
    q_idx_tie = q_idx.copy()
    q_idx_tie[0, 4, 0] = 0.0
    res_t = O.prefill(q, kk, vv, q_idx_tie, k_idx, top_k=k, block=blk, scale=sc, rows=[(0, 4)])
    np.testing.assert_array_equal(res_t["sel"][0, 0, 4], ex["tie_sel_t4"])
    dec = O.decode(q[:, 4], q_idx[:, 4], kk, vv, k_idx, [5], top_k=k, block=blk, scale=sc)
    np.testing.assert_array_equal(dec["sel"][0, 0], ex["decode_seq_len_5"]["sel"])
    np.testing.assert_allclose(dec["out"][0], np.array(ex["decode_seq_len_5"]["out"]), rtol=0, atol=1e-14)


def _gqa_sdpa(q, k, v, mask=None, is_causal=False):
    """torch SDPA (fp64, CPU) with k/v repeated over the heads of each group."""
    qt = torch.from_numpy(q).permute(0, 2, 1, 3)          # [B,H,L,d]
    r = q.shape[2] // k.shape[2]
    kt = torch.from_numpy(k).permute(0, 2, 1, 3).repeat_interleave(r, dim=1)
    vt = torch.from_numpy(v).permute(0, 2, 1, 3).repeat_interleave(r, dim=1)
    o = F.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, is_causal=is_causal)
    return o.permute(0, 2, 1, 3).numpy()


def _small_problem(seed, B=2, L=96, H=4, G=2, d=16, di=8):
    x = I.prefill_inputs_small(B, L, H, G, d, di, seed)
    return {n: O.as_f64(x[n]) for n in ("q", "k", "v", "q_idx", "k_idx")}


def check_dense_limit():
    blk = 16
    p = _small_problem(11)
    nb = p["q"].shape[1] // blk
    for k in (nb, nb + 3):
        res = O.prefill(p["q"], p["k"], p["v"], p["q_idx"], p["k_idx"], top_k=k, block=blk)
        ref = _gqa_sdpa(p["q"], p["k"], p["v"], is_causal=True)
        np.testing.assert_allclose(res["out"], ref, rtol=1e-11, atol=1e-12)


def check_block_local_limit():
    blk = 16
    p = _small_problem(12, L=80)  # 5 blocks
    L = p["q"].shape[1]
    res = O.prefill(p["q"], p["k"], p["v"], p["q_idx"], p["k_idx"], top_k=1, block=blk)
    t = np.arange(L)[:, None]
    s = np.arange(L)[None, :]
    mask = torch.from_numpy((s <= t) & (s // blk == t // blk))
    ref = _gqa_sdpa(p["q"], p["k"], p["v"], mask=mask)
    np.testing.assert_allclose(res["out"], ref, rtol=1e-11, atol=1e-12)


def _brute_sel(q_idx_row, k_idx, t, blk, k):
    """Pure-Python: token scores by explicit loops, block max by loops over
    visible tokens, then the best (k-1)-subset of earlier blocks by total
    score, ties to the lexicographically smallest id tuple."""
    n_vis = t + 1
    tok = []
    for s in range(n_vis):
        acc = 0.0
        for i in range(len(q_idx_row)):
            acc += float(q_idx_row[i]) * float(k_idx[s][i])
        tok.append(acc)
    bt = t // blk
    bscore = []
    for j in range(bt + 1):
        m = -math.inf
        for s in range(j * blk, min((j + 1) * blk, n_vis)):
            m = max(m, tok[s])
        bscore.append(m)
    if bt + 1 <= k:
        return list(range(bt + 1)), bscore
    best, best_sum = None, -math.inf
    for comb in itertools.combinations(range(bt), k - 1):
        ssum = sum(bscore[j] for j in comb)
        if ssum > best_sum or (ssum == best_sum and comb < best):
            best, best_sum = comb, ssum
    return sorted(list(best) + [bt]), bscore


def check_selection_brute_force(integer_inputs):
    blk, k = 8, 3
    x = I.prefill_inputs_small(1, 64, 2, 2, 4, 6, seed=21)
    if integer_inputs:
        x["q_idx"] = I.small_integer_like(x["q_idx"], 5, -2, 2)
        x["k_idx"] = I.small_integer_like(x["k_idx"], 6, -2, 2)
    q_idx, k_idx = O.as_f64(x["q_idx"]), O.as_f64(x["k_idx"])
    res = O.prefill(O.as_f64(x["q"]), O.as_f64(x["k"]), O.as_f64(x["v"]), q_idx, k_idx,
                    top_k=k, block=blk)
    kl = k_idx[0].tolist()
    for t in range(64):
        for g in range(2):
            want, bscore = _brute_sel(q_idx[0, t, g].tolist(), kl, t, blk, k)
            got = [int(j) for j in res["sel"][0, g, t] if j >= 0]
            assert got == want, (t, g, got, want)
            np.testing.assert_array_equal(O.block_scores_row(q_idx[0, t, g], k_idx[0], t, blk), bscore)


def check_selection_structure():
    blk, k = 16, 4
    p = _small_problem(31, B=1, L=160, G=2)
    res = O.prefill(p["q"], p["k"], p["v"], p["q_idx"], p["k_idx"], top_k=k, block=blk)
    sel = res["sel"]
    for g in range(2):
        for t in range(160):
            bt = t // blk
            row = sel[0, g, t]
            valid = [int(j) for j in row if j >= 0]
            assert len(valid) == min(k, bt + 1)
            assert valid == sorted(valid) and len(set(valid)) == len(valid)
            assert valid[-1] == bt                        # local block forced in
            assert all(j < bt for j in valid[:-1])
            assert all(j == -1 for j in row[len(valid):])  # -1 padding at the end


def check_zero_index_key_ties():
    blk, k = 16, 4
    p = _small_problem(41, B=1, L=128, G=2)
    p["k_idx"][:] = 0.0
    res = O.prefill(p["q"], p["k"], p["v"], p["q_idx"], p["k_idx"], top_k=k, block=blk)
    for t in range(128):
        bt = t // blk
        want = list(range(bt + 1)) if bt + 1 <= k else list(range(k - 1)) + [bt]
        for g in range(2):
            assert [int(j) for j in res["sel"][0, g, t] if j >= 0] == want


def check_needles():
    shape = I.PrefillShape(B=1, L=640, H=4, G=2, d=16, d_idx=32, block=16, top_k=8)
    alpha = 3.0 * math.sqrt(shape.d_idx)
    x = I.prefill_inputs(shape, seed=51, needles=6, needle_alpha=alpha)
    nb_ids = x["needle_blocks"].numpy()
    p = {n: O.as_f64(x[n]) for n in ("q", "k", "v", "q_idx", "k_idx")}
    rows = [(0, t) for t in range(0, 640, 7)]
    res = O.prefill(p["q"], p["k"], p["v"], p["q_idx"], p["k_idx"], top_k=shape.top_k,
                    block=shape.block, rows=rows)
    checked = 0
    for (_, t) in rows:
        bt = t // shape.block
        for g in range(shape.G):
            first = nb_ids[g].min()
            if t < (first + 1) * shape.block:
                continue
            sel = set(int(j) for j in res["sel"][0, g, t] if j >= 0)
            for j in nb_ids[g]:
                if j < bt:
                    assert j in sel, (t, g, j, sel)
                    checked += 1
    assert checked > 50


def check_probs_sum_to_one():
    p = _small_problem(61, B=1, L=64, G=2)
    res = O.prefill(p["q"], p["k"], p["v"], p["q_idx"], p["k_idx"], top_k=2, block=16,
                    want_probs=True)
    for pr in res["probs"].values():
        assert np.all(pr >= 0)
        assert abs(pr.sum() - 1.0) < 1e-12


def check_sel_order_invariance():
    p = _small_problem(71, B=1, L=128, G=2)
    res = O.prefill(p["q"], p["k"], p["v"], p["q_idx"], p["k_idx"], top_k=4, block=16)
    perm = res["sel"].copy()
    rng = np.random.default_rng(0)
    for g in range(2):
        for t in range(128):
            n = int((perm[0, g, t] >= 0).sum())
            perm[0, g, t, :n] = perm[0, g, t, :n][rng.permutation(n)]
    res2 = O.prefill(p["q"], p["k"], p["v"], p["q_idx"], p["k_idx"], top_k=4, block=16,
                     sel_override=perm)
    np.testing.assert_allclose(res2["out"], res["out"], rtol=0, atol=1e-13)


def check_zero_query_mean():
    """q = 0: every attended token gets the same weight, so the output is the
    plain mean of v over the attended tokens (tokens of the selected blocks
    with s <= t), built here from a boolean mask."""
    blk, k = 16, 3
    p = _small_problem(81, B=1, L=112, G=2)
    p["q"][:] = 0.0
    res = O.prefill(p["q"], p["k"], p["v"], p["q_idx"], p["k_idx"], top_k=k, block=blk)
    L, H, G = 112, p["q"].shape[2], 2
    r = H // G
    for t in range(L):
        for h in range(H):
            g = h // r
            sel = set(int(j) for j in res["sel"][0, g, t] if j >= 0)
            mask = np.array([(s <= t) and (s // blk in sel) for s in range(L)])
            np.testing.assert_allclose(res["out"][0, t, h], p["v"][0, mask, g].mean(axis=0),
                                       rtol=0, atol=1e-13)
            np.testing.assert_allclose(res["lse"][0, t, h], math.log(mask.sum()), rtol=0, atol=1e-13)


def check_decode_is_last_prefill_row():
    blk, k = 16, 3
    p = _small_problem(91, B=2, L=96, G=2)
    lens = [96, 59]
    pre = O.prefill(p["q"], p["k"], p["v"], p["q_idx"], p["k_idx"], top_k=k, block=blk,
                    rows=[(0, 95), (1, 58)])
    q = np.stack([p["q"][0, 95], p["q"][1, 58]])
    qi = np.stack([p["q_idx"][0, 95], p["q_idx"][1, 58]])
    dec = O.decode(q, qi, p["k"], p["v"], p["k_idx"], lens, top_k=k, block=blk)
    np.testing.assert_allclose(dec["out"][0], pre["out"][0, 95], rtol=0, atol=1e-14)
    np.testing.assert_allclose(dec["out"][1], pre["out"][1, 58], rtol=0, atol=1e-14)
    np.testing.assert_array_equal(dec["sel"][0], pre["sel"][0, :, 95])
    np.testing.assert_array_equal(dec["sel"][1], pre["sel"][1, :, 58])


def check_e4m3_against_library_and_closed_forms():
    # every one of the 256 codes against torch's float8_e4m3fn conversion
    codes = np.arange(256, dtype=np.uint8)
    lib = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = O.e4m3_to_f64(codes)
    assert np.array_equal(np.isnan(got), np.isnan(lib))
    np.testing.assert_array_equal(got[~np.isnan(got)], lib[~np.isnan(lib)])
    # values fixed by the format's definition
    want = {0x00: 0.0, 0x38: 1.0, 0x3C: 1.5, 0xB8: -1.0, 0x7E: 448.0, 0xFE: -448.0,
            0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0x40: 2.0, 0x30: 0.5}
    for c, v in want.items():
        assert O.e4m3_to_f64(np.uint8(c)) == v, hex(c)
    assert math.copysign(1.0, float(O.e4m3_to_f64(np.uint8(0x80)))) == -1.0
    assert np.isnan(O.e4m3_to_f64(np.uint8(0x7F))) and np.isnan(O.e4m3_to_f64(np.uint8(0xFF)))
    # dequantization: one scale per row
    rows = np.array([[0x38, 0x40], [0x3C, 0xB8]], dtype=np.uint8)
    np.testing.assert_array_equal(O.dequant_rows(rows, [0.25, 4.0]), [[0.25, 0.5], [6.0, -4.0]])


def _bwd_problem(seed, top_k=2, L=64):
    """Small fp64 problem with a sparse selection (4 blocks of 16, top_k=2)."""
    blk = 16
    p = _small_problem(seed, B=1, L=L, H=4, G=2, d=8, di=8)
    sel = O.prefill(p["q"], p["k"], p["v"], p["q_idx"], p["k_idx"], top_k=top_k, block=blk)["sel"]
    dout = np.random.default_rng(seed).standard_normal(p["q"].shape)
    return p, sel, dout, blk


def check_backward_finite_differences():
    """Directional derivatives of sum(dout * out) by central differences
    (fp64, h = 1e-5) against the oracle's gradients: random directions over
    whole tensors, and directions confined to the diagonal (local) block and
    to one earlier key block."""
    p, sel, dout, blk = _bwd_problem(101)
    g = O.prefill_backward(p["q"], p["k"], p["v"], sel, dout, block=blk)
    grads = {"q": g["dq"], "k": g["dk"], "v": g["dv"]}

    def loss(**kw):
        x = {n: kw.get(n, p[n]) for n in ("q", "k", "v")}
        out = O.prefill(x["q"], x["k"], x["v"], p["q_idx"], p["k_idx"], top_k=sel.shape[-1],
                        block=blk, sel_override=sel)["out"]
        return float(np.sum(out * dout))

    rng = np.random.default_rng(7)
    h = 1e-5
    L = p["q"].shape[1]
    for name in ("q", "k", "v"):
        dirs = [rng.standard_normal(p[name].shape) for _ in range(3)]
        for lo, hi in ((L - blk, L), (blk, 2 * blk)):
            u = np.zeros(p[name].shape)
            u[:, lo:hi] = rng.standard_normal(u[:, lo:hi].shape)
            dirs.append(u)
        for u in dirs:
            fd = (loss(**{name: p[name] + h * u}) - loss(**{name: p[name] - h * u})) / (2 * h)
            an = float(np.sum(grads[name] * u))
            assert abs(fd - an) <= 1e-6 * (1.0 + abs(an)), (name, fd, an)


def check_backward_dense_limit():
    """top_k >= nb: every earlier block is selected, so the gradients are
    those of dense causal GQA attention -- torch autograd through
    scaled_dot_product_attention in fp64."""
    p, _, dout, blk = _bwd_problem(102)
    nb = p["q"].shape[1] // blk
    sel = O.prefill(p["q"], p["k"], p["v"], p["q_idx"], p["k_idx"], top_k=nb, block=blk)["sel"]
    g = O.prefill_backward(p["q"], p["k"], p["v"], sel, dout, block=blk)
    qt, kt, vt = (torch.from_numpy(p[n].copy()).requires_grad_() for n in ("q", "k", "v"))
    r = qt.shape[2] // kt.shape[2]
    o = F.scaled_dot_product_attention(qt.permute(0, 2, 1, 3),
                                       kt.permute(0, 2, 1, 3).repeat_interleave(r, dim=1),
                                       vt.permute(0, 2, 1, 3).repeat_interleave(r, dim=1),
                                       is_causal=True).permute(0, 2, 1, 3)
    (o * torch.from_numpy(dout)).sum().backward()
    np.testing.assert_allclose(g["dq"], qt.grad.numpy(), rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(g["dk"], kt.grad.numpy(), rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(g["dv"], vt.grad.numpy(), rtol=1e-10, atol=1e-11)


def check_backward_sums():
    """Closed forms that hold for any selection: each softmax row sums to 1,
    so the value gradients of a group sum to the group's summed output
    gradient, and the logit gradients of a row sum to 0, so the key
    gradients of a group sum to 0."""
    p, sel, dout, blk = _bwd_problem(103, top_k=2, L=80)
    g = O.prefill_backward(p["q"], p["k"], p["v"], sel, dout, block=blk)
    G = p["k"].shape[2]
    r = p["q"].shape[2] // G
    for gi in range(G):
        want_v = dout[0, :, gi * r:(gi + 1) * r].sum(axis=(0, 1))
        np.testing.assert_allclose(g["dv"][0, :, gi].sum(axis=0), want_v, rtol=0, atol=1e-11)
        np.testing.assert_allclose(g["dk"][0, :, gi].sum(axis=0), 0.0, rtol=0, atol=1e-11)
    # keys of blocks that no query selects get no gradient
    used = set(int(j) for j in sel.ravel() if j >= 0)
    for j in range(p["k"].shape[1] // blk):
        if j not in used:
            assert not g["dk"][0, j * blk:(j + 1) * blk].any()


def _nsa_problem(seed, L=96, blk=16, top_k=3):
    p = _small_problem(seed, L=L)
    sel = O.prefill(p["q"], p["k"], p["v"], p["q_idx"], p["k_idx"], top_k=top_k, block=blk)["sel"]
    return p, sel, blk


def _band_mask(L, lo_off, device=None):
    """[L, L] boolean: key s visible to query t iff t - lo_off <= s <= t."""
    ones = torch.ones(L, L, dtype=torch.bool)
    return torch.tril(ones) & torch.triu(ones, diagonal=-lo_off)


def check_nsa_window():
    """Sliding-window branch against torch SDPA (fp64) with a band mask built
    from tril/triu; window = 1 gives v[t] exactly; window >= L is dense
    causal attention."""
    p, sel, blk = _nsa_problem(121)
    L = p["q"].shape[1]
    for w in (1, 5, 16, 37):
        br = O.nsa_branches(p["q"], p["k"], p["v"], sel, window=w, block=blk)
        want = _gqa_sdpa(p["q"], p["k"], p["v"], mask=_band_mask(L, w - 1))
        np.testing.assert_allclose(br["out_win"], want, rtol=1e-11, atol=1e-12)
        if w == 1:
            r = p["q"].shape[2] // p["k"].shape[2]
            np.testing.assert_array_equal(br["out_win"], np.repeat(p["v"], r, axis=2))
    br = O.nsa_branches(p["q"], p["k"], p["v"], sel, window=L + 7, block=blk)
    np.testing.assert_allclose(br["out_win"], _gqa_sdpa(p["q"], p["k"], p["v"], is_causal=True),
                               rtol=1e-11, atol=1e-12)


def check_nsa_compression():
    """Compression branch: block means against torch's avg_pool1d (a partial
    last block averaged over its own tokens), the branch output against SDPA
    over those pooled tokens with compressed token c visible to t iff block
    c ends at or before t, zero output where no block is complete; block = 1
    is dense causal attention."""
    for L, blk in ((96, 16), (90, 16), (40, 1)):
        p, sel, _ = _nsa_problem(122, L=L, blk=max(blk, 2))
        B, _, G, d = p["k"].shape
        pool = lambda x: F.avg_pool1d(torch.from_numpy(x).permute(0, 2, 3, 1).reshape(B * G * d, 1, L),
                                      blk, blk, ceil_mode=True).reshape(B, G, d, -1).permute(0, 3, 1, 2)
        kc, vc = O.compress_kv(p["k"], p["v"], blk)
        np.testing.assert_allclose(kc, pool(p["k"]).numpy(), rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(vc, pool(p["v"]).numpy(), rtol=1e-13, atol=1e-14)
        br = O.nsa_branches(p["q"], p["k"], p["v"], sel, window=4, block=blk)
        nb = kc.shape[1]
        t_ = torch.arange(L)[:, None]
        c_ = torch.arange(nb)[None, :]
        mask = (c_ + 1) * blk - 1 <= t_                      # [L, nb]
        has = mask.any(dim=1).numpy()
        want = _gqa_sdpa(p["q"][:, has], kc, vc, mask=mask[torch.from_numpy(has)])
        np.testing.assert_allclose(br["out_cmp"][:, has], want, rtol=1e-11, atol=1e-12)
        assert not br["out_cmp"][:, ~has].any()
        assert np.all(br["lse_cmp"][:, ~has] == -np.inf)
        if blk == 1:
            np.testing.assert_allclose(br["out_cmp"], _gqa_sdpa(p["q"], p["k"], p["v"], is_causal=True),
                                       rtol=1e-11, atol=1e-12)


def check_nsa_gate():
    """One-hot gates give each branch alone (the selection branch is MSA's
    prefill output on the same selection); the output is linear in the
    gates."""
    p, sel, blk = _nsa_problem(123)
    B, L, H, _ = p["q"].shape
    rng = np.random.default_rng(5)
    out_slc = O.prefill(p["q"], p["k"], p["v"], p["q_idx"], p["k_idx"], top_k=3, block=blk,
                        sel_override=sel)["out"]
    outs = []
    for i in range(3):
        gates = np.zeros((B, L, H, 3))
        gates[..., i] = 1.0
        o, br = O.nsa_forward(p["q"], p["k"], p["v"], sel, gates, window=9, block=blk)
        np.testing.assert_array_equal(o, br["out_" + ("cmp", "slc", "win")[i]])
        outs.append(o)
    np.testing.assert_allclose(outs[1], out_slc, rtol=0, atol=1e-13)
    gates = rng.uniform(0, 1, (B, L, H, 3))
    o, _ = O.nsa_forward(p["q"], p["k"], p["v"], sel, gates, window=9, block=blk)
    want = sum(gates[..., i:i + 1] * outs[i] for i in range(3))
    np.testing.assert_allclose(o, want, rtol=1e-13, atol=1e-14)


CHECKS = {
    "golden": check_golden,
    "e4m3": check_e4m3_against_library_and_closed_forms,
    "dense_limit": check_dense_limit,
    "block_local_limit": check_block_local_limit,
    "brute_force_float": lambda: check_selection_brute_force(False),
    "brute_force_int": lambda: check_selection_brute_force(True),
    "structure": check_selection_structure,
    "zero_key_ties": check_zero_index_key_ties,
    "needles": check_needles,
    "probs": check_probs_sum_to_one,
    "order_invariance": check_sel_order_invariance,
    "zero_query_mean": check_zero_query_mean,
    "decode_last_row": check_decode_is_last_prefill_row,
    "backward_finite_differences": check_backward_finite_differences,
    "backward_dense_limit": check_backward_dense_limit,
    "backward_sums": check_backward_sums,
    "nsa_window": check_nsa_window,
    "nsa_compression": check_nsa_compression,
    "nsa_gate": check_nsa_gate,
}


@pytest.mark.parametrize("name", list(CHECKS))
def test_oracle_pin(name):
    CHECKS[name]()


# ---------------------------------------------------------------------------
# mutation tests: a planted mistake in the oracle must trip some pin
# ---------------------------------------------------------------------------

def _select_no_local(bscores, t, block, top_k):
    bt = t // block
    if bt + 1 <= top_k:
        return list(range(bt + 1))
    return sorted(sorted(range(bt + 1), key=lambda j: (-bscores[j], j))[:top_k])


def _select_high_tie(bscores, t, block, top_k):
    bt = t // block
    if bt + 1 <= top_k:
        return list(range(bt + 1))
    return sorted(sorted(range(bt), key=lambda j: (-bscores[j], -j))[: top_k - 1] + [bt])


def _select_local_not_counted(bscores, t, block, top_k):
    bt = t // block
    if bt + 1 <= top_k:
        return list(range(bt + 1))
    return sorted(sorted(range(bt), key=lambda j: (-bscores[j], j))[:top_k] + [bt])


def _block_mean(q_idx_row, k_idx, t, block):
    s = k_idx[: t + 1] @ q_idx_row
    n = t // block + 1
    return np.array([s[j * block: min((j + 1) * block, t + 1)].mean() for j in range(n)])


def _tokens_strict(blocks, t, block):
    ids = [s for j in blocks if j >= 0 for s in range(j * block, min((j + 1) * block, t + 1)) if s < t or t == 0]
    return np.asarray(sorted(ids), dtype=np.int64)


def _attend_no_scale(q_rows, k_tok, v_tok, scale):
    return _orig_attend(q_rows, k_tok, v_tok, 1.0)


def _attend_swapped_kv(q_rows, k_tok, v_tok, scale):
    return _orig_attend(q_rows, v_tok, k_tok, scale)


_orig_attend = O.attend_rows


def _e4m3_bias8(codes):
    return _orig_e4m3(codes) * 0.5      # exponent bias 8 instead of 7


def _e4m3_no_subnormals(codes):
    v = _orig_e4m3(codes)
    c = np.asarray(codes).astype(np.uint8)
    return np.where(((c >> 3) & 0xF) == 0, np.sign(v) * 0.0, v)


_orig_e4m3 = O.e4m3_to_f64


def _grad_no_delta(q_rows, k_tok, v_tok, do_rows, scale):
    _, _, p = _orig_attend(q_rows, k_tok, v_tok, scale)
    dz = p * (do_rows @ v_tok.T)                 # the rowsum(do * o) term dropped
    return scale * (dz @ k_tok), scale * (dz.T @ q_rows), p.T @ do_rows


def _grad_dk_unscaled(q_rows, k_tok, v_tok, do_rows, scale):
    dq, dk, dv = _orig_grad(q_rows, k_tok, v_tok, do_rows, scale)
    return dq, dk / scale, dv


def _grad_dq_through_v(q_rows, k_tok, v_tok, do_rows, scale):
    o, _, p = _orig_attend(q_rows, k_tok, v_tok, scale)
    dz = p * (do_rows @ v_tok.T - np.sum(do_rows * o, axis=1, keepdims=True))
    return scale * (dz @ v_tok), scale * (dz.T @ q_rows), p.T @ do_rows


_orig_grad = O.attend_rows_grad


def _window_one_more(t, window):
    return np.arange(max(0, t - window), t + 1, dtype=np.int64)


def _compressed_partial_visible(t, block):
    return np.arange(t // block + 1, dtype=np.int64)


def _compressed_before_local(t, block):
    return np.arange(t // block, dtype=np.int64)


def _compress_sum(k, v, block):
    kc, vc = _orig_compress(k, v, block)
    return kc * block, vc * block


_orig_compress = O.compress_kv


def _nsa_gates_swapped(q, k, v, sel, gates, window, block=128, scale=None, rows=None):
    return _orig_nsa_forward(q, k, v, sel, np.asarray(gates)[..., ::-1], window, block, scale, rows)


_orig_nsa_forward = O.nsa_forward

MUTANTS = {
    "no_forced_local": ("select_blocks_row", _select_no_local),
    "ties_to_higher_id": ("select_blocks_row", _select_high_tie),
    "local_not_counted_in_top_k": ("select_blocks_row", _select_local_not_counted),
    "mean_pool": ("block_scores_row", _block_mean),
    "strict_causal": ("selected_tokens", _tokens_strict),
    "scale_dropped": ("attend_rows", _attend_no_scale),
    "k_v_swapped": ("attend_rows", _attend_swapped_kv),
    "e4m3_bias_8": ("e4m3_to_f64", _e4m3_bias8),
    "e4m3_no_subnormals": ("e4m3_to_f64", _e4m3_no_subnormals),
    "bwd_delta_dropped": ("attend_rows_grad", _grad_no_delta),
    "bwd_dk_unscaled": ("attend_rows_grad", _grad_dk_unscaled),
    "bwd_dq_through_v": ("attend_rows_grad", _grad_dq_through_v),
    "nsa_window_one_too_many": ("window_tokens", _window_one_more),
    "nsa_partial_block_compressed": ("compressed_tokens", _compressed_partial_visible),
    "nsa_completed_block_left_out": ("compressed_tokens", _compressed_before_local),
    "nsa_compress_sum": ("compress_kv", _compress_sum),
    "nsa_gates_swapped": ("nsa_forward", _nsa_gates_swapped),
}


@pytest.mark.parametrize("mutant", list(MUTANTS))
def test_planted_oracle_mistake_is_caught(mutant, monkeypatch):
    attr, fn = MUTANTS[mutant]
    monkeypatch.setattr(O, attr, fn)
    failed = []
    for name, chk in CHECKS.items():
        try:
            chk()
        except Exception:  # a failed assertion, or the mutant breaking a shape
            failed.append(name)
    assert failed, f"no pin caught the planted mistake {mutant}"
