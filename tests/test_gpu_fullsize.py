"""GPU parity at the full workload sizes, in the launch configuration the
benchmark times: msa_index_select (fused top-k) + msa_sparse_attn_prefill +
msa_sparse_attn_decode with their own workspaces, on device-drawn inputs
with the benchmark's seeds.  The oracle evaluates sampled rows one by one
(every group and head of each), covering the first and last rows, rows with
fewer than top_k visible blocks and every block-boundary class; decode is
checked for every sequence.  Tolerances as in test_gpu_parity.py.
"""
import numpy as np
import pytest
import torch

import oracle.msa_oracle as O
from block_sparse_long_08_b200 import inputs as I
from block_sparse_long_08_b200 import msa as M
from tests import _parity as P

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _sample_rows(L, n, seed, top_k, block=128):
    rng = np.random.default_rng(seed)
    nb = L // block
    rows = {0, 1, block - 1, block, top_k * block - 1, top_k * block, L - 1, L - 2}
    for j in (nb // 4, nb // 2, (3 * nb) // 4, nb - 2):
        rows |= {j * block, j * block + 63, (j + 1) * block - 1}
    rows |= set(rng.integers(0, L, size=max(0, n - len(rows))).tolist())
    return sorted(t for t in rows if 0 <= t < L)


def _run_prefill(shape, x):
    B, L, H, G, K, blk = shape.B, shape.L, shape.H, shape.G, shape.top_k, shape.block
    p = M.make_params(B, L, H, G, 128, shape.d_idx, blk, K)
    ws_idx = M.new_workspace(p, M.MSA_OP_INDEX_SELECT, DEV)
    ws_att = M.new_workspace(p, M.MSA_OP_PREFILL_ATTN, DEV)
    sel = torch.empty((B, G, L, K), dtype=torch.int32, device=DEV)
    out = torch.empty_like(x["q"])
    M.msa_index_select(x["q_idx"], x["k_idx"], K, sel=sel, ws=ws_idx, block=blk)
    M.msa_sparse_attn_prefill(x["q"], x["k"], x["v"], sel, out=out, ws=ws_att, block=blk)
    torch.cuda.synchronize()
    assert M.msa_read_status(ws_idx) == M.MSA_OK
    assert M.msa_read_status(ws_att) == M.MSA_OK
    return sel, out


def _check_prefill_rows(shape, x, sel, out, rows):
    cpu = {n: x[n][0].to("cpu") for n in ("k", "v", "k_idx")}
    k_idx64 = cpu["k_idx"].double().numpy()
    G, r, K, blk = shape.G, shape.H // shape.G, shape.top_k, shape.block
    sc = 1.0 / np.sqrt(shape.d)
    q_rows = x["q"][0, rows].to("cpu")
    qi_rows = x["q_idx"][0, rows].to("cpu")
    sel_c = sel[0, :, rows].to("cpu").numpy()          # [G, n, K]
    out_c = out[0, rows].float().to("cpu").numpy()    # [n, H, d]
    errs, swaps = [], 0
    for n, t in enumerate(rows):
        for g in range(G):
            bs = O.block_scores_row(O.as_f64(qi_rows[n, g]), k_idx64, t, blk)
            want = O.select_blocks_row(bs, t, blk, K)
            exact = P.check_selection_row(sel_c[g, n], want + [-1] * (K - len(want)), bs, t, K,
                                          block=blk)
            swaps += 0 if exact else 1
            blocks = P.sel_set(sel_c[g, n])      # validated GPU selection
            tok = torch.from_numpy(O.selected_tokens(blocks, t, blk))
            o, _, _ = O.attend_rows(O.as_f64(q_rows[n, g * r:(g + 1) * r]), O.as_f64(cpu["k"][tok, g]),
                                    O.as_f64(cpu["v"][tok, g]), sc)
            errs.append(np.abs(out_c[n, g * r:(g + 1) * r] - o).ravel())
    e = np.concatenate(errs)
    assert e.max() <= P.OUT_MAX_ABS and e.mean() <= P.OUT_MEAN_ABS, (e.max(), e.mean())
    return swaps


def _check_decode(dshape, y, out, sel):
    lens = y["seq_lens"].to("cpu").numpy()
    r = dshape.H // dshape.G
    sc = 1.0 / np.sqrt(dshape.d)
    sel_c = sel.to("cpu").numpy()
    out_c = out.float().to("cpu").numpy()
    errs = []
    for b in range(dshape.B):
        t = int(lens[b]) - 1
        ki64 = y["k_idx_cache"][b, : t + 1].to("cpu").double().numpy()
        kc, vc = y["k_cache"][b].to("cpu"), y["v_cache"][b].to("cpu")
        for g in range(dshape.G):
            bs = O.block_scores_row(O.as_f64(y["q_idx"][b, g].cpu()), ki64, t, 128)
            want = O.select_blocks_row(bs, t, 128, dshape.top_k)
            P.check_selection_row(sel_c[b, g], want + [-1] * (dshape.top_k - len(want)), bs, t,
                                  dshape.top_k)
            tok = torch.from_numpy(O.selected_tokens(P.sel_set(sel_c[b, g]), t, 128))
            o, _, _ = O.attend_rows(O.as_f64(y["q"][b, g * r:(g + 1) * r].cpu()), O.as_f64(kc[tok, g]),
                                    O.as_f64(vc[tok, g]), sc)
            errs.append(np.abs(out_c[b, g * r:(g + 1) * r] - o).ravel())
    e = np.concatenate(errs)
    assert e.max() <= P.OUT_MAX_ABS and e.mean() <= P.OUT_MEAN_ABS, (e.max(), e.mean())


def _run_decode(dshape, y):
    pd = M.make_params(dshape.B, dshape.Lmax, dshape.H, dshape.G, dshape.d, dshape.d_idx, 128,
                       dshape.top_k)
    ws = M.new_workspace(pd, M.MSA_OP_DECODE, DEV)
    out, sel = M.msa_sparse_attn_decode(y["q"], y["q_idx"], y["k_cache"], y["v_cache"],
                                        y["k_idx_cache"], y["seq_lens"].to(DEV), dshape.top_k,
                                        want_sel=True, ws=ws)
    torch.cuda.synchronize()
    assert M.msa_read_status(ws) == M.MSA_OK
    return out, sel


def test_prefill_32k():
    shape = I.PREFILL_32K
    x = I.prefill_inputs(shape, I.SEEDS["32k"], device=DEV)
    sel, out = _run_prefill(shape, x)
    rows = _sample_rows(shape.L, 48, 1, shape.top_k)
    swaps = _check_prefill_rows(shape, x, sel, out, rows)
    assert swaps <= 0.05 * len(rows) * shape.G


def test_prefill_32k_block64():
    """The 64-token block variant at the 2048-token budget (top_k = 32)."""
    shape = I.PREFILL_32K_BLOCK64
    x = I.prefill_inputs(shape, I.SEEDS["32k"], device=DEV)
    sel, out = _run_prefill(shape, x)
    rows = _sample_rows(shape.L, 48, 1, shape.top_k, block=64)
    swaps = _check_prefill_rows(shape, x, sel, out, rows)
    assert swaps <= 0.05 * len(rows) * shape.G


def test_prefill_128k_planted():
    shape = I.PREFILL_128K_PLANTED
    x = I.prefill_inputs(shape, I.SEEDS["128k_planted"], device=DEV, needles=12, needle_alpha=3.0)
    sel, out = _run_prefill(shape, x)
    rows = _sample_rows(shape.L, 32, 2, shape.top_k)
    _check_prefill_rows(shape, x, sel, out, rows)
    # needle hit rate (reported; at alpha = 3 the pages' claim does not hold,
    # the oracle's pin uses alpha = 3*sqrt(d_idx))
    nb_ids = x["needle_blocks"].numpy()
    sel_c = sel[0, :, rows].to("cpu").numpy()
    hit = tot = 0
    for n, t in enumerate(rows):
        bt = t // 128
        for g in range(shape.G):
            if t < (nb_ids[g].min() + 1) * 128:
                continue
            s = set(int(j) for j in sel_c[g, n] if j >= 0)
            for j in nb_ids[g]:
                if j < bt:
                    tot += 1
                    hit += int(j) in s
    print(f"needle hit rate at alpha=3: {hit}/{tot}")


def test_decode_128k():
    dshape = I.DECODE_128K
    y = I.decode_inputs(dshape, I.SEEDS["decode_128k"], device=DEV)
    out, sel = _run_decode(dshape, y)
    _check_decode(dshape, y, out, sel)


def _rows_per_chunk(shape, per_chunk, seed):
    """Boundary rows plus per_chunk uniform rows inside every query chunk of
    the prefill attention (msa_prefill_chunk_len), so that a fault confined
    to one chunk of the 1M path shows."""
    p = M.make_params(shape.B, shape.L, shape.H, shape.G, 128, shape.d_idx, 128, shape.top_k)
    lc = M.msa_prefill_chunk_len(p)
    rng = np.random.default_rng(seed)
    rows = set(_sample_rows(shape.L, 0, seed, shape.top_k))
    for c0 in range(0, shape.L, lc):
        c1 = min(shape.L, c0 + lc)
        rows |= {c0, c1 - 1}
        rows |= set(rng.integers(c0, c1, size=per_chunk).tolist())
    return sorted(rows), (shape.L + lc - 1) // lc


def test_1m_prefill_and_decode():
    shape, dshape = I.PREFILL_1M, I.DECODE_1M
    x = I.prefill_inputs(shape, I.SEEDS["1m"], device=DEV)
    sel, out = _run_prefill(shape, x)
    rows, n_chunks = _rows_per_chunk(shape, 14, 4)
    assert n_chunks >= 9 and len(rows) >= 128
    _check_prefill_rows(shape, x, sel, out, rows)
    del x, sel, out
    torch.cuda.empty_cache()
    y = I.decode_inputs(dshape, I.SEEDS["1m"], device=DEV)
    dout, dsel = _run_decode(dshape, y)
    _check_decode(dshape, y, dout, dsel)
