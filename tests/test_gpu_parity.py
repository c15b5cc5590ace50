"""GPU parity: the CUDA path, called through the C ABI, against the fp64
oracle on the same seeded inputs.

Tolerances:
  * block scores: |S_gpu - S_oracle| <= 4 * d_idx * 2^-24 * sum_i |q_i k_i|
    + 1e-6 (fp32 accumulation of d_idx bf16 products; the max over a block
    moves by no more than the largest element error);
  * selections: bit-equal except boundary swaps within 1e-4*|S| + 1e-4;
  * outputs: max-abs <= 2e-2, mean-abs <= 2e-3 against the oracle run on
    the GPU's validated selection (bf16 in/out, fp32 accumulation).
"""
import math

import numpy as np
import pytest
import torch

import oracle.msa_oracle as O
from block_sparse_long_08_b200 import inputs as I
from block_sparse_long_08_b200 import msa as M
from tests import _parity as P

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _prefill(shape: I.PrefillShape, seed: int, device=DEV, **kw):
    x = I.prefill_inputs(shape, seed, device="cpu", **kw)
    return {n: (t.to(device) if isinstance(t, torch.Tensor) and t.dtype == torch.bfloat16 else t)
            for n, t in x.items()}


def _score_tol(q_idx_row: np.ndarray, k_idx: np.ndarray, t: int, block: int) -> np.ndarray:
    """Per-block bound on the fp32 error of a block score."""
    absdot = np.abs(k_idx[: t + 1]) @ np.abs(q_idx_row)
    nblk = t // block + 1
    bound = np.array([absdot[j * block:min((j + 1) * block, t + 1)].max() for j in range(nblk)])
    return 4 * q_idx_row.shape[0] * 2.0 ** -24 * bound + 1e-6


def _rows_sample(L, n, seed, block=128):
    rng = np.random.default_rng(seed)
    nb = L // block
    base = {0, 1, block - 1, block, L - 1, L - 2, L // 2}
    for j in (nb // 3, nb // 2, nb - 2):   # every boundary class
        base |= {j * block, j * block + 1, (j + 1) * block - 1}
    extra = set(rng.integers(0, L, size=max(0, n - len(base))).tolist())
    return sorted(t for t in base | extra if 0 <= t < L)


# ------------------------------------------------------------------ index
@pytest.mark.parametrize("L,G,di,top_k,seed", [(2048, 2, 64, 4, 0), (1024, 8, 128, 3, 5),
                                               (640, 1, 128, 2, 6), (1152, 4, 64, 17, 7),
                                               (2048, 2, 128, 9, 8), (2560, 2, 64, 5, 9),
                                               (3200, 1, 64, 17, 10), (2048, 4, 128, 12, 11),
                                               (1000, 2, 64, 4, 12), (2049, 4, 128, 5, 13)])
def test_block_scores_and_selection(L, G, di, top_k, seed):
    shape = I.PrefillShape(B=2, L=L, H=G * 4, G=G, d=128, d_idx=di, top_k=top_k)
    x = _prefill(shape, seed)
    sel_f = M.msa_index_select(x["q_idx"], x["k_idx"], top_k)
    sel_u, scores = M.msa_index_select(x["q_idx"], x["k_idx"], top_k, block_scores=True)
    torch.cuda.synchronize()
    # the fused and stored-score routes give bit-identical selections
    assert torch.equal(sel_f, sel_u)
    sc = scores.cpu().numpy()
    sel = sel_f.cpu().numpy()
    qi, ki = P.f64(x["q_idx"]), P.f64(x["k_idx"])
    nb = (L + 127) // 128       # the last block may be partial
    n_swaps = 0
    for b in range(2):
        for t in range(0, L, 3 if L > 1024 else 1):
            bt = t // 128
            for g in range(G):
                ref = O.block_scores_row(qi[b, t, g], ki[b], t, 128)
                tol = _score_tol(qi[b, t, g], ki[b], t, 128)
                got = sc[b, g, t]
                assert np.all(np.abs(got[:bt] - ref[:bt]) <= tol[:bt]), (b, t, g)
                assert np.all(np.isneginf(got[bt:nb]))
                ref_sel = O.select_blocks_row(ref, t, 128, top_k)
                ref_row = ref_sel + [-1] * (top_k - len(ref_sel))
                if not P.check_selection_row(sel[b, g, t], ref_row, ref, t, top_k):
                    n_swaps += 1
    assert n_swaps <= 0.02 * 2 * G * L


def test_integer_inputs_select_bit_exact():
    """Small-integer bf16 inputs make every score exact in fp32, so ties are
    real ties and the lower-id rule must match bit for bit."""
    shape = I.PrefillShape(B=1, L=2048, H=8, G=2, d=128, d_idx=64, top_k=4)
    x = I.prefill_inputs(shape, 3)
    q_idx = I.small_integer_like(x["q_idx"], 11, -1, 1)
    k_idx = I.small_integer_like(x["k_idx"], 12, -1, 1)
    sel = M.msa_index_select(q_idx.to(DEV), k_idx.to(DEV), 4).cpu().numpy()
    qi, ki = O.as_f64(q_idx), O.as_f64(k_idx)
    ties = 0
    for t in range(2048):
        for g in range(2):
            bs = O.block_scores_row(qi[0, t, g], ki[0], t, 128)
            want = O.select_blocks_row(bs, t, 128, 4)
            want = want + [-1] * (4 - len(want))
            assert list(sel[0, g, t]) == want, (t, g, sel[0, g, t], want)
            ties += len(bs) != len(set(bs.tolist()))
    assert ties > 100   # the case really exercises ties


@pytest.mark.parametrize("blk,top_k", [(128, 16), (64, 32)])
def test_many_work_items_keep_ties_bit_exact(blk, top_k):
    """512 index work items over 148 CTAs, so every CTA takes items in
    several rounds.  Small-integer inputs make scores exact and ties common,
    so the fused route must equal the stored-score route, and sampled rows
    of every round the oracle's selection, bit for bit."""
    shape = I.PrefillShape(B=2, L=8192, H=32, G=8, d=128, d_idx=128, top_k=top_k, block=blk)
    x = I.prefill_inputs(shape, 14)
    q_idx = I.small_integer_like(x["q_idx"], 15, -1, 1)
    k_idx = I.small_integer_like(x["k_idx"], 16, -1, 1)
    sel_f = M.msa_index_select(q_idx.to(DEV), k_idx.to(DEV), top_k, block=blk)
    sel_u, _ = M.msa_index_select(q_idx.to(DEV), k_idx.to(DEV), top_k, block_scores=True, block=blk)
    torch.cuda.synchronize()
    assert torch.equal(sel_f, sel_u)
    sel = sel_f.cpu().numpy()
    qi, ki = O.as_f64(q_idx), O.as_f64(k_idx)
    # query tiles 63..0 are items 8*(63-i) .. 8*(63-i)+7: a tile every 3
    # covers rounds 0-3 (148 items each)
    for i in range(2, 64, 3):
        for t in (i * 128, i * 128 + 77, i * 128 + 127):
            for b in range(2):
                for g in (0, 5):
                    bs = O.block_scores_row(qi[b, t, g], ki[b], t, blk)
                    want = O.select_blocks_row(bs, t, blk, top_k)
                    assert list(sel[b, g, t]) == want + [-1] * (top_k - len(want)), (b, g, t)


def test_zero_index_keys_all_ties():
    shape = I.PrefillShape(B=1, L=1024, H=8, G=2, d=128, d_idx=128, top_k=5)
    x = _prefill(shape, 4)
    sel = M.msa_index_select(x["q_idx"], torch.zeros_like(x["k_idx"]), 5).cpu().numpy()
    for t in range(1024):
        bt = t // 128
        want = list(range(bt + 1)) + [-1] * (4 - bt) if bt + 1 <= 5 else [0, 1, 2, 3, bt]
        assert list(sel[0, 0, t]) == want and list(sel[0, 1, t]) == want


# ------------------------------------------------------------------ prefill attention
@pytest.mark.parametrize("L,H,G,top_k,seed", [(2048, 8, 2, 4, 0), (1024, 32, 8, 3, 21),
                                              (768, 16, 16, 2, 22), (512, 16, 1, 3, 23),
                                              (512, 16, 8, 8, 24), (1024, 16, 2, 5, 25),
                                              (1000, 8, 2, 4, 26), (2049, 16, 4, 5, 27)])
def test_prefill_attention_on_oracle_selection(L, H, G, top_k, seed):
    di = 64 if L == 2048 else 128
    shape = I.PrefillShape(B=2, L=L, H=H, G=G, d=128, d_idx=di, top_k=top_k)
    x = _prefill(shape, seed)
    ref = O.prefill(x["q"].cpu(), x["k"].cpu(), x["v"].cpu(), x["q_idx"].cpu(), x["k_idx"].cpu(),
                    top_k=top_k, rows=[(b, t) for b in range(2) for t in range(L)])
    sel = torch.from_numpy(ref["sel"]).to(DEV)
    out, lse = M.msa_sparse_attn_prefill(x["q"], x["k"], x["v"], sel, want_lse=True)
    torch.cuda.synchronize()
    o = out.float().cpu().numpy()
    mx, mean = P.out_errors(o, ref["out"])
    assert mx <= P.OUT_MAX_ABS and mean <= P.OUT_MEAN_ABS, (mx, mean)
    lse_err = np.abs(lse.cpu().numpy() - ref["lse"]).max()
    assert lse_err < 1e-2, lse_err


def test_prefill_dense_limit_and_permuted_selection():
    """top_k >= nb: every block selected, the result is dense causal attention;
    the selection's order inside a row must not matter."""
    shape = I.PrefillShape(B=1, L=1024, H=8, G=2, d=128, d_idx=64, top_k=8)
    x = _prefill(shape, 31)
    out_sel = M.msa_forward(x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"], 8, want_sel=True)
    out, sel = out_sel
    import torch.nn.functional as F
    qt = x["q"].float().permute(0, 2, 1, 3)
    kt = x["k"].float().permute(0, 2, 1, 3).repeat_interleave(4, dim=1)
    vt = x["v"].float().permute(0, 2, 1, 3).repeat_interleave(4, dim=1)
    dense = F.scaled_dot_product_attention(qt, kt, vt, is_causal=True).permute(0, 2, 1, 3)
    err = (out.float() - dense).abs()
    assert err.max().item() <= P.OUT_MAX_ABS and err.mean().item() <= P.OUT_MEAN_ABS
    perm = sel.clone()
    perm[..., :4] = sel[..., :4].flip(-1)
    out2 = M.msa_sparse_attn_prefill(x["q"], x["k"], x["v"], perm)
    assert (out2.float() - out.float()).abs().max().item() <= 1e-2


# ------------------------------------------------------------------ forward end to end
@pytest.mark.parametrize("shape,seed,nrows", [
    (I.PREFILL_TINY, I.SEEDS["tiny"], None),
    (I.PrefillShape(B=1, L=8192, H=32, G=8, d=128, d_idx=128, top_k=16), 8, 40),
    # lengths that are not a multiple of the block: a partial last block
    (I.PrefillShape(B=1, L=1000, H=8, G=2, d=128, d_idx=64, top_k=4), 14, None),
    (I.PrefillShape(B=1, L=2049, H=16, G=4, d=128, d_idx=128, top_k=5), 15, None),
])
def test_forward_matches_oracle(shape, seed, nrows):
    x = _prefill(shape, seed)
    out, sel, lse = M.msa_forward(x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"], shape.top_k,
                                  want_sel=True, want_lse=True)
    torch.cuda.synchronize()
    L = shape.L
    rows = [(0, t) for t in (range(L) if nrows is None else _rows_sample(L, nrows, seed))]
    cpu = {n: x[n].cpu() for n in ("q", "k", "v", "q_idx", "k_idx")}
    ref = P.oracle_rows(cpu["q"], cpu["k"], cpu["v"], cpu["q_idx"], cpu["k_idx"], rows,
                        shape.top_k)
    sel_c = sel.cpu().numpy()
    out_c = out.float().cpu().numpy()
    r = shape.H // shape.G
    errs = []
    for (b, t) in rows:
        for g in range(shape.G):
            bs, blocks, o_ref, lse_ref = ref[(b, t, g)]
            ref_row = blocks + [-1] * (shape.top_k - len(blocks))
            exact = P.check_selection_row(sel_c[b, g, t], ref_row, bs, t, shape.top_k)
            if not exact:   # score the output against the GPU's (validated) selection
                o_ref = P.oracle_rows(cpu["q"], cpu["k"], cpu["v"], cpu["q_idx"], cpu["k_idx"],
                                      [(b, t)], shape.top_k, sel_override=sel_c)[(b, t, g)][2]
            errs.append(np.abs(out_c[b, t, g * r:(g + 1) * r] - o_ref))
    e = np.concatenate([x.ravel() for x in errs])
    assert e.max() <= P.OUT_MAX_ABS and e.mean() <= P.OUT_MEAN_ABS, (e.max(), e.mean())


def test_single_block_and_topk_one():
    shape = I.PrefillShape(B=3, L=128, H=8, G=2, d=128, d_idx=128, top_k=1)
    x = _prefill(shape, 41)
    out = M.msa_forward(x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"], 1)
    ref = O.prefill(x["q"].cpu(), x["k"].cpu(), x["v"].cpu(), x["q_idx"].cpu(), x["k_idx"].cpu(),
                    top_k=1)
    mx, mean = P.out_errors(out.float().cpu().numpy(), ref["out"])
    assert mx <= P.OUT_MAX_ABS and mean <= P.OUT_MEAN_ABS
    shape = I.PrefillShape(B=1, L=640, H=8, G=2, d=128, d_idx=128, top_k=1)
    x = _prefill(shape, 42)
    out = M.msa_forward(x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"], 1)
    ref = O.prefill(x["q"].cpu(), x["k"].cpu(), x["v"].cpu(), x["q_idx"].cpu(), x["k_idx"].cpu(),
                    top_k=1)
    mx, mean = P.out_errors(out.float().cpu().numpy(), ref["out"])
    assert mx <= P.OUT_MAX_ABS and mean <= P.OUT_MEAN_ABS


# ------------------------------------------------------------------ decode
@pytest.mark.parametrize("B,Lmax,G,H,di,top_k,lens", [
    (4, 4096, 8, 32, 128, 16, [4096, 1, 129, 3000]),
    (5, 2048, 2, 8, 64, 4, [2048, 128, 127, 777, 1500]),
    (3, 8192, 8, 32, 128, 16, [8192, 8191, 5000]),
])
def test_decode_matches_oracle(B, Lmax, G, H, di, top_k, lens):
    shape = I.DecodeShape(B=B, Lmax=Lmax, H=H, G=G, d=128, d_idx=di, top_k=top_k)
    x = I.decode_inputs(shape, 9)
    seq = torch.tensor(lens, dtype=torch.int32)
    dev = {n: x[n].to(DEV) for n in ("q", "q_idx", "k_cache", "v_cache", "k_idx_cache")}
    out, sel = M.msa_sparse_attn_decode(dev["q"], dev["q_idx"], dev["k_cache"], dev["v_cache"],
                                        dev["k_idx_cache"], seq.to(DEV), top_k, want_sel=True)
    torch.cuda.synchronize()
    ref = O.decode(x["q"], x["q_idx"], x["k_cache"], x["v_cache"], x["k_idx_cache"], lens, top_k)
    sel_c = sel.cpu().numpy()
    qi, ki = P.f64(x["q_idx"]), P.f64(x["k_idx_cache"])
    any_swap = False
    for b in range(B):
        t = lens[b] - 1
        for g in range(G):
            bs = O.block_scores_row(qi[b, g], ki[b], t, 128)
            if not P.check_selection_row(sel_c[b, g], ref["sel"][b, g], bs, t, top_k):
                any_swap = True
    if any_swap:
        ref = O.decode(x["q"], x["q_idx"], x["k_cache"], x["v_cache"], x["k_idx_cache"], lens,
                       top_k, sel_override=sel_c)
    mx, mean = P.out_errors(out.float().cpu().numpy(), ref["out"])
    assert mx <= P.OUT_MAX_ABS and mean <= P.OUT_MEAN_ABS, (mx, mean)


@pytest.mark.parametrize("zero_keys", [False, True])
def test_decode_integer_inputs_select_bit_exact(zero_keys):
    """Exact scores (small integers) make ties real: the multi-warp top-k
    merge must keep the lower block id exactly as the oracle does."""
    shape = I.DecodeShape(B=3, Lmax=8192, H=8, G=2, d=128, d_idx=64, top_k=6)
    x = I.decode_inputs(shape, 12)
    qi = I.small_integer_like(x["q_idx"], 13, -1, 1)
    ki = torch.zeros_like(x["k_idx_cache"]) if zero_keys else I.small_integer_like(x["k_idx_cache"], 14, -1, 1)
    lens = [8192, 5000, 700]
    d = {n: x[n].to(DEV) for n in ("q", "k_cache", "v_cache")}
    _, sel = M.msa_sparse_attn_decode(d["q"], qi.to(DEV), d["k_cache"], d["v_cache"], ki.to(DEV),
                                      torch.tensor(lens, dtype=torch.int32, device=DEV), 6,
                                      want_sel=True)
    sel = sel.cpu().numpy()
    q64, k64 = O.as_f64(qi), O.as_f64(ki)
    for b in range(3):
        t = lens[b] - 1
        for g in range(2):
            bs = O.block_scores_row(q64[b, g], k64[b], t, 128)
            want = O.select_blocks_row(bs, t, 128, 6)
            assert list(sel[b, g]) == want + [-1] * (6 - len(want)), (b, g, sel[b, g], want)


def test_decode_long_row_integer_ties():
    """One sequence at 1M tokens (8192 blocks): every one of the 16 scanning
    warps holds candidates, and integer scores force exact ties."""
    Lmax = 1048576
    shape = I.DecodeShape(B=1, Lmax=Lmax, H=8, G=2, d=128, d_idx=64, top_k=16)
    gen = torch.Generator().manual_seed(15)
    qi = torch.randint(-1, 2, (1, 2, 64), generator=gen).to(torch.bfloat16)
    ki = torch.randint(-1, 2, (1, Lmax, 64), generator=gen).to(torch.bfloat16)
    q = torch.randn((1, 8, 128), generator=gen).to(torch.bfloat16)
    kc = torch.zeros((1, Lmax, 2, 128), dtype=torch.bfloat16)
    _, sel = M.msa_sparse_attn_decode(q.to(DEV), qi.to(DEV), kc.to(DEV), kc.to(DEV), ki.to(DEV),
                                      torch.tensor([Lmax], dtype=torch.int32, device=DEV), 16,
                                      want_sel=True)
    sel = sel.cpu().numpy()
    q64, k64 = O.as_f64(qi), O.as_f64(ki)
    for g in range(2):
        bs = O.block_scores_row(q64[0, g], k64[0], Lmax - 1, 128)
        want = O.select_blocks_row(bs, Lmax - 1, 128, 16)
        assert list(sel[0, g]) == want, (g, sel[0, g], want)


def test_decode_bad_length_sets_status():
    shape = I.DecodeShape(B=2, Lmax=1024, H=8, G=2, d=128, d_idx=128, top_k=4)
    x = {n: t.to(DEV) for n, t in I.decode_inputs(shape, 10).items() if t.dtype == torch.bfloat16}
    p = M.make_params(2, 1024, 8, 2, 128, 128, 128, 4)
    ws = M.new_workspace(p, M.MSA_OP_DECODE, DEV)
    seq = torch.tensor([1024, 5000], dtype=torch.int32, device=DEV)
    out = M.msa_sparse_attn_decode(x["q"], x["q_idx"], x["k_cache"], x["v_cache"], x["k_idx_cache"],
                                   seq, 4, ws=ws)
    assert M.msa_read_status(ws) == M.MSA_ERR_DEVICE_INPUT
    assert M.msa_read_status(ws) == M.MSA_OK
    assert torch.all(out[1] == 0)


def test_status_clean_after_valid_calls():
    shape = I.PREFILL_TINY
    x = _prefill(shape, 0)
    p = M.make_params(1, shape.L, shape.H, shape.G, 128, shape.d_idx, 128, shape.top_k)
    ws = M.new_workspace(p, M.MSA_OP_FORWARD, DEV)
    M.msa_forward(x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"], shape.top_k, ws=ws)
    assert M.msa_read_status(ws) == M.MSA_OK
