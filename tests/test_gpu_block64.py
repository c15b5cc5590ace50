"""GPU parity of the 64-token block variant ("MiniMax M3 sparse attention"
explainer, §4.2, reasons with 64-token blocks) against the fp64 oracle, whose
every function takes the block length as a parameter.  The same budget of
2048 KV tokens per (query, group) is top_k = 32 blocks of 64.

Tolerances and the selection rule are those of test_gpu_parity.py: block
scores within the fp32 accumulation bound, selections bit-equal except
allowed boundary swaps, outputs within max-abs 2e-2 / mean-abs 2e-3 of the
oracle on the validated GPU selection.  Cached and ragged calls must equal
the whole-sequence rows bit for bit, as with 128-token blocks.
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
BLK = 64


def _score_tol(q_idx_row, k_idx, t, block):
    absdot = np.abs(k_idx[: t + 1]) @ np.abs(q_idx_row)
    nblk = t // block + 1
    bound = np.array([absdot[j * block:min((j + 1) * block, t + 1)].max() for j in range(nblk)])
    return 4 * q_idx_row.shape[0] * 2.0 ** -24 * bound + 1e-6


@pytest.mark.parametrize("L,G,di,top_k,seed", [(2048, 2, 64, 8, 60), (1000, 4, 128, 5, 61),
                                               (3072, 1, 128, 32, 62), (2048, 8, 128, 17, 63),
                                               (640, 2, 64, 2, 64), (1111, 2, 128, 9, 65)])
def test_block_scores_and_selection(L, G, di, top_k, seed):
    shape = I.PrefillShape(B=2, L=L, H=G * 4, G=G, d=128, d_idx=di, top_k=top_k)
    x = {n: t.to(DEV) for n, t in I.prefill_inputs(shape, seed).items()}
    sel_f = M.msa_index_select(x["q_idx"], x["k_idx"], top_k, block=BLK)
    sel_u, scores = M.msa_index_select(x["q_idx"], x["k_idx"], top_k, block_scores=True, block=BLK)
    torch.cuda.synchronize()
    assert torch.equal(sel_f, sel_u)      # fused and stored-score routes agree
    sc, sel = scores.cpu().numpy(), sel_f.cpu().numpy()
    qi, ki = P.f64(x["q_idx"]), P.f64(x["k_idx"])
    nb = (L + BLK - 1) // BLK
    n_swaps = 0
    for b in range(2):
        for t in range(0, L, 3 if L > 1024 else 1):
            bt = t // BLK
            for g in range(G):
                ref = O.block_scores_row(qi[b, t, g], ki[b], t, BLK)
                tol = _score_tol(qi[b, t, g], ki[b], t, BLK)
                assert np.all(np.abs(sc[b, g, t, :bt] - ref[:bt]) <= tol[:bt]), (b, t, g)
                assert np.all(np.isneginf(sc[b, g, t, bt:nb]))
                want = O.select_blocks_row(ref, t, BLK, top_k)
                if not P.check_selection_row(sel[b, g, t], want + [-1] * (top_k - len(want)), ref, t,
                                             top_k, block=BLK):
                    n_swaps += 1
    assert n_swaps <= 0.02 * 2 * G * L


def test_integer_inputs_select_bit_exact():
    shape = I.PrefillShape(B=1, L=2048, H=8, G=2, d=128, d_idx=64, top_k=6)
    x = I.prefill_inputs(shape, 66)
    q_idx = I.small_integer_like(x["q_idx"], 67, -1, 1)
    k_idx = I.small_integer_like(x["k_idx"], 68, -1, 1)
    sel = M.msa_index_select(q_idx.to(DEV), k_idx.to(DEV), 6, block=BLK).cpu().numpy()
    qi, ki = O.as_f64(q_idx), O.as_f64(k_idx)
    for t in range(2048):
        for g in range(2):
            bs = O.block_scores_row(qi[0, t, g], ki[0], t, BLK)
            want = O.select_blocks_row(bs, t, BLK, 6)
            assert list(sel[0, g, t]) == want + [-1] * (6 - len(want)), (t, g)


def _check_forward(shape, x, out, sel, rows):
    cpu = {n: x[n].cpu() for n in ("q", "k", "v", "q_idx", "k_idx")}
    ref = P.oracle_rows(cpu["q"], cpu["k"], cpu["v"], cpu["q_idx"], cpu["k_idx"], rows,
                        shape.top_k, block=BLK)
    sel_c = sel.cpu().numpy()
    out_c = out.float().cpu().numpy()
    r = shape.H // shape.G
    errs = []
    for (b, t) in rows:
        for g in range(shape.G):
            bs, blocks, o_ref, _ = ref[(b, t, g)]
            exact = P.check_selection_row(sel_c[b, g, t], blocks + [-1] * (shape.top_k - len(blocks)),
                                          bs, t, shape.top_k, block=BLK)
            if not exact:
                o_ref = P.oracle_rows(cpu["q"], cpu["k"], cpu["v"], cpu["q_idx"], cpu["k_idx"],
                                      [(b, t)], shape.top_k, block=BLK,
                                      sel_override=sel_c)[(b, t, g)][2]
            errs.append(np.abs(out_c[b, t, g * r:(g + 1) * r] - o_ref).ravel())
    e = np.concatenate(errs)
    assert e.max() <= P.OUT_MAX_ABS and e.mean() <= P.OUT_MEAN_ABS, (e.max(), e.mean())


@pytest.mark.parametrize("L,H,G,di,top_k,seed", [(2048, 8, 2, 64, 8, 70), (1000, 16, 4, 128, 5, 71),
                                                 (1536, 16, 16, 128, 3, 72),
                                                 (1024, 16, 1, 64, 4, 73)])
def test_forward_matches_oracle(L, H, G, di, top_k, seed):
    shape = I.PrefillShape(B=1, L=L, H=H, G=G, d=128, d_idx=di, top_k=top_k)
    x = {n: t.to(DEV) for n, t in I.prefill_inputs(shape, seed).items()}
    out, sel, lse = M.msa_forward(x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"], top_k,
                                  want_sel=True, want_lse=True, block=BLK)
    torch.cuda.synchronize()
    _check_forward(shape, x, out, sel, [(0, t) for t in range(L)])


def test_forward_8k_top32_sampled():
    """The 2048-token budget as 32 blocks of 64, sampled rows of every
    boundary class."""
    shape = I.PrefillShape(B=1, L=8192, H=32, G=8, d=128, d_idx=128, top_k=32)
    x = {n: t.to(DEV) for n, t in I.prefill_inputs(shape, 74).items()}
    out, sel = M.msa_forward(x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"], 32, want_sel=True,
                             block=BLK)
    torch.cuda.synchronize()
    rows = sorted({0, 1, 63, 64, 65, 127, 128, 2047, 2048, 2049, 4095, 4096, 8190, 8191} |
                  set(np.random.default_rng(74).integers(0, 8192, 30).tolist()))
    _check_forward(shape, x, out, sel, [(0, t) for t in rows])


def test_dense_limit():
    """top_k >= nb: every block kept, dense causal GQA attention."""
    import torch.nn.functional as F
    shape = I.PrefillShape(B=1, L=1000, H=8, G=2, d=128, d_idx=64, top_k=16)
    x = {n: t.to(DEV) for n, t in I.prefill_inputs(shape, 75).items()}
    out = M.msa_forward(x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"], 16, block=BLK)
    qt = x["q"].float().permute(0, 2, 1, 3)
    kt = x["k"].float().permute(0, 2, 1, 3).repeat_interleave(4, dim=1)
    vt = x["v"].float().permute(0, 2, 1, 3).repeat_interleave(4, dim=1)
    dense = F.scaled_dot_product_attention(qt, kt, vt, is_causal=True).permute(0, 2, 1, 3)
    err = (out.float() - dense).abs()
    assert err.max().item() <= P.OUT_MAX_ABS and err.mean().item() <= P.OUT_MEAN_ABS


def test_cached_and_ragged_equal_whole_rows():
    shape = I.PrefillShape(B=2, L=4096, H=16, G=4, d=128, d_idx=128, top_k=12)
    x = I.prefill_inputs(shape, 76, device=DEV)
    out, sel, lse = M.msa_forward(x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"], 12,
                                  want_sel=True, want_lse=True, block=BLK)
    for t0, n in ((100, 700), (64, 64), (4000, 96), (0, 4096)):
        cache = {nm: x[nm].clone() for nm in ("k", "v", "k_idx")}
        for c in cache.values():
            c[:, t0 + n:] = float("nan")
        o_c, s_c, l_c = M.msa_forward_cached(x["q"][:, t0:t0 + n].contiguous(),
                                             x["q_idx"][:, t0:t0 + n].contiguous(), cache["k"],
                                             cache["v"], cache["k_idx"], t0, 12, want_sel=True,
                                             want_lse=True, block=BLK)
        torch.cuda.synchronize()
        assert torch.equal(s_c, sel[:, :, t0:t0 + n]), (t0, n)
        assert torch.equal(o_c, out[:, t0:t0 + n]), (t0, n)
        assert torch.equal(l_c, lse[:, t0:t0 + n]), (t0, n)
    t0, n = [100, 2047], [700, 2049]
    q = torch.cat([x["q"][b, t0[b]:t0[b] + n[b]] for b in range(2)])
    q_idx = torch.cat([x["q_idx"][b, t0[b]:t0[b] + n[b]] for b in range(2)])
    cache = {nm: x[nm].clone() for nm in ("k", "v", "k_idx")}
    for c in cache.values():
        for b in range(2):
            c[b, t0[b] + n[b]:] = float("nan")
    o_v = M.msa_forward_cached_varlen(q, q_idx, cache["k"], cache["v"], cache["k_idx"], t0, n, 12,
                                      block=BLK)
    torch.cuda.synchronize()
    assert torch.equal(o_v, torch.cat([out[b, t0[b]:t0[b] + n[b]] for b in range(2)]))


@pytest.mark.parametrize("B,Lmax,G,H,di,top_k,lens", [
    (6, 4096, 8, 32, 128, 32, [4096, 1, 63, 64, 65, 3001]),
    (4, 2000, 2, 8, 64, 8, [2000, 129, 1999, 700]),
])
def test_decode_matches_oracle(B, Lmax, G, H, di, top_k, lens):
    shape = I.DecodeShape(B=B, Lmax=Lmax, H=H, G=G, d=128, d_idx=di, top_k=top_k)
    x = I.decode_inputs(shape, 77)
    dev = {n: x[n].to(DEV) for n in ("q", "q_idx", "k_cache", "v_cache", "k_idx_cache")}
    seq = torch.tensor(lens, dtype=torch.int32, device=DEV)
    out, sel = M.msa_sparse_attn_decode(dev["q"], dev["q_idx"], dev["k_cache"], dev["v_cache"],
                                        dev["k_idx_cache"], seq, top_k, want_sel=True, block=BLK)
    torch.cuda.synchronize()
    ref = O.decode(x["q"], x["q_idx"], x["k_cache"], x["v_cache"], x["k_idx_cache"], lens, top_k,
                   block=BLK)
    sel_c = sel.cpu().numpy()
    qi, ki = P.f64(x["q_idx"]), P.f64(x["k_idx_cache"])
    any_swap = False
    for b in range(B):
        t = lens[b] - 1
        for g in range(G):
            bs = O.block_scores_row(qi[b, g], ki[b], t, BLK)
            if not P.check_selection_row(sel_c[b, g], ref["sel"][b, g], bs, t, top_k, block=BLK):
                any_swap = True
    if any_swap:
        ref = O.decode(x["q"], x["q_idx"], x["k_cache"], x["v_cache"], x["k_idx_cache"], lens,
                       top_k, block=BLK, sel_override=sel_c)
    mx, mean = P.out_errors(out.float().cpu().numpy(), ref["out"])
    assert mx <= P.OUT_MAX_ABS and mean <= P.OUT_MEAN_ABS, (mx, mean)


def test_decode_integer_ties_and_fp8_caches():
    """Exact integer scores force ties in the decode top-k; the FP8 decodes
    (index keys, then every cache) against the oracle on the dequantized
    caches, with 64-token blocks."""
    shape = I.DecodeShape(B=3, Lmax=8192, H=16, G=4, d=128, d_idx=64, top_k=10)
    x = I.decode_inputs(shape, 78)
    qi = I.small_integer_like(x["q_idx"], 79, -1, 1)
    ki = I.small_integer_like(x["k_idx_cache"], 80, -1, 1)
    lens = [8192, 5000, 65]
    seq = torch.tensor(lens, dtype=torch.int32, device=DEV)
    d = {n: x[n].to(DEV) for n in ("q", "k_cache", "v_cache")}
    _, sel = M.msa_sparse_attn_decode(d["q"], qi.to(DEV), d["k_cache"], d["v_cache"], ki.to(DEV),
                                      seq, 10, want_sel=True, block=BLK)
    sel = sel.cpu().numpy()
    q64, k64 = O.as_f64(qi), O.as_f64(ki)
    for b in range(3):
        t = lens[b] - 1
        for g in range(4):
            want = O.select_blocks_row(O.block_scores_row(q64[b, g], k64[b], t, BLK), t, BLK, 10)
            assert list(sel[b, g]) == want + [-1] * (10 - len(want)), (b, g)
    # FP8 caches (N(0,1) values, per-row scales)
    codes, scale = I.fp8_index_cache(x["k_idx_cache"])
    k8, ks = I.fp8_rows(x["k_cache"])
    v8, vs = I.fp8_rows(x["v_cache"])
    out8, sel8 = M.msa_sparse_attn_decode_fp8(d["q"], x["q_idx"].to(DEV), k8.to(DEV), ks.to(DEV),
                                              v8.to(DEV), vs.to(DEV), codes.to(DEV),
                                              scale.to(DEV), seq, 10, want_sel=True, block=BLK)
    out8i, sel8i = M.msa_sparse_attn_decode_fp8idx(d["q"], x["q_idx"].to(DEV), d["k_cache"],
                                                   d["v_cache"], codes.to(DEV), scale.to(DEV), seq,
                                                   10, want_sel=True, block=BLK)
    torch.cuda.synchronize()
    kid = O.dequant_rows(codes.numpy(), scale.numpy())
    kc = O.dequant_rows(k8.numpy(), ks.numpy())
    vc = O.dequant_rows(v8.numpy(), vs.numpy())
    qi64 = P.f64(x["q_idx"])
    for out_, sel_, kk, vv in ((out8, sel8, kc, vc), (out8i, sel8i, x["k_cache"], x["v_cache"])):
        s = sel_.cpu().numpy()
        for b in range(3):
            t = lens[b] - 1
            for g in range(4):
                bs = O.block_scores_row(qi64[b, g], kid[b], t, BLK)
                want = O.select_blocks_row(bs, t, BLK, 10)
                P.check_selection_row(s[b, g], want + [-1] * (10 - len(want)), bs, t, 10, block=BLK)
        ref = O.decode(x["q"], x["q_idx"], kk, vv, kid, lens, 10, block=BLK, sel_override=s)
        mx, mean = P.out_errors(out_.float().cpu().numpy(), ref["out"])
        assert mx <= P.OUT_MAX_ABS and mean <= P.OUT_MEAN_ABS, (mx, mean)
