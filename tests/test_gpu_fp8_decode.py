"""GPU tests of the FP8 caches for decode (msa_sparse_attn_decode_fp8idx: index
keys in FP8; msa_sparse_attn_decode_fp8: index keys, keys and values in FP8)
and of the row quantizer (msa_quantize_e4m3_rows).

The oracle reads the same E4M3 codes and per-token scales, decoded by its own
e4m3_to_f64 (pinned in test_oracle_pins.py), so the selection and the output
are held to the same parity rule as the bf16 decode: sets equal except
boundary swaps of near-tied blocks, outputs within the tolerances of the
parity helpers.  Integer-valued codes make scores exact, and then the
selection must match bit for bit, ties included.
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


def test_quantize_matches_library_conversion():
    gen = torch.Generator().manual_seed(51)
    x = torch.randn((333, 128), generator=gen).to(torch.bfloat16)
    x[7] = 0                                      # all-zero row: scale 1
    x[8] *= 1000                                  # large row
    x[9, :] = 2.0 ** -20                          # tiny row
    codes, scale = M.msa_quantize_e4m3_rows(x.to(DEV))
    torch.cuda.synchronize()
    want_c, want_s = I.fp8_index_cache(x[None])
    assert torch.equal(scale.cpu(), want_s[0])
    assert torch.equal(codes.cpu(), want_c[0])
    # decoded rows reproduce the input to E4M3 precision (3 mantissa bits)
    deq = O.dequant_rows(codes.cpu().numpy(), scale.cpu().numpy())
    x64 = x.double().numpy()
    assert np.all(np.abs(deq - x64) <= np.abs(x64) * 2.0 ** -4 + scale.cpu().numpy()[:, None] * 2.0 ** -9)


@pytest.mark.parametrize("B,Lmax,G,H,di,top_k,lens", [
    (4, 4096, 8, 32, 128, 16, [4096, 1, 129, 3000]),
    (5, 2048, 2, 8, 64, 4, [2048, 128, 127, 777, 1500]),
])
def test_fp8idx_decode_matches_oracle(B, Lmax, G, H, di, top_k, lens):
    shape = I.DecodeShape(B=B, Lmax=Lmax, H=H, G=G, d=128, d_idx=di, top_k=top_k)
    x = I.decode_inputs(shape, 52)
    codes, scale = I.fp8_index_cache(x["k_idx_cache"])
    d = {n: x[n].to(DEV) for n in ("q", "q_idx", "k_cache", "v_cache")}
    out, sel = M.msa_sparse_attn_decode_fp8idx(d["q"], d["q_idx"], d["k_cache"], d["v_cache"],
                                               codes.to(DEV), scale.to(DEV),
                                               torch.tensor(lens, dtype=torch.int32, device=DEV),
                                               top_k, want_sel=True)
    torch.cuda.synchronize()
    ki = O.dequant_rows(codes.numpy(), scale.numpy())          # [B, Lmax, d_idx] fp64
    ref = O.decode(x["q"], x["q_idx"], x["k_cache"], x["v_cache"], ki, lens, top_k)
    sel_c = sel.cpu().numpy()
    qi = P.f64(x["q_idx"])
    any_swap = False
    for b in range(B):
        t = lens[b] - 1
        for g in range(G):
            bs = O.block_scores_row(qi[b, g], ki[b], t, 128)
            if not P.check_selection_row(sel_c[b, g], ref["sel"][b, g], bs, t, top_k):
                any_swap = True
    if any_swap:
        ref = O.decode(x["q"], x["q_idx"], x["k_cache"], x["v_cache"], ki, lens, top_k,
                       sel_override=sel_c)
    mx, mean = P.out_errors(out.float().cpu().numpy(), ref["out"])
    assert mx <= P.OUT_MAX_ABS and mean <= P.OUT_MEAN_ABS, (mx, mean)


def test_fp8idx_integer_codes_select_bit_exact():
    """Codes of the values -2..2 with power-of-two scales and integer index
    queries: every score is exact on both sides, ties included."""
    shape = I.DecodeShape(B=3, Lmax=8192, H=8, G=2, d=128, d_idx=128, top_k=6)
    x = I.decode_inputs(shape, 53)
    gen = torch.Generator().manual_seed(54)
    vals = torch.randint(-2, 3, (3, 8192, 128), generator=gen).float()
    codes = vals.to(torch.float8_e4m3fn).view(torch.uint8)
    scale = (2.0 ** torch.randint(-2, 3, (3, 8192), generator=gen)).float()
    qi = I.small_integer_like(x["q_idx"], 55, -1, 1)
    lens = [8192, 5000, 700]
    d = {n: x[n].to(DEV) for n in ("q", "k_cache", "v_cache")}
    _, sel = M.msa_sparse_attn_decode_fp8idx(d["q"], qi.to(DEV), d["k_cache"], d["v_cache"],
                                             codes.to(DEV), scale.to(DEV),
                                             torch.tensor(lens, dtype=torch.int32, device=DEV), 6,
                                             want_sel=True)
    sel = sel.cpu().numpy()
    q64 = O.as_f64(qi)
    k64 = O.dequant_rows(codes.numpy(), scale.numpy())
    for b in range(3):
        t = lens[b] - 1
        for g in range(2):
            bs = O.block_scores_row(q64[b, g], k64[b], t, 128)
            want = O.select_blocks_row(bs, t, 128, 6)
            assert list(sel[b, g]) == want + [-1] * (6 - len(want)), (b, g, sel[b, g], want)


@pytest.mark.parametrize("B,Lmax,G,H,di,top_k,lens", [
    (4, 4096, 8, 32, 128, 16, [4096, 1, 129, 3000]),
    (5, 2048, 2, 8, 64, 4, [2048, 128, 127, 777, 1500]),
    (2, 1024, 1, 16, 128, 3, [1024, 300]),
])
def test_all_fp8_decode_matches_oracle(B, Lmax, G, H, di, top_k, lens):
    shape = I.DecodeShape(B=B, Lmax=Lmax, H=H, G=G, d=128, d_idx=di, top_k=top_k)
    x = I.decode_inputs(shape, 56)
    ki8, kis = I.fp8_rows(x["k_idx_cache"])
    k8, ks = I.fp8_rows(x["k_cache"])
    v8, vs = I.fp8_rows(x["v_cache"])
    # garbage past each sequence's length, including NaN codes: never read
    for b, n in enumerate(lens):
        for t in (ki8, k8, v8):
            t[b, n:] = 0x7F
    dv = lambda t: t.to(DEV)
    out, sel = M.msa_sparse_attn_decode_fp8(dv(x["q"]), dv(x["q_idx"]), dv(k8), dv(ks), dv(v8),
                                            dv(vs), dv(ki8), dv(kis),
                                            torch.tensor(lens, dtype=torch.int32, device=DEV),
                                            top_k, want_sel=True)
    torch.cuda.synchronize()
    kd = O.dequant_rows(k8.numpy(), ks.numpy())
    vd = O.dequant_rows(v8.numpy(), vs.numpy())
    kid = O.dequant_rows(ki8.numpy(), kis.numpy())
    ref = O.decode(x["q"], x["q_idx"], kd, vd, kid, lens, top_k)
    sel_c = sel.cpu().numpy()
    qi = P.f64(x["q_idx"])
    any_swap = False
    for b in range(B):
        t = lens[b] - 1
        for g in range(G):
            bs = O.block_scores_row(qi[b, g], kid[b], t, 128)
            if not P.check_selection_row(sel_c[b, g], ref["sel"][b, g], bs, t, top_k):
                any_swap = True
    if any_swap:
        ref = O.decode(x["q"], x["q_idx"], kd, vd, kid, lens, top_k, sel_override=sel_c)
    mx, mean = P.out_errors(out.float().cpu().numpy(), ref["out"])
    assert mx <= P.OUT_MAX_ABS and mean <= P.OUT_MEAN_ABS, (mx, mean)
