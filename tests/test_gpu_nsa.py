"""GPU parity of the NSA-style variant (compression and sliding-window
branches beside MSA's selection, mixed by caller-given gates; "MiniMax M3
sparse attention" explainer, §3.1) against the fp64 oracle's compress_kv,
nsa_branches and nsa_forward.

Tolerances: branch and gated outputs within the prefill's max-abs 2e-2 /
mean-abs 2e-3 of the oracle (bf16 P and output, fp32 accumulation, and for
the compression branch the compressed tokens rounded to bf16, relative
2^-9, which moves a logit by about 2e-3); lse within 2e-3 absolute.
Compressed tokens within 2^-8 relative (one bf16 rounding of an fp32 mean)
plus 1e-6.  Rows that see no compressed token are exactly zero with lse
-inf.
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
LSE_ABS = 2e-3


def _inputs(B, L, H, G, seed, top_k=4):
    shape = I.PrefillShape(B=B, L=L, H=H, G=G, d=128, d_idx=128, top_k=top_k)
    return shape, I.prefill_inputs(shape, seed, device=DEV)


def _close(gpu, ref, name):
    g = gpu.float().cpu().numpy()
    e = np.abs(g - ref)
    assert e.max() <= P.OUT_MAX_ABS and e.mean() <= P.OUT_MEAN_ABS, (name, e.max(), e.mean())


def _lse_close(gpu, ref, name):
    g = gpu.cpu().numpy().astype(np.float64)
    fin = np.isfinite(ref)
    assert np.array_equal(np.isfinite(g), fin), name
    assert np.all(g[~fin] == -np.inf), name
    if fin.any():
        err = np.abs(g[fin] - ref[fin]).max()
        assert err <= LSE_ABS, (name, err)


@pytest.mark.parametrize("L,G,blk", [(1000, 4, 128), (777, 2, 64), (256, 8, 128), (1, 1, 64)])
def test_compress_kv(L, G, blk):
    _, x = _inputs(2, L, G, G, 60)
    kc, vc = M.msa_nsa_compress_kv(x["k"], x["v"], block=blk)
    torch.cuda.synchronize()
    rk, rv = O.compress_kv(x["k"].cpu(), x["v"].cpu(), blk)
    for g_, r_ in ((kc, rk), (vc, rv)):
        e = np.abs(P.f64(g_) - r_)
        assert np.all(e <= 2.0 ** -8 * np.abs(r_) + 1e-6), e.max()


@pytest.mark.parametrize("B,L,H,G,window,seed", [
    (2, 1000, 8, 2, 100, 61),     # R = 4, windows across query and key tiles, ragged tail
    (1, 777, 16, 4, 1, 62),       # window 1: v[t]
    (1, 2049, 8, 8, 512, 63),     # R = 1 (128 queries per tile), one key in the last tile
    (2, 640, 32, 2, 4096, 64),    # R = 16, window > L: dense causal attention
    (1, 300, 4, 4, 130, 65),      # R = 1, window just over one key tile
])
def test_window_branch(B, L, H, G, window, seed):
    _, x = _inputs(B, L, H, G, seed)
    out, lse = M.msa_nsa_window_attn(x["q"], x["k"], x["v"], window, want_lse=True)
    torch.cuda.synchronize()
    sel = np.full((B, G, L, 1), -1, dtype=np.int32)
    ref = O.nsa_branches(x["q"].cpu(), x["k"].cpu(), x["v"].cpu(), sel, window=window, block=128)
    _close(out, ref["out_win"], "out_win")
    _lse_close(lse, ref["lse_win"], "lse_win")


@pytest.mark.parametrize("B,L,H,G,blk,seed", [
    (2, 1000, 8, 2, 128, 66),     # R = 4: rows of the first block see nothing
    (1, 2049, 16, 4, 64, 67),     # 64-token blocks: 32 compressed tokens, one partial tile
    (1, 20000, 8, 8, 128, 68),    # R = 1, 157 compressed tokens: two key tiles
    (2, 100, 4, 2, 128, 69),      # L < block: every row sees nothing
])
def test_compressed_branch(B, L, H, G, blk, seed):
    _, x = _inputs(B, L, H, G, seed)
    kc, vc = M.msa_nsa_compress_kv(x["k"], x["v"], block=blk)
    out, lse = M.msa_nsa_compressed_attn(x["q"], kc, vc, block=blk, want_lse=True)
    torch.cuda.synchronize()
    sel = np.full((B, G, L, 1), -1, dtype=np.int32)
    if L > 4096:   # sampled rows: both ends, block boundaries, the tail
        rows = sorted({(b, t) for b in range(B) for t in
                       [0, blk - 2, blk - 1, blk, 2 * blk - 1, 128 * blk - 1, 128 * blk, L // 2,
                        L - 2, L - 1] if 0 <= t < L})
    else:
        rows = None
    ref = O.nsa_branches(x["q"].cpu(), x["k"].cpu(), x["v"].cpu(), sel, window=1, block=blk,
                         rows=rows)
    if rows is None:
        _close(out, ref["out_cmp"], "out_cmp")
        _lse_close(lse, ref["lse_cmp"], "lse_cmp")
    else:
        bi = [b for b, _ in rows]
        ti = [t for _, t in rows]
        _close(out[bi, ti], ref["out_cmp"][bi, ti], "out_cmp")
        _lse_close(lse[bi, ti], ref["lse_cmp"][bi, ti], "lse_cmp")
    # no complete block at or before t: exactly zero
    t_none = min(L, blk - 1)
    assert not out[:, :t_none].any()
    assert torch.all(lse[:, :t_none] == -float("inf"))


@pytest.mark.parametrize("B,L,H,G,top_k,blk,window,seed", [
    (1, 1000, 8, 2, 4, 128, 200, 70),
    (2, 777, 16, 4, 6, 64, 64, 71),
])
def test_nsa_forward(B, L, H, G, top_k, blk, window, seed):
    """The whole call against the oracle on the GPU's own (validated)
    selection, with random gates."""
    shape, x = _inputs(B, L, H, G, seed, top_k=top_k)
    rng = np.random.default_rng(seed)
    gates = torch.from_numpy(rng.uniform(0, 1, (B, L, H, 3)).astype(np.float32)).to(DEV)
    out, sel = M.msa_nsa_forward(x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"], gates, top_k,
                                 window, block=blk, want_sel=True)
    torch.cuda.synchronize()
    cpu = {n: x[n].cpu() for n in ("q", "k", "v", "q_idx", "k_idx")}
    sel_c = sel.cpu().numpy()
    k_idx64 = cpu["k_idx"].double().numpy()
    for b in range(B):
        for t in range(0, L, 37):
            for g in range(G):
                bs = O.block_scores_row(O.as_f64(cpu["q_idx"][b, t, g]), k_idx64[b], t, blk)
                want = O.select_blocks_row(bs, t, blk, top_k)
                P.check_selection_row(sel_c[b, g, t], want + [-1] * (top_k - len(want)), bs, t,
                                      top_k, block=blk)
    ref, _ = O.nsa_forward(cpu["q"], cpu["k"], cpu["v"], sel_c, gates.cpu().numpy(), window,
                           block=blk)
    _close(out, ref, "nsa out")


def test_gate_in_place():
    """The gate kernel against the oracle's combination of the same bf16
    branch outputs, written over its selection-branch input."""
    g = torch.Generator(device="cpu").manual_seed(72)
    shape = (2, 300, 8, 128)
    o = [torch.randn(shape, generator=g).to(torch.bfloat16).to(DEV) for _ in range(3)]
    gates = torch.rand(shape[:3] + (3,), generator=g).to(DEV)
    want = sum(gates[..., i:i + 1].double().cpu() * o[i].double().cpu() for i in range(3))
    out = o[1].clone()
    M.msa_nsa_gate(gates, o[0], out, o[2], out=out)
    torch.cuda.synchronize()
    e = (out.double().cpu() - want).abs()
    assert (e <= 2.0 ** -8 * want.abs() + 1e-6).all(), e.max()


def _growing_keys(x, period):
    """Keys scaled by 2^(s/period) along the sequence, so that a row's
    maximum keeps rising from key tile to key tile by far more than the 2^8
    the kernel allows before it rescales its accumulator."""
    L = x["k"].shape[1]
    f = torch.pow(2.0, torch.arange(L, dtype=torch.float32, device=x["k"].device) / period)
    k = (x["k"].float() * f[None, :, None, None]).to(torch.bfloat16)
    return dict(x, k=k.contiguous())


def test_window_branch_rescales_as_the_maximum_grows():
    """Keys growing 2x every 128 positions: every key tile raises the row
    maximum, so O and l are rescaled in place tile after tile (window 1024
    over L = 1024 and 600: dense causal attention)."""
    for L in (1024, 600):
        _, x = _inputs(1, L, 8, 2, 73)
        x = _growing_keys(x, 128.0)
        out, lse = M.msa_nsa_window_attn(x["q"], x["k"], x["v"], 1024, want_lse=True)
        torch.cuda.synchronize()
        sel = np.full((1, 2, L, 1), -1, dtype=np.int32)
        ref = O.nsa_branches(x["q"].cpu(), x["k"].cpu(), x["v"].cpu(), sel, window=1024)
        _close(out, ref["out_win"], "out_win (growing keys)")
        g = lse.cpu().numpy().astype(np.float64)
        rel = np.abs(g - ref["lse_win"]) / np.maximum(1.0, np.abs(ref["lse_win"]))
        assert rel.max() <= 1e-3, rel.max()


def test_compressed_branch_rescales_as_the_maximum_grows():
    """Compressed keys growing along the sequence (2x every 3000 tokens):
    the second compressed-token tile raises a late row's maximum by about
    140 raw score units over the first's, past the kernel's 2^8 threshold
    (63 units at scale 1/sqrt(128)), while the scores (about 250) stay
    small enough for the bf16 rounding of the compressed keys to move a
    logit by only ~0.04."""
    _, x = _inputs(1, 20000, 8, 8, 74)
    x = _growing_keys(x, 3000.0)
    kc, vc = M.msa_nsa_compress_kv(x["k"], x["v"])
    out, lse = M.msa_nsa_compressed_attn(x["q"], kc, vc, want_lse=True)
    torch.cuda.synchronize()
    rows = [(0, t) for t in (127, 5000, 16383, 16384, 16511, 16512, 19999)]
    sel = np.full((1, 8, 20000, 1), -1, dtype=np.int32)
    ref = O.nsa_branches(x["q"].cpu(), x["k"].cpu(), x["v"].cpu(), sel, window=1, rows=rows)
    ti = [t for _, t in rows]
    _close(out[0, ti], ref["out_cmp"][0, ti], "out_cmp (growing keys)")
    g = lse[0, ti].cpu().numpy().astype(np.float64)
    r = ref["lse_cmp"][0, ti]
    rel = np.abs(g - r) / np.maximum(1.0, np.abs(r))
    assert rel.max() <= 3e-3, rel.max()
