"""GPU parity of the main-branch backward pass (msa_sparse_attn_backward,
through the C ABI) against the fp64 oracle's prefill_backward on the GPU's
own selection.

Tolerance, for each of dq, dk, dv against the fp64 gradients:
  max |gpu - ref| <= 2e-2 * max |ref|   and   ||gpu - ref||_2 <= 1e-2 ||ref||_2.
The kernel rounds P and dZ to bf16 for the tensor-core products (relative
error 2^-9 each), computes D = do . o from the bf16 forward output, and
rounds dq, dk, dv to bf16 (2^-9); accumulation is fp32.  These are
independent relative errors of a few 2^-9 per element, and the bounds leave
a factor of about 3 over them.
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
REL_MAX = 2e-2
REL_L2 = 1e-2


def _grad_close(name, gpu, ref):
    g = np.asarray(gpu, dtype=np.float64)
    e = np.abs(g - ref)
    m = float(np.abs(ref).max())
    rel_max = float(e.max()) / m if m > 0 else float(e.max())
    nr = float(np.linalg.norm(ref))
    rel_l2 = float(np.linalg.norm(g - ref)) / nr if nr > 0 else float(np.linalg.norm(g))
    print(f"{name}: max|ref|={m:.3g} rel_max={rel_max:.2e} rel_l2={rel_l2:.2e}")
    assert rel_max <= REL_MAX and rel_l2 <= REL_L2, (name, rel_max, rel_l2)


def _inputs(shape, seed):
    x = I.prefill_inputs(shape, seed, device="cpu")
    x = {n: x[n].to(DEV) for n in ("q", "k", "v", "q_idx", "k_idx")}
    x["dout"] = I.output_grad(shape, seed, device="cpu").to(DEV)
    return x


def _forward_backward(x, top_k, sel=None, block=128, chunk=0):
    if sel is None:
        out, sel, lse = M.msa_forward(x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"], top_k,
                                      want_sel=True, want_lse=True, block=block)
    else:
        out, lse = M.msa_sparse_attn_prefill(x["q"], x["k"], x["v"], sel, want_lse=True,
                                             block=block)
    dq, dk, dv = M.msa_sparse_attn_backward(x["q"], x["k"], x["v"], out, lse, x["dout"], sel,
                                            block=block, chunk=chunk)
    torch.cuda.synchronize()
    return sel, dq, dk, dv


@pytest.mark.parametrize("B,L,H,G,top_k,seed", [
    (1, 1024, 8, 2, 4, 20),      # R = 4, ragged item lists, several key blocks
    (2, 640, 4, 4, 3, 21),       # R = 1 (128 queries per item), two sequences
    (1, 768, 32, 2, 2, 22),      # R = 16 (8 queries per item)
    (1, 512, 8, 1, 8, 23),       # top_k >= nb: dense causal attention
    (1, 1152, 16, 8, 1, 24),     # top_k = 1: the local block only
    (1, 2560, 16, 2, 17, 28),    # R = 8, top_k = 17 (32-slot dq reduction)
])
def test_backward_matches_oracle(B, L, H, G, top_k, seed):
    shape = I.PrefillShape(B=B, L=L, H=H, G=G, d=128, d_idx=128, top_k=top_k)
    x = _inputs(shape, seed)
    sel, dq, dk, dv = _forward_backward(x, top_k)
    ref = O.prefill_backward(x["q"], x["k"], x["v"], sel.cpu().numpy(), x["dout"], block=128)
    _grad_close("dq", P.f64(dq), ref["dq"])
    _grad_close("dk", P.f64(dk), ref["dk"])
    _grad_close("dv", P.f64(dv), ref["dv"])


def test_backward_blocks_nobody_selects_get_zero():
    """A selection of block 0 only (for every query): key blocks 1.. are
    attended by nobody, so their units are empty and dk, dv there are 0."""
    shape = I.PrefillShape(B=1, L=512, H=8, G=2, d=128, d_idx=128, top_k=2)
    x = _inputs(shape, 25)
    sel = torch.full((1, 2, 512, 2), -1, dtype=torch.int32)
    sel[..., 0] = 0
    sel = sel.to(DEV)
    sel_, dq, dk, dv = _forward_backward(x, 2, sel=sel)
    assert not dk[:, 128:].any() and not dv[:, 128:].any()
    ref = O.prefill_backward(x["q"], x["k"], x["v"], sel.cpu().numpy(), x["dout"], block=128)
    _grad_close("dq", P.f64(dq), ref["dq"])
    _grad_close("dk", P.f64(dk), ref["dk"])
    _grad_close("dv", P.f64(dv), ref["dv"])


@pytest.mark.parametrize("L,top_k,chunk", [(2048, 5, 0), (2048, 5, 640), (2304, 18, 0)])
def test_backward_run_to_run(L, top_k, chunk):
    """dq rows are each computed from their own (query, slot) rows and summed
    in slot order; dk and dv sum a key block's items in the order of the
    reverse index's lists, which are sorted by query position.  So all
    three are bit-identical across runs, one chunk or several.  With
    top_k = 18 over 18 blocks every query selects every earlier block, so
    the lists of blocks 0 and 1 (2304 and 2176 entries) take the bitmap
    route of the ordering step and the others the direct one."""
    shape = I.PrefillShape(B=1, L=L, H=16, G=4, d=128, d_idx=128, top_k=top_k)
    x = _inputs(shape, 26)
    sel, dq1, dk1, dv1 = _forward_backward(x, top_k, chunk=chunk)
    for _ in range(2):
        _, dq2, dk2, dv2 = _forward_backward(x, top_k, sel=sel, chunk=chunk)
        assert torch.equal(dq1, dq2)
        assert torch.equal(dk1, dk2)
        assert torch.equal(dv1, dv2)
    ref = O.prefill_backward(x["q"], x["k"], x["v"], sel.cpu().numpy(), x["dout"], block=128)
    for name, g in (("dq", dq1), ("dk", dk1), ("dv", dv1)):
        _grad_close(name, P.f64(g), ref[name])


def test_backward_32k_sampled():
    """32K prefill (H=32, G=8, top_k=16): sampled dq rows, and dk/dv of whole
    key blocks (the last block, a middle one, block 0 of group 0, the one
    with the longest query list), each summed by the oracle over every
    (query, group) row whose GPU selection holds the block."""
    shape = I.PrefillShape(B=1, L=32768, H=32, G=8, d=128, d_idx=128, top_k=16)
    x = _inputs(shape, 1)
    sel, dq, dk, dv = _forward_backward(x, 16)
    sel_np = sel.cpu().numpy()
    L, H, G, r, blk = 32768, 32, 8, 4, 128
    sc = 1.0 / np.sqrt(128.0)
    rng = np.random.default_rng(5)
    q_cpu = x["q"][0].cpu()
    k_cpu, v_cpu = x["k"][0].cpu(), x["v"][0].cpu()
    dout = x["dout"].cpu()

    def qrow(t):
        return P.f64(q_cpu[t])

    dq_np = P.f64(dq[0])
    ts = sorted(set([0, 127, 128, L - 1] + rng.integers(0, L, 40).tolist()))
    for t in ts:
        for g in (0, 5):
            blocks = P.sel_set(sel_np[0, g, t])
            tok = O.selected_tokens(blocks, t, blk)
            tk = torch.from_numpy(tok)
            gq, _, _ = O.attend_rows_grad(qrow(t)[g * r:(g + 1) * r], P.f64(k_cpu[tk, g]),
                                          P.f64(v_cpu[tk, g]),
                                          P.f64(dout[0, t, g * r:(g + 1) * r]), sc)
            _grad_close(f"dq t={t} g={g}", dq_np[t, g * r:(g + 1) * r], gq)
    nb = L // blk
    for (j, g) in ((nb - 1, 3), (nb // 2, 6), (0, 0)):
        k64 = P.f64(k_cpu[:, g])
        v64 = P.f64(v_cpu[:, g])
        rows = np.nonzero((sel_np[0, g] == j).any(axis=1))[0]
        gk = np.zeros((blk, 128))
        gv = np.zeros((blk, 128))
        for t in rows.tolist():
            tok = O.selected_tokens(P.sel_set(sel_np[0, g, t]), int(t), blk)
            _, gkt, gvt = O.attend_rows_grad(qrow(int(t))[g * r:(g + 1) * r], k64[tok], v64[tok],
                                             P.f64(dout[0, int(t), g * r:(g + 1) * r]), sc)
            m = (tok >= j * blk) & (tok < (j + 1) * blk)
            gk[tok[m] - j * blk] += gkt[m]
            gv[tok[m] - j * blk] += gvt[m]
        _grad_close(f"dk block {j} g={g} ({rows.size} rows)", P.f64(dk[0, j * blk:(j + 1) * blk, g]), gk)
        _grad_close(f"dv block {j} g={g}", P.f64(dv[0, j * blk:(j + 1) * blk, g]), gv)


def test_backward_query_chunks():
    """Four query chunks of 256 (p->chunk): dq equals the one-chunk run bit
    for bit (each partial row depends only on its own query row); dk and dv
    are summed across chunks in fp32 and match the oracle under the same
    bounds.  A selection leaving blocks unselected keeps them at zero
    through every chunk."""
    shape = I.PrefillShape(B=2, L=1024, H=8, G=2, d=128, d_idx=128, top_k=3)
    x = _inputs(shape, 27)
    out, sel, lse = M.msa_forward(x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"], 3,
                                  want_sel=True, want_lse=True)
    one = M.msa_sparse_attn_backward(x["q"], x["k"], x["v"], out, lse, x["dout"], sel)
    four = M.msa_sparse_attn_backward(x["q"], x["k"], x["v"], out, lse, x["dout"], sel, chunk=256)
    torch.cuda.synchronize()
    assert torch.equal(one[0], four[0])
    ref = O.prefill_backward(x["q"], x["k"], x["v"], sel.cpu().numpy(), x["dout"], block=128)
    for name, g in zip(("dq", "dk", "dv"), four):
        _grad_close(f"{name} (4 chunks)", P.f64(g), ref[name])
    # block 0 only: blocks 1.. are attended by nobody in any chunk
    sel0 = torch.full_like(sel, -1)
    sel0[..., 0] = 0
    out0, lse0 = M.msa_sparse_attn_prefill(x["q"], x["k"], x["v"], sel0, want_lse=True)
    dq0, dk0, dv0 = M.msa_sparse_attn_backward(x["q"], x["k"], x["v"], out0, lse0, x["dout"], sel0,
                                               chunk=128)
    torch.cuda.synchronize()
    assert not dk0[:, 128:].any() and not dv0[:, 128:].any()
    ref0 = O.prefill_backward(x["q"], x["k"], x["v"], sel0.cpu().numpy(), x["dout"], block=128)
    _grad_close("dk block 0 (8 chunks)", P.f64(dk0[:, :128]), ref0["dk"][:, :128])
    _grad_close("dv block 0 (8 chunks)", P.f64(dv0[:, :128]), ref0["dv"][:, :128])


@pytest.mark.parametrize("B,L,H,G,top_k,blk,seed", [
    (2, 1000, 8, 2, 4, 128, 40),    # partial last block (104 keys), two sequences
    (1, 2049, 16, 4, 5, 128, 41),   # a last block of one key
    (1, 1024, 8, 2, 6, 64, 42),     # 64-token blocks: half of the key tile
    (2, 777, 4, 4, 8, 64, 43),      # 64-token blocks, partial last block, R = 1
    (1, 640, 32, 2, 32, 64, 44),    # R = 16, top_k = 32 >= nb: dense causal
])
def test_backward_any_length_and_block64(B, L, H, G, top_k, blk, seed):
    shape = I.PrefillShape(B=B, L=L, H=H, G=G, d=128, d_idx=128, top_k=top_k, block=blk)
    x = _inputs(shape, seed)
    sel, dq, dk, dv = _forward_backward(x, top_k, block=blk)
    ref = O.prefill_backward(x["q"], x["k"], x["v"], sel.cpu().numpy(), x["dout"], block=blk)
    _grad_close("dq", P.f64(dq), ref["dq"])
    _grad_close("dk", P.f64(dk), ref["dk"])
    _grad_close("dv", P.f64(dv), ref["dv"])


@pytest.mark.parametrize("blk", [64, 128])
def test_backward_chunks_any_length(blk):
    """Query chunks of 384 packed rows over two sequences of 1000 (chunks
    that straddle the sequence boundary): dq equals the one-chunk run bit
    for bit, dk and dv match the oracle."""
    shape = I.PrefillShape(B=2, L=1000, H=8, G=2, d=128, d_idx=128, top_k=5, block=blk)
    x = _inputs(shape, 45)
    sel, dq1, _, _ = _forward_backward(x, 5, block=blk)
    _, dq, dk, dv = _forward_backward(x, 5, sel=sel, block=blk, chunk=384)
    assert torch.equal(dq, dq1)
    ref = O.prefill_backward(x["q"], x["k"], x["v"], sel.cpu().numpy(), x["dout"], block=blk)
    for name, g in (("dq", dq), ("dk", dk), ("dv", dv)):
        _grad_close(f"{name} (chunks of 384)", P.f64(g), ref[name])


def test_backward_ordering_routes_bit_reproducible():
    """A selection of block 0 plus the local block for every row: block 0's
    list holds all 8192 rows (the ordering step's bitmap route, over 4096
    entries), the local blocks' lists 128 each (direct rank count).  dq, dk
    and dv must be bit-identical over runs and match the oracle."""
    L, top_k = 8192, 2
    shape = I.PrefillShape(B=1, L=L, H=8, G=2, d=128, d_idx=128, top_k=top_k)
    x = _inputs(shape, 46)
    t = torch.arange(L, dtype=torch.int32)
    sel = torch.full((1, 2, L, top_k), -1, dtype=torch.int32)
    sel[..., 0] = 0
    sel[..., 1] = torch.where(t // 128 > 0, t // 128, torch.full_like(t, -1))
    sel = sel.to(DEV)
    _, dq1, dk1, dv1 = _forward_backward(x, top_k, sel=sel)
    _, dq2, dk2, dv2 = _forward_backward(x, top_k, sel=sel)
    assert torch.equal(dq1, dq2) and torch.equal(dk1, dk2) and torch.equal(dv1, dv2)
    ref = O.prefill_backward(x["q"], x["k"], x["v"], sel.cpu().numpy(), x["dout"], block=128)
    for name, g in (("dq", dq1), ("dk", dk1), ("dv", dv1)):
        _grad_close(f"{name} (block 0 for every row)", P.f64(g), ref[name])
