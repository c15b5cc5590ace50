"""GPU tests of msa_forward_cached: prefill of a chunk of new tokens at
positions [t0, t0+n) against key caches that already hold every row up to
t0+n.  Each new query attends exactly as in a whole-sequence prefill of
length t0+n (rows are computed independently of one another), so out, sel
and lse must equal rows [t0, t0+n) of msa_forward bit for bit; the
whole-sequence path is checked against the oracle elsewhere.  Cache rows at
or beyond t0+n are filled with NaN to show they are never read.
"""
import numpy as np
import pytest
import torch

from block_sparse_long_08_b200 import inputs as I
from block_sparse_long_08_b200 import msa as M
from tests import _parity as P

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def full_run():
    shape = I.PrefillShape(B=2, L=4096, H=16, G=4, d=128, d_idx=128, top_k=8)
    x = I.prefill_inputs(shape, 41, device=DEV)
    out, sel, lse = M.msa_forward(x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"], shape.top_k,
                                  want_sel=True, want_lse=True)
    torch.cuda.synchronize()
    return shape, x, out, sel, lse


@pytest.mark.parametrize("t0,n,chunk", [(0, 1024, 0), (1536, 1024, 0), (3072, 1024, 0),
                                        (1024, 2048, 512),
                                        # positions and counts of any size
                                        (100, 700, 0), (1000, 1, 0), (4000, 96, 0),
                                        (1, 4095, 1024), (2047, 2, 0), (0, 77, 0)])
def test_cached_prefill_equals_whole_sequence_rows(full_run, t0, n, chunk):
    shape, x, out, sel, lse = full_run
    cache = {nm: x[nm].clone() for nm in ("k", "v", "k_idx")}
    for t in cache.values():
        t[:, t0 + n:] = float("nan")           # never read
    q = x["q"][:, t0:t0 + n].contiguous()
    q_idx = x["q_idx"][:, t0:t0 + n].contiguous()
    o_c, s_c, l_c = M.msa_forward_cached(q, q_idx, cache["k"], cache["v"], cache["k_idx"], t0,
                                         shape.top_k, want_sel=True, want_lse=True, chunk=chunk)
    torch.cuda.synchronize()
    assert torch.equal(s_c, sel[:, :, t0:t0 + n])
    assert torch.equal(o_c, out[:, t0:t0 + n])
    assert torch.equal(l_c, lse[:, t0:t0 + n])


def test_cached_prefill_against_oracle():
    # a prefix of 3 blocks continued by 2 blocks; the oracle sees the whole
    # sequence and evaluates the new rows
    shape = I.PrefillShape(B=1, L=2048, H=8, G=2, d=128, d_idx=64, top_k=4)
    x = I.prefill_inputs(shape, 42, device=DEV)
    t0, n = 384, 256
    o_c, s_c = M.msa_forward_cached(x["q"][:, t0:t0 + n].contiguous(),
                                    x["q_idx"][:, t0:t0 + n].contiguous(), x["k"], x["v"],
                                    x["k_idx"], t0, shape.top_k, want_sel=True)
    torch.cuda.synchronize()
    cpu = {nm: x[nm].cpu() for nm in ("q", "k", "v", "q_idx", "k_idx")}
    rows = [(0, t) for t in range(t0, t0 + n)]
    ref = P.oracle_rows(cpu["q"], cpu["k"], cpu["v"], cpu["q_idx"], cpu["k_idx"], rows,
                        shape.top_k)
    sel_c = s_c.cpu().numpy()                   # [1, G, n, top_k]
    # the GPU selection laid out over the whole sequence, to score against
    sel_full = np.full((1, shape.G, shape.L, shape.top_k), -1, dtype=np.int32)
    sel_full[:, :, t0:t0 + n] = sel_c
    out_c = o_c.float().cpu().numpy()           # [1, n, H, d]
    r = shape.H // shape.G
    errs = []
    for (b, t) in rows:
        for g in range(shape.G):
            bs, blocks, o_ref, _ = ref[(b, t, g)]
            ref_row = blocks + [-1] * (shape.top_k - len(blocks))
            exact = P.check_selection_row(sel_c[b, g, t - t0], ref_row, bs, t, shape.top_k)
            if not exact:   # score against the GPU's (validated) selection
                o_ref = P.oracle_rows(cpu["q"], cpu["k"], cpu["v"], cpu["q_idx"], cpu["k_idx"],
                                      [(b, t)], shape.top_k, sel_override=sel_full)[(b, t, g)][2]
            errs.append(np.abs(out_c[b, t - t0, g * r:(g + 1) * r] - o_ref))
    e = np.concatenate([v.ravel() for v in errs])
    assert e.max() <= P.OUT_MAX_ABS and e.mean() <= P.OUT_MEAN_ABS, (e.max(), e.mean())


@pytest.mark.parametrize("t0,n,chunk", [([1024, 2944], [768, 1152], 0),
                                        ([100, 2947], [700, 1149], 0),
                                        ([0, 3000], [77, 1], 0),
                                        ([5, 129], [3000, 3967], 1024)])
def test_ragged_batch_equals_whole_sequence_rows(full_run, t0, n, chunk):
    """Sequences continuing at different positions with different numbers of
    new tokens (one with none), query rows packed, the whole batch in one
    launch per kernel.  Cache rows past each sequence's t0 + n hold NaN:
    they must never be read."""
    shape, x, out, sel, lse = full_run
    t0, n = t0 + [0], n + [0]          # a third sequence with no new tokens
    B = 2
    q = torch.cat([x["q"][b, t0[b]:t0[b] + n[b]] for b in range(B)])
    q_idx = torch.cat([x["q_idx"][b, t0[b]:t0[b] + n[b]] for b in range(B)])
    cache = {nm: x[nm].clone() for nm in ("k", "v", "k_idx")}
    for c in cache.values():
        for b in range(B):
            c[b, t0[b] + n[b]:] = float("nan")
    o_c, l_c = M.msa_forward_cached_varlen(q, q_idx, cache["k"], cache["v"], cache["k_idx"],
                                           t0[:B], n[:B], shape.top_k, want_lse=True, chunk=chunk)
    torch.cuda.synchronize()
    want_o = torch.cat([out[b, t0[b]:t0[b] + n[b]] for b in range(B)])
    want_l = torch.cat([lse[b, t0[b]:t0[b] + n[b]] for b in range(B)])
    assert torch.equal(o_c, want_o)
    assert torch.equal(l_c, want_l)
    # an empty sequence in the batch
    k3 = torch.cat([cache["k"], cache["k"][:1]])
    v3 = torch.cat([cache["v"], cache["v"][:1]])
    ki3 = torch.cat([cache["k_idx"], cache["k_idx"][:1]])
    o3 = M.msa_forward_cached_varlen(q, q_idx, k3, v3, ki3, t0, n, shape.top_k)
    torch.cuda.synchronize()
    assert torch.equal(o3, want_o)
    # an empty sequence first, then the others
    o4 = M.msa_forward_cached_varlen(q, q_idx, torch.cat([k3[2:], cache["k"]]),
                                     torch.cat([v3[2:], cache["v"]]),
                                     torch.cat([ki3[2:], cache["k_idx"]]), [0] + t0[:B],
                                     [0] + n[:B], shape.top_k)
    torch.cuda.synchronize()
    assert torch.equal(o4, want_o)
