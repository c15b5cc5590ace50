"""Group-sharded deployment on one GPU: every stage of the path is per GQA
group, with k_idx shared by all groups ("MiniMax M3 sparse attention"
explainer, §2.1: one index query per group against one shared index key;
§2.2: the heads of a group share its selection).  A GPU that holds groups
[g0, g1) -- their q heads, q_idx columns, K/V heads -- plus a replica of
k_idx therefore computes exactly those groups' rows with no exchange.  Here
the two halves run as two calls on contiguous copies of their slices, and
their concatenation must equal the whole call bit for bit."""
import pytest
import torch

from block_sparse_long_08_b200 import inputs as I
from block_sparse_long_08_b200 import msa as M

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _half(t: torch.Tensor, dim: int, n: int, part: int) -> torch.Tensor:
    w = t.shape[dim] // n
    return t.narrow(dim, part * w, w).contiguous()


@pytest.mark.parametrize("L,H,G,di,top_k", [(4096, 16, 4, 128, 5), (2048, 32, 8, 64, 4)])
def test_prefill_group_halves_equal_whole(L, H, G, di, top_k):
    x = I.prefill_inputs(I.PrefillShape(B=2, L=L, H=H, G=G, d=128, d_idx=di), 31)
    x = {n: x[n].to(DEV) for n in ("q", "k", "v", "q_idx", "k_idx")}
    out, sel, lse = M.msa_forward(x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"], top_k,
                                  want_sel=True, want_lse=True)
    parts = []
    for part in range(2):
        parts.append(M.msa_forward(_half(x["q"], 2, 2, part), _half(x["k"], 2, 2, part),
                                   _half(x["v"], 2, 2, part), _half(x["q_idx"], 2, 2, part),
                                   x["k_idx"], top_k, want_sel=True, want_lse=True))
    torch.cuda.synchronize()
    assert torch.equal(torch.cat([p[0] for p in parts], dim=2), out)
    assert torch.equal(torch.cat([p[1] for p in parts], dim=1), sel)
    assert torch.equal(torch.cat([p[2] for p in parts], dim=2), lse)


def test_decode_group_halves_equal_whole():
    ds = I.DecodeShape(B=5, Lmax=8192, H=32, G=8, d=128, d_idx=128, top_k=16)
    y = I.decode_inputs(ds, 32)
    y = {n: y[n].to(DEV) for n in ("q", "q_idx", "k_cache", "v_cache", "k_idx_cache")}
    lens = torch.tensor([8192, 1, 3000, 129, 7777], dtype=torch.int32, device=DEV)
    out, sel = M.msa_sparse_attn_decode(y["q"], y["q_idx"], y["k_cache"], y["v_cache"],
                                        y["k_idx_cache"], lens, 16, want_sel=True)
    parts = []
    for part in range(2):
        parts.append(M.msa_sparse_attn_decode(
            _half(y["q"], 1, 2, part), _half(y["q_idx"], 1, 2, part),
            _half(y["k_cache"], 2, 2, part), _half(y["v_cache"], 2, 2, part), y["k_idx_cache"],
            lens, 16, want_sel=True))
    torch.cuda.synchronize()
    assert torch.equal(torch.cat([p[0] for p in parts], dim=1), out)
    assert torch.equal(torch.cat([p[1] for p in parts], dim=1), sel)
