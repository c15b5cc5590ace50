"""GPU tests of the query-chunk knob and of msa_forward_host (inputs and
outputs in host memory, transfers overlapped with the computation).

Rows are computed independently of which queries share a work item or a
query chunk, so chunked runs and the host-buffer path must reproduce the
device path bit for bit; the device path itself is checked against the
oracle in test_gpu_parity.py and test_gpu_fullsize.py.
"""
import pytest
import torch

from block_sparse_long_08_b200 import inputs as I
from block_sparse_long_08_b200 import msa as M

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _inputs(shape, seed):
    return I.prefill_inputs(shape, seed, device=DEV)


@pytest.mark.parametrize("L", [4096, 3000])
def test_chunked_prefill_is_bit_identical(L):
    """Chunks are ranges of the packed query rows b*L + t, so with B = 2 some
    chunks span the end of one sequence and the start of the next."""
    shape = I.PrefillShape(B=2, L=L, H=16, G=4, d=128, d_idx=128, top_k=8)
    x = _inputs(shape, 31)
    sel = M.msa_index_select(x["q_idx"], x["k_idx"], shape.top_k)
    o_ref, l_ref = M.msa_sparse_attn_prefill(x["q"], x["k"], x["v"], sel, want_lse=True)
    for chunk in (128, 1024, 1536):
        o, l = M.msa_sparse_attn_prefill(x["q"], x["k"], x["v"], sel, want_lse=True, chunk=chunk)
        torch.cuda.synchronize()
        assert torch.equal(o, o_ref), chunk
        assert torch.equal(l, l_ref), chunk


@pytest.mark.parametrize("L", [4096, 2049])
def test_forward_host_matches_device_forward(L):
    shape = I.PrefillShape(B=2, L=L, H=32, G=8, d=128, d_idx=128, top_k=16)
    x = _inputs(shape, 32)
    o_ref, l_ref = M.msa_forward(x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"], shape.top_k,
                                 want_lse=True)
    torch.cuda.synchronize()
    host = {n: x[n].cpu().pin_memory() for n in ("q", "k", "v", "q_idx", "k_idx")}
    out_h = torch.empty(x["q"].shape, dtype=torch.bfloat16).pin_memory()
    lse_h = torch.empty(l_ref.shape, dtype=torch.float32).pin_memory()
    stream = torch.cuda.current_stream()
    copy_stream = torch.cuda.Stream()
    staging = None
    for rep in range(2):   # the second call reuses the staging buffers and events
        out_h.fill_(0)
        lse_h.fill_(0)
        if staging is None:
            staging = {n: torch.empty_like(x[n]) for n in ("q", "k", "v", "q_idx", "k_idx")}
            staging["out"] = torch.empty_like(x["q"])
            staging["lse"] = torch.empty_like(l_ref)
        M.msa_forward_host(host["q"], host["k"], host["v"], host["q_idx"], host["k_idx"],
                           shape.top_k, out=out_h, lse=lse_h, staging=staging, stream=stream,
                           copy_stream=copy_stream, chunk=1024)   # 4 chunks per sequence
        stream.synchronize()
        assert torch.equal(out_h, o_ref.cpu()), rep
        assert torch.equal(lse_h, l_ref.cpu()), rep


def test_forward_host_same_stream_and_no_lse():
    shape = I.PrefillShape(B=1, L=2048, H=8, G=2, d=128, d_idx=64, top_k=4)
    x = _inputs(shape, 33)
    o_ref = M.msa_forward(x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"], shape.top_k)
    torch.cuda.synchronize()
    host = {n: x[n].cpu() for n in ("q", "k", "v", "q_idx", "k_idx")}   # pageable
    out_h = torch.empty(x["q"].shape, dtype=torch.bfloat16)
    s = torch.cuda.current_stream()
    M.msa_forward_host(host["q"], host["k"], host["v"], host["q_idx"], host["k_idx"], shape.top_k,
                       out=out_h, stream=s, copy_stream=s)
    s.synchronize()
    assert torch.equal(out_h, o_ref.cpu())
