"""The decode entry point that allocates nothing (msa_sparse_attn_decode_noalloc).

Callers that cannot allocate device memory where they run a decode step --
engines whose device buffers are all planned at start-up, plugin hosts that
hand the library only the call's tensors -- use this variant; it keeps its
scratch in a 16 MiB device array owned by the library.  These tests call it
through the C ABI twice in a row, on two different problems, and check each
result against the regular workspace-taking entry point within the parity
tolerances the other GPU tests use; the second call shows that the first
call's leftovers in the shared scratch do not leak into the next result.
The file is named to be collected last.
"""
import ctypes
import os
import subprocess
import sys

import pytest
import torch

from block_sparse_long_08_b200 import inputs as I
from block_sparse_long_08_b200 import msa as M

pytestmark = pytest.mark.gpu
DEV = "cuda"
OUT_MAX_ABS = 2e-2
OUT_MEAN_ABS = 2e-3


def _problem(B, Lmax, G, H, di, top_k, lens, seed):
    shape = I.DecodeShape(B=B, Lmax=Lmax, H=H, G=G, d=128, d_idx=di, top_k=top_k)
    x = I.decode_inputs(shape, seed)
    d = {n: x[n].to(DEV) for n in ("q", "q_idx", "k_cache", "v_cache", "k_idx_cache")}
    d["seq_lens"] = torch.tensor(lens, dtype=torch.int32, device=DEV)
    return d


def _both(d, top_k):
    ref, ref_sel = M.msa_sparse_attn_decode(d["q"], d["q_idx"], d["k_cache"], d["v_cache"],
                                            d["k_idx_cache"], d["seq_lens"], top_k, want_sel=True)
    got, got_sel = M.msa_sparse_attn_decode_noalloc(d["q"], d["q_idx"], d["k_cache"], d["v_cache"],
                                                    d["k_idx_cache"], d["seq_lens"], top_k,
                                                    want_sel=True)
    torch.cuda.synchronize()
    return ref, ref_sel, got, got_sel


def test_noalloc_decode_matches_workspace_decode_twice():
    problems = [
        (_problem(6, 8192, 8, 32, 128, 16, [8192, 1, 300, 4097, 8000, 129], seed=101), 16),
        (_problem(3, 4096, 2, 8, 64, 4, [4096, 2000, 128], seed=102), 4),
    ]
    for d, top_k in problems:   # two calls in a row on the shared scratch
        ref, ref_sel, got, got_sel = _both(d, top_k)
        err = (got.float() - ref.float()).abs()
        assert err.max().item() <= OUT_MAX_ABS and err.mean().item() <= OUT_MEAN_ABS
        assert torch.equal(got_sel, ref_sel)


def test_noalloc_rejects_problems_beyond_its_scratch():
    # 32 sequences at 1M tokens need ~16.3 MB of decode scratch > 16 MiB.
    p = M.make_params(32, 1048576, 32, 8, 128, 128, 128, 16)
    assert M.msa_workspace_bytes(p, M.MSA_OP_DECODE) > (16 << 20)
    fake = ctypes.c_void_p(1 << 20)   # never dereferenced: the size check comes first
    rc = M.lib().msa_sparse_attn_decode_noalloc(ctypes.byref(p), fake, fake, fake, fake, fake, fake,
                                                fake, None, None)
    assert rc == M.MSA_ERR_WORKSPACE
    assert "no-allocation" in M.msa_last_error()


def test_noalloc_without_sel_and_with_a_bad_length():
    """sel = NULL (the selection then lives in the shared scratch) and a
    length above Lmax: that sequence's output is zero, the others match the
    workspace entry point (which also reports the bad length on the device)."""
    d = _problem(4, 4096, 2, 8, 64, 4, [4096, 5000, 300, 1], seed=103)
    ws = M.new_workspace(M.make_params(4, 4096, 8, 2, 128, 64, 128, 4), M.MSA_OP_DECODE, DEV)
    ref = M.msa_sparse_attn_decode(d["q"], d["q_idx"], d["k_cache"], d["v_cache"], d["k_idx_cache"],
                                   d["seq_lens"], 4, ws=ws)
    assert M.msa_read_status(ws) == M.MSA_ERR_DEVICE_INPUT
    for _ in range(2):
        got = M.msa_sparse_attn_decode_noalloc(d["q"], d["q_idx"], d["k_cache"], d["v_cache"],
                                               d["k_idx_cache"], d["seq_lens"], 4)
        torch.cuda.synchronize()
        assert torch.count_nonzero(got[1]).item() == 0
        err = (got.float() - ref.float()).abs()
        assert err.max().item() <= OUT_MAX_ABS and err.mean().item() <= OUT_MEAN_ABS


def test_noalloc_across_device_reset():
    """A reset rebuilds the context and may move the scratch array; the
    entry point must look its address up again (run in a child process
    without torch, see _noalloc_reset_child.py)."""
    child = os.path.join(os.path.dirname(os.path.abspath(__file__)), "_noalloc_reset_child.py")
    r = subprocess.run([sys.executable, child], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "ok" in r.stdout
