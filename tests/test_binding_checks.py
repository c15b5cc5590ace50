"""Host-side argument checks of the Python binding (no GPU).

Every binding function validates the buffers it hands to the C ABI against
the element counts the call reads or writes, derived from the same
parameters it passes, so a short caller buffer raises ValueError instead of
reaching a kernel.  These tests run the binding with the library replaced by
a stub that records calls, and CPU tensors standing in for device tensors:
correctly sized arguments of each entry point reach the stub, and one short
buffer per entry point is refused before any library call.
"""
import ctypes

import pytest
import torch

from block_sparse_long_08_b200 import inputs as I
from block_sparse_long_08_b200 import msa as M

BF16 = torch.bfloat16


class _StubLib:
    def __init__(self):
        self.calls = []

    def msa_workspace_bytes(self, p, op):
        return 64

    def msa_last_error(self):
        return b"stub"

    def __getattr__(self, name):
        def fn(*args):
            self.calls.append(name)
            return M.MSA_OK
        return fn


@pytest.fixture
def stub(monkeypatch):
    lib = _StubLib()

    def req_any_device(t, name, dtype):   # the binding's checks minus "is CUDA"
        if not isinstance(t, torch.Tensor):
            raise ValueError(f"{name} must be a tensor")
        if t.dtype != dtype:
            raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        return t

    monkeypatch.setattr(M, "lib", lambda: lib)
    monkeypatch.setattr(M, "_req", req_any_device)
    monkeypatch.setattr(M, "_stream", lambda s=None: ctypes.c_void_p(0))
    return lib


def _short(t):
    """The same tensor one leading row short (a buffer too small by a row)."""
    return t[:-1].contiguous() if t.shape[0] > 1 else t.reshape(-1)[:-1].contiguous()


PF = I.PrefillShape(B=2, L=300, H=8, G=2, d=128, d_idx=64, top_k=4)


@pytest.fixture
def pre():
    x = I.prefill_inputs(PF, 5)
    x["sel"] = torch.zeros((PF.B, PF.G, PF.L, PF.top_k), dtype=torch.int32)
    x["out"] = torch.empty_like(x["q"])
    x["lse"] = torch.empty((PF.B, PF.L, PF.H), dtype=torch.float32)
    x["dout"] = torch.empty_like(x["q"])
    return x


def _refused(lib, fn, *args, match="the call needs", **kw):
    n = len(lib.calls)
    with pytest.raises(ValueError, match=match):
        fn(*args, **kw)
    assert len(lib.calls) == n, "a refused call must not reach the library"


def test_index_select(stub, pre):
    for blk in (64, 128):
        M.msa_index_select(pre["q_idx"], pre["k_idx"], PF.top_k, sel=pre["sel"], block=blk)
    assert stub.calls == ["msa_index_select"] * 2
    _refused(stub, M.msa_index_select, pre["q_idx"], _short(pre["k_idx"]), PF.top_k)
    _refused(stub, M.msa_index_select, pre["q_idx"], pre["k_idx"], PF.top_k,
             sel=pre["sel"][:, :, :-1].contiguous())
    _refused(stub, M.msa_index_select, pre["q_idx"], pre["k_idx"], PF.top_k,
             sel=pre["sel"].to(torch.int64), match="must be torch.int32")


def test_prefill_and_backward(stub, pre):
    x = pre
    M.msa_sparse_attn_prefill(x["q"], x["k"], x["v"], x["sel"], out=x["out"], want_lse=True,
                              chunk=128, block=64)
    M.msa_sparse_attn_backward(x["q"], x["k"], x["v"], x["out"], x["lse"], x["dout"], x["sel"])
    assert stub.calls == ["msa_sparse_attn_prefill", "msa_sparse_attn_backward"]
    _refused(stub, M.msa_sparse_attn_prefill, x["q"], _short(x["k"]), x["v"], x["sel"])
    _refused(stub, M.msa_sparse_attn_prefill, x["q"], x["k"], x["v"], x["sel"], out=_short(x["out"]))
    _refused(stub, M.msa_sparse_attn_backward, x["q"], x["k"], x["v"], x["out"], _short(x["lse"]),
             x["dout"], x["sel"])
    _refused(stub, M.msa_sparse_attn_backward, x["q"], x["k"], x["v"], x["out"], x["lse"],
             x["dout"], x["sel"], dk=_short(torch.empty_like(x["k"])))
    _refused(stub, M.msa_sparse_attn_backward, x["q"], x["k"], x["v"], x["out"], x["lse"],
             _short(x["dout"]), x["sel"])


def test_forward_and_nsa(stub, pre):
    x = pre
    args = (x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"])
    M.msa_forward(*args, PF.top_k, want_sel=True, want_lse=True)
    M.msa_forward(*args, PF.top_k, out=x["out"], sel=x["sel"])
    gates = torch.rand((PF.B, PF.L, PF.H, 3))
    M.msa_nsa_forward(*args, gates, PF.top_k, 64, want_sel=True)
    kc, vc = M.msa_nsa_compress_kv(x["k"], x["v"], block=64)
    assert kc.shape == (PF.B, 5, PF.G, PF.d)
    M.msa_nsa_window_attn(x["q"], x["k"], x["v"], 64, want_lse=True)
    M.msa_nsa_compressed_attn(x["q"], kc, vc, block=64, out=x["out"])
    M.msa_nsa_gate(gates, x["out"], x["q"], x["dout"], out=x["out"])   # out may alias an input
    assert stub.calls == ["msa_forward", "msa_forward", "msa_nsa_forward", "msa_nsa_compress_kv",
                          "msa_nsa_window_attn", "msa_nsa_compressed_attn", "msa_nsa_gate"]
    _refused(stub, M.msa_forward, x["q"], x["k"], x["v"], _short(x["q_idx"]), x["k_idx"], PF.top_k)
    _refused(stub, M.msa_forward, *args, PF.top_k, sel=_short(x["sel"]))
    _refused(stub, M.msa_nsa_forward, *args, _short(gates), PF.top_k, 64)
    _refused(stub, M.msa_nsa_compress_kv, x["k"], _short(x["v"]))
    _refused(stub, M.msa_nsa_compress_kv, x["k"], x["v"], k_cmp=_short(kc))
    _refused(stub, M.msa_nsa_window_attn, x["q"], x["k"], _short(x["v"]), 64)
    _refused(stub, M.msa_nsa_compressed_attn, x["q"], kc, _short(vc), block=64)
    _refused(stub, M.msa_nsa_gate, gates, x["out"], _short(x["q"]), x["dout"])


def test_cached_and_ragged(stub):
    sh = I.DecodeShape(B=3, Lmax=1000, H=8, G=2, d=128, d_idx=64, top_k=4)
    y = I.decode_inputs(sh, 6)
    n = 37
    q = torch.zeros((sh.B, n, sh.H, sh.d), dtype=BF16)
    q_idx = torch.zeros((sh.B, n, sh.G, sh.d_idx), dtype=BF16)
    caches = (y["k_cache"], y["v_cache"], y["k_idx_cache"])
    M.msa_forward_cached(q, q_idx, *caches, 500, sh.top_k, want_sel=True, want_lse=True)
    ns = [5, 0, 40]
    qv = torch.zeros((sum(ns), sh.H, sh.d), dtype=BF16)
    qiv = torch.zeros((sum(ns), sh.G, sh.d_idx), dtype=BF16)
    M.msa_forward_cached_varlen(qv, qiv, *caches, [0, 10, 900], ns, sh.top_k, want_lse=True)
    assert stub.calls == ["msa_forward_cached", "msa_forward_cached_varlen"]
    _refused(stub, M.msa_forward_cached, q, _short(q_idx), *caches, 500, sh.top_k)
    _refused(stub, M.msa_forward_cached, q, q_idx, y["k_cache"], _short(y["v_cache"]),
             y["k_idx_cache"], 500, sh.top_k)
    _refused(stub, M.msa_forward_cached, q, q_idx, *caches, 500, sh.top_k,
             sel=torch.zeros((sh.B, sh.G, n - 1, sh.top_k), dtype=torch.int32))
    _refused(stub, M.msa_forward_cached_varlen, qv, _short(qiv), *caches, [0, 10, 900], ns,
             sh.top_k)
    _refused(stub, M.msa_forward_cached_varlen, qv, qiv, *caches, [0, 10], ns, sh.top_k,
             match="one entry per cached sequence")
    _refused(stub, M.msa_forward_cached_varlen, qv, qiv, *caches, [0, 10, 900], ns, sh.top_k,
             out=_short(torch.empty_like(qv)))


def test_host_forward(stub, pre):
    x = pre
    names = ("q", "k", "v", "q_idx", "k_idx")
    staging = {n: torch.empty_like(x[n]) for n in names}
    staging["out"] = torch.empty_like(x["q"])
    staging["lse"] = torch.empty_like(x["lse"])
    out_h = torch.empty_like(x["q"])
    args = tuple(x[n] for n in names)
    M.msa_forward_host(*args, PF.top_k, out=out_h, lse=x["lse"], staging=staging,
                       copy_stream=object(), device="cpu")
    assert stub.calls == ["msa_forward_host"]
    _refused(stub, M.msa_forward_host, *args, PF.top_k, out=_short(out_h), staging=staging,
             copy_stream=object(), device="cpu")
    bad = dict(staging, k=_short(staging["k"]))
    _refused(stub, M.msa_forward_host, *args, PF.top_k, out=out_h, staging=bad,
             copy_stream=object(), device="cpu")
    bad = dict(staging, lse=_short(staging["lse"]))
    _refused(stub, M.msa_forward_host, *args, PF.top_k, out=out_h, lse=x["lse"], staging=bad,
             copy_stream=object(), device="cpu")


def test_decode_variants(stub):
    sh = I.DecodeShape(B=3, Lmax=700, H=8, G=2, d=128, d_idx=64, top_k=4)
    y = I.decode_inputs(sh, 7)
    seq = y["seq_lens"]
    bf = (y["q"], y["q_idx"], y["k_cache"], y["v_cache"], y["k_idx_cache"])
    codes, kscale = I.fp8_index_cache(y["k_idx_cache"])
    k8, ks8 = I.fp8_rows(y["k_cache"])
    v8, vs8 = I.fp8_rows(y["v_cache"])
    M.msa_sparse_attn_decode(*bf, seq, sh.top_k, want_sel=True, block=64)
    M.msa_sparse_attn_decode_noalloc(*bf, seq, sh.top_k, want_sel=True)
    M.msa_sparse_attn_decode_fp8idx(y["q"], y["q_idx"], y["k_cache"], y["v_cache"], codes, kscale,
                                    seq, sh.top_k, want_sel=True)
    M.msa_sparse_attn_decode_fp8(y["q"], y["q_idx"], k8, ks8, v8, vs8, codes, kscale, seq,
                                 sh.top_k, want_sel=True)
    c, s = M.msa_quantize_e4m3_rows(y["k_idx_cache"])
    assert c.shape == y["k_idx_cache"].shape and s.shape == y["k_idx_cache"].shape[:2]
    assert stub.calls == ["msa_sparse_attn_decode", "msa_sparse_attn_decode_noalloc",
                          "msa_sparse_attn_decode_fp8idx", "msa_sparse_attn_decode_fp8",
                          "msa_quantize_e4m3_rows"]
    _refused(stub, M.msa_sparse_attn_decode, y["q"], y["q_idx"], y["k_cache"], _short(y["v_cache"]),
             y["k_idx_cache"], seq, sh.top_k)
    _refused(stub, M.msa_sparse_attn_decode, *bf, seq[:-1].contiguous(), sh.top_k)
    _refused(stub, M.msa_sparse_attn_decode, *bf, seq, sh.top_k,
             sel=torch.zeros((sh.B, sh.G, sh.top_k - 1), dtype=torch.int32))
    _refused(stub, M.msa_sparse_attn_decode_noalloc, y["q"], _short(y["q_idx"]), y["k_cache"],
             y["v_cache"], y["k_idx_cache"], seq, sh.top_k)
    _refused(stub, M.msa_sparse_attn_decode_fp8idx, y["q"], y["q_idx"], y["k_cache"],
             y["v_cache"], codes, _short(kscale), seq, sh.top_k)
    _refused(stub, M.msa_sparse_attn_decode_fp8, y["q"], y["q_idx"], k8, _short(ks8), v8, vs8,
             codes, kscale, seq, sh.top_k)
    _refused(stub, M.msa_sparse_attn_decode_fp8, y["q"], y["q_idx"], k8, ks8, _short(v8), vs8,
             codes, kscale, seq, sh.top_k, out=torch.empty_like(y["q"]))
    _refused(stub, M.msa_quantize_e4m3_rows, y["k_idx_cache"], scale=_short(s))


def test_workspace_must_be_bytes(stub, pre):
    x = pre
    with pytest.raises(ValueError, match="ws must be torch.uint8"):
        M.msa_sparse_attn_prefill(x["q"], x["k"], x["v"], x["sel"],
                                  ws=torch.zeros(64, dtype=torch.int32))
    with pytest.raises(M.MSAError):
        M.msa_sparse_attn_prefill(x["q"], x["k"], x["v"], x["sel"],
                                  ws=torch.zeros(63, dtype=torch.uint8))
    assert stub.calls == []
