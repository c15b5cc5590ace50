"""Python binding of libmsa.so (ctypes).  Argument marshalling only: every
step of the computation runs in the library's CUDA kernels; PyTorch supplies
device memory and the current stream.

The functions carry the C names (msa_index_select, msa_sparse_attn_prefill,
msa_sparse_attn_decode, msa_forward, msa_workspace_bytes, msa_read_status,
msa_last_error).  Tensors must be CUDA, contiguous, bf16 (int32 for
selections and lengths).  Outputs are allocated here unless passed in.
Every tensor handed to the library, passed in or allocated, is checked
against the number of elements the call reads or writes (derived from the
same parameters the call receives), so a short buffer raises ValueError
here instead of being read or written past its end on the device.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmsa.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "msa.h")

MSA_OK = 0
MSA_ERR_INVALID_ARG = -1
MSA_ERR_UNSUPPORTED = -2
MSA_ERR_WORKSPACE = -3
MSA_ERR_CUDA = -4
MSA_ERR_DEVICE_TIMEOUT = -5
MSA_ERR_DEVICE_INPUT = -6

MSA_OP_INDEX_SELECT = 0
MSA_OP_PREFILL_ATTN = 1
MSA_OP_DECODE = 2
MSA_OP_FORWARD = 3
MSA_OP_BACKWARD = 4
MSA_OP_FORWARD_VARLEN = 5
MSA_OP_NSA_BRANCH = 6
MSA_OP_NSA_FORWARD = 7


class MSAError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"msa error {code}: {msg}")
        self.code = code


class msa_params(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("L", ctypes.c_int32), ("H", ctypes.c_int32),
                ("G", ctypes.c_int32), ("d", ctypes.c_int32), ("d_idx", ctypes.c_int32),
                ("block", ctypes.c_int32), ("top_k", ctypes.c_int32), ("scale", ctypes.c_float),
                ("chunk", ctypes.c_int32)]


class msa_staging(ctypes.Structure):
    _fields_ = [("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
                ("q_idx", ctypes.c_void_p), ("k_idx", ctypes.c_void_p), ("out", ctypes.c_void_p),
                ("lse", ctypes.c_void_p)]


_lib = None
_P = ctypes.c_void_p
_SZ = ctypes.c_size_t


def lib() -> ctypes.CDLL:
    """Load libmsa.so (built in-tree by block_sparse_long_08_b200.build)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: run `python -m block_sparse_long_08_b200.build`")
        torch.cuda.is_available()  # make sure torch's CUDA runtime is loaded first
        L = ctypes.CDLL(LIB_PATH)
        pp = ctypes.POINTER(msa_params)
        L.msa_index_select.argtypes = [pp, _P, _P, _P, _P, _P, _SZ, _P]
        L.msa_sparse_attn_prefill.argtypes = [pp, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]
        L.msa_sparse_attn_decode.argtypes = [pp, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]
        L.msa_forward.argtypes = [pp, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]
        L.msa_forward_cached.argtypes = [pp, ctypes.c_int, ctypes.c_int, _P, _P, _P, _P, _P, _P, _P,
                                         _P, _P, _SZ, _P]
        L.msa_forward_cached_varlen.argtypes = [pp, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ,
                                                _P]
        L.msa_forward_host.argtypes = [pp, _P, _P, _P, _P, _P, _P, _P,
                                       ctypes.POINTER(msa_staging), _P, _SZ, _P, _P]
        L.msa_sparse_attn_decode_noalloc.argtypes = [pp, _P, _P, _P, _P, _P, _P, _P, _P, _P]
        L.msa_sparse_attn_decode_fp8idx.argtypes = [pp, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ,
                                                    _P]
        L.msa_quantize_e4m3_rows.argtypes = [_P, ctypes.c_longlong, ctypes.c_int, _P, _P, _P]
        L.msa_sparse_attn_decode_fp8.argtypes = [pp, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                                 _P, _SZ, _P]
        L.msa_sparse_attn_decode_noalloc.restype = ctypes.c_int
        L.msa_sparse_attn_backward.argtypes = [pp, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                               _SZ, _P]
        L.msa_nsa_compress_kv.argtypes = [pp, _P, _P, _P, _P, _P]
        L.msa_nsa_window_attn.argtypes = [pp, ctypes.c_int32, _P, _P, _P, _P, _P, _P, _SZ, _P]
        L.msa_nsa_compressed_attn.argtypes = [pp, _P, _P, _P, _P, _P, _P, _SZ, _P]
        L.msa_nsa_gate.argtypes = [pp, _P, _P, _P, _P, _P, _P]
        L.msa_nsa_forward.argtypes = [pp, ctypes.c_int32, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ,
                                      _P]
        L.msa_workspace_bytes.argtypes = [pp, ctypes.c_int]
        L.msa_workspace_bytes.restype = _SZ
        L.msa_read_status.argtypes = [_P, _P]
        L.msa_prefill_chunk_len.argtypes = [pp]
        L.msa_prefill_chunk_len.restype = ctypes.c_int
        L.msa_last_error.restype = ctypes.c_char_p
        L.msa_version.restype = ctypes.c_char_p
        for f in ("msa_index_select", "msa_sparse_attn_prefill", "msa_sparse_attn_decode",
                  "msa_forward", "msa_forward_host", "msa_forward_cached", "msa_read_status",
                  "msa_sparse_attn_decode_fp8idx", "msa_quantize_e4m3_rows",
                  "msa_sparse_attn_decode_fp8", "msa_forward_cached_varlen",
                  "msa_sparse_attn_backward", "msa_nsa_compress_kv", "msa_nsa_window_attn",
                  "msa_nsa_compressed_attn", "msa_nsa_gate", "msa_nsa_forward"):
            getattr(L, f).restype = ctypes.c_int
        _lib = L
    return _lib


def header_functions() -> list[str]:
    """Entry points declared in include/msa.h."""
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(msa_\w+)\s*\(", txt, re.M)))


def msa_last_error() -> str:
    return lib().msa_last_error().decode()


def _check(rc: int):
    if rc != MSA_OK:
        raise MSAError(rc, msa_last_error())


def make_params(B, L, H, G, d=128, d_idx=128, block=128, top_k=16, scale=0.0,
                chunk=0) -> msa_params:
    return msa_params(int(B), int(L), int(H), int(G), int(d), int(d_idx), int(block), int(top_k),
                      float(scale), int(chunk))


def msa_workspace_bytes(p: msa_params, op: int) -> int:
    n = lib().msa_workspace_bytes(ctypes.byref(p), op)
    if n == 0:
        raise MSAError(MSA_ERR_INVALID_ARG, msa_last_error())
    return int(n)


def msa_prefill_chunk_len(p: msa_params) -> int:
    return int(lib().msa_prefill_chunk_len(ctypes.byref(p)))


def new_workspace(p: msa_params, op: int, device) -> torch.Tensor:
    """Zeroed workspace (the status word must start at zero)."""
    return torch.zeros(msa_workspace_bytes(p, op), dtype=torch.uint8, device=device)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _req(t: torch.Tensor, name: str, dtype) -> torch.Tensor:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _size(t: torch.Tensor, name: str, dtype, numel: int) -> torch.Tensor:
    """_req plus the element count the call reads or writes: a short buffer
    is an error here rather than an access past its end on the device."""
    _req(t, name, dtype)
    if t.numel() < numel:
        raise ValueError(f"{name} has {t.numel()} elements, the call needs {numel}")
    return t


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _ensure_ws(ws, p, op, device):
    need = msa_workspace_bytes(p, op)
    if ws is None:
        return torch.zeros(need, dtype=torch.uint8, device=device)
    _req(ws, "ws", torch.uint8)
    if ws.numel() < need:
        raise MSAError(MSA_ERR_WORKSPACE, f"workspace has {ws.numel()} bytes, need {need}")
    return ws


def msa_index_select(q_idx: torch.Tensor, k_idx: torch.Tensor, top_k: int, *,
                     block_scores: bool = False, sel: Optional[torch.Tensor] = None,
                     ws: Optional[torch.Tensor] = None, stream=None, block: int = 128):
    """q_idx [B,L,G,d_idx], k_idx [B,L,d_idx] -> sel [B,G,L,top_k] int32
    (and block scores [B,G,L,nb] fp32 when block_scores=True)."""
    _req(q_idx, "q_idx", torch.bfloat16)
    _req(k_idx, "k_idx", torch.bfloat16)
    B, L, G, di = q_idx.shape
    _size(k_idx, "k_idx", torch.bfloat16, B * L * di)
    p = make_params(B, L, G, G, 128, di, block, top_k)
    dev = q_idx.device
    if sel is None:
        sel = torch.empty((B, G, L, top_k), dtype=torch.int32, device=dev)
    _size(sel, "sel", torch.int32, B * G * L * top_k)
    scores = torch.empty((B, G, L, (L + block - 1) // block), dtype=torch.float32,
                         device=dev) if block_scores else None
    ws = _ensure_ws(ws, p, MSA_OP_INDEX_SELECT, dev)
    _check(lib().msa_index_select(ctypes.byref(p), _ptr(q_idx), _ptr(k_idx), _ptr(sel), _ptr(scores),
                                  _ptr(ws), ws.numel(), _stream(stream)))
    return (sel, scores) if block_scores else sel


def msa_sparse_attn_prefill(q, k, v, sel, *, scale: float = 0.0, want_lse: bool = False,
                            out=None, ws=None, stream=None, chunk: int = 0, block: int = 128):
    """q [B,L,H,d], k/v [B,L,G,d] bf16, sel [B,G,L,top_k] int32 -> out [B,L,H,d]
    (and lse [B,L,H] fp32 when want_lse)."""
    for n, t in (("q", q), ("k", k), ("v", v)):
        _req(t, n, torch.bfloat16)
    _req(sel, "sel", torch.int32)
    B, L, H, d = q.shape
    G = k.shape[2]
    top_k = sel.shape[3]
    for n, t in (("k", k), ("v", v)):
        _size(t, n, torch.bfloat16, B * L * G * d)
    _size(sel, "sel", torch.int32, B * G * L * top_k)
    p = make_params(B, L, H, G, d, 128, block, top_k, scale, chunk)
    dev = q.device
    if out is None:
        out = torch.empty_like(q)
    _size(out, "out", torch.bfloat16, B * L * H * d)
    lse = torch.empty((B, L, H), dtype=torch.float32, device=dev) if want_lse else None
    ws = _ensure_ws(ws, p, MSA_OP_PREFILL_ATTN, dev)
    _check(lib().msa_sparse_attn_prefill(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(sel),
                                         _ptr(out), _ptr(lse), _ptr(ws), ws.numel(), _stream(stream)))
    return (out, lse) if want_lse else out


def msa_sparse_attn_backward(q, k, v, out, lse, dout, sel, *, scale: float = 0.0, dq=None,
                             dk=None, dv=None, ws=None, stream=None, chunk: int = 0,
                             block: int = 128):
    """Main-branch gradients for a fixed selection: q [B,L,H,d], k/v
    [B,L,G,d], the forward's out [B,L,H,d] and lse [B,L,H] fp32, dout
    [B,L,H,d], sel [B,G,L,top_k] (block ids of `block` tokens) -> (dq, dk,
    dv) bf16, shaped like q, k, v."""
    for n, t in (("q", q), ("k", k), ("v", v), ("out", out), ("dout", dout)):
        _req(t, n, torch.bfloat16)
    _req(lse, "lse", torch.float32)
    _req(sel, "sel", torch.int32)
    B, L, H, d = q.shape
    G = k.shape[2]
    top_k = sel.shape[3]
    p = make_params(B, L, H, G, d, 128, block, top_k, scale, chunk)
    dev = q.device
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    for n, t in (("k", k), ("v", v), ("dk", dk), ("dv", dv)):
        _size(t, n, torch.bfloat16, B * L * G * d)
    for n, t in (("out", out), ("dout", dout), ("dq", dq)):
        _size(t, n, torch.bfloat16, B * L * H * d)
    _size(lse, "lse", torch.float32, B * L * H)
    _size(sel, "sel", torch.int32, B * G * L * top_k)
    ws = _ensure_ws(ws, p, MSA_OP_BACKWARD, dev)
    _check(lib().msa_sparse_attn_backward(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(out),
                                          _ptr(lse), _ptr(dout), _ptr(sel), _ptr(dq), _ptr(dk),
                                          _ptr(dv), _ptr(ws), ws.numel(), _stream(stream)))
    return dq, dk, dv


def msa_forward(q, k, v, q_idx, k_idx, top_k: int, *, scale: float = 0.0, want_sel: bool = False,
                want_lse: bool = False, out=None, sel=None, ws=None, stream=None, chunk: int = 0, block: int = 128):
    """Whole prefill: index branch with fused top-k, then the sparse main branch."""
    for n, t in (("q", q), ("k", k), ("v", v), ("q_idx", q_idx), ("k_idx", k_idx)):
        _req(t, n, torch.bfloat16)
    B, L, H, d = q.shape
    G = k.shape[2]
    di = q_idx.shape[3]
    _check_prefill_inputs(B, L, G, d, di, k, v, q_idx, k_idx)
    p = make_params(B, L, H, G, d, di, block, top_k, scale, chunk)
    dev = q.device
    if out is None:
        out = torch.empty_like(q)
    _size(out, "out", torch.bfloat16, B * L * H * d)
    if sel is None and want_sel:
        sel = torch.empty((B, G, L, top_k), dtype=torch.int32, device=dev)
    if sel is not None:
        _size(sel, "sel", torch.int32, B * G * L * top_k)
    lse = torch.empty((B, L, H), dtype=torch.float32, device=dev) if want_lse else None
    ws = _ensure_ws(ws, p, MSA_OP_FORWARD, dev)
    _check(lib().msa_forward(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(q_idx), _ptr(k_idx),
                             _ptr(out), _ptr(sel), _ptr(lse), _ptr(ws), ws.numel(), _stream(stream)))
    res = [out]
    if want_sel:
        res.append(sel)
    if want_lse:
        res.append(lse)
    return res[0] if len(res) == 1 else tuple(res)


def _check_prefill_inputs(B, L, G, d, di, k, v, q_idx, k_idx):
    for n, t in (("k", k), ("v", v)):
        _size(t, n, torch.bfloat16, B * L * G * d)
    _size(q_idx, "q_idx", torch.bfloat16, B * L * G * di)
    _size(k_idx, "k_idx", torch.bfloat16, B * L * di)


# ---- NSA-style variant: compression and sliding-window branches beside the
# selection, mixed by caller-given gates (see include/msa.h)

def _nsa_params(q, k, block, scale, top_k=16, d_idx=128):
    B, L, H, d = q.shape
    return make_params(B, L, H, k.shape[2], d, d_idx, block, top_k, scale)


def msa_nsa_compress_kv(k, v, *, block: int = 128, k_cmp=None, v_cmp=None, stream=None):
    """Block means of k and v [B,L,G,d] -> (k_cmp, v_cmp) [B,ceil(L/block),G,d]."""
    _req(k, "k", torch.bfloat16)
    _req(v, "v", torch.bfloat16)
    B, L, G, d = k.shape
    p = make_params(B, L, G, G, d, 128, block, 1)
    nb = (L + block - 1) // block
    k_cmp = torch.empty((B, nb, G, d), dtype=torch.bfloat16, device=k.device) if k_cmp is None else k_cmp
    v_cmp = torch.empty((B, nb, G, d), dtype=torch.bfloat16, device=k.device) if v_cmp is None else v_cmp
    _size(v, "v", torch.bfloat16, B * L * G * d)
    for n, t in (("k_cmp", k_cmp), ("v_cmp", v_cmp)):
        _size(t, n, torch.bfloat16, B * nb * G * d)
    _check(lib().msa_nsa_compress_kv(ctypes.byref(p), _ptr(k), _ptr(v), _ptr(k_cmp), _ptr(v_cmp),
                                     _stream(stream)))
    return k_cmp, v_cmp


def msa_nsa_window_attn(q, k, v, window: int, *, scale: float = 0.0, want_lse: bool = False,
                        out=None, ws=None, stream=None):
    """Sliding-window branch: each query over its `window` most recent tokens."""
    for n, t in (("q", q), ("k", k), ("v", v)):
        _req(t, n, torch.bfloat16)
    p = _nsa_params(q, k, 128, scale)
    B, L, H, d = q.shape
    for n, t in (("k", k), ("v", v)):
        _size(t, n, torch.bfloat16, B * L * k.shape[2] * d)
    out = torch.empty_like(q) if out is None else out
    _size(out, "out", torch.bfloat16, B * L * H * d)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device) if want_lse else None
    ws = _ensure_ws(ws, p, MSA_OP_NSA_BRANCH, q.device)
    _check(lib().msa_nsa_window_attn(ctypes.byref(p), int(window), _ptr(q), _ptr(k), _ptr(v),
                                     _ptr(out), _ptr(lse), _ptr(ws), ws.numel(), _stream(stream)))
    return (out, lse) if want_lse else out


def msa_nsa_compressed_attn(q, k_cmp, v_cmp, *, block: int = 128, scale: float = 0.0,
                            want_lse: bool = False, out=None, ws=None, stream=None):
    """Compression branch: each query over the compressed tokens of the blocks
    whose every token lies at or before it."""
    for n, t in (("q", q), ("k_cmp", k_cmp), ("v_cmp", v_cmp)):
        _req(t, n, torch.bfloat16)
    p = _nsa_params(q, k_cmp, block, scale)
    if k_cmp.shape[1] != (q.shape[1] + block - 1) // block:
        raise ValueError("k_cmp must hold ceil(L / block) compressed tokens")
    B, L, H, d = q.shape
    for n, t in (("k_cmp", k_cmp), ("v_cmp", v_cmp)):
        _size(t, n, torch.bfloat16, B * k_cmp.shape[1] * k_cmp.shape[2] * d)
    out = torch.empty_like(q) if out is None else out
    _size(out, "out", torch.bfloat16, B * L * H * d)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device) if want_lse else None
    ws = _ensure_ws(ws, p, MSA_OP_NSA_BRANCH, q.device)
    _check(lib().msa_nsa_compressed_attn(ctypes.byref(p), _ptr(q), _ptr(k_cmp), _ptr(v_cmp),
                                         _ptr(out), _ptr(lse), _ptr(ws), ws.numel(),
                                         _stream(stream)))
    return (out, lse) if want_lse else out


def msa_nsa_gate(gates, o_cmp, o_slc, o_win, *, out=None, stream=None):
    """out = g_cmp o_cmp + g_slc o_slc + g_win o_win, gates [B,L,H,3] fp32."""
    _req(gates, "gates", torch.float32)
    for n, t in (("o_cmp", o_cmp), ("o_slc", o_slc), ("o_win", o_win)):
        _req(t, n, torch.bfloat16)
    B, L, H, d = o_cmp.shape
    p = make_params(B, L, H, H, d, 128, 128, 1)   # the gate is per head: any grouping
    out = torch.empty_like(o_cmp) if out is None else out
    _size(gates, "gates", torch.float32, B * L * H * 3)
    for n, t in (("o_slc", o_slc), ("o_win", o_win), ("out", out)):
        _size(t, n, torch.bfloat16, B * L * H * d)
    _check(lib().msa_nsa_gate(ctypes.byref(p), _ptr(gates), _ptr(o_cmp), _ptr(o_slc), _ptr(o_win),
                              _ptr(out), _stream(stream)))
    return out


def msa_nsa_forward(q, k, v, q_idx, k_idx, gates, top_k: int, window: int, *, block: int = 128,
                    scale: float = 0.0, want_sel: bool = False, out=None, sel=None, ws=None,
                    stream=None):
    """NSA-style prefill: MSA's selection branch, the compression and window
    branches, and the gate, in one call."""
    for n, t in (("q", q), ("k", k), ("v", v), ("q_idx", q_idx), ("k_idx", k_idx)):
        _req(t, n, torch.bfloat16)
    _req(gates, "gates", torch.float32)
    B, L, H, d = q.shape
    G = k.shape[2]
    _check_prefill_inputs(B, L, G, d, q_idx.shape[3], k, v, q_idx, k_idx)
    _size(gates, "gates", torch.float32, B * L * H * 3)
    p = make_params(B, L, H, G, d, q_idx.shape[3], block, top_k, scale)
    out = torch.empty_like(q) if out is None else out
    _size(out, "out", torch.bfloat16, B * L * H * d)
    if sel is None and want_sel:
        sel = torch.empty((B, G, L, top_k), dtype=torch.int32, device=q.device)
    if sel is not None:
        _size(sel, "sel", torch.int32, B * G * L * top_k)
    ws = _ensure_ws(ws, p, MSA_OP_NSA_FORWARD, q.device)
    _check(lib().msa_nsa_forward(ctypes.byref(p), int(window), _ptr(q), _ptr(k), _ptr(v),
                                 _ptr(q_idx), _ptr(k_idx), _ptr(gates), _ptr(out), _ptr(sel),
                                 _ptr(ws), ws.numel(), _stream(stream)))
    return (out, sel) if want_sel else out


def _check_cache_inputs(B, Lmax, G, d, di, k_cache, v_cache, k_idx_cache):
    for n, t in (("k_cache", k_cache), ("v_cache", v_cache)):
        _size(t, n, torch.bfloat16, B * Lmax * G * d)
    _size(k_idx_cache, "k_idx_cache", torch.bfloat16, B * Lmax * di)


def msa_forward_cached(q, q_idx, k_cache, v_cache, k_idx_cache, t0: int, top_k: int, *,
                       scale: float = 0.0, want_sel: bool = False, want_lse: bool = False,
                       out=None, sel=None, ws=None, stream=None, chunk: int = 0, block: int = 128):
    """Prefill of the n new tokens at positions [t0, t0+n) against caches that
    already hold every key up to t0+n: q [B,n,H,d], q_idx [B,n,G,d_idx];
    k_cache/v_cache [B,Lmax,G,d], k_idx_cache [B,Lmax,d_idx] -> out [B,n,H,d]
    (and sel [B,G,n,top_k], lse [B,n,H]); equal to rows [t0, t0+n) of
    msa_forward over a sequence of length t0+n."""
    for n_, t in (("q", q), ("q_idx", q_idx), ("k_cache", k_cache), ("v_cache", v_cache),
                  ("k_idx_cache", k_idx_cache)):
        _req(t, n_, torch.bfloat16)
    B, n, H, d = q.shape
    Lmax, G = k_cache.shape[1], k_cache.shape[2]
    di = q_idx.shape[3]
    _check_cache_inputs(B, Lmax, G, d, di, k_cache, v_cache, k_idx_cache)
    _size(q_idx, "q_idx", torch.bfloat16, B * n * G * di)
    p = make_params(B, Lmax, H, G, d, di, block, top_k, scale, chunk)
    dev = q.device
    if out is None:
        out = torch.empty_like(q)
    _size(out, "out", torch.bfloat16, B * n * H * d)
    if sel is None and want_sel:
        sel = torch.empty((B, G, n, top_k), dtype=torch.int32, device=dev)
    if sel is not None:
        _size(sel, "sel", torch.int32, B * G * n * top_k)
    lse = torch.empty((B, n, H), dtype=torch.float32, device=dev) if want_lse else None
    ws = _ensure_ws(ws, p, MSA_OP_FORWARD, dev)
    _check(lib().msa_forward_cached(ctypes.byref(p), int(t0), int(n), _ptr(q), _ptr(q_idx),
                                    _ptr(k_cache), _ptr(v_cache), _ptr(k_idx_cache), _ptr(out),
                                    _ptr(sel), _ptr(lse), _ptr(ws), ws.numel(), _stream(stream)))
    res = [out]
    if want_sel:
        res.append(sel)
    if want_lse:
        res.append(lse)
    return res[0] if len(res) == 1 else tuple(res)


def msa_forward_cached_varlen(q, q_idx, k_cache, v_cache, k_idx_cache, t0, n, top_k: int, *,
                              scale: float = 0.0, want_lse: bool = False, out=None, ws=None,
                              stream=None, chunk: int = 0, block: int = 128):
    """Ragged batch of cached prefills: sequence b continues at position t0[b]
    with n[b] new tokens whose query rows are packed in q [sum n,H,d] and
    q_idx [sum n,G,d_idx]; caches [B,Lmax,...].  Returns out [sum n,H,d]
    (and lse [sum n,H])."""
    for n_, t in (("q", q), ("q_idx", q_idx), ("k_cache", k_cache), ("v_cache", v_cache),
                  ("k_idx_cache", k_idx_cache)):
        _req(t, n_, torch.bfloat16)
    B, Lmax, G = k_cache.shape[0], k_cache.shape[1], k_cache.shape[2]
    H, d = q.shape[1], q.shape[2]
    if len(t0) != B or len(n) != B:
        raise ValueError(f"t0 and n need one entry per cached sequence ({B})")
    t0a = (ctypes.c_int32 * B)(*[int(v) for v in t0])
    na = (ctypes.c_int32 * B)(*[int(v) for v in n])
    N = q.shape[0]
    if sum(int(v) for v in n) != N:
        raise ValueError("q rows must equal sum(n)")
    di = q_idx.shape[2]
    _check_cache_inputs(B, Lmax, G, d, di, k_cache, v_cache, k_idx_cache)
    _size(q_idx, "q_idx", torch.bfloat16, N * G * di)
    p = make_params(B, Lmax, H, G, d, di, block, top_k, scale, chunk)
    dev = q.device
    if out is None:
        out = torch.empty_like(q)
    _size(out, "out", torch.bfloat16, N * H * d)
    lse = torch.empty((q.shape[0], H), dtype=torch.float32, device=dev) if want_lse else None
    ws = _ensure_ws(ws, p, MSA_OP_FORWARD_VARLEN, dev)
    _check(lib().msa_forward_cached_varlen(ctypes.byref(p), t0a, na, _ptr(q), _ptr(q_idx),
                                           _ptr(k_cache), _ptr(v_cache), _ptr(k_idx_cache),
                                           _ptr(out), _ptr(lse), _ptr(ws), ws.numel(),
                                           _stream(stream)))
    return (out, lse) if want_lse else out


def _req_host(t: torch.Tensor, name: str, dtype) -> torch.Tensor:
    if not isinstance(t, torch.Tensor) or t.is_cuda:
        raise ValueError(f"{name} must be a host (CPU) tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def msa_forward_host(q, k, v, q_idx, k_idx, top_k: int, *, out, lse=None, staging=None,
                     scale: float = 0.0, ws=None, stream=None, copy_stream=None, chunk: int = 0,
                     device=None, block: int = 128):
    """msa_forward on HOST tensors (pinned for overlap): q [B,L,H,d], k/v [B,L,G,d],
    q_idx [B,L,G,d_idx], k_idx [B,L,d_idx] bf16 in; out [B,L,H,d] bf16 (and lse
    [B,L,H] fp32) host tensors filled.  `staging` holds the device buffers
    (dict with q, k, v, q_idx, k_idx, out and, with lse, lse); created when
    None.  Transfers run on copy_stream (default: a new stream) overlapped
    with the computation on `stream`; synchronise `stream` before reading out."""
    for n, t in (("q", q), ("k", k), ("v", v), ("q_idx", q_idx), ("k_idx", k_idx), ("out", out)):
        _req_host(t, n, torch.bfloat16)
    if lse is not None:
        _req_host(lse, "lse", torch.float32)
    B, L, H, d = q.shape
    G = k.shape[2]
    di = q_idx.shape[3]
    need = {"q": B * L * H * d, "k": B * L * G * d, "v": B * L * G * d, "q_idx": B * L * G * di,
            "k_idx": B * L * di, "out": B * L * H * d}
    for n, t in (("k", k), ("v", v), ("q_idx", q_idx), ("k_idx", k_idx), ("out", out)):
        if t.numel() < need[n]:
            raise ValueError(f"{n} has {t.numel()} elements, the call needs {need[n]}")
    if lse is not None and lse.numel() < B * L * H:
        raise ValueError(f"lse has {lse.numel()} elements, the call needs {B * L * H}")
    p = make_params(B, L, H, G, d, di, block, top_k, scale, chunk)
    dev = torch.device("cuda") if device is None else torch.device(device)
    if staging is None:
        staging = {n: torch.empty(t.shape, dtype=t.dtype, device=dev)
                   for n, t in (("q", q), ("k", k), ("v", v), ("q_idx", q_idx), ("k_idx", k_idx),
                                ("out", out))}
        if lse is not None:
            staging["lse"] = torch.empty(lse.shape, dtype=torch.float32, device=dev)
    for n in ("q", "k", "v", "q_idx", "k_idx", "out"):
        _size(staging[n], "staging " + n, torch.bfloat16, need[n])
    if lse is not None:
        _size(staging["lse"], "staging lse", torch.float32, B * L * H)
    st = msa_staging(*(staging[n].data_ptr() for n in ("q", "k", "v", "q_idx", "k_idx", "out")),
                     staging["lse"].data_ptr() if lse is not None else None)
    ws = _ensure_ws(ws, p, MSA_OP_FORWARD, dev)
    if copy_stream is None:
        copy_stream = torch.cuda.Stream(device=dev)
    _check(lib().msa_forward_host(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(q_idx),
                                  _ptr(k_idx), _ptr(out), _ptr(lse), ctypes.byref(st), _ptr(ws),
                                  ws.numel(), _stream(stream), _stream(copy_stream)))
    return (out, lse) if lse is not None else out


def _check_decode_outputs(B, H, G, d, top_k, out, sel):
    _size(out, "out", torch.bfloat16, B * H * d)
    if sel is not None:
        _size(sel, "sel", torch.int32, B * G * top_k)


def msa_sparse_attn_decode(q, q_idx, k_cache, v_cache, k_idx_cache, seq_lens, top_k: int, *,
                           scale: float = 0.0, want_sel: bool = False, out=None, sel=None,
                           ws=None, stream=None, block: int = 128):
    """q [B,H,d], q_idx [B,G,d_idx], caches [B,Lmax,G,d] / [B,Lmax,d_idx],
    seq_lens [B] int32 (device) -> out [B,H,d] (and sel [B,G,top_k])."""
    for n, t in (("q", q), ("q_idx", q_idx), ("k_cache", k_cache), ("v_cache", v_cache),
                 ("k_idx_cache", k_idx_cache)):
        _req(t, n, torch.bfloat16)
    _req(seq_lens, "seq_lens", torch.int32)
    B, H, d = q.shape
    Lmax, G = k_cache.shape[1], k_cache.shape[2]
    di = q_idx.shape[2]
    _check_cache_inputs(B, Lmax, G, d, di, k_cache, v_cache, k_idx_cache)
    _size(q_idx, "q_idx", torch.bfloat16, B * G * di)
    _size(seq_lens, "seq_lens", torch.int32, B)
    p = make_params(B, Lmax, H, G, d, di, block, top_k, scale)
    dev = q.device
    if out is None:
        out = torch.empty_like(q)
    if sel is None and want_sel:
        sel = torch.empty((B, G, top_k), dtype=torch.int32, device=dev)
    _check_decode_outputs(B, H, G, d, top_k, out, sel)
    ws = _ensure_ws(ws, p, MSA_OP_DECODE, dev)
    _check(lib().msa_sparse_attn_decode(ctypes.byref(p), _ptr(q), _ptr(q_idx), _ptr(k_cache),
                                        _ptr(v_cache), _ptr(k_idx_cache), _ptr(seq_lens), _ptr(out),
                                        _ptr(sel), _ptr(ws), ws.numel(), _stream(stream)))
    return (out, sel) if want_sel else out


def msa_sparse_attn_decode_fp8idx(q, q_idx, k_cache, v_cache, k_idx8, k_idx_scale, seq_lens,
                                  top_k: int, *, scale: float = 0.0, want_sel: bool = False,
                                  out=None, sel=None, ws=None, stream=None, block: int = 128):
    """msa_sparse_attn_decode with the index-key cache in FP8: k_idx8 [B,Lmax,d_idx]
    uint8 E4M3 codes and k_idx_scale [B,Lmax] fp32 (stored key = scale * E4M3(code))."""
    _req(q, "q", torch.bfloat16)
    _req(q_idx, "q_idx", torch.bfloat16)
    _req(k_cache, "k_cache", torch.bfloat16)
    _req(v_cache, "v_cache", torch.bfloat16)
    _req(k_idx8, "k_idx8", torch.uint8)
    _req(k_idx_scale, "k_idx_scale", torch.float32)
    _req(seq_lens, "seq_lens", torch.int32)
    B, H, d = q.shape
    Lmax, G = k_cache.shape[1], k_cache.shape[2]
    di = k_idx8.shape[2]
    for n_, t in (("k_cache", k_cache), ("v_cache", v_cache)):
        _size(t, n_, torch.bfloat16, B * Lmax * G * d)
    _size(k_idx8, "k_idx8", torch.uint8, B * Lmax * di)
    _size(k_idx_scale, "k_idx_scale", torch.float32, B * Lmax)
    _size(q_idx, "q_idx", torch.bfloat16, B * G * di)
    _size(seq_lens, "seq_lens", torch.int32, B)
    p = make_params(B, Lmax, H, G, d, di, block, top_k, scale)
    dev = q.device
    if out is None:
        out = torch.empty_like(q)
    if sel is None and want_sel:
        sel = torch.empty((B, G, top_k), dtype=torch.int32, device=dev)
    _check_decode_outputs(B, H, G, d, top_k, out, sel)
    ws = _ensure_ws(ws, p, MSA_OP_DECODE, dev)
    _check(lib().msa_sparse_attn_decode_fp8idx(ctypes.byref(p), _ptr(q), _ptr(q_idx), _ptr(k_cache),
                                               _ptr(v_cache), _ptr(k_idx8), _ptr(k_idx_scale),
                                               _ptr(seq_lens), _ptr(out), _ptr(sel), _ptr(ws),
                                               ws.numel(), _stream(stream)))
    return (out, sel) if want_sel else out


def msa_sparse_attn_decode_fp8(q, q_idx, k8, k_scale, v8, v_scale, k_idx8, k_idx_scale,
                               seq_lens, top_k: int, *, scale: float = 0.0, want_sel: bool = False,
                               out=None, sel=None, ws=None, stream=None, block: int = 128):
    """Decode step with every cache in FP8: k8/v8 [B,Lmax,G,d] uint8 E4M3 with
    k_scale/v_scale [B,Lmax,G] fp32, k_idx8 [B,Lmax,d_idx] with k_idx_scale [B,Lmax]."""
    _req(q, "q", torch.bfloat16)
    _req(q_idx, "q_idx", torch.bfloat16)
    for n_, t in (("k8", k8), ("v8", v8), ("k_idx8", k_idx8)):
        _req(t, n_, torch.uint8)
    for n_, t in (("k_scale", k_scale), ("v_scale", v_scale), ("k_idx_scale", k_idx_scale)):
        _req(t, n_, torch.float32)
    _req(seq_lens, "seq_lens", torch.int32)
    B, H, d = q.shape
    Lmax, G = k8.shape[1], k8.shape[2]
    di = k_idx8.shape[2]
    for n_, t in (("k8", k8), ("v8", v8)):
        _size(t, n_, torch.uint8, B * Lmax * G * d)
    for n_, t in (("k_scale", k_scale), ("v_scale", v_scale)):
        _size(t, n_, torch.float32, B * Lmax * G)
    _size(k_idx8, "k_idx8", torch.uint8, B * Lmax * di)
    _size(k_idx_scale, "k_idx_scale", torch.float32, B * Lmax)
    _size(q_idx, "q_idx", torch.bfloat16, B * G * di)
    _size(seq_lens, "seq_lens", torch.int32, B)
    p = make_params(B, Lmax, H, G, d, di, block, top_k, scale)
    dev = q.device
    if out is None:
        out = torch.empty_like(q)
    if sel is None and want_sel:
        sel = torch.empty((B, G, top_k), dtype=torch.int32, device=dev)
    _check_decode_outputs(B, H, G, d, top_k, out, sel)
    ws = _ensure_ws(ws, p, MSA_OP_DECODE, dev)
    _check(lib().msa_sparse_attn_decode_fp8(ctypes.byref(p), _ptr(q), _ptr(q_idx), _ptr(k8),
                                            _ptr(k_scale), _ptr(v8), _ptr(v_scale), _ptr(k_idx8),
                                            _ptr(k_idx_scale), _ptr(seq_lens), _ptr(out),
                                            _ptr(sel), _ptr(ws), ws.numel(), _stream(stream)))
    return (out, sel) if want_sel else out


def msa_quantize_e4m3_rows(x, *, codes=None, scale=None, stream=None):
    """bf16 [..., cols] -> (E4M3 codes uint8 [..., cols], fp32 scale [...]), one scale per row."""
    _req(x, "x", torch.bfloat16)
    cols = x.shape[-1]
    rows = x.numel() // cols
    if codes is None:
        codes = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    if scale is None:
        scale = torch.empty(x.shape[:-1], dtype=torch.float32, device=x.device)
    _size(codes, "codes", torch.uint8, rows * cols)
    _size(scale, "scale", torch.float32, rows)
    _check(lib().msa_quantize_e4m3_rows(_ptr(x), rows, cols, _ptr(codes), _ptr(scale),
                                        _stream(stream)))
    return codes, scale


def msa_sparse_attn_decode_noalloc(q, q_idx, k_cache, v_cache, k_idx_cache, seq_lens, top_k: int, *,
                                   scale: float = 0.0, want_sel: bool = False, out=None, sel=None,
                                   stream=None, block: int = 128):
    """Decode step that passes no workspace: the library uses its own 16 MiB
    device scratch (for callers that cannot allocate device memory at the
    call site).  Same arguments and results as msa_sparse_attn_decode.  Only
    the outputs are allocated here, and only when not passed in."""
    for n, t in (("q", q), ("q_idx", q_idx), ("k_cache", k_cache), ("v_cache", v_cache),
                 ("k_idx_cache", k_idx_cache)):
        _req(t, n, torch.bfloat16)
    _req(seq_lens, "seq_lens", torch.int32)
    B, H, d = q.shape
    Lmax, G = k_cache.shape[1], k_cache.shape[2]
    di = q_idx.shape[2]
    _check_cache_inputs(B, Lmax, G, d, di, k_cache, v_cache, k_idx_cache)
    _size(q_idx, "q_idx", torch.bfloat16, B * G * di)
    _size(seq_lens, "seq_lens", torch.int32, B)
    p = make_params(B, Lmax, H, G, d, di, block, top_k, scale)
    if out is None:
        out = torch.empty_like(q)
    if sel is None and want_sel:
        sel = torch.empty((B, G, top_k), dtype=torch.int32, device=q.device)
    _check_decode_outputs(B, H, G, d, top_k, out, sel)
    _check(lib().msa_sparse_attn_decode_noalloc(ctypes.byref(p), _ptr(q), _ptr(q_idx), _ptr(k_cache),
                                                _ptr(v_cache), _ptr(k_idx_cache), _ptr(seq_lens),
                                                _ptr(out), _ptr(sel), _stream(stream)))
    return (out, sel) if want_sel else out


def msa_read_status(ws: torch.Tensor, stream=None) -> int:
    """Synchronise and return (then clear) the device status word in ws."""
    return lib().msa_read_status(_ptr(ws), _stream(stream))
