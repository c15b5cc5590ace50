"""CPU tests of the C-ABI boundary: the library loads, exports every entry
point its header declares, sizes workspaces and rejects bad arguments
before touching the device."""
import ctypes
import os

import pytest

import block_sparse_long_08_b200.msa as M


def test_library_exports_header_symbols():
    lib = M.lib()
    names = M.header_functions()
    assert {"msa_index_select", "msa_sparse_attn_prefill", "msa_sparse_attn_decode",
            "msa_forward", "msa_workspace_bytes", "msa_last_error"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n


def test_version():
    assert b"sm_100a" in M.lib().msa_version()


@pytest.mark.parametrize("L,top_k,G,H,di", [(2048, 4, 2, 8, 64), (32768, 16, 8, 32, 128),
                                             (1048576, 16, 8, 32, 128)])
def test_workspace_sizes(L, top_k, G, H, di):
    p = M.make_params(1, L, H, G, 128, di, 128, top_k)
    ws_sel = M.msa_workspace_bytes(p, M.MSA_OP_INDEX_SELECT)
    ws_att = M.msa_workspace_bytes(p, M.MSA_OP_PREFILL_ATTN)
    ws_fwd = M.msa_workspace_bytes(p, M.MSA_OP_FORWARD)
    ws_dec = M.msa_workspace_bytes(p, M.MSA_OP_DECODE)
    assert ws_sel >= 4
    # forward = selection buffer + attention workspace
    assert ws_fwd >= ws_att + 4 * L * G * top_k
    # the partial-result budget (16 GiB) bounds the prefill workspace; the
    # chunk always holds the partials of whole queries
    assert ws_att < 17 * 2**30
    lc = M.msa_prefill_chunk_len(p)
    assert lc % 128 == 0 and 128 <= lc <= L
    assert ws_att >= lc * H * top_k * 128 * 2
    assert ws_dec < 64 * 2**20
    # backward: per query chunk a reverse index and one bf16 dq row per
    # (query, head, slot); D for every row; fp32 dk/dv accumulators when
    # there is more than one chunk
    ws_bwd = M.msa_workspace_bytes(p, M.MSA_OP_BACKWARD)
    entries = lc * G * top_k
    acc = 2 * L * G * 128 * 4 if lc < L else 0
    need = entries * (H // G) * 128 * 2 + 2 * 4 * entries + 4 * L * H + acc
    assert need <= ws_bwd <= need + 2 * 2**20
    assert ws_bwd < 27 * 2**30


@pytest.mark.parametrize("field,value,code", [
    ("d", 64, M.MSA_ERR_UNSUPPORTED), ("d_idx", 96, M.MSA_ERR_UNSUPPORTED),
    ("block", 32, M.MSA_ERR_UNSUPPORTED), ("top_k", 33, M.MSA_ERR_UNSUPPORTED),
    ("top_k", 0, M.MSA_ERR_INVALID_ARG), ("L", -5, M.MSA_ERR_INVALID_ARG),
    ("H", 12, M.MSA_ERR_UNSUPPORTED), ("G", 3, M.MSA_ERR_INVALID_ARG),
    ("B", -1, M.MSA_ERR_INVALID_ARG), ("chunk", 100, M.MSA_ERR_INVALID_ARG),
    ("chunk", -128, M.MSA_ERR_INVALID_ARG)])
def test_bad_params_rejected_before_launch(field, value, code):
    p = M.make_params(1, 2048, 8, 2, 128, 64, 128, 4)
    setattr(p, field, value)
    lib = M.lib()
    dummy = ctypes.c_void_p(256)  # never dereferenced: the check fails first
    rc = lib.msa_index_select(ctypes.byref(p), dummy, dummy, dummy, None, dummy, 1 << 20, None)
    assert rc == code, (rc, M.msa_last_error())
    assert M.msa_last_error()
    assert lib.msa_workspace_bytes(ctypes.byref(p), 0) == 0


def test_null_and_misaligned_pointers_rejected():
    p = M.make_params(1, 2048, 8, 2, 128, 64, 128, 4)
    lib = M.lib()
    ok = ctypes.c_void_p(4096)
    rc = lib.msa_index_select(ctypes.byref(p), None, ok, ok, None, ok, 1 << 20, None)
    assert rc == M.MSA_ERR_INVALID_ARG
    rc = lib.msa_index_select(ctypes.byref(p), ctypes.c_void_p(4098), ok, ok, None, ok, 1 << 20, None)
    assert rc == M.MSA_ERR_INVALID_ARG
    rc = lib.msa_index_select(ctypes.byref(p), ok, ok, ok, None, ctypes.c_void_p(4096 + 16), 1 << 20, None)
    assert rc == M.MSA_ERR_WORKSPACE
    rc = lib.msa_index_select(ctypes.byref(p), ok, ok, ok, None, ok, 8, None)
    assert rc == M.MSA_ERR_WORKSPACE


def test_empty_problem_is_noop():
    p = M.make_params(0, 2048, 8, 2, 128, 64, 128, 4)
    lib = M.lib()
    assert lib.msa_index_select(ctypes.byref(p), None, None, None, None, None, 0, None) == M.MSA_OK
    p = M.make_params(1, 0, 8, 2, 128, 64, 128, 4)
    assert lib.msa_forward(ctypes.byref(p), None, None, None, None, None, None, None, None, None, 0,
                           None) == M.MSA_OK


def test_chunk_length_follows_params():
    p = M.make_params(2, 8192, 32, 8, 128, 128, 128, 16)
    full = M.msa_prefill_chunk_len(p)
    assert full == 16384                      # small problems run as one chunk of packed rows
    for c, want in ((1024, 1024), (128, 128), (16384, 16384), (32768, 16384)):
        p.chunk = c
        assert M.msa_prefill_chunk_len(p) == want
    # a shorter chunk needs a smaller prefill workspace
    p.chunk = 1024
    small = M.msa_workspace_bytes(p, M.MSA_OP_PREFILL_ATTN)
    p.chunk = 0
    assert small < M.msa_workspace_bytes(p, M.MSA_OP_PREFILL_ATTN)


def test_forward_host_rejects_bad_arguments():
    p = M.make_params(1, 2048, 8, 2, 128, 64, 128, 4)
    lib = M.lib()
    h = ctypes.c_void_p(4096)
    st = M.msa_staging(4096, 4096, 4096, 4096, 4096, 4096, None)
    rc = lib.msa_forward_host(ctypes.byref(p), h, h, h, h, h, h, None, None, h, 1 << 30, None, None)
    assert rc == M.MSA_ERR_INVALID_ARG          # no staging buffers
    bad = M.msa_staging(4096 + 8, 4096, 4096, 4096, 4096, 4096, None)
    rc = lib.msa_forward_host(ctypes.byref(p), h, h, h, h, h, h, None, ctypes.byref(bad), h,
                              1 << 30, None, None)
    assert rc == M.MSA_ERR_INVALID_ARG          # misaligned staging
    rc = lib.msa_forward_host(ctypes.byref(p), h, h, h, h, h, h, h, ctypes.byref(st), h, 1 << 30,
                              None, None)
    assert rc == M.MSA_ERR_INVALID_ARG          # lse requested without device lse
    rc = lib.msa_forward_host(ctypes.byref(p), h, h, h, h, h, h, None, ctypes.byref(st), h, 64,
                              None, None)
    assert rc == M.MSA_ERR_WORKSPACE


@pytest.mark.parametrize("t0,n", [(-128, 128), (3968, 256), (0, -128), (4000, 97), (-1, 1)])
def test_cached_prefill_rejects_bad_ranges(t0, n):
    p = M.make_params(1, 4096, 8, 2, 128, 64, 128, 4)
    ok = ctypes.c_void_p(4096)
    rc = M.lib().msa_forward_cached(ctypes.byref(p), t0, n, ok, ok, ok, ok, ok, ok, None, None, ok,
                                    1 << 30, None)
    assert rc == M.MSA_ERR_INVALID_ARG, (rc, M.msa_last_error())


def test_varlen_rejects_bad_ranges():
    p = M.make_params(2, 4096, 8, 2, 128, 64, 128, 4)
    ok = ctypes.c_void_p(4096)
    for t0, n in (([0, 4000], [128, 100]), ([0, 3968], [128, 256]), ([-128, 0], [128, 128]),
                  ([5, 0], [-1, 128])):
        rc = M.lib().msa_forward_cached_varlen(ctypes.byref(p), (ctypes.c_int32 * 2)(*t0),
                                               (ctypes.c_int32 * 2)(*n), ok, ok, ok, ok, ok, ok,
                                               None, ok, 1 << 30, None)
        assert rc == M.MSA_ERR_INVALID_ARG, (t0, n, M.msa_last_error())


def test_decode_rejects_more_than_eight_groups():
    p = M.make_params(2, 4096, 32, 16, 128, 128, 128, 16)
    assert M.lib().msa_workspace_bytes(ctypes.byref(p), M.MSA_OP_DECODE) == 0


def test_backward_rejects_bad_arguments():
    """Argument checks of msa_sparse_attn_backward run before any CUDA call."""
    p = M.make_params(1, 1024, 8, 2, 128, 128, 128, 4)
    lib = M.lib()
    ok = ctypes.c_void_p(4096)
    need = M.msa_workspace_bytes(p, M.MSA_OP_BACKWARD)
    args = [ok] * 10
    rc = lib.msa_sparse_attn_backward(ctypes.byref(p), *args[:4], None, *args[5:], ok, need, None)
    assert rc == M.MSA_ERR_INVALID_ARG                       # lse is required
    bad = list(args)
    bad[6] = ctypes.c_void_p(4096 + 4)                        # misaligned sel
    rc = lib.msa_sparse_attn_backward(ctypes.byref(p), *bad, ok, need, None)
    assert rc == M.MSA_ERR_INVALID_ARG
    rc = lib.msa_sparse_attn_backward(ctypes.byref(p), *args, ok, need - 1, None)
    assert rc == M.MSA_ERR_WORKSPACE
    # workspace: reverse index + D + one fp32 dq row per (query, head, slot)
    assert need >= 1024 * 8 * 4 * 128 * 2 + 1024 * 8 * 4
    p0 = M.make_params(0, 1024, 8, 2, 128, 128, 128, 4)
    assert lib.msa_sparse_attn_backward(ctypes.byref(p0), *([None] * 10), None, 0, None) == M.MSA_OK


def test_nsa_entry_points_reject_bad_arguments():
    """Argument checks of the NSA-style entry points run before any CUDA
    call: window >= 1, no NULL tensors, 16-byte alignment, workspace size."""
    p = M.make_params(1, 1000, 8, 2, 128, 128, 128, 4)
    lib = M.lib()
    ok = ctypes.c_void_p(4096)
    odd = ctypes.c_void_p(4096 + 8)
    hdr = M.msa_workspace_bytes(p, M.MSA_OP_NSA_BRANCH)
    assert hdr == 256
    assert lib.msa_nsa_window_attn(ctypes.byref(p), 0, ok, ok, ok, ok, None, ok, hdr,
                                   None) == M.MSA_ERR_INVALID_ARG
    assert lib.msa_nsa_window_attn(ctypes.byref(p), 64, ok, None, ok, ok, None, ok, hdr,
                                   None) == M.MSA_ERR_INVALID_ARG
    assert lib.msa_nsa_window_attn(ctypes.byref(p), 64, ok, ok, ok, ok, odd, ok, hdr,
                                   None) == M.MSA_ERR_INVALID_ARG
    assert lib.msa_nsa_window_attn(ctypes.byref(p), 64, ok, ok, ok, ok, None, ok, hdr - 1,
                                   None) == M.MSA_ERR_WORKSPACE
    assert lib.msa_nsa_compressed_attn(ctypes.byref(p), ok, ok, odd, ok, None, ok, hdr,
                                       None) == M.MSA_ERR_INVALID_ARG
    assert lib.msa_nsa_compress_kv(ctypes.byref(p), ok, ok, None, ok, None) == M.MSA_ERR_INVALID_ARG
    assert lib.msa_nsa_gate(ctypes.byref(p), odd, ok, ok, ok, ok, None) == M.MSA_ERR_INVALID_ARG
    need = M.msa_workspace_bytes(p, M.MSA_OP_NSA_FORWARD)
    # msa_forward's workspace, then k_cmp, v_cmp (8 blocks) and two outputs
    assert need >= (M.msa_workspace_bytes(p, M.MSA_OP_FORWARD) + 2 * 8 * 2 * 128 * 2
                    + 2 * 1000 * 8 * 128 * 2)
    args = [ok] * 7
    assert lib.msa_nsa_forward(ctypes.byref(p), 0, *args, None, ok, need,
                               None) == M.MSA_ERR_INVALID_ARG
    assert lib.msa_nsa_forward(ctypes.byref(p), 512, *args, None, ok, need - 1,
                               None) == M.MSA_ERR_WORKSPACE
    p0 = M.make_params(0, 1000, 8, 2, 128, 128, 128, 4)
    assert lib.msa_nsa_window_attn(ctypes.byref(p0), 5, *([None] * 5), None, 0, None) == M.MSA_OK


def test_plain_c_program_uses_the_library(tmp_path):
    """The boundary is a C ABI: a C99 program, compiled with warnings as
    errors against include/msa.h alone, links libmsa.so and calls its
    host-side entry points (workspace sizing, argument checks, version)
    without Python or torch."""
    import shutil
    import subprocess

    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not available")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    libdir = os.path.dirname(M.LIB_PATH)
    src = tmp_path / "use_msa.c"
    src.write_text(r'''
#include <stdio.h>
#include <string.h>
#include "msa.h"
int main(void) {
  msa_params p;
  memset(&p, 0, sizeof p);
  p.B = 1; p.L = 32768; p.H = 32; p.G = 8; p.d = 128; p.d_idx = 128; p.block = 128;
  p.top_k = 16;
  size_t w = msa_workspace_bytes(&p, MSA_OP_BACKWARD);
  int rc = msa_index_select(&p, NULL, NULL, NULL, NULL, NULL, 0, NULL);
  printf("%s|%zu|%d|%s\n", msa_version(), w, rc, msa_last_error());
  return (w > 0 && rc == MSA_ERR_INVALID_ARG) ? 0 : 1;
}
''')
    exe = tmp_path / "use_msa"
    cuda_lib = "/usr/local/cuda/lib64"
    cmd = [gcc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
           "-I" + os.path.join(root, "include"), str(src), "-o", str(exe),
           "-L" + libdir, "-lmsa", "-Wl,-rpath," + libdir]
    if os.path.isdir(cuda_lib):
        cmd += ["-L" + cuda_lib, "-Wl,-rpath," + cuda_lib]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, (r.stdout, r.stderr)
    version, ws, rc, msg = r.stdout.strip().split("|")
    assert "sm_100a" in version
    assert int(ws) == M.msa_workspace_bytes(M.make_params(1, 32768, 32, 8, top_k=16),
                                            M.MSA_OP_BACKWARD)
    assert int(rc) == M.MSA_ERR_INVALID_ARG and msg


def test_backward_workspace_follows_chunking():
    """One chunk: no dk/dv accumulators.  Several chunks (p.chunk): the
    reverse index and dq partials shrink to one chunk, and fp32 dk/dv
    accumulators for the whole sequence are added."""
    L, H, G, K = 4096, 16, 4, 8
    whole = M.msa_workspace_bytes(M.make_params(1, L, H, G, top_k=K), M.MSA_OP_BACKWARD)
    half = M.msa_workspace_bytes(M.make_params(1, L, H, G, top_k=K, chunk=L // 2),
                                 M.MSA_OP_BACKWARD)
    per_chunk = lambda lc: lc * G * K * (H // G) * 128 * 2 + 2 * 4 * lc * G * K
    acc = 2 * L * G * 128 * 4
    assert abs((whole - per_chunk(L)) - (half - per_chunk(L // 2) - acc)) <= 4096
    assert M.msa_prefill_chunk_len(M.make_params(1, L, H, G, top_k=K, chunk=L // 2)) == L // 2


def test_any_length_and_either_block_in_every_operation():
    """L need not be a multiple of the block length: the last block of a
    sequence is partial.  Every operation takes 64- and 128-token blocks."""
    lib = M.lib()
    for L in (1, 127, 1000, 2049):
        for blk in (64, 128):
            p = M.make_params(2, L, 16, 4, 128, 128, blk, 5)
            for op in (M.MSA_OP_INDEX_SELECT, M.MSA_OP_PREFILL_ATTN, M.MSA_OP_DECODE,
                       M.MSA_OP_FORWARD, M.MSA_OP_FORWARD_VARLEN, M.MSA_OP_BACKWARD):
                assert lib.msa_workspace_bytes(ctypes.byref(p), op) > 0, (L, blk, op,
                                                                         M.msa_last_error())
    # the ragged-batch workspace holds the uniform forward's plus its tables
    p = M.make_params(4, 4096, 16, 4, 128, 128, 128, 8)
    assert (M.msa_workspace_bytes(p, M.MSA_OP_FORWARD_VARLEN)
            >= M.msa_workspace_bytes(p, M.MSA_OP_FORWARD) + 4 * (2 * 128 + 16 + 32 * 8))


def test_decode_entry_points_reject_bad_arguments():
    """The bf16 and both FP8 decodes check pointers, alignment (scales
    4-byte) and the workspace before any launch."""
    p = M.make_params(2, 4096, 8, 2, 128, 64, 128, 4)
    lib = M.lib()
    ok, odd, odd4 = ctypes.c_void_p(4096), ctypes.c_void_p(4104), ctypes.c_void_p(4098)
    need = M.msa_workspace_bytes(p, M.MSA_OP_DECODE)
    dec = lambda q, out, ws, nbytes: lib.msa_sparse_attn_decode(ctypes.byref(p), q, ok, ok, ok, ok,
                                                               ok, out, None, ws, nbytes, None)
    assert dec(None, ok, ok, need) == M.MSA_ERR_INVALID_ARG
    assert dec(ok, odd, ok, need) == M.MSA_ERR_INVALID_ARG
    assert dec(ok, ok, ok, need - 1) == M.MSA_ERR_WORKSPACE
    assert dec(ok, ok, None, need) == M.MSA_ERR_WORKSPACE
    p0 = M.make_params(2, 0, 8, 2, 128, 64, 128, 4)   # a decode needs a cache
    assert lib.msa_sparse_attn_decode(ctypes.byref(p0), ok, ok, ok, ok, ok, ok, ok, None, ok, need,
                                      None) == M.MSA_ERR_INVALID_ARG

    def fp8idx(k_idx8, scale):
        return lib.msa_sparse_attn_decode_fp8idx(ctypes.byref(p), ok, ok, ok, ok, k_idx8, scale, ok,
                                                 ok, None, ok, need, None)
    assert fp8idx(None, ok) == M.MSA_ERR_INVALID_ARG
    assert fp8idx(ok, None) == M.MSA_ERR_INVALID_ARG
    assert fp8idx(odd, ok) == M.MSA_ERR_INVALID_ARG
    assert fp8idx(ok, odd4) == M.MSA_ERR_INVALID_ARG     # scales need 4-byte alignment

    def fp8(k8, ks, v8, vs, nbytes=need):
        return lib.msa_sparse_attn_decode_fp8(ctypes.byref(p), ok, ok, k8, ks, v8, vs, ok, ok, ok,
                                              ok, None, ok, nbytes, None)
    assert fp8(None, ok, ok, ok) == M.MSA_ERR_INVALID_ARG
    assert fp8(ok, ok, None, ok) == M.MSA_ERR_INVALID_ARG
    assert fp8(ok, None, ok, ok) == M.MSA_ERR_INVALID_ARG
    assert fp8(odd, ok, ok, ok) == M.MSA_ERR_INVALID_ARG
    assert fp8(ok, ok, ok, odd4) == M.MSA_ERR_INVALID_ARG
    assert fp8(ok, ok, ok, ok, need - 16) == M.MSA_ERR_WORKSPACE
    # the no-allocation decode reports bad parameters like the regular one
    bad = M.make_params(2, 4096, 8, 2, 128, 64, 128, 0)
    assert lib.msa_sparse_attn_decode_noalloc(ctypes.byref(bad), ok, ok, ok, ok, ok, ok, ok, None,
                                              None) == M.MSA_ERR_INVALID_ARG


def test_prefill_attention_and_quantizer_reject_bad_arguments():
    p = M.make_params(1, 2048, 8, 2, 128, 64, 128, 4)
    lib = M.lib()
    ok, odd = ctypes.c_void_p(4096), ctypes.c_void_p(4104)
    need = M.msa_workspace_bytes(p, M.MSA_OP_PREFILL_ATTN)
    att = lambda sel, lse, nbytes: lib.msa_sparse_attn_prefill(ctypes.byref(p), ok, ok, ok, sel, ok,
                                                               lse, ok, nbytes, None)
    assert att(None, None, need) == M.MSA_ERR_INVALID_ARG
    assert att(ok, odd, need) == M.MSA_ERR_INVALID_ARG
    assert att(ok, None, need - 1) == M.MSA_ERR_WORKSPACE
    q8 = lambda x, rows, cols, codes, scale: lib.msa_quantize_e4m3_rows(x, rows, cols, codes, scale,
                                                                        None)
    assert q8(ok, 4, 0, ok, ok) == M.MSA_ERR_INVALID_ARG
    assert q8(ok, 4, 24, ok, ok) == M.MSA_ERR_INVALID_ARG    # columns come in 16-byte granules
    assert q8(ok, -1, 16, ok, ok) == M.MSA_ERR_INVALID_ARG
    assert q8(None, 0, 16, None, None) == M.MSA_OK           # no rows: nothing to do
    assert q8(ok, 4, 16, None, ok) == M.MSA_ERR_INVALID_ARG
    assert q8(ok, 4, 16, ok, odd) == M.MSA_ERR_INVALID_ARG
