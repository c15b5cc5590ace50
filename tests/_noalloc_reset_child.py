"""Child process of tests/test_zz_no_alloc.py: the no-allocation decode
before and after cudaDeviceReset.

cudaDeviceReset destroys the device's primary context; the next runtime call
builds a new one and loads the library's module into it again, so the
scratch array may sit at a new device address.  This process calls
msa_sparse_attn_decode_noalloc, resets the device, makes new inputs and calls
it again, each time checking it against msa_sparse_attn_decode with a
workspace.  It drives the CUDA runtime through ctypes only: torch is not
imported, because a reset would pull the context from under torch's
allocator.  Exit status 0 means both rounds agreed.
"""
import ctypes
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIB = os.path.join(ROOT, "block_sparse_long_08_b200", "libmsa.so")
H2D, D2H = 1, 2   # cudaMemcpyHostToDevice, cudaMemcpyDeviceToHost


class Params(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("B", "L", "H", "G", "d", "d_idx", "block",
                                               "top_k")] + [("scale", ctypes.c_float),
                                                            ("chunk", ctypes.c_int32)]


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round to nearest even (finite inputs)."""
    u = x.astype(np.float32).view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def bf16_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32)


def main() -> int:
    rt = ctypes.CDLL("libcudart.so.12", mode=ctypes.RTLD_GLOBAL)
    lib = ctypes.CDLL(LIB)
    P, SZ = ctypes.c_void_p, ctypes.c_size_t
    pp = ctypes.POINTER(Params)
    lib.msa_workspace_bytes.argtypes = [pp, ctypes.c_int]
    lib.msa_workspace_bytes.restype = SZ
    lib.msa_sparse_attn_decode.argtypes = [pp] + [P] * 9 + [SZ, P]
    lib.msa_sparse_attn_decode_noalloc.argtypes = [pp] + [P] * 9
    lib.msa_last_error.restype = ctypes.c_char_p
    rt.cudaMalloc.argtypes = [ctypes.POINTER(P), SZ]
    rt.cudaMemcpy.argtypes = [P, P, SZ, ctypes.c_int]
    rt.cudaMemset.argtypes = [P, ctypes.c_int, SZ]
    rt.cudaFree.argtypes = [P]

    def ck(e, what):
        if e != 0:
            raise SystemExit(f"{what}: CUDA error {e}")

    def upload(a: np.ndarray) -> P:
        p = P()
        ck(rt.cudaMalloc(ctypes.byref(p), a.nbytes), "cudaMalloc")
        ck(rt.cudaMemcpy(p, a.ctypes.data_as(P), a.nbytes, H2D), "upload")
        return p

    def empty(nbytes: int) -> P:
        p = P()
        ck(rt.cudaMalloc(ctypes.byref(p), nbytes), "cudaMalloc")
        ck(rt.cudaMemset(p, 0, nbytes), "cudaMemset")
        return p

    def download(p: P, shape, dtype) -> np.ndarray:
        a = np.empty(shape, dtype=dtype)
        ck(rt.cudaMemcpy(a.ctypes.data_as(P), p, a.nbytes, D2H), "download")
        return a

    def one_round(seed: int):
        B, Lmax, H, G, di, top_k = 3, 4096, 8, 2, 64, 4
        rng = np.random.default_rng(seed)
        lens = np.array([4096, 2000, 129], dtype=np.int32)
        host = {"q": bf16_bits(rng.standard_normal((B, H, 128))),
                "q_idx": bf16_bits(rng.standard_normal((B, G, di))),
                "k": bf16_bits(rng.standard_normal((B, Lmax, G, 128))),
                "v": bf16_bits(rng.standard_normal((B, Lmax, G, 128))),
                "k_idx": bf16_bits(rng.standard_normal((B, Lmax, di)))}
        dev = {n: upload(a) for n, a in host.items()}
        d_lens = upload(lens)
        p = Params(B, Lmax, H, G, 128, di, 128, top_k, 0.0, 0)
        ws_bytes = lib.msa_workspace_bytes(ctypes.byref(p), 2)
        ws = empty(ws_bytes)
        outs, sels = [empty(B * H * 128 * 2) for _ in range(2)], [empty(B * G * top_k * 4)
                                                                 for _ in range(2)]
        args = (dev["q"], dev["q_idx"], dev["k"], dev["v"], dev["k_idx"], d_lens)
        rc = lib.msa_sparse_attn_decode(ctypes.byref(p), *args, outs[0], sels[0], ws, ws_bytes, None)
        ck(rc, "msa_sparse_attn_decode " + lib.msa_last_error().decode())
        rc = lib.msa_sparse_attn_decode_noalloc(ctypes.byref(p), *args, outs[1], sels[1], None)
        ck(rc, "msa_sparse_attn_decode_noalloc " + lib.msa_last_error().decode())
        ck(rt.cudaDeviceSynchronize(), "kernels")
        ref, got = (bf16_f32(download(o, (B, H, 128), np.uint16)) for o in outs)
        sref, sgot = (download(s, (B, G, top_k), np.int32) for s in sels)
        err = np.abs(got.astype(np.float64) - ref)
        assert np.array_equal(sref, sgot), (sref, sgot)
        assert np.isfinite(got).all() and err.max() <= 2e-2 and err.mean() <= 2e-3, err.max()
        for a in list(dev.values()) + [d_lens, ws] + outs + sels:
            ck(rt.cudaFree(a), "cudaFree")

    ck(rt.cudaSetDevice(0), "cudaSetDevice")
    one_round(301)
    ck(rt.cudaDeviceReset(), "cudaDeviceReset")
    one_round(302)   # a new context: the scratch address is looked up again
    print("noalloc across cudaDeviceReset: ok")
    return 0


if __name__ == "__main__":
    sys.exit(main())
