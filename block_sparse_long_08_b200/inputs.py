"""Seeded synthetic inputs for MSA prefill and decode.

This module only draws random numbers and lays them out; it holds none of
the attention arithmetic.  Both the CUDA path's tests/benchmark and the CPU
oracle's tests take their inputs from here, so the two sides always see the
same bf16 bit patterns.

Recipe: every tensor is drawn i.i.d. N(0, 1) in fp32 from one
`torch.Generator` seeded per workload, in the fixed order q, k, v, q_idx,
k_idx (prefill) or q, q_idx, k_cache, v_cache, k_idx_cache (decode), then
rounded to bf16 (round-to-nearest-even).  Ragged decode lengths and planted
needle structure come from a separate CPU generator seeded with the same
seed, so they do not depend on the device the tensors are drawn on.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import torch

BF16 = torch.bfloat16


@dataclasses.dataclass(frozen=True)
class PrefillShape:
    B: int
    L: int
    H: int
    G: int
    d: int = 128
    d_idx: int = 128
    block: int = 128
    top_k: int = 16


@dataclasses.dataclass(frozen=True)
class DecodeShape:
    B: int
    Lmax: int
    H: int
    G: int
    d: int = 128
    d_idx: int = 128
    block: int = 128
    top_k: int = 16
    len_lo: int = 0   # ragged lengths uniform in [len_lo, len_hi]
    len_hi: int = 0


# The pages' workloads (MiniMax Sparse Attention, "2048 个 KV token" section:
# 16 blocks of 128 tokens) at the sizes the benchmarks use.
PREFILL_TINY = PrefillShape(B=1, L=2048, H=8, G=2, d=128, d_idx=64, top_k=4)
PREFILL_32K = PrefillShape(B=1, L=32768, H=32, G=8)
PREFILL_128K_PLANTED = PrefillShape(B=1, L=131072, H=32, G=8)
DECODE_128K = DecodeShape(B=32, Lmax=131072, H=32, G=8, len_lo=65536, len_hi=131072)
PREFILL_1M = PrefillShape(B=1, L=1048576, H=32, G=8)
DECODE_1M = DecodeShape(B=4, Lmax=1048576, H=32, G=8, len_lo=1048576, len_hi=1048576)

# The 64-token block variant of the 32K prefill at the same 2048-token
# budget ("MiniMax M3 sparse attention" explainer §4.2 reasons with 64-token
# blocks): 32 blocks of 64.
PREFILL_32K_BLOCK64 = PrefillShape(B=1, L=32768, H=32, G=8, block=64, top_k=32)


@dataclasses.dataclass(frozen=True)
class RaggedBatchShape:
    """Prompt chunks continuing cached prefixes: B sequences, caches of Lmax
    tokens, n_b new tokens uniform in [1, n_hi], positions t0_b uniform in
    [0, Lmax - n_b]."""
    B: int
    Lmax: int
    n_hi: int
    H: int
    G: int
    d: int = 128
    d_idx: int = 128
    top_k: int = 16


RAGGED_BATCH = RaggedBatchShape(B=16, Lmax=131072, n_hi=16384, H=32, G=8)

SEEDS = {"tiny": 0, "32k": 1, "128k_planted": 2, "decode_128k": 3, "1m": 4, "ragged": 5}


def _normal_bf16(gen: torch.Generator, shape, device) -> torch.Tensor:
    return torch.randn(shape, generator=gen, device=device, dtype=torch.float32).to(BF16)


def prefill_inputs(shape: PrefillShape, seed: int, device="cpu",
                   needles: int = 0, needle_alpha: float = 3.0) -> dict:
    """q [B,L,H,d], k/v [B,L,G,d], q_idx [B,L,G,d_idx], k_idx [B,L,d_idx], bf16.

    needles > 0 plants, per group g, `needles` seeded blocks (drawn without
    replacement from blocks 0..nb-2) whose k_idx rows get +alpha*u_g, with
    u_g a seeded unit vector, and adds +alpha*u_g to q_idx[:, t, g] for every
    t at or after the block following g's first needle.  The additions are
    made in fp32 before the bf16 rounding.  The planted block ids are
    returned under "needle_blocks" ([G, needles] int64).
    """
    s = shape
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    f32 = {}
    for name, shp in (("q", (s.B, s.L, s.H, s.d)), ("k", (s.B, s.L, s.G, s.d)),
                      ("v", (s.B, s.L, s.G, s.d)), ("q_idx", (s.B, s.L, s.G, s.d_idx)),
                      ("k_idx", (s.B, s.L, s.d_idx))):
        f32[name] = torch.randn(shp, generator=gen, device=device, dtype=torch.float32)
    out = {}
    if needles > 0:
        nb = (s.L + s.block - 1) // s.block
        cpu = torch.Generator().manual_seed(seed + 1_000_003)
        u = torch.randn((s.G, s.d_idx), generator=cpu, dtype=torch.float32)
        u = u / u.norm(dim=1, keepdim=True)
        blocks = torch.stack([torch.randperm(nb - 1, generator=cpu)[:needles] for _ in range(s.G)])
        for g in range(s.G):
            ug = (needle_alpha * u[g]).to(device)
            for j in blocks[g].tolist():
                f32["k_idx"][:, j * s.block:(j + 1) * s.block, :] += ug
            first = int(blocks[g].min())
            f32["q_idx"][:, (first + 1) * s.block:, g, :] += ug
        out["needle_blocks"] = blocks.to(torch.int64)
        out["needle_u"] = u
    for name, x in f32.items():
        out[name] = x.to(BF16)
    del f32
    return out


def output_grad(shape: PrefillShape, seed: int, device="cpu") -> torch.Tensor:
    """Gradient arriving at the attention output, dout [B,L,H,d]: i.i.d.
    N(0,1) sampled in fp32 and rounded to bf16, from its own seed stream
    (seed + 3_000_017) so the forward inputs of the same seed are unchanged."""
    s = shape
    gen = torch.Generator(device=device)
    gen.manual_seed(seed + 3_000_017)
    return _normal_bf16(gen, (s.B, s.L, s.H, s.d), device)


def decode_lengths(shape: DecodeShape, seed: int) -> torch.Tensor:
    """Ragged cache lengths, uniform integers in [len_lo, len_hi] (CPU int32)."""
    s = shape
    cpu = torch.Generator().manual_seed(seed + 2_000_003)
    if s.len_lo == s.len_hi:
        return torch.full((s.B,), s.len_hi, dtype=torch.int32)
    return torch.randint(s.len_lo, s.len_hi + 1, (s.B,), generator=cpu, dtype=torch.int64).to(torch.int32)


def decode_inputs(shape: DecodeShape, seed: int, device="cpu") -> dict:
    """q [B,H,d], q_idx [B,G,d_idx], k_cache/v_cache [B,Lmax,G,d],
    k_idx_cache [B,Lmax,d_idx] (bf16) and seq_lens [B] (int32, CPU).
    Cache rows past a sequence's length hold random data as well; the
    definition never reads them."""
    s = shape
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    out = {
        "q": _normal_bf16(gen, (s.B, s.H, s.d), device),
        "q_idx": _normal_bf16(gen, (s.B, s.G, s.d_idx), device),
        "k_cache": _normal_bf16(gen, (s.B, s.Lmax, s.G, s.d), device),
        "v_cache": _normal_bf16(gen, (s.B, s.Lmax, s.G, s.d), device),
        "k_idx_cache": _normal_bf16(gen, (s.B, s.Lmax, s.d_idx), device),
    }
    out["seq_lens"] = decode_lengths(s, seed)
    return out


def fp8_index_cache(k_idx_cache: torch.Tensor) -> tuple:
    """An FP8 index-key cache holding the given bf16 cache [B,Lmax,d_idx]:
    E4M3 codes (uint8, same shape) and one fp32 scale per token [B,Lmax]
    (fp8_rows of it)."""
    return fp8_rows(k_idx_cache)


def fp8_rows(t: torch.Tensor) -> tuple:
    """E4M3 codes of a bf16 tensor [..., D] with one fp32 scale per row
    [...]: scale = max|row| / 448, codes = the row divided by its scale,
    rounded to E4M3 by torch's float8_e4m3fn conversion.  (Input
    preparation: the method consumes codes and scales as given.)"""
    x = t.float()
    amax = x.abs().amax(dim=-1)
    scale = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
    codes = (x / scale[..., None]).to(torch.float8_e4m3fn).view(torch.uint8)
    return codes.contiguous(), scale.contiguous()


def small_integer_like(t: torch.Tensor, seed: int, lo: int = -4, hi: int = 4) -> torch.Tensor:
    """Same shape/dtype/device as t, integers drawn uniformly from [lo, hi].
    Dot products of such bf16 values are exact in fp32 and fp64 alike, which
    makes score ties exact on both sides."""
    gen = torch.Generator(device="cpu").manual_seed(seed)
    x = torch.randint(lo, hi + 1, tuple(t.shape), generator=gen, dtype=torch.int32)
    return x.to(t.dtype).to(t.device)


def prefill_inputs_small(B: int, L: int, H: int, G: int, d: int, d_idx: int,
                         seed: int, device="cpu") -> dict:
    """Small i.i.d. N(0,1) bf16 prefill problem of any shape."""
    return prefill_inputs(PrefillShape(B=B, L=L, H=H, G=G, d=d, d_idx=d_idx), seed, device)
