"""Plain fp64 CPU oracle for MiniMax Sparse Attention (MSA) prefill and decode.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library and
its Python binding) imports or calls this module; only the tests, the smoke
entry point and the benchmark's CPU-baseline leg do.  It shares no code with
the CUDA path.

Sources (cited by page title / address and section):

* [P2] "MiniMax M3 sparse attention" explainer, mlqm.cn/news/533796:
  §2.1 (Index Branch: one index query per GQA group, one shared single-head
  index key, score = Q_idx . K_idx^T, block max pooling, top-k block choice),
  §2.2 (sparse branch: gather the selected K/V blocks and run ordinary
  attention; all query heads of one GQA group share one top-k choice),
  §4.1 (decode: one new query scores the cache and attends to its blocks).
* [P4] "MiniMax Sparse Attention:百万上下文稀疏注意力" (researchpapers.dev),
  section "机制" (the index scores visible KV tokens, pools them to block
  level, keeps top-k blocks per query and group and always keeps the most
  recent local block; the main branch does exact softmax attention on the
  selected blocks) and section "2048 个 KV token 是真正压力测试" (budget of
  16 blocks x 128 tokens per query group).
* [P3] "揭秘MiniMax闪电注意力机制", §1: textbook softmax attention, the
  quadratic baseline that sparse attention avoids.
* [P1] the long-context engineering essay (the FP8-KV paragraphs): low-
  precision (FP8) cache storage as the direction to pursue, with error
  control as its concern.  The FP8 cache format itself is the OCP 8-bit
  floating point E4M3 encoding; its definition, not the pages, fixes
  e4m3_to_f64.
* Training paragraph of [P4] "机制": the index branch learns from a KL loss
  against the main branch on the selected blocks, and the index path's
  gradient into the main attention is cut.  The main branch's backward pass
  is therefore the gradient of its exact attention over the selected tokens
  with the selection held fixed (prefill_backward).
* [P2] §3.1 (comparison with DeepSeek NSA): NSA runs three parallel
  branches -- compression, selection and a sliding window -- mixed by a
  learned gate, where MSA keeps the selection branch alone.  The NSA-style
  variant here (nsa_branches, nsa_forward) adds the other two branches to
  MSA's selection.  The page names them without formulas; the readings
  taken are listed below.

Readings taken where the pages are silent (each is also listed in the
design notes):

* index score = raw dot product q_idx . k_idx (no scale, no activation);
* main-branch scale = 1/sqrt(d) unless the caller passes one;
* top_k counts the forced local block (16 blocks = 2048 tokens);
* ties between equal block scores go to the lower block id;
* with no more than top_k visible blocks, every visible block is selected;
* the local block is attended only up to the query itself (s <= t);
* selections are stored sorted ascending and padded with -1;
* NSA-style variant: the sliding window of a query t is its `window` most
  recent tokens, s in [t-window+1, t]; the compression branch summarises
  block c by the mean of its keys and of its values (no learned weights
  exist here), and a query attends the summaries of the blocks whose every
  token is at or before it; a branch with no visible token contributes 0;
  the gate is given per (query, head, branch) by the caller, and the output
  is the gate-weighted sum of the three branch outputs.

Every function here is pinned by a CPU test (tests/test_oracle_pins.py)
against a closed form, a library routine, brute force or an invariant.

Layouts (row-major): q [B,L,H,d]; k, v [B,L,G,d]; q_idx [B,L,G,d_idx];
k_idx [B,L,d_idx]; sel [B,G,L,top_k] int32; out [B,L,H,d]; lse [B,L,H].
Query head h belongs to group h // (H // G).
"""
from __future__ import annotations

import math
from typing import Iterable, Optional, Sequence

import numpy as np

__all__ = [
    "as_f64",
    "e4m3_to_f64",
    "dequant_rows",
    "token_index_scores",
    "block_scores_row",
    "select_blocks_row",
    "selected_tokens",
    "attend_rows",
    "prefill",
    "decode",
    "block_scores_all",
    "attend_rows_grad",
    "prefill_backward",
    "window_tokens",
    "compress_kv",
    "compressed_tokens",
    "attend_rows_or_zero",
    "nsa_branches",
    "nsa_forward",
]


def e4m3_to_f64(codes) -> np.ndarray:
    """Value of 8-bit E4M3 floating-point codes (OCP FP8 E4M3, the 'fn'
    variant): bit 7 sign, bits 6..3 exponent e (bias 7), bits 2..0 mantissa m.
    e = 0: subnormal, (m / 8) * 2^-6; e = 1..15: (1 + m / 8) * 2^(e - 7),
    except e = 15, m = 7, which is NaN (the format has no infinities).  The
    largest finite magnitude is 1.75 * 2^8 = 448."""
    c = np.asarray(codes).astype(np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, (m / 8.0) * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return sign * mag


def dequant_rows(codes, scale) -> np.ndarray:
    """Rows of E4M3 codes [..., D] with one scale per row [...]: the stored
    row is scale * e4m3_to_f64(codes)."""
    return e4m3_to_f64(codes) * np.asarray(scale, dtype=np.float64)[..., None]


def as_f64(x) -> np.ndarray:
    """Exact upcast of a bf16/fp32 torch tensor or array to numpy fp64."""
    try:
        import torch  # local import: the oracle also works on plain arrays

        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


# ---------------------------------------------------------------------------
# Index Branch  ([P2] §2.1, [P4] "机制")
# ---------------------------------------------------------------------------

def token_index_scores(q_idx_row: np.ndarray, k_idx_prefix: np.ndarray) -> np.ndarray:
    """Index score of one (query, group) against every visible token.

    [P2] §2.1: the score is the plain product Q_idx . K_idx^T, with one index
    query per GQA group and one shared index-key head.  `k_idx_prefix` holds
    the index keys of tokens 0..t (the visible ones, s <= t).
    """
    return k_idx_prefix @ q_idx_row


def block_scores_row(q_idx_row: np.ndarray, k_idx: np.ndarray, t: int, block: int) -> np.ndarray:
    """Block score of every block that holds a visible token, for query t.

    [P2] §2.1 "Block Max Pooling": a block's score is the maximum of the token
    scores inside it.  Only tokens s <= t are visible ([P4] "机制": the index
    scores *visible* KV tokens), so the query's own block b_t = t // block is
    pooled over its first (t mod block) + 1 tokens.  Returns an array of
    length b_t + 1.
    """
    s = token_index_scores(q_idx_row, k_idx[: t + 1])
    nblk = t // block + 1
    out = np.empty(nblk, dtype=np.float64)
    for j in range(nblk):
        out[j] = np.max(s[j * block: min((j + 1) * block, t + 1)])
    return out


def select_blocks_row(bscores: np.ndarray, t: int, block: int, top_k: int) -> list[int]:
    """Top-k block choice for one (query, group), local block forced in.

    [P4] "机制": keep the top-k blocks and always keep the most recent local
    block; [P4] "2048 个 KV token": the budget of 16 blocks counts every block
    attended, so the local block takes one of the top_k places and the other
    top_k - 1 come from the strictly earlier blocks, highest score first.
    Equal scores go to the lower block id.  With b_t + 1 <= top_k every
    visible block is kept.  Returned sorted ascending (length min(top_k, b_t+1)).
    """
    bt = t // block
    if bt + 1 <= top_k:
        return list(range(bt + 1))
    candidates = sorted(range(bt), key=lambda j: (-bscores[j], j))
    return sorted(candidates[: top_k - 1] + [bt])


def selected_tokens(blocks: Iterable[int], t: int, block: int) -> np.ndarray:
    """Token ids a query at position t attends to, given its selected blocks.

    [P2] §2.2: the sparse branch gathers the K/V of the selected blocks; the
    attention stays causal, so only tokens s <= t are kept (this only trims
    the local block, every other selected block is entirely before t).
    """
    ids = []
    for j in blocks:
        if j < 0:
            continue
        lo, hi = j * block, min((j + 1) * block, t + 1)
        ids.extend(range(lo, hi))
    return np.asarray(sorted(ids), dtype=np.int64)


# ---------------------------------------------------------------------------
# Main Branch  ([P2] §2.2, [P3] §1)
# ---------------------------------------------------------------------------

def attend_rows(q_rows: np.ndarray, k_tok: np.ndarray, v_tok: np.ndarray, scale: float):
    """Exact softmax attention of r query rows over one gathered token set.

    [P3] §1 / [P2] §2.2: o = softmax(q k^T * scale) v over the gathered
    tokens.  Max-subtracted fp64 softmax.  Returns (o [r,d], lse [r],
    P [r,n]) where lse = log sum_s exp(scale * q.k_s).
    """
    logits = (q_rows @ k_tok.T) * scale  # [r, n]
    m = logits.max(axis=1, keepdims=True)
    e = np.exp(logits - m)
    z = e.sum(axis=1, keepdims=True)
    p = e / z
    o = p @ v_tok
    lse = (m + np.log(z))[:, 0]
    return o, lse, p


def _scale_of(d: int, scale: Optional[float]) -> float:
    return (1.0 / math.sqrt(d)) if (scale is None or scale == 0.0) else float(scale)


def block_scores_all(q_idx, k_idx, block: int) -> np.ndarray:
    """Block scores for every (b, g, t, j) of a small problem, -inf where block
    j holds no visible token (j > t // block).  Shape [B, G, L, nb]."""
    q_idx = as_f64(q_idx)
    k_idx = as_f64(k_idx)
    B, L, G, _ = q_idx.shape
    nb = (L + block - 1) // block
    out = np.full((B, G, L, nb), -np.inf)
    for b in range(B):
        for g in range(G):
            for t in range(L):
                bs = block_scores_row(q_idx[b, t, g], k_idx[b], t, block)
                out[b, g, t, : bs.shape[0]] = bs
    return out


def prefill(q, k, v, q_idx, k_idx, top_k: int, block: int = 128,
            scale: Optional[float] = None, rows: Optional[Sequence[tuple]] = None,
            sel_override: Optional[np.ndarray] = None, want_probs: bool = False):
    """MSA prefill for a batch of sequences.

    For every query t and group g: block scores ([P2] §2.1), top-k + forced
    local block ([P4] "机制"), then, for every query head of the group
    (shared selection, [P2] §2.2), exact causal softmax attention over the
    tokens of the selected blocks.

    rows: optional list of (b, t) pairs to evaluate (all rows when None).
    sel_override: optional [B,G,L,top_k] selection to attend with instead of
      the oracle's own (used to score an output against a given selection).
    Returns dict with
      sel [B,G,L,top_k] int32 (-1 padded; rows not evaluated stay -1),
      out [B,L,H,d] fp64 and lse [B,L,H] fp64 (NaN for rows not evaluated),
      probs {(b,t,h): P row} when want_probs.
    """
    q, k, v = as_f64(q), as_f64(k), as_f64(v)
    q_idx, k_idx = as_f64(q_idx), as_f64(k_idx)
    B, L, H, d = q.shape
    G = k.shape[2]
    r = H // G
    sc = _scale_of(d, scale)
    if rows is None:
        rows = [(b, t) for b in range(B) for t in range(L)]
    sel = np.full((B, G, L, top_k), -1, dtype=np.int32)
    out = np.full((B, L, H, d), np.nan)
    lse = np.full((B, L, H), np.nan)
    probs = {}
    for (b, t) in rows:
        for g in range(G):
            if sel_override is not None:
                blocks = [int(x) for x in sel_override[b, g, t] if x >= 0]
            else:
                bs = block_scores_row(q_idx[b, t, g], k_idx[b], t, block)
                blocks = select_blocks_row(bs, t, block, top_k)
            sel[b, g, t, : len(blocks)] = sorted(blocks)
            tok = selected_tokens(blocks, t, block)
            heads = list(range(g * r, (g + 1) * r))
            o, l_, p = attend_rows(q[b, t, heads], k[b, tok, g], v[b, tok, g], sc)
            out[b, t, heads] = o
            lse[b, t, heads] = l_
            if want_probs:
                for i, h in enumerate(heads):
                    probs[(b, t, h)] = p[i]
    res = {"sel": sel, "out": out, "lse": lse}
    if want_probs:
        res["probs"] = probs
    return res


def decode(q, q_idx, k_cache, v_cache, k_idx_cache, seq_lens, top_k: int,
           block: int = 128, scale: Optional[float] = None,
           sel_override: Optional[np.ndarray] = None):
    """MSA decode step: one new query per sequence at position n_b - 1.

    [P2] §4.1: each generated token only interacts with its selected KV
    blocks.  The caller has already appended the new token's k, v and k_idx,
    so sequence b holds n_b = seq_lens[b] cached tokens and the query sits at
    t = n_b - 1.  The selection and attention are the prefill definitions at
    that single position.

    Shapes: q [B,H,d], q_idx [B,G,d_idx], k_cache/v_cache [B,Lmax,G,d],
    k_idx_cache [B,Lmax,d_idx].  Returns dict(out [B,H,d], lse [B,H],
    sel [B,G,top_k]).
    """
    q, q_idx = as_f64(q), as_f64(q_idx)
    k_cache, v_cache, k_idx_cache = as_f64(k_cache), as_f64(v_cache), as_f64(k_idx_cache)
    seq_lens = np.asarray(seq_lens, dtype=np.int64)
    B, H, d = q.shape
    G = k_cache.shape[2]
    r = H // G
    sc = _scale_of(d, scale)
    sel = np.full((B, G, top_k), -1, dtype=np.int32)
    out = np.empty((B, H, d))
    lse = np.empty((B, H))
    for b in range(B):
        t = int(seq_lens[b]) - 1
        for g in range(G):
            if sel_override is not None:
                blocks = [int(x) for x in sel_override[b, g] if x >= 0]
            else:
                bs = block_scores_row(q_idx[b, g], k_idx_cache[b], t, block)
                blocks = select_blocks_row(bs, t, block, top_k)
            sel[b, g, : len(blocks)] = sorted(blocks)
            tok = selected_tokens(blocks, t, block)
            heads = list(range(g * r, (g + 1) * r))
            o, l_, _ = attend_rows(q[b, heads], k_cache[b, tok, g], v_cache[b, tok, g], sc)
            out[b, heads] = o
            lse[b, heads] = l_
    return {"sel": sel, "out": out, "lse": lse}


# ---------------------------------------------------------------------------
# Main Branch backward  ([P4] "机制", training paragraph)
# ---------------------------------------------------------------------------

def attend_rows_grad(q_rows: np.ndarray, k_tok: np.ndarray, v_tok: np.ndarray,
                     do_rows: np.ndarray, scale: float):
    """Gradient of sum(do * o) for o = attend_rows(q_rows, k_tok, v_tok).

    With P the softmax probabilities and dP = do v^T, the softmax Jacobian
    gives dZ = P * (dP - rowsum(P * dP)) for the scaled logits Z, and
    rowsum(P * dP) = rowsum(do * o).  Then dq = scale dZ k, dk = scale dZ^T q
    and dv = P^T do.  Returns (dq [r,d], dk [n,d], dv [n,d]).
    """
    o, _, p = attend_rows(q_rows, k_tok, v_tok, scale)
    dp = do_rows @ v_tok.T
    delta = np.sum(do_rows * o, axis=1, keepdims=True)
    dz = p * (dp - delta)
    return scale * (dz @ k_tok), scale * (dz.T @ q_rows), p.T @ do_rows


def prefill_backward(q, k, v, sel, dout, block: int = 128, scale: Optional[float] = None):
    """Main-branch backward of MSA prefill for a given selection.

    The index path is detached from the main attention ([P4] "机制"), so the
    selection sel [B,G,L,top_k] is a constant here and only q, k and v get
    gradients: every (query, group) row contributes through the tokens of its
    selected blocks with s <= t (the same token set as prefill), and a key or
    value token sums the contributions of every row that attends to it.
    dout has the shape of the output [B,L,H,d].  Returns dict(dq [B,L,H,d],
    dk [B,L,G,d], dv [B,L,G,d]) in fp64.
    """
    q, k, v, dout = as_f64(q), as_f64(k), as_f64(v), as_f64(dout)
    sel = np.asarray(sel)
    B, L, H, d = q.shape
    G = k.shape[2]
    r = H // G
    sc = _scale_of(d, scale)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(B):
        for t in range(L):
            for g in range(G):
                blocks = [int(x) for x in sel[b, g, t] if x >= 0]
                tok = selected_tokens(blocks, t, block)
                if tok.size == 0:
                    continue
                heads = list(range(g * r, (g + 1) * r))
                gq, gk, gv = attend_rows_grad(q[b, t, heads], k[b, tok, g], v[b, tok, g],
                                              dout[b, t, heads], sc)
                dq[b, t, heads] = gq
                np.add.at(dk[b, :, g], tok, gk)
                np.add.at(dv[b, :, g], tok, gv)
    return {"dq": dq, "dk": dk, "dv": dv}


# ---------------------------------------------------------------------------
# NSA-style variant: compression and sliding-window branches  ([P2] §3.1)
# ---------------------------------------------------------------------------

def window_tokens(t: int, window: int) -> np.ndarray:
    """Tokens the sliding-window branch attends for a query at position t:
    its `window` most recent positions, s in [t-window+1, t] (clipped at 0)."""
    return np.arange(max(0, t - window + 1), t + 1, dtype=np.int64)


def compress_kv(k, v, block: int):
    """Keys and values of the compression branch: compressed token c stands
    for block c and is the mean of the block's keys (values).  k, v
    [B,L,G,d] -> (k_cmp, v_cmp) [B,nb,G,d] fp64, nb = ceil(L/block); a
    partial last block averages the tokens it has."""
    k, v = as_f64(k), as_f64(v)
    B, L, G, d = k.shape
    nb = (L + block - 1) // block
    k_cmp = np.zeros((B, nb, G, d))
    v_cmp = np.zeros((B, nb, G, d))
    for c in range(nb):
        lo, hi = c * block, min((c + 1) * block, L)
        k_cmp[:, c] = k[:, lo:hi].sum(axis=1) / (hi - lo)
        v_cmp[:, c] = v[:, lo:hi].sum(axis=1) / (hi - lo)
    return k_cmp, v_cmp


def compressed_tokens(t: int, block: int) -> np.ndarray:
    """Compressed tokens a query at position t may attend: those of the blocks
    whose every token is at or before t, i.e. c <= (t + 1) // block - 1."""
    return np.arange((t + 1) // block, dtype=np.int64)


def attend_rows_or_zero(q_rows: np.ndarray, k_tok: np.ndarray, v_tok: np.ndarray, scale: float):
    """attend_rows, except that an empty token set gives a zero output and an
    lse of -inf (a branch with nothing to attend contributes nothing)."""
    if k_tok.shape[0] == 0:
        r = q_rows.shape[0]
        return np.zeros((r, v_tok.shape[-1])), np.full(r, -np.inf)
    o, lse, _ = attend_rows(q_rows, k_tok, v_tok, scale)
    return o, lse


def nsa_branches(q, k, v, sel, window: int, block: int = 128, scale: Optional[float] = None,
                 rows: Optional[Sequence[tuple]] = None):
    """The three branch outputs of the NSA-style variant, each an exact
    softmax attention of the query head over its own token set:
      cmp  compressed tokens compressed_tokens(t) of (k_cmp, v_cmp),
      slc  MSA's selection: the tokens s <= t of the blocks in sel[b, g, t],
      win  window_tokens(t, window) of (k, v).
    rows: optional (b, t) pairs to evaluate (all when None).  Returns dict of
    out_cmp, out_slc, out_win [B,L,H,d] and lse_cmp, lse_slc, lse_win
    [B,L,H] (NaN for rows not evaluated)."""
    q, k, v = as_f64(q), as_f64(k), as_f64(v)
    sel = np.asarray(sel)
    B, L, H, d = q.shape
    G = k.shape[2]
    r = H // G
    sc = _scale_of(d, scale)
    k_cmp, v_cmp = compress_kv(k, v, block)
    if rows is None:
        rows = [(b, t) for b in range(B) for t in range(L)]
    res = {}
    for name in ("cmp", "slc", "win"):
        res["out_" + name] = np.full((B, L, H, d), np.nan)
        res["lse_" + name] = np.full((B, L, H), np.nan)
    for (b, t) in rows:
        for g in range(G):
            heads = list(range(g * r, (g + 1) * r))
            qr = q[b, t, heads]
            c = compressed_tokens(t, block)
            s_tok = selected_tokens([int(x) for x in sel[b, g, t] if x >= 0], t, block)
            w_tok = window_tokens(t, window)
            for name, kk, vv in (("cmp", k_cmp[b, c, g], v_cmp[b, c, g]),
                                 ("slc", k[b, s_tok, g], v[b, s_tok, g]),
                                 ("win", k[b, w_tok, g], v[b, w_tok, g])):
                o, l_ = attend_rows_or_zero(qr, kk, vv, sc)
                res["out_" + name][b, t, heads] = o
                res["lse_" + name][b, t, heads] = l_
    return res


def nsa_forward(q, k, v, sel, gates, window: int, block: int = 128,
                scale: Optional[float] = None, rows: Optional[Sequence[tuple]] = None):
    """NSA-style output: o[t,h] = g_cmp o_cmp + g_slc o_slc + g_win o_win with
    gates [B,L,H,3] in the order (cmp, slc, win) given by the caller (the
    learned gate of [P2] §3.1 needs trained weights, which do not exist
    here).  Returns (out [B,L,H,d], branches dict of nsa_branches)."""
    br = nsa_branches(q, k, v, sel, window, block, scale, rows)
    g = np.asarray(gates, dtype=np.float64)
    out = (g[..., 0:1] * br["out_cmp"] + g[..., 1:2] * br["out_slc"]
           + g[..., 2:3] * br["out_win"])
    return out, br
