#!/usr/bin/env python
"""MSA (MiniMax Sparse Attention) benchmark on B200.

One step = one pass of the whole hot path over one batch of synthetic input:
  msa_index_select      index scores + block max-pool + fused top-k
  msa_sparse_attn_prefill  reverse index, gathered-query tcgen05 attention,
                        partial merge
  msa_sparse_attn_decode   decode step (index scan, top-k, split attention)
on the 1M-token workload: prefill B=1, L=1,048,576 plus a decode step of 4
sequences at 1,048,576 cached tokens; 32 query heads, 8 groups, d=128,
d_idx=128, block=128, top_k=16; i.i.d. N(0,1) bf16 inputs (seed 4).  The
decode-128K workload (32 sequences, lengths uniform in [65536, 131072]) is
timed alongside and reported under "decode_128k".

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

--impl reference times the fp64 CPU oracle (the only reference this method
has) on a bounded sample of the same workload per step.
Prints one JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

METRIC = "MSA prefill tokens/s & decode µs/step at 128K/1M; % of B200 roofline"
BLOCK = 128
SPEC_BF16_TFLOPS = 2250.0   # dense bf16 tensor peak of the part (spec sheet)
SPEC_HBM_GBS = 8000.0       # HBM3e bandwidth of the part (spec sheet)

# DRAM bytes (read + write) of one msa_index_kernel launch on the 1M-token
# workload, from one ncu capture (dram__bytes_read.sum + dram__bytes_write.sum,
# a single-pass metric set).  Keyed to the kernel source it was measured on:
# a changed kernel reports null.
INDEX_TRAFFIC_1M = {"bytes": 1.21216e11, "source_sha256_16": "2709ffa72db0ee6d"}


def index_traffic(workload: str):
    import hashlib
    src = os.path.join(ROOT, "block_sparse_long_08_b200", "csrc", "index_kernel.cu")
    try:
        h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    except OSError:
        return None
    if workload != "1m" or h != INDEX_TRAFFIC_1M["source_sha256_16"]:
        return None
    return INDEX_TRAFFIC_1M["bytes"]


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        clk = d.get("clocks_under_load", {}).get("sm_mhz_median")
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d["bf16_tflops_sustained"], "sm_mhz": clk,
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "sm_mhz": None, "source": "fallback"}


# --------------------------------------------------------------------- work
def n_sel(t: np.ndarray, top_k: int, block: int = BLOCK) -> np.ndarray:
    """Tokens a query at position t attends to (selected blocks, s <= t)."""
    bt = t // block
    return block * (np.minimum(top_k, bt + 1) - 1) + (t % block) + 1


def prefill_index_flops(B, L, G, d_idx, top_k, block=BLOCK):
    """Index scores a prefill must compute: every row whose local block b_t
    is at least top_k scores the b_t * block keys of its earlier blocks."""
    bt = np.arange(L, dtype=np.int64) // block
    keys = float(np.where(bt >= top_k, bt * block, 0).sum())
    return B * G * 2.0 * d_idx * keys


def prefill_main_flops(B, L, H, d, top_k, block=BLOCK):
    t = np.arange(L, dtype=np.int64)
    return B * float(H) * 4.0 * d * float(n_sel(t, top_k, block).sum())


def prefill_attn_bytes(B, L, H, G, d, top_k, block=BLOCK):
    """Bytes the key-block-outer prefill attention must move: every selected
    (query, group, block) entry gathers its R = H/G q rows once and writes and
    reads back one bf16 partial row (+ fp32 lse) per head, and the merged
    output is written once.  K/V block reads (once per query chunk that
    selects the block) are not counted."""
    t = np.arange(L, dtype=np.int64)
    entries = B * G * float(np.minimum(top_k, t // block + 1).sum())
    r = H // G
    return entries * r * (d * 2 * 3 + 4 * 2) + B * float(L) * H * d * 2


def prefill_bwd_bytes(B, L, H, G, d, top_k):
    """Bytes the key-block-outer backward must move: every selected (query,
    group, block) entry gathers its R q rows and R do rows, reads R lse and
    D values, and writes and reads back R bf16 dq partial rows; K/V are read
    once per key block and dk/dv written once; D = do . o reads o and do,
    and dq is written once."""
    t = np.arange(L, dtype=np.int64)
    entries = B * G * float(np.minimum(top_k, t // BLOCK + 1).sum())
    r = H // G
    rows = B * float(L) * H * d * 2
    kv = B * float(L) * G * d * 2
    return entries * r * (d * 2 * 2 + d * 2 * 2 + 8) + 3 * rows + 4 * kv


def prefill_bwd_flops(B, L, H, d, top_k):
    """Five products per (query, head, attended token) of 2d flops each:
    S, dP, dV, dK, dQ."""
    t = np.arange(L, dtype=np.int64)
    return B * float(H) * 10.0 * d * float(n_sel(t, top_k).sum())


def decode_bytes(seq_lens, H, G, d, d_idx, top_k, fp8_index=False, fp8_kv=False, block=BLOCK):
    """Bytes a decode step must read: the index-key scan over every cached
    token (bf16, or E4M3 codes + one fp32 scale per token), the selected K/V
    tokens (bf16, or codes + one scale per token and head), and the small
    per-step tensors."""
    n = np.asarray(seq_lens, dtype=np.int64)
    t = n - 1
    kv = G * 2 * ((d + 4) if fp8_kv else d * 2) * n_sel(t, top_k, block)
    scan = n * (d_idx + 4) if fp8_index else n * d_idx * 2
    small = len(n) * (H * d * 2 * 2 + G * d_idx * 2)
    return float((kv + scan).sum() + small)


# --------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        # nvidia-smi numbers GPUs differently from a masked CUDA device list:
        # address the device by its UUID.
        try:
            self.gpu = "GPU-" + str(torch.cuda.get_device_properties(gpu_index).uuid)
        except Exception:
            self.gpu = str(gpu_index)
        self.lines = []
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            threading.Thread(target=self._read, daemon=True).start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# --------------------------------------------------------------------- dist
def dist_setup():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime

        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return ws, rank, local


def dist_max(x: float, ws: int) -> float:
    if ws == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def dist_barrier(ws: int):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


# --------------------------------------------------------------------- oracle leg
def _bits(t: torch.Tensor) -> np.ndarray:
    """Host copy of a bf16 tensor as its raw 16-bit patterns (numpy)."""
    return t.to("cpu").contiguous().view(torch.int16).numpy()


def _f64(bits: np.ndarray) -> np.ndarray:
    """Exact fp64 values of bf16 bit patterns (a bf16 value is the upper half
    of the fp32 with the same bits)."""
    return (bits.astype(np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


class OracleLeg:
    """Times the fp64 oracle, as it stands, on the host cores.

    Prefill work is timed per query position (every group and head of the
    position); decode work per whole sequence.  Host copies (bf16 K/V rows,
    the fp64 index keys) are made before any clock starts.  A prefill
    position's cost grows with t, so sampled positions are stratified: [0, L)
    is cut into n equal strata with one uniform position in each, and the
    whole prefill's oracle time is extrapolated as the sum over strata of the
    stratum's width times its position's time."""

    def __init__(self, x=None, dx=None, shape=None, dshape=None):
        self.x, self.dx, self.shape, self.dshape = x, dx, shape, dshape
        self._pre = None

    def _prefill_host(self):
        if self._pre is None:
            x, B = self.x, self.shape.B
            self._pre = [(_bits(x["k"][b]), _bits(x["v"][b]),
                          x["k_idx"][b].to("cpu").double().numpy()) for b in range(B)]
        return self._pre

    def prefill_positions(self, positions):
        """Oracle seconds of each (b, t) position (all groups and heads)."""
        import oracle.msa_oracle as O
        f64 = O.as_f64
        s = self.shape
        r = s.H // s.G
        sc = 1.0 / math.sqrt(s.d)
        host = self._prefill_host()
        pos = list(positions)
        q_rows = [self.x["q"][b, t].to("cpu") for (b, t) in pos]
        qi_rows = [self.x["q_idx"][b, t].to("cpu") for (b, t) in pos]
        times = []
        for n, (b, t) in enumerate(pos):
            k, v, k_idx64 = host[b]
            t0 = time.perf_counter()
            for g in range(s.G):
                bs = O.block_scores_row(f64(qi_rows[n][g]), k_idx64, t, s.block)
                blocks = O.select_blocks_row(bs, t, s.block, s.top_k)
                tok = O.selected_tokens(blocks, t, s.block)
                O.attend_rows(f64(q_rows[n][g * r:(g + 1) * r]), _f64(k[tok, g]), _f64(v[tok, g]),
                              sc)
            times.append(time.perf_counter() - t0)
        return times

    def nsa_positions(self, positions, window):
        """Oracle seconds of each (b, t) position of the NSA-style variant: the
        selection branch as in prefill_positions, the window branch and the
        compression branch (every group and head).  The compressed keys and
        values are made once, before the clock starts, and timed apart
        (returned second)."""
        import oracle.msa_oracle as O
        f64 = O.as_f64
        s = self.shape
        r = s.H // s.G
        sc = 1.0 / math.sqrt(s.d)
        host = self._prefill_host()
        t0 = time.perf_counter()
        cmp_kv = [O.compress_kv(_f64(k)[None], _f64(v)[None], s.block) for (k, v, _) in host]
        t_cmp = time.perf_counter() - t0
        pos = list(positions)
        q_rows = [self.x["q"][b, t].to("cpu") for (b, t) in pos]
        qi_rows = [self.x["q_idx"][b, t].to("cpu") for (b, t) in pos]
        times = []
        for n, (b, t) in enumerate(pos):
            k, v, k_idx64 = host[b]
            kc, vc = cmp_kv[b]
            t0 = time.perf_counter()
            c = O.compressed_tokens(t, s.block)
            w_tok = O.window_tokens(t, window)
            for g in range(s.G):
                qr = f64(q_rows[n][g * r:(g + 1) * r])
                bs = O.block_scores_row(f64(qi_rows[n][g]), k_idx64, t, s.block)
                tok = O.selected_tokens(O.select_blocks_row(bs, t, s.block, s.top_k), t, s.block)
                O.attend_rows(qr, _f64(k[tok, g]), _f64(v[tok, g]), sc)
                O.attend_rows(qr, _f64(k[w_tok, g]), _f64(v[w_tok, g]), sc)
                O.attend_rows_or_zero(qr, kc[0, c, g], vc[0, c, g], sc)
            times.append(time.perf_counter() - t0)
        return times, t_cmp

    def prefill_full(self):
        """(seconds, (query, group) rows) of the oracle over every position."""
        s = self.shape
        times = self.prefill_positions([(b, t) for b in range(s.B) for t in range(s.L)])
        return sum(times), s.B * s.L * s.G

    def prefill_stratified(self, rng, n_strata):
        """(sampled seconds, extrapolated whole-prefill seconds, sampled rows)."""
        s = self.shape
        pos, width = [], []
        for b in range(s.B):
            for i in range(n_strata):
                lo, hi = i * s.L // n_strata, (i + 1) * s.L // n_strata
                if hi > lo:
                    pos.append((b, int(rng.integers(lo, hi))))
                    width.append(hi - lo)
        times = self.prefill_positions(pos)
        return sum(times), sum(w * tm for w, tm in zip(width, times)), len(pos) * s.G

    def decode_sequences(self, seqs):
        """Oracle seconds of whole decode sequences (every group and head).
        One sequence's caches are on the host at a time."""
        import oracle.msa_oracle as O
        f64 = O.as_f64
        dx, s = self.dx, self.dshape
        r = s.H // s.G
        sc = 1.0 / math.sqrt(s.d)
        total = 0.0
        for b in seqs:
            n = int(dx["seq_lens"][b])
            q, qi = dx["q"][b].to("cpu"), dx["q_idx"][b].to("cpu")
            kc, vc = _bits(dx["k_cache"][b, :n]), _bits(dx["v_cache"][b, :n])
            ki64 = dx["k_idx_cache"][b, :n].to("cpu").double().numpy()
            t = n - 1
            t0 = time.perf_counter()
            for g in range(s.G):
                bs = O.block_scores_row(f64(qi[g]), ki64, t, s.block)
                blocks = O.select_blocks_row(bs, t, s.block, s.top_k)
                tok = O.selected_tokens(blocks, t, s.block)
                O.attend_rows(f64(q[g * r:(g + 1) * r]), _f64(kc[tok, g]), _f64(vc[tok, g]), sc)
            total += time.perf_counter() - t0
            del kc, vc, ki64
        return total

    def sample(self, rng, n_tok, n_dec):
        """Bounded sample of one step (the reference arm): n_tok stratified
        prefill positions and n_dec decode sequences.  Returns (sampled
        seconds, extrapolated seconds of the whole step)."""
        t_pre, est_pre, _ = self.prefill_stratified(rng, n_tok)
        bsel = sorted(rng.choice(self.dshape.B, size=n_dec, replace=False).tolist())
        t_dec = self.decode_sequences(bsel)
        return t_pre + t_dec, est_pre + t_dec * (self.dshape.B / n_dec)


# --------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the tiny / 32K / 128K-planted prefill legs")
    ap.add_argument("--workload", default="1m", choices=["1m", "512k", "128k", "32k", "8k"],
                    help="prefill length of the step (1m is the headline workload; 8k is a "
                         "small-footprint case for profiler captures, 512k the smallest "
                         "whose index keys (134 MB) exceed the 126 MB L2)")
    ap.add_argument("--op", default="step",
                    choices=["step", "index", "scores", "attn", "decode", "decode8", "cached",
                             "bwd", "nsa_window", "nsa_compressed"],
                    help="time one operation of the step alone (profiling runs; 'cached' runs "
                         "the whole prefill as 8 msa_forward_cached chunks against the caches); "
                         "prints its own short JSON line")
    ap.add_argument("--decode-batch", type=int, default=0,
                    help="override the decode batch (profiling runs on a smaller footprint)")
    args = ap.parse_args()
    ws_n, rank, local = dist_setup()

    from block_sparse_long_08_b200 import inputs as I

    if args.workload == "1m":
        shape, dshape, seed = I.PREFILL_1M, I.DECODE_1M, I.SEEDS["1m"]
    elif args.workload == "512k":
        import dataclasses
        shape, dshape, seed = (dataclasses.replace(I.PREFILL_1M, L=524288), I.DECODE_128K,
                               I.SEEDS["1m"])
    elif args.workload == "128k":
        shape, dshape, seed = I.PREFILL_128K_PLANTED, I.DECODE_128K, I.SEEDS["128k_planted"]
    elif args.workload == "32k":
        shape, dshape, seed = I.PREFILL_32K, I.DECODE_128K, I.SEEDS["32k"]
    else:
        import dataclasses
        shape, dshape, seed = (dataclasses.replace(I.PREFILL_32K, L=8192), I.DECODE_128K,
                               I.SEEDS["32k"])
    cfg = {"workload": f"MSA prefill B={shape.B} L={shape.L} + decode batch {dshape.B} at "
                       f"{'%d' % dshape.len_hi if dshape.len_lo == dshape.len_hi else 'U[%d,%d]' % (dshape.len_lo, dshape.len_hi)}",
           "B": shape.B, "L": shape.L, "H": shape.H, "G": shape.G, "d": shape.d,
           "d_idx": shape.d_idx, "block": shape.block, "top_k": shape.top_k,
           "decode_batch": dshape.B, "seed": seed,
           "l2": "inputs larger than L2 (126 MB) every step; no flush needed"}

    if args.decode_batch > 0:
        import dataclasses
        dshape = dataclasses.replace(dshape, B=args.decode_batch)
        cfg["decode_batch"] = dshape.B
    if args.impl == "reference":
        return run_reference(args, shape, dshape, seed, cfg, ws_n, rank)
    return run_ours(args, shape, dshape, seed, cfg, ws_n, rank, local)


def run_reference(args, shape, dshape, seed, cfg, ws_n, rank):
    if rank != 0:
        return
    from block_sparse_long_08_b200 import inputs as I
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    x = I.prefill_inputs(shape, seed, device=dev)
    dx = I.decode_inputs(dshape, seed, device=dev)
    leg = OracleLeg(x, dx, shape, dshape)
    rng = np.random.default_rng(seed)
    n_tok, n_dec = 4, 1
    ests = []
    for i in range(args.warmup + args.steps):
        _, est = leg.sample(rng, n_tok, n_dec)
        if i >= args.warmup:
            ests.append(est)
    step_s = statistics.mean(ests)
    tokens = shape.B * shape.L + dshape.B
    value = tokens / step_s
    cores = os.cpu_count()
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": step_s * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": cfg,
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": f"per step {n_tok} prefill query positions (all {shape.G} groups) "
                                       f"+ {n_dec} decode sequence, scaled to the full step"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_ours(args, shape, dshape, seed, cfg, ws_n, rank, local):
    from block_sparse_long_08_b200 import inputs as I
    from block_sparse_long_08_b200 import msa as M

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the product path has no CPU fallback)")
    dev = torch.device("cuda", local)
    M.lib()
    peaks = load_peaks()

    # ---- inputs (device-resident for the kernel-timed leg)
    need_pre = args.op in ("step", "index", "scores", "attn", "cached", "bwd", "nsa_window",
                           "nsa_compressed")
    need_dec = args.op in ("step", "decode", "decode8")
    if not need_pre:   # a decode-only profiling run keeps the footprint small
        import dataclasses
        shape = dataclasses.replace(shape, L=128)
    x = I.prefill_inputs(shape, seed, device=dev)
    if not need_dec:
        import dataclasses
        dshape = dataclasses.replace(dshape, B=1, Lmax=128, len_lo=128, len_hi=128)
    dx = I.decode_inputs(dshape, seed, device=dev)
    dx["seq_lens"] = dx["seq_lens"].to(dev)
    B, L, H, G, d, di, K = shape.B, shape.L, shape.H, shape.G, shape.d, shape.d_idx, shape.top_k
    p = M.make_params(B, L, H, G, d, di, BLOCK, K)
    pd = M.make_params(dshape.B, dshape.Lmax, dshape.H, dshape.G, dshape.d, dshape.d_idx, BLOCK, dshape.top_k)
    ws_idx = M.new_workspace(p, M.MSA_OP_INDEX_SELECT, dev)
    ws_att = M.new_workspace(p, M.MSA_OP_PREFILL_ATTN, dev)
    ws_dec = M.new_workspace(pd, M.MSA_OP_DECODE, dev)
    sel = torch.empty((B, G, L, K), dtype=torch.int32, device=dev)
    out = torch.empty_like(x["q"])
    dout = torch.empty_like(dx["q"])
    stream = torch.cuda.current_stream()

    def step(ev=None):
        if ev:
            ev[0].record(stream)
        M.msa_index_select(x["q_idx"], x["k_idx"], K, sel=sel, ws=ws_idx)
        if ev:
            ev[1].record(stream)
        M.msa_sparse_attn_prefill(x["q"], x["k"], x["v"], sel, out=out, ws=ws_att)
        if ev:
            ev[2].record(stream)
        M.msa_sparse_attn_decode(dx["q"], dx["q_idx"], dx["k_cache"], dx["v_cache"], dx["k_idx_cache"],
                                 dx["seq_lens"], dshape.top_k, out=dout, ws=ws_dec)
        if ev:
            ev[3].record(stream)

    if args.op != "step":
        return run_single_op(args, M, x, dx, dshape, K, sel, out, dout, ws_idx, ws_att, ws_dec, stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    for w in (ws_idx, ws_att, ws_dec):
        rc = M.msa_read_status(w)
        if rc != 0:
            raise SystemExit(f"device status {rc} after warm-up")
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    dist_barrier(ws_n)
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for i in range(args.steps):
        step(evs[i])
    t_end.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    dist_barrier(ws_n)
    total_ms = t_start.elapsed_time(t_end)
    total_ms = dist_max(total_ms, ws_n)
    idx_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    att_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    dec_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in evs)
    ms_per_step = total_ms / args.steps
    tokens_per_step = B * L + dshape.B
    value = ws_n * tokens_per_step / (ms_per_step / 1e3)

    # ---- rooflines
    f_idx = prefill_index_flops(B, L, G, di, K)
    f_main = prefill_main_flops(B, L, H, d, K)
    seq_lens_host = dx["seq_lens"].cpu().numpy()
    dbytes = decode_bytes(seq_lens_host, dshape.H, dshape.G, dshape.d, dshape.d_idx, dshape.top_k)
    peak_t = peaks["bf16_tflops_sustained"]
    roof_idx = {"bound": "tensor", "achieved": f_idx / (idx_ms / 1e3) / 1e12, "peak": peak_t,
                "unit": "TFLOP/s", "frac": None, "traffic": index_traffic(args.workload),
                "kernel": "msa_index_kernel", "peak_kind": f"bf16 sustained ({peaks['source']})"}
    roof_idx["frac"] = roof_idx["achieved"] / peak_t
    # The sustained peak was measured at a power-capped median clock; the
    # index kernel runs at its own power-capped clock.  Secondary fractions:
    # against the measured peak scaled to the clock sampled during this run,
    # and against the 2.25 PFLOP/s dense bf16 spec.
    if clk.get("sm_mhz") and peaks.get("sm_mhz"):
        scaled = peak_t * clk["sm_mhz"] / peaks["sm_mhz"]
        roof_idx["peak_clock_scaled"] = scaled
        roof_idx["frac_clock_scaled"] = roof_idx["achieved"] / scaled
    roof_idx["frac_of_spec"] = roof_idx["achieved"] / SPEC_BF16_TFLOPS
    b_att = prefill_attn_bytes(B, L, H, G, d, K)
    roof_att = {"bound": "hbm", "achieved": b_att / (att_ms / 1e3) / 1e9, "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "bytes": b_att,
                "tflops": f_main / (att_ms / 1e3) / 1e12}
    roof_att["frac"] = roof_att["achieved"] / peaks["hbm_gbs"]
    roof_dec = {"bound": "hbm", "achieved": dbytes / (dec_ms / 1e3) / 1e9, "peak": peaks["hbm_gbs"],
                "unit": "GB/s"}
    roof_dec["frac"] = roof_dec["achieved"] / peaks["hbm_gbs"]

    nchunks = math.ceil(L / M.msa_prefill_chunk_len(p))
    launches_per_step = 1 + 5 * nchunks + 3   # index; per chunk 3 reverse-index + attention + merge; decode 3
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws_n,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "config": cfg, "roofline": roof_idx,
            "breakdown": {"index_ms": idx_ms, "prefill_attn_ms": att_ms, "decode_us": dec_ms * 1e3,
                          "prefill_tokens_per_s": B * L / ((idx_ms + att_ms) / 1e3),
                          "index_flops": f_idx, "main_flops": f_main, "decode_bytes": dbytes,
                          "prefill_attn_roofline": roof_att, "decode_roofline": roof_dec},
            "gpu_launches": launches_per_step * args.steps, "clocks": clk}

    # ---- decode at 128K (the decode workload of the pages' 128K setting)
    if args.workload == "1m" and rank == 0 or args.workload != "1m":
        line["decode_128k"] = bench_decode_128k(M, I, dev, args, peaks)

    # ---- main-branch backward at 32K
    if args.workload == "1m" and rank == 0 or args.workload != "1m":
        line["backward_32k"] = bench_backward_32k(M, I, dev, args, peaks)

    # ---- end to end through the public API with host buffers (the timed
    # leg's workspace and outputs are released first)
    del ws_att, sel, out
    torch.cuda.empty_cache()
    if not args.no_e2e:
        line["e2e"] = bench_e2e(M, x, dx, shape, dshape, K, args, ws_n, stream)

    # ---- every configuration at 1 GPU: the 1M step above, decode-128K, and
    # the tiny, 32K and 128K-planted prefills, each beside the oracle
    if rank == 0 and ws_n == 1 and not args.no_configs:
        line["per_config"] = bench_configs(M, I, dev, args, peaks, line)

    # ---- oracle on the host cores
    if not args.no_cpu_baseline and rank == 0 and ws_n == 1:
        leg = OracleLeg(x, dx, shape, dshape)
        rng = np.random.default_rng(seed)
        n_strata = 64
        t_pre, est_pre, rows = leg.prefill_stratified(rng, n_strata)
        t_dec = leg.decode_sequences(range(dshape.B))
        est = est_pre + t_dec
        line["cpu_baseline"] = {
            "value": tokens_per_step / est, "unit": "tokens/s", "cores": oracle_threads(),
            "kind": "oracle", "extrapolated": True, "seconds_per_step": est,
            "sample": f"prefill: {rows} (query, group) rows, one uniform position in each of "
                      f"{n_strata} equal strata of [0,L) with all {G} groups and {H} heads, "
                      f"{t_pre:.1f} s, extrapolated to the whole prefill by stratum width; "
                      f"decode: all {dshape.B} sequences in full, {t_dec:.1f} s"}
        if "per_config" in line:
            line["per_config"]["1m"]["oracle"] = line["cpu_baseline"]
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws_n > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_single_op(args, M, x, dx, dshape, K, sel, out, dout, ws_idx, ws_att, ws_dec, stream):
    """One operation alone, W untimed + K timed launches (profiling aid)."""
    M.msa_index_select(x["q_idx"], x["k_idx"], K, sel=sel, ws=ws_idx)  # the attention op needs sel

    if args.op == "decode8":
        from block_sparse_long_08_b200 import inputs as I
        codes8, scale8 = I.fp8_index_cache(dx["k_idx_cache"])
    L = x["q"].shape[1]
    n_c = L // 8
    qc = [(x["q"][:, t0:t0 + n_c].contiguous(), x["q_idx"][:, t0:t0 + n_c].contiguous())
          for t0 in range(0, L, n_c)] if args.op == "cached" else []
    outc = torch.empty_like(qc[0][0]) if qc else None
    ws_c = None
    if qc:
        pc = M.make_params(x["q"].shape[0], L, x["q"].shape[2], x["k"].shape[2], 128,
                           x["q_idx"].shape[3], 128, K)
        ws_c = M.new_workspace(pc, M.MSA_OP_FORWARD, x["q"].device)

    if args.op == "bwd":
        from block_sparse_long_08_b200 import inputs as I
        Bq, Lq, Hq, dq_ = x["q"].shape
        sh_b = I.PrefillShape(B=Bq, L=Lq, H=Hq, G=x["k"].shape[2], d=dq_, d_idx=x["q_idx"].shape[3],
                              top_k=K)
        dout_b = I.output_grad(sh_b, 0, device=x["q"].device)
        out, lse_b = M.msa_sparse_attn_prefill(x["q"], x["k"], x["v"], sel, want_lse=True)
        ws_b = M.new_workspace(M.make_params(Bq, Lq, Hq, sh_b.G, dq_, sh_b.d_idx, 128, K),
                               M.MSA_OP_BACKWARD, x["q"].device)

    if args.op in ("nsa_window", "nsa_compressed"):   # NSA-style branch kernels (window 512)
        Bq, Lq, Hq, dq_ = x["q"].shape
        p_n = M.make_params(Bq, Lq, Hq, x["k"].shape[2], dq_, x["q_idx"].shape[3], 128, K)
        ws_nsa = M.new_workspace(p_n, M.MSA_OP_NSA_BRANCH, x["q"].device)
        kc, vc = M.msa_nsa_compress_kv(x["k"], x["v"])

    def op():
        if args.op == "nsa_window":
            M.msa_nsa_window_attn(x["q"], x["k"], x["v"], 512, out=out, ws=ws_nsa)
        elif args.op == "nsa_compressed":
            M.msa_nsa_compressed_attn(x["q"], kc, vc, out=out, ws=ws_nsa)
        elif args.op == "cached":   # the prefill as the serving form: 8 chunks against the caches
            for c, (q, q_idx) in enumerate(qc):
                M.msa_forward_cached(q, q_idx, x["k"], x["v"], x["k_idx"], c * n_c, K, out=outc,
                                     ws=ws_c)
        elif args.op == "index":
            M.msa_index_select(x["q_idx"], x["k_idx"], K, sel=sel, ws=ws_idx)
        elif args.op == "scores":   # stored block scores + the standalone top-k kernel
            M.msa_index_select(x["q_idx"], x["k_idx"], K, sel=sel, ws=ws_idx, block_scores=True)
        elif args.op == "attn":
            M.msa_sparse_attn_prefill(x["q"], x["k"], x["v"], sel, out=out, ws=ws_att)
        elif args.op == "bwd":
            M.msa_sparse_attn_backward(x["q"], x["k"], x["v"], out, lse_b, dout_b, sel, ws=ws_b)
        elif args.op == "decode8":   # FP8 index-key cache
            M.msa_sparse_attn_decode_fp8idx(dx["q"], dx["q_idx"], dx["k_cache"], dx["v_cache"],
                                            codes8, scale8, dx["seq_lens"], dshape.top_k,
                                            out=dout, ws=ws_dec)
        else:
            M.msa_sparse_attn_decode(dx["q"], dx["q_idx"], dx["k_cache"], dx["v_cache"],
                                     dx["k_idx_cache"], dx["seq_lens"], dshape.top_k, out=dout, ws=ws_dec)

    for _ in range(args.warmup):
        op()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(args.steps):
        op()
    b.record(stream)
    torch.cuda.synchronize()
    extra = ((ws_c,) if ws_c is not None else ()) + ((ws_b,) if args.op == "bwd" else ()) \
        + ((ws_nsa,) if args.op in ("nsa_window", "nsa_compressed") else ())
    for w in (ws_idx, ws_att, ws_dec) + extra:
        if M.msa_read_status(w) != 0:
            raise SystemExit("device status error")
    ms = a.elapsed_time(b) / args.steps
    line = {"op": args.op, "workload": args.workload, "ms_per_launch": ms}
    if args.op == "cached":
        line["tokens_per_s"] = L * x["q"].shape[0] / (ms / 1e3)
        line["chunks"] = len(qc)
    print(json.dumps(line), flush=True)


def bench_decode_128k(M, I, dev, args, peaks):
    ds = I.DECODE_128K
    y = I.decode_inputs(ds, I.SEEDS["decode_128k"], device=dev)
    seq = y["seq_lens"].to(dev)
    pd = M.make_params(ds.B, ds.Lmax, ds.H, ds.G, ds.d, ds.d_idx, BLOCK, ds.top_k)
    ws = M.new_workspace(pd, M.MSA_OP_DECODE, dev)
    out = torch.empty_like(y["q"])
    stream = torch.cuda.current_stream()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    codes, kscale = I.fp8_index_cache(y["k_idx_cache"])   # the same caches stored in FP8
    k8, ks8 = I.fp8_rows(y["k_cache"])
    v8, vs8 = I.fp8_rows(y["v_cache"])

    def run():
        M.msa_sparse_attn_decode(y["q"], y["q_idx"], y["k_cache"], y["v_cache"], y["k_idx_cache"], seq,
                                 ds.top_k, out=out, ws=ws)

    def run_fp8():
        M.msa_sparse_attn_decode_fp8idx(y["q"], y["q_idx"], y["k_cache"], y["v_cache"], codes,
                                        kscale, seq, ds.top_k, out=out, ws=ws)

    def run_all_fp8():
        M.msa_sparse_attn_decode_fp8(y["q"], y["q_idx"], k8, ks8, v8, vs8, codes, kscale, seq,
                                     ds.top_k, out=out, ws=ws)

    def timed(fn):
        for _ in range(max(3, args.warmup)):
            fn()
        torch.cuda.synchronize()
        if M.msa_read_status(ws) != 0:
            raise SystemExit("decode-128k device status error")
        times = []
        for _ in range(iters):
            flush.zero_()   # L2 flush (256 MB > 126 MB L2) outside the timed span
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            torch.cuda.synchronize()
            times.append(a.elapsed_time(b))
        return statistics.median(times) * 1e3

    def roof(byts, us):
        return {"bound": "hbm", "achieved": byts / (us / 1e6) / 1e9, "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": byts / (us / 1e6) / 1e9 / peaks["hbm_gbs"], "bytes": byts}

    iters = 20
    us = timed(run)
    us8 = timed(run_fp8)
    us88 = timed(run_all_fp8)
    lens = y["seq_lens"].numpy()
    oracle = None
    if not args.no_cpu_baseline:   # the full oracle: every sequence, every group and head
        del codes, kscale, k8, ks8, v8, vs8
        secs = OracleLeg(None, y, None, ds).decode_sequences(range(ds.B))
        oracle = {"seconds": secs, "us_per_step": secs * 1e6, "cores": oracle_threads(),
                  "kind": "oracle", "extrapolated": False,
                  "sample": f"all {ds.B} sequences, every group and head"}
        codes = kscale = k8 = ks8 = v8 = vs8 = None
    byts = decode_bytes(lens, ds.H, ds.G, ds.d, ds.d_idx, ds.top_k)
    byts8 = decode_bytes(lens, ds.H, ds.G, ds.d, ds.d_idx, ds.top_k, fp8_index=True)
    byts88 = decode_bytes(lens, ds.H, ds.G, ds.d, ds.d_idx, ds.top_k, fp8_index=True, fp8_kv=True)
    del y, codes, kscale, k8, ks8, v8, vs8
    return {"us_per_step": us, "iters": iters, "batch": ds.B,
            "seq_lens": f"U[{ds.len_lo},{ds.len_hi}] seed {I.SEEDS['decode_128k']}",
            "l2": "256 MB buffer written between iterations",
            "roofline": roof(byts, us),
            "fp8_index_cache": {"us_per_step": us8, "roofline": roof(byts8, us8),
                                "cache": "k_idx as E4M3 codes + fp32 scale per token"},
            "fp8_all_caches": {"us_per_step": us88, "roofline": roof(byts88, us88),
                               "cache": "k_idx, K and V as E4M3 codes + fp32 scales"},
            "gpu_launches": 9 * iters, "oracle": oracle}


def bench_backward_32k(M, I, dev, args, peaks):
    """Main-branch backward at the 32K prefill workload (seed of the 32K
    config), on the forward's own selection, output and lse."""
    sh = I.PREFILL_32K
    x = I.prefill_inputs(sh, I.SEEDS["32k"], device=dev)
    dout = I.output_grad(sh, I.SEEDS["32k"], device=dev)
    out, sel, lse = M.msa_forward(x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"], sh.top_k,
                                  want_sel=True, want_lse=True)
    p = M.make_params(sh.B, sh.L, sh.H, sh.G, sh.d, sh.d_idx, BLOCK, sh.top_k)
    ws = M.new_workspace(p, M.MSA_OP_BACKWARD, dev)
    dq, dk, dv = torch.empty_like(x["q"]), torch.empty_like(x["k"]), torch.empty_like(x["v"])
    stream = torch.cuda.current_stream()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def run():
        M.msa_sparse_attn_backward(x["q"], x["k"], x["v"], out, lse, dout, sel, dq=dq, dk=dk,
                                   dv=dv, ws=ws)

    for _ in range(max(3, args.warmup)):
        run()
    torch.cuda.synchronize()
    if M.msa_read_status(ws) != 0:
        raise SystemExit("backward device status error")
    iters = 10
    times = []
    for _ in range(iters):
        flush.zero_()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        run()
        b.record(stream)
        torch.cuda.synchronize()
        times.append(a.elapsed_time(b))
    ms = statistics.median(times)
    byts = prefill_bwd_bytes(sh.B, sh.L, sh.H, sh.G, sh.d, sh.top_k)
    fl = prefill_bwd_flops(sh.B, sh.L, sh.H, sh.d, sh.top_k)
    del x, dout, out, sel, lse, ws, dq, dk, dv
    return {"ms": ms, "iters": iters, "tokens_per_s": sh.B * sh.L / (ms / 1e3),
            "workload": f"B={sh.B} L={sh.L} H={sh.H} G={sh.G} d={sh.d} top_k={sh.top_k}",
            "roofline": {"bound": "hbm", "achieved": byts / (ms / 1e3) / 1e9,
                         "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": byts / (ms / 1e3) / 1e9 / peaks["hbm_gbs"], "bytes": byts},
            "tensor": {"flops": fl, "tflops": fl / (ms / 1e3) / 1e12,
                       "frac_of_sustained": fl / (ms / 1e3) / 1e12 / peaks["bf16_tflops_sustained"]},
            "gpu_launches": 6 * iters}


def oracle_threads() -> int:
    """Threads the oracle runs on: numpy's BLAS pool (matrix products) or
    torch's intra-op pool (row gathers), whichever is larger."""
    n = torch.get_num_threads()
    try:
        from threadpoolctl import threadpool_info
        n = max([n] + [int(i.get("num_threads", 1)) for i in threadpool_info()])
    except Exception:
        pass
    return int(n)


def needle_hit_rate(sel: torch.Tensor, needle_blocks: torch.Tensor):
    """Over every query t after group g's first needle block and every needle
    block j < t/128 of g: how often j is in sel[0, g, t].  sel [1,G,L,K]."""
    G, L = sel.shape[1], sel.shape[2]
    bt = torch.arange(L, device=sel.device) // BLOCK
    hit = tot = 0
    for g in range(G):
        js = needle_blocks[g].tolist()
        start = (min(js) + 1) * BLOCK
        rows, btg = sel[0, g, start:], bt[start:]
        for j in js:
            vis = btg > j
            tot += int(vis.sum())
            hit += int(((rows == j).any(-1) & vis).sum())
    return hit, tot


def bench_prefill_config(M, I, dev, args, peaks, name, shape, seed, needles=0,
                         oracle_full=False, n_strata=64, iters=10):
    """One prefill configuration at 1 GPU: msa_index_select (fused top-k) then
    msa_sparse_attn_prefill, as in the step, timed per launch with CUDA events
    and an L2 flush between iterations; rooflines of both ops; the oracle on
    the host cores beside it (every position, or stratified positions
    extrapolated to the whole prefill)."""
    x = I.prefill_inputs(shape, seed, device=dev, needles=needles, needle_alpha=3.0)
    B, L, H, G, d, di, K = shape.B, shape.L, shape.H, shape.G, shape.d, shape.d_idx, shape.top_k
    blk = shape.block
    p = M.make_params(B, L, H, G, d, di, blk, K)
    ws_idx = M.new_workspace(p, M.MSA_OP_INDEX_SELECT, dev)
    ws_att = M.new_workspace(p, M.MSA_OP_PREFILL_ATTN, dev)
    sel = torch.empty((B, G, L, K), dtype=torch.int32, device=dev)
    out = torch.empty_like(x["q"])
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    for _ in range(max(3, args.warmup)):
        M.msa_index_select(x["q_idx"], x["k_idx"], K, sel=sel, ws=ws_idx, block=blk)
        M.msa_sparse_attn_prefill(x["q"], x["k"], x["v"], sel, out=out, ws=ws_att, block=blk)
    torch.cuda.synchronize()
    if M.msa_read_status(ws_idx) != 0 or M.msa_read_status(ws_att) != 0:
        raise SystemExit(f"{name}: device status error")
    t_idx, t_att, t_pre = [], [], []
    for _ in range(iters):
        flush.zero_()   # L2 flush (256 MB > 126 MB L2) outside the timed span
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        ev[0].record(stream)
        M.msa_index_select(x["q_idx"], x["k_idx"], K, sel=sel, ws=ws_idx, block=blk)
        ev[1].record(stream)
        M.msa_sparse_attn_prefill(x["q"], x["k"], x["v"], sel, out=out, ws=ws_att, block=blk)
        ev[2].record(stream)
        torch.cuda.synchronize()
        t_idx.append(ev[0].elapsed_time(ev[1]))
        t_att.append(ev[1].elapsed_time(ev[2]))
        t_pre.append(ev[0].elapsed_time(ev[2]))
    idx_ms, att_ms, pre_ms = (statistics.median(v) for v in (t_idx, t_att, t_pre))
    f_idx = prefill_index_flops(B, L, G, di, K, blk)
    f_main = prefill_main_flops(B, L, H, d, K, blk)
    b_att = prefill_attn_bytes(B, L, H, G, d, K, blk)
    burst = peaks["bf16_tflops"]
    nchunks = math.ceil(B * L / M.msa_prefill_chunk_len(p))
    res = {"workload": f"B={B} L={L} H={H} G={G} d={d} d_idx={di} block={blk} top_k={K}"
                       + (f", {needles} planted needle blocks per group (alpha 3)" if needles else ""),
           "seed": seed, "iters": iters, "l2": "256 MB buffer written between iterations",
           "prefill_ms": pre_ms, "tokens_per_s": B * L / (pre_ms / 1e3),
           "index_ms": idx_ms, "attn_ms": att_ms,
           "prefill_tensor": {"flops": f_idx + f_main,
                              "tflops": (f_idx + f_main) / (pre_ms / 1e3) / 1e12,
                              "frac_of_burst": (f_idx + f_main) / (pre_ms / 1e3) / 1e12 / burst,
                              "frac_of_spec": (f_idx + f_main) / (pre_ms / 1e3) / 1e12
                              / SPEC_BF16_TFLOPS},
           "index_roofline": {"bound": "tensor", "achieved": f_idx / (idx_ms / 1e3) / 1e12,
                              "peak": burst, "unit": "TFLOP/s",
                              "frac": f_idx / (idx_ms / 1e3) / 1e12 / burst, "flops": f_idx,
                              "peak_kind": f"bf16 burst ({peaks['source']}): kernel timed alone"},
           "attn_roofline": {"bound": "hbm", "achieved": b_att / (att_ms / 1e3) / 1e9,
                             "peak": peaks["hbm_gbs"], "unit": "GB/s",
                             "frac": b_att / (att_ms / 1e3) / 1e9 / peaks["hbm_gbs"],
                             "bytes": b_att, "tflops": f_main / (att_ms / 1e3) / 1e12},
           "gpu_launches": (1 + 5 * nchunks) * iters}
    if needles:
        hit, tot = needle_hit_rate(sel, x["needle_blocks"])
        res["needle_hit_rate"] = {"alpha": 3.0, "hits": hit, "of": tot,
                                  "rate": hit / tot if tot else None}
    del ws_att, out, flush
    torch.cuda.empty_cache()
    if not args.no_cpu_baseline:
        leg = OracleLeg(x, None, shape, None)
        if oracle_full:
            secs, rows = leg.prefill_full()
            sample = f"every position: {rows} (query, group) rows"
        else:
            rng = np.random.default_rng(seed)
            t_s, secs, rows = leg.prefill_stratified(rng, n_strata)
            sample = (f"{rows} (query, group) rows: one uniform position in each of {n_strata} "
                      f"equal strata of [0,L), all groups and heads; {t_s:.1f} s, extrapolated to "
                      f"the whole prefill by stratum width")
        res["oracle"] = {"seconds": secs, "tokens_per_s": B * L / secs, "cores": oracle_threads(),
                         "kind": "oracle", "extrapolated": not oracle_full, "sample": sample}
        res["gpu_over_oracle"] = secs / (pre_ms / 1e3)
    del x, sel
    torch.cuda.empty_cache()
    return res


def nsa_branch_flops(B, L, H, d, window, block):
    """Algorithmic FLOPs of the window and compression branches: per query and
    head 4*d per attended key (q.k and p*v), over min(window, t+1) tokens and
    (t+1)//block compressed tokens."""
    t = np.arange(L, dtype=np.float64)
    f_win = B * H * 4 * d * float(np.minimum(window, t + 1).sum())
    f_cmp = B * H * 4 * d * float(((t + 1) // block).sum())
    return f_win, f_cmp


def bench_nsa_32k(M, I, dev, args, peaks, window=512, iters=10):
    """The NSA-style variant at the 32K prefill: msa_nsa_forward (MSA's index
    and selection branches, block compression, the compression and window
    branches, the gate) timed whole and branch by branch, with an L2 flush
    between iterations; tensor rooflines of the two query-outer branch
    kernels; the oracle on stratified positions beside it."""
    shape = I.PREFILL_32K
    seed = I.SEEDS["32k"]
    x = I.prefill_inputs(shape, seed, device=dev)
    B, L, H, G, d, di, K, blk = (shape.B, shape.L, shape.H, shape.G, shape.d, shape.d_idx,
                                 shape.top_k, shape.block)
    p = M.make_params(B, L, H, G, d, di, blk, K)
    gen = torch.Generator(device="cpu").manual_seed(seed)
    gates = torch.rand((B, L, H, 3), generator=gen).to(dev)
    ws = M.new_workspace(p, M.MSA_OP_NSA_FORWARD, dev)
    ws_b = M.new_workspace(p, M.MSA_OP_NSA_BRANCH, dev)
    out = torch.empty_like(x["q"])
    o_b = torch.empty_like(x["q"])
    nb = (L + blk - 1) // blk
    kc = torch.empty((B, nb, G, d), dtype=torch.bfloat16, device=dev)
    vc = torch.empty_like(kc)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def run_all():
        M.msa_nsa_forward(x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"], gates, K, window,
                          block=blk, out=out, ws=ws)

    def run_win():
        M.msa_nsa_window_attn(x["q"], x["k"], x["v"], window, out=o_b, ws=ws_b)

    def run_cmp():
        M.msa_nsa_compressed_attn(x["q"], kc, vc, block=blk, out=o_b, ws=ws_b)

    def run_compress():
        M.msa_nsa_compress_kv(x["k"], x["v"], block=blk, k_cmp=kc, v_cmp=vc)

    legs = {"forward": run_all, "window": run_win, "compress_kv": run_compress,
            "compressed": run_cmp}
    for _ in range(max(3, args.warmup)):
        for f in legs.values():
            f()
    torch.cuda.synchronize()
    if M.msa_read_status(ws) != 0 or M.msa_read_status(ws_b) != 0:
        raise SystemExit("nsa_32k: device status error")
    times = {k: [] for k in legs}
    for _ in range(iters):
        for k, f in legs.items():
            flush.zero_()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            f()
            b.record(stream)
            torch.cuda.synchronize()
            times[k].append(a.elapsed_time(b))
    ms = {k: statistics.median(v) for k, v in times.items()}
    f_win, f_cmp = nsa_branch_flops(B, L, H, d, window, blk)
    burst = peaks["bf16_tflops"]

    def tensor_roofline(f, t_ms):
        return {"bound": "tensor", "achieved": f / (t_ms / 1e3) / 1e12, "peak": burst,
                "unit": "TFLOP/s", "frac": f / (t_ms / 1e3) / 1e12 / burst, "flops": f,
                "peak_kind": f"bf16 burst ({peaks['source']}): kernel timed alone"}

    nchunks = math.ceil(B * L / M.msa_prefill_chunk_len(p))
    res = {"workload": f"B={B} L={L} H={H} G={G} d={d} d_idx={di} block={blk} top_k={K}, "
                       f"window {window}, gates U[0,1)",
           "seed": seed, "iters": iters, "l2": "256 MB buffer written before every timed call",
           "forward_ms": ms["forward"], "tokens_per_s": B * L / (ms["forward"] / 1e3),
           "window_ms": ms["window"], "compress_kv_ms": ms["compress_kv"],
           "compressed_ms": ms["compressed"],
           "window_roofline": tensor_roofline(f_win, ms["window"]),
           "compressed_roofline": tensor_roofline(f_cmp, ms["compressed"]),
           "compress_kv_roofline": {"bound": "hbm", "unit": "GB/s", "peak": peaks["hbm_gbs"],
                                    "bytes": 2 * B * L * G * d * 2 + 2 * B * nb * G * d * 2,
                                    "achieved": (2 * B * L * G * d * 2 + 2 * B * nb * G * d * 2)
                                    / (ms["compress_kv"] / 1e3) / 1e9},
           "gpu_launches": (1 + 5 * nchunks + 4) * iters}
    res["compress_kv_roofline"]["frac"] = res["compress_kv_roofline"]["achieved"] / peaks["hbm_gbs"]
    del ws, ws_b, out, o_b, kc, vc, flush
    torch.cuda.empty_cache()
    if not args.no_cpu_baseline:
        leg = OracleLeg(x, None, shape, None)
        rng = np.random.default_rng(seed)
        n_strata = 64
        pos, width = [], []
        for i in range(n_strata):
            lo, hi = i * L // n_strata, (i + 1) * L // n_strata
            pos.append((0, int(rng.integers(lo, hi))))
            width.append(hi - lo)
        tms, t_cmp = leg.nsa_positions(pos, window)
        secs = t_cmp + sum(w * tm for w, tm in zip(width, tms))
        res["oracle"] = {"seconds": secs, "tokens_per_s": B * L / secs, "cores": oracle_threads(),
                         "kind": "oracle", "extrapolated": True,
                         "sample": f"{len(pos) * G} (query, group) rows: one uniform position in "
                                   f"each of {n_strata} equal strata of [0,L), all groups and "
                                   f"heads, the three branches; {sum(tms):.1f} s, extrapolated "
                                   f"by stratum width, plus the block compression "
                                   f"({t_cmp:.2f} s)"}
        res["gpu_over_oracle"] = secs / (ms["forward"] / 1e3)
    del x, gates
    torch.cuda.empty_cache()
    return res


def bench_ragged_batch(M, I, dev, args, peaks):
    """A serving batch of prompt chunks continuing cached prefixes: 16
    sequences with caches of 131,072 tokens, each continuing at a seeded
    position t0 with n new tokens (n uniform in [1, 16384], t0 uniform in
    [0, Lmax - n]), every length unaligned.  msa_forward_cached_varlen runs
    the batch with one launch per kernel; the same batch sequence by sequence
    (msa_forward_cached, B = 1 each) is timed beside it."""
    s = I.RAGGED_BATCH
    rng = np.random.default_rng(I.SEEDS["ragged"])
    n = rng.integers(1, s.n_hi + 1, size=s.B).tolist()
    t0 = [int(rng.integers(0, s.Lmax - nb + 1)) for nb in n]
    gen = torch.Generator(device=dev)
    gen.manual_seed(I.SEEDS["ragged"])
    N = int(sum(n))
    mk = lambda shp: torch.randn(shp, generator=gen, device=dev, dtype=torch.float32).to(torch.bfloat16)
    q, q_idx = mk((N, s.H, s.d)), mk((N, s.G, s.d_idx))
    k, v, k_idx = mk((s.B, s.Lmax, s.G, s.d)), mk((s.B, s.Lmax, s.G, s.d)), mk((s.B, s.Lmax, s.d_idx))
    out = torch.empty_like(q)
    p = M.make_params(s.B, s.Lmax, s.H, s.G, s.d, s.d_idx, BLOCK, s.top_k)
    ws = M.new_workspace(p, M.MSA_OP_FORWARD_VARLEN, dev)
    p1 = M.make_params(1, s.Lmax, s.H, s.G, s.d, s.d_idx, BLOCK, s.top_k)
    ws1 = M.new_workspace(p1, M.MSA_OP_FORWARD, dev)
    rows0 = np.concatenate([[0], np.cumsum(n)]).tolist()
    stream = torch.cuda.current_stream()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def one_launch():
        M.msa_forward_cached_varlen(q, q_idx, k, v, k_idx, t0, n, s.top_k, out=out, ws=ws)

    def per_sequence():
        for b in range(s.B):
            r0, r1 = rows0[b], rows0[b + 1]
            M.msa_forward_cached(q[r0:r1].unsqueeze(0), q_idx[r0:r1].unsqueeze(0), k[b:b + 1],
                                 v[b:b + 1], k_idx[b:b + 1], t0[b], s.top_k,
                                 out=out[r0:r1].unsqueeze(0), ws=ws1)

    def timed(fn, iters=5):
        for _ in range(max(3, args.warmup)):
            fn()
        torch.cuda.synchronize()
        if M.msa_read_status(ws) != 0 or M.msa_read_status(ws1) != 0:
            raise SystemExit("ragged batch: device status error")
        ts = []
        for _ in range(iters):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        return statistics.median(ts)

    ms = timed(one_launch)
    ms_seq = timed(per_sequence)
    f = 0.0
    for b in range(s.B):
        t = np.arange(t0[b], t0[b] + n[b], dtype=np.int64)
        bt = t // BLOCK
        f += s.G * 2.0 * s.d_idx * float(np.where(bt >= s.top_k, bt * BLOCK, 0).sum())
        f += s.H * 4.0 * s.d * float(n_sel(t, s.top_k).sum())
    del q, q_idx, k, v, k_idx, out, ws, ws1, flush
    torch.cuda.empty_cache()
    return {"workload": f"{s.B} sequences, caches of {s.Lmax}, n uniform in [1, {s.n_hi}], "
                        f"H={s.H} G={s.G} d={s.d} d_idx={s.d_idx} block={BLOCK} top_k={s.top_k}",
            "seed": I.SEEDS["ragged"], "new_tokens": N, "ms": ms,
            "tokens_per_s": N / (ms / 1e3), "ms_sequence_by_sequence": ms_seq,
            "one_launch_speedup": ms_seq / ms,
            "tensor": {"flops": f, "tflops": f / (ms / 1e3) / 1e12,
                       "frac_of_burst": f / (ms / 1e3) / 1e12 / peaks["bf16_tflops"]},
            "l2": "256 MB buffer written between iterations"}


def bench_configs(M, I, dev, args, peaks, line):
    """Every configuration at 1 GPU.  The 1M step and decode-128K were timed
    above; the tiny, 32K and 128K-planted prefills are timed here."""
    cfgs = {}
    cfgs["tiny"] = bench_prefill_config(M, I, dev, args, peaks, "tiny", I.PREFILL_TINY,
                                        I.SEEDS["tiny"], oracle_full=True, iters=20)
    cfgs["32k"] = bench_prefill_config(M, I, dev, args, peaks, "32k", I.PREFILL_32K,
                                       I.SEEDS["32k"], iters=10)
    cfgs["128k_planted"] = bench_prefill_config(M, I, dev, args, peaks, "128k_planted",
                                                I.PREFILL_128K_PLANTED, I.SEEDS["128k_planted"],
                                                needles=12, iters=5)
    # the 64-token block variant at the same 2048-token budget (32 blocks)
    cfgs["32k_block64"] = bench_prefill_config(M, I, dev, args, peaks, "32k_block64",
                                               I.PREFILL_32K_BLOCK64, I.SEEDS["32k"], iters=10)
    cfgs["ragged_batch"] = bench_ragged_batch(M, I, dev, args, peaks)
    cfgs["nsa_32k"] = bench_nsa_32k(M, I, dev, args, peaks)
    if "decode_128k" in line:
        d = line["decode_128k"]
        cfgs["decode_128k"] = {"us_per_step": d["us_per_step"], "roofline": d["roofline"],
                               "frac_of_8tbs": d["roofline"]["achieved"] / SPEC_HBM_GBS,
                               "oracle": d.get("oracle")}
    bd = line["breakdown"]
    cfgs["1m"] = {"ms_per_step": line["ms_per_step"], "tokens_per_s": line["value"],
                  "prefill_tokens_per_s": bd["prefill_tokens_per_s"],
                  "index_roofline": line["roofline"],
                  "prefill_tensor_frac_of_spec": (bd["index_flops"] + bd["main_flops"])
                  / ((bd["index_ms"] + bd["prefill_attn_ms"]) / 1e3) / 1e12 / SPEC_BF16_TFLOPS,
                  "attn_roofline": bd["prefill_attn_roofline"],
                  "decode_us": bd["decode_us"], "decode_roofline": bd["decode_roofline"],
                  "decode_frac_of_8tbs": bd["decode_roofline"]["achieved"] / SPEC_HBM_GBS}
    return cfgs


def bench_e2e(M, x, dx, shape, dshape, K, args, ws_n, stream):
    """Same step through the public API (msa_forward + msa_sparse_attn_decode),
    inputs copied from pinned host memory and outputs read back every step."""
    dev = x["q"].device
    names = ("q", "k", "v", "q_idx", "k_idx")
    host = {n: x[n].to("cpu").pin_memory() for n in names}
    dnames = ("q", "q_idx")
    dhost = {n: dx[n].to("cpu").pin_memory() for n in dnames}
    dbuf = {n: torch.empty_like(x[n]) for n in names}
    ddbuf = {n: torch.empty_like(dx[n]) for n in dnames}
    out_h = torch.empty(x["q"].shape, dtype=torch.bfloat16).pin_memory()
    dout_h = torch.empty(dx["q"].shape, dtype=torch.bfloat16).pin_memory()
    p = M.make_params(shape.B, shape.L, shape.H, shape.G, shape.d, shape.d_idx, BLOCK, K)
    pd = M.make_params(dshape.B, dshape.Lmax, dshape.H, dshape.G, dshape.d, dshape.d_idx, BLOCK,
                       dshape.top_k)
    ws = M.new_workspace(p, M.MSA_OP_FORWARD, dev)
    wsd = M.new_workspace(pd, M.MSA_OP_DECODE, dev)
    staging = dict(dbuf)
    staging["out"] = torch.empty_like(x["q"])
    dout = torch.empty_like(dx["q"])
    copy_stream = torch.cuda.Stream(device=dev)
    h2d = sum(host[n].numel() * 2 for n in names) + sum(dhost[n].numel() * 2 for n in dnames)
    d2h = out_h.numel() * 2 + dout_h.numel() * 2

    def step():
        # prefill from host buffers: uploads overlap the index branch and each
        # query chunk's output is downloaded while the next chunk computes
        M.msa_forward_host(host["q"], host["k"], host["v"], host["q_idx"], host["k_idx"], K,
                           out=out_h, staging=staging, ws=ws, stream=stream,
                           copy_stream=copy_stream)
        for n in dnames:
            ddbuf[n].copy_(dhost[n], non_blocking=True)
        M.msa_sparse_attn_decode(ddbuf["q"], ddbuf["q_idx"], dx["k_cache"], dx["v_cache"],
                                 dx["k_idx_cache"], dx["seq_lens"], dshape.top_k, out=dout, ws=wsd)
        dout_h.copy_(dout, non_blocking=True)

    for _ in range(max(1, min(args.warmup, 2))):
        step()
    torch.cuda.synchronize()
    n = max(1, min(args.steps, 3))
    dist_barrier(ws_n)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(n):
        step()
    b.record(stream)
    torch.cuda.synchronize()
    ms = dist_max(a.elapsed_time(b) / n, ws_n)
    tokens = shape.B * shape.L + dshape.B
    del host, dhost, dbuf, ddbuf, out_h, dout_h, staging
    return {"value": ws_n * tokens / (ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": ms, "steps": n,
            "path": "msa_forward_host (host buffers, transfers overlapped) + msa_sparse_attn_decode "
                    "(C ABI via the Python binding)"}


if __name__ == "__main__":
    main()
