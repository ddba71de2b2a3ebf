#!/usr/bin/env python3
"""Benchmark of the SALA hybrid attention forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {sala,reference}]

One step = one attention prefill pass over a 262144-token sequence through the 32-layer hybrid
stack: 24 linear-attention layers (sala_linear_prefill) and 8 sparse-attention layers
(sala_block_compress -> sala_block_topk -> sala_sparse_prefill), sparse layers at 3, 7, ..., 31,
each layer with its own seeded Q/K/V (all resident in HBM before timing; every tensor is 2 GiB or
128 MiB, far larger than L2, so no flush is needed).  The printed JSON line reports whole-job
tokens/s (device time, CUDA events, max over ranks), plus:
  decode   : one decode token per step at a 2^20-token context through the same 32-layer stack
             (24 x sala_linear_decode + 8 x sala_sparse_decode with in-kernel selection),
             L2 flushed before every step, us/token;
  e2e      : the prefill step through the same calls with the layer inputs streamed from pinned
             host memory and the outputs copied back (copies inside the timed region);
  roofline : the dominant kernel (sparse prefill, tensor-bound) -- algorithmic FLOPs per launch /
             its mean launch time, against the measured bf16 peak;
  cpu_baseline : the fp64 oracle on a bounded sample of the same workload, scaled to tokens/s.
--impl reference times only the oracle (the CPU baseline arm) and prints its own line.
With --gpus N > 1 (torchrun) every rank runs an independent replica (weak scaling).
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
sys.path.insert(0, ROOT)

N_TOK = 262144
H, HKV, D = 32, 2, 128
TOPK, N_INIT, N_LOCAL, BLOCK = 64, 1, 2, 64
N_LAYERS = 32
SPARSE_LAYERS = [l for l in range(N_LAYERS) if l % 4 == 3]
DECODE_T = 1 << 20
METRIC = "SALA attn prefill tokens/s @256K; decode µs/token @1M; % of roofline"


# ----------------------------------------------------------------------------------------------
# algorithmic work (closed forms of the selection rule; independent of the GPU's output)

def attended_keys(N: int, topk=TOPK, n_init=N_INIT, n_local=N_LOCAL, block=BLOCK) -> int:
    """Sum over query tokens of |J_i| (keys each token attends to; shared by the group's heads)."""
    total = 0
    nblk = (N + block - 1) // block
    for c in range(nblk):
        rows = min(block, N - c * block)
        ncand = max(0, c - n_local + 1 - n_init)
        if ncand <= topk:
            full_before = c                      # every block 0..c-1 plus the diagonal
        else:
            full_before = n_init + topk + (n_local - 1)
        # token at offset t of block c attends full_before * block + (t + 1) keys
        total += rows * full_before * block + rows * (rows + 1) // 2
    return total


def sparse_layer_flops(N: int) -> float:
    return 4.0 * D * H * attended_keys(N)        # QK^T and PV, 2 FLOP per MAC each


# DRAM traffic of the sparse prefill kernel (dram__bytes_read.sum + dram__bytes_write.sum) from one
# ncu capture of the single-layer N = 131072 case, 2.323e9 bytes per launch, scaled by the tokens
# processed to N = 262144 (Q reads, O writes and the K/V re-reads per 16-token unit all grow with N).
# Valid only for the kernel sources it was taken on: any change to them reports null.
SPARSE_TRAFFIC = {"bytes_per_token": (1288783104 + 1033887232) / 131072,
                  "sources": {"sparse_tc.cu": "0b1ebdf2db4727e0e23f510939c7096e1ceba114f6c618463cff01c4d788a173",
                              "fastexp.cuh": "b6d9ae064f35b9fd752ec893180eaf72ade6f0495d57f5699832618f42784c06",
                              "ptx.cuh": "fd104364a691e71bb755a0a84573920e3263e23dbfbee024db781170b73eb422"}}


def sparse_traffic(N: int):
    import hashlib
    src = os.path.join(os.path.dirname(os.path.abspath(__file__)), "hybrid_sparse_linear_b200", "csrc")
    for name, digest in SPARSE_TRAFFIC["sources"].items():
        try:
            with open(os.path.join(src, name), "rb") as f:
                if hashlib.sha256(f.read()).hexdigest() != digest:
                    return None
        except OSError:
            return None
    return SPARSE_TRAFFIC["bytes_per_token"] * N


# Tensor-core work the sparse prefill kernel executes per (8-token tile, block of the union of
# the tile's 8 selections): S = Q K^T (M128 N64 K128) and O += P V (M128 N128 K64).
EXEC_FLOPS_PER_TILE_BLOCK = 2.0 * 128 * 64 * 128 * 2


def tile_union_blocks(torch, idx, tq: int = 8, heads: int = 1) -> int:
    """Sum over 8-token tiles of |union of the tile's selections| (idx [B, Hkv, N, slots], -1 pad).
    heads > 1: idx is [B, Hkv * heads, N, slots], one row per query head, and a tile's union runs
    over its 8 tokens of all `heads` heads of the KV group (one KV group at a time)."""
    if heads > 1:
        B, Hq, N, S = idx.shape
        return sum(tile_union_blocks(torch, idx[:, g * heads:(g + 1) * heads].permute(0, 2, 1, 3)
                                     .reshape(B, 1, N, heads * S), tq)
                   for g in range(Hq // heads))
    B, G, N, S = idx.shape
    pad = (-N) % tq
    if pad:
        idx = torch.cat([idx, idx.new_full((B, G, pad, S), -1)], dim=2)
    t, _ = torch.sort(idx.reshape(B, G, -1, tq * S), dim=-1)
    n = ((t[..., 1:] != t[..., :-1]) & (t[..., 1:] >= 0)).sum() + (t[..., 0] >= 0).sum()
    return int(n.item())


def linear_layer_bytes(N: int) -> float:
    return 4.0 * H * N * D * 2                    # read Q, K, V and write O, bf16


def decode_bytes(T: int) -> dict:
    lin = H * D * D * 4 * 2 + 4 * H * D * 2       # state read + write, q/k/v/o
    nb = T // BLOCK
    sp = HKV * nb * D * 2 + HKV * (N_INIT + N_LOCAL + TOPK) * BLOCK * D * 2 * 2 + 2 * H * D * 2
    return {"linear": lin, "sparse": sp, "step": 24 * lin + 8 * sp}


# ----------------------------------------------------------------------------------------------
# distributed plumbing (host-side only: barrier and max over ranks; no data-path collective)

def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def init_dist(backend: str):
    import torch.distributed as dist
    ws, rank, _ = dist_env()
    if ws > 1 and not dist.is_initialized():
        import datetime
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return ws, rank


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def max_over_ranks(x: float, device="cpu") -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ----------------------------------------------------------------------------------------------
class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 200 ms while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.reader = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.reader = threading.Thread(target=self._read, daemon=True)
        self.reader.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.reader:
            self.reader.join(timeout=2)
        sm, smax, reasons, power = [], None, set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
                power.append(float(parts[3]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": smax, "reasons": ["no samples"]}
        loaded = [s for s, p in zip(sm, power) if p > 300.0] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------------------------
def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained", p["bf16_tflops"]),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


# Prefill workloads: (sequence length, layer kinds).  The first is the benchmark; the single-layer
# ones are the small cases used for kernel profiles.
WORKLOADS = {
    "hybrid_prefill_n256k": (N_TOK, ["sparse" if l in SPARSE_LAYERS else "linear" for l in range(N_LAYERS)]),
    "sparse_prefill_n128k": (131072, ["sparse"]),
    "linear_prefill_n32k": (32768, ["linear"]),
    "sparse_prefill_n32k": (32768, ["sparse"]),
    "linear_prefill_n256k": (N_TOK, ["linear"]),
    # a linear layer with its RoPE (HyPE) fused into the load path, base 10000, positions 0..N-1
    "linear_rope_prefill_n256k": (N_TOK, ["linear_rope"]),
    # a sparse layer whose 64-token query blocks each share one selection (the variant)
    "sparse_qblock_prefill_n256k": (N_TOK, ["sparse_qblock"]),
    "sparse_qblock_softmax_prefill_n256k": (N_TOK, ["sparse_qsoft"]),
    # a sparse layer whose query heads each choose their own blocks (the per-head variant)
    "sparse_per_head_prefill_n256k": (N_TOK, ["sparse_per_head"]),
    "linear_rope_prologue_prefill_n256k": (N_TOK, ["linear_rope_pro"]),
}


def run_prefill(sala, synth, torch, steps, warmup, stream, workload="hybrid_prefill_n256k"):
    """Device-timed prefill of a workload.  Returns timing dict."""
    dev = torch.device("cuda")
    n_tok, kinds = WORKLOADS[workload]
    lam = synth.decays(H).to(dev)
    layers = []
    for l, kind in enumerate(kinds):
        if kind.startswith("sparse"):
            sl = synth.sparse_layer(1, H, HKV, n_tok, D, torch.bfloat16, dev, layer=l)
            layers.append((kind, sl.q, sl.k, sl.v))
        else:
            q, k, v = synth.linear_layer(1, H, n_tok, D, torch.bfloat16, dev, layer=l)
            layers.append((kind, q, k, v))
    out = torch.empty((1, H, n_tok, D), device=dev, dtype=torch.bfloat16)
    nb = n_tok // BLOCK
    kbar = torch.empty((1, HKV, nb, D), device=dev, dtype=torch.bfloat16)
    slots = N_INIT + N_LOCAL + TOPK
    sel_heads = H if "sparse_per_head" in kinds else HKV   # selection rows per token
    idx = torch.empty((1, sel_heads, n_tok, slots), device=dev, dtype=torch.int32)
    # scratch of the sequence-parallel linear prefill (the segments' states)
    lws = torch.empty(max(sala.linear_prefill_workspace_bytes(1, H, n_tok, D), 16), device=dev,
                      dtype=torch.uint8)
    # rotated q and k of a RoPE layer run as the one-pass prologue + the plain prefill
    qr = kr = None
    if "linear_rope_pro" in kinds:
        qr = torch.empty((1, H, n_tok, D), device=dev, dtype=torch.bfloat16)
        kr = torch.empty_like(qr)
    torch.cuda.synchronize()

    ev = lambda: torch.cuda.Event(enable_timing=True)
    sparse_ev, linear_ev, topk_ev = [], [], []

    def select(kind, q):
        if kind == "sparse":
            sala.block_topk(q, kbar, TOPK, N_INIT, N_LOCAL, idx=idx, stream=stream)
        elif kind == "sparse_qblock":
            sala.block_topk_qblock(q, kbar, TOPK, N_INIT, N_LOCAL, idx=idx, stream=stream)
        elif kind == "sparse_per_head":
            sala.block_topk_per_head(q, kbar, TOPK, N_INIT, N_LOCAL, idx=idx, stream=stream)
        else:
            sala.block_topk_qblock_softmax(q, kbar, TOPK, N_INIT, N_LOCAL, idx=idx, stream=stream)

    def one_step(record):
        launches = 0
        for kind, q, k, v in layers:
            if kind in ("linear", "linear_rope", "linear_rope_pro"):
                e0, e1 = (ev(), ev()) if record else (None, None)
                if record: e0.record(stream)
                if kind == "linear":
                    sala.linear_prefill(q, k, v, lam, o=out, workspace=lws, stream=stream)
                elif kind == "linear_rope":
                    sala.linear_prefill(q, k, v, lam, o=out, workspace=lws, stream=stream,
                                        rope_base=10000.0, pos0=0)
                else:
                    sala.qk_prologue(q, k, q_out=qr, k_out=kr, rope_base=10000.0, pos0=0,
                                     stream=stream)
                    sala.linear_prefill(qr, kr, v, lam, o=out, workspace=lws, stream=stream)
                    launches += 1
                if record: e1.record(stream); linear_ev.append((e0, e1))
                launches += 3  # segment states, their chain, the output pass
            else:
                t0, t1 = (ev(), ev()) if record else (None, None)
                if record: t0.record(stream)
                sala.block_compress(k, kbar, stream=stream)
                select(kind, q)
                if record: t1.record(stream); topk_ev.append((t0, t1))
                e0, e1 = (ev(), ev()) if record else (None, None)
                if record: e0.record(stream)
                if kind == "sparse_per_head":
                    sala.sparse_prefill_per_head(q, k, v, idx, o=out, stream=stream)
                else:
                    sala.sparse_prefill(q, k, v, idx, o=out, stream=stream)
                if record: e1.record(stream); sparse_ev.append((e0, e1))
                launches += 3
        return launches

    with torch.cuda.stream(stream):
        for _ in range(warmup):
            one_step(False)
        sala.check_status(stream)
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        start, end = ev(), ev()
        start.record(stream)
        launches = 0
        for _ in range(steps):
            launches += one_step(True)
        end.record(stream)
        torch.cuda.synchronize()
        barrier()
    sala.check_status(stream)
    total_ms = start.elapsed_time(end)
    mean = lambda pairs: sum(a.elapsed_time(b) for a, b in pairs) / max(1, len(pairs))
    res = {"total_ms": total_ms, "launches": launches,
           "sparse_ms": mean(sparse_ev), "linear_ms": mean(linear_ev), "select_ms": mean(topk_ev)}
    # Executed tensor-core work of the sparse kernel, counted after the timed region from each
    # sparse layer's selection (recomputed: the timed steps overwrite one shared buffer).
    union, n_sp = 0, 0
    with torch.cuda.stream(stream):
        for kind, q, k, v in layers:
            if kind.startswith("sparse"):
                sala.block_compress(k, kbar, stream=stream)
                select(kind, q)
                union += tile_union_blocks(torch, idx, heads=H // HKV if kind == "sparse_per_head" else 1)
                n_sp += 1
    res["sparse_exec_flops"] = EXEC_FLOPS_PER_TILE_BLOCK * union / max(1, n_sp)
    del layers, out, kbar, idx
    torch.cuda.empty_cache()
    return res


def run_decode_paged(sala, synth, torch, steps, warmup, stream, B=8):
    """One sparse layer's decode for B sequences at their own positions (64K .. 256K tokens), the
    KV cache in pages of one block scattered over a pool; CUDA-graph replays, L2 flushed."""
    import numpy as np
    dev = torch.device("cuda")
    lengths = [int(n) // 64 * 64 + 17 for n in np.linspace(1 << 16, 1 << 18, B)]
    nblk = [(n + 63) // 64 for n in lengths]
    max_pages, n_pages = max(nblk), sum(nblk)
    perm = torch.randperm(n_pages, generator=torch.Generator().manual_seed(5))
    k_pages = torch.empty((n_pages, HKV, BLOCK, D), dtype=torch.bfloat16, device=dev)
    v_pages = torch.empty_like(k_pages)
    table = torch.full((B, max_pages), -1, dtype=torch.int32)
    nb_cap = max(n // BLOCK for n in lengths)
    kbar = torch.zeros((B, HKV, nb_cap, D), dtype=torch.bfloat16, device=dev)
    qs, at = [], 0
    for b, n in enumerate(lengths):
        sl = synth.sparse_layer(1, H, HKV, n, D, torch.bfloat16, dev, layer=40 + b, q_rows=1)
        pad = nblk[b] * BLOCK - n
        kk = torch.nn.functional.pad(sl.k[0], (0, 0, 0, pad)).view(HKV, nblk[b], BLOCK, D)
        vv = torch.nn.functional.pad(sl.v[0], (0, 0, 0, pad)).view(HKV, nblk[b], BLOCK, D)
        ids = perm[at:at + nblk[b]]
        at += nblk[b]
        table[b, :nblk[b]] = ids.to(torch.int32)
        k_pages[ids.to(dev)] = kk.transpose(0, 1)
        v_pages[ids.to(dev)] = vv.transpose(0, 1)
        kbar[b, :, :n // BLOCK] = sala.block_compress(sl.k, stream=stream)[0, :, :n // BLOCK]
        qs.append(sl.q[0, :, 0])
        del sl
    q = torch.stack(qs).contiguous()
    table = table.to(dev)
    pos = torch.tensor([n - 1 for n in lengths], dtype=torch.int32, device=dev)
    max_pos = max(lengths) - 1
    need = sala.sparse_decode_paged_workspace_bytes(B, H, HKV, max_pos, TOPK, N_INIT, N_LOCAL, D)
    ws = torch.zeros(max(need, 256), dtype=torch.uint8, device=dev)
    o = torch.empty_like(q)
    flush = torch.empty(512 << 20, device=dev, dtype=torch.uint8)
    call = lambda: sala.sparse_decode_paged(q, k_pages, v_pages, table, kbar, pos, max_pos, TOPK,
                                            N_INIT, N_LOCAL, o=o, workspace=ws, stream=stream)
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            call()
        torch.cuda.synchronize()
        sala.check_status(stream)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            call()
        times = []
        for _ in range(max(steps, 20)):
            flush.zero_()
            a, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            g.replay()
            e.record(stream)
            times.append((a, e))
        torch.cuda.synchronize()
    sala.check_status(stream)
    us = sorted(a.elapsed_time(e) * 1000.0 for a, e in times)[len(times) // 2]
    slots = N_INIT + N_LOCAL + TOPK
    nbytes = sum(HKV * (n // BLOCK) * D * 2 + HKV * slots * BLOCK * D * 2 * 2 + 2 * H * D * 2
                 for n in lengths)
    del g, k_pages, v_pages, kbar, flush
    torch.cuda.empty_cache()
    return {"us_per_call": us, "bytes": nbytes, "lengths": lengths}


def run_linear_backward(sala, synth, torch, steps, warmup, stream, n_tok=N_TOK):
    """The backward pass of one linear layer (dq, dk, dv from dout) at N tokens, 32 heads."""
    dev = torch.device("cuda")
    q, k, v = synth.linear_layer(1, H, n_tok, D, torch.bfloat16, dev, layer=0)
    dout = synth.linear_layer(1, H, n_tok, D, torch.bfloat16, dev, layer=1)[0]
    lam = synth.decays(H).to(dev)
    ws = torch.empty(max(sala._lib.sala_linear_backward_workspace(1, H, n_tok, D, 1), 16),
                     dtype=torch.uint8, device=dev)
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            sala.linear_backward(q, k, v, lam, dout, workspace=ws, stream=stream)
        torch.cuda.synchronize()
        a, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(steps):
            sala.linear_backward(q, k, v, lam, dout, workspace=ws, stream=stream)
        e.record(stream)
        torch.cuda.synchronize()
    sala.check_status(stream)
    ms = a.elapsed_time(e) / steps
    del q, k, v, dout, ws
    torch.cuda.empty_cache()
    return {"ms": ms, "bytes": 7.0 * H * n_tok * D * 2}  # read q, k, v, dout; write dq, dk, dv


def run_sparse_backward(sala, synth, torch, steps, warmup, stream, n_tok=N_TOK):
    """Training step of one sparse layer at N tokens (32 query / 2 KV heads, top-64 + 1 init +
    2 local): the training forward (lse, o's residual), then the backward (dq, dk, dv), each
    timed with CUDA events over `steps` back-to-back calls.  Executed FLOPs are counted from the
    selection: the query-side pass runs 4 MMAs of 2.10 MFLOP per (8-token tile, union block), the
    key-side pass 4 per 8-token tile of each block's token list."""
    dev = torch.device("cuda")
    sl = synth.sparse_layer(1, H, HKV, n_tok, D, torch.bfloat16, dev, layer=3)
    dout = synth.normal((1, H, n_tok, D), synth.seed(3, 7), dev, torch.bfloat16)
    kbar = sala.block_compress(sl.k, stream=stream)
    idx = sala.block_topk(sl.q, kbar, TOPK, N_INIT, N_LOCAL, stream=stream)
    o, lse, o_lo = sala.sparse_prefill(sl.q, sl.k, sl.v, idx, lse=True, o_lo=True, stream=stream)
    ws = torch.empty(sala.sparse_backward_workspace_bytes(1, H, HKV, n_tok, D, idx.shape[3]),
                     dtype=torch.uint8, device=dev)
    ev = lambda: torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            sala.sparse_prefill(sl.q, sl.k, sl.v, idx, o=o, lse=lse, o_lo=o_lo, stream=stream)
            sala.sparse_backward(sl.q, sl.k, sl.v, idx, o, lse, dout, o_lo=o_lo, workspace=ws,
                                 stream=stream)
        torch.cuda.synchronize()
        a, b, c = ev(), ev(), ev()
        a.record(stream)
        for _ in range(steps):
            sala.sparse_prefill(sl.q, sl.k, sl.v, idx, o=o, lse=lse, o_lo=o_lo, stream=stream)
        b.record(stream)
        for _ in range(steps):
            sala.sparse_backward(sl.q, sl.k, sl.v, idx, o, lse, dout, o_lo=o_lo, workspace=ws,
                                 stream=stream)
        c.record(stream)
        torch.cuda.synchronize()
    sala.check_status(stream)
    mma = 2.0 * 128 * 64 * 128
    union = tile_union_blocks(torch, idx)
    nb = (n_tok + BLOCK - 1) // BLOCK
    keys = (idx + torch.arange(HKV, device=dev, dtype=torch.int32).view(1, HKV, 1, 1) * nb)[idx >= 0]
    cnt = torch.bincount(keys.long(), minlength=HKV * nb)
    kv_tiles = int(((cnt + 7) // 8).sum().item())
    out = {"fwd_ms": a.elapsed_time(b) / steps, "bwd_ms": b.elapsed_time(c) / steps,
           "alg_flops": 10.0 * D * H * attended_keys(n_tok),
           "exec_flops_dq": 4 * mma * union, "exec_flops_dkv": 4 * mma * kv_tiles}
    del sl, dout, kbar, idx, o, lse, o_lo, ws
    torch.cuda.empty_cache()
    return out


def run_qk_norm(sala, synth, torch, steps, warmup, stream, n_tok=N_TOK):
    """QK normalisation of one linear layer's q and k (32 heads each, d 128) at N tokens, in
    place, one launch per call."""
    dev = torch.device("cuda")
    q = synth.prenorm((1, H, n_tok, D), synth.seed(0, synth.Q), dev, torch.bfloat16)
    k = synth.prenorm((1, H, n_tok, D), synth.seed(0, synth.K), dev, torch.bfloat16)
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            sala.qk_norm(q, k, q_out=q, k_out=k, stream=stream)
        torch.cuda.synchronize()
        a, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(steps):
            sala.qk_norm(q, k, q_out=q, k_out=k, stream=stream)
        e.record(stream)
        torch.cuda.synchronize()
    sala.check_status(stream)
    ms = a.elapsed_time(e) / steps
    del q, k
    torch.cuda.empty_cache()
    return {"ms": ms, "bytes": 2.0 * 2 * H * n_tok * D * 2}  # q and k read once, written once


def run_decode(sala, synth, torch, steps, warmup, stream, T=DECODE_T):
    """Decode at a T-token context (2^20 by default), 24 linear + 8 sparse layers per token, L2
    flushed."""
    dev = torch.device("cuda")
    pos = T - 1
    lam = synth.decays(H).to(dev)
    g = torch.Generator(device=dev)
    lin = []
    for l in range(N_LAYERS):
        if l in SPARSE_LAYERS:
            continue
        g.manual_seed(synth.seed(l, synth.U) + 17)
        S = torch.randn((1, H, D, D), generator=g, device=dev) / D
        q, k, v = synth.linear_layer(1, H, 1, D, torch.bfloat16, dev, layer=l)
        lin.append((S, q[:, :, 0].contiguous(), k[:, :, 0].contiguous(), v[:, :, 0].contiguous()))
    sp = []
    for l in SPARSE_LAYERS:
        sl = synth.sparse_layer(1, H, HKV, T, D, torch.bfloat16, dev, layer=l, q_rows=1)
        kbar = sala.block_compress(sl.k, stream=stream)
        sp.append((sl.q[:, :, 0].contiguous(), sl.k, sl.v, kbar))
    ws_bytes = sala.sparse_decode_workspace_bytes(1, H, HKV, pos, TOPK, N_INIT, N_LOCAL, D)
    ws = torch.zeros(max(ws_bytes, 256), device=dev, dtype=torch.uint8)  # counters start at 0
    o = torch.empty((1, H, D), device=dev, dtype=torch.bfloat16)
    flush = torch.empty(512 << 20, device=dev, dtype=torch.uint8)
    torch.cuda.synchronize()

    # Every layer launches as a programmatic dependent of the kernel before it (a linear layer
    # reads its own state, a sparse layer its share of k_bar, while the previous layer finishes);
    # the token is also timed without that.
    def one_token(pdl=True):
        for l in range(N_LAYERS):
            if l in SPARSE_LAYERS:
                q, kc, vc, kbar = sp[SPARSE_LAYERS.index(l)]
                sala.sparse_decode(q, kc, vc, kbar, pos, TOPK, N_INIT, N_LOCAL, o=o, workspace=ws,
                                   stream=stream, pdl=pdl)
            else:
                S, q, k, v = lin[l - sum(1 for s in SPARSE_LAYERS if s < l)]
                sala.linear_decode(q, k, v, lam, S, o=o, stream=stream, pdl=pdl)

    times = []
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            one_token()
        torch.cuda.synchronize()
        sala.check_status(stream)
        # One decode token (all 32 layers' calls) captured once and replayed: the library's calls
        # only enqueue kernels on the given stream, so the graph holds exactly those launches.
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            one_token()
        graph_plain = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph_plain, stream=stream):
            one_token(pdl=False)
        for _ in range(warmup):
            graph.replay()
            graph_plain.replay()
        times_plain = []
        for _ in range(steps):
            for g_, ts_ in ((graph, times), (graph_plain, times_plain)):
                flush.zero_()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                g_.replay()
                b.record(stream)
                ts_.append((a, b))
        torch.cuda.synchronize()
    sala.check_status(stream)
    us = [a.elapsed_time(b) * 1000.0 for a, b in times]
    us_plain = [a.elapsed_time(b) * 1000.0 for a, b in times_plain]

    def per_layer(kind):
        # The same calls of one kind only, captured and replayed the same way: where the time goes.
        calls = [l for l in range(N_LAYERS) if (l in SPARSE_LAYERS) == (kind == "sparse")]
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            with torch.cuda.graph(g, stream=stream):
                for l in calls:
                    if kind == "sparse":
                        q, kc, vc, kbar = sp[SPARSE_LAYERS.index(l)]
                        sala.sparse_decode(q, kc, vc, kbar, pos, TOPK, N_INIT, N_LOCAL, o=o,
                                           workspace=ws, stream=stream, pdl=True)
                    else:
                        S, q, k, v = lin[l - sum(1 for s in SPARSE_LAYERS if s < l)]
                        sala.linear_decode(q, k, v, lam, S, o=o, stream=stream, pdl=True)
            for _ in range(warmup):
                g.replay()
            ts = []
            for _ in range(steps):
                flush.zero_()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                g.replay()
                b.record(stream)
                ts.append((a, b))
            torch.cuda.synchronize()
        del g
        return statistics.median(a.elapsed_time(b) * 1000.0 for a, b in ts) / len(calls)

    lin_us, sp_us = per_layer("linear"), per_layer("sparse")
    sala.check_status(stream)
    del graph, graph_plain, lin, sp, ws, flush
    torch.cuda.empty_cache()
    # launches per token: linear 1 each; sparse 2 each (the score kernel over every SM, then the
    # attend kernel of one cluster per KV group)
    return {"us_per_token": statistics.median(us), "us_min": min(us), "samples": len(us),
            "us_per_token_without_pdl": statistics.median(us_plain),
            "launches_per_token": 24 * 1 + 8 * 2,
            "us_per_linear_layer": lin_us, "us_per_sparse_layer": sp_us}


def run_e2e(sala, synth, torch, steps, warmup):
    """Prefill step with every layer's inputs streamed from pinned host memory and the outputs
    copied back, through the same calls.  Copies run on their own streams into double-buffered
    device inputs, so the host->device copy of layer l+1 and the device->host copy of layer l-1
    overlap the kernels of layer l.  One pinned host copy of a linear and of a sparse layer is
    streamed for every layer of its kind (host RAM cannot hold 164 GiB of distinct inputs)."""
    dev = torch.device("cuda")
    lam = synth.decays(H).to(dev)
    ql, kl, vl = synth.linear_layer(1, H, N_TOK, D, torch.bfloat16, dev, layer=0)
    sl = synth.sparse_layer(1, H, HKV, N_TOK, D, torch.bfloat16, dev, layer=3)
    host = {"linear": [t.cpu().pin_memory() for t in (ql, kl, vl)],
            "sparse": [t.cpu().pin_memory() for t in (sl.q, sl.k, sl.v)]}
    del ql, kl, vl, sl
    torch.cuda.empty_cache()
    shape = {"linear": [(1, H, N_TOK, D)] * 3,
             "sparse": [(1, H, N_TOK, D), (1, HKV, N_TOK, D), (1, HKV, N_TOK, D)]}
    dbuf = {kind: [[torch.empty(sh, device=dev, dtype=torch.bfloat16) for sh in shape[kind]]
                   for _ in range(2)] for kind in ("linear", "sparse")}
    outs = [torch.empty((1, H, N_TOK, D), device=dev, dtype=torch.bfloat16) for _ in range(2)]
    out_host = torch.empty((1, H, N_TOK, D), dtype=torch.bfloat16).pin_memory()
    kbar = torch.empty((1, HKV, N_TOK // BLOCK, D), device=dev, dtype=torch.bfloat16)
    lws = torch.empty(max(sala.linear_prefill_workspace_bytes(1, H, N_TOK, D), 16), device=dev,
                      dtype=torch.uint8)
    idx = torch.empty((1, HKV, N_TOK, N_INIT + N_LOCAL + TOPK), device=dev, dtype=torch.int32)
    s_h2d, s_cmp, s_d2h = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()
    counts = {"h2d": 0, "d2h": 0}
    # per buffer slot: inputs copied / inputs consumed; per output slot: written / read back
    in_ready = {k: [None, None] for k in dbuf}
    in_free = {k: [None, None] for k in dbuf}
    out_ready, out_free = [None, None], [None, None]
    use = {"linear": 0, "sparse": 0}

    def step():
        for l in range(N_LAYERS):
            kind = "sparse" if l in SPARSE_LAYERS else "linear"
            slot = use[kind] & 1
            use[kind] += 1
            with torch.cuda.stream(s_h2d):
                if in_free[kind][slot] is not None:
                    s_h2d.wait_event(in_free[kind][slot])
                for dst, src in zip(dbuf[kind][slot], host[kind]):
                    dst.copy_(src, non_blocking=True)
                    counts["h2d"] += src.numel() * 2
                e = ev(); e.record(s_h2d); in_ready[kind][slot] = e
            o = outs[l & 1]
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(in_ready[kind][slot])
                if out_free[l & 1] is not None:
                    s_cmp.wait_event(out_free[l & 1])
                q, k, v = dbuf[kind][slot]
                if kind == "linear":
                    sala.linear_prefill(q, k, v, lam, o=o, workspace=lws, stream=s_cmp)
                else:
                    sala.block_compress(k, kbar, stream=s_cmp)
                    sala.block_topk(q, kbar, TOPK, N_INIT, N_LOCAL, idx=idx, stream=s_cmp)
                    sala.sparse_prefill(q, k, v, idx, o=o, stream=s_cmp)
                e = ev(); e.record(s_cmp); in_free[kind][slot] = e; out_ready[l & 1] = e
            with torch.cuda.stream(s_d2h):
                s_d2h.wait_event(out_ready[l & 1])
                out_host.copy_(o, non_blocking=True)
                counts["d2h"] += o.numel() * 2
                e = ev(); e.record(s_d2h); out_free[l & 1] = e

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    counts["h2d"] = counts["d2h"] = 0
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(s_h2d)
    s_cmp.wait_event(a); s_d2h.wait_event(a)
    for _ in range(steps):
        step()
    s_d2h.wait_stream(s_h2d); s_d2h.wait_stream(s_cmp)
    b.record(s_d2h)
    torch.cuda.synchronize()
    sala.check_status(s_cmp)
    ms = a.elapsed_time(b) / steps
    del host, dbuf, outs, out_host, kbar, idx
    torch.cuda.empty_cache()
    return {"ms_per_step": ms, "h2d": counts["h2d"] // steps, "d2h": counts["d2h"] // steps}


# ----------------------------------------------------------------------------------------------
# CPU baseline: the fp64 oracle on bounded samples, scaled to the full workloads.

def oracle_linear_layer(torch, synth, n_tok, budget_s):
    """Seconds of one linear layer (32 heads x n_tok tokens) in the oracle's chunked form, from a
    sample of `cores` heads; a 4096-token pilot sizes it to about 40 % of the budget."""
    import oracle
    cores = oracle.default_threads()
    hs = min(cores, H)
    lam = synth.decays(H)[:hs]
    f = oracle.from_tensor

    def lin_sample(n):
        q, k, v = synth.linear_layer(1, hs, n, D, torch.bfloat16, "cpu", layer=0)
        t0 = time.perf_counter()
        oracle.linear_chunked(f(q), f(k), f(v), f(lam), 64, threads=cores)
        return time.perf_counter() - t0

    n_lin = min(4096, n_tok)
    t_lin = lin_sample(n_lin)
    grow = int(min(n_tok // n_lin, max(1.0, 0.4 * budget_s / max(t_lin, 1e-6))))
    if grow > 1:
        n_lin *= 1 << (grow.bit_length() - 1)
        t_lin = lin_sample(n_lin)
    return {"s": t_lin * (H / hs) * (n_tok / n_lin), "cores": cores,
            "sample": f"{hs} heads x {n_lin} tokens (scaled x{H / hs:.0f} heads, x{n_tok / n_lin:g} length)"}


def oracle_sparse_layer(torch, synth, n_tok, budget_s):
    """Seconds of one sparse layer (selection + attention, 32 query heads over 2 KV heads) at n_tok
    tokens: sampled query rows from the second half of a 32768-token layer, the attention scaled by
    attended keys and the selection by candidate blocks."""
    import numpy as np
    import oracle
    cores = oracle.default_threads()
    f = oracle.from_tensor
    n_s = 32768
    sl = synth.sparse_layer(1, H, HKV, n_s, D, torch.bfloat16, "cpu", layer=3)
    q64, k64, v64 = f(sl.q), f(sl.k), f(sl.v)
    kbar = oracle.block_compress(k64, BLOCK)
    rng = np.random.default_rng(0)

    def sparse_sample(n_rows):
        rows_tok = np.sort(rng.choice(np.arange(n_s // 2, n_s), size=n_rows, replace=False))
        t0 = time.perf_counter()
        sel = []
        for r in rows_tok:
            ix, _ = oracle.block_select(q64[:, :, r:r + 1], kbar, BLOCK, TOPK, N_INIT, N_LOCAL,
                                        q_pos0=int(r), threads=1)
            sel.append(ix)
        t_sel = time.perf_counter() - t0
        idx = np.full((1, HKV, n_s, N_INIT + N_LOCAL + TOPK), -1, dtype=np.int32)
        for r, ix in zip(rows_tok, sel):
            idx[:, :, r] = ix[:, :, 0]
        rows = np.array([[h, r] for r in rows_tok for h in range(H)])
        t0 = time.perf_counter()
        oracle.sparse_attention(q64, k64, v64, idx, BLOCK, rows=rows, threads=cores)
        return rows_tok, t_sel, time.perf_counter() - t0

    n_rows = max(2 * cores, 32)
    rows_tok, t_sel, t_att = sparse_sample(n_rows)
    grow = int(min((n_s // 2) // n_rows, max(1.0, 0.4 * budget_s / max(t_sel + t_att, 1e-6))))
    if grow > 1:
        rows_tok, t_sel, t_att = sparse_sample(n_rows * grow)
    keys_sample = cand_sample = 0
    for r in rows_tok:
        c = r // BLOCK
        ncand = max(0, c - N_LOCAL + 1 - N_INIT)
        full_before = c if ncand <= TOPK else N_INIT + TOPK + N_LOCAL - 1
        keys_sample += full_before * BLOCK + (r % BLOCK) + 1
        cand_sample += ncand
    keys_full = attended_keys(n_tok)
    cand_full = sum(max(0, i // BLOCK - N_LOCAL + 1 - N_INIT) for i in range(0, n_tok, BLOCK)) * BLOCK
    return {"s": t_att * keys_full / keys_sample + t_sel * cand_full / cand_sample, "cores": cores,
            "sample": (f"selection + attention of {len(rows_tok)} query tokens x {H} heads sampled "
                       f"from the second half of a {n_s}-token layer (scaled to {n_tok} tokens by "
                       f"attended keys and candidate blocks)")}


def oracle_decode_token(torch, synth, T):
    """Seconds of one decode token at a T-token context in the oracle, at full size: a linear decode
    step (32 heads, 128 x 128 state) counted 24 times, and a sparse step counted 8 times --
    selection over the T/64 blocks' k_bar, then softmax attention over 67 blocks (a cache holding
    exactly those blocks' keys, so the attended work is that of the real step)."""
    import numpy as np
    import oracle
    f = oracle.from_tensor
    cores = oracle.default_threads()
    g = torch.Generator().manual_seed(5)
    lam = f(synth.decays(H))
    t_lin = 0.0
    for _ in range(2):
        S = torch.randn((1, H, D, D), generator=g, dtype=torch.float64).numpy() / D
        q, k, v = (f(torch.randn((1, H, D), generator=g).to(torch.bfloat16)) for _ in range(3))
        t0 = time.perf_counter()
        oracle.linear_decode(q, k, v, lam, S)
        t_lin += (time.perf_counter() - t0) / 2
    nb = T // BLOCK
    kbar = f(torch.randn((1, HKV, nb, D), generator=g).to(torch.bfloat16))
    qd = f(torch.randn((1, H, 1, D), generator=g).to(torch.bfloat16))
    t0 = time.perf_counter()
    oracle.block_select(qd, kbar, BLOCK, TOPK, N_INIT, N_LOCAL, q_pos0=T - 1, threads=cores)
    t_sel = time.perf_counter() - t0
    slots = N_INIT + N_LOCAL + TOPK
    n_c = slots * BLOCK
    kc = f(torch.randn((1, HKV, n_c, D), generator=g).to(torch.bfloat16))
    vc = f(torch.randn((1, HKV, n_c, D), generator=g).to(torch.bfloat16))
    idx = np.tile(np.arange(slots, dtype=np.int32), (1, HKV, 1, 1))
    t0 = time.perf_counter()
    oracle.sparse_attention(qd, kc, vc, idx, BLOCK, q_pos0=n_c - 1, threads=cores)
    t_att = time.perf_counter() - t0
    s = 24 * t_lin + 8 * (t_sel + t_att)
    return {"s": s, "cores": cores,
            "sample": (f"one token at full size, each kind of step timed once and counted per "
                       f"layer: 24 x linear decode step ({t_lin * 1e3:.2f} ms, mean of 2) + 8 x "
                       f"(selection over {nb} blocks {t_sel * 1e3:.1f} ms + attention over {slots} "
                       f"blocks {t_att * 1e3:.1f} ms)")}


def cpu_baseline(torch, synth, budget_s: float = 20.0):
    t_start = time.time()
    lin = oracle_linear_layer(torch, synth, N_TOK, budget_s)
    sp = oracle_sparse_layer(torch, synth, N_TOK, budget_s)
    step_s = 24 * lin["s"] + 8 * sp["s"]
    return {"value": N_TOK / step_s, "unit": "tokens/s", "cores": lin["cores"], "kind": "oracle",
            "sample": (f"linear: {lin['sample']}; sparse: {sp['sample']}; "
                       f"{time.time() - t_start:.1f} s of CPU work"),
            "step_s_extrapolated": step_s}


def config_lines(sala, synth, torch, stream, peaks, steps, warmup, decode=None, cpu=True,
                 budget_s=8.0):
    """One record per further benchmark configuration: the 32K linear prefill, the 128K sparse
    prefill and the 1M-context decode -- absolute throughput, roofline fraction and, on rank 0, the
    oracle timed on the host cores beside it."""
    out = {}
    hbm, tc = peaks["hbm_gbs"], peaks["bf16_tflops_sustained"]
    n = 32768
    pre = run_prefill(sala, synth, torch, steps, warmup, stream, "linear_prefill_n32k")
    ms = pre["total_ms"] / steps
    gbs = linear_layer_bytes(n) / (ms * 1e-3) / 1e9
    rec = {"workload": "linear_prefill_n32k: B=1, 32 heads, d=128, N=32768, bf16, chunk 64",
           "tokens_per_s": n / (ms * 1e-3), "ms": ms, "bound": "hbm", "achieved_gbs": gbs,
           "roofline_frac": gbs / hbm, "algorithmic_bytes": linear_layer_bytes(n)}
    if cpu:
        o = oracle_linear_layer(torch, synth, n, budget_s)
        rec["oracle"] = {"tokens_per_s": n / o["s"], "s": o["s"], "cores": o["cores"],
                         "sample": o["sample"]}
    out["linear_prefill_n32k"] = rec
    n = 131072
    pre = run_prefill(sala, synth, torch, steps, warmup, stream, "sparse_prefill_n128k")
    ms = pre["total_ms"] / steps
    fl = sparse_layer_flops(n)
    rec = {"workload": "sparse_prefill_n128k: B=1, 32 query / 2 KV heads, d=128, N=131072, bf16, "
                       "block 64, top-64 + init + 2 local (compress, select, attend)",
           "tokens_per_s": n / (ms * 1e-3), "ms": ms, "bound": "tensor",
           "attention_ms": pre["sparse_ms"], "selection_ms": pre["select_ms"],
           "achieved_tflops": fl / (pre["sparse_ms"] * 1e-3) / 1e12,
           "roofline_frac": fl / (pre["sparse_ms"] * 1e-3) / 1e12 / tc,
           "executed_frac": pre["sparse_exec_flops"] / (pre["sparse_ms"] * 1e-3) / 1e12 / tc,
           "algorithmic_flops": fl, "peak": f"{tc} TFLOP/s bf16 sustained ({peaks['source']})"}
    if cpu:
        o = oracle_sparse_layer(torch, synth, n, budget_s)
        rec["oracle"] = {"tokens_per_s": n / o["s"], "s": o["s"], "cores": o["cores"],
                         "sample": o["sample"]}
    out["sparse_prefill_n128k"] = rec
    n = N_TOK
    pre = run_prefill(sala, synth, torch, steps, warmup, stream, "sparse_per_head_prefill_n256k")
    ms = pre["total_ms"] / steps
    fl = sparse_layer_flops(n)
    out["sparse_per_head_prefill_n256k"] = {
        "workload": "sparse_per_head_prefill_n256k (selection variant): B=1, 32 query / 2 KV heads, "
                    "d=128, N=262144, bf16, block 64, top-64 + init + 2 local chosen per query head",
        "tokens_per_s": n / (ms * 1e-3), "ms": ms, "bound": "tensor",
        "attention_ms": pre["sparse_ms"], "selection_ms": pre["select_ms"],
        "achieved_tflops": fl / (pre["sparse_ms"] * 1e-3) / 1e12,
        "roofline_frac": fl / (pre["sparse_ms"] * 1e-3) / 1e12 / tc,
        "executed_frac": pre["sparse_exec_flops"] / (pre["sparse_ms"] * 1e-3) / 1e12 / tc,
        "union_overhead": pre["sparse_exec_flops"] / fl,
        "algorithmic_flops": fl, "peak": f"{tc} TFLOP/s bf16 sustained ({peaks['source']})"}
    if decode is not None:
        us = decode["us_per_token"]
        db = decode_bytes(DECODE_T)
        rec = {"workload": "decode_1m: one token through 24 linear + 8 sparse layers at a 2^20-token "
                           "context, batch 1",
               "tokens_per_s": 1e6 / us, "us_per_token": us, "bound": "hbm",
               "achieved_gbs": db["step"] / (us * 1e-6) / 1e9,
               "roofline_frac": db["step"] / (us * 1e-6) / 1e9 / hbm, "bytes_per_token": db["step"]}
        if cpu:
            o = oracle_decode_token(torch, synth, DECODE_T)
            rec["oracle"] = {"tokens_per_s": 1.0 / o["s"], "s": o["s"], "cores": o["cores"],
                             "sample": o["sample"]}
        out["decode_1m"] = rec
    return out


# ----------------------------------------------------------------------------------------------
def bench_config(ws: int) -> dict:
    return {"workload": "hybrid_prefill_n256k: 24 linear + 8 sparse layers, N=262144, "
                        "32 heads (2 KV heads in sparse layers), d=128, chunk 64, "
                        "block 64, top-64 + init + 2 local",
            "global_batch": ws, "seq_len": N_TOK,
            "parallelism": f"replicas x{ws}" if ws > 1 else "single GPU",
            "l2": "inputs larger than L2 (2 GiB per tensor); decode flushes L2 per step"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["sala", "reference"], default="sala")
    ap.add_argument("--cpu-budget", type=float, default=0.0,
                    help="seconds of oracle work per CPU-baseline sample (0: the default sizing)")
    ap.add_argument("--phases", default="prefill,decode,e2e,cpu,configs",
                    help="comma list of prefill,decode,e2e,cpu,configs,paged,backward,qknorm,"
                         "sparse_bwd (default: the first five)")
    ap.add_argument("--decode-steps", type=int, default=200)
    ap.add_argument("--decode-t", type=int, default=DECODE_T,
                    help="decode context length (default 2^20, the benchmark; smaller only for profiles)")
    ap.add_argument("--wait-limit-s", type=float, default=0.0,
                    help="bound of the kernels' device-side waits in seconds (0: the library's 2 s; "
                         "a profiler replaying kernels pass by pass needs more)")
    ap.add_argument("--bwd-n", type=int, default=N_TOK,
                    help="sequence length of the sparse_bwd phase (a smaller one for profiling)")
    ap.add_argument("--workload", default="hybrid_prefill_n256k", choices=sorted(WORKLOADS),
                    help="prefill workload (default: the 32-layer hybrid stack at 256K)")
    args = ap.parse_args()
    if args.workload != "hybrid_prefill_n256k" and "--phases" not in " ".join(sys.argv):
        args.phases = "prefill"
    phases = set(args.phases.split(","))

    import torch
    ws, rank, local = dist_env()

    if args.impl == "reference":
        if ws > 1:
            init_dist("gloo")
            if rank != 0:
                barrier()
                return
        from hybrid_sparse_linear_b200 import synth
        vals = []
        # each step a bounded sample, so that the whole arm stays within a few minutes
        budget = args.cpu_budget or max(5.0, min(20.0, 150.0 / (args.warmup + args.steps)))
        for i in range(args.warmup + args.steps):
            r = cpu_baseline(torch, synth, budget)
            if i >= args.warmup:
                vals.append(r)
        v = statistics.median(x["value"] for x in vals)
        # each step is a bounded sample scaled to the full step: ms_per_step is extrapolated
        line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s",
                "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": 1000.0 * N_TOK / v, "extrapolated": True,
                "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": bench_config(ws),
                "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": vals[-1]["cores"],
                                 "kind": "oracle", "sample": vals[-1]["sample"]},
                "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        if ws > 1:
            barrier()
        return

    if not torch.cuda.is_available():
        print(json.dumps({"error": "no CUDA device"}))
        sys.exit(1)
    torch.cuda.set_device(local)
    init_dist("nccl")
    from hybrid_sparse_linear_b200 import sala, synth
    if args.wait_limit_s > 0:
        sala.set_wait_limit_ns(int(args.wait_limit_s * 1e9))
    stream = torch.cuda.Stream()
    peaks = measured_peaks()
    line = {"metric": METRIC, "unit": "tokens/s", "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded normal Q/K/V per layer)",
            "config": bench_config(ws)}
    if "prefill" in phases:
        vis = [x for x in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",") if x.strip()]
        sampler = ClockSampler(vis[local] if local < len(vis) else str(local))
        sampler.start()
        pre = run_prefill(sala, synth, torch, args.steps, args.warmup, stream, args.workload)
        clocks = sampler.stop()
        n_tok, kinds = WORKLOADS[args.workload]
        ms = max_over_ranks(pre["total_ms"], "cuda") / args.steps
        line.update({"value": ws * n_tok / (ms / 1000.0), "ms_per_step": ms,
                     "gpu_launches": pre["launches"], "clocks": clocks})
        if args.workload != "hybrid_prefill_n256k":
            line["config"]["workload"] = f"{args.workload}: {len(kinds)} x {kinds[0]} layer, N={n_tok}"
            line["config"]["seq_len"] = n_tok
        line["kernels"] = {}
        if any(k.startswith("sparse") for k in kinds):
            fl = sparse_layer_flops(n_tok)
            achieved = fl / (pre["sparse_ms"] / 1000.0) / 1e12
            executed = pre["sparse_exec_flops"] / (pre["sparse_ms"] / 1000.0) / 1e12
            peak = peaks["bf16_tflops_sustained"]
            line["roofline"] = {"kernel": "sparse_prefill_tc_kernel", "bound": "tensor",
                                "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                                "frac": achieved / peak,
                                "traffic": sparse_traffic(n_tok) if "sparse" in kinds else None,
                                "peak_source": f"{peaks['source']} bf16 sustained",
                                "algorithmic_flops_per_launch": fl,
                                "mean_launch_ms": pre["sparse_ms"],
                                "executed_flops_per_launch": pre["sparse_exec_flops"],
                                "executed_tflops": executed, "executed_frac": executed / peak}
            line["kernels"]["sparse_prefill"] = {"mean_ms": pre["sparse_ms"], "achieved_tflops": achieved,
                                                 "executed_tflops": executed,
                                                 "union_overhead": pre["sparse_exec_flops"] / fl}
            line["kernels"]["compress_plus_select"] = {"mean_ms": pre["select_ms"]}
        if "linear" in kinds or "linear_rope" in kinds or "linear_rope_pro" in kinds:
            lin_gbs = linear_layer_bytes(n_tok) / (pre["linear_ms"] / 1000.0) / 1e9
            line["kernels"]["linear_prefill"] = {"mean_ms": pre["linear_ms"], "achieved_gbs": lin_gbs,
                                                 "hbm_frac": lin_gbs / peaks["hbm_gbs"]}
            if "sparse" not in kinds:
                line["roofline"] = {"kernel": "linear_prefill_tc_kernel", "bound": "hbm",
                                    "achieved": lin_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                    "frac": lin_gbs / peaks["hbm_gbs"], "traffic": None,
                                    "peak_source": f"{peaks['source']} HBM copy",
                                    "algorithmic_bytes_per_launch": linear_layer_bytes(n_tok),
                                    "mean_launch_ms": pre["linear_ms"]}
    if "backward" in phases:
        bw = run_linear_backward(sala, synth, torch, max(args.steps, 3), max(3, args.warmup), stream)
        gbs = bw["bytes"] / (bw["ms"] * 1e-3) / 1e9
        line["linear_backward"] = {"metric": "linear-attention backward ms per layer @256K (dq, dk, dv)",
                                   "ms": bw["ms"], "algorithmic_bytes": bw["bytes"],
                                   "achieved_gbs": gbs, "hbm_frac": gbs / peaks["hbm_gbs"],
                                   "composition": "three forward linear attentions (two of the "
                                                  "reversed sequence) and six row reversals"}
    if "sparse_bwd" in phases:
        sb = run_sparse_backward(sala, synth, torch, max(args.steps, 3), max(3, args.warmup), stream,
                                 args.bwd_n)
        ex = sb["exec_flops_dq"] + sb["exec_flops_dkv"]
        line["sparse_backward"] = {
            "metric": f"sparse-attention training step ms per layer @{args.bwd_n} (forward with "
                      "lse, then dq, dk, dv)",
            "forward_ms": sb["fwd_ms"], "backward_ms": sb["bwd_ms"],
            "algorithmic_tflops": sb["alg_flops"] / (sb["bwd_ms"] * 1e-3) / 1e12,
            "executed_tflops": ex / (sb["bwd_ms"] * 1e-3) / 1e12,
            "executed_tflop": {"dq_pass": sb["exec_flops_dq"] / 1e12, "dkv_pass": sb["exec_flops_dkv"] / 1e12},
            "algorithmic_tflop": sb["alg_flops"] / 1e12,
            "peak_tflops": peaks["bf16_tflops_sustained"],
            "timing": "CUDA events around back-to-back calls on resident inputs"}
    if "qknorm" in phases:
        qn = run_qk_norm(sala, synth, torch, max(args.steps, 5), max(3, args.warmup), stream)
        gbs = qn["bytes"] / (qn["ms"] * 1e-3) / 1e9
        line["qk_norm"] = {"metric": "QK normalisation ms per layer @256K (q and k, 32 heads each, "
                                     "in place)",
                           "ms": qn["ms"], "algorithmic_bytes": qn["bytes"], "achieved_gbs": gbs,
                           "hbm_frac": gbs / peaks["hbm_gbs"],
                           "timing": "CUDA events around back-to-back launches; 8.6 GB moved per "
                                     "launch, far above L2"}
    if "paged" in phases:
        pg = run_decode_paged(sala, synth, torch, args.decode_steps, max(3, args.warmup), stream)
        gbs = pg["bytes"] / (pg["us_per_call"] * 1e-6) / 1e9
        line["decode_paged"] = {"metric": "paged sparse decode us per call (8 sequences, own positions)",
                                "us_per_call": pg["us_per_call"], "sequence_tokens": pg["lengths"],
                                "bytes_per_call": pg["bytes"], "achieved_gbs": gbs,
                                "hbm_frac": gbs / peaks["hbm_gbs"],
                                "timing": "CUDA events around one CUDA-graph replay, L2 flushed "
                                          "before each, median"}
    if "decode" in phases:
        dec = run_decode(sala, synth, torch, args.decode_steps, max(3, args.warmup), stream, args.decode_t)
        db = decode_bytes(args.decode_t)
        gbs = db["step"] / (dec["us_per_token"] * 1e-6) / 1e9
        ctx = "1M" if args.decode_t == DECODE_T else str(args.decode_t)
        line["decode"] = {"metric": f"decode us/token @{ctx} (24 linear + 8 sparse layers)",
                          "us_per_token": dec["us_per_token"], "us_min": dec["us_min"],
                          "bytes_per_token": db["step"], "achieved_gbs": gbs,
                          "hbm_frac": gbs / peaks["hbm_gbs"],
                          "launches_per_token": dec["launches_per_token"],
                          "us_per_linear_layer": dec["us_per_linear_layer"],
                          "us_per_sparse_layer": dec["us_per_sparse_layer"],
                          "us_per_token_without_pdl": dec["us_per_token_without_pdl"],
                          "timing": "CUDA events around one CUDA-graph replay of a token's 32 layer "
                                    "calls, L2 flushed before each token, median; every layer "
                                    "launched as a programmatic dependent (linear state and sparse "
                                    "k_bar reads overlapping the previous layer); per-layer figures "
                                    "from graphs of one kind of call only"}
    dec_result = None
    if "decode" in phases:
        dec_result = {"us_per_token": line["decode"]["us_per_token"]}
    if "configs" in phases and args.workload == "hybrid_prefill_n256k":
        line["configs"] = config_lines(sala, synth, torch, stream, peaks, max(args.steps, 3),
                                       max(args.warmup, 3), dec_result,
                                       cpu=(rank == 0 and ws == 1), budget_s=args.cpu_budget or 8.0)
    if "e2e" in phases:
        e = run_e2e(sala, synth, torch, max(1, min(args.steps, 2)), 1)
        line["e2e"] = {"value": ws * N_TOK / (max_over_ranks(e["ms_per_step"], "cuda") / 1000.0),
                       "unit": "tokens/s", "h2d_bytes_per_step": e["h2d"],
                       "d2h_bytes_per_step": e["d2h"],
                       "note": "per layer: pinned host -> device copy of Q/K/V, the layer's calls, "
                               "device -> pinned host copy of O; copies on their own streams, "
                               "overlapping the neighbouring layers' kernels"}
    if "cpu" in phases and rank == 0 and ws == 1:
        line["cpu_baseline"] = cpu_baseline(torch, synth, args.cpu_budget or 20.0)
    if rank == 0:
        print(json.dumps(line), flush=True)
    barrier()
    import torch.distributed as dist
    if dist.is_initialized():
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
