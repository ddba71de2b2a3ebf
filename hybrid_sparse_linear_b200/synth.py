"""Seeded synthetic inputs for the SALA hybrid attention forward.

This module only draws random numbers and lays them out; it holds none of the method's
arithmetic.  The same tensors feed the CUDA path and the fp64 oracle (which reads them back to
the host), so both sides always see identical values.

Recipe (every draw is a standard normal from torch's Philox generator):

* ``seed(base, layer, what)`` = ``base + 1000 * layer + what`` with what = 0 (Q), 1 (K), 2 (V),
  3 (u, the per-group shift direction), 4 (choice of shifted blocks).  ``base`` defaults to
  20260212.
* each ``[b, h]`` slice of a tensor is drawn on its own generator, seeded
  ``seed * 4096 + b * heads + h``, so huge tensors are drawn slice by slice with bounded
  temporary memory and any slice can be regenerated alone.
* linear-attention layers: Q, K, V ~ N(0, 1) / sqrt(d); per-head decay
  ``lambda_h = exp(-2^(-8 (h+1) / H))`` (0.431 ... 0.9961 at H = 32), or the two fixed decays
  0.99 / 0.999 of the tiny fp32 case.
* decode draws queries only for the last ``q_rows`` positions (a [.., q_rows, d] tensor seeded
  like the others).
* sparse-attention layers: K ~ N(0, 1); round(0.02 * n_blocks) complete blocks per (batch, KV
  head), chosen without replacement, get ``3 u`` added to every key row; Q ~ N(0, 1) + u for
  every query head of the group; V ~ N(0, 1); u ~ N(0, I_d), one per (layer, batch, KV head).
  The tiny fp32 case instead uses Q, K, V ~ N(0, 1) / sqrt(d) with no shift.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

BASE_SEED = 20260212
Q, K, V, U, MASK = 0, 1, 2, 3, 4


def seed(layer: int, what: int, base: int = BASE_SEED) -> int:
    return base + 1000 * layer + what


def _gen(device, s: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(s)
    return g


def normal(shape, s: int, device="cpu", dtype=torch.float32, scale: float = 1.0,
           add=None) -> torch.Tensor:
    """[B, heads, rows, d] standard normals * scale (+ add[b, h] broadcast over rows), per-slice
    seeded, materialised in ``dtype`` on ``device``."""
    B, Hh, N, d = shape
    out = torch.empty(shape, device=device, dtype=dtype)
    for b in range(B):
        for h in range(Hh):
            x = torch.randn((N, d), generator=_gen(device, s * 4096 + b * Hh + h),
                            device=device, dtype=torch.float32)
            if scale != 1.0:
                x.mul_(scale)
            if add is not None:
                x.add_(add[b, h].to(device=device, dtype=torch.float32))
            out[b, h].copy_(x)
    return out


def prenorm(shape, s: int, device="cpu", dtype=torch.float32, spread: float = 3.0) -> torch.Tensor:
    """q or k ahead of the QK normalisation: [B, heads, rows, d] standard normals, each row
    scaled by e^u with u uniform in [-spread, spread] (row magnitudes from e^-3 to e^3)."""
    x = normal(shape, s, device, torch.float32)
    u = (torch.rand(tuple(shape[:-1]) + (1,), generator=_gen("cpu", s * 7919 + 1)) * 2 - 1) * spread
    return (x * torch.exp(u).to(device)).to(dtype)


def decays(H: int, kind: str = "geometric") -> torch.Tensor:
    """Per-head decay lambda_h as fp32 (an input of the method, not part of it)."""
    if kind == "tiny":
        assert H == 2
        return torch.tensor([0.99, 0.999], dtype=torch.float32)
    h = torch.arange(H, dtype=torch.float64)
    return torch.exp(-torch.pow(2.0, -8.0 * (h + 1) / H)).to(torch.float32)


def linear_layer(B, H, N, d, dtype, device="cpu", layer=0, base=BASE_SEED):
    sc = 1.0 / math.sqrt(d)
    q = normal((B, H, N, d), seed(layer, Q, base), device, dtype, sc)
    k = normal((B, H, N, d), seed(layer, K, base), device, dtype, sc)
    v = normal((B, H, N, d), seed(layer, V, base), device, dtype, sc)
    return q, k, v


@dataclass
class SparseLayer:
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    shifted: list = field(default_factory=list)   # [b][g] -> sorted list of shifted block ids
    u: torch.Tensor | None = None                 # [B, Hkv, d] fp32


def sparse_layer(B, H, Hkv, N, d, dtype, device="cpu", layer=0, block=64, shift_frac=0.02,
                 shift_mult=3.0, base=BASE_SEED, q_rows=None) -> SparseLayer:
    """q_rows: draw queries only for the last q_rows positions (decode), Q is [B, H, q_rows, d]."""
    G = H // Hkv
    nb = N // block
    gu = _gen("cpu", seed(layer, U, base))
    u = torch.randn((B, Hkv, d), generator=gu, dtype=torch.float32)
    gm = _gen("cpu", seed(layer, MASK, base))
    n_shift = int(round(shift_frac * nb))
    shifted = [[sorted(torch.randperm(nb, generator=gm)[:n_shift].tolist()) for _ in range(Hkv)]
               for _ in range(B)]
    k = normal((B, Hkv, N, d), seed(layer, K, base), device, dtype)
    for b in range(B):
        for g in range(Hkv):
            if not shifted[b][g]:
                continue
            shift = (shift_mult * u[b, g]).to(device)
            rows = torch.cat([torch.arange(blk * block, (blk + 1) * block) for blk in shifted[b][g]])
            rows = rows.to(device)
            kk = k[b, g].index_select(0, rows).float() + shift
            k[b, g].index_copy_(0, rows, kk.to(dtype))
    uq = u.repeat_interleave(G, dim=1)  # [B, H, d]
    q = normal((B, H, q_rows or N, d), seed(layer, Q, base), device, dtype, 1.0, add=uq)
    v = normal((B, Hkv, N, d), seed(layer, V, base), device, dtype)
    return SparseLayer(q, k, v, shifted, u)


def tiny_sparse_layer(B, H, Hkv, N, d, dtype, device="cpu", layer=0, base=BASE_SEED) -> SparseLayer:
    sc = 1.0 / math.sqrt(d)
    q = normal((B, H, N, d), seed(layer, Q, base), device, dtype, sc)
    k = normal((B, Hkv, N, d), seed(layer, K, base), device, dtype, sc)
    v = normal((B, Hkv, N, d), seed(layer, V, base), device, dtype, sc)
    return SparseLayer(q, k, v, [], None)


# Named workloads, by what they are.  Sizes follow the hybrid attention of the pages' 9B model
# (32 query heads, head dim 128; GQA 16:1 in the sparse layers; 3 linear : 1 sparse).
WORKLOADS = {
    "tiny_fp32_n512": dict(B=1, H=2, Hkv=2, d=64, N=512, dtype="f32", chunk=64, block=64,
                           topk=2, n_init=1, n_local=1, decay="tiny"),
    "linear_prefill_n32k": dict(B=1, H=32, d=128, N=32768, dtype="bf16", chunk=64),
    "sparse_prefill_n128k": dict(B=1, H=32, Hkv=2, d=128, N=131072, dtype="bf16", block=64,
                                 topk=64, n_init=1, n_local=2),
    "hybrid_prefill_n256k": dict(B=1, H=32, Hkv=2, d=128, N=262144, dtype="bf16", chunk=64,
                                 block=64, topk=64, n_init=1, n_local=2, n_linear=24, n_sparse=8),
    "decode_1m": dict(B=1, H=32, Hkv=2, d=128, T=1 << 20, dtype="bf16", block=64, topk=64,
                      n_init=1, n_local=2, n_linear=24, n_sparse=8),
}
