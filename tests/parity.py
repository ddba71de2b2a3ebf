"""Comparison rules shared by the parity tests (test infrastructure, not collected).

Tolerances:
* bf16 inputs: max|err| <= 1e-2 * max|ref| + 1e-3 over the whole output tensor;
* fp32 inputs: max|err| <= 1e-5 * max|ref| (normwise relative).
Selection: the GPU and oracle block sets of a row may differ only by near-ties: each block in the
symmetric difference must score within 1e-3 relative of the oracle's k-th selected score,
|s_a - s_k| <= 1e-3 * max(|s_a|, |s_k|); forced blocks and set sizes must agree exactly.
"""
from __future__ import annotations

import numpy as np

import oracle


def tol_ok(out: np.ndarray, ref: np.ndarray, dtype: str):
    err = float(np.max(np.abs(out - ref))) if out.size else 0.0
    mref = float(np.max(np.abs(ref))) if ref.size else 0.0
    bound = (1e-2 * mref + 1e-3) if dtype == "bf16" else 1e-5 * mref
    return err <= bound, err, bound


def assert_close(out, ref, dtype: str, what: str = ""):
    out = np.asarray(out, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert out.shape == ref.shape, (out.shape, ref.shape)
    assert np.all(np.isfinite(out)), f"{what}: non-finite output"
    ok, err, bound = tol_ok(out, ref, dtype)
    assert ok, f"{what}: max|err| {err:.3e} > bound {bound:.3e}"
    return err, bound


def check_selection(gpu_idx, ref_idx, q64, kbar64, kth, topk, n_init, n_local, q_pos0=0,
                    block=64, rel=1e-3, row_ids=None):
    """gpu_idx/ref_idx: [B,Hkv,Nr,slots] (rows may be a subset: row_ids gives their index in q).
    Returns the number of rows that differ only by allowed near-ties."""
    gpu_idx = np.asarray(gpu_idx)
    ref_idx = np.asarray(ref_idx)
    assert gpu_idx.shape == ref_idx.shape, (gpu_idx.shape, ref_idx.shape)
    diff_rows = np.argwhere(np.any(gpu_idx != ref_idx, axis=-1))
    quads, checks = [], []
    for b, g, r in diff_rows:
        rr = int(row_ids[r]) if row_ids is not None else int(r)
        a = [x for x in gpu_idx[b, g, r] if x >= 0]
        e = [x for x in ref_idx[b, g, r] if x >= 0]
        assert a == sorted(set(a)), f"row {(b, g, rr)} not strictly ascending: {a}"
        assert len(a) == len(e), f"row {(b, g, rr)}: {len(a)} vs {len(e)} blocks"
        pos = q_pos0 + rr
        c = pos // block
        forced = set(range(min(n_init, c + 1))) | set(range(max(0, c - n_local + 1), c + 1))
        assert forced <= set(a), f"row {(b, g, rr)} misses forced blocks"
        sym = sorted(set(a) ^ set(e))
        for x in sym:
            assert n_init <= x <= c - n_local, f"row {(b, g, rr)}: block {x} is not a candidate"
            quads.append((b, g, rr, x))
            checks.append((b, g, r))
    if quads:
        s = oracle.block_scores_at(q64, kbar64, np.array(quads))
        for (b, g, r), sc, quad in zip(checks, s, quads):
            sk = kth[b, g, r]
            assert np.isfinite(sk), f"row {quad[:3]}: differing sets with fewer than k candidates"
            assert abs(sc - sk) <= rel * max(abs(sc), abs(sk)), \
                f"row {quad[:3]} block {quad[3]}: score {sc} vs k-th {sk} is not a near-tie"
    return len(diff_rows)
