"""Host-side accounting of bench.py, on the CPU.

The roofline fractions the bench reports divide work counts by measured times, so the counts are
pinned here against independent computations:
  - attended_keys (the closed form behind the sparse layer's algorithmic FLOPs) against the keys
    the oracle's own selections attend, counted block by block;
  - tile_union_blocks (the executed work of the union walk) against Python set unions;
  - the reference arm's JSON line (run here: it times only the oracle) for the contract's keys.
"""
import json
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _keys_from_selection(idx, block):
    """Sum over rows of the keys a row attends: per chosen block, its keys at or before the row."""
    B, G, N, S = idx.shape
    total = np.zeros((B, G), dtype=np.int64)
    for i in range(N):
        blk = idx[:, :, i, :].astype(np.int64)
        keys = np.where(blk >= 0, np.minimum(block, i - blk * block + 1), 0)
        assert (keys[blk >= 0] >= 1).all(), "a chosen block lies after its row"
        total += keys.sum(axis=-1)
    return total


@pytest.mark.parametrize("N,topk,n_init,n_local", [
    (64 * 9 + 17, 3, 1, 2),      # ragged tail, rows with and without more candidates than k
    (64 * 12, 4, 2, 1),          # whole blocks, two init blocks, a local window of one
    (40, 2, 1, 2),               # a single partial block
])
def test_attended_keys_matches_the_oracle_selection(N, topk, n_init, n_local):
    from hybrid_sparse_linear_b200 import synth
    layer = synth.sparse_layer(1, 4, 2, N, 32, torch.float32, layer=41)
    q64, k64 = oracle.from_tensor(layer.q), oracle.from_tensor(layer.k)
    kbar = oracle.block_compress(k64, 64, round_to_bf16=False) if N >= 64 else \
        np.zeros((1, 2, 0, 32))
    idx, _ = oracle.block_select(q64, kbar, 64, topk, n_init, n_local)
    got = _keys_from_selection(idx, 64)
    want = bench.attended_keys(N, topk=topk, n_init=n_init, n_local=n_local, block=64)
    assert (got == want).all(), (got, want)


def test_sparse_layer_flops_counts_both_products_for_every_head():
    n = 64 * 5 + 3
    assert bench.sparse_layer_flops(n) == 4.0 * bench.D * bench.H * bench.attended_keys(n)


def _union_brute(idx, tq, heads):
    B, Hq, N, S = idx.shape
    total = 0
    for b in range(B):
        for g in range(Hq // heads):
            for t0 in range(0, N, tq):
                rows = idx[b, g * heads:(g + 1) * heads, t0:t0 + tq].reshape(-1)
                total += len({int(x) for x in rows if x >= 0})
    return total


@pytest.mark.parametrize("heads", [1, 4])
def test_tile_union_blocks_matches_set_unions(heads):
    rng = np.random.default_rng(5)
    B, G, N, S = 2, 3, 8 * 7 + 5, 6           # ragged last tile
    idx = rng.integers(-1, 20, size=(B, G * heads, N, S)).astype(np.int32)
    idx[0, 0, 3] = -1                          # a row with no block at all
    want = _union_brute(idx, 8, heads)
    got = bench.tile_union_blocks(torch, torch.from_numpy(idx), 8, heads=heads)
    assert got == want


def test_tile_union_of_identical_rows_is_one_row():
    row = np.array([0, 3, 7, -1, 9], dtype=np.int32)
    idx = np.broadcast_to(row, (1, 2, 16, 5)).copy()
    assert bench.tile_union_blocks(torch, torch.from_numpy(idx), 8) == 2 * 2 * 4


def test_reference_arm_prints_the_contract_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0", "--cpu-budget", "1"],
                       capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["metric"] == bench.METRIC and line["unit"] == "tokens/s"
    assert line["higher_is_better"] is True and line["extrapolated"] is True
    assert line["config"] == bench.bench_config(1)
    assert line["value"] > 0 and line["cpu_baseline"]["value"] == line["value"]
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"] == {"value": line["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    assert abs(line["ms_per_step"] - 1000.0 * bench.N_TOK / line["value"]) < 1e-6 * line["ms_per_step"]
