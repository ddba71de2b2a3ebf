"""Full-size parity in the launch configuration the benchmark times: one sparse layer at
N = 131072 and 262144 (32 query heads, 2 KV heads, d 128, top-64 + init + 2 local), the same with
per-head selections at 262144, and one linear layer at N = 262144.  The oracle checks sampled outputs one by one (first/last rows, block and tile
boundaries, the row where top-k starts to bind, random rows); compression is checked on every
block, selection on the sampled rows with the near-tie rule."""
import numpy as np
import pytest
import torch

import oracle
from parity import assert_close, check_selection

pytestmark = pytest.mark.gpu

TOPK, N_INIT, N_LOCAL = 64, 1, 2


def _rows(N, seed):
    fixed = [0, 1, 7, 8, 63, 64, 65, 127, 128, 64 * 66 - 1, 64 * 67, 64 * 67 + 1, N // 2,
             N // 2 + 5, N - 65, N - 64, N - 9, N - 8, N - 1]
    rng = np.random.default_rng(seed)
    rnd = rng.integers(0, N, size=24).tolist()
    return sorted(set(r for r in fixed + rnd if 0 <= r < N))


@pytest.mark.parametrize("N", [131072, 262144])
def test_sparse_layer_full_size(N):
    from hybrid_sparse_linear_b200 import sala, synth
    layer = synth.sparse_layer(1, 32, 2, N, 128, torch.bfloat16, "cuda", layer=7)
    kbar = sala.block_compress(layer.k)
    idx = sala.block_topk(layer.q, kbar, TOPK, N_INIT, N_LOCAL)
    o = sala.sparse_prefill(layer.q, layer.k, layer.v, idx)
    sala.check_status()
    f = oracle.from_tensor
    k64, v64 = f(layer.k), f(layer.v)
    kbar_ref = oracle.block_compress(k64, 64)
    np.testing.assert_array_equal(f(kbar), kbar_ref)
    rows = _rows(N, N)
    gidx = idx.cpu().numpy()
    got, ref = [], []
    for r in rows:
        q64 = f(layer.q[:, :, r:r + 1])
        ridx, kth = oracle.block_select(q64, kbar_ref, 64, TOPK, N_INIT, N_LOCAL, q_pos0=r)
        check_selection(gidx[:, :, r:r + 1], ridx, q64, kbar_ref, kth, TOPK, N_INIT, N_LOCAL,
                        q_pos0=r, row_ids=np.array([0]))
        ref.append(oracle.sparse_attention(q64, k64, v64, gidx[:, :, r:r + 1], 64, q_pos0=r)[0, :, 0])
        got.append(f(o[0, :, r]))
    assert_close(np.stack(got), np.stack(ref), "bf16", f"sparse N={N} sampled rows")


def test_sparse_layer_per_head_full_size():
    # the per-query-head variant at the benchmark's N = 262144: selection rows per head, each head
    # checked against the oracle's per-head selection (a group of one, its KV head's kbar), and
    # the attention over every head's own blocks on sampled rows
    from hybrid_sparse_linear_b200 import sala, synth
    N = 262144
    layer = synth.sparse_layer(1, 32, 2, N, 128, torch.bfloat16, "cuda", layer=8)
    kbar = sala.block_compress(layer.k)
    idx = sala.block_topk_per_head(layer.q, kbar, TOPK, N_INIT, N_LOCAL)
    o = sala.sparse_prefill_per_head(layer.q, layer.k, layer.v, idx)
    sala.check_status()
    f = oracle.from_tensor
    k64, v64 = f(layer.k), f(layer.v)
    kbar_ref = oracle.block_compress(k64, 64)
    np.testing.assert_array_equal(f(kbar), kbar_ref)
    kbar_h = np.repeat(kbar_ref, 16, axis=1)
    rows = _rows(N, N + 1)
    gidx = idx.cpu().numpy()
    got, ref = [], []
    for r in rows:
        q64 = f(layer.q[:, :, r:r + 1])
        ridx, kth = oracle.block_select_per_head(q64, kbar_ref, 64, TOPK, N_INIT, N_LOCAL, q_pos0=r)
        check_selection(gidx[:, :, r:r + 1], ridx, q64, kbar_h, kth, TOPK, N_INIT, N_LOCAL,
                        q_pos0=r, row_ids=np.array([0]))
        ref.append(oracle.sparse_attention_per_head(q64, k64, v64, gidx[:, :, r:r + 1], 64,
                                                    q_pos0=r)[0, :, 0])
        got.append(f(o[0, :, r]))
    assert_close(np.stack(got), np.stack(ref), "bf16", "per-head sparse N=262144 sampled rows")


def test_linear_layer_full_size():
    from hybrid_sparse_linear_b200 import sala, synth
    N, H, d = 262144, 32, 128
    q, k, v = synth.linear_layer(1, H, N, d, torch.bfloat16, "cuda", layer=1)
    lam = synth.decays(H).cuda()
    o = sala.linear_prefill(q, k, v, lam)
    sala.check_status()
    heads = [0, 13, 31]
    toks = [0, 1, 63, 64, 65, 127, 128, 131071, 131072, N - 129, N - 128, N - 1]
    sub = lambda t: oracle.from_tensor(t[:, heads])
    rows = np.array([[hi, t] for hi in range(len(heads)) for t in toks])
    ref = oracle.linear_quadratic(sub(q), sub(k), sub(v), oracle.from_tensor(lam.cpu()[heads]),
                                  rows=rows)
    got = np.stack([oracle.from_tensor(o[0, heads[hi], t]) for hi, t in rows])
    assert_close(got, ref, "bf16", "linear N=262144 sampled rows")


def test_linear_rope_layer_full_size():
    # the RoPE linear layer at N = 262144 in the launch configuration the benchmark times
    # (parallel segments), sampled rows against the oracle's quadratic form on rotated q, k
    from hybrid_sparse_linear_b200 import sala, synth
    N, H, d = 262144, 32, 128
    q, k, v = synth.linear_layer(1, H, N, d, torch.bfloat16, "cuda", layer=2)
    lam = synth.decays(H).cuda()
    ws = torch.empty(max(sala.linear_prefill_workspace_bytes(1, H, N, d), 16), dtype=torch.uint8,
                     device="cuda")
    o = sala.linear_prefill(q, k, v, lam, workspace=ws, rope_base=10000.0, pos0=0)
    sala.check_status()
    heads = [0, 21]
    toks = [0, 1, 127, 128, 16383, 16384, 131071, N - 129, N - 1]
    sub = lambda t: oracle.from_tensor(t[:, heads])
    rows = np.array([[hi, t] for hi in range(len(heads)) for t in toks])
    ref = oracle.linear_quadratic(oracle.rope(sub(q), 0), oracle.rope(sub(k), 0), sub(v),
                                  oracle.from_tensor(lam.cpu()[heads]), rows=rows)
    got = np.stack([oracle.from_tensor(o[0, heads[hi], t]) for hi, t in rows])
    assert_close(got, ref, "bf16", "RoPE linear N=262144 sampled rows")
