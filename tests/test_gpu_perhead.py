"""GPU parity of the per-query-head selection variant (sala_block_topk_per_head and
sala_sparse_prefill_per_head) against the fp64 oracle, through the C ABI.

Selections are checked with the near-tie rule of tests/parity.py, each head its own group of one
(the oracle's kbar repeated per head).  Attention is checked on the GPU's own per-head selection.
The tensor-core attention walks each 16-token unit's union over 16 heads x 16 tokens and masks
every row to its own blocks, so the cases below include selections that agree across heads
(the union of the group path), that differ per head, that are padded mid-row, and that cover
every block (the widest union)."""
import numpy as np
import pytest
import torch

import oracle
from parity import assert_close, check_selection

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sala():
    from hybrid_sparse_linear_b200 import sala as s
    return s


def _f64(t):
    return oracle.from_tensor(t)


def _per_head_pipeline(sala, layer, kind, topk, n_init, n_local):
    q, k, v = layer.q.cuda(), layer.k.cuda(), layer.v.cuda()
    H, Hkv = q.shape[1], k.shape[1]
    kbar = sala.block_compress(k)
    idx = sala.block_topk_per_head(q, kbar, topk, n_init, n_local)
    o = sala.sparse_prefill_per_head(q, k, v, idx)
    sala.check_status()
    q64, k64, v64 = _f64(layer.q), _f64(layer.k), _f64(layer.v)
    kbar_ref = oracle.block_compress(k64, 64, round_to_bf16=(kind == "bf16"))
    if kind == "f32":
        kbar_ref = kbar_ref.astype(np.float32).astype(np.float64)
    np.testing.assert_array_equal(_f64(kbar), kbar_ref)
    idx_ref, kth = oracle.block_select_per_head(q64, kbar_ref, 64, topk, n_init, n_local)
    got = idx.cpu().numpy()
    assert got.shape == idx_ref.shape
    kbar_h = np.repeat(kbar_ref, H // Hkv, axis=1)   # head h scores against its KV head's kbar
    ndiff = check_selection(got, idx_ref, q64, kbar_h, kth, topk, n_init, n_local)
    o_ref = oracle.sparse_attention_per_head(q64, k64, v64, got, 64)
    assert_close(_f64(o), o_ref, kind, "o")
    return got, ndiff


@pytest.mark.parametrize("N,topk,n_local", [(64 * 70 + 17, 16, 2), (64 * 40, 64, 2),
                                             (100, 4, 2), (64 * 9 + 1, 3, 1)])
def test_bf16_per_head_pipeline_gqa16(sala, N, topk, n_local):
    from hybrid_sparse_linear_b200 import synth
    layer = synth.sparse_layer(1, 32, 2, N, 128, torch.bfloat16, layer=21, shift_frac=0.05)
    got, _ = _per_head_pipeline(sala, layer, "bf16", topk, 1, n_local)
    # the heads of a group do not all agree (else this would only test the group path's union)
    c = (N - 1) // 64
    if c - n_local + 1 - 1 > topk:
        assert (got[0, :16, N - 1] != got[0, :1, N - 1]).any()


def test_bf16_per_head_batch2_short_rows(sala):
    # batch 2, fewer than 17 query rows (the CUDA-core selection), two KV heads.
    from hybrid_sparse_linear_b200 import synth
    layer = synth.sparse_layer(2, 32, 2, 13, 128, torch.bfloat16, layer=22)
    _per_head_pipeline(sala, layer, "bf16", 2, 1, 1)


def test_fp32_and_d64_per_head_cuda_core_paths(sala):
    from hybrid_sparse_linear_b200 import synth
    layer = synth.sparse_layer(1, 8, 2, 64 * 12 + 5, 128, torch.float32, layer=23, shift_frac=0.1)
    _per_head_pipeline(sala, layer, "f32", 3, 1, 2)
    layer = synth.sparse_layer(1, 8, 2, 64 * 20 + 3, 64, torch.bfloat16, layer=24, shift_frac=0.1)
    _per_head_pipeline(sala, layer, "bf16", 5, 1, 2)


def test_equal_heads_give_the_group_attention_bitwise(sala):
    # Every head of a group given the group's selection: the per-head union and row masks equal
    # the group path's, so the two tensor-core walks run the same MMAs and exponentials.
    from hybrid_sparse_linear_b200 import synth
    N = 64 * 50 + 9
    layer = synth.sparse_layer(1, 32, 2, N, 128, torch.bfloat16, layer=25, shift_frac=0.05)
    q, k, v = layer.q.cuda(), layer.k.cuda(), layer.v.cuda()
    kbar = sala.block_compress(k)
    idx_g = sala.block_topk(q, kbar, 16, 1, 2)
    idx_h = idx_g.repeat_interleave(16, dim=1).contiguous()
    o_g = sala.sparse_prefill(q, k, v, idx_g)
    o_h = sala.sparse_prefill_per_head(q, k, v, idx_h)
    sala.check_status()
    assert torch.equal(o_g, o_h)


def _given_idx(rng, B, H, N, slots, n_pick, pad_mid):
    """Random per-head rows: each row picks n_pick distinct blocks of 0..c (always c), ascending,
    -1 padded; with pad_mid the -1 slots are scattered among the blocks instead of trailing."""
    idx = np.full((B, H, N, slots), -1, dtype=np.int32)
    for b in range(B):
        for h in range(H):
            for i in range(N):
                c = i // 64
                m = min(n_pick, c + 1)
                pick = np.sort(np.concatenate([[c], rng.choice(c, m - 1, replace=False)])) \
                    if c > 0 else np.array([0])
                row = np.full(slots, -1, dtype=np.int32)
                if pad_mid:
                    pos = np.sort(rng.choice(slots, len(pick), replace=False))
                    row[pos] = pick
                else:
                    row[:len(pick)] = pick
                idx[b, h, i] = row
    return idx


@pytest.mark.parametrize("n_pick,pad_mid", [(6, True), (40, False)])
def test_given_per_head_selection(sala, n_pick, pad_mid):
    # n_pick 40 of at most 30 blocks: every row takes all its blocks (the widest union); 6 blocks
    # per row, padded mid-row, gives each (head, token) its own random set.
    from hybrid_sparse_linear_b200 import synth
    N = 64 * 29 + 50
    layer = synth.sparse_layer(1, 32, 2, N, 128, torch.bfloat16, layer=26)
    rng = np.random.default_rng(7)
    idx = _given_idx(rng, 1, 32, N, 48, n_pick, pad_mid)
    o = sala.sparse_prefill_per_head(layer.q.cuda(), layer.k.cuda(), layer.v.cuda(),
                                     torch.from_numpy(idx).cuda())
    sala.check_status()
    o_ref = oracle.sparse_attention_per_head(_f64(layer.q), _f64(layer.k), _f64(layer.v), idx, 64)
    assert_close(_f64(o), o_ref, "bf16", "o")


def test_per_head_out_of_range_index_is_flagged(sala):
    from hybrid_sparse_linear_b200 import synth
    layer = synth.sparse_layer(1, 32, 2, 256, 128, torch.bfloat16, layer=27)
    idx = torch.full((1, 32, 256, 3), -1, dtype=torch.int32)
    idx[..., 0] = 0
    idx[0, 17, 5, 1] = 3  # block 3 is in the future of row 5
    o = sala.sparse_prefill_per_head(layer.q.cuda(), layer.k.cuda(), layer.v.cuda(), idx.cuda())
    with pytest.raises(sala.SalaError) as ei:
        sala.check_status()
    assert ei.value.code == sala.ERR_BOUNDS
    assert torch.isfinite(o.float()).all()
    sala.check_status()


def test_bf16_per_head_batch2_tensor_core_paths(sala):
    # batch 2 through the tensor-core selection (more than 16 rows) and attention
    from hybrid_sparse_linear_b200 import synth
    layer = synth.sparse_layer(2, 32, 2, 64 * 10 + 7, 128, torch.bfloat16, layer=28, shift_frac=0.1)
    _per_head_pipeline(sala, layer, "bf16", 8, 1, 2)


def test_per_head_top0_forced_blocks_only(sala):
    # k = 0: rows of three slots (init + two local), shorter than the four-entry look-ahead each
    # softmax thread keeps over its own row
    from hybrid_sparse_linear_b200 import synth
    layer = synth.sparse_layer(1, 32, 2, 64 * 7 + 33, 128, torch.bfloat16, layer=29)
    got, _ = _per_head_pipeline(sala, layer, "bf16", 0, 1, 2)
    assert got.shape[-1] == 3
