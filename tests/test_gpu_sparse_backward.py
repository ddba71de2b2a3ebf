"""GPU parity of the sparse attention's training path (sala_sparse_prefill_lse and
sala_sparse_backward) against the fp64 oracle, through the C ABI.

The selection comes from the GPU (sala_block_topk) and is held fixed: the oracle differentiates the
softmax over exactly the blocks the GPU chose.  dq, dk, dv are compared element by element with the
bf16 tolerance of tests/parity.py; lse within 2e-3 absolute (the forward sums its exponentials in
fp32, a quarter of them through a polynomial exp2 of relative error <= 8e-5).  At N = 32768 the check
is sampled dq rows plus the two column identities of softmax attention (per KV group, the dk rows
sum to zero and the dv rows to the group's summed dout).
"""
import numpy as np
import pytest
import torch

import oracle
from parity import assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sala():
    from hybrid_sparse_linear_b200 import sala as s
    return s


def _f64(t):
    return oracle.from_tensor(t)


def _layer(B, Hkv, N, seed):
    from hybrid_sparse_linear_b200 import synth
    layer = synth.sparse_layer(B, 16 * Hkv, Hkv, N, 128, torch.bfloat16, layer=seed, shift_frac=0.05)
    dout = synth.normal((B, 16 * Hkv, N, 128), synth.seed(seed, 7), "cpu", torch.bfloat16)
    return layer.q, layer.k, layer.v, dout


def _run(sala, q, k, v, dout, topk, n_local=2):
    qd, kd, vd, dd = q.cuda(), k.cuda(), v.cuda(), dout.cuda()
    kbar = sala.block_compress(kd)
    idx = sala.block_topk(qd, kbar, topk, 1, n_local)
    o, lse, o_lo = sala.sparse_prefill(qd, kd, vd, idx, lse=True, o_lo=True)
    dq, dk, dv = sala.sparse_backward(qd, kd, vd, idx, o, lse, dd, o_lo=o_lo)
    sala.check_status()
    return idx.cpu().numpy(), o, lse, dq, dk, dv, o_lo


@pytest.mark.parametrize("B,Hkv,N,topk", [(1, 2, 1000, 4), (1, 2, 333, 64), (2, 1, 200, 2),
                                          (1, 1, 40, 4), (1, 2, 2048, 8)])
def test_backward_matches_oracle(sala, B, Hkv, N, topk):
    q, k, v, dout = _layer(B, Hkv, N, 5 + N % 7)
    idx, o, lse, dq, dk, dv, o_lo = _run(sala, q, k, v, dout, topk)
    q64, k64, v64, do64 = _f64(q), _f64(k), _f64(v), _f64(dout)
    # the training forward's o + o_lo carries o to ~2^-16 (P V as P_hi V + P_lo V)
    o_ref = oracle.sparse_attention(q64, k64, v64, idx, 64)
    err = np.abs(_f64(o) + _f64(o_lo) - o_ref).max()
    assert err <= 2e-4 * np.abs(o_ref).max(), f"o + o_lo max error {err}"
    assert_close(_f64(o), o_ref, "bf16", "o")
    lse_ref = oracle.sparse_lse(q64, k64, idx, 64)
    err = np.abs(_f64(lse) - lse_ref)
    assert err.max() <= 2e-3, f"lse max error {err.max()}"
    dq_ref, dk_ref, dv_ref = oracle.sparse_attention_backward(q64, k64, v64, idx, do64, 64)
    assert_close(_f64(dq), dq_ref, "bf16", "dq")
    assert_close(_f64(dk), dk_ref, "bf16", "dk")
    assert_close(_f64(dv), dv_ref, "bf16", "dv")


def test_future_block_is_flagged(sala):
    q, k, v, dout = _layer(1, 1, 256, 3)
    qd, kd, vd, dd = q.cuda(), k.cuda(), v.cuda(), dout.cuda()
    idx = sala.block_topk(qd, sala.block_compress(kd), 2, 1, 1)
    o, lse, _ = sala.sparse_prefill(qd, kd, vd, idx, lse=True)
    sala.check_status()
    bad = idx.clone()
    bad[0, 0, 5, 2] = 3  # token 5 sits in block 0; block 3 is in its future
    sala.sparse_backward(qd, kd, vd, bad, o, lse, dd)
    with pytest.raises(sala.SalaError) as e:
        sala.check_status()
    assert e.value.code == sala.ERR_BOUNDS


def test_full_size_32k_sampled(sala):
    B, Hkv, N, topk = 1, 2, 32768, 64
    q, k, v, dout = _layer(B, Hkv, N, 9)
    idx, o, lse, dq, dk, dv, _ = _run(sala, q, k, v, dout, topk)
    g = np.random.default_rng(4)
    rows = np.stack([np.zeros(48, dtype=np.int64), g.integers(0, 32, 48), g.integers(0, N, 48)], 1)
    rows[:4, 2] = [0, 63, 64, N - 1]
    ref = oracle.sparse_dq_rows(q.float().numpy(), k.float().numpy(), v.float().numpy(), idx,
                                dout.float().numpy(), 64, rows)
    got = _f64(dq)[rows[:, 0], rows[:, 1], rows[:, 2]]
    assert_close(got, ref, "bf16", "dq rows")
    dk64, dv64, do64 = _f64(dk), _f64(dv), _f64(dout)
    for gr in range(Hkv):
        s_dk = dk64[0, gr].sum(axis=0)
        scale_dk = np.abs(dk64[0, gr]).sum(axis=0)
        assert np.all(np.abs(s_dk) <= 2e-2 * scale_dk + 1e-3), "dk rows do not sum to zero"
        s_dv = dv64[0, gr].sum(axis=0)
        s_do = do64[0, 16 * gr:16 * (gr + 1)].sum(axis=(0, 1))
        scale_dv = np.abs(dv64[0, gr]).sum(axis=0)
        assert np.all(np.abs(s_dv - s_do) <= 1e-2 * scale_dv + 1e-2), "dv rows do not sum to dout"
