"""GPU parity of the QK normalisation (sala_qk_norm) against the fp64 oracle, through the C ABI.

Beyond the whole-tensor tolerance of tests/parity.py, each bf16 element is checked against the
oracle's value within 2^-8 relative (one bf16 rounding of an fp32 product, plus the fp32 sum of
squares and rsqrt), and fp32 within 1e-6 relative: a wrong row norm shows up on every element of
its row, however small the row.
"""
import numpy as np
import pytest
import torch

import oracle
from parity import assert_close

pytestmark = pytest.mark.gpu

EPS = 1e-6


@pytest.fixture(scope="module")
def sala():
    from hybrid_sparse_linear_b200 import sala as s
    return s


def _pre(shape, seed, dtype):
    from hybrid_sparse_linear_b200 import synth
    return synth.prenorm(shape, seed, "cpu", dtype)


def _check(out, x, dtype):
    ref = oracle.qk_norm(oracle.from_tensor(x), EPS)
    got = oracle.from_tensor(out)
    assert_close(got, ref, "bf16" if dtype == torch.bfloat16 else "f32")
    rel = 2.0 ** -8 if dtype == torch.bfloat16 else 1e-6
    bad = np.abs(got - ref) > rel * np.abs(ref) + 1e-30
    assert not bad.any(), f"{bad.sum()} elements beyond {rel} relative, first at {np.argwhere(bad)[0]}"


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.bfloat16, 64),
                                     (torch.float32, 128), (torch.float32, 64)])
def test_q_and_k_ragged(sala, dtype, d):
    # 3 * 333 q rows + 333 k rows: a tail that is no multiple of a warp's four rows
    q = _pre((1, 3, 333, d), 21, dtype)
    k = _pre((1, 1, 333, d), 22, dtype)
    qo, ko = sala.qk_norm(q.cuda(), k.cuda(), eps=EPS)
    sala.check_status()
    _check(qo.cpu(), q, dtype)
    _check(ko.cpu(), k, dtype)


def test_in_place_and_q_only(sala):
    q = _pre((2, 4, 77, 128), 23, torch.bfloat16)
    qd = q.cuda()
    qo, ko = sala.qk_norm(qd, q_out=qd, eps=EPS)
    sala.check_status()
    assert qo.data_ptr() == qd.data_ptr() and ko is None
    _check(qd.cpu(), q, torch.bfloat16)


def test_extreme_rows(sala):
    # rows of one large element, constant rows, tiny rows and a zero row (eps keeps it at 0)
    x = torch.zeros((6, 128), dtype=torch.float32)
    x[0, 5] = 3.0e4
    x[1] = -2.5
    x[2] = torch.linspace(-1e-3, 1e-3, 128)
    x[4, ::2] = 1.0
    x[5] = torch.randn(128, generator=torch.Generator().manual_seed(3)) * 1e-8
    for dtype in (torch.float32, torch.bfloat16):
        xx = x.to(dtype)
        qo, _ = sala.qk_norm(xx.cuda(), eps=EPS)
        sala.check_status()
        got = qo.cpu().double().numpy()
        ref = oracle.qk_norm(oracle.from_tensor(xx), EPS)
        assert np.all(got[3] == 0.0)
        rel = 2.0 ** -8 if dtype == torch.bfloat16 else 1e-6
        assert np.all(np.abs(got - ref) <= rel * np.abs(ref) + 1e-30)


def test_empty_and_errors(sala):
    z = torch.empty((0, 128), device="cuda", dtype=torch.bfloat16)
    sala.qk_norm(z, z)
    sala.check_status()
    q = torch.ones((4, 128), device="cuda", dtype=torch.bfloat16)
    with pytest.raises(sala.SalaError):
        sala.qk_norm(q, eps=0.0)
    with pytest.raises(sala.SalaError):
        sala.qk_norm(torch.ones((4, 96), device="cuda", dtype=torch.bfloat16))
    # an output that overlaps its input without being it is refused
    buf = torch.ones((8, 128), device="cuda", dtype=torch.bfloat16)
    with pytest.raises(sala.SalaError):
        sala.qk_norm(buf[:4], q_out=buf[2:6])


def test_full_size_sampled(sala):
    # one sparse layer's q and k at N = 262144 (32 + 2 heads, d 128): 8.9M rows, more than the
    # grid covers in one sweep; sampled rows against the oracle
    from hybrid_sparse_linear_b200 import synth
    N = 262144
    q = synth.prenorm((1, 32, N, 128), 31, "cuda", torch.bfloat16)
    k = synth.prenorm((1, 2, N, 128), 32, "cuda", torch.bfloat16)
    qo, ko = sala.qk_norm(q, k, eps=EPS)
    sala.check_status()
    g = torch.Generator().manual_seed(5)
    for x, y in ((q, qo), (k, ko)):
        rows = x.reshape(-1, 128)
        idx = torch.cat([torch.randint(0, rows.shape[0], (4000,), generator=g),
                         torch.tensor([0, rows.shape[0] - 1])]).cuda()
        xs = rows.index_select(0, idx).cpu()
        ys = y.reshape(-1, 128).index_select(0, idx).cpu()
        _check(ys, xs, torch.bfloat16)


# ---------------------------------------------------------------------------------------------
# The layer prologue (sala_qk_prologue): QK norm and/or RoPE in one pass

@pytest.mark.parametrize("dtype,d,norm,rope", [(torch.bfloat16, 128, False, True),
                                               (torch.bfloat16, 128, True, True),
                                               (torch.bfloat16, 64, True, True),
                                               (torch.float32, 128, False, True),
                                               (torch.float32, 64, True, False)])
def test_prologue_matches_oracle(sala, dtype, d, norm, rope):
    N, pos0, base = 333, 4099, 10000.0
    q = _pre((2, 3, N, d), 41, dtype)
    k = _pre((2, 1, N, d), 42, dtype)
    qo, ko = sala.qk_prologue(q.cuda(), k.cuda(), eps=EPS if norm else 0.0,
                              rope_base=base if rope else 0.0, pos0=pos0)
    sala.check_status()
    kind = "bf16" if dtype == torch.bfloat16 else "f32"
    for x, y in ((q, qo), (k, ko)):
        ref = oracle.from_tensor(x)
        if norm:
            ref = oracle.qk_norm(ref, EPS)
        if rope:
            ref = oracle.rope(ref, pos0, base)
        assert_close(oracle.from_tensor(y.cpu()), ref, kind)


def test_rope_layer_as_prologue_plus_plain_prefill(sala):
    # a linear layer with RoPE: rotate q, k in one pass, then the plain (tensor-core) prefill
    from hybrid_sparse_linear_b200 import synth
    B, H, N, d = 1, 4, 64 * 37 + 11, 128
    q, k, v = synth.linear_layer(B, H, N, d, torch.bfloat16, "cpu", layer=5)
    lam = synth.decays(H)
    qd, kd = q.cuda(), k.cuda()
    qr, kr = sala.qk_prologue(qd, kd, rope_base=10000.0, pos0=0)
    ws = torch.empty(max(sala.linear_prefill_workspace_bytes(B, H, N, d), 16), device="cuda",
                     dtype=torch.uint8)
    o = sala.linear_prefill(qr, kr, v.cuda(), lam.cuda(), workspace=ws)
    sala.check_status()
    f = oracle.from_tensor
    ref, _ = oracle.linear_chunked_rope(f(q), f(k), f(v), f(lam), 64, 0, 10000.0)
    assert_close(f(o.cpu()), ref, "bf16", "o")
