"""GPU parity of the linear-attention calls (sala_linear_prefill / sala_linear_decode) against the
fp64 oracle, through the C ABI.  Tolerances: see tests/parity.py."""
import math

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


def _inputs(B, H, N, d, dtype, seed, layer=0):
    from hybrid_sparse_linear_b200 import synth
    q, k, v = synth.linear_layer(B, H, N, d, dtype, "cpu", layer=layer, base=seed)
    return q, k, v


def _f64(t):
    return oracle.from_tensor(t)


def test_tiny_fp32_prefill(sala):
    from hybrid_sparse_linear_b200 import synth
    w = synth.WORKLOADS["tiny_fp32_n512"]
    q, k, v = _inputs(1, w["H"], w["N"], w["d"], torch.float32, 11)
    lam = synth.decays(w["H"], "tiny")
    so = torch.zeros((1, w["H"], w["d"], w["d"]), device="cuda")
    o = sala.linear_prefill(q.cuda(), k.cuda(), v.cuda(), lam.cuda(), state_out=so, chunk=64)
    sala.check_status()
    ref, s_ref = oracle.linear_chunked(_f64(q), _f64(k), _f64(v), _f64(lam), 64)
    assert_close(_f64(o), ref, "f32", "o")
    assert_close(_f64(so), s_ref, "f32", "state_out")


@pytest.mark.parametrize("d,N,B,H", [(128, 333, 2, 3), (64, 200, 1, 4), (128, 64, 1, 2),
                                     (128, 1, 1, 2), (128, 1100, 1, 32)])
def test_bf16_prefill_ragged_with_state(sala, d, N, B, H):
    from hybrid_sparse_linear_b200 import synth
    q, k, v = _inputs(B, H, N, d, torch.bfloat16, 100 + N)
    lam = synth.decays(H)
    g = torch.Generator().manual_seed(5)
    s_in = torch.randn((B, H, d, d), generator=g) / d
    so = torch.empty((B, H, d, d), device="cuda")
    o = sala.linear_prefill(q.cuda(), k.cuda(), v.cuda(), lam.cuda(), state_in=s_in.cuda(),
                            state_out=so)
    sala.check_status()
    ref, s_ref = oracle.linear_recurrent(_f64(q), _f64(k), _f64(v), _f64(lam), _f64(s_in))
    assert_close(_f64(o), ref, "bf16", "o")
    assert_close(_f64(so), s_ref, "bf16", "state_out")


def test_fp32_prefill_split_resume(sala):
    from hybrid_sparse_linear_b200 import synth
    B, H, N, d = 1, 2, 300, 64
    q, k, v = _inputs(B, H, N, d, torch.float32, 21)
    lam = synth.decays(H, "tiny").cuda()
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    s_full = torch.empty((B, H, d, d), device="cuda")
    o_full = sala.linear_prefill(qc, kc, vc, lam, state_out=s_full)
    s1 = torch.empty_like(s_full)
    o1 = sala.linear_prefill(qc[:, :, :131].contiguous(), kc[:, :, :131].contiguous(),
                             vc[:, :, :131].contiguous(), lam, state_out=s1)
    o2 = sala.linear_prefill(qc[:, :, 131:].contiguous(), kc[:, :, 131:].contiguous(),
                             vc[:, :, 131:].contiguous(), lam, state_in=s1, state_out=s1)
    sala.check_status()
    ref, s_ref = oracle.linear_recurrent(_f64(q), _f64(k), _f64(v), _f64(lam.cpu()))
    assert_close(_f64(torch.cat([o1, o2], dim=2)), ref, "f32", "resumed o")
    assert_close(_f64(s1), s_ref, "f32", "resumed state")
    assert_close(_f64(o_full), ref, "f32", "o")


def test_prefill_empty_sequence_passes_state(sala):
    B, H, d = 1, 2, 64
    lam = torch.full((H,), 0.9, device="cuda")
    s_in = torch.randn((B, H, d, d), device="cuda")
    s_out = torch.zeros_like(s_in)
    e = torch.empty((B, H, 0, d), device="cuda")
    sala.linear_prefill(e, e, e, lam, o=e, state_in=s_in, state_out=s_out)
    sala.check_status()
    assert torch.equal(s_in, s_out)


@pytest.mark.parametrize("dtype,d", [(torch.float32, 64), (torch.bfloat16, 128), (torch.float32, 128)])
def test_decode_steps_match_oracle(sala, dtype, d):
    from hybrid_sparse_linear_b200 import synth
    B, H, steps = 2, 4, 5
    lam = synth.decays(H)
    g = torch.Generator().manual_seed(9)
    S0 = (torch.randn((B, H, d, d), generator=g) / d).float()
    S = S0.cuda().clone()
    S_ref = _f64(S0)
    q, k, v = _inputs(B, H, steps, d, dtype, 31)
    kind = "bf16" if dtype == torch.bfloat16 else "f32"
    for t in range(steps):
        qt, kt, vt = (x[:, :, t].contiguous() for x in (q, k, v))
        o = sala.linear_decode(qt.cuda(), kt.cuda(), vt.cuda(), lam.cuda(), S)
        o_ref, S_ref = oracle.linear_decode(_f64(qt), _f64(kt), _f64(vt), _f64(lam), S_ref)
        assert_close(_f64(o), o_ref, kind, f"o step {t}")
    sala.check_status()
    assert_close(_f64(S), S_ref, kind, "state")


def test_decode_continues_prefill(sala):
    # decode at position p reproduces prefill row p when started from the prefill state.
    from hybrid_sparse_linear_b200 import synth
    B, H, N, d = 1, 4, 129, 128
    q, k, v = _inputs(B, H, N, d, torch.bfloat16, 41)
    lam = synth.decays(H).cuda()
    S = torch.empty((B, H, d, d), device="cuda")
    o_pre = sala.linear_prefill(q.cuda(), k.cuda(), v.cuda(), lam)
    sala.linear_prefill(q[:, :, :-1].contiguous().cuda(), k[:, :, :-1].contiguous().cuda(),
                        v[:, :, :-1].contiguous().cuda(), lam, state_out=S)
    o_dec = sala.linear_decode(q[:, :, -1].contiguous().cuda(), k[:, :, -1].contiguous().cuda(),
                               v[:, :, -1].contiguous().cuda(), lam, S)
    sala.check_status()
    ref = oracle.linear_quadratic(_f64(q), _f64(k), _f64(v), _f64(lam.cpu()),
                                  rows=np.array([[h, N - 1] for h in range(H)]))
    assert_close(_f64(o_dec), ref.reshape(1, H, d), "bf16", "decode row")
    assert_close(_f64(o_pre[:, :, -1]), ref.reshape(1, H, d), "bf16", "prefill row")


@pytest.mark.parametrize("segments", [False, True])
def test_linear_prefill_full_size_sampled(sala, segments):
    """32 heads x 32768 tokens x d 128 (bf16), checked on sampled rows of four heads, including
    the first and last rows and rows on both sides of 64- and 128-row boundaries; in one pass and
    split into parallel segments (then also on rows at segment boundaries)."""
    from hybrid_sparse_linear_b200 import synth
    B, H, N, d = 1, 32, 32768, 128
    q, k, v = synth.linear_layer(B, H, N, d, torch.bfloat16, "cuda", layer=0)
    lam = synth.decays(H).cuda()
    ws = None
    if segments:
        nbytes = sala.linear_prefill_workspace_bytes(B, H, N, d)
        assert nbytes > 0, "expected this shape to run as segments"
        ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    o = sala.linear_prefill(q, k, v, lam, workspace=ws)
    sala.check_status()
    heads = [0, 7, 19, 31]
    toks = [0, 1, 63, 64, 127, 128, 129, 4095, 4096, 20000, N - 129, N - 128, N - 2, N - 1]
    sub = lambda t: oracle.from_tensor(t[:, heads])
    rows = np.array([[hi, t] for hi in range(len(heads)) for t in toks])
    ref = oracle.linear_quadratic(sub(q), sub(k), sub(v), _f64(lam.cpu()[heads]), rows=rows)
    got = np.stack([_f64(o[0, heads[hi], t]) for hi, t in rows])
    assert_close(got, ref, "bf16", "sampled rows")


def test_bf16_prefill_segments_ragged_with_state(sala):
    """The segment-parallel form on every row of a ragged length, with a carried-in state and the
    state out (the chained state after the last segment) against the fp64 recurrence."""
    from hybrid_sparse_linear_b200 import synth
    B, H, N, d = 1, 32, 5000, 128
    nbytes = sala.linear_prefill_workspace_bytes(B, H, N, d)
    assert nbytes > 0, "expected this shape to run as segments"
    q, k, v = _inputs(B, H, N, d, torch.bfloat16, 700)
    lam = synth.decays(H)
    g = torch.Generator().manual_seed(9)
    s_in = torch.randn((B, H, d, d), generator=g) / d
    so = torch.empty((B, H, d, d), device="cuda")
    ws = torch.full((nbytes,), 0xFF, dtype=torch.uint8, device="cuda")  # no initial value needed
    o = sala.linear_prefill(q.cuda(), k.cuda(), v.cuda(), lam.cuda(), state_in=s_in.cuda(),
                            state_out=so, workspace=ws)
    sala.check_status()
    ref, s_ref = oracle.linear_recurrent(_f64(q), _f64(k), _f64(v), _f64(lam), _f64(s_in))
    assert_close(_f64(o), ref, "bf16", "o")
    assert_close(_f64(so), s_ref, "bf16", "state_out")


def test_prefill_workspace_size_contract(sala):
    """Short sequences need no workspace; fp32 never uses one; a NULL workspace falls back to one
    pass (covered by the unsegmented runs above)."""
    assert sala.linear_prefill_workspace_bytes(1, 32, 512, 128) == 0
    assert sala.linear_prefill_workspace_bytes(1, 32, 32768, 128, torch.float32) == 0
    n = sala.linear_prefill_workspace_bytes(1, 32, 32768, 128)
    assert n > 0 and n % (32 * 128 * 128 * 4) == 0


# ---------------------------------------------------------------------------------------------
# RoPE (the linear layers' half of HyPE): sala_linear_prefill_rope / sala_linear_decode_rope

@pytest.mark.parametrize("d,N,B,H,pos0,ws,dtype", [
    (128, 333, 2, 3, 0, False, torch.bfloat16),        # tensor cores, one pass, ragged tail
    (128, 5000, 1, 4, 1234, True, torch.bfloat16),     # tensor cores, parallel segments
    (128, 130, 1, 2, 2 ** 20 + 5, True, torch.bfloat16),  # positions past 2^20
    (64, 200, 1, 4, 77, False, torch.bfloat16),        # CUDA cores, bf16
    (64, 150, 2, 2, 9, False, torch.float32),          # CUDA cores, fp32
])
def test_rope_prefill_with_state(sala, d, N, B, H, pos0, ws, dtype):
    from hybrid_sparse_linear_b200 import synth
    q, k, v = _inputs(B, H, N, d, dtype, 300 + N)
    lam = synth.decays(H)
    g = torch.Generator().manual_seed(6)
    s_in = torch.randn((B, H, d, d), generator=g) / d
    so = torch.empty((B, H, d, d), device="cuda")
    work = None
    if ws:
        nbytes = sala.linear_prefill_workspace_bytes(B, H, N, d)
        work = torch.full((max(nbytes, 16),), 0xFF, dtype=torch.uint8, device="cuda")
    o = sala.linear_prefill(q.cuda(), k.cuda(), v.cuda(), lam.cuda(), state_in=s_in.cuda(),
                            state_out=so, workspace=work, rope_base=10000.0, pos0=pos0)
    sala.check_status()
    ref, s_ref = oracle.linear_chunked_rope(_f64(q), _f64(k), _f64(v), _f64(lam), 64, pos0=pos0,
                                            s_in=_f64(s_in))
    kind = "bf16" if dtype == torch.bfloat16 else "f32"
    assert_close(_f64(o), ref, kind, "o")
    assert_close(_f64(so), s_ref, kind, "state_out")


def test_rope_decode_continues_prefill(sala):
    # decode at position P + N - 1 from the rotated prefill's state reproduces that prefill row
    from hybrid_sparse_linear_b200 import synth
    B, H, N, d, P = 1, 4, 129, 128, 4000
    q, k, v = _inputs(B, H, N, d, torch.bfloat16, 51)
    lam = synth.decays(H).cuda()
    S = torch.empty((B, H, d, d), device="cuda")
    o_pre = sala.linear_prefill(q.cuda(), k.cuda(), v.cuda(), lam, rope_base=10000.0, pos0=P)
    sala.linear_prefill(q[:, :, :-1].contiguous().cuda(), k[:, :, :-1].contiguous().cuda(),
                        v[:, :, :-1].contiguous().cuda(), lam, state_out=S, rope_base=10000.0,
                        pos0=P)
    o_dec = sala.linear_decode(q[:, :, -1].contiguous().cuda(), k[:, :, -1].contiguous().cuda(),
                               v[:, :, -1].contiguous().cuda(), lam, S, rope_base=10000.0,
                               pos=P + N - 1)
    sala.check_status()
    ref, _ = oracle.linear_chunked_rope(_f64(q), _f64(k), _f64(v), _f64(lam.cpu()), 64, pos0=P)
    assert_close(_f64(o_pre), ref, "bf16", "rope prefill")
    assert_close(_f64(o_dec), ref[:, :, -1], "bf16", "rope decode row")


@pytest.mark.parametrize("d", [64, 128])
def test_rope_decode_fp32(sala, d):
    from hybrid_sparse_linear_b200 import synth
    B, H, pos = 2, 3, 123457
    lam = synth.decays(H)
    g = torch.Generator().manual_seed(8)
    S0 = (torch.randn((B, H, d, d), generator=g) / d).float()
    q, k, v = (x[:, :, 0].contiguous() for x in _inputs(B, H, 1, d, torch.float32, 61))
    S = S0.cuda().clone()
    o = sala.linear_decode(q.cuda(), k.cuda(), v.cuda(), lam.cuda(), S, rope_base=500000.0, pos=pos)
    sala.check_status()
    rq = oracle.rope(_f64(q)[:, :, None], pos, 500000.0)[:, :, 0]
    rk = oracle.rope(_f64(k)[:, :, None], pos, 500000.0)[:, :, 0]
    o_ref, s_ref = oracle.linear_decode(rq, rk, _f64(v), _f64(lam), _f64(S0))
    assert_close(_f64(o), o_ref, "f32", "rope decode o")
    assert_close(_f64(S), s_ref, "f32", "rope decode state")


# ---------------------------------------------------------------------------------------------
# Backward pass of the linear attention (sala_linear_backward)

@pytest.mark.parametrize("d,N,B,H,dtype", [
    (128, 333, 2, 3, torch.bfloat16),    # tensor cores, one pass
    (128, 3000, 1, 4, torch.bfloat16),   # tensor cores, parallel segments
    (64, 150, 1, 2, torch.float32),      # CUDA cores, fp32
    (128, 65, 1, 2, torch.float32),
])
def test_linear_backward(sala, d, N, B, H, dtype):
    from hybrid_sparse_linear_b200 import synth
    q, k, v = _inputs(B, H, N, d, dtype, 700 + N)
    g = torch.Generator().manual_seed(7)
    dout = (torch.randn((B, H, N, d), generator=g) / math.sqrt(d)).to(dtype)
    lam = synth.decays(H)
    dq, dk, dv = sala.linear_backward(q.cuda(), k.cuda(), v.cuda(), lam.cuda(), dout.cuda())
    sala.check_status()
    rq, rk, rv = oracle.linear_backward(_f64(q), _f64(k), _f64(v), _f64(lam), _f64(dout))
    kind = "bf16" if dtype == torch.bfloat16 else "f32"
    assert_close(_f64(dq), rq, kind, "dq")
    assert_close(_f64(dk), rk, kind, "dk")
    assert_close(_f64(dv), rv, kind, "dv")


# ---------------------------------------------------------------------------------------------
# Decode steps launched as programmatic dependents (sala_linear_decode_pdl)

@pytest.mark.parametrize("graph", [False, True])
def test_pdl_decode_chain_of_layers(sala, graph):
    # Three layers' decode steps back to back, each launched while the previous one may still run
    # (it reads only its own state early); then a second token.  Every output and state against
    # the oracle.  The middle layer rotates q and k (RoPE), the others do not.
    from hybrid_sparse_linear_b200 import synth
    B, H, d, L = 2, 32, 128, 3
    g = torch.Generator().manual_seed(77)
    lam = synth.decays(H)
    states = [torch.randn((B, H, d, d), generator=g) / d for _ in range(L)]
    toks = [[(torch.randn((B, H, d), generator=g) / 4).to(torch.bfloat16) for _ in range(3)]
            for _ in range(2 * L)]
    S_dev = [s.clone().cuda() for s in states]
    outs = [torch.empty((B, H, d), device="cuda", dtype=torch.bfloat16) for _ in range(2 * L)]
    qkv = [[x.cuda() for x in t] for t in toks]
    lam_d = lam.cuda()
    pos = 4097
    stream = torch.cuda.Stream()

    def run():
        for step in range(2):
            for l in range(L):
                q, k, v = qkv[step * L + l]
                sala.linear_decode(q, k, v, lam_d, S_dev[l], o=outs[step * L + l], stream=stream,
                                   pdl=True, rope_base=10000.0 if l == 1 else None, pos=pos + step)

    with torch.cuda.stream(stream):
        if graph:
            G = torch.cuda.CUDAGraph()
            with torch.cuda.graph(G, stream=stream):
                run()
            for l in range(L):  # capture ran nothing: start from the initial states
                S_dev[l].copy_(states[l])
            G.replay()
        else:
            run()
    torch.cuda.synchronize()
    sala.check_status(stream)
    S_ref = [_f64(s) for s in states]
    for step in range(2):
        for l in range(L):
            q, k, v = (_f64(x) for x in toks[step * L + l])
            if l == 1:
                q = oracle.rope(q[:, :, None], pos + step, 10000.0)[:, :, 0]
                k = oracle.rope(k[:, :, None], pos + step, 10000.0)[:, :, 0]
            o_ref, S_ref[l] = oracle.linear_decode(q, k, v, _f64(lam), S_ref[l])
            assert_close(_f64(outs[step * L + l]), o_ref, "bf16", f"o step {step} layer {l}")
    for l in range(L):
        assert_close(_f64(S_dev[l]), S_ref[l], "bf16", f"state layer {l}")
