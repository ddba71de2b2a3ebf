"""sala_sparse_decode_noalloc: the sparse decode step for callers that may not allocate device
memory (serving loops that size every buffer up front, plug-ins whose host application owns the
device memory pool).  It must give the same result as sala_sparse_decode with a caller-provided
workspace, call after call (its built-in scratch area keeps the previous call's contents), and it
must refuse problems larger than that area before launching anything.

This file is collected last on purpose (test_zz_*): if it fails, a run that stops at the first
failure has already run every other test.  It is self-contained, so it also passes alone in a
fresh process."""
import ctypes
import os

import pytest
import torch

from parity import assert_close

pytestmark = pytest.mark.gpu

LIB = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "hybrid_sparse_linear_b200", "libsala.so")


def _lib():
    lib = ctypes.CDLL(LIB)
    vp, i = ctypes.c_void_p, ctypes.c_int
    lib.sala_sparse_decode_noalloc.argtypes = [vp] * 7 + [i] * 11 + [ctypes.c_float, i, vp]
    lib.sala_sparse_decode_noalloc.restype = i
    lib.sala_last_error.restype = ctypes.c_char_p
    return lib


def _call(lib, q, kc, vc, kbar, idx_out, o, pos, topk, n_init, n_local):
    B, H, d = q.shape
    Hkv, Tmax = kc.shape[1], kc.shape[2]
    dt = 1 if q.dtype == torch.bfloat16 else 0
    return lib.sala_sparse_decode_noalloc(
        q.data_ptr(), kc.data_ptr(), vc.data_ptr(), kbar.data_ptr(), None, idx_out.data_ptr(),
        o.data_ptr(), B, H, Hkv, pos, Tmax, kbar.shape[2], d, 64, topk, n_init, n_local,
        ctypes.c_float(0.0), dt, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("T", [64 * 300 + 5, 1 << 20])
def test_noalloc_matches_workspace_version_twice(T):
    from hybrid_sparse_linear_b200 import sala, synth
    lib = _lib()
    topk, n_init, n_local, H, Hkv, d = 64, 1, 2, 32, 2, 128
    slots = n_init + n_local + topk
    layer = synth.sparse_layer(1, H, Hkv, T, d, torch.bfloat16, "cuda", layer=11, q_rows=1)
    kbar = sala.block_compress(layer.k)
    q = layer.q[:, :, 0].contiguous()
    idx_ref = torch.empty((1, Hkv, slots), dtype=torch.int32, device="cuda")
    o_ref = sala.sparse_decode(q, layer.k, layer.v, kbar, T - 1, topk, n_init, n_local,
                               idx_out=idx_ref)
    sala.check_status()
    for call in range(2):
        o = torch.full_like(o_ref, float("nan"))
        idx = torch.full_like(idx_ref, -7)
        r = _call(lib, q, layer.k, layer.v, kbar, idx, o, T - 1, topk, n_init, n_local)
        assert r == 0, lib.sala_last_error()
        sala.check_status()
        assert torch.equal(idx, idx_ref), f"call {call}: selection differs"
        assert_close(o.double().cpu().numpy(), o_ref.double().cpu().numpy(), "bf16",
                     f"no-alloc call {call}")


def test_noalloc_recovers_after_a_timed_out_call():
    # The built-in area carries the grid barrier counters of the one-launch cooperative kernel
    # (the fp32 decode takes it) from call to call, and no caller can reach the area to clear them.
    # Make one call give up on its waits (a 1 ns wait limit: every CTA but the last to arrive stops
    # waiting at once, records SALA_ERR_TIMEOUT and returns; nothing faults), then check that the
    # next calls with the normal limit give exactly the result of sala_sparse_decode with its own
    # workspace.
    from hybrid_sparse_linear_b200 import sala, synth
    lib = _lib()
    lib.sala_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
    lib.sala_check_status.argtypes = [ctypes.c_void_p]
    lib.sala_check_status.restype = ctypes.c_int
    T, topk, n_init, n_local, H, Hkv, d = 64 * 3000 + 5, 64, 1, 2, 32, 2, 128
    slots = n_init + n_local + topk
    layer = synth.sparse_layer(1, H, Hkv, T, d, torch.float32, "cuda", layer=12, q_rows=1)
    kbar = sala.block_compress(layer.k)
    q = layer.q[:, :, 0].contiguous()
    idx_ref = torch.empty((1, Hkv, slots), dtype=torch.int32, device="cuda")
    o_ref = sala.sparse_decode(q, layer.k, layer.v, kbar, T - 1, topk, n_init, n_local,
                               idx_out=idx_ref)
    sala.check_status()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    o = torch.empty_like(o_ref)
    idx = torch.empty_like(idx_ref)
    lib.sala_set_wait_limit_ns(1)
    try:
        r = _call(lib, q, layer.k, layer.v, kbar, idx, o, T - 1, topk, n_init, n_local)
        assert r == 0, lib.sala_last_error()
        assert lib.sala_check_status(stream) == 4  # SALA_ERR_TIMEOUT
    finally:
        lib.sala_set_wait_limit_ns(2_000_000_000)
    for call in range(2):
        o = torch.full_like(o_ref, float("nan"))
        idx = torch.full_like(idx_ref, -7)
        r = _call(lib, q, layer.k, layer.v, kbar, idx, o, T - 1, topk, n_init, n_local)
        assert r == 0, lib.sala_last_error()
        assert lib.sala_check_status(stream) == 0, f"call {call} after the timeout did not complete"
        assert torch.equal(idx, idx_ref), f"call {call} after the timeout: selection differs"
        assert torch.equal(o, o_ref), f"call {call} after the timeout: output differs"


def test_noalloc_refuses_oversized_problem():
    lib = _lib()
    vp = ctypes.c_void_p
    dummy = vp(1 << 20)  # never dereferenced: the size check comes first
    r = lib.sala_sparse_decode_noalloc(dummy, dummy, dummy, dummy, None, None, dummy, 64, 32, 2,
                                       (1 << 20) - 1, 1 << 20, 1 << 14, 128, 64, 64, 1, 2,
                                       ctypes.c_float(0.0), 1, None)
    assert r == 2  # SALA_ERR_UNSUPPORTED
    assert b"built-in" in lib.sala_last_error()
