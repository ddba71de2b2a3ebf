"""Device-level self-tests: one tcgen05 MMA tile per operand layout the kernels use (TMA with the
128-byte swizzle, K-major and MN-major B, A from shared memory or from TMEM) against a host
product, and the bounded-wait timeout path (a barrier that never completes; the kernel gives up,
records the timeout and returns -- no fault, no trap)."""
import ctypes
import os

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SELFTEST = os.path.join(ROOT, "hybrid_sparse_linear_b200", "libsala_selftest.so")


@pytest.fixture(scope="module")
def st():
    lib = ctypes.CDLL(SELFTEST)
    lib.sala_selftest_mma.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int] * 4 + [ctypes.c_void_p] * 2
    lib.sala_selftest_mma.restype = ctypes.c_int
    lib.sala_selftest_exp2_poly.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p]
    lib.sala_selftest_exp2_poly.restype = ctypes.c_int
    return lib


@pytest.mark.parametrize("N", [64, 128, 256])
@pytest.mark.parametrize("K", [64, 128])
@pytest.mark.parametrize("b_mn_major", [0, 1])
@pytest.mark.parametrize("a_mode", [0, 1, 2])  # A in SMEM K-major, in TMEM, in SMEM M-major
def test_mma_tile(st, N, K, b_mn_major, a_mode):
    g = torch.Generator().manual_seed(N * 7 + K + 3 * b_mn_major + a_mode)
    A = torch.randn((128, K), generator=g).to(torch.bfloat16)
    if b_mn_major:
        Bm = torch.randn((K, N), generator=g).to(torch.bfloat16)
        ref = A.double() @ Bm.double()
    else:
        Bm = torch.randn((N, K), generator=g).to(torch.bfloat16)
        ref = A.double() @ Bm.double().T
    Ad = (A.T.contiguous() if a_mode == 2 else A).cuda()
    Bd = Bm.cuda()
    D = torch.full((128, N), float("nan"), device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    r = st.sala_selftest_mma(Ad.data_ptr(), Bd.data_ptr(), D.data_ptr(), N, K, b_mn_major, a_mode,
                             status.data_ptr(), torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert r == 0
    assert int(status.item()) == 0, "device wait timed out"
    err = (D.double().cpu() - ref).abs().max().item()
    assert err <= 1e-4 * ref.abs().max().item(), f"max err {err}"


def test_exp2_polynomial_against_exact(st):
    """The FMA-pipe 2^y of the softmax: relative error within the fitted bound (7.5e-5, plus fp32
    rounding of the argument reduction) against an exact 2^y, over the range the softmax feeds it
    (y <= 8, including the stale-max excess) down to the clamp at -125; below the clamp (and at
    -inf, a masked key) it returns 2^-125 scaled by the polynomial, a normal number far below any
    ulp of the sums it enters."""
    g = torch.Generator().manual_seed(11)
    y = torch.cat([torch.linspace(-125.0, 8.0, 200001, dtype=torch.float64),
                   torch.rand(100000, generator=g, dtype=torch.float64) * 40 - 32,
                   torch.tensor([0.0, 0.5, -0.5, 1.0, -1.0, 7.999, 8.0, -124.999, -125.0])]).float()
    yd = y.cuda()
    out = torch.empty_like(yd)
    assert st.sala_selftest_exp2_poly(yd.data_ptr(), out.data_ptr(), y.numel(),
                                      torch.cuda.current_stream().cuda_stream) == 0
    torch.cuda.synchronize()
    ref = torch.exp2(y.double())
    rel = ((out.cpu().double() - ref) / ref).abs()
    assert rel.max().item() <= 8e-5, f"max rel err {rel.max().item()}"
    low = torch.tensor([-126.0, -200.0, -1e30, float("-inf")]).cuda()
    lo_out = torch.empty_like(low)
    assert st.sala_selftest_exp2_poly(low.data_ptr(), lo_out.data_ptr(), 4,
                                      torch.cuda.current_stream().cuda_stream) == 0
    torch.cuda.synchronize()
    v = lo_out.cpu().double()
    assert bool(((v > 0) & (v <= 2.0 ** -125 * 1.0001)).all()), v


def test_wait_timeout_is_reported_not_fatal():
    from hybrid_sparse_linear_b200 import sala
    sala.check_status()
    sala.set_wait_limit_ns(20_000_000)  # 20 ms
    try:
        sala.selftest_wait_timeout()
        with pytest.raises(sala.SalaError) as ei:
            sala.check_status()
        assert ei.value.code == sala.ERR_TIMEOUT
    finally:
        sala.set_wait_limit_ns(2_000_000_000)
    # the context is still usable and the word was cleared
    x = torch.ones(1024, device="cuda")
    assert float(x.sum()) == 1024.0
    sala.check_status()
