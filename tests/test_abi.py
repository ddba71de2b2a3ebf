"""The C-ABI library loads, exports every entry point include/sala.h declares, and rejects bad
arguments on the host before touching the GPU (no compute call is made here)."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sala.h")
LIB = os.path.join(ROOT, "hybrid_sparse_linear_b200", "libsala.so")
DEBUG_LIB = os.path.join(ROOT, "hybrid_sparse_linear_b200", "libsala_debug.so")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sala_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(LIB):
        from hybrid_sparse_linear_b200 import build
        build.build()
    import torch  # noqa: F401  (loads the shared CUDA runtime the library links against)
    return ctypes.CDLL(LIB)


def test_header_declares_the_boundary():
    names = _declared()
    for n in ("sala_linear_prefill", "sala_linear_decode", "sala_block_compress",
              "sala_block_topk", "sala_sparse_prefill", "sala_sparse_decode",
              "sala_check_status", "sala_status_string"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", LIB], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\bT (sala_\w+)", out))
    missing = [n for n in _declared() if n not in exported]
    assert not missing, missing
    for n in _declared():
        assert hasattr(lib, n)


def test_debug_build_exports_the_same_boundary(lib):
    # the bounds-checking build is a drop-in for the release one, and each says which it is
    out = subprocess.run(["nm", "-D", "--defined-only", DEBUG_LIB], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\bT (sala_\w+)", out))
    assert not [n for n in _declared() if n not in exported]
    dbg = ctypes.CDLL(DEBUG_LIB)
    assert dbg.sala_debug_bounds_build() == 1
    assert lib.sala_debug_bounds_build() == 0


def test_library_is_sm100a_only():
    out = subprocess.run(["cuobjdump", "--list-elf", LIB], capture_output=True, text=True).stdout
    arches = set(re.findall(r"sm_(\d+a?)", out))
    assert arches == {"100a"}, arches


def test_status_strings(lib):
    lib.sala_status_string.restype = ctypes.c_char_p
    for code, name in enumerate(["SALA_OK", "SALA_ERR_INVALID_ARG", "SALA_ERR_UNSUPPORTED",
                                 "SALA_ERR_CUDA", "SALA_ERR_TIMEOUT", "SALA_ERR_BOUNDS"]):
        assert lib.sala_status_string(code).decode() == name


def test_host_validation_rejects_before_launch(lib):
    vp = ctypes.c_void_p
    lib.sala_last_error.restype = ctypes.c_char_p
    good = vp(1 << 20)  # never dereferenced: every case below fails validation first
    # head dim 96 is unsupported
    r = lib.sala_linear_prefill(good, good, good, good, good, None, None, 1, 1, 64, 96, 0, 1, None)
    assert r == 2 and b"head dim" in lib.sala_last_error()
    # NULL q with work to do
    r = lib.sala_linear_prefill(None, good, good, good, good, None, None, 1, 1, 64, 128, 0, 1, None)
    assert r == 1 and b"q must be" in lib.sala_last_error()
    # misaligned pointer
    r = lib.sala_linear_prefill(vp((1 << 20) + 2), good, good, good, good, None, None, 1, 1, 64,
                                128, 0, 1, None)
    assert r == 1
    # unsupported chunk
    r = lib.sala_linear_prefill(good, good, good, good, good, None, None, 1, 1, 64, 128, 32, 1, None)
    assert r == 2
    # block compress past the end of the keys
    r = lib.sala_block_compress(good, good, 1, 2, 100, 128, 64, 1, 1, 4, 1, None)
    assert r == 1
    # H not a multiple of Hkv
    r = lib.sala_sparse_prefill(good, good, good, good, good, 1, 6, 4, 128, 128, 64, 3,
                                ctypes.c_float(0.0), 1, None)
    assert r == 1
    # block size other than 64
    r = lib.sala_sparse_prefill(good, good, good, good, good, 1, 4, 2, 128, 128, 32, 3,
                                ctypes.c_float(0.0), 1, None)
    assert r == 2
    # kbar too short for the last query row
    r = lib.sala_block_topk(good, good, good, 1, 4, 2, 640, 0, 3, 128, 64, 2, 1, 1, None, 0, 1, None)
    assert r == 1 and b"kbar holds" in lib.sala_last_error()
    # top-k above 64 with more candidates than that
    r = lib.sala_block_topk(good, good, good, 1, 4, 2, 64 * 200, 0, 200, 128, 64, 65, 1, 1, None,
                            0, 1, None)
    assert r == 2
    # decode position outside the cache
    r = lib.sala_sparse_decode(good, good, good, good, None, None, good, 1, 4, 2, 100, 100, 2, 128,
                               64, 1, 1, 1, ctypes.c_float(0.0), good, 1 << 20, 1, None)
    assert r == 1


def test_empty_problems_are_noops(lib):
    # B = 0 / N = 0: nothing to do, nothing launched, no device needed.
    assert lib.sala_linear_prefill(None, None, None, None, None, None, None, 0, 4, 64, 128, 0, 1, None) == 0
    assert lib.sala_sparse_prefill(None, None, None, None, None, 1, 4, 2, 0, 128, 64, 3,
                                   ctypes.c_float(0.0), 1, None) == 0
    assert lib.sala_block_compress(None, None, 1, 2, 64, 128, 64, 0, 0, 1, 1, None) == 0
    assert lib.sala_block_topk(None, None, None, 1, 4, 2, 0, 0, 0, 128, 64, 2, 1, 1, None, 0, 1, None) == 0
    assert lib.sala_block_topk_per_head(None, None, None, 1, 4, 2, 0, 0, 128, 64, 2, 1, 1, 1, None) == 0
    assert lib.sala_sparse_prefill_per_head(None, None, None, None, None, 1, 4, 2, 0, 128, 64, 3,
                                            ctypes.c_float(0.0), 1, None) == 0


def test_per_head_calls_validate_before_launch(lib):
    vp = ctypes.c_void_p
    lib.sala_last_error.restype = ctypes.c_char_p
    good = vp(1 << 20)  # never dereferenced: every case below fails validation first
    # block 32 is unsupported
    r = lib.sala_block_topk_per_head(good, good, good, 1, 4, 2, 64, 2, 128, 32, 2, 1, 1, 1, None)
    assert r == 2
    # H not a multiple of Hkv
    r = lib.sala_sparse_prefill_per_head(good, good, good, good, good, 1, 5, 2, 64, 128, 64, 3,
                                         ctypes.c_float(0.0), 1, None)
    assert r == 1 and b"multiple" in lib.sala_last_error()
    # NULL idx with work to do
    r = lib.sala_sparse_prefill_per_head(good, good, good, None, good, 1, 4, 2, 64, 128, 64, 3,
                                         ctypes.c_float(0.0), 1, None)
    assert r == 1 and b"idx" in lib.sala_last_error()


def test_product_never_imports_the_oracle():
    pkg = os.path.join(ROOT, "hybrid_sparse_linear_b200")
    bad = re.compile(r"^\s*(import\s+oracle|from\s+oracle\b)|liborc|sala_oracle", re.M)
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                assert not bad.search(open(os.path.join(dirpath, f)).read()), f
    for f in os.listdir(os.path.join(ROOT, "oracle")):
        if f.endswith((".py", ".cpp")):
            text = open(os.path.join(ROOT, "oracle", f)).read()
            assert not re.search(r"^\s*(import|from)\s+hybrid_sparse_linear_b200|libsala|sala\.h",
                                 text, re.M), f


def test_host_validation_of_the_training_and_variant_calls(lib):
    vp, i64, f32, f64 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_float, ctypes.c_double
    lib.sala_last_error.restype = ctypes.c_char_p
    good = vp(1 << 20)
    # QK normalisation: head dim 96, eps 0, negative rows, an output overlapping its input
    lib.sala_qk_norm.argtypes = [vp, vp, i64, vp, vp, i64, ctypes.c_int, f64, ctypes.c_int, vp]
    assert lib.sala_qk_norm(good, good, 4, None, None, 0, 96, 1e-6, 1, None) == 2
    assert lib.sala_qk_norm(good, good, 4, None, None, 0, 128, 0.0, 1, None) == 1
    assert lib.sala_qk_norm(good, good, -1, None, None, 0, 128, 1e-6, 1, None) == 1
    assert lib.sala_qk_norm(good, vp((1 << 20) + 256), 4, None, None, 0, 128, 1e-6, 1, None) == 1
    assert b"overlaps" in lib.sala_last_error()
    assert lib.sala_qk_norm(None, None, 0, None, None, 0, 128, 1e-6, 1, None) == 0  # nothing to do
    # sparse training calls: only bf16, d 128, 16 query heads per KV head
    lib.sala_sparse_prefill_lse.argtypes = [vp] * 7 + [ctypes.c_int] * 7 + [f32, ctypes.c_int, vp]
    assert lib.sala_sparse_prefill_lse(good, good, good, good, good, good, None, 1, 8, 2, 128, 128,
                                       64, 67, f32(0.0), 1, None) == 2
    lib.sala_sparse_backward.argtypes = [vp] * 11 + [ctypes.c_int] * 7 + [f32, vp, ctypes.c_size_t,
                                                                          ctypes.c_int, vp]
    assert lib.sala_sparse_backward(good, good, good, good, good, None, good, good, good, good, good,
                                    1, 32, 2, 128, 64, 64, 67, f32(0.0), good, 1 << 30, 1,
                                    None) == 2                       # d 64
    assert lib.sala_sparse_backward(good, good, good, good, good, None, good, good, good, good, good,
                                    1, 32, 2, 128, 128, 64, 67, f32(0.0), good, 16, 1, None) == 1
    assert b"workspace" in lib.sala_last_error()                    # workspace too small
    lib.sala_sparse_backward_workspace.restype = ctypes.c_size_t
    assert lib.sala_sparse_backward_workspace(1, 32, 2, 262144, 128, 67) > 2 * 2 * 262144 * 128 * 4
    # softmax-aggregated selection: more than 16 query heads per KV head
    lib.sala_block_topk_qblock_softmax.argtypes = [vp, vp, vp] + [ctypes.c_int] * 10 + [
        f32, ctypes.c_int, vp]
    assert lib.sala_block_topk_qblock_softmax(good, good, good, 1, 34, 2, 640, 10, 128, 64, 4, 1, 2,
                                              f32(0.0), 1, None) == 2
    # programmatic-dependent decode: a RoPE base in (0, 1] is rejected
    lib.sala_linear_decode_pdl.argtypes = [vp] * 6 + [ctypes.c_int] * 3 + [i64, f64, ctypes.c_int, vp]
    assert lib.sala_linear_decode_pdl(good, good, good, good, good, good, 1, 4, 128, 5, 0.5, 1,
                                      None) == 1
