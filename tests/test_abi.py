"""The C-ABI library loads, exports every symbol include/tq.h declares, and rejects bad
arguments on the host (no GPU needed: no call here reaches a launch)."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tq.h")


@pytest.fixture(scope="module")
def lib():
    from kv_cache_vector_compress_b200 import build
    path = build.build()
    return ctypes.CDLL(path), path


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(tq_[a-z_0-9]+)\s*\(", src)))


def test_header_declares_the_five_calls():
    names = declared_functions()
    for n in ["tq_codebook", "tq_compress_keys", "tq_compress_values", "tq_scores", "tq_attend"]:
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    L, path = lib
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (tq_[a-z_0-9]+)$", out, flags=re.M))
    for n in declared_functions():
        assert n in exported, n
        getattr(L, n)  # resolvable through the dynamic loader too


def test_binding_names_match_header():
    from kv_cache_vector_compress_b200 import tq
    assert sorted(tq.EXPORTS) == declared_functions()
    for n in tq.EXPORTS:
        assert hasattr(tq, n) or n in ("tq_status_string", "tq_version", "tq_workspace_bytes")


def test_status_strings(lib):
    L, _ = lib
    L.tq_status_string.restype = ctypes.c_char_p
    assert L.tq_status_string(0) == b"TQ_OK"
    assert L.tq_status_string(1) == b"TQ_ERR_INVALID_ARG"
    assert L.tq_status_string(4) == b"TQ_ERR_TIMEOUT"
    assert L.tq_status_string(99) == b"TQ_ERR_UNKNOWN"


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
@pytest.mark.parametrize("dim", [32, 128, 256, 1024])
def test_host_codebook_within_one_ulp_of_oracle(lib, dim, bits):
    # the library's Lloyd-Max (independent code) against the oracle's, after fp32 rounding
    L, _ = lib
    K = 1 << bits
    b = np.zeros(K - 1, np.float32)
    c = np.zeros(K, np.float32)
    assert L.tq_codebook(dim, bits, b.ctypes.data, c.ctypes.data) == 0
    ob, oc = oracle.codebook_f32(dim, bits)
    ulp = lambda a, o: np.abs(a.view(np.int32).astype(np.int64) - o.view(np.int32).astype(np.int64))
    assert ulp(c, oc).max() <= 1
    assert ulp(b, ob).max() <= 1
    assert b[K // 2 - 1] == 0.0
    np.testing.assert_array_equal(c, -c[::-1])


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
@pytest.mark.parametrize("dim", [32, 128, 1024])
def test_host_beta_codebook_within_one_ulp_of_oracle(lib, dim, bits):
    # the library's exact-law Lloyd-Max (cumulative table + Hermite interpolation, positive half)
    # against the oracle's (Gauss-Legendre quadrature in theta, all cells), after fp32 rounding
    L, _ = lib
    K = 1 << bits
    b = np.zeros(K - 1, np.float32)
    c = np.zeros(K, np.float32)
    assert L.tq_codebook_beta(dim, bits, b.ctypes.data, c.ctypes.data) == 0
    ob, oc = oracle.codebook_f32(dim, bits, law="beta")
    ulp = lambda a, o: np.abs(a.view(np.int32).astype(np.int64) - o.view(np.int32).astype(np.int64))
    assert ulp(c, oc).max() <= 1
    assert ulp(b, ob).max() <= 1
    np.testing.assert_array_equal(c, -c[::-1])
    assert L.tq_codebook_beta(2, bits, b.ctypes.data, c.ctypes.data) == 1


def test_codebook_rejects_bad_args(lib):
    L, _ = lib
    b = np.zeros(16, np.float32)
    c = np.zeros(16, np.float32)
    assert L.tq_codebook(128, 0, b.ctypes.data, c.ctypes.data) == 1
    assert L.tq_codebook(128, 5, b.ctypes.data, c.ctypes.data) == 1
    assert L.tq_codebook(0, 3, b.ctypes.data, c.ctypes.data) == 1
    assert L.tq_codebook(128, 3, None, c.ctypes.data) == 1


def test_workspace_bytes(lib):
    L, _ = lib
    L.tq_workspace_bytes.restype = ctypes.c_size_t
    assert L.tq_workspace_bytes(128, 3, 64) > 128 * 128 * 4
    assert L.tq_workspace_bytes(100, 3, 64) == 0  # not a multiple of 32
    assert L.tq_workspace_bytes(128, 0, 64) == 0
    assert L.tq_workspace_bytes(128, 3, 48) == 0
    assert L.tq_workspace_bytes(2048, 3, 64) == 0


class _Params(ctypes.Structure):
    _fields_ = [("dim", ctypes.c_int), ("bits", ctypes.c_int), ("proj_dim", ctypes.c_int),
                ("R", ctypes.c_void_p), ("S", ctypes.c_void_p), ("workspace", ctypes.c_void_p),
                ("workspace_bytes", ctypes.c_size_t)]


def test_argument_errors_return_before_any_launch(lib):
    # Every call below is rejected by the host-side checks, so no CUDA call is made (this
    # test runs on a machine without a GPU).  Fake device addresses are never dereferenced.
    L, _ = lib
    L.tq_workspace_bytes.restype = ctypes.c_size_t
    ws = L.tq_workspace_bytes(128, 3, 64)
    fake = 0x10000
    good = _Params(128, 3, 64, fake, fake, fake, ws)
    P = ctypes.byref
    # null params / bad dims / bits
    assert L.tq_compress_keys(None, fake, 0, 10, fake, fake, fake, fake, None, None) == 1
    bad = _Params(100, 3, 64, fake, fake, fake, ws)
    assert L.tq_compress_values(P(bad), fake, 0, 10, fake, fake, None, None) == 1
    bad = _Params(128, 1, 64, fake, fake, fake, ws)  # keys need bits >= 2
    assert L.tq_compress_keys(P(bad), fake, 0, 10, fake, fake, fake, fake, None, None) == 1
    bad = _Params(128, 3, 0, fake, fake, fake, ws)  # keys need a projection
    assert L.tq_compress_keys(P(bad), fake, 0, 10, fake, fake, fake, fake, None, None) == 1
    small = _Params(128, 3, 64, fake, fake, fake, ws - 1)
    assert L.tq_compress_values(P(small), fake, 0, 10, fake, fake, None, None) == 1
    # misaligned pointers
    assert L.tq_compress_values(P(good), fake + 4, 0, 10, fake, fake, None, None) == 1
    assert L.tq_compress_keys(P(good), fake, 0, 10, fake, fake + 2, fake, fake, None, None) == 1
    # bad dtype / negative n
    assert L.tq_compress_values(P(good), fake, 7, 10, fake, fake, None, None) == 1
    assert L.tq_compress_values(P(good), fake, 0, -1, fake, fake, None, None) == 1
    # n == 0 is a valid no-op
    assert L.tq_compress_values(P(good), fake, 0, 0, fake, fake, None, None) == 0
    # unsupported (valid multiple of 32, no kernel instance)
    ws96 = L.tq_workspace_bytes(96, 3, 64)
    p96 = _Params(96, 3, 64, fake, fake, fake, ws96)
    assert L.tq_compress_values(P(p96), fake, 0, 10, fake, fake, None, None) == 2
    # scores / attend shapes
    L.tq_scores.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                            ctypes.c_int, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
                            ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_void_p]
    L.tq_search.argtypes = L.tq_scores.argtypes
    for fn in (L.tq_scores, L.tq_search):  # tq_search takes tq_scores' arguments and checks
        call = lambda B, Hq, Hkv, Nq, T, topk=0, sc=fake, sb=1 << 40: fn(
            P(good), fake, B, Hq, Hkv, Nq, T, fake, fake, fake, fake, sc, topk, fake, fake, fake, sb, None, None)
        assert call(1, 3, 2, 1, 10) == 1      # Hq not a multiple of Hkv
        assert call(1, 4, 2, 1, 0) == 1       # empty cache
        assert call(1, 4, 2, 0, 10) == 1      # no queries
        assert call(1, 4, 2, 1, 10, topk=11) == 1  # topk > T
        assert call(1, 4, 2, 1, 100, topk=65) == 1  # topk above the maximum
        assert call(1, 4, 2, 1, 10, sc=None) == 1  # nothing to return
        assert call(1, 4, 2, 1, 10, sb=0) == 1  # scratch too small
    L.tq_attend.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                            ctypes.c_int, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_float, ctypes.c_void_p,
                            ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_void_p]
    att = lambda T, out=fake, sb=1 << 40, scale=0.0: L.tq_attend(
        P(good), fake, 1, 4, 2, 1, T, fake, fake, fake, fake, fake, fake, scale, out, fake, sb, None, None)
    assert att(0) == 1
    assert att(10, out=None) == 1
    assert att(10, sb=16) == 1
    assert att(10, scale=float("nan")) == 1
    # host-buffer step: missing host pointers, bad dtype, scratch too small
    L.tq_compress_attend_host.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                                          ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                          ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                          ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_float,
                                          ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p,
                                          ctypes.c_void_p]
    host = lambda kh=fake, oh=fake, dt=0, T=10, sb=1 << 40: L.tq_compress_attend_host(
        P(good), kh, fake, dt, fake, 1, 4, 2, 1, T, fake, fake, fake, fake, fake, fake, 0.0, oh, fake, sb, None,
        None)
    assert host(kh=None) == 1
    assert host(oh=None) == 1
    assert host(dt=5) == 1
    assert host(T=0) == 1
    assert host(sb=16) == 1
    # decode-step append: slot outside the cache, bad dtype, missing or misaligned new rows
    L.tq_append_attend.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                   ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                   ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p,
                                   ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                   ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t,
                                   ctypes.c_void_p, ctypes.c_void_p]
    app = lambda t, cap, kn=fake, dt=0, sb=1 << 40: L.tq_append_attend(
        P(good), fake, kn, fake, dt, 1, 4, 2, 1, t, cap, fake, fake, fake, fake, fake, fake, 0.0, fake, fake,
        sb, None, None)
    assert app(10, 10) == 1        # slot t must be below the capacity
    assert app(-1, 10) == 1
    assert app(3, 10, dt=5) == 1   # dtype
    assert app(3, 10, kn=None) == 1
    assert app(3, 10, kn=fake + 8) == 1
    assert app(3, 10, sb=16) == 1  # scratch too small


def test_scratch_size_helpers(lib):
    L, _ = lib
    L.tq_workspace_bytes.restype = ctypes.c_size_t
    L.tq_attend_scratch_bytes.restype = ctypes.c_size_t
    L.tq_attend_scratch_bytes.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                          ctypes.c_int, ctypes.c_int64]
    L.tq_scores_scratch_bytes.restype = ctypes.c_size_t
    L.tq_scores_scratch_bytes.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                          ctypes.c_int, ctypes.c_int64, ctypes.c_int]
    ws = L.tq_workspace_bytes(128, 3, 64)
    p = _Params(128, 3, 64, 0x10000, 0x10000, 0x10000, ws)
    a = L.tq_attend_scratch_bytes(ctypes.byref(p), 32, 32, 8, 1, 32768)
    assert a >= 32 * 32 * (128 + 64) * 4
    # few rows: a top-k pass over a full score buffer in scratch
    f0 = L.tq_scores_scratch_bytes(ctypes.byref(p), 1, 1, 1, 16, 1000, 0)
    f1 = L.tq_scores_scratch_bytes(ctypes.byref(p), 1, 1, 1, 16, 1000, 10)
    assert f1 >= f0 + 16 * 1000 * 4
    # many rows: a short top-k is fused (per-CTA lists only), a long one needs the score buffer
    s0 = L.tq_scores_scratch_bytes(ctypes.byref(p), 1, 1, 1, 1024, 1000, 0)
    s1 = L.tq_scores_scratch_bytes(ctypes.byref(p), 1, 1, 1, 1024, 1000, 10)
    s2 = L.tq_scores_scratch_bytes(ctypes.byref(p), 1, 1, 1, 1024, 1000, 64)
    assert s0 < s1 < s0 + 1024 * 1000 * 4
    assert s2 >= s0 + 1024 * 1000 * 4
    assert L.tq_attend_scratch_bytes(ctypes.byref(p), 1, 3, 2, 1, 10) == 0
