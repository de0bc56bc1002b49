"""CPU oracle for the TurboQuant compression hot path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``
may import this package.  The product path (the CUDA library and its binding) never
touches it, and the two share no code: the oracle is plain C in double precision
(``tq_oracle.c``), wrapped here with ctypes and numpy for argument marshalling only.

Every function follows the steps the pages give (see the header of ``tq_oracle.c``
for the list of sources and readings).  Pins that tie it to the pages and to
mathematics other than itself live in ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "tq_oracle.c")
_LIB = os.path.join(_HERE, "libtq_oracle.so")

# The compile line is deliberately plain: -O2, no fast-math, OpenMP over independent units.
CFLAGS = ["-O2", "-std=c99", "-fPIC", "-shared", "-fopenmp", "-fno-fast-math", "-ffp-contract=off"]


def build(force: bool = False) -> str:
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", *CFLAGS, "-o", _LIB, _SRC, "-lm"])
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        L = _lib
        P = ctypes.c_void_p
        I = ctypes.c_int
        I64 = ctypes.c_int64
        D = ctypes.c_double
        L.ora_f64_to_f16.argtypes = [D]
        L.ora_f64_to_f16.restype = ctypes.c_uint16
        L.ora_f16_to_f64.argtypes = [ctypes.c_uint16]
        L.ora_f16_to_f64.restype = D
        L.ora_codebook.argtypes = [I, I, P, P]
        L.ora_codebook.restype = I
        L.ora_codebook_f32.argtypes = [I, I, P, P]
        L.ora_codebook_f32.restype = I
        L.ora_codebook_beta.argtypes = [I, I, P, P]
        L.ora_codebook_beta.restype = I
        L.ora_codebook_law_f32.argtypes = [I, I, I, P, P]
        L.ora_codebook_law_f32.restype = I
        L.ora_pack_codes.argtypes = [P, I, I, P]
        L.ora_unpack_codes.argtypes = [P, I, I, P]
        L.ora_compress.argtypes = [I, I, I, I, P, P, P, I, I64, P, P, P, P, P, P, I]
        L.ora_compress.restype = I
        L.ora_dequantize.argtypes = [I, I, P, P, P, I64, P, I]
        L.ora_dequantize.restype = I
        L.ora_scores.argtypes = [I, I, I, P, P, P, I, I, I, I, I64, P, P, P, P, P, I]
        L.ora_scores.restype = I
        L.ora_attend.argtypes = [I, I, I, P, P, P, I, I, I, I, I64, P, P, P, P, P, P, D, P, I]
        L.ora_attend.restype = I
        L.ora_topk.argtypes = [P, I64, I64, I, P, P]
        L.ora_topk.restype = I
        L.ora_nominal_bytes.argtypes = [I, I, I64, I, I]
        L.ora_nominal_bytes.restype = D
        L.ora_fp16_bytes.argtypes = [I, I, I64, I]
        L.ora_fp16_bytes.restype = D
        L.ora_num_threads.argtypes = []
        L.ora_num_threads.restype = I
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def num_threads() -> int:
    return lib().ora_num_threads()


def f64_to_f16_bits(v: float) -> int:
    return int(lib().ora_f64_to_f16(float(v)))


def f16_bits_to_f64(h: int) -> float:
    return float(lib().ora_f16_to_f64(int(h)))


def codebook(dim: int, bits: int):
    """Lloyd-Max codebook for N(0, 1/dim) in double: (boundaries[K-1], centroids[K], iterations)."""
    K = 1 << bits
    b = np.zeros(K - 1, np.float64)
    c = np.zeros(K, np.float64)
    it = lib().ora_codebook(dim, bits, _p(b), _p(c))
    if it < 0:
        raise ValueError("codebook did not converge / bad arguments")
    return b, c, it


def codebook_beta(dim: int, bits: int):
    """Lloyd-Max codebook for the exact coordinate law of a random unit vector in R^dim (density
    proportional to (1 - y^2)^((dim-3)/2)), in double: (boundaries[K-1], centroids[K], iterations)."""
    K = 1 << bits
    b = np.zeros(K - 1, np.float64)
    c = np.zeros(K, np.float64)
    it = lib().ora_codebook_beta(dim, bits, _p(b), _p(c))
    if it < 0:
        raise ValueError("codebook did not converge / bad arguments")
    return b, c, it


LAWS = {"gaussian": 0, "beta": 1}


def codebook_f32(dim: int, bits: int, law: str = "gaussian"):
    K = 1 << bits
    b = np.zeros(K - 1, np.float32)
    c = np.zeros(K, np.float32)
    if lib().ora_codebook_law_f32(dim, bits, LAWS[law], _p(b), _p(c)) < 0:
        raise ValueError("codebook did not converge / bad arguments")
    return b, c


def pack_codes(idx: np.ndarray, dim: int, beta: int) -> np.ndarray:
    idx = _c(idx, np.int32)
    w = np.zeros(beta * dim // 32, np.uint32)
    lib().ora_pack_codes(_p(idx), dim, beta, _p(w))
    return w


def unpack_codes(words: np.ndarray, dim: int, beta: int) -> np.ndarray:
    words = _c(words, np.uint32)
    idx = np.zeros(dim, np.int32)
    lib().ora_unpack_codes(_p(words), dim, beta, _p(idx))
    return idx


def compress(x: np.ndarray, R: np.ndarray, S: np.ndarray | None, bits: int, is_key: bool,
             want_y: bool = False, want_p: bool = False, law: str = "gaussian"):
    """Compress rows of x ([n, dim], fp16 or fp32).  Returns a dict of packed arrays
    (codes, norm as fp16 bits; keys also signs and rnorm) plus optional y32 / p32."""
    x = np.ascontiguousarray(x)
    if x.dtype == np.float16:
        xf16 = 1
        xb = x.view(np.uint16)
    elif x.dtype == np.float32:
        xf16 = 0
        xb = x
    else:
        raise TypeError("x must be float16 or float32")
    n, dim = x.shape
    R = _c(R, np.float32)
    beta = bits - 1 if is_key else bits
    m = 0
    if is_key:
        S = _c(S, np.float32)
        m = S.shape[0]
    codes = np.zeros((n, beta * dim // 32), np.uint32)
    signs = np.zeros((n, max(m // 32, 1)), np.uint32)
    norm = np.zeros(n, np.uint16)
    rnorm = np.zeros(n, np.uint16)
    y32 = np.zeros((n, dim), np.float32) if want_y else None
    p32 = np.zeros((n, max(m, 1)), np.float32) if (want_p and is_key) else None
    rc = lib().ora_compress(1 if is_key else 0, dim, bits, m, _p(R), _p(S) if is_key else None,
                            _p(xb), xf16, n, _p(codes), _p(signs), _p(norm), _p(rnorm),
                            _p(y32) if y32 is not None else None,
                            _p(p32) if p32 is not None else None, LAWS[law])
    if rc:
        raise ValueError("ora_compress rejected its arguments")
    out = {"codes": codes, "norm": norm}
    if is_key:
        out["signs"] = signs[:, : m // 32]
        out["rnorm"] = rnorm
    if y32 is not None:
        out["y32"] = y32
    if p32 is not None:
        out["p32"] = p32
    return out


def dequantize(codes: np.ndarray, norm: np.ndarray, R: np.ndarray, beta: int, law: str = "gaussian") -> np.ndarray:
    codes = _c(codes, np.uint32)
    norm = _c(norm, np.uint16)
    R = _c(R, np.float32)
    n = norm.shape[0]
    dim = R.shape[0]
    out = np.zeros((n, dim), np.float64)
    if lib().ora_dequantize(dim, beta, _p(R), _p(codes), _p(norm), n, _p(out), LAWS[law]):
        raise ValueError("bad arguments")
    return out


def scores(q, R, S, bits, B, Hq, Hkv, Nq, T, kcodes, ksigns, knorm, krnorm, law: str = "gaussian") -> np.ndarray:
    q = _c(q, np.float32)
    R = _c(R, np.float32)
    S = _c(S, np.float32)
    dim = R.shape[0]
    m = S.shape[0]
    out = np.zeros((B, Hq, Nq, T), np.float64)
    rc = lib().ora_scores(dim, bits, m, _p(R), _p(S), _p(q), B, Hq, Hkv, Nq, T,
                          _p(_c(kcodes, np.uint32)), _p(_c(ksigns, np.uint32)),
                          _p(_c(knorm, np.uint16)), _p(_c(krnorm, np.uint16)), _p(out), LAWS[law])
    if rc:
        raise ValueError("bad arguments")
    return out


def attend(q, R, S, bits, B, Hq, Hkv, Nq, T, kcodes, ksigns, knorm, krnorm, vcodes, vnorm,
           scale: float | None = None, law: str = "gaussian") -> np.ndarray:
    q = _c(q, np.float32)
    R = _c(R, np.float32)
    S = _c(S, np.float32)
    dim = R.shape[0]
    m = S.shape[0]
    if scale is None or scale <= 0:
        scale = 1.0 / np.sqrt(dim)
    out = np.zeros((B, Hq, Nq, dim), np.float64)
    rc = lib().ora_attend(dim, bits, m, _p(R), _p(S), _p(q), B, Hq, Hkv, Nq, T,
                          _p(_c(kcodes, np.uint32)), _p(_c(ksigns, np.uint32)),
                          _p(_c(knorm, np.uint16)), _p(_c(krnorm, np.uint16)),
                          _p(_c(vcodes, np.uint32)), _p(_c(vnorm, np.uint16)), float(scale), _p(out),
                          LAWS[law])
    if rc:
        raise ValueError("bad arguments")
    return out


def topk(scores_: np.ndarray, k: int):
    s = _c(scores_, np.float64)
    T = s.shape[-1]
    rows = s.size // T
    idx = np.zeros((rows, k), np.int64)
    val = np.zeros((rows, k), np.float64)
    if lib().ora_topk(_p(s), rows, T, k, _p(idx), _p(val)):
        raise ValueError("bad arguments")
    shp = s.shape[:-1] + (k,)
    return idx.reshape(shp), val.reshape(shp)


def nominal_bytes(layers: int, kv_heads: int, seq: int, dim: int, bits: int) -> float:
    return float(lib().ora_nominal_bytes(layers, kv_heads, seq, dim, bits))


def fp16_bytes(layers: int, kv_heads: int, seq: int, dim: int) -> float:
    return float(lib().ora_fp16_bytes(layers, kv_heads, seq, dim))
