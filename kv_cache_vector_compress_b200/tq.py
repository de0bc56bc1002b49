"""Thin Python binding of libtq (the C ABI in include/tq.h) over torch CUDA tensors.

Argument marshalling only: every step of the hot path runs in the library's kernels.
Importing this module loads ``libtq.so`` and raises ImportError if it is missing; there
is no fallback implementation.

Tensor conventions: norms are ``torch.float16`` tensors (their bits are the IEEE half the
library writes); packed codes and signs are ``torch.int32`` tensors holding the uint32
words; all tensors must be contiguous CUDA tensors on the current device, and work is
enqueued on ``torch.cuda.current_stream()``.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtq.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"libtq.so not built at {LIB_PATH}; run python -m kv_cache_vector_compress_b200.build")
_lib = ctypes.CDLL(LIB_PATH)

TQ_OK, TQ_ERR_INVALID_ARG, TQ_ERR_UNSUPPORTED, TQ_ERR_CUDA, TQ_ERR_TIMEOUT = 0, 1, 2, 3, 4
TQ_F16, TQ_F32 = 0, 1


class tq_params(ctypes.Structure):
    _fields_ = [("dim", ctypes.c_int), ("bits", ctypes.c_int), ("proj_dim", ctypes.c_int),
                ("R", ctypes.c_void_p), ("S", ctypes.c_void_p), ("workspace", ctypes.c_void_p),
                ("workspace_bytes", ctypes.c_size_t)]


_P = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64
_SZ = ctypes.c_size_t
_PP = ctypes.POINTER(tq_params)

_lib.tq_status_string.argtypes = [_I]
_lib.tq_status_string.restype = ctypes.c_char_p
_lib.tq_version.restype = _I
_lib.tq_codebook.argtypes = [_I, _I, _P, _P]
_lib.tq_codebook.restype = _I
_lib.tq_codebook_beta.argtypes = [_I, _I, _P, _P]
_lib.tq_codebook_beta.restype = _I
_lib.tq_workspace_bytes.argtypes = [_I, _I, _I]
_lib.tq_workspace_bytes.restype = _SZ
_lib.tq_prepare.argtypes = [_PP, _P, _P]
_lib.tq_prepare_law.argtypes = [_PP, _I, _P, _P]
_lib.tq_prepare_law.restype = _I
_lib.tq_prepare.restype = _I
_lib.tq_compress_keys.argtypes = [_PP, _P, _I, _I64, _P, _P, _P, _P, _P, _P]
_lib.tq_compress_keys.restype = _I
_lib.tq_compress_values.argtypes = [_PP, _P, _I, _I64, _P, _P, _P, _P]
_lib.tq_compress_values.restype = _I
_lib.tq_scores_scratch_bytes.argtypes = [_PP, _I, _I, _I, _I, _I64, _I]
_lib.tq_scores_scratch_bytes.restype = _SZ
_lib.tq_scores.argtypes = [_PP, _P, _I, _I, _I, _I, _I64, _P, _P, _P, _P, _P, _I, _P, _P, _P, _SZ, _P, _P]
_lib.tq_scores.restype = _I
_lib.tq_search.argtypes = _lib.tq_scores.argtypes
_lib.tq_search.restype = _I
_lib.tq_append_attend.argtypes = [_PP, _P, _P, _P, _I, _I, _I, _I, _I, _I64, _I64, _P, _P, _P, _P, _P, _P,
                                  ctypes.c_float, _P, _P, _SZ, _P, _P]
_lib.tq_append_attend.restype = _I
_lib.tq_attend_scratch_bytes.argtypes = [_PP, _I, _I, _I, _I, _I64]
_lib.tq_attend_scratch_bytes.restype = _SZ
_lib.tq_compress_attend_host_scratch_bytes.argtypes = [_PP, _I, _I, _I, _I, _I, _I64]
_lib.tq_compress_attend_host_scratch_bytes.restype = _SZ
_lib.tq_compress_attend_host.argtypes = [_PP, _P, _P, _I, _P, _I, _I, _I, _I, _I64, _P, _P, _P, _P, _P, _P,
                                         ctypes.c_float, _P, _P, _SZ, _P, _P]
_lib.tq_compress_attend_host.restype = _I
_lib.tq_attend.argtypes = [_PP, _P, _I, _I, _I, _I, _I64, _P, _P, _P, _P, _P, _P, ctypes.c_float, _P, _P,
                           _SZ, _P, _P]
_lib.tq_attend.restype = _I

_lib.tq_attend_partial.argtypes = [_PP, _P, _I, _I, _I, _I, _I64, _P, _P, _P, _P, _P, _P, ctypes.c_float, _P, _P,
                                   _SZ, _P, _P]
_lib.tq_attend_partial.restype = _I
_lib.tq_attend_merge.argtypes = [_PP, _P, _I, _I64, _P, _P, _P]
_lib.tq_attend_merge.restype = _I
_lib.tq_attend_static.argtypes = [_PP, _P, _I, _I, _I, _I, _I64, _P, _P, _P, _P, _P, _P, ctypes.c_float, _P,
                                  _P, _P]
_lib.tq_attend_static.restype = _I
_lib.tq_selftest_wait_timeout.argtypes = [_P, ctypes.c_uint32, _P]
_lib.tq_selftest_wait_timeout.restype = _I

TQ_STATIC_SCRATCH_BYTES = 16 << 20

TQ_LAW_GAUSSIAN, TQ_LAW_BETA = 0, 1
LAWS = {"gaussian": TQ_LAW_GAUSSIAN, "beta": TQ_LAW_BETA}

EXPORTS = ["tq_status_string", "tq_version", "tq_codebook", "tq_codebook_beta", "tq_workspace_bytes",
           "tq_prepare", "tq_prepare_law",
           "tq_compress_keys", "tq_compress_values", "tq_scores_scratch_bytes", "tq_scores", "tq_search",
           "tq_attend_scratch_bytes", "tq_attend", "tq_attend_partial", "tq_attend_merge", "tq_append_attend",
           "tq_compress_attend_host_scratch_bytes", "tq_compress_attend_host",
           "tq_selftest_wait_timeout",
           "tq_attend_static"]


class TQError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {_lib.tq_status_string(status).decode()}")
        self.status = status


def _check(st: int, what: str):
    if st != TQ_OK:
        raise TQError(st, what)


def _ptr(t):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def version() -> int:
    return _lib.tq_version()


def tq_codebook(dim: int, bits: int):
    """Host Lloyd-Max codebook: (boundaries[2^bits-1], centroids[2^bits]) as float32 tensors (CPU)."""
    K = 1 << bits
    b = torch.zeros(K - 1, dtype=torch.float32)
    c = torch.zeros(K, dtype=torch.float32)
    _check(_lib.tq_codebook(dim, bits, _ptr(b), _ptr(c)), "tq_codebook")
    return b, c


def tq_codebook_beta(dim: int, bits: int):
    """Host Lloyd-Max codebook for the exact (Beta) coordinate law of a random unit vector in R^dim."""
    K = 1 << bits
    b = torch.zeros(K - 1, dtype=torch.float32)
    c = torch.zeros(K, dtype=torch.float32)
    _check(_lib.tq_codebook_beta(dim, bits, _ptr(b), _ptr(c)), "tq_codebook_beta")
    return b, c


class Params:
    """A prepared parameter set: owns the device workspace and keeps R and S alive."""

    def __init__(self, dim: int, bits: int, proj_dim: int, R: torch.Tensor, S: torch.Tensor | None,
                 prepare: bool = True, law: str = "gaussian"):
        dev = R.device
        self.R = R.to(torch.float32).contiguous()
        self.S = S.to(device=dev, dtype=torch.float32).contiguous() if S is not None else None
        nbytes = _lib.tq_workspace_bytes(dim, bits, proj_dim)
        if nbytes == 0:
            raise TQError(TQ_ERR_INVALID_ARG, "tq_workspace_bytes")
        self.workspace = torch.empty(nbytes, dtype=torch.uint8, device=dev)
        self.c = tq_params(dim, bits, proj_dim, self.R.data_ptr(),
                           self.S.data_ptr() if self.S is not None else None,
                           self.workspace.data_ptr(), nbytes)
        self.dim, self.bits, self.proj_dim = dim, bits, proj_dim
        self.law = law
        if prepare:
            tq_prepare(self, law=law)

    @property
    def ref(self):
        return ctypes.byref(self.c)

    def key_words(self) -> int:
        return (self.bits - 1) * self.dim // 32

    def value_words(self) -> int:
        return self.bits * self.dim // 32


def tq_prepare_law(p: Params, law: str, dev_status: torch.Tensor | None = None):
    """Fill p's workspace with the codebooks of `law` ("gaussian" or "beta")."""
    _check(_lib.tq_prepare_law(p.ref, LAWS[law], _ptr(dev_status), _stream()), "tq_prepare_law")


def tq_prepare(p: Params, dev_status: torch.Tensor | None = None, law: str = "gaussian"):
    """Fill p's workspace; law "gaussian" (tq_prepare) or "beta" (tq_prepare_law)."""
    if law == "gaussian":
        _check(_lib.tq_prepare(p.ref, _ptr(dev_status), _stream()), "tq_prepare")
    else:
        tq_prepare_law(p, law, dev_status)


def _dtype_code(x: torch.Tensor) -> int:
    if x.dtype == torch.float16:
        return TQ_F16
    if x.dtype == torch.float32:
        return TQ_F32
    raise TypeError("x must be float16 or float32")


def tq_compress_keys(p: Params, x: torch.Tensor, codes=None, signs=None, norm=None, rnorm=None,
                     dev_status=None):
    """Compress rows of x ([n, dim]) as keys.  Returns (codes, signs, norm, rnorm)."""
    n = x.numel() // p.dim
    dev = x.device
    if codes is None:
        codes = torch.empty((n, p.key_words()), dtype=torch.int32, device=dev)
    if signs is None:
        signs = torch.empty((n, p.proj_dim // 32), dtype=torch.int32, device=dev)
    if norm is None:
        norm = torch.empty(n, dtype=torch.float16, device=dev)
    if rnorm is None:
        rnorm = torch.empty(n, dtype=torch.float16, device=dev)
    _check(_lib.tq_compress_keys(p.ref, _ptr(x), _dtype_code(x), n, _ptr(codes), _ptr(signs), _ptr(norm),
                                 _ptr(rnorm), _ptr(dev_status), _stream()), "tq_compress_keys")
    return codes, signs, norm, rnorm


def tq_compress_values(p: Params, x: torch.Tensor, codes=None, norm=None, dev_status=None):
    """Compress rows of x ([n, dim]) as values.  Returns (codes, norm)."""
    n = x.numel() // p.dim
    dev = x.device
    if codes is None:
        codes = torch.empty((n, p.value_words()), dtype=torch.int32, device=dev)
    if norm is None:
        norm = torch.empty(n, dtype=torch.float16, device=dev)
    _check(_lib.tq_compress_values(p.ref, _ptr(x), _dtype_code(x), n, _ptr(codes), _ptr(norm),
                                   _ptr(dev_status), _stream()), "tq_compress_values")
    return codes, norm


def tq_scores_scratch_bytes(p: Params, B, Hq, Hkv, Nq, T, topk=0) -> int:
    return _lib.tq_scores_scratch_bytes(p.ref, B, Hq, Hkv, Nq, T, topk)


def tq_scores(p: Params, q: torch.Tensor, keys, Hkv: int, T: int, want_scores: bool = True, topk: int = 0,
              scores=None, topk_idx=None, topk_val=None, scratch=None, dev_status=None, _fn="tq_scores"):
    """Scores [B, Hq, Nq, T] (fp32) of queries q [B, Hq, Nq, dim] against packed keys
    (codes, signs, norm, rnorm) laid out [B, Hkv, T].  With topk > 0 also returns the top-k
    indices and values per row.  Returns (scores or None, topk_idx or None, topk_val or None)."""
    B, Hq, Nq, _ = q.shape
    kc, ks, kn, kr = keys
    dev = q.device
    if want_scores and scores is None:
        scores = torch.empty((B, Hq, Nq, T), dtype=torch.float32, device=dev)
    if topk > 0:
        if topk_idx is None:
            topk_idx = torch.empty((B, Hq, Nq, topk), dtype=torch.int32, device=dev)
        if topk_val is None:
            topk_val = torch.empty((B, Hq, Nq, topk), dtype=torch.float32, device=dev)
    need = tq_scores_scratch_bytes(p, B, Hq, Hkv, Nq, T, topk)
    if scratch is None:
        scratch = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    _check(getattr(_lib, _fn)(p.ref, _ptr(q), B, Hq, Hkv, Nq, T, _ptr(kc), _ptr(ks), _ptr(kn), _ptr(kr),
                              _ptr(scores) if want_scores else None, topk, _ptr(topk_idx), _ptr(topk_val),
                              _ptr(scratch), scratch.numel(), _ptr(dev_status), _stream()), _fn)
    return scores, topk_idx, topk_val


def tq_search(p: Params, q: torch.Tensor, keys, Hkv: int, T: int, want_scores: bool = True, topk: int = 0,
              scores=None, topk_idx=None, topk_val=None, scratch=None, dev_status=None):
    """tq_scores with single fp16 operand products on the tensor-core search path (vector
    search; the score error bound is stated in the C header).  Same arguments and results."""
    return tq_scores(p, q, keys, Hkv, T, want_scores, topk, scores, topk_idx, topk_val, scratch, dev_status,
                     _fn="tq_search")


def tq_attend_scratch_bytes(p: Params, B, Hq, Hkv, Nq, T) -> int:
    return _lib.tq_attend_scratch_bytes(p.ref, B, Hq, Hkv, Nq, T)


def tq_compress_attend_host_scratch_bytes(p: Params, dtype: torch.dtype, B, Hq, Hkv, Nq, T) -> int:
    return _lib.tq_compress_attend_host_scratch_bytes(p.ref, TQ_F16 if dtype == torch.float16 else TQ_F32, B, Hq,
                                                      Hkv, Nq, T)


def tq_compress_attend_host(p: Params, k_host: torch.Tensor, v_host: torch.Tensor, q_host: torch.Tensor, Hkv: int,
                            T: int, keys, values, out_host: torch.Tensor, scale: float = 0.0, scratch=None,
                            dev_status=None):
    """One step from host memory: k_host / v_host [B, Hkv, T, dim] (fp16 or fp32) and q_host
    [B, Hq, Nq, dim] fp32 on the host (pinned for asynchronous copies), compressed into the device
    cache arrays keys (codes, signs, norm, rnorm) and values (codes, norm), attended, and the
    output written to out_host [B, Hq, Nq, dim] fp32 (valid after the stream synchronises)."""
    B, Hq, Nq, _ = q_host.shape
    kc, ks, kn, kr = keys
    vc, vn = values
    need = tq_compress_attend_host_scratch_bytes(p, k_host.dtype, B, Hq, Hkv, Nq, T)
    if scratch is None:
        scratch = torch.empty(max(need, 16), dtype=torch.uint8, device=kc.device)
    _check(_lib.tq_compress_attend_host(p.ref, _ptr(k_host), _ptr(v_host), _dtype_code(k_host), _ptr(q_host), B, Hq,
                                        Hkv, Nq, T, _ptr(kc), _ptr(ks), _ptr(kn), _ptr(kr), _ptr(vc), _ptr(vn),
                                        float(scale), _ptr(out_host), _ptr(scratch), scratch.numel(),
                                        _ptr(dev_status), _stream()), "tq_compress_attend_host")
    return out_host


def tq_attend(p: Params, q: torch.Tensor, keys, values, Hkv: int, T: int, scale: float = 0.0, out=None,
              scratch=None, dev_status=None):
    """Fused attention over a compressed cache: out [B, Hq, Nq, dim] fp32."""
    B, Hq, Nq, d = q.shape
    kc, ks, kn, kr = keys
    vc, vn = values
    dev = q.device
    if out is None:
        out = torch.empty((B, Hq, Nq, d), dtype=torch.float32, device=dev)
    if scratch is None:
        scratch = torch.empty(max(tq_attend_scratch_bytes(p, B, Hq, Hkv, Nq, T), 16), dtype=torch.uint8,
                              device=dev)
    _check(_lib.tq_attend(p.ref, _ptr(q), B, Hq, Hkv, Nq, T, _ptr(kc), _ptr(ks), _ptr(kn), _ptr(kr),
                          _ptr(vc), _ptr(vn), float(scale), _ptr(out), _ptr(scratch), scratch.numel(),
                          _ptr(dev_status), _stream()), "tq_attend")
    return out


def tq_append_attend(p: Params, q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor, keys, values,
                     Hkv: int, t: int, t_cap: int, scale: float = 0.0, out=None, scratch=None, dev_status=None):
    """One decode step: compress the new token of every (batch, KV head) (k_new, v_new: [B, Hkv, dim],
    fp16 or fp32) into slot t of the caches (keys / values as returned by the compress calls, holding
    B * Hkv * t_cap records), then attend over slots 0 .. t.  Returns out [B, Hq, Nq, dim] fp32."""
    B, Hq, Nq, d = q.shape
    kc, ks, kn, kr = keys
    vc, vn = values
    if k_new.dtype != v_new.dtype or k_new.dtype not in (torch.float16, torch.float32):
        raise ValueError("k_new and v_new must both be float16 or both float32")
    dt = 0 if k_new.dtype == torch.float16 else 1
    dev = q.device
    if out is None:
        out = torch.empty((B, Hq, Nq, d), dtype=torch.float32, device=dev)
    if scratch is None:
        scratch = torch.empty(max(tq_attend_scratch_bytes(p, B, Hq, Hkv, Nq, t + 1), 16), dtype=torch.uint8,
                              device=dev)
    _check(_lib.tq_append_attend(p.ref, _ptr(q), _ptr(k_new), _ptr(v_new), dt, B, Hq, Hkv, Nq, t, t_cap,
                                 _ptr(kc), _ptr(ks), _ptr(kn), _ptr(kr), _ptr(vc), _ptr(vn), float(scale),
                                 _ptr(out), _ptr(scratch), scratch.numel(), _ptr(dev_status), _stream()),
           "tq_append_attend")
    return out


def tq_attend_partial(p: Params, q: torch.Tensor, keys, values, Hkv: int, T: int, scale: float = 0.0,
                      partial=None, scratch=None, dev_status=None):
    """Attention partial over one piece of a context: [B, Hq, Nq, dim + 2] fp32 holding, per query
    row, the piece's largest logit, the sum of e^(logit - max), and the unnormalised rotated
    weighted value sum (see tq_attend_merge)."""
    B, Hq, Nq, d = q.shape
    kc, ks, kn, kr = keys
    vc, vn = values
    dev = q.device
    if partial is None:
        partial = torch.empty((B, Hq, Nq, d + 2), dtype=torch.float32, device=dev)
    if scratch is None:
        scratch = torch.empty(max(tq_attend_scratch_bytes(p, B, Hq, Hkv, Nq, T), 16), dtype=torch.uint8, device=dev)
    _check(_lib.tq_attend_partial(p.ref, _ptr(q), B, Hq, Hkv, Nq, T, _ptr(kc), _ptr(ks), _ptr(kn), _ptr(kr),
                                  _ptr(vc), _ptr(vn), float(scale), _ptr(partial), _ptr(scratch), scratch.numel(),
                                  _ptr(dev_status), _stream()), "tq_attend_partial")
    return partial


def tq_attend_merge(p: Params, partials: torch.Tensor, out=None, dev_status=None):
    """Merge partials [parts, B, Hq, Nq, dim + 2] of the pieces of one context into the attention
    output [B, Hq, Nq, dim]."""
    parts = partials.shape[0]
    shape = partials.shape[1:-1]
    rows = int(torch.tensor(shape).prod().item()) if len(shape) else 1
    if out is None:
        out = torch.empty((*shape, p.dim), dtype=torch.float32, device=partials.device)
    _check(_lib.tq_attend_merge(p.ref, _ptr(partials), parts, rows, _ptr(out), _ptr(dev_status), _stream()),
           "tq_attend_merge")
    return out


def tq_attend_static(p: Params, q: torch.Tensor, keys, values, Hkv: int, T: int, scale: float = 0.0, out=None,
                     dev_status=None):
    """tq_attend with the library-owned scratch array (no scratch argument, no allocation inside
    the library).  `out` may be passed in so that the call allocates nothing at all."""
    B, Hq, Nq, d = q.shape
    kc, ks, kn, kr = keys
    vc, vn = values
    if out is None:
        out = torch.empty((B, Hq, Nq, d), dtype=torch.float32, device=q.device)
    _check(_lib.tq_attend_static(p.ref, _ptr(q), B, Hq, Hkv, Nq, T, _ptr(kc), _ptr(ks), _ptr(kn), _ptr(kr),
                                 _ptr(vc), _ptr(vn), float(scale), _ptr(out), _ptr(dev_status), _stream()),
           "tq_attend_static")
    return out


def tq_selftest_wait_timeout(dev_status: torch.Tensor, timeout_ms: int = 100):
    """Launch the library's bounded-wait self-test: a kernel whose wait can only end by its time
    limit, which must leave TQ_ERR_TIMEOUT in dev_status (a device int32 tensor)."""
    _check(_lib.tq_selftest_wait_timeout(_ptr(dev_status), timeout_ms, _stream()), "tq_selftest_wait_timeout")

