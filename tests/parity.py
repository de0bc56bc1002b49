"""Comparison rules between the CUDA path and the oracle.

- Codes: bit-exact, except coordinates whose oracle fp32 rotated value lies within 1e-5 of
  a codebook boundary; such mismatches must also stay below 1e-4 of all coordinates.
- Signs: bit-exact, except projections whose oracle fp32 value is within 1e-5 of zero, and
  except keys whose codes already differ (a different code gives a different residual).
- Norms: within one fp16 ulp (an fp32 norm can land on the other side of an fp16 rounding
  midpoint than the double one).  Residual norms of keys with differing codes are exempt.
- Scores and attention outputs: |gpu - oracle| <= 1e-4 + 1e-3 |oracle|.
"""
from __future__ import annotations

import numpy as np

CODE_TOL = 1e-5
SIGN_TOL = 1e-5
MAX_MISMATCH_FRAC = 1e-4
ATOL, RTOL = 1e-4, 1e-3


def as_u32(a) -> np.ndarray:
    a = a.cpu().numpy() if hasattr(a, "cpu") else np.asarray(a)
    return np.ascontiguousarray(a).view(np.uint32)


def as_u16(a) -> np.ndarray:
    a = a.cpu().numpy() if hasattr(a, "cpu") else np.asarray(a)
    return np.ascontiguousarray(a).view(np.uint16)


def _bit_positions(x: int):
    out = []
    while x:
        low = x & -x
        out.append(low.bit_length() - 1)
        x ^= low
    return out


def code_mismatches(gpu_codes, ora_codes, d: int, beta: int):
    """(row, coordinate) pairs whose packed codes differ."""
    g = as_u32(gpu_codes).reshape(-1, beta * d // 32)
    o = as_u32(ora_codes).reshape(-1, beta * d // 32)
    diff = g ^ o
    rows, words = np.nonzero(diff)
    pairs = set()
    for r, w in zip(rows.tolist(), words.tolist()):
        grp = w // beta
        for l in _bit_positions(int(diff[r, w])):
            pairs.add((r, 32 * grp + l))
    return sorted(pairs)


def check_codes(gpu_codes, ora_codes, ora_y32, bounds32, d: int, beta: int, what: str = "codes"):
    """Assert the code parity rule; returns the set of rows with (exempt) mismatches."""
    mm = code_mismatches(gpu_codes, ora_codes, d, beta)
    n = as_u32(ora_codes).reshape(-1, beta * d // 32).shape[0]
    b = np.asarray(bounds32, np.float64)
    bad = []
    for r, j in mm:
        y = float(ora_y32[r, j])
        if np.min(np.abs(y - b)) >= CODE_TOL:
            bad.append((r, j, y))
    assert not bad, f"{what}: {len(bad)} code mismatches outside the boundary band, e.g. {bad[:5]}"
    assert len(mm) < max(1.0, MAX_MISMATCH_FRAC * n * d), f"{what}: {len(mm)} boundary mismatches of {n * d}"
    return {r for r, _ in mm}


def check_signs(gpu_signs, ora_signs, ora_p32, m: int, exempt_rows=frozenset(), what: str = "signs"):
    g = as_u32(gpu_signs).reshape(-1, m // 32)
    o = as_u32(ora_signs).reshape(-1, m // 32)
    diff = g ^ o
    rows, words = np.nonzero(diff)
    bad, near = [], 0
    for r, w in zip(rows.tolist(), words.tolist()):
        if r in exempt_rows:
            continue
        for l in _bit_positions(int(diff[r, w])):
            a = 32 * w + l
            p = float(ora_p32[r, a])
            if abs(p) >= SIGN_TOL:
                bad.append((r, a, p))
            else:
                near += 1
    assert not bad, f"{what}: {len(bad)} sign mismatches with |p| >= {SIGN_TOL}, e.g. {bad[:5]}"
    assert near < max(1.0, MAX_MISMATCH_FRAC * g.size * 32)
    return near


def f16_ordered(bits: np.ndarray) -> np.ndarray:
    b = bits.astype(np.int64)
    return np.where(b & 0x8000, -(b & 0x7FFF), b)


def check_f16_close(gpu, ora, exempt_rows=frozenset(), what: str = "norm"):
    g = as_u16(gpu).reshape(-1)
    o = as_u16(ora).reshape(-1)
    d = np.abs(f16_ordered(g) - f16_ordered(o))
    if exempt_rows:
        keep = np.ones(len(d), bool)
        keep[list(exempt_rows)] = False
        d = d[keep]
    assert d.size == 0 or d.max() <= 1, f"{what}: {np.count_nonzero(d > 1)} values differ by more than 1 fp16 ulp"


def check_close(gpu, ora, what: str = "values", atol: float = ATOL, rtol: float = RTOL):
    g = gpu.detach().cpu().double().numpy() if hasattr(gpu, "cpu") else np.asarray(gpu, np.float64)
    o = np.asarray(ora, np.float64)
    assert g.shape == o.shape, (g.shape, o.shape)
    err = np.abs(g - o)
    lim = atol + rtol * np.abs(o)
    bad = np.count_nonzero(~(err <= lim))
    assert bad == 0, (f"{what}: {bad} of {err.size} outside {atol} + {rtol}|ref|; worst excess "
                      f"{float(np.max(err - lim)):.3g} (max err {float(err.max()):.3g})")
    return float(err.max())


def check_topk(gpu_idx, gpu_val, ora_scores_row, k: int, what: str = "topk"):
    """The GPU top-k set equals the oracle's, except indices whose oracle score lies within
    the tolerance of the oracle's k-th score (near-ties); GPU values agree with the oracle's
    scores at the returned indices; GPU order is by value descending."""
    s = np.asarray(ora_scores_row, np.float64)
    gi = np.asarray(gpu_idx).astype(np.int64).reshape(-1)
    gv = np.asarray(gpu_val, np.float64).reshape(-1)
    order = np.lexsort((np.arange(len(s)), -s))
    top = order[:k]
    kth = s[top[-1]]
    band = ATOL + RTOL * abs(kth)
    assert len(set(gi.tolist())) == k and gi.min() >= 0 and gi.max() < len(s)
    for i in set(gi.tolist()) ^ set(top.tolist()):
        assert abs(s[i] - kth) <= 2 * band, f"{what}: index {i} (score {s[i]}) vs k-th {kth}"
    check_close(gv, s[gi], what + " values")
    assert np.all(np.diff(gv) <= 0), f"{what}: values not descending"
