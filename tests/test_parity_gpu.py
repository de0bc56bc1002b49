"""GPU parity: the CUDA path through the C ABI against the oracle, element by element, on
seeded inputs that span several tiles, ragged tails and the degenerate cases."""
import math

import numpy as np
import pytest

import oracle
from kv_cache_vector_compress_b200 import synth

from .parity import (as_u16, as_u32, check_close, check_codes, check_f16_close, check_signs, check_topk)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tq():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from kv_cache_vector_compress_b200 import tq as _tq  # raises if libtq.so is missing
    return _tq


def _params(tq, R, S, bits, m):
    import torch
    d = R.shape[0]
    Rt = torch.from_numpy(R).cuda()
    St = torch.from_numpy(S).cuda() if S is not None else None
    return tq.Params(d, bits, m, Rt, St)


def _compress_both(tq, x, R, S, bits, is_key):
    """GPU and oracle compression of the same rows; asserts the parity rules and returns both."""
    import torch
    d = R.shape[0]
    m = S.shape[0] if S is not None else 0
    p = _params(tq, R, S, bits, m)
    xt = torch.from_numpy(x).cuda()
    ora = oracle.compress(x, R, S, bits, is_key=is_key, want_y=True, want_p=is_key)
    if is_key:
        codes, signs, norm, rnorm = tq.tq_compress_keys(p, xt)
    else:
        codes, norm = tq.tq_compress_values(p, xt)
    torch.cuda.synchronize()
    beta = bits - 1 if is_key else bits
    bnd, _ = oracle.codebook_f32(d, beta)
    rows = check_codes(codes, ora["codes"], ora["y32"], bnd, d, beta)
    check_f16_close(norm, ora["norm"], what="norm")
    gpu = {"codes": codes, "norm": norm}
    if is_key:
        check_signs(signs, ora["signs"], ora["p32"], m, exempt_rows=rows)
        check_f16_close(rnorm, ora["rnorm"], exempt_rows=rows, what="rnorm")
        gpu.update(signs=signs, rnorm=rnorm)
    return gpu, ora, rows, p


# ------------------------------------------------------------------ compress

def test_compress_workload1(tq):
    w = synth.workload1()
    _, _, rk, _ = _compress_both(tq, w["K"], w["R"], w["S"], 3, True)
    _, _, rv, _ = _compress_both(tq, w["V"], w["R"], None, 3, False)
    assert len(rk) <= 2 and len(rv) <= 2


@pytest.mark.parametrize("d", [32, 64, 128, 256, 512, 1024])
@pytest.mark.parametrize("n", [1, 31, 33, 257])
@pytest.mark.parametrize("f16", [True, False])
def test_compress_shapes(tq, d, n, f16):
    R = synth.rotation(d, 1000 + d)
    S = synth.gaussian(max(32, d // 2), d, 2000 + d)
    x = synth.gaussian(n, d, 3000 + n + d)
    x = x.astype(np.float16) if f16 else x
    for bits in (2, 3, 4):
        _compress_both(tq, x, R, S, bits, True)
    for bits in (1, 2, 3, 4):
        _compress_both(tq, x, R, None, bits, False)


@pytest.mark.parametrize("d", [128, 256])
def test_compress_zero_and_outlier_rows(tq, d):
    R = synth.rotation(d, 11)
    S = synth.gaussian(d // 2, d, 12)
    x = synth.channel_scaled_f16(96, d, 13, 14, 3)
    x[5] = 0
    x[40, :3] = np.float16(60000.0)  # near the top of the fp16 range
    gk, ok, _, _ = _compress_both(tq, x, R, S, 3, True)
    gv, ov, _, _ = _compress_both(tq, x, R, None, 3, False)
    assert as_u16(gk["norm"])[5] == 0 and as_u16(gv["norm"])[5] == 0


def test_compress_large_projection(tq):
    d, m = 64, 256
    R = synth.rotation(d, 21)
    S = synth.gaussian(m, d, 22)
    x = synth.gaussian(300, d, 23)
    _compress_both(tq, x, R, S, 2, True)


@pytest.mark.parametrize("m", [32, 96, 192, 256])
def test_compress_wide_head_projection_widths(tq, m):
    """d = 256 fp16 keys: one rotation chunk and one projection chunk of any width up to 256,
    a ragged tail and several tiles per CTA."""
    d = 256
    R = synth.rotation(d, 31)
    S = synth.gaussian(m, d, 32 + m)
    x = synth.gaussian(128 * 148 + 300, d, 33).astype(np.float16)
    for bits in (2, 3, 4):
        _compress_both(tq, x, R, S, bits, True)


# -------------------------------------------------------------------- scores

def _oracle_cache(seed, d, m, bits, B, Hkv, T, f16=True):
    R = synth.rotation(d, seed)
    S = synth.gaussian(m, d, seed + 1)
    K = synth.gaussian(B * Hkv * T, d, seed + 2)
    V = synth.gaussian(B * Hkv * T, d, seed + 3)
    if f16:
        K, V = K.astype(np.float16), V.astype(np.float16)
    k = oracle.compress(K, R, S, bits, is_key=True)
    v = oracle.compress(V, R, None, bits, is_key=False)
    return R, S, k, v


def _to_dev(k, v=None):
    import torch
    kk = (torch.from_numpy(k["codes"].view(np.int32)).cuda(), torch.from_numpy(k["signs"].view(np.int32)).cuda(),
          torch.from_numpy(k["norm"].view(np.float16)).cuda(), torch.from_numpy(k["rnorm"].view(np.float16)).cuda())
    if v is None:
        return kk
    vv = (torch.from_numpy(v["codes"].view(np.int32)).cuda(), torch.from_numpy(v["norm"].view(np.float16)).cuda())
    return kk, vv


@pytest.mark.parametrize("cfg", [
    dict(d=128, m=64, bits=3, B=1, Hkv=1, G=1, Nq=16, T=4096),   # workload 1 shape
    dict(d=64, m=32, bits=2, B=2, Hkv=2, G=4, Nq=1, T=300),      # GQA, ragged tail
    dict(d=128, m=64, bits=4, B=1, Hkv=1, G=1, Nq=20, T=129),    # more rows than one pass
    dict(d=256, m=128, bits=2, B=1, Hkv=2, G=2, Nq=2, T=77),     # wide head, 1-bit keys
    dict(d=32, m=32, bits=3, B=3, Hkv=1, G=1, Nq=1, T=1),        # single token
])
def test_scores_on_oracle_cache(tq, cfg):
    import torch
    c = cfg
    R, S, k, _ = _oracle_cache(100 + c["d"] + c["T"], c["d"], c["m"], c["bits"], c["B"], c["Hkv"], c["T"])
    Hq = c["Hkv"] * c["G"]
    q = synth.gaussian(c["B"] * Hq * c["Nq"], c["d"], 7).reshape(c["B"], Hq, c["Nq"], c["d"])
    ora = oracle.scores(q, R, S, c["bits"], c["B"], Hq, c["Hkv"], c["Nq"], c["T"],
                        k["codes"], k["signs"], k["norm"], k["rnorm"])
    p = _params(tq, R, S, c["bits"], c["m"])
    s, _, _ = tq.tq_scores(p, torch.from_numpy(q).cuda(), _to_dev(k), c["Hkv"], c["T"])
    torch.cuda.synchronize()
    check_close(s, ora, "scores")


@pytest.mark.parametrize("k_", [1, 10, 64])
def test_scores_topk(tq, k_):
    import torch
    d, m, bits, T, Nq = 64, 32, 3, 3000, 18
    R, S, k, _ = _oracle_cache(500 + k_, d, m, bits, 1, 1, T, f16=False)
    q = synth.gaussian(Nq, d, 8).reshape(1, 1, Nq, d)
    ora = oracle.scores(q, R, S, bits, 1, 1, 1, Nq, T, k["codes"], k["signs"], k["norm"], k["rnorm"])
    p = _params(tq, R, S, bits, m)
    for want_scores in (True, False):
        s, ti, tv = tq.tq_scores(p, torch.from_numpy(q).cuda(), _to_dev(k), 1, T, want_scores=want_scores,
                                 topk=k_)
        torch.cuda.synchronize()
        if want_scores:
            check_close(s, ora, "scores")
        for r in range(Nq):
            check_topk(ti[0, 0, r].cpu().numpy(), tv[0, 0, r].cpu().numpy(), ora[0, 0, r], k_, f"row {r}")


def test_scores_topk_exact_ties(tq):
    # identical keys give identical scores: ties resolve to the smaller token index
    import torch
    d, m, bits, T = 32, 32, 2, 500
    R = synth.rotation(d, 1)
    S = synth.gaussian(m, d, 2)
    K = np.repeat(synth.gaussian(5, d, 3), 100, axis=0)
    k = oracle.compress(K, R, S, bits, is_key=True)
    q = synth.gaussian(1, d, 4).reshape(1, 1, 1, d)
    p = _params(tq, R, S, bits, m)
    _, ti, tv = tq.tq_scores(p, torch.from_numpy(q).cuda(), _to_dev(k), 1, T, want_scores=False, topk=10)
    ora = oracle.scores(q, R, S, bits, 1, 1, 1, 1, T, k["codes"], k["signs"], k["norm"], k["rnorm"])[0, 0, 0]
    best = int(np.argmax(ora[::100]))
    np.testing.assert_array_equal(ti[0, 0, 0].cpu().numpy(), np.arange(100 * best, 100 * best + 10))


@pytest.mark.parametrize("cfg", [
    dict(d=128, m=64, bits=3, B=1, Hkv=1, G=1, Nq=200, T=1000),   # two row blocks, ragged keys
    dict(d=64, m=64, bits=2, B=2, Hkv=2, G=3, Nq=30, T=300),      # GQA slices, 1-bit keys
    dict(d=256, m=128, bits=4, B=1, Hkv=1, G=1, Nq=129, T=129),   # one row past a block
    # vector-search width with the search workload's unit keys and queries: the 1e-4 absolute
    # bound presumes that scale (with |q| |k| ~ d = 1024, plain fp32 summation alone already
    # rounds near-zero scores by more than 1e-4)
    dict(d=1024, m=512, bits=4, B=1, Hkv=1, G=1, Nq=130, T=300, unit=True),
    dict(d=128, m=128, bits=3, B=1, Hkv=1, G=1, Nq=65, T=1),      # single key
])
def test_search_scores_and_topk(tq, cfg):
    """Many query rows per KV head (the tensor-core path): full scores, and the top-k both fused
    (k <= 16) and as a separate pass (k > 16), against the oracle."""
    import torch
    c = cfg
    seed = 300 + c["d"] + c["T"]
    if c.get("unit"):
        R = synth.rotation(c["d"], seed)
        S = synth.gaussian(c["m"], c["d"], seed + 1)
        K = synth.unit_rows(c["B"] * c["Hkv"] * c["T"], c["d"], seed + 2)
        k = oracle.compress(K, R, S, c["bits"], is_key=True)
    else:
        R, S, k, _ = _oracle_cache(seed, c["d"], c["m"], c["bits"], c["B"], c["Hkv"], c["T"], f16=False)
    Hq = c["Hkv"] * c["G"]
    rows = c["B"] * Hq * c["Nq"]
    q = (synth.unit_rows(rows, c["d"], 9) if c.get("unit") else synth.gaussian(rows, c["d"], 9))
    q = q.reshape(c["B"], Hq, c["Nq"], c["d"])
    ora = oracle.scores(q, R, S, c["bits"], c["B"], Hq, c["Hkv"], c["Nq"], c["T"],
                        k["codes"], k["signs"], k["norm"], k["rnorm"])
    p = _params(tq, R, S, c["bits"], c["m"])
    qd = torch.from_numpy(q).cuda()
    s, _, _ = tq.tq_scores(p, qd, _to_dev(k), c["Hkv"], c["T"])
    torch.cuda.synchronize()
    check_close(s, ora, "scores")
    for k_ in (1, 10, 16, 20):
        if k_ > c["T"]:
            continue
        for want_scores in (False, True):
            s2, ti, tv = tq.tq_scores(p, qd, _to_dev(k), c["Hkv"], c["T"], want_scores=want_scores, topk=k_)
            torch.cuda.synchronize()
            ti, tv = ti.cpu().numpy(), tv.cpu().numpy()
            for b in range(c["B"]):
                for h in range(Hq):
                    for r in range(0, c["Nq"], 7):
                        check_topk(ti[b, h, r], tv[b, h, r], ora[b, h, r], k_, f"k={k_} row {b},{h},{r}")
            if want_scores:
                # the top-k is exactly the k best of the returned scores
                sc = s2.cpu().numpy()
                for r in range(0, c["Nq"], 11):
                    row = sc[0, 0, r].astype(np.float64)
                    order = np.lexsort((np.arange(c["T"]), -row))[:k_]
                    np.testing.assert_array_equal(ti[0, 0, r], order)


@pytest.mark.parametrize("cfg", [
    dict(d=1024, m=512, bits=4, Nq=130, T=300),   # the vector-search width
    dict(d=128, m=64, bits=3, Nq=200, T=1000),    # two row blocks, ragged keys
    dict(d=128, m=64, bits=3, Nq=16, T=500),      # few rows: not the tensor-core search path
])
def test_search_fp16_operands(tq, cfg):
    """tq_search (single fp16 operand products) on unit keys and queries: every score within the
    header's bound 2^-10 ||k|| (sum_i |q_rot,i c_i| + rho gamma sum_j |(S q)_j|) of the exact
    tq_scores; at the vector-search width (d = 1024, typical error ~1e-5) also within the scores
    tolerance of the oracle, which d = 128 (typical error ~3e-5, tail ~1.5e-4) does not promise;
    top-k against the oracle.  Shapes outside the tensor-core search run exactly as tq_scores."""
    import torch
    c = cfg
    d, m, bits, Nq, T = c["d"], c["m"], c["bits"], c["Nq"], c["T"]
    seed = 700 + d + T
    R = synth.rotation(d, seed)
    S = synth.gaussian(m, d, seed + 1)
    K = synth.unit_rows(T, d, seed + 2)
    k = oracle.compress(K, R, S, bits, is_key=True)
    q = synth.unit_rows(Nq, d, seed + 3).reshape(1, 1, Nq, d)
    ora = oracle.scores(q, R, S, bits, 1, 1, 1, Nq, T, k["codes"], k["signs"], k["norm"], k["rnorm"])
    p = _params(tq, R, S, bits, m)
    qd = torch.from_numpy(q).cuda()
    s16, _, _ = tq.tq_search(p, qd, _to_dev(k), 1, T)
    s32, _, _ = tq.tq_scores(p, qd, _to_dev(k), 1, T)
    torch.cuda.synchronize()
    s16, s32 = s16.cpu().numpy()[0, 0].astype(np.float64), s32.cpu().numpy()[0, 0].astype(np.float64)
    if d >= 1024 or Nq <= 64:
        check_close(s16, ora[0, 0], "fp16-operand scores")
    # the stated bound, per score, from the oracle's own quantities
    nk = np.array([oracle.f16_bits_to_f64(int(h)) for h in as_u16(k["norm"])])
    rho = np.array([oracle.f16_bits_to_f64(int(h)) for h in as_u16(k["rnorm"])])
    idx = np.stack([oracle.unpack_codes(w, d, bits - 1) for w in k["codes"]])  # [T, d]
    cvals = oracle.codebook(d, bits - 1)[1][idx]                     # centroids c[idx] [T, d]
    qr = q[0, 0].astype(np.float64) @ R.astype(np.float64).T       # q_rot [Nq, d]
    sq = q[0, 0].astype(np.float64) @ S.astype(np.float64).T       # S q [Nq, m]
    gamma = math.sqrt(math.pi / 2) / m
    bound = 2.0 ** -10 * nk[None, :] * (np.abs(qr) @ np.abs(cvals).T + gamma * rho[None, :] *
                                        np.abs(sq).sum(1)[:, None])
    err = np.abs(s16 - s32)
    assert np.all(err <= bound + 1e-6), f"max excess {np.max(err - bound)}"
    if Nq <= 64:
        np.testing.assert_array_equal(s16, s32)
    for k_ in (1, 10, 20):  # 20: past the fused top-k, a separate pass over the fp16-operand scores
        _, ti, tv = tq.tq_search(p, qd, _to_dev(k), 1, T, want_scores=False, topk=k_)
        torch.cuda.synchronize()
        ti, tv = ti.cpu().numpy()[0, 0], tv.cpu().numpy()[0, 0]
        for r in range(0, Nq, 7):
            check_topk(ti[r], tv[r], ora[0, 0, r], k_, f"k={k_} row {r}")


@pytest.mark.parametrize("fn", ["tq_scores", "tq_search"])
def test_sharded_search_topk_merge(tq, fn):
    """The sharded vector search on one GPU: a database split into two row ranges, the fused
    top-k of each range (indices made global by the range's offset) merged by dist.merge_topk,
    equals the top-k of one call over the whole database, and matches the oracle's top-k."""
    import torch
    from kv_cache_vector_compress_b200 import dist
    d, m, bits, Nq, T, k = 1024, 512, 4, 130, 700, 10
    R = synth.rotation(d, 41)
    S = synth.gaussian(m, d, 42)
    K = synth.unit_rows(T, d, 43)
    kk = oracle.compress(K, R, S, bits, is_key=True)
    q = synth.unit_rows(Nq, d, 44).reshape(1, 1, Nq, d)
    ora = oracle.scores(q, R, S, bits, 1, 1, 1, Nq, T, kk["codes"], kk["signs"], kk["norm"], kk["rnorm"])
    p = _params(tq, R, S, bits, m)
    qd = torch.from_numpy(q).cuda()
    call = getattr(tq, fn)
    dev = _to_dev(kk)
    _, ti, tv = call(p, qd, dev, 1, T, want_scores=False, topk=k)
    cut = 300  # a range boundary inside a 128-key tile
    parts_v, parts_i = [], []
    for a, b in ((0, cut), (cut, T)):
        sub = tuple(x[a:b].clone() for x in dev)  # each shard in its own (16-byte aligned) buffers
        _, si, sv = call(p, qd, sub, 1, b - a, want_scores=False, topk=k)
        parts_v.append(sv)
        parts_i.append(si.to(torch.int64) + a)
    mi, mv = dist.merge_topk(torch.cat(parts_v, -1), torch.cat(parts_i, -1), k)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(mi.cpu().numpy(), ti.cpu().numpy().astype(np.int64))
    np.testing.assert_array_equal(mv.cpu().numpy(), tv.cpu().numpy())
    for r in range(0, Nq, 13):
        check_topk(ti[0, 0, r].cpu().numpy(), tv[0, 0, r].cpu().numpy(), ora[0, 0, r], k, f"{fn} row {r}")


def test_search_topk_exact_ties(tq):
    # identical keys, many query rows: ties resolve to the smaller token index across CTAs too
    import torch
    d, m, bits, T, Nq = 64, 64, 3, 4000, 100
    R = synth.rotation(d, 11)
    S = synth.gaussian(m, d, 12)
    K = np.repeat(synth.gaussian(8, d, 13), 500, axis=0)
    k = oracle.compress(K, R, S, bits, is_key=True)
    q = synth.gaussian(Nq, d, 14).reshape(1, 1, Nq, d)
    p = _params(tq, R, S, bits, m)
    _, ti, _ = tq.tq_scores(p, torch.from_numpy(q).cuda(), _to_dev(k), 1, T, want_scores=False, topk=16)
    ora = oracle.scores(q, R, S, bits, 1, 1, 1, Nq, T, k["codes"], k["signs"], k["norm"], k["rnorm"])[0, 0]
    for r in range(Nq):
        vals = ora[r, ::500]
        best = int(np.argmax(vals))
        if np.sort(vals)[-2] > vals[best] - 1e-3 * abs(vals[best]) - 1e-4:
            continue  # two groups too close to call
        np.testing.assert_array_equal(ti[0, 0, r].cpu().numpy(), np.arange(500 * best, 500 * best + 16))


def test_search_topk_increasing_scores(tq):
    # scaled copies of one direction: each query's scores rise (or fall) with the key index, so
    # every tile brings new top-k entries for half of the rows
    import torch
    d, m, bits, T, Nq = 128, 64, 3, 3000, 100
    R = synth.rotation(d, 31)
    S = synth.gaussian(m, d, 32)
    v = synth.unit_rows(1, d, 33)
    K = (v * (1.0 + np.arange(T, dtype=np.float32)[:, None] / T)).astype(np.float32)
    k = oracle.compress(K, R, S, bits, is_key=True)
    q = synth.gaussian(Nq, d, 34).reshape(1, 1, Nq, d)
    p = _params(tq, R, S, bits, m)
    ora = oracle.scores(q, R, S, bits, 1, 1, 1, Nq, T, k["codes"], k["signs"], k["norm"], k["rnorm"])[0, 0]
    for k_ in (1, 10, 16):
        _, ti, tv = tq.tq_scores(p, torch.from_numpy(q).cuda(), _to_dev(k), 1, T, want_scores=False, topk=k_)
        torch.cuda.synchronize()
        for r in range(Nq):
            check_topk(ti[0, 0, r].cpu().numpy(), tv[0, 0, r].cpu().numpy(), ora[r], k_, f"k={k_} row {r}")


# -------------------------------------------------------------------- attend

@pytest.mark.parametrize("cfg", [
    dict(d=128, m=64, bits=3, B=1, Hkv=1, G=1, Nq=16, T=4096),
    dict(d=128, m=64, bits=3, B=2, Hkv=2, G=4, Nq=1, T=1000),
    dict(d=64, m=32, bits=2, B=1, Hkv=1, G=2, Nq=10, T=1),
    dict(d=64, m=32, bits=4, B=1, Hkv=2, G=1, Nq=17, T=129),
    dict(d=256, m=128, bits=2, B=1, Hkv=1, G=4, Nq=1, T=3000),
    dict(d=256, m=128, bits=4, B=1, Hkv=1, G=4, Nq=1, T=513),
    dict(d=32, m=32, bits=1 + 1, B=1, Hkv=1, G=1, Nq=1, T=127),
    # bit-plane shapes (at most 4 query rows per KV head, proj_dim = dim / 2) at their edges
    dict(d=64, m=32, bits=3, B=2, Hkv=1, G=4, Nq=1, T=1),      # a single token
    dict(d=128, m=64, bits=4, B=1, Hkv=2, G=2, Nq=2, T=31),    # under one 32-token stage
    dict(d=64, m=32, bits=2, B=1, Hkv=1, G=1, Nq=3, T=2049),   # three ranges, 3 rows, ragged tail
])
def test_attend_on_oracle_cache(tq, cfg):
    import torch
    c = cfg
    R, S, k, v = _oracle_cache(300 + c["d"] + c["T"], c["d"], c["m"], c["bits"], c["B"], c["Hkv"], c["T"])
    Hq = c["Hkv"] * c["G"]
    q = synth.gaussian(c["B"] * Hq * c["Nq"], c["d"], 9).reshape(c["B"], Hq, c["Nq"], c["d"])
    ora = oracle.attend(q, R, S, c["bits"], c["B"], Hq, c["Hkv"], c["Nq"], c["T"], k["codes"], k["signs"],
                        k["norm"], k["rnorm"], v["codes"], v["norm"])
    p = _params(tq, R, S, c["bits"], c["m"])
    kk, vv = _to_dev(k, v)
    out = tq.tq_attend(p, torch.from_numpy(q).cuda(), kk, vv, c["Hkv"], c["T"])
    torch.cuda.synchronize()
    check_close(out, ora, "attend")
    # an explicit temperature
    ora2 = oracle.attend(q, R, S, c["bits"], c["B"], Hq, c["Hkv"], c["Nq"], c["T"], k["codes"], k["signs"],
                         k["norm"], k["rnorm"], v["codes"], v["norm"], scale=0.02)
    out2 = tq.tq_attend(p, torch.from_numpy(q).cuda(), kk, vv, c["Hkv"], c["T"], scale=0.02)
    torch.cuda.synchronize()
    check_close(out2, ora2, "attend scale=0.02")


@pytest.mark.parametrize("dtype", ["f16", "f32"])
def test_compress_attend_host(tq, dtype):
    """tq_compress_attend_host: host K/V/Q in, host output out, through one C-ABI call.  The cache
    arrays it writes equal those of tq_compress_keys / tq_compress_values on the same inputs, its
    output equals tq_attend's over them, and the output matches the oracle's attention over the
    oracle's own compression of the inputs where the packed records agree (all of them here)."""
    import torch
    d, m, bits, B, Hq, Hkv, Nq, T = 128, 64, 3, 2, 8, 2, 1, 300
    seed = 900 + (dtype == "f32")
    R = synth.rotation(d, seed)
    S = synth.gaussian(m, d, seed + 1)
    n = B * Hkv * T
    K = synth.gaussian(n, d, seed + 2)
    V = synth.gaussian(n, d, seed + 3)
    if dtype == "f16":
        K, V = K.astype(np.float16), V.astype(np.float16)
    q = synth.gaussian(B * Hq * Nq, d, seed + 4).reshape(B, Hq, Nq, d)
    p = _params(tq, R, S, bits, m)
    hK = torch.from_numpy(K).reshape(B, Hkv, T, d).pin_memory()
    hV = torch.from_numpy(V).reshape(B, Hkv, T, d).pin_memory()
    hQ = torch.from_numpy(q).pin_memory()
    hO = torch.full((B, Hq, Nq, d), float("nan"), dtype=torch.float32).pin_memory()
    kz = (torch.zeros((n, p.key_words()), dtype=torch.int32, device="cuda"),
          torch.zeros((n, m // 32), dtype=torch.int32, device="cuda"),
          torch.zeros(n, dtype=torch.float16, device="cuda"), torch.zeros(n, dtype=torch.float16, device="cuda"))
    vz = (torch.zeros((n, p.value_words()), dtype=torch.int32, device="cuda"),
          torch.zeros(n, dtype=torch.float16, device="cuda"))
    tq.tq_compress_attend_host(p, hK, hV, hQ, Hkv, T, kz, vz, hO)
    torch.cuda.synchronize()
    Kd, Vd = hK.cuda().view(n, d), hV.cuda().view(n, d)
    kt, vt = tq.tq_compress_keys(p, Kd), tq.tq_compress_values(p, Vd)
    ref = tq.tq_attend(p, hQ.cuda(), kt, vt, Hkv, T)
    torch.cuda.synchronize()
    for a, b in zip(kz + vz, kt + vt):
        assert torch.equal(a, b)
    np.testing.assert_array_equal(hO.numpy(), ref.cpu().numpy())
    k = oracle.compress(K.astype(np.float32) if dtype == "f32" else K, R, S, bits, is_key=True)
    v = oracle.compress(V.astype(np.float32) if dtype == "f32" else V, R, None, bits, is_key=False)
    ora = oracle.attend(q, R, S, bits, B, Hq, Hkv, Nq, T, k["codes"], k["signs"], k["norm"], k["rnorm"],
                        v["codes"], v["norm"])
    same = ((as_u32(kz[0]) == k["codes"]).all(1) & (as_u32(kz[1]) == k["signs"]).all(1)
            & (as_u16(kz[2]) == k["norm"]) & (as_u16(kz[3]) == k["rnorm"])
            & (as_u32(vz[0]) == v["codes"]).all(1) & (as_u16(vz[1]) == v["norm"]))
    if same.all():
        check_close(hO, ora, "host-step attend")


def test_end_to_end_workload1(tq):
    """Compress with the GPU, attend with the GPU; oracle does the same from the same inputs."""
    import torch
    w = synth.workload1()
    R, S = w["R"], w["S"]
    p = _params(tq, R, S, 3, 64)
    kt = tq.tq_compress_keys(p, torch.from_numpy(w["K"]).cuda())
    vt = tq.tq_compress_values(p, torch.from_numpy(w["V"]).cuda())
    q = torch.from_numpy(w["Q"]).cuda()
    out = tq.tq_attend(p, q, kt, vt, 1, 4096)
    s, _, _ = tq.tq_scores(p, q, kt, 1, 4096)
    torch.cuda.synchronize()
    k = oracle.compress(w["K"], R, S, 3, is_key=True)
    v = oracle.compress(w["V"], R, None, 3, is_key=False)
    ora_out = oracle.attend(w["Q"], R, S, 3, 1, 1, 1, 16, 4096, k["codes"], k["signs"], k["norm"], k["rnorm"],
                            v["codes"], v["norm"])
    check_close(out, ora_out, "end-to-end attend")
    ora_s = oracle.scores(w["Q"], R, S, 3, 1, 1, 1, 16, 4096, k["codes"], k["signs"], k["norm"], k["rnorm"])
    # keys whose packed records are identical must score within tolerance
    same = ((as_u32(kt[0]) == k["codes"]).all(1) & (as_u32(kt[1]) == k["signs"]).all(1)
            & (as_u16(kt[2]) == k["norm"]) & (as_u16(kt[3]) == k["rnorm"]))
    assert same.mean() > 0.999
    check_close(s[0, 0][:, torch.from_numpy(same).cuda()], ora_s[0, 0][:, same], "end-to-end scores")


# ------------------------------------------------------- decode-step append + attend

@pytest.mark.parametrize("cfg", [
    dict(d=128, m=64, bits=3, B=2, Hkv=2, G=4, Nq=1, t=1000, cap=1100, f16=True),   # GQA decode step
    dict(d=64, m=32, bits=2, B=1, Hkv=3, G=1, Nq=2, t=0, cap=5, f16=False),         # empty cache, fp32 rows
    dict(d=256, m=128, bits=4, B=1, Hkv=1, G=8, Nq=1, t=4094, cap=4095, f16=True),  # last slot, wide head
    dict(d=128, m=64, bits=2, B=1, Hkv=1, G=16, Nq=1, t=333, cap=400, f16=True),    # two row groups
    dict(d=32, m=32, bits=3, B=2, Hkv=1, G=2, Nq=1, t=50, cap=64, f16=True),        # append kernel + CUDA-core attention
    dict(d=128, m=128, bits=3, B=1, Hkv=2, G=2, Nq=3, t=200, cap=256, f16=False),   # proj_dim = dim: same path
    dict(d=128, m=64, bits=3, B=1, Hkv=2, G=2, Nq=2, t=77, cap=90, f16=False),      # bit-plane shape, fp32 rows
    dict(d=256, m=128, bits=2, B=1, Hkv=2, G=4, Nq=1, t=600, cap=700, f16=True),    # bit-plane shape, wide head
])
def test_append_attend(tq, cfg):
    """tq_append_attend writes the oracle's records for the new token into slot t, leaves every other
    slot alone, and attends over slots 0..t exactly as the oracle does over that cache."""
    import torch
    c = cfg
    d, m, bits, B, Hkv, t, cap = c["d"], c["m"], c["bits"], c["B"], c["Hkv"], c["t"], c["cap"]
    Hq, nsl = Hkv * c["G"], B * Hkv
    seed = 500 + d + t
    R, S = synth.rotation(d, seed), synth.gaussian(m, d, seed + 1)
    dt = np.float16 if c["f16"] else np.float32
    # every slot of the cache holds a valid record, so reading past slot t would change the output
    K = synth.gaussian(nsl * cap, d, seed + 2).astype(np.float16)
    V = synth.gaussian(nsl * cap, d, seed + 3).astype(np.float16)
    k = oracle.compress(K, R, S, bits, is_key=True)
    v = oracle.compress(V, R, None, bits, is_key=False)
    k_new = synth.gaussian(nsl, d, seed + 4).astype(dt)
    v_new = synth.gaussian(nsl, d, seed + 5).astype(dt)
    q = synth.gaussian(B * Hq * c["Nq"], d, seed + 6).reshape(B, Hq, c["Nq"], d)
    p = _params(tq, R, S, bits, m)
    kk, vv = _to_dev(k, v)
    out = tq.tq_append_attend(p, torch.from_numpy(q).cuda(), torch.from_numpy(k_new).cuda(),
                              torch.from_numpy(v_new).cuda(), kk, vv, Hkv, t, cap)
    torch.cuda.synchronize()

    def slots(a):
        a = a.cpu().numpy() if hasattr(a, "cpu") else a
        return a.reshape(nsl, cap, -1)

    g = {n: slots(x) for n, x in zip(("kc", "ks", "kn", "kr"), kk)}
    g.update({n: slots(x) for n, x in zip(("vc", "vn"), vv)})
    # the new records against the oracle's compression of the new rows
    kb, vb = bits - 1, bits
    ok_ = oracle.compress(k_new, R, S, bits, is_key=True, want_y=True, want_p=True)
    ov_ = oracle.compress(v_new, R, None, bits, is_key=False, want_y=True)
    rows = check_codes(g["kc"][:, t].view(np.uint32), ok_["codes"], ok_["y32"], oracle.codebook_f32(d, kb)[0], d, kb,
                       what="appended key codes")
    check_signs(g["ks"][:, t].view(np.uint32), ok_["signs"], ok_["p32"], m, exempt_rows=rows, what="appended signs")
    check_f16_close(g["kn"][:, t].view(np.uint16).ravel(), ok_["norm"], what="appended key norm")
    check_f16_close(g["kr"][:, t].view(np.uint16).ravel(), ok_["rnorm"], exempt_rows=rows, what="appended rnorm")
    check_codes(g["vc"][:, t].view(np.uint32), ov_["codes"], ov_["y32"], oracle.codebook_f32(d, vb)[0], d, vb,
                what="appended value codes")
    check_f16_close(g["vn"][:, t].view(np.uint16).ravel(), ov_["norm"], what="appended value norm")
    # every other slot untouched
    other = np.ones(cap, bool)
    other[t] = False
    for name, ref in (("kc", k["codes"]), ("ks", k["signs"]), ("kn", k["norm"]), ("kr", k["rnorm"]),
                      ("vc", v["codes"]), ("vn", v["norm"])):
        gv = g[name][:, other].reshape(-1).view(np.uint16 if name in ("kn", "kr", "vn") else np.uint32)
        rv = ref.reshape(nsl, cap, -1)[:, other].reshape(-1)
        assert np.array_equal(gv, rv), f"slot other than t changed in {name}"
    # attention over slots 0..t of the cache as the GPU left it
    def upto(a, dtype):
        r = np.ascontiguousarray(a[:, : t + 1]).view(dtype).reshape(nsl * (t + 1), -1)
        return r[:, 0] if r.shape[1] == 1 else r
    ora = oracle.attend(q, R, S, bits, B, Hq, Hkv, c["Nq"], t + 1, upto(g["kc"], np.uint32), upto(g["ks"], np.uint32),
                        upto(g["kn"], np.uint16), upto(g["kr"], np.uint16), upto(g["vc"], np.uint32),
                        upto(g["vn"], np.uint16))
    check_close(out, ora, "append + attend")


# ------------------------------------------------------- the exact (Beta) coordinate law

@pytest.mark.parametrize("d,bits", [(128, 3), (256, 2), (64, 4)])
def test_beta_law_compress_scores_attend(tq, d, bits):
    """Parameter sets prepared with the Beta-law codebooks (tq_prepare_law): compression, scores
    and attention against the oracle using the same law."""
    import torch
    m = d // 2
    seed = 700 + d + bits
    R, S = synth.rotation(d, seed), synth.gaussian(m, d, seed + 1)
    p = tq.Params(d, bits, m, torch.from_numpy(R).cuda(), torch.from_numpy(S).cuda(), law="beta")
    B, Hkv, G, T = 1, 2, 4, 700
    x = synth.gaussian(B * Hkv * T, d, seed + 2).astype(np.float16)
    v = synth.gaussian(B * Hkv * T, d, seed + 3).astype(np.float16)
    gk = tq.tq_compress_keys(p, torch.from_numpy(x).cuda())
    gv = tq.tq_compress_values(p, torch.from_numpy(v).cuda())
    torch.cuda.synchronize()
    ok = oracle.compress(x, R, S, bits, is_key=True, want_y=True, want_p=True, law="beta")
    ov = oracle.compress(v, R, None, bits, is_key=False, want_y=True, law="beta")
    rows = check_codes(gk[0], ok["codes"], ok["y32"], oracle.codebook_f32(d, bits - 1, law="beta")[0], d, bits - 1)
    check_signs(gk[1], ok["signs"], ok["p32"], m, exempt_rows=rows)
    check_f16_close(gk[2], ok["norm"], what="norm")
    check_codes(gv[0], ov["codes"], ov["y32"], oracle.codebook_f32(d, bits, law="beta")[0], d, bits)
    # scores and attention over the oracle's records (same law on both sides)
    Hq = Hkv * G
    q = synth.gaussian(B * Hq, d, seed + 4).reshape(B, Hq, 1, d)
    qd = torch.from_numpy(q).cuda()
    kk, vv = _to_dev(ok, ov)
    s, _, _ = tq.tq_scores(p, qd, kk, Hkv, T)
    out = tq.tq_attend(p, qd, kk, vv, Hkv, T)
    torch.cuda.synchronize()
    ora_s = oracle.scores(q, R, S, bits, B, Hq, Hkv, 1, T, ok["codes"], ok["signs"], ok["norm"], ok["rnorm"],
                          law="beta")
    check_close(s, ora_s, "beta-law scores")
    ora_o = oracle.attend(q, R, S, bits, B, Hq, Hkv, 1, T, ok["codes"], ok["signs"], ok["norm"], ok["rnorm"],
                          ov["codes"], ov["norm"], law="beta")
    check_close(out, ora_o, "beta-law attention")


# ------------------------------------------- one long context split into pieces (multi-GPU)

@pytest.mark.parametrize("cfg", [
    dict(d=128, m=64, bits=3, B=2, Hkv=2, G=4, Nq=1, cuts=(0, 1000, 2100, 3000)),  # bit-plane kernel
    dict(d=256, m=128, bits=2, B=1, Hkv=1, G=4, Nq=1, cuts=(0, 1, 700)),          # a one-token piece
    dict(d=64, m=32, bits=4, B=1, Hkv=2, G=1, Nq=9, cuts=(0, 129, 400)),          # register-MMA kernel
    dict(d=32, m=32, bits=3, B=1, Hkv=1, G=2, Nq=1, cuts=(0, 60, 61, 127)),       # CUDA-core kernel
])
def test_context_pieces_merge_to_whole_attention(tq, cfg):
    """The context of every (batch, KV head) cut into pieces, as ranks that each hold one token
    range would hold them: tq_attend_partial on each piece, tq_attend_merge of the stacked
    partials, against the oracle's attention over the whole context."""
    import torch
    c = cfg
    cuts = c["cuts"]
    T = cuts[-1]
    R, S, k, v = _oracle_cache(900 + c["d"] + T, c["d"], c["m"], c["bits"], c["B"], c["Hkv"], T)
    Hq = c["Hkv"] * c["G"]
    q = synth.gaussian(c["B"] * Hq * c["Nq"], c["d"], 19).reshape(c["B"], Hq, c["Nq"], c["d"])
    ora = oracle.attend(q, R, S, c["bits"], c["B"], Hq, c["Hkv"], c["Nq"], T, k["codes"], k["signs"], k["norm"],
                        k["rnorm"], v["codes"], v["norm"])
    p = _params(tq, R, S, c["bits"], c["m"])
    qd = torch.from_numpy(q).cuda()
    nsl = c["B"] * c["Hkv"]

    def piece(a, t0, t1):
        return np.ascontiguousarray(a.reshape(nsl, T, -1)[:, t0:t1]).reshape(nsl * (t1 - t0), -1)

    parts = []
    for t0, t1 in zip(cuts[:-1], cuts[1:]):
        kp = {n: piece(k[n], t0, t1) for n in ("codes", "signs")}
        kp.update({n: piece(k[n].reshape(-1, 1), t0, t1).reshape(-1) for n in ("norm", "rnorm")})
        vp = {"codes": piece(v["codes"], t0, t1), "norm": piece(v["norm"].reshape(-1, 1), t0, t1).reshape(-1)}
        kk, vv = _to_dev(kp, vp)
        parts.append(tq.tq_attend_partial(p, qd, kk, vv, c["Hkv"], t1 - t0))
    out = tq.tq_attend_merge(p, torch.stack(parts))
    torch.cuda.synchronize()
    check_close(out, ora, "merged context pieces")
