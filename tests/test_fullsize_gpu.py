"""Full-size workloads on the GPU, checked against the oracle on sampled outputs (the oracle
recomputes those rows, slices or scores from the same inputs) and by properties that hold at
any size.  Inputs are generated on the device with a seeded generator and the sampled rows
are copied to the host for the oracle."""
import numpy as np
import pytest

import oracle
from kv_cache_vector_compress_b200 import synth

from .parity import as_u16, as_u32, check_close, check_codes, check_f16_close, check_signs, check_topk

pytestmark = pytest.mark.gpu

N_SAMPLE = 2048


@pytest.fixture(scope="module")
def tq():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from kv_cache_vector_compress_b200 import tq as _tq
    return _tq


def _sample_rows(n, k, seed):
    rng = np.random.default_rng(seed)
    rows = np.unique(np.concatenate([rng.choice(n, size=k, replace=False), [0, n - 1]]))
    return rows


def _check_sampled_compress(gpu, x_dev, rows, R, S, bits, is_key):
    import torch
    d = R.shape[0]
    xs = x_dev[torch.from_numpy(rows).cuda()].cpu().numpy()
    ora = oracle.compress(xs, R, S, bits, is_key=is_key, want_y=True, want_p=is_key)
    idx = torch.from_numpy(rows).cuda()
    beta = bits - 1 if is_key else bits
    bnd, _ = oracle.codebook_f32(d, beta)
    bad_rows = check_codes(gpu[0][idx], ora["codes"], ora["y32"], bnd, d, beta)
    if is_key:
        check_signs(gpu[1][idx], ora["signs"], ora["p32"], S.shape[0], exempt_rows=bad_rows)
        check_f16_close(gpu[2][idx], ora["norm"])
        check_f16_close(gpu[3][idx], ora["rnorm"], exempt_rows=bad_rows, what="rnorm")
    else:
        check_f16_close(gpu[1][idx], ora["norm"])
    return bad_rows


def _qwen_shaped(n_groups, T, d, seed, scale_seed):
    """N(0,1) x per-(layer, head, channel) lognormal(0,1) scales, fp16, on the device."""
    import torch
    base = synth.torch_normal_f16((n_groups * T, d), seed)
    sc = np.exp(np.random.Generator(np.random.PCG64(scale_seed)).standard_normal((n_groups, d)))
    sct = torch.from_numpy(sc.astype(np.float32)).cuda()
    x = (base.view(n_groups, T, d).float() * sct[:, None, :]).half().view(n_groups * T, d)
    return x


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_workload2_qwen_shaped_prefill(tq, bits):
    import torch
    d, m, L, H, T = 128, 64, 36, 2, 8192
    s = synth.seeds(2)
    R = synth.rotation(d, s["R"])
    S = synth.gaussian(m, d, s["S"])
    p = tq.Params(d, bits, m, torch.from_numpy(R).cuda(), torch.from_numpy(S).cuda())
    K = _qwen_shaped(L * H, T, d, s["keys"], s["scales"])
    V = _qwen_shaped(L * H, T, d, s["values"], s["scales"] + 100)
    keys = tq.tq_compress_keys(p, K)
    vals = tq.tq_compress_values(p, V)
    torch.cuda.synchronize()
    n = L * H * T
    rows = _sample_rows(n, N_SAMPLE, bits)
    _check_sampled_compress(keys, K, rows, R, S, bits, True)
    _check_sampled_compress(vals, V, rows, R, None, bits, False)
    # the packed cache has the size the record layout states
    nbytes = sum(t.numel() * t.element_size() for t in keys + vals)
    assert nbytes == n * (((bits - 1) * d + m) // 8 + 4 + bits * d // 8 + 2)


def _decode_workload(tq, d, m, bits, B, Hq, Hkv, T, s, key_outliers=None):
    import torch
    n = B * Hkv * T
    R = synth.rotation(d, s["R"])
    S = synth.gaussian(m, d, s["S"])
    p = tq.Params(d, bits, m, torch.from_numpy(R).cuda(), torch.from_numpy(S).cuda())
    K = synth.torch_normal_f16((n, d), s["keys"])
    if key_outliers is not None:
        K[:, torch.from_numpy(key_outliers).cuda()] *= 20
    V = synth.torch_normal_f16((n, d), s["values"])
    Q = synth.torch_normal_f32((B, Hq, 1, d), s["queries"])
    keys = tq.tq_compress_keys(p, K)
    vals = tq.tq_compress_values(p, V)
    out = tq.tq_attend(p, Q, keys, vals, Hkv, T)
    torch.cuda.synchronize()
    return p, R, S, K, V, Q, keys, vals, out


def _check_slice(tq, p, R, S, bits, K, V, Q, keys, vals, b, kv, Hq, Hkv, T):
    """Attention parity of one (batch, KV-head) slice in the full-size launch: the oracle
    compresses the slice's T keys and values from the same inputs; its packed records are
    written over that slice of the GPU cache; the full-size tq_attend runs again and the
    slice's output rows are compared with the oracle's attention over its own records.
    The GPU's own records of the slice must agree with the oracle's almost everywhere."""
    import torch
    G = Hq // Hkv
    sl = b * Hkv + kv
    rows = slice(sl * T, (sl + 1) * T)
    Ks = K[rows].cpu().numpy()
    Vs = V[rows].cpu().numpy()
    q = Q[b, kv * G:(kv + 1) * G].cpu().numpy().reshape(1, G, 1, -1)
    k = oracle.compress(Ks, R, S, bits, is_key=True)
    v = oracle.compress(Vs, R, None, bits, is_key=False)
    same = ((as_u32(keys[0][rows]) == k["codes"]).all(1) & (as_u32(keys[1][rows]) == k["signs"]).all(1)
            & (as_u32(vals[0][rows]) == v["codes"]).all(1))
    assert same.mean() > 0.995, f"only {same.mean():.4%} of the slice's records match"
    ref = oracle.attend(q, R, S, bits, 1, G, 1, 1, T, k["codes"], k["signs"], k["norm"], k["rnorm"],
                        v["codes"], v["norm"])
    for dst, src in ((keys[0], k["codes"].view(np.int32)), (keys[1], k["signs"].view(np.int32)),
                     (keys[2], k["norm"].view(np.float16)), (keys[3], k["rnorm"].view(np.float16)),
                     (vals[0], v["codes"].view(np.int32)), (vals[1], v["norm"].view(np.float16))):
        dst[rows] = torch.from_numpy(np.ascontiguousarray(src)).cuda()
    out = tq.tq_attend(p, Q, keys, vals, Hkv, T)
    torch.cuda.synchronize()
    check_close(out[b, kv * G:(kv + 1) * G].cpu().numpy().reshape(ref.shape), ref, f"slice ({b},{kv})")


def test_workload3_decode_attention(tq):
    d, m, bits, B, Hq, Hkv, T = 128, 64, 3, 32, 32, 8, 32768
    s = synth.seeds(3)
    p, R, S, K, V, Q, keys, vals, out = _decode_workload(tq, d, m, bits, B, Hq, Hkv, T, s)
    rows = _sample_rows(B * Hkv * T, N_SAMPLE, 3)
    _check_sampled_compress(keys, K, rows, R, S, bits, True)
    _check_sampled_compress(vals, V, rows, R, None, bits, False)
    for b, kv in [(0, 0), (17, 5), (31, 7)]:
        _check_slice(tq, p, R, S, bits, K, V, Q, keys, vals, b, kv, Hq, Hkv, T)


@pytest.mark.parametrize("bits", [2, 4])
def test_workload4_wide_heads(tq, bits):
    d, m, B, Hq, Hkv, T = 256, 128, 8, 16, 4, 65536
    s = synth.seeds(4)
    outl = synth.outlier_channels(d, s["scales"])
    p, R, S, K, V, Q, keys, vals, out = _decode_workload(tq, d, m, bits, B, Hq, Hkv, T, s, key_outliers=outl)
    rows = _sample_rows(B * Hkv * T, N_SAMPLE // 2, 40 + bits)
    _check_sampled_compress(keys, K, rows, R, S, bits, True)
    _check_sampled_compress(vals, V, rows, R, None, bits, False)
    _check_slice(tq, p, R, S, bits, K, V, Q, keys, vals, 5, 2, Hq, Hkv, T)


def test_workload5_vector_search(tq):
    import torch
    d, m, bits, N, Nq, k = 1024, 512, 4, 1_000_000, 1024, 10
    s = synth.seeds(5)
    R = synth.rotation(d, s["R"])
    S = synth.gaussian(m, d, s["S"])
    p = tq.Params(d, bits, m, torch.from_numpy(R).cuda(), torch.from_numpy(S).cuda())
    X = synth.torch_normal_f32((N, d), s["keys"])
    X /= X.norm(dim=1, keepdim=True)
    Q = synth.torch_normal_f32((1, 1, Nq, d), s["queries"])
    Q /= Q.norm(dim=-1, keepdim=True)
    keys = tq.tq_compress_keys(p, X)
    sc, ti, tv = tq.tq_scores(p, Q, keys, 1, N, want_scores=True, topk=k)
    torch.cuda.synchronize()
    rows = _sample_rows(N, 256, 5)
    bad = _check_sampled_compress(keys, X, rows, R, S, bits, True)
    # sampled scores: oracle scores of the sampled keys (compressed by the oracle from the same
    # inputs) for 16 queries, compared where the packed records agree
    xs = X[torch.from_numpy(rows).cuda()].cpu().numpy()
    ok = oracle.compress(xs, R, S, bits, is_key=True)
    qs = Q[0, 0, :16].cpu().numpy().reshape(1, 1, 16, d)
    ora = oracle.scores(qs, R, S, bits, 1, 1, 1, 16, len(rows), ok["codes"], ok["signs"], ok["norm"], ok["rnorm"])
    keep = np.array([i for i in range(len(rows)) if i not in bad])
    g = sc[0, 0, :16][:, torch.from_numpy(rows[keep]).cuda()].cpu().numpy()
    check_close(g, ora[0, 0][:, keep], "sampled scores")
    # the fp16-operand search (the launch the vector-search benchmark times) on the same keys
    sc16, ti16, tv16 = tq.tq_search(p, Q, keys, 1, N, want_scores=True, topk=k)
    torch.cuda.synchronize()
    g16 = sc16[0, 0, :16][:, torch.from_numpy(rows[keep]).cuda()].cpu().numpy()
    check_close(g16, ora[0, 0][:, keep], "sampled fp16-operand scores")
    for r in range(0, Nq, 97):
        row = sc16[0, 0, r].cpu().numpy().astype(np.float64)
        order = np.lexsort((np.arange(N), -row))[:k]
        np.testing.assert_array_equal(ti16[0, 0, r].cpu().numpy(), order)
    del sc16
    # top-k is exactly the k best of the returned scores (value desc, index asc)
    for r in range(0, Nq, 97):
        row = sc[0, 0, r].cpu().numpy().astype(np.float64)
        order = np.lexsort((np.arange(N), -row))[:k]
        np.testing.assert_array_equal(ti[0, 0, r].cpu().numpy(), order)
        np.testing.assert_array_equal(tv[0, 0, r].cpu().numpy(), row[order].astype(np.float32))


def test_workload5_topk_against_oracle(tq):
    """The vector-search launches (1M packed keys, d=1024, 4-bit, 1024 query rows, top-10 fused into
    the search kernel; tq_scores and the fp16-operand tq_search) against the oracle's exact top-10
    over the whole database, for 8 of the query rows.  Both sides score the same packed records, seeded random code and sign words with
    unit key norms and residual norms of the 3-bit stage's size, so no oracle input comes from the
    GPU; the compression of real inputs is checked on sampled rows above."""
    import torch
    d, m, bits, N, Nq, k = 1024, 512, 4, 1_000_000, 1024, 10
    s = synth.seeds(5)
    R = synth.rotation(d, s["R"])
    S = synth.gaussian(m, d, s["S"])
    rec = synth.random_packed_keys(N, d, bits - 1, m, s["keys"] + 100)
    Q = synth.unit_rows(Nq, d, s["queries"] + 100)
    p = tq.Params(d, bits, m, torch.from_numpy(R).cuda(), torch.from_numpy(S).cuda())
    keys = (torch.from_numpy(rec["codes"].view(np.int32)).cuda(), torch.from_numpy(rec["signs"].view(np.int32)).cuda(),
            torch.from_numpy(rec["norm"].view(np.float16)).cuda(),
            torch.from_numpy(rec["rnorm"].view(np.float16)).cuda())
    qd = torch.from_numpy(Q.reshape(1, 1, Nq, d)).cuda()
    got = {}
    for fn in (tq.tq_scores, tq.tq_search):
        _, ti, tv = fn(p, qd, keys, 1, N, want_scores=False, topk=k)
        torch.cuda.synchronize()
        got[fn.__name__] = (ti.cpu().numpy()[0, 0], tv.cpu().numpy()[0, 0])
    rows = np.arange(0, Nq, Nq // 8)
    ora = oracle.scores(Q[rows].reshape(1, 1, len(rows), d), R, S, bits, 1, 1, 1, len(rows), N, rec["codes"],
                        rec["signs"], rec["norm"], rec["rnorm"])[0, 0]
    oi, ov = oracle.topk(ora, k)
    for name, (ti, tv) in got.items():
        for j, r in enumerate(rows):
            check_topk(ti[r], tv[r], ora[j], k, f"{name} row {r}")
            # where no near-tie straddles the k-th place, the sets are equal
            if ov[j, k - 1] - np.sort(ora[j])[::-1][k] > 2 * (1e-4 + 1e-3 * abs(ov[j, k - 1])):
                assert set(ti[r].tolist()) == set(oi[j].tolist()), f"{name} row {r}: top-{k} sets differ"
