"""Pins of the CPU oracle to facts other than itself (no GPU needed).

Each test ties one oracle function to what the pages print, to a closed form, to a
textbook table, to an independent library routine or to brute force, chosen so that a
plausible slip (dropped term, wrong sign or index, transposed operand) fails one of them.
"""
import math
import os

import numpy as np
import pytest
from scipy import integrate, special, stats

import oracle
from kv_cache_vector_compress_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            rows.append(line.split())
    return rows


# ------------------------------------------------------------------ codebook

@pytest.mark.parametrize("d", [1, 32, 128, 256, 1024])
def test_one_bit_codebook_closed_form(d):
    # 1-bit Lloyd-Max for N(0, 1/d): centroids +-E|Z|/sqrt(d) = +-sqrt(2/(pi d)), boundary 0
    b, c, _ = oracle.codebook(d, 1)
    assert b[0] == 0.0
    np.testing.assert_allclose(c, [-math.sqrt(2 / (math.pi * d)), math.sqrt(2 / (math.pi * d))],
                               rtol=1e-13)


def test_codebook_matches_max_1960_table():
    rows = _read_golden("lloyd_max_gaussian_max1960.txt")
    seen = 0
    for bits, kind, *vals in rows:
        bits = int(bits)
        vals = np.array([float(v) for v in vals])
        b, c, _ = oracle.codebook(1, bits)
        K = 1 << bits
        if kind == "level":
            got = c[K // 2:]
        elif kind == "threshold":
            got = b[K // 2:]
        else:
            # distortion of the oracle's codebook, integrated independently
            got = np.array([_gauss_distortion(b, c, 1.0)])
        # the table prints 4 significant digits
        np.testing.assert_allclose(got, vals, rtol=6e-4, atol=6e-5)
        seen += 1
    assert seen == 11


def _gauss_distortion(b, c, sigma):
    edges = np.concatenate([[-np.inf], b, [np.inf]])
    tot = 0.0
    for k in range(len(c)):
        f = lambda y, ck=c[k]: (y - ck) ** 2 * stats.norm.pdf(y, scale=sigma)
        tot += integrate.quad(f, edges[k], edges[k + 1], epsabs=1e-14, epsrel=1e-12)[0]
    return tot


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
@pytest.mark.parametrize("d", [64, 128])
def test_codebook_is_lloyd_fixed_point_by_quadrature(bits, d):
    # each centroid is the conditional mean of its cell under N(0,1/d) (computed here by
    # numerical quadrature, not the closed form the oracle uses); boundaries are midpoints
    b, c, _ = oracle.codebook(d, bits)
    s = 1 / math.sqrt(d)
    edges = np.concatenate([[-np.inf], b, [np.inf]])
    for k in range(len(c)):
        num = integrate.quad(lambda y: y * stats.norm.pdf(y, scale=s), edges[k], edges[k + 1],
                             epsabs=1e-15, epsrel=1e-13)[0]
        den = integrate.quad(lambda y: stats.norm.pdf(y, scale=s), edges[k], edges[k + 1],
                             epsabs=1e-15, epsrel=1e-13)[0]
        assert abs(num / den - c[k]) < 1e-9 * max(1.0, abs(c[k]) * math.sqrt(d))
    np.testing.assert_allclose(b, 0.5 * (c[1:] + c[:-1]), atol=1e-15)
    np.testing.assert_array_equal(c, -c[::-1])
    assert b[len(b) // 2] == 0.0


@pytest.mark.parametrize("bits,ratio", [(1, 1.45), (2, 1.88), (3, 2.21), (4, 2.43)])
def test_distortion_within_shannon_factor(bits, ratio):
    # "distortion within ~2.7x of Shannon's lower bound" (jansverre.net, "Hva er TurboQuant"):
    # D_b <= (sqrt(3) pi / 2) 4^-b for unit vectors; D_b >= 4^-b (Shannon)
    b, c, _ = oracle.codebook(1, bits)
    D = _gauss_distortion(b, c, 1.0)
    assert 4.0 ** -bits <= D <= math.sqrt(3) * math.pi / 2 * 4.0 ** -bits
    assert abs(D / 4.0 ** -bits - ratio) < 0.01


# ------------------------------------------------- codebook under the exact (Beta) law
# jansverre.net, "Hva er TurboQuant, kort fortalt?": after the rotation a coordinate follows a
# concentrated Beta law; for a uniform unit vector in R^d, (y + 1) / 2 ~ Beta((d-1)/2, (d-1)/2).

@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_beta_codebook_d3_is_the_uniform_quantizer(bits):
    # d = 3: the coordinate of a uniform point on the 2-sphere is uniform on [-1, 1]
    # (Archimedes' hat-box theorem), whose Lloyd-Max quantizer is the uniform one
    K = 1 << bits
    b, c, _ = oracle.codebook_beta(3, bits)
    np.testing.assert_allclose(c, (2 * np.arange(K) + 1) / K - 1, atol=1e-12)
    np.testing.assert_allclose(b, 2 * np.arange(1, K) / K - 1, atol=1e-12)


@pytest.mark.parametrize("d", [3, 4, 32, 128, 1024])
def test_beta_codebook_one_bit_closed_form(d):
    # 1 bit: +-E|y| = +-Gamma(d/2) / (sqrt(pi) Gamma((d+1)/2)), boundary 0
    b, c, _ = oracle.codebook_beta(d, 1)
    e = math.exp(special.gammaln(d / 2) - special.gammaln((d + 1) / 2)) / math.sqrt(math.pi)
    assert b[0] == 0.0
    np.testing.assert_allclose(c, [-e, e], rtol=1e-12)


@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("d", [32, 128])
def test_beta_codebook_is_lloyd_fixed_point_under_scipy_beta(bits, d):
    # each centroid is the conditional mean of its cell under scipy's Beta((d-1)/2, (d-1)/2)
    # mapped to [-1, 1]; boundaries are midpoints; the codebook is antisymmetric
    b, c, _ = oracle.codebook_beta(d, bits)
    law = stats.beta((d - 1) / 2, (d - 1) / 2, loc=-1.0, scale=2.0)
    edges = np.concatenate([[-1.0], b, [1.0]])
    for k in range(len(c)):
        num = integrate.quad(lambda y: y * law.pdf(y), edges[k], edges[k + 1], epsabs=1e-15, epsrel=1e-13,
                             limit=200)[0]
        den = law.cdf(edges[k + 1]) - law.cdf(edges[k])
        assert abs(num / den - c[k]) < 1e-9 * max(1.0, abs(c[k]) * math.sqrt(d))
    np.testing.assert_allclose(b, 0.5 * (c[1:] + c[:-1]), atol=1e-15)
    np.testing.assert_array_equal(c, -c[::-1])


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_beta_codebook_tends_to_the_gaussian_one(bits):
    # N(0, 1/d) is the large-d limit of the law: sqrt(d) * centroids approach the standard
    # Lloyd-Max table, with a gap that shrinks roughly like 1/d
    _, g, _ = oracle.codebook(1, bits)
    gaps = []
    for d in (64, 256, 1024, 4096):
        _, c, _ = oracle.codebook_beta(d, bits)
        gaps.append(np.max(np.abs(c * math.sqrt(d) - g)))
    assert all(gaps[i + 1] < gaps[i] / 3 for i in range(3)), gaps
    assert gaps[-1] < 2e-3 * np.max(np.abs(g)), gaps


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
@pytest.mark.parametrize("d", [32, 128])
def test_beta_codebook_beats_the_gaussian_one_under_the_exact_law(bits, d):
    # optimality: under the exact law the Lloyd-Max codebook for that law has the lower
    # distortion (integrated independently with scipy); at d = 32 the gap is clearly visible
    bb, cb, _ = oracle.codebook_beta(d, bits)
    bg, cg, _ = oracle.codebook(d, bits)
    db = _beta_law_distortion(bb, cb, d)
    dg = _beta_law_distortion(bg, cg, d)
    assert db < dg, (db, dg)


def test_beta_law_compression_distortion_matches_its_integral():
    # values compressed with the Beta-law codebook: E||u - x_hat||^2 equals that codebook's
    # distortion integral under the exact law (as for the Gaussian codebook above)
    d, n, bits = 64, 3000, 2
    R = synth.rotation(d, 51)
    x = synth.gaussian(n, d, 52)
    out = oracle.compress(x, R, None, bits, is_key=False, law="beta")
    xh = oracle.dequantize(out["codes"], out["norm"], R, bits, law="beta")
    u = x.astype(np.float64) / np.linalg.norm(x.astype(np.float64), axis=1, keepdims=True)
    nrm = np.array([oracle.f16_bits_to_f64(h) for h in out["norm"]])
    err = np.sum((u - xh / nrm[:, None]) ** 2, axis=1)
    bnd, cen = oracle.codebook_f32(d, bits, law="beta")
    want = _beta_law_distortion(bnd, cen, d)
    se = err.std(ddof=1) / math.sqrt(n)
    assert abs(err.mean() - want) < 4 * se, (err.mean(), want, se)


# --------------------------------------------------------------------- fp16

def test_fp16_rounding_matches_numpy():
    rng = np.random.default_rng(1)
    vals = np.concatenate([rng.standard_normal(2000) * 10.0 ** rng.integers(-9, 5, 2000),
                           [0.0, -0.0, 65504.0, 65519.99, 65520.0, 2 ** -24, 2 ** -25, 3 * 2 ** -26,
                            6.097555e-05, 1.0 + 2 ** -11, 1.0 + 3 * 2 ** -11]])
    with np.errstate(over="ignore"):
        want = vals.astype(np.float16).view(np.uint16)
    got = np.array([oracle.f64_to_f16_bits(v) for v in vals], np.uint16)
    np.testing.assert_array_equal(got, want)
    back = np.array([oracle.f16_bits_to_f64(h) for h in want])
    np.testing.assert_array_equal(back, want.view(np.float16).astype(np.float64))


# --------------------------------------------------------------- packing

def test_pack_hand_computed_words():
    # coordinate j of a 32-group gets code j % K: plane p collects bit p of j
    for beta, words in [(1, [0xAAAAAAAA]), (2, [0xAAAAAAAA, 0xCCCCCCCC]),
                        (3, [0xAAAAAAAA, 0xCCCCCCCC, 0xF0F0F0F0]),
                        (4, [0xAAAAAAAA, 0xCCCCCCCC, 0xF0F0F0F0, 0xFF00FF00])]:
        idx = np.arange(32) % (1 << beta)
        np.testing.assert_array_equal(oracle.pack_codes(idx, 32, beta), np.array(words, np.uint32))


@pytest.mark.parametrize("beta", [1, 2, 3, 4])
@pytest.mark.parametrize("d", [32, 64, 128])
def test_pack_roundtrip(beta, d):
    rng = np.random.default_rng(beta * 1000 + d)
    for _ in range(20):
        idx = rng.integers(0, 1 << beta, d)
        w = oracle.pack_codes(idx, d, beta)
        np.testing.assert_array_equal(oracle.unpack_codes(w, d, beta), idx)
        # group g only touches words g*beta .. g*beta+beta-1
        for g in range(d // 32):
            idx2 = idx.copy()
            idx2[32 * g:32 * g + 32] = 0
            w2 = oracle.pack_codes(idx2, d, beta)
            assert np.all(w2[g * beta:(g + 1) * beta] == 0)
            others = np.ones(len(w), bool)
            others[g * beta:(g + 1) * beta] = False
            np.testing.assert_array_equal(w2[others], w[others])


# ------------------------------------------------------------ quantization

def test_generator_rotation_is_orthogonal():
    # spec: R orthogonal to 1e-6 (checked in double from the fp32 matrix)
    for d in (32, 128, 256, 1024):
        R = synth.rotation(d, 7 + d).astype(np.float64)
        assert np.abs(R.T @ R - np.eye(d)).max() <= 1e-6
        sign, logdet = np.linalg.slogdet(R)
        assert abs(sign) == 1.0 and abs(logdet) < 1e-5


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_signed_permutation_rotation_reduces_to_searchsorted(bits):
    # with R a signed permutation P, y = P u exactly, and the codes are the textbook
    # searchsorted of y against the boundaries ("left": ties go to the lower cell)
    d = 64
    rng = np.random.default_rng(bits)
    perm = rng.permutation(d)
    sgn = rng.choice([-1.0, 1.0], d)
    P = np.zeros((d, d), np.float32)
    P[np.arange(d), perm] = sgn
    x = synth.unit_rows(50, d, 99 + bits)
    out = oracle.compress(x, P, None, bits, is_key=False, want_y=True)
    bnd, _ = oracle.codebook_f32(d, bits)
    y = (x.astype(np.float64)[:, perm] * sgn[None, :]) / np.linalg.norm(x.astype(np.float64), axis=1,
                                                                           keepdims=True)
    want_idx = np.searchsorted(bnd, y.astype(np.float32), side="left")
    for v in range(50):
        np.testing.assert_array_equal(oracle.unpack_codes(out["codes"][v], d, bits), want_idx[v])
    # y = P u, not P^T u: the transposed rotation gives different codes
    yT = (x.astype(np.float64) @ P.astype(np.float64)) / np.linalg.norm(x.astype(np.float64), axis=1,
                                                                         keepdims=True)
    assert not np.array_equal(np.searchsorted(bnd, yT.astype(np.float32)), want_idx)


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_codes_are_nearest_centroid_brute_force(bits):
    # Lloyd-Max cells with midpoint boundaries are nearest-centroid cells: brute-force argmin
    d = 32
    R = synth.rotation(d, 3)
    x = synth.gaussian(200, d, 5)
    out = oracle.compress(x, R, None, bits, is_key=False, want_y=True)
    _, cen = oracle.codebook_f32(d, bits)
    y = out["y32"].astype(np.float64)
    brute = np.argmin(np.abs(y[..., None] - cen.astype(np.float64)[None, None, :]), axis=-1)
    got = np.stack([oracle.unpack_codes(out["codes"][v], d, bits) for v in range(200)])
    # away from exact midpoints the two must agree everywhere
    np.testing.assert_array_equal(got, brute)


def test_zero_vector_codes_and_norm():
    d, bits = 64, 3
    R = synth.rotation(d, 11)
    S = synth.gaussian(32, d, 12)
    x = np.zeros((2, d), np.float32)
    v = oracle.compress(x, R, None, bits, is_key=False)
    assert np.all(v["norm"] == 0)
    # y = 0 exactly; the middle boundary is 0 and ties go down: code K/2-1 = 3 = 0b011
    np.testing.assert_array_equal(v["codes"][0], np.array([0xFFFFFFFF, 0xFFFFFFFF, 0] * 2, np.uint32))
    k = oracle.compress(x, R, S, bits, is_key=True)
    assert np.all(k["norm"] == 0)
    # key MSE bits = 2: code 1 = 0b01; centroid -c0, residual = -R^T c -> nonzero rho
    np.testing.assert_array_equal(k["codes"][0], np.array([0xFFFFFFFF, 0] * 2, np.uint32))
    assert k["rnorm"][0] != 0


def _beta_law_distortion(bnd, cen, d):
    # one coordinate of a uniform unit vector in R^d has density
    # f(y) = Gamma(d/2) / (sqrt(pi) Gamma((d-1)/2)) (1 - y^2)^((d-3)/2) on [-1, 1]
    logc = special.gammaln(d / 2) - 0.5 * math.log(math.pi) - special.gammaln((d - 1) / 2)
    f = lambda y: math.exp(logc + (d - 3) / 2 * math.log1p(-y * y))
    edges = np.concatenate([[-1.0], bnd.astype(np.float64), [1.0]])
    tot = 0.0
    for k in range(len(cen)):
        tot += integrate.quad(lambda y, c=float(cen[k]): (y - c) ** 2 * f(y), edges[k], edges[k + 1],
                              epsabs=1e-16, epsrel=1e-12, limit=200)[0]
    return d * tot


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_mse_distortion_matches_exact_law_integral(bits):
    # E||u - x_hat||^2 over random unit vectors equals the codebook's distortion integral
    # under the exact coordinate law of a rotated unit vector; fails for a transposed
    # dequantization, a dropped rotation or a wrong codebook
    d, n = 128, 3000
    R = synth.rotation(d, 21)
    x = synth.gaussian(n, d, 22 + bits)
    out = oracle.compress(x, R, None, bits, is_key=False)
    xh = oracle.dequantize(out["codes"], out["norm"], R, bits)
    u = x.astype(np.float64) / np.linalg.norm(x.astype(np.float64), axis=1, keepdims=True)
    nrm = np.array([oracle.f16_bits_to_f64(h) for h in out["norm"]])
    err = np.sum((u - xh / nrm[:, None]) ** 2, axis=1)
    bnd, cen = oracle.codebook_f32(d, bits)
    want = _beta_law_distortion(bnd, cen, d)
    se = err.std(ddof=1) / math.sqrt(n)
    assert abs(err.mean() - want) < 4 * se, (err.mean(), want, se)


# ------------------------------------------------------------------- QJL

def _one_key_estimate(q, u, R, S, bits):
    k = oracle.compress(u[None, :].astype(np.float32), R, S, bits, is_key=True)
    s = oracle.scores(q.reshape(1, 1, 1, -1), R, S, bits, 1, 1, 1, 1, 1,
                      k["codes"], k["signs"], k["norm"], k["rnorm"])
    return float(s.reshape(-1)[0]), k


def test_qjl_estimate_is_unbiased_and_has_closed_form_variance():
    # "QJL residual correction -- 1-bit sign projection that makes inner product estimates
    # unbiased" (atskills.one, "What It Does"): averaged over many independent S the
    # estimate converges to <q, u>; its variance is (rho^2/m)((pi/2)||q||^2 - <q, r/rho>^2)
    d, m, bits, N = 64, 32, 2, 6000
    R = synth.rotation(d, 31)
    u = synth.unit_rows(1, d, 32)[0].astype(np.float64)
    q = synth.gaussian(1, d, 33)[0].astype(np.float64)
    rng = np.random.Generator(np.random.PCG64(34))
    est = np.empty(N)
    k0 = None
    for i in range(N):
        S = rng.standard_normal((m, d)).astype(np.float32)
        est[i], k = _one_key_estimate(q.astype(np.float32), u.astype(np.float32), R, S, bits)
        k0 = k0 or k
    # MSE part and residual, independent of S
    xh = oracle.dequantize(k0["codes"], np.array([0x3C00], np.uint16), R, bits - 1)[0]
    uu = u.astype(np.float32).astype(np.float64)
    uu /= np.linalg.norm(uu)
    r = uu - xh
    rho = np.linalg.norm(r)
    truth = float(q.astype(np.float32).astype(np.float64) @ uu)
    mse_only = float(q.astype(np.float32).astype(np.float64) @ xh)
    se = est.std(ddof=1) / math.sqrt(N)
    assert abs(est.mean() - truth) < 4 * se, (est.mean(), truth, se)
    # the MSE-only estimate is biased by <q, r>, many standard errors away
    assert abs(mse_only - truth) > 10 * se
    qq = q.astype(np.float32).astype(np.float64)
    var = rho ** 2 / m * (math.pi / 2 * qq @ qq - (qq @ r / rho) ** 2)
    assert abs(est.var(ddof=1) / var - 1.0) < 0.08, (est.var(ddof=1), var)


def test_score_scales_with_stored_key_norm():
    d, m, bits = 64, 32, 3
    R = synth.rotation(d, 41)
    S = synth.gaussian(m, d, 42)
    u = synth.unit_rows(1, d, 43)[0]
    q = synth.gaussian(1, d, 44)[0]
    s1, _ = _one_key_estimate(q, u, R, S, bits)
    s2, k2 = _one_key_estimate(q, 2.0 * u, R, S, bits)  # codes identical, norm exactly 2x
    assert k2["norm"][0] == 0x4000
    assert s2 == pytest.approx(2 * s1, rel=1e-12)


def test_large_projection_estimate_concentrates():
    # with m >> d the sign sketch term concentrates: estimate error ~ 1/sqrt(m)
    d, bits = 32, 2
    R = synth.rotation(d, 51)
    x = synth.unit_rows(40, d, 52)
    q = synth.gaussian(1, d, 53)[0]
    errs = {}
    for m in (32, 2048):
        S = synth.gaussian(m, d, 54 + m)
        k = oracle.compress(x, R, S, bits, is_key=True)
        s = oracle.scores(q.reshape(1, 1, 1, d), R, S, bits, 1, 1, 1, 1, 40,
                          k["codes"], k["signs"], k["norm"], k["rnorm"]).reshape(-1)
        errs[m] = np.sqrt(np.mean((s - x.astype(np.float64) @ q.astype(np.float64)) ** 2))
    assert errs[2048] < errs[32] / 4


# -------------------------------------------------------------- attention

def _small_cache(seed, d=64, m=32, bits=3, B=2, Hkv=2, G=2, Nq=3, T=37):
    R = synth.rotation(d, seed)
    S = synth.gaussian(m, d, seed + 1)
    K = synth.gaussian(B * Hkv * T, d, seed + 2)
    V = synth.gaussian(B * Hkv * T, d, seed + 3)
    Q = synth.gaussian(B * Hkv * G * Nq, d, seed + 4).reshape(B, Hkv * G, Nq, d)
    k = oracle.compress(K, R, S, bits, is_key=True)
    v = oracle.compress(V, R, None, bits, is_key=False)
    return dict(R=R, S=S, K=K, V=V, Q=Q, k=k, v=v, d=d, m=m, bits=bits, B=B, Hkv=Hkv, Hq=Hkv * G,
                G=G, Nq=Nq, T=T)


def test_attend_equals_softmax_weighted_dequantized_values():
    c = _small_cache(61)
    k, v = c["k"], c["v"]
    args = (c["Q"], c["R"], c["S"], c["bits"], c["B"], c["Hq"], c["Hkv"], c["Nq"], c["T"],
            k["codes"], k["signs"], k["norm"], k["rnorm"])
    sc = oracle.scores(*args)
    out = oracle.attend(*args, v["codes"], v["norm"])
    vh = oracle.dequantize(v["codes"], v["norm"], c["R"], c["bits"]).reshape(c["B"], c["Hkv"], c["T"], c["d"])
    scale = 1 / math.sqrt(c["d"])
    for b in range(c["B"]):
        for h in range(c["Hq"]):
            a = special.softmax(scale * sc[b, h], axis=-1)  # independent softmax
            np.testing.assert_allclose(out[b, h], a @ vh[b, h // c["G"]], rtol=1e-12, atol=1e-13)


def test_attend_single_token_and_uniform_scores():
    c = _small_cache(71, T=1)
    k, v = c["k"], c["v"]
    out = oracle.attend(c["Q"], c["R"], c["S"], c["bits"], c["B"], c["Hq"], c["Hkv"], c["Nq"], 1,
                        k["codes"], k["signs"], k["norm"], k["rnorm"], v["codes"], v["norm"])
    vh = oracle.dequantize(v["codes"], v["norm"], c["R"], c["bits"]).reshape(c["B"], c["Hkv"], c["d"])
    for b in range(c["B"]):
        for h in range(c["Hq"]):
            for i in range(c["Nq"]):
                np.testing.assert_allclose(out[b, h, i], vh[b, h // c["G"]], rtol=1e-13, atol=1e-15)
    # zero-norm keys give every token the same score -> plain mean of the values
    c = _small_cache(72, T=9)
    k, v = c["k"], c["v"]
    out = oracle.attend(c["Q"], c["R"], c["S"], c["bits"], c["B"], c["Hq"], c["Hkv"], c["Nq"], 9,
                        k["codes"], k["signs"], np.zeros_like(k["norm"]), k["rnorm"], v["codes"], v["norm"])
    vh = oracle.dequantize(v["codes"], v["norm"], c["R"], c["bits"]).reshape(c["B"], c["Hkv"], 9, c["d"])
    for b in range(c["B"]):
        for h in range(c["Hq"]):
            np.testing.assert_allclose(out[b, h], np.broadcast_to(vh[b, h // c["G"]].mean(0), out[b, h].shape),
                                       rtol=1e-12, atol=1e-14)


def test_gqa_head_mapping():
    # query head h reads KV head h // G: permuting the KV heads permutes head groups
    c = _small_cache(81, B=1, Hkv=2, G=2, Nq=1, T=16)
    k, v = c["k"], c["v"]
    out = oracle.attend(c["Q"], c["R"], c["S"], c["bits"], 1, 4, 2, 1, 16, k["codes"], k["signs"],
                        k["norm"], k["rnorm"], v["codes"], v["norm"])
    sw = lambda a: np.concatenate([a.reshape(2, 16, -1)[1], a.reshape(2, 16, -1)[0]]).reshape(a.shape)
    Q2 = c["Q"][:, [2, 3, 0, 1]]
    out2 = oracle.attend(Q2, c["R"], c["S"], c["bits"], 1, 4, 2, 1, 16, sw(k["codes"]), sw(k["signs"]),
                         sw(k["norm"]), sw(k["rnorm"]), sw(v["codes"]), sw(v["norm"]))
    np.testing.assert_allclose(out2[:, [2, 3, 0, 1]], out, rtol=1e-13, atol=1e-15)


def test_topk_matches_lexsort():
    rng = np.random.default_rng(91)
    s = np.round(rng.standard_normal((5, 300)), 1)  # many exact ties
    idx, val = oracle.topk(s, 10)
    for r in range(5):
        order = np.lexsort((np.arange(300), -s[r]))[:10]
        np.testing.assert_array_equal(idx[r], order)
        np.testing.assert_array_equal(val[r], s[r, order])


# ------------------------------------------------------------- size table

def test_nominal_sizes_reproduce_printed_table():
    # 289 MB fp16 -> 76 / 58 / 40 MB at 4 / 3 / 2 bits (3.8x / 5.0x / 7.3x) for Qwen2.5-3B at 8K
    rows = {int(r[0]): (float(r[1]), float(r[2])) for r in _read_golden("kv_cache_sizes.txt")}
    L, H, T, d = 36, 2, 8192, 128
    MiB = float(1 << 20)
    base = oracle.fp16_bytes(L, H, T, d)
    assert abs(base / MiB - rows[16][0]) <= 1.0  # 288.0 MiB vs the printed 289
    for bits in (4, 3, 2):
        sz = oracle.nominal_bytes(L, H, T, d, bits)
        assert math.ceil(sz / MiB) == rows[bits][0]
        assert abs(sz / MiB - rows[bits][0]) <= 1.0
        assert round(base / sz, 1) == rows[bits][1]
