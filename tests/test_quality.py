"""Attention-quality measurement (the pages' validation of compression quality: cosine similarity
of exact and estimated attention distributions and top-1 match, "turboquant-pytorch",
nav.superapi.store, 常见使用模式 / 算法细节), on synthetic inputs."""
import math

import numpy as np
import pytest

import oracle
from kv_cache_vector_compress_b200 import synth


def test_distribution_metrics_hand_case():
    import torch
    from kv_cache_vector_compress_b200.quality import distribution_metrics
    # identical distributions
    s = torch.tensor([[0.3, -1.0, 2.0, 0.5]])
    cos, top1 = distribution_metrics(s, s.clone(), 1.0)
    assert abs(cos.item() - 1.0) < 1e-12 and top1.item() == 1.0
    # softmax([0, 0]) = (1/2, 1/2) against softmax([0, ln 3]) = (1/4, 3/4):
    # cosine = (1/8 + 3/8) / (sqrt(1/2) sqrt(10/16)) = 2 / sqrt(5); argmax 0 (first of a tie) vs 1
    cos, top1 = distribution_metrics(torch.tensor([[0.0, 0.0]], dtype=torch.float64),
                                     torch.tensor([[0.0, math.log(3.0) / 0.5]], dtype=torch.float64), 0.5)
    assert abs(cos.item() - 2.0 / math.sqrt(5.0)) < 1e-12
    assert top1.item() == 0.0


@pytest.mark.gpu
def test_quality_against_oracle():
    """The GPU measurement on a cache compressed by the oracle equals the same measurement made
    from the oracle's scores and attention, and improves with the bit width."""
    import torch
    from kv_cache_vector_compress_b200 import quality, tq
    d, m, B, Hkv, G, T = 128, 64, 1, 2, 4, 512
    Hq = Hkv * G
    R, S = synth.rotation(d, 711), synth.gaussian(m, d, 712)
    sc = np.exp(np.random.Generator(np.random.PCG64(713)).standard_normal((B, Hkv, 1, d))).astype(np.float32)
    K = (synth.gaussian(B * Hkv * T, d, 714).reshape(B, Hkv, T, d) * sc).astype(np.float16)
    V = synth.gaussian(B * Hkv * T, d, 715).reshape(B, Hkv, T, d).astype(np.float16)
    Q = (synth.gaussian(B * Hq, d, 716).reshape(B, Hkv, G, d) * sc).reshape(B, Hq, 1, d).astype(np.float32)
    scale = 1.0 / math.sqrt(d)
    # exact side in float64 numpy
    Kd, Vd = K.astype(np.float64).repeat(G, axis=1), V.astype(np.float64).repeat(G, axis=1)
    ex_s = np.einsum("bhnd,bhtd->bhnt", Q.astype(np.float64), Kd)
    ex_p = np.exp(scale * ex_s - (scale * ex_s).max(-1, keepdims=True))
    ex_p /= ex_p.sum(-1, keepdims=True)
    ex_o = np.einsum("bhnt,bhtd->bhnd", ex_p, Vd)
    got = {}
    for bits in (2, 3, 4):
        k = oracle.compress(K.reshape(-1, d), R, S, bits, is_key=True)
        v = oracle.compress(V.reshape(-1, d), R, None, bits, is_key=False)
        o_s = oracle.scores(Q, R, S, bits, B, Hq, Hkv, 1, T, k["codes"], k["signs"], k["norm"], k["rnorm"])
        o_o = oracle.attend(Q, R, S, bits, B, Hq, Hkv, 1, T, k["codes"], k["signs"], k["norm"], k["rnorm"],
                            v["codes"], v["norm"])
        o_p = np.exp(scale * o_s - (scale * o_s).max(-1, keepdims=True))
        o_p /= o_p.sum(-1, keepdims=True)
        cos = (o_p * ex_p).sum(-1) / np.linalg.norm(o_p, axis=-1) / np.linalg.norm(ex_p, axis=-1)
        top1 = (o_p.argmax(-1) == ex_p.argmax(-1)).mean()
        ocos = (o_o * ex_o).sum(-1) / np.linalg.norm(o_o, axis=-1) / np.linalg.norm(ex_o, axis=-1)
        p = tq.Params(d, bits, m, torch.from_numpy(R).cuda(), torch.from_numpy(S).cuda())
        kk = (torch.from_numpy(k["codes"].view(np.int32)).cuda(), torch.from_numpy(k["signs"].view(np.int32)).cuda(),
              torch.from_numpy(k["norm"].view(np.float16)).cuda(), torch.from_numpy(k["rnorm"].view(np.float16)).cuda())
        vv = (torch.from_numpy(v["codes"].view(np.int32)).cuda(), torch.from_numpy(v["norm"].view(np.float16)).cuda())
        g = quality.attention_quality(p, torch.from_numpy(Q).cuda(), torch.from_numpy(K).cuda(),
                                      torch.from_numpy(V).cuda(), kk, vv)
        assert abs(g["score_cosine"] - cos.mean()) < 1e-5, (bits, g, cos.mean())
        assert abs(g["top1"] - top1) <= 1.0 / (B * Hq) + 1e-12, (bits, g, top1)
        assert abs(g["out_cosine"] - ocos.mean()) < 1e-5, (bits, g, ocos.mean())
        got[bits] = g
    assert got[2]["score_cosine"] < got[3]["score_cosine"] < got[4]["score_cosine"]
    assert got[2]["out_cosine"] < got[3]["out_cosine"] < got[4]["out_cosine"]


@pytest.mark.gpu
def test_mse_only_keys_scores_match_dequantized_dot():
    """MSE-only keys scored through tq_scores (zero residual norm, key codebook of the same bits)
    equal q . dequantize(key) from the oracle, and differ from the two-stage estimate."""
    import torch
    from kv_cache_vector_compress_b200 import quality, tq
    d, m, T, Hq = 128, 64, 700, 3
    R, S = synth.rotation(d, 721), synth.gaussian(m, d, 722)
    K = synth.gaussian(T, d, 723).astype(np.float16)
    Q = synth.gaussian(Hq, d, 724).reshape(1, Hq, 1, d)
    for b in (2, 3):
        v = oracle.compress(K, R, None, b, is_key=False)
        ref = Q.reshape(Hq, d).astype(np.float64) @ oracle.dequantize(v["codes"], v["norm"], R, b).T
        ps = tq.Params(d, b + 1, m, torch.from_numpy(R).cuda(), torch.from_numpy(S).cuda())
        codes = torch.from_numpy(v["codes"].view(np.int32)).cuda()
        norm = torch.from_numpy(v["norm"].view(np.float16)).cuda()
        s, _, _ = tq.tq_scores(ps, torch.from_numpy(Q).cuda(), quality.mse_only_keys(ps, codes, norm), 1, T)
        torch.cuda.synchronize()
        from .parity import check_close
        check_close(s[0, :, 0], ref, f"MSE-only scores, {b} bits")
