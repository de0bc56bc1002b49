"""Attention quality of a compressed cache against exact attention on the same inputs.

The measurement the pages describe for validating compression ("turboquant-pytorch",
nav.superapi.store, 常见使用模式 and the quality table of 算法细节): the cosine similarity between
the exact attention distribution and the one estimated from the compressed keys, and how often
both put their largest weight on the same token (top-1 match).  The attention output (the
softmax-weighted values) is compared the same way.  The estimated scores and outputs come from
the library's kernels; the exact side is plain fp32 PyTorch on the uncompressed cache."""
import math

import torch

from . import tq


def distribution_metrics(est_scores: torch.Tensor, exact_scores: torch.Tensor, scale: float):
    """Per query row (last axis = tokens): cosine similarity of softmax(scale * est) and
    softmax(scale * exact), and whether their argmax agrees.  Returns (cosine, top1) tensors."""
    pe = torch.softmax(scale * est_scores.double(), dim=-1)
    px = torch.softmax(scale * exact_scores.double(), dim=-1)
    cos = torch.nn.functional.cosine_similarity(pe, px, dim=-1)
    top1 = (pe.argmax(dim=-1) == px.argmax(dim=-1)).double()
    return cos, top1


def exact_attention(q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, scale: float):
    """q [B, Hq, Nq, d]; K, V [B, Hkv, T, d] (grouped query heads share a KV head).
    Returns (scores [B, Hq, Nq, T], out [B, Hq, Nq, d]) in fp32."""
    B, Hq, Nq, d = q.shape
    Hkv = K.shape[1]
    G = Hq // Hkv
    Kf = K.float().repeat_interleave(G, dim=1)
    Vf = V.float().repeat_interleave(G, dim=1)
    s = torch.matmul(q.float(), Kf.transpose(-1, -2))
    out = torch.matmul(torch.softmax(scale * s, dim=-1), Vf)
    return s, out


def score_quality(p, q: torch.Tensor, K: torch.Tensor, keys, scale: float = 0.0):
    """score_cosine and top1 of the compressed keys alone (no values)."""
    B, Hq, Nq, d = q.shape
    Hkv, T = K.shape[1], K.shape[2]
    scale = scale if scale > 0 else 1.0 / math.sqrt(d)
    est, _, _ = tq.tq_scores(p, q, keys, Hkv, T)
    Kf = K.float().repeat_interleave(Hq // Hkv, dim=1)
    cos, top1 = distribution_metrics(est, torch.matmul(q.float(), Kf.transpose(-1, -2)), scale)
    return {"score_cosine": cos.mean().item(), "top1": top1.mean().item()}


def mse_only_keys(p_scorer, codes: torch.Tensor, norm: torch.Tensor):
    """Keys compressed with b MSE bits and no QJL stage (tq_compress_values with b bits), as a key
    cache for a scorer whose key codebook has the same b bits (parameters of b + 1 bits): a zero
    residual norm removes the QJL term, leaving the MSE-only estimate ||k|| <R q, c[idx]>."""
    n = norm.numel()
    signs = torch.zeros((n, p_scorer.proj_dim // 32), dtype=torch.int32, device=codes.device)
    rnorm = torch.zeros(n, dtype=torch.float16, device=codes.device)
    return codes, signs, norm, rnorm


def attention_quality(p, q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, keys, values, scale: float = 0.0):
    """Quality of the compressed cache (keys, values: the outputs of tq_compress_keys /
    tq_compress_values of K and V viewed as [B * Hkv * T, d]) for the queries q.  Returns a dict
    of means over query rows: score_cosine, top1, out_cosine."""
    B, Hq, Nq, d = q.shape
    Hkv, T = K.shape[1], K.shape[2]
    scale = scale if scale > 0 else 1.0 / math.sqrt(d)
    est, _, _ = tq.tq_scores(p, q, keys, Hkv, T)
    out = tq.tq_attend(p, q, keys, values, Hkv, T, scale=scale)
    ex_s, ex_out = exact_attention(q, K, V, scale)
    cos, top1 = distribution_metrics(est, ex_s, scale)
    ocos = torch.nn.functional.cosine_similarity(out.double(), ex_out.double(), dim=-1)
    return {"score_cosine": cos.mean().item(), "top1": top1.mean().item(), "out_cosine": ocos.mean().item()}
