"""Seeded synthetic inputs for the five workloads.

This module generates inputs only: random matrices, random vectors and the scaling
recipes of each workload.  It holds none of the compression method's arithmetic and
is shared by the tests, the benchmark and the smoke check (both the CUDA path and the
CPU oracle consume what it produces).

Seeds: base s0 = 20260000 + workload number; streams R = s0+1, S = s0+2, keys = s0+3,
values = s0+4, queries = s0+5, channel scales / outlier channels = s0+6.

Host generation uses numpy's PCG64; device generation (for the large workloads, where
host generation would take minutes) uses torch's CUDA generator.  The two give different
numbers; each parity check uses one of them for both sides.
"""
from __future__ import annotations

import numpy as np

SEED_BASE = 20260000


def seeds(workload: int) -> dict:
    s0 = SEED_BASE + workload
    return {"R": s0 + 1, "S": s0 + 2, "keys": s0 + 3, "values": s0 + 4, "queries": s0 + 5,
            "scales": s0 + 6}


def rotation(d: int, seed: int) -> np.ndarray:
    """Haar-distributed orthogonal matrix: QR of a seeded Gaussian d x d matrix with the
    signs of R's diagonal folded into Q.  Returned as fp32 [d, d]."""
    rng = np.random.Generator(np.random.PCG64(seed))
    g = rng.standard_normal((d, d))
    q, r = np.linalg.qr(g)
    q = q * np.sign(np.diag(r))[None, :]
    return np.ascontiguousarray(q.astype(np.float32))


def gaussian(rows: int, cols: int, seed: int, dtype=np.float32) -> np.ndarray:
    rng = np.random.Generator(np.random.PCG64(seed))
    return np.ascontiguousarray(rng.standard_normal((rows, cols)).astype(dtype))


def unit_rows(rows: int, cols: int, seed: int) -> np.ndarray:
    """i.i.d. N(0,1) rows scaled to unit length (fp32)."""
    x = np.random.Generator(np.random.PCG64(seed)).standard_normal((rows, cols))
    x /= np.linalg.norm(x, axis=1, keepdims=True)
    return np.ascontiguousarray(x.astype(np.float32))


# --------------------------------------------------------------------- workloads

WORKLOADS = {
    1: dict(name="single-head d128 3-bit (4096 K + 4096 V fp32 unit, 16 queries)",
            dim=128, bits=3, proj_dim=64, B=1, Hq=1, Hkv=1, Nq=16, T=4096, dtype="f32"),
    2: dict(name="Qwen2.5-3B-shaped prefill compress (36 layers x 2 KV heads x 8192 x 128 fp16)",
            dim=128, bits=3, proj_dim=64, layers=36, Hkv=2, T=8192, dtype="f16", bits_sweep=(2, 3, 4)),
    3: dict(name="decode attention B32 Hq32/Hkv8 T32768 d128 3-bit",
            dim=128, bits=3, proj_dim=64, B=32, Hq=32, Hkv=8, Nq=1, T=32768, dtype="f16"),
    4: dict(name="wide-head decode B8 Hq16/Hkv4 T65536 d256",
            dim=256, bits=4, proj_dim=128, B=8, Hq=16, Hkv=4, Nq=1, T=65536, dtype="f16",
            bits_sweep=(2, 4)),
    5: dict(name="vector search 1M x d1024 4-bit Prod, 1024 queries, top-10",
            dim=1024, bits=4, proj_dim=512, N=1_000_000, Nq=1024, topk=10, dtype="f32"),
}


def workload1(scale_T: int | None = None):
    """Workload 1: one head, d=128, 4096 keys and values (fp32, N(0,1) then unit length),
    16 queries N(0,1); R = QR of a seeded Gaussian 128x128; S seeded Gaussian 64x128."""
    w = WORKLOADS[1]
    s = seeds(1)
    d, m, T = w["dim"], w["proj_dim"], scale_T or w["T"]
    return dict(R=rotation(d, s["R"]), S=gaussian(m, d, s["S"]),
                K=unit_rows(T, d, s["keys"]), V=unit_rows(T, d, s["values"]),
                Q=gaussian(w["Nq"], d, s["queries"]).reshape(1, 1, w["Nq"], d))


def channel_scaled_f16(rows: int, d: int, seed: int, scale_seed: int, groups: int) -> np.ndarray:
    """N(0,1) rows times per-(group, channel) lognormal(0,1) scales (outlier channels),
    as fp16: rows are split evenly into `groups` (layer, head) blocks."""
    rng = np.random.Generator(np.random.PCG64(seed))
    srng = np.random.Generator(np.random.PCG64(scale_seed))
    sc = np.exp(srng.standard_normal((groups, d)))
    x = rng.standard_normal((rows, d)).reshape(groups, rows // groups, d) * sc[:, None, :]
    return np.ascontiguousarray(x.reshape(rows, d).astype(np.float16))


def outlier_channels(d: int, seed: int, frac: float = 0.01) -> np.ndarray:
    """Indices of round(frac*d) channels (at least 1) that are scaled x20 in workload 4."""
    k = max(1, int(round(frac * d)))
    rng = np.random.Generator(np.random.PCG64(seed))
    return np.sort(rng.choice(d, size=k, replace=False))


# ------------------------------------------------------------ device generation

def torch_normal_f16(shape, seed: int, device="cuda", chunk_rows: int = 1 << 20):
    """N(0,1) fp16 tensor generated on the device in chunks (bounded temporary memory)."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    out = torch.empty(shape, dtype=torch.float16, device=device)
    flat = out.view(-1, shape[-1])
    for r0 in range(0, flat.shape[0], chunk_rows):
        r1 = min(flat.shape[0], r0 + chunk_rows)
        flat[r0:r1] = torch.randn((r1 - r0, shape[-1]), generator=g, device=device,
                                  dtype=torch.float32).half()
    return out


def torch_normal_f32(shape, seed: int, device="cuda"):
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32)


def random_packed_keys(n: int, d: int, beta: int, m: int, seed: int, rho=(0.17, 0.20)):
    """Seeded packed key records without a compression step: uniformly random code and sign
    words, key norms 1 (fp16 1.0, unit keys) and residual norms uniform in `rho` (fp16), in the
    layout of the library's key arrays.  Used to check scoring and top-k at full size where
    compressing the inputs on the host would take too long."""
    rng = np.random.Generator(np.random.PCG64(seed))
    codes = rng.integers(0, 1 << 32, size=(n, beta * d // 32), dtype=np.uint64).astype(np.uint32)
    signs = rng.integers(0, 1 << 32, size=(n, m // 32), dtype=np.uint64).astype(np.uint32)
    norm = np.full(n, 0x3C00, np.uint16)
    rnorm = rng.uniform(rho[0], rho[1], size=n).astype(np.float16).view(np.uint16)
    return {"codes": codes, "signs": signs, "norm": norm, "rnorm": rnorm}
