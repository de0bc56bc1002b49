"""tq_attend_static, the attention call for callers that cannot allocate device memory at call
time (a serving loop whose memory is all in its own pool, or code that must not pay the device
synchronisation of cudaMalloc / cudaFree inside a decode step): it takes its scratch from a
library-owned array instead of from the caller.  Checked through the C ABI on two calls in a row,
with different problems, so that the second call runs on top of whatever the first left in the
shared array: against tq_attend (which takes caller scratch) and against the oracle's attention
over the same packed records.  This file is collected last."""
import numpy as np
import pytest

import oracle
from kv_cache_vector_compress_b200 import synth

from .parity import check_close

pytestmark = pytest.mark.gpu


def _problem(tq, seed, d, bits, B, Hq, Hkv, T):
    """The oracle's packed records of seeded keys and values, on the device, with the queries."""
    import torch
    m = d // 2
    R, S = synth.rotation(d, seed), synth.gaussian(m, d, seed + 1)
    n = B * Hkv * T
    K = synth.gaussian(n, d, seed + 2).astype(np.float16)
    V = synth.gaussian(n, d, seed + 3).astype(np.float16)
    q = synth.gaussian(B * Hq, d, seed + 4).reshape(B, Hq, 1, d)
    k = oracle.compress(K, R, S, bits, is_key=True)
    v = oracle.compress(V, R, None, bits, is_key=False)
    ora = oracle.attend(q, R, S, bits, B, Hq, Hkv, 1, T, k["codes"], k["signs"], k["norm"], k["rnorm"],
                        v["codes"], v["norm"])
    p = tq.Params(d, bits, m, torch.from_numpy(R).cuda(), torch.from_numpy(S).cuda())
    dev = lambda a, t: torch.from_numpy(np.ascontiguousarray(a).view(t)).cuda()
    keys = (dev(k["codes"], np.int32), dev(k["signs"], np.int32), dev(k["norm"], np.float16),
            dev(k["rnorm"], np.float16))
    vals = (dev(v["codes"], np.int32), dev(v["norm"], np.float16))
    return p, torch.from_numpy(q).cuda(), keys, vals, ora


def test_attend_static_matches_attend_and_oracle_on_two_calls():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from kv_cache_vector_compress_b200 import tq
    cases = [dict(seed=11, d=128, bits=3, B=4, Hq=32, Hkv=8, T=4096),
             dict(seed=23, d=256, bits=2, B=2, Hq=16, Hkv=4, T=3000)]
    for c in cases:
        p, Q, keys, vals, ora = _problem(tq, c["seed"], c["d"], c["bits"], c["B"], c["Hq"], c["Hkv"], c["T"])
        need = tq.tq_attend_scratch_bytes(p, c["B"], c["Hq"], c["Hkv"], 1, c["T"])
        assert 0 < need <= tq.TQ_STATIC_SCRATCH_BYTES
        ref = tq.tq_attend(p, Q, keys, vals, c["Hkv"], c["T"])
        out = torch.full_like(ref, float("nan"))
        tq.tq_attend_static(p, Q, keys, vals, c["Hkv"], c["T"], out=out)
        torch.cuda.synchronize()
        check_close(out, ref.double().cpu().numpy(), "tq_attend_static vs tq_attend")
        check_close(out, ora, "tq_attend_static vs the oracle")


def test_attend_static_rejects_oversized_problems():
    import torch
    from kv_cache_vector_compress_b200 import tq
    p, Q, keys, vals, _ = _problem(tq, 5, 128, 3, 1, 4, 1, 64)
    # a problem whose scratch would not fit the fixed array is refused before any work
    B, Hq, Hkv, T = 64, 256, 64, 1 << 16
    assert tq.tq_attend_scratch_bytes(p, B, Hq, Hkv, 1, T) > tq.TQ_STATIC_SCRATCH_BYTES
    q = torch.empty((B, Hq, 1, 128), dtype=torch.float32, device="cuda")
    with pytest.raises(tq.TQError) as e:
        tq.tq_attend_static(p, q, keys, vals, Hkv, T)
    assert e.value.status == tq.TQ_ERR_UNSUPPORTED
