"""tq_attend_static, the attention call for callers that cannot allocate device memory at call
time (a serving loop whose memory is all in its own pool, or code that must not pay the device
synchronisation of cudaMalloc / cudaFree inside a decode step): it takes its scratch from a
library-owned array instead of from the caller.  Checked through the C ABI against tq_attend
(which takes caller scratch) on two calls in a row, with different problems, so that the second
call runs on top of whatever the first left in the shared array.  This file is collected last."""
import numpy as np
import pytest

from kv_cache_vector_compress_b200 import synth

from .parity import check_close

pytestmark = pytest.mark.gpu


def _problem(tq, seed, d, bits, B, Hq, Hkv, T):
    import torch
    m = d // 2
    p = tq.Params(d, bits, m, torch.from_numpy(synth.rotation(d, seed)).cuda(),
                  torch.from_numpy(synth.gaussian(m, d, seed + 1)).cuda())
    n = B * Hkv * T
    K = synth.torch_normal_f16((n, d), seed + 2)
    V = synth.torch_normal_f16((n, d), seed + 3)
    Q = synth.torch_normal_f32((B, Hq, 1, d), seed + 4)
    keys = tq.tq_compress_keys(p, K)
    vals = tq.tq_compress_values(p, V)
    return p, Q, keys, vals


def test_attend_static_matches_attend_on_two_calls():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from kv_cache_vector_compress_b200 import tq
    cases = [dict(seed=11, d=128, bits=3, B=4, Hq=32, Hkv=8, T=4096),
             dict(seed=23, d=256, bits=2, B=2, Hq=16, Hkv=4, T=3000)]
    for c in cases:
        p, Q, keys, vals = _problem(tq, c["seed"], c["d"], c["bits"], c["B"], c["Hq"], c["Hkv"], c["T"])
        need = tq.tq_attend_scratch_bytes(p, c["B"], c["Hq"], c["Hkv"], 1, c["T"])
        assert 0 < need <= tq.TQ_STATIC_SCRATCH_BYTES
        ref = tq.tq_attend(p, Q, keys, vals, c["Hkv"], c["T"])
        out = torch.full_like(ref, float("nan"))
        tq.tq_attend_static(p, Q, keys, vals, c["Hkv"], c["T"], out=out)
        torch.cuda.synchronize()
        check_close(out, ref.double().cpu().numpy(), "tq_attend_static vs tq_attend")


def test_attend_static_rejects_oversized_problems():
    import torch
    from kv_cache_vector_compress_b200 import tq
    p, Q, keys, vals = _problem(tq, 5, 128, 3, 1, 4, 1, 64)
    # a problem whose scratch would not fit the fixed array is refused before any work
    B, Hq, Hkv, T = 64, 256, 64, 1 << 16
    assert tq.tq_attend_scratch_bytes(p, B, Hq, Hkv, 1, T) > tq.TQ_STATIC_SCRATCH_BYTES
    q = torch.empty((B, Hq, 1, 128), dtype=torch.float32, device="cuda")
    with pytest.raises(tq.TQError) as e:
        tq.tq_attend_static(p, q, keys, vals, Hkv, T)
    assert e.value.status == tq.TQ_ERR_UNSUPPORTED
