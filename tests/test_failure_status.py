"""Device-side failure detection without a GPU fault: a bounded wait that nothing completes
must run out, record TQ_ERR_TIMEOUT in dev_status and return, after which the same context
keeps working (a normal compression right after gives the oracle's codes)."""
import time

import numpy as np
import pytest

import oracle
from kv_cache_vector_compress_b200 import synth

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    import torch
    from kv_cache_vector_compress_b200 import tq
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    t0 = time.perf_counter()
    tq.tq_selftest_wait_timeout(status, 200)
    torch.cuda.synchronize()
    waited = time.perf_counter() - t0
    assert int(status.item()) == tq.TQ_ERR_TIMEOUT
    assert 0.15 < waited < 5.0
    # the context is still usable: a compression after the timeout matches the oracle
    d, m, bits = 128, 64, 3
    R = synth.rotation(d, 41)
    S = synth.gaussian(m, d, 42)
    x = synth.gaussian(256, d, 43).astype(np.float16)
    p = tq.Params(d, bits, m, torch.from_numpy(R).cuda(), torch.from_numpy(S).cuda())
    fresh = torch.zeros(1, dtype=torch.int32, device="cuda")
    codes, signs, norm, rnorm = tq.tq_compress_keys(p, torch.from_numpy(x).cuda(), dev_status=fresh)
    torch.cuda.synchronize()
    assert int(fresh.item()) == 0
    ora = oracle.compress(x, R, S, bits, is_key=True)
    same = (codes.cpu().numpy().view(np.uint32) == ora["codes"]).mean()
    assert same > 0.999


def test_selftest_rejects_bad_arguments():
    import torch
    from kv_cache_vector_compress_b200 import tq
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(tq.TQError):
        tq.tq_selftest_wait_timeout(status, 0)
    with pytest.raises(tq.TQError):
        tq.tq_selftest_wait_timeout(status, 20000)
