"""The N > 1 path's host logic on CPU: two gloo ranks, each compressing and attending its own
(batch, KV-head) slice with the oracle as the stand-in compute, then the max-over-ranks timing
reduction and the whole-job throughput the benchmark reports."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from kv_cache_vector_compress_b200 import dist as tqdist


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import time

    import oracle
    from kv_cache_vector_compress_b200 import synth
    ri = tqdist.init("gloo", timeout_s=60)
    assert (ri.rank, ri.world) == (rank, world)
    d, m, bits, T, G = 64, 32, 3, 256, 2
    off = tqdist.seed_offset(rank)
    R = synth.rotation(d, 1)
    S = synth.gaussian(m, d, 2)
    K = synth.gaussian(T, d, 3 + off).astype(np.float16)
    V = synth.gaussian(T, d, 4 + off).astype(np.float16)
    q = synth.gaussian(G, d, 5 + off).reshape(1, G, 1, d)
    tqdist.barrier()
    t0 = time.perf_counter()
    k = oracle.compress(K, R, S, bits, is_key=True)
    v = oracle.compress(V, R, None, bits, is_key=False)
    o = oracle.attend(q, R, S, bits, 1, G, 1, 1, T, k["codes"], k["signs"], k["norm"], k["rnorm"],
                      v["codes"], v["norm"])
    elapsed = time.perf_counter() - t0 + 0.05 * rank  # make the ranks' times differ
    tqdist.barrier()
    mx = tqdist.max_over_ranks(elapsed)
    out_q.put((rank, elapsed, mx, float(np.abs(o).sum()), tqdist.weak_scaling_value(T, world, mx)))
    tqdist.destroy()


def test_two_gloo_ranks_time_as_max_and_work_independently():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    times = [r[1] for r in res]
    for r in res:
        assert r[2] == pytest.approx(max(times))            # every rank sees the max
        assert r[4] == pytest.approx(world * 256 / max(times))  # whole-job weak-scaling value
    assert res[0][3] != res[1][3]  # different seeds: the ranks did their own work


@pytest.mark.parametrize("n,world", [(10, 2), (7, 3), (256, 8), (1, 4), (0, 2)])
def test_shards_cover_every_unit_once(n, world):
    seen = []
    for r in range(world):
        s, c = tqdist.shard(n, world, r)
        seen.extend(range(s, s + c))
    assert seen == list(range(n))


def test_single_rank_is_identity():
    assert tqdist.max_over_ranks(3.5) == 3.5
    assert tqdist.rank_info().world >= 1


def _topk_worker(rank, world, port, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import torch
    tqdist.init("gloo", timeout_s=60)
    nq, n, k = 5, 1003, 10
    g = np.random.Generator(np.random.PCG64(77))
    full = np.round(g.standard_normal((nq, n)), 1).astype(np.float32)  # many exact ties
    start, cnt = tqdist.shard(n, world, rank)
    local = torch.from_numpy(full[:, start:start + cnt])
    # the shard's own top-k, as the search kernel returns it (local indices)
    li, lv = tqdist.merge_topk(local, torch.arange(cnt, dtype=torch.int64).expand(nq, cnt), k)
    gi, gv = tqdist.sharded_topk(li, lv, k, start)
    out_q.put((rank, gi.numpy(), gv.numpy(), full))
    tqdist.destroy()


def test_sharded_topk_over_two_gloo_ranks():
    """A database split over two ranks: the merged per-rank top-k lists equal the top-k of the whole
    database (score descending, ties to the smaller index), on every rank."""
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_topk_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    full = res[0][3]
    k = 10
    for r in range(full.shape[0]):
        order = np.lexsort((np.arange(full.shape[1]), -full[r]))[:k]
        for _, gi, gv, _ in res:
            assert np.array_equal(gi[r], order), (r, gi[r], order)
            assert np.array_equal(gv[r], full[r, order])



def _piece_partial(q, R, S, bits, k, v, T0, T1, T, scale):
    """(max, sum, rotated weighted value sum) of tokens [T0, T1) of a one-slice cache, from the
    oracle's scores and dequantized values (numpy), per query row."""
    import oracle
    d = R.shape[0]
    G = q.shape[1]
    sc = oracle.scores(q, R, S, bits, 1, G, 1, 1, T, k["codes"], k["signs"], k["norm"], k["rnorm"])[0, :, 0]
    vh = oracle.dequantize(v["codes"], v["norm"], R, bits)  # original space, norm included
    z = scale * sc[:, T0:T1]
    M = z.max(axis=1)
    w = np.exp(z - M[:, None])
    o = w @ vh[T0:T1] @ R.astype(np.float64).T  # rotated: R o
    return np.concatenate([M[:, None], w.sum(axis=1)[:, None], o], axis=1)


def _context_worker(rank, world, port, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import oracle
    import torch
    from kv_cache_vector_compress_b200 import synth
    tqdist.init("gloo", timeout_s=60)
    d, m, bits, T, G = 64, 32, 3, 301, 4
    R = synth.rotation(d, 61)
    S = synth.gaussian(m, d, 62)
    K = synth.gaussian(T, d, 63).astype(np.float16)
    V = synth.gaussian(T, d, 64).astype(np.float16)
    q = synth.gaussian(G, d, 65).reshape(1, G, 1, d)
    k = oracle.compress(K, R, S, bits, is_key=True)
    v = oracle.compress(V, R, None, bits, is_key=False)
    start, count = tqdist.context_shard(T, world, rank)
    part = _piece_partial(q, R, S, bits, k, v, start, start + count, T, 1 / np.sqrt(d))
    parts = tqdist.gather_partials(torch.from_numpy(part)).numpy()
    # the merge of the gathered pieces: log-sum-exp over ranks, then the rotation back
    M = parts[:, :, 0].max(axis=0)
    w = np.exp(parts[:, :, 0] - M[None, :])
    L = (w * parts[:, :, 1]).sum(axis=0)
    o_rot = (w[:, :, None] * parts[:, :, 2:]).sum(axis=0) / L[:, None]
    merged = o_rot @ R.astype(np.float64)  # R^T o_rot per row
    whole = oracle.attend(q, R, S, bits, 1, G, 1, 1, T, k["codes"], k["signs"], k["norm"], k["rnorm"],
                          v["codes"], v["norm"])[0, :, 0]
    out_q.put((rank, start, count, float(np.abs(merged - whole).max()), float(np.abs(whole).max())))
    tqdist.destroy()


def test_context_split_over_two_gloo_ranks():
    """One context split over two ranks (contiguous token ranges): every rank's partial is
    gathered in rank order and the merged result equals the oracle's attention over the whole
    context; the ranges tile the context."""
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_context_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res[0][1] == 0 and res[0][1] + res[0][2] == res[1][1] and res[1][1] + res[1][2] == 301
    # R is fp32, orthogonal to ~1e-7: rotating into and out of its frame costs about that much
    for _, _, _, err, scale in res:
        assert err <= 1e-6 * max(1.0, scale), err
