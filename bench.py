"""Benchmark of the TurboQuant compression hot path on B200.

One step = the whole hot path over the decode-attention workload
(B=32, Hq=32 / Hkv=8, T=32768, head_dim 128, 3-bit: keys 2-bit MSE + 64 QJL signs,
values 3-bit MSE): compress all 8.4 M keys and 8.4 M values of the fp16 cache, then
fused scores + softmax + weighted value sum for one new query token per sequence.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl tq|reference]

Multi-GPU (torchrun): every rank compresses and attends its own batch (weak scaling,
no data-path collective); timing is the max over ranks.  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "packed keys scored/s and vectors compressed/s; % of B200 HBM roofline"
UNIT = "keys/s (each key compressed with its value, then scored and attended)"

W3 = dict(B=32, Hq=32, Hkv=8, Nq=1, T=32768, d=128, bits=3, m=64)
WORKLOAD_NAME = ("decode attention over a compressed cache: B32, Hq32/Hkv8 (GQA 4), T32768, d128, "
                 "3-bit keys (2-bit MSE + 64 QJL signs) and 3-bit values; fp16 K/V compressed, then "
                 "one query token per sequence attended")


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            j = json.load(f)
        return {"hbm_gbs": float(j["hbm_gbs"]), "bf16_tflops": float(j["bf16_tflops"]), "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "source": "fallback"}


def record_bytes(w):
    d, m, b = w["d"], w["m"], w["bits"]
    key = (b - 1) * d // 8 + m // 8 + 4
    val = b * d // 8 + 2
    return key, val


def algorithmic_bytes(w):
    n = w["B"] * w["Hkv"] * w["T"]
    key, val = record_bytes(w)
    d = w["d"]
    comp_k = n * (d * 2 + key)        # read fp16 keys, write packed keys
    comp_v = n * (d * 2 + val)
    attend = n * (key + val) + w["B"] * w["Hq"] * w["Nq"] * d * 4 * 2  # packed cache + q + out
    return {"compress_keys": comp_k, "compress_values": comp_v, "attend": attend}


# --------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        sm.sort()
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------- CPU arm

def oracle_sample(w, seed: int, T: int):
    """Oracle on one (batch, KV-head) slice of the workload: compress T keys and values and
    attend the slice's G query heads.  Returns (seconds, tokens)."""
    import numpy as np
    import oracle
    from kv_cache_vector_compress_b200 import synth
    d, m, bits, G = w["d"], w["m"], w["bits"], w["Hq"] // w["Hkv"]
    R = synth.rotation(d, seed + 1)
    S = synth.gaussian(m, d, seed + 2)
    K = synth.gaussian(T, d, seed + 3).astype(np.float16)
    V = synth.gaussian(T, d, seed + 4).astype(np.float16)
    q = synth.gaussian(G, d, seed + 5).reshape(1, G, 1, d)
    t0 = time.perf_counter()
    k = oracle.compress(K, R, S, bits, is_key=True)
    v = oracle.compress(V, R, None, bits, is_key=False)
    oracle.attend(q, R, S, bits, 1, G, 1, 1, T, k["codes"], k["signs"], k["norm"], k["rnorm"], v["codes"],
                  v["norm"])
    return time.perf_counter() - t0, T


def cpu_baseline(w, budget_s: float = 10.0):
    """The oracle, as it stands, on whole (batch, KV-head) slices of the workload until about
    budget_s seconds of CPU work have been timed."""
    import oracle
    oracle.build()
    secs = toks = 0
    i = 0
    while secs < budget_s and i < 64:
        s_, t_ = oracle_sample(w, 20260003 + i, w["T"])
        secs += s_
        toks += t_
        i += 1
    return {"value": toks / secs, "unit": "keys/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{i} (batch, KV-head) slices of {w['T']} tokens each: keys and values compressed and "
                      f"attended by {w['Hq'] // w['Hkv']} query heads, {secs:.1f} s of CPU wall time"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    oracle.build()
    w = W3
    T = w["T"]
    times = []
    for i in range(args.warmup + args.steps):
        secs, toks = oracle_sample(w, 20260003 + i, T)
        if i >= args.warmup:
            times.append(secs)
    per = sum(times) / len(times)
    value = T / per
    line = {"metric": METRIC, "value": value, "unit": "keys/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": per * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": WORKLOAD_NAME, "sample_tokens_per_step": T, **w},
            "cpu_baseline": {"value": value, "unit": "keys/s", "cores": oracle.num_threads(), "kind": "oracle",
                             "sample": f"per step one (batch, KV-head) slice of {T} tokens (K+V compress, "
                                       f"attend by {w['Hq'] // w['Hkv']} heads)"},
            "e2e": {"value": value, "unit": "keys/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# -------------------------------------------------------------------- GPU arm

def source_closure(path: str) -> list[str]:
    """Repo-relative paths of `path` and of every file it includes with #include "...", followed
    recursively (looked up beside the including file, then in the package's csrc/ and include/)."""
    import re
    seen, todo = [], [path]
    dirs = [os.path.join("kv_cache_vector_compress_b200", "csrc"), "include"]
    while todo:
        rel = todo.pop()
        if rel in seen:
            continue
        seen.append(rel)
        try:
            text = open(os.path.join(ROOT, rel)).read()
        except OSError:
            continue
        for inc in re.findall(r'^\s*#\s*include\s+"([^"]+)"', text, flags=re.M):
            for base in [os.path.dirname(rel)] + dirs:
                cand = os.path.normpath(os.path.join(base, inc))
                if os.path.exists(os.path.join(ROOT, cand)):
                    todo.append(cand)
                    break
    return sorted(seen)


def sources_sha1(path: str) -> str:
    """sha1 over the kernel source and everything it includes (names and contents)."""
    import hashlib
    h = hashlib.sha1()
    for rel in source_closure(path):
        h.update(rel.encode() + b"\0")
        h.update(open(os.path.join(ROOT, rel), "rb").read())
    return h.hexdigest()


def traffic_per_unit(kernel: str):
    """DRAM bytes per unit of `kernel` from the committed counters (profiles/dram_traffic.json),
    or None when the kernel's source or anything it includes has changed since they were taken."""
    try:
        rec = json.load(open(os.path.join(ROOT, "profiles", "dram_traffic.json")))["kernels"][kernel]
    except (OSError, ValueError, KeyError):
        return None
    if sources_sha1(rec["source"]) != rec["sources_sha1"]:
        return None
    return float(rec["bytes_per_unit"])


def run_tq(args):
    import numpy as np
    import torch

    from kv_cache_vector_compress_b200 import dist as tqdist
    ri = tqdist.rank_info()
    world, rank, local = ri.world, ri.rank, ri.local
    torch.cuda.set_device(local)
    tqdist.init("nccl", timeout_s=120)
    from kv_cache_vector_compress_b200 import synth, tq

    w = dict(W3)
    if args.batch:
        w["B"] = args.batch
    d, m, bits = w["d"], w["m"], w["bits"]
    B, Hq, Hkv, Nq, T = w["B"], w["Hq"], w["Hkv"], w["Nq"], w["T"]
    n = B * Hkv * T
    s = synth.seeds(3)
    off = tqdist.seed_offset(rank)
    R = torch.from_numpy(synth.rotation(d, s["R"])).cuda()
    S = torch.from_numpy(synth.gaussian(m, d, s["S"])).cuda()
    p = tq.Params(d, bits, m, R, S)
    K = synth.torch_normal_f16((n, d), s["keys"] + off)
    V = synth.torch_normal_f16((n, d), s["values"] + off)
    Q = synth.torch_normal_f32((B, Hq, Nq, d), s["queries"] + off)
    kc = torch.empty((n, (bits - 1) * d // 32), dtype=torch.int32, device="cuda")
    ks = torch.empty((n, m // 32), dtype=torch.int32, device="cuda")
    kn = torch.empty(n, dtype=torch.float16, device="cuda")
    kr = torch.empty(n, dtype=torch.float16, device="cuda")
    vc = torch.empty((n, bits * d // 32), dtype=torch.int32, device="cuda")
    vn = torch.empty(n, dtype=torch.float16, device="cuda")
    out = torch.empty((B, Hq, Nq, d), dtype=torch.float32, device="cuda")
    scratch = torch.empty(tq.tq_attend_scratch_bytes(p, B, Hq, Hkv, Nq, T), dtype=torch.uint8, device="cuda")
    keys, vals = (kc, ks, kn, kr), (vc, vn)
    stream = torch.cuda.current_stream()

    def step(ev=None):
        if ev:
            ev[0].record(stream)
        tq.tq_compress_keys(p, K, kc, ks, kn, kr)
        if ev:
            ev[1].record(stream)
        tq.tq_compress_values(p, V, vc, vn)
        if ev:
            ev[2].record(stream)
        tq.tq_attend(p, Q, keys, vals, Hkv, T, out=out, scratch=scratch)
        if ev:
            ev[3].record(stream)

    def barrier():
        tqdist.barrier()
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        step()
    barrier()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    with ClockSampler(local) as clk:
        time.sleep(0.3)
        barrier()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for i in range(args.steps):
            step(evs[i])
        t1.record(stream)
        barrier()
    ms = t0.elapsed_time(t1)
    # scores alone over the same cache (not part of the step): tq_scores into a [B, Hq, Nq, T] buffer
    sc_buf = torch.empty((B, Hq, Nq, T), dtype=torch.float32, device="cuda")
    sc_scr = torch.empty(tq.tq_scores_scratch_bytes(p, B, Hq, Hkv, Nq, T, 0), dtype=torch.uint8, device="cuda")
    for _ in range(args.warmup):
        tq.tq_scores(p, Q, keys, Hkv, T, scores=sc_buf, scratch=sc_scr)
    barrier()
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s0.record(stream)
    for _ in range(args.steps):
        tq.tq_scores(p, Q, keys, Hkv, T, scores=sc_buf, scratch=sc_scr)
    s1.record(stream)
    barrier()
    scores_ms = s0.elapsed_time(s1) / args.steps
    del sc_buf, sc_scr
    op_ms = {"compress_keys": 0.0, "compress_values": 0.0, "attend": 0.0}
    for e in evs:
        op_ms["compress_keys"] += e[0].elapsed_time(e[1]) / args.steps
        op_ms["compress_values"] += e[1].elapsed_time(e[2]) / args.steps
        op_ms["attend"] += e[2].elapsed_time(e[3]) / args.steps
    ms = tqdist.max_over_ranks(ms, device="cuda")
    ms_step = ms / args.steps

    # end to end through the C-ABI with host buffers: one tq_compress_attend_host call per step
    # copies the pinned host K/V/Q in, compresses, attends and copies the output back
    hK = torch.empty((n, d), dtype=torch.float16, pin_memory=True)
    hV = torch.empty((n, d), dtype=torch.float16, pin_memory=True)
    hQ = torch.empty((B, Hq, Nq, d), dtype=torch.float32, pin_memory=True)
    hO = torch.empty((B, Hq, Nq, d), dtype=torch.float32, pin_memory=True)
    hK.copy_(K)
    hV.copy_(V)
    hQ.copy_(Q)
    hscr = torch.empty(tq.tq_compress_attend_host_scratch_bytes(p, torch.float16, B, Hq, Hkv, Nq, T),
                       dtype=torch.uint8, device="cuda")

    def e2e_step():
        tq.tq_compress_attend_host(p, hK, hV, hQ, Hkv, T, keys, vals, hO, scratch=hscr)

    for _ in range(args.warmup):
        e2e_step()
    barrier()
    a0 = torch.cuda.Event(enable_timing=True)
    a1 = torch.cuda.Event(enable_timing=True)
    a0.record(stream)
    for _ in range(args.steps):
        e2e_step()
    a1.record(stream)
    barrier()
    e2e_ms = a0.elapsed_time(a1) / args.steps
    e2e_ms = tqdist.max_over_ranks(e2e_ms, device="cuda")

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w)

    if rank == 0:
        pk = peaks()
        ab = algorithmic_bytes(w)
        breakdown = {}
        for op, t in op_ms.items():
            gbs = ab[op] / (t * 1e-3) / 1e9
            breakdown[op] = {"ms": t, "algorithmic_bytes": ab[op], "GB/s": gbs, "frac_hbm": gbs / pk["hbm_gbs"]}
        breakdown["compress_keys"]["vectors_per_s"] = n / (op_ms["compress_keys"] * 1e-3)
        breakdown["compress_values"]["vectors_per_s"] = n / (op_ms["compress_values"] * 1e-3)
        breakdown["attend"]["packed_keys_scored_per_s"] = n / (op_ms["attend"] * 1e-3)
        # scores only (outside the step): packed keys read, fp32 scores written
        kbytes = n * record_bytes(w)[0]
        sbytes = B * Hq * Nq * T * 4
        sgbs = (kbytes + sbytes) / (scores_ms * 1e-3) / 1e9
        breakdown["scores_only"] = {"ms": scores_ms, "algorithmic_bytes": kbytes + sbytes,
                                    "bytes_note": "packed keys read + fp32 scores written", "GB/s": sgbs,
                                    "frac_hbm": sgbs / pk["hbm_gbs"],
                                    "packed_keys_scored_per_s": n / (scores_ms * 1e-3)}
        dom = max(op_ms, key=lambda k: op_ms[k])
        ach = ab[dom] / (op_ms[dom] * 1e-3) / 1e9
        tpu = traffic_per_unit(dom)
        traffic = None if tpu is None else tpu * n
        value = tqdist.weak_scaling_value(n, world, ms_step * 1e-3)
        line = {
            "metric": METRIC, "value": value, "unit": "keys/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": WORKLOAD_NAME, "parallelism": f"dp{world} (independent batches)", **w,
                       "l2": f"inputs larger than L2 ({2 * n * d * 2 / 1e9:.2f} GB of fp16 K/V read per step)"},
            "breakdown": breakdown,
            "roofline": {"kernel": dom, "bound": "hbm", "achieved": ach, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": ach / pk["hbm_gbs"], "traffic": traffic, "peak_source": pk["source"]},
            "e2e": {"value": world * n / (e2e_ms * 1e-3), "unit": "keys/s",
                    "h2d_bytes_per_step": int(hK.numel() * 2 + hV.numel() * 2 + hQ.numel() * 4),
                    "d2h_bytes_per_step": int(hO.numel() * 4)},
            # per step: compress keys, compress values, query operands + bit-plane attention
            "gpu_launches": 4 * args.steps,
            "clocks": clk.summary(),
        }
        if cpu:
            line["cpu_baseline"] = cpu
        print(json.dumps(line), flush=True)
    tqdist.barrier()
    tqdist.destroy()
    return 0


def run_workload(args):
    """Secondary measurements of the other workloads (one JSON line each, not the headline):
    per-op device time with CUDA events after warm-up, rates, and HBM fractions."""
    import numpy as np
    import torch
    from kv_cache_vector_compress_b200 import dist as tqdist
    from kv_cache_vector_compress_b200 import synth, tq
    ri = tqdist.rank_info()
    torch.cuda.set_device(ri.local)
    pk = peaks()
    wl = args.workload
    if ri.world > 1 and wl != 5:
        raise SystemExit("only the vector-search workload (5) shards over ranks; the others run on one GPU")
    s = synth.seeds(wl)
    st = torch.cuda.current_stream()

    def timed(fn, steps=args.steps, warmup=args.warmup):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(st)
        for _ in range(steps):
            fn()
        b.record(st)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / steps

    def rec(op, ms, units, unit, nbytes, gpus=1):
        # nbytes and units are whole-job figures; the HBM fraction is taken against the peak of
        # all `gpus` devices that shared the work
        gbs = nbytes / (ms * 1e-3) / 1e9
        return {"op": op, "ms": ms, "units": units, f"{unit}_per_s": units / (ms * 1e-3), "GB/s": gbs,
                "frac_hbm": gbs / (gpus * pk["hbm_gbs"])}

    out = []
    if wl == 1:
        w = synth.workload1()
        d, m, bits, T = 128, 64, 3, 4096
        p = tq.Params(d, bits, m, torch.from_numpy(w["R"]).cuda(), torch.from_numpy(w["S"]).cuda())
        K, V, Q = (torch.from_numpy(w[k]).cuda() for k in ("K", "V", "Q"))
        keys = tq.tq_compress_keys(p, K)
        vals = tq.tq_compress_values(p, V)
        ms = timed(lambda: tq.tq_compress_keys(p, K, *keys))
        out.append(rec("compress_keys", ms, T, "vectors", T * (d * 4 + 44)))
        ms = timed(lambda: tq.tq_compress_values(p, V, *vals))
        out.append(rec("compress_values", ms, T, "vectors", T * (d * 4 + 50)))
        sc = torch.empty((1, 1, 16, T), dtype=torch.float32, device="cuda")
        ms = timed(lambda: tq.tq_scores(p, Q, keys, 1, T, scores=sc))
        out.append(rec("scores", ms, T, "keys", T * 44 + 16 * T * 4))
        o = torch.empty((1, 1, 16, d), dtype=torch.float32, device="cuda")
        ms = timed(lambda: tq.tq_attend(p, Q, keys, vals, 1, T, out=o))
        out.append(rec("attend", ms, T, "keys", T * 94))
        name = "single head d128 3-bit: 4096 K + 4096 V fp32 unit vectors, 16 queries (latency)"
    elif wl == 2:
        d, m, L, H, T = 128, 64, 36, 2, 8192
        n = L * H * T
        R = torch.from_numpy(synth.rotation(d, s["R"])).cuda()
        S = torch.from_numpy(synth.gaussian(m, d, s["S"])).cuda()
        sc = np.exp(np.random.Generator(np.random.PCG64(s["scales"])).standard_normal((L * H, d)))
        K = (synth.torch_normal_f16((L * H, T, d), s["keys"]).float()
             * torch.from_numpy(sc.astype(np.float32)).cuda()[:, None, :]).half().view(n, d)
        V = synth.torch_normal_f16((n, d), s["values"])
        for bits in (2, 3, 4):
            p = tq.Params(d, bits, m, R, S)
            keys = tq.tq_compress_keys(p, K)
            vals = tq.tq_compress_values(p, V)
            kb = (bits - 1) * d // 8 + m // 8 + 4
            vb = bits * d // 8 + 2
            ms = timed(lambda: tq.tq_compress_keys(p, K, *keys))
            out.append(rec(f"compress_keys_b{bits}", ms, n, "vectors", n * (2 * d + kb)))
            ms = timed(lambda: tq.tq_compress_values(p, V, *vals))
            out.append(rec(f"compress_values_b{bits}", ms, n, "vectors", n * (2 * d + vb)))
        name = "Qwen2.5-3B-shaped prefill compress: 36 layers x 2 KV heads x 8192 x 128 fp16, bits 2/3/4"
    elif wl == 4:
        d, m, B, Hq, Hkv, T = 256, 128, 8, 16, 4, 65536
        B = args.batch if args.batch > 0 else B
        n = B * Hkv * T
        R = torch.from_numpy(synth.rotation(d, s["R"])).cuda()
        S = torch.from_numpy(synth.gaussian(m, d, s["S"])).cuda()
        K = synth.torch_normal_f16((n, d), s["keys"])
        K[:, torch.from_numpy(synth.outlier_channels(d, s["scales"])).cuda()] *= 20
        V = synth.torch_normal_f16((n, d), s["values"])
        Q = synth.torch_normal_f32((B, Hq, 1, d), s["queries"])
        for bits in (2, 4):
            p = tq.Params(d, bits, m, R, S)
            keys = tq.tq_compress_keys(p, K)
            vals = tq.tq_compress_values(p, V)
            kb = (bits - 1) * d // 8 + m // 8 + 4
            vb = bits * d // 8 + 2
            ms = timed(lambda: tq.tq_compress_keys(p, K, *keys), steps=3)
            out.append(rec(f"compress_keys_b{bits}", ms, n, "vectors", n * (2 * d + kb)))
            ms = timed(lambda: tq.tq_compress_values(p, V, *vals), steps=3)
            out.append(rec(f"compress_values_b{bits}", ms, n, "vectors", n * (2 * d + vb)))
            o = torch.empty((B, Hq, 1, d), dtype=torch.float32, device="cuda")
            scr = torch.empty(tq.tq_attend_scratch_bytes(p, B, Hq, Hkv, 1, T), dtype=torch.uint8, device="cuda")
            ms = timed(lambda: tq.tq_attend(p, Q, keys, vals, Hkv, T, out=o, scratch=scr))
            out.append(rec(f"attend_b{bits}", ms, n, "keys", n * (kb + vb)))
        name = "wide-head decode: B8 Hq16/Hkv4 T65536 d256 m128, bits 2 and 4, 1% key channels x20"
    elif wl == 5:
        d, m, bits, Nq, k = 1024, 512, 4, 1024, 10
        N = args.db if args.db > 0 else 1_000_000
        # with several ranks the database of N keys is sharded (contiguous rows per rank, each
        # shard generated from its own seed); the per-rank top-k lists meet in sharded_topk
        tqdist.init("nccl", timeout_s=120)
        start, Nl = tqdist.shard(N, ri.world, ri.rank)
        R = torch.from_numpy(synth.rotation(d, s["R"])).cuda()
        S = torch.from_numpy(synth.gaussian(m, d, s["S"])).cuda()
        p = tq.Params(d, bits, m, R, S)
        X = synth.torch_normal_f32((Nl, d), s["keys"] + tqdist.seed_offset(ri.rank))
        X /= X.norm(dim=1, keepdim=True)
        Qv = synth.torch_normal_f32((1, 1, Nq, d), s["queries"])
        Qv /= Qv.norm(dim=-1, keepdim=True)
        keys = tq.tq_compress_keys(p, X)
        kb = (bits - 1) * d // 8 + m // 8 + 4

        def timed_ranks(fn, steps, warmup):
            # device time on every rank between barriers; the slowest rank's time is reported
            for _ in range(warmup):
                fn()
            torch.cuda.synchronize()
            tqdist.barrier()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(st)
            for _ in range(steps):
                fn()
            b.record(st)
            torch.cuda.synchronize()
            tqdist.barrier()
            return tqdist.max_over_ranks(a.elapsed_time(b) / steps, device="cuda")
        ms = timed_ranks(lambda: tq.tq_compress_keys(p, X, *keys), steps=2, warmup=1)
        out.append(rec("compress_db", ms, N, "vectors", N * (4 * d + kb), gpus=ri.world))
        ti = torch.empty((1, 1, Nq, k), dtype=torch.int32, device="cuda")
        tv = torch.empty((1, 1, Nq, k), dtype=torch.float32, device="cuda")
        scr = torch.empty(tq.tq_scores_scratch_bytes(p, 1, 1, 1, Nq, Nl, k), dtype=torch.uint8, device="cuda")

        def search():
            tq.tq_scores(p, Qv, keys, 1, Nl, want_scores=False, topk=k, topk_idx=ti, topk_val=tv, scratch=scr)
            if ri.world > 1:
                tqdist.sharded_topk(ti.view(Nq, k), tv.view(Nq, k), k, start)
        ms = timed_ranks(search, steps=5, warmup=3)
        r = rec("scores_top10", ms, N * Nq, "query_key_pairs", N * kb, gpus=ri.world)
        r["tflops_equiv"] = 2.0 * Nq * N * (d + m) / (ms * 1e-3) / 1e12
        # tensor-core work actually issued: fp16 hi/lo split products, 3 per centroid column and
        # 2 per sign column, on 128-padded tiles
        pad = lambda x: (x + 127) // 128 * 128
        r["tflops_mma"] = 2.0 * pad(Nq) * pad(N) * (3 * d + 2 * m) / (ms * 1e-3) / 1e12
        r["frac_tensor"] = r["tflops_mma"] / (ri.world * pk["bf16_tflops"]) if pk.get("bf16_tflops") else None
        out.append(r)

        # tq_search: the same launch with single fp16 operand products (one per column)
        def search16():
            tq.tq_search(p, Qv, keys, 1, Nl, want_scores=False, topk=k, topk_idx=ti, topk_val=tv, scratch=scr)
            if ri.world > 1:
                tqdist.sharded_topk(ti.view(Nq, k), tv.view(Nq, k), k, start)
        ms = timed_ranks(search16, steps=5, warmup=3)
        r = rec("search_top10_fp16", ms, N * Nq, "query_key_pairs", N * kb, gpus=ri.world)
        r["tflops_equiv"] = 2.0 * Nq * N * (d + m) / (ms * 1e-3) / 1e12
        r["tflops_mma"] = 2.0 * pad(Nq) * pad(N) * (d + m) / (ms * 1e-3) / 1e12
        r["frac_tensor"] = r["tflops_mma"] / (ri.world * pk["bf16_tflops"]) if pk.get("bf16_tflops") else None
        out.append(r)
        name = (f"vector search: {N} x d1024 4-bit Prod (m=512) fp32 DB, 1024 queries, top-10"
                + (f", sharded over {ri.world} GPUs (per-rank top-k lists gathered and merged)" if ri.world > 1 else ""))
    elif wl == 6:
        # one decode step on the decode-attention shape: append the new token of every (batch, KV
        # head) into slot t of a cache of capacity T, then attend over slots 0..t
        d, m, bits, B, Hq, Hkv, T = 128, 64, 3, 32, 32, 8, 32768
        B = args.batch if args.batch > 0 else B
        t, ns = T - 1, B * Hkv
        n = ns * T
        R = torch.from_numpy(synth.rotation(d, s["R"])).cuda()
        S = torch.from_numpy(synth.gaussian(m, d, s["S"])).cuda()
        p = tq.Params(d, bits, m, R, S)
        keys = tq.tq_compress_keys(p, synth.torch_normal_f16((n, d), s["keys"]))
        vals = tq.tq_compress_values(p, synth.torch_normal_f16((n, d), s["values"]))
        kn = synth.torch_normal_f16((B, Hkv, d), s["scales"] + 1)
        vn = synth.torch_normal_f16((B, Hkv, d), s["scales"] + 2)
        Q = synth.torch_normal_f32((B, Hq, 1, d), s["queries"])
        o = torch.empty((B, Hq, 1, d), dtype=torch.float32, device="cuda")
        scr = torch.empty(tq.tq_attend_scratch_bytes(p, B, Hq, Hkv, 1, T), dtype=torch.uint8, device="cuda")
        kb, vb = (bits - 1) * d // 8 + m // 8 + 4, bits * d // 8 + 2
        nbytes = ns * (t + 1) * (kb + vb) + ns * 2 * d * 2
        ms = timed(lambda: tq.tq_append_attend(p, Q, kn, vn, keys, vals, Hkv, t, T, out=o, scratch=scr))
        out.append(rec("append_attend", ms, ns * (t + 1), "keys", nbytes))
        # the same step unfused: compress the B * Hkv new rows, then attend over the cache
        nk = tq.tq_compress_keys(p, kn.view(ns, d))
        nv = tq.tq_compress_values(p, vn.view(ns, d))

        def unfused():
            tq.tq_compress_keys(p, kn.view(ns, d), *nk)
            tq.tq_compress_values(p, vn.view(ns, d), *nv)
            tq.tq_attend(p, Q, keys, vals, Hkv, T, out=o, scratch=scr)
        ms = timed(unfused)
        out.append(rec("compress_new_then_attend", ms, ns * (t + 1), "keys", nbytes))
        name = (f"decode step: B{B} Hq32/Hkv8 d128 3-bit, append the new token into slot {t} of a "
                f"{T}-slot cache, attend over {t + 1} tokens")
    elif wl == 7:
        # attention quality of the compressed cache on synthetic Qwen2.5-3B-shaped decode inputs
        # (36 layers x 2 KV heads as the batch, 16 query heads, 8K context, one query per head),
        # two input recipes: "gaussian" (keys, values, queries N(0,1): the coordinate model the
        # method is built on) and "key_outliers" (keys N(0,1) x lognormal(0,1) per (layer, KV
        # head, channel), as real key caches have outlier channels; values, queries N(0,1))
        from kv_cache_vector_compress_b200 import quality
        d, m, L, Hkv, Hq, T = 128, 64, 36, 2, 16, 8192
        R = torch.from_numpy(synth.rotation(d, s["R"])).cuda()
        S = torch.from_numpy(synth.gaussian(m, d, s["S"])).cuda()
        sc = torch.from_numpy(np.exp(np.random.Generator(np.random.PCG64(s["scales"])).standard_normal(
            (L, Hkv, 1, d))).astype(np.float32)).cuda()
        V = synth.torch_normal_f16((L, Hkv, T, d), s["values"])
        Q = synth.torch_normal_f32((L, Hq, 1, d), s["queries"])
        res = {}
        for recipe in ("gaussian", "key_outliers"):
            K = synth.torch_normal_f16((L, Hkv, T, d), s["keys"])
            if recipe == "key_outliers":
                K = (K.float() * sc).half()
            res[recipe] = []
            for bits in (2, 3, 4):
                p = tq.Params(d, bits, m, R, S)
                keys = tq.tq_compress_keys(p, K.view(-1, d))
                vals = tq.tq_compress_values(p, V.view(-1, d))
                res[recipe].append({"bits": bits, **quality.attention_quality(p, Q, K, V, keys, vals)})
        # proj_dim sweep at 3 bits on the gaussian recipe: the QJL term's variance falls as 1/m
        K = synth.torch_normal_f16((L, Hkv, T, d), s["keys"])
        sweep = []
        for mm in (32, 64, 128):
            Sm = torch.from_numpy(synth.gaussian(mm, d, s["S"] + mm)).cuda()
            p = tq.Params(d, 3, mm, R, Sm)
            keys = tq.tq_compress_keys(p, K.view(-1, d))
            vals = tq.tq_compress_values(p, V.view(-1, d))
            sweep.append({"proj_dim": mm, **quality.attention_quality(p, Q, K, V, keys, vals)})
        # ablation: MSE-only keys (b MSE bits, no QJL) against the two-stage keys, scores only
        mse = []
        for b in (2, 3):
            pv = tq.Params(d, b, m, R, S)
            codes, norm = tq.tq_compress_values(pv, K.view(-1, d))
            ps = tq.Params(d, b + 1, m, R, S)
            mse.append({"mse_bits": b, **quality.score_quality(ps, Q, K, quality.mse_only_keys(ps, codes, norm))})
        print(json.dumps({"workload": wl, "name": "attention quality, synthetic Qwen2.5-3B-shaped decode: "
                          "36 layers x 2 KV heads, 16 query heads, T8192, d128 (means over 576 query rows)",
                          "quality": res, "proj_dim_sweep_3bit_gaussian": sweep,
                          "mse_only_keys_gaussian": mse,
                          "pages_qwen_validation": {"note": "real activations, not comparable",
                                                    "cosine": {"4": 0.999, "3": 0.995, "2": 0.988},
                                                    "top1": {"4": 0.87, "3": 0.82, "2": 0.66}}}), flush=True)
        return 0
    else:
        raise SystemExit("unknown workload")
    if ri.rank == 0:
        print(json.dumps({"workload": wl, "name": name, "ops": out, "n_gpus": ri.world,
                          "peak_hbm_gbs": pk["hbm_gbs"]}), flush=True)
    tqdist.destroy()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="tq", choices=["tq", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--batch", type=int, default=0, help="sequences per GPU (default: the workload's 32)")
    ap.add_argument("--db", type=int, default=0,
                    help="database vectors of the vector-search workload (default 1,000,000; smaller for profiling)")
    ap.add_argument("--workload", type=int, default=3,
                    help="3 (default) prints the headline line; 1, 2, 4, 5, 6 print secondary per-op "
                         "measurements, 7 the attention quality of the compressed cache")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)
    if args.workload != 3:
        return run_workload(args)
    return run_tq(args)


if __name__ == "__main__":
    sys.exit(main())
