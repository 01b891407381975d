#!/usr/bin/env python
"""Benchmark of compressed decode attention over a packed KV cache on B200.

One step = one decode step of the whole hot path for a batch of sequences, in
one tq_decode_step call (three launches): quantize the newest token's K and V
into the packed cache (rotation, Lloyd-Max codes, QJL sketch) and pre-rotate
the queries, split-K attention straight from the packed codes, log-sum-exp
merge and the final inverse rotation.

Headline `value`: KV tokens attended per second (B * T per step) with the
packed cache and the step inputs resident in HBM.  `e2e`: the same metric with
the step inputs (query, new K/V token) copied from pinned host memory and the
output copied back inside the timed region.  Also reported: the roofline of
the attention call against the measured HBM copy bandwidth, quantize
throughput (Mvec/s) on the prefill-shaped sweep, SM clocks sampled during the
run, and the CPU oracle timed on a bounded sample (`cpu_baseline`).

`--impl reference` times the fp64 CPU oracle (the only reference
implementation this method has here) on a bounded sample of the same workload.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
Under torchrun (N > 1) each rank runs an independent replica (the decode path
needs no exchange between GPUs); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time
from pathlib import Path

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

METRIC = "compressed decode-attn KV tokens/s (% HBM roofline); quantize Mvec/s"
UNIT = "KV tokens/s"

WORKLOADS = {
    # Llama-3-8B-shaped decode: GQA 4, k3v4 (keys 2 Lloyd-Max bits + 1 QJL bit, m=128; values 4 bits)
    "llama3-8b-decode": dict(B=16, Hq=32, Hkv=8, d=128, T=32768, bits_k=3, bits_v=4, m=128),
    # 70B-shaped long-context decode: GQA 8
    "70b-decode-k3v4": dict(B=4, Hq=64, Hkv=8, d=128, T=131072, bits_k=3, bits_v=4, m=128),
    "70b-decode-k4v4": dict(B=4, Hq=64, Hkv=8, d=128, T=131072, bits_k=4, bits_v=4, m=128),
}
QUANT_SWEEP = dict(tokens=131072, heads=8, d=128, bits=(2, 3, 4))
# The other cache formats of the vLLM study (norm-corrected MSE-only, and
# 8-bit keys), timed on the Llama-3-8B decode shape.
FORMAT_VARIANTS = ("k3v4_nc", "4bit_nc", "3bit_nc", "k8v4")


def peaks():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        j = json.loads(p.read_text())
        return float(j["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def tensor_peak():
    """Dense bf16 tensor peak (burst), measured, else the machine's fallback."""
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        j = json.loads(p.read_text())
        for key in ("bf16_tflops", "bf16_tflops_burst"):
            if key in j:
                return float(j[key]), f"measured {key} (cuBLAS bf16 burst; fp16 same nominal rate)"
    return 1590.0, "fallback 1.59 PFLOP/s bf16"


def kernel_source_hash(files) -> str:
    """Hash of the sources a decode-attention kernel is built from (its
    counters go stale when these change)."""
    h = hashlib.sha256()
    csrc = ROOT / "compressed_decode_attention_quantize_b200" / "csrc"
    for name in files:
        h.update((csrc / name).read_bytes())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str):
    """DRAM bytes per attention launch from a committed ncu summary, or None if
    the sources of that workload's kernel changed since the counters were
    taken."""
    p = ROOT / "profiles" / "attn_traffic.json"
    if not p.exists():
        return None
    j = json.loads(p.read_text())
    e = j.get(workload)
    if not e or e.get("source_hash") != kernel_source_hash(e.get("source_files", [])):
        return None
    return e.get("dram_bytes_per_launch")


def max_over_ranks(vals, world: int, device):
    """Element-wise max of vals over all ranks: the slowest rank sets the
    job's time.  One all-reduce on the process group when world > 1."""
    import torch
    t = torch.tensor(vals, dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def whole_job_rate(units_per_rank: float, world: int, ms: float) -> float:
    """Units all ranks processed per second, over the max-over-ranks time."""
    return world * units_per_rank / (ms / 1e3)


def kv_bytes(w, ctx) -> int:
    kb = ctx.key_layout["bytes_per_vector"]
    vb = ctx.value_layout["bytes_per_vector"]
    return w["B"] * w["Hkv"] * w["T"] * (kb + vb)


class ClockSampler:
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.proc = None
        self.windows = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.f, stderr=subprocess.DEVNULL)
        except FileNotFoundError:
            self.proc = None

    def mark(self, t0, t1):
        self.windows.append((t0, t1))

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        time.sleep(0.25)
        self.proc.terminate()
        self.proc.wait()
        self.f.flush()
        rows = []
        for ln in Path(self.f.name).read_text().splitlines():
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 10:
                continue
            try:
                ts = time.mktime(time.strptime(parts[0].split(".")[0], "%Y/%m/%d %H:%M:%S"))
                ts += float("0." + parts[0].split(".")[1]) if "." in parts[0] else 0.0
                rows.append((ts, float(parts[2]), float(parts[3]), parts[6:10]))
            except (ValueError, IndexError):
                continue
        os.unlink(self.f.name)
        inside = [r for r in rows if any(a - 0.15 <= r[0] <= b + 0.15 for a, b in self.windows)]
        use = inside or rows
        if not use:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in use for i, v in enumerate(r[3]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[1] for r in use), "sm_max_mhz": max(r[2] for r in use),
                "reasons": reasons, "samples": len(use), "in_timed_region": bool(inside)}


# ---------------------------------------------------------------------------
# CPU oracle arms (the only places this script runs the oracle)
# ---------------------------------------------------------------------------
def oracle_decode_sample(w, kc_host, vc_host, q_host, tab):
    """Oracle attention for the G query heads of one (sequence, kv head) slice."""
    from oracle import tq_oracle as o
    T = kc_host["norm"].shape[2]
    return o.attention(tab, q_host, kc_host["codes"], kc_host.get("qjl"), kc_host["norm"],
                       kc_host.get("rnorm"), vc_host["codes"], vc_host["norm"], [T], 1)


def cpu_baseline_from_device(w, ctx, kc, vc, q, gpu_out, budget_s: float = 10.0):
    """The fp64 oracle on whole (sequence, kv head) slices of the bench's own
    cache, one after another until about budget_s seconds of CPU work.  The
    same oracle outputs are compared with the GPU's attention output for
    these slices (gpu_out: host [B, Hq, d] from the same query and cache)."""
    import numpy as np
    import torch
    from oracle import tq_oracle as o
    G = w["Hq"] // w["Hkv"]
    T = w["T"]

    def host(t, b, h):
        if t is None:
            return None
        a = t[b:b + 1, h:h + 1, :T].cpu()
        return a.numpy().view(np.uint32) if a.dtype == torch.int32 else a.numpy()

    tab = o.make_tables(w["d"], w["bits_k"], w["bits_v"], w["m"], 0)
    slices, dt, worst = 0, 0.0, 0.0
    for b in range(w["B"]):
        for h in range(w["Hkv"]):
            kh = {k: host(v, b, h) for k, v in kc.items()}
            vh = {k: host(v, b, h) for k, v in vc.items()}
            qh = q[b:b + 1, h * G:(h + 1) * G].float().cpu().numpy().astype(np.float64)
            t0 = time.perf_counter()
            ref = oracle_decode_sample(w, kh, vh, qh, tab)
            dt += time.perf_counter() - t0
            got = gpu_out[b, h * G:(h + 1) * G].astype(np.float64)
            rel = np.linalg.norm(got - ref[0], axis=-1) / np.linalg.norm(ref[0], axis=-1)
            worst = max(worst, float(rel.max()))
            slices += 1
            if dt >= budget_s:
                break
        if dt >= budget_s:
            break
    tokens_equiv = slices * T / w["Hkv"]   # Hkv slices of T tokens make T full-width KV tokens
    base = {"value": tokens_equiv / dt, "unit": UNIT, "cores": len(os.sched_getaffinity(0)),
            "kind": "oracle",
            "sample": f"fp64 oracle attention of the {G} query heads of {slices} (sequence, kv head) slices "
                      f"of {T} packed tokens ({dt:.1f} s); tokens/s counts {w['Hkv']} slices as {T} "
                      f"full-width KV tokens"}
    attn = {"pairs": slices * G, "max_rel_l2": worst, "tol": 2e-3, "ok": worst <= 2e-3,
            "sample": f"the GPU attention output of the same {slices} (sequence, kv head) slices "
                      f"against the oracle's (same query, same packed cache)"}
    return base, attn


def code_parity(w, kc, vc, xs):
    """Excused-index counts: the oracle quantizes the sampled input slices
    (bf16 K/V kept on the host when the cache was built) and compares its
    indices and QJL bits with the cache's codes for the same tokens.  An index
    may differ only within 1e-5 of a decision boundary on the rotated
    unit-vector scale; the counts also give the in-band fraction on the
    standardized sqrt(d) scale."""
    import numpy as np
    import torch
    from oracle import tq_oracle as o
    tab = o.make_tables(w["d"], w["bits_k"], w["bits_v"], w["m"], 0)

    def host(t, b, h, n):
        if t is None:
            return None
        a = t[b, h, :n].cpu()
        return a.numpy().view(np.uint32) if a.dtype == torch.int32 else a.numpy()

    out = {}
    for which, cache in (("k", kc), ("v", vc)):
        tot = {}
        for (b, h), (xk, xv) in xs.items():
            x = (xk if which == "k" else xv).astype(np.float64)
            n = x.shape[0]
            c = o.code_agreement(tab, which, x, host(cache["codes"], b, h, n),
                                 host(cache.get("qjl"), b, h, n))
            for k, v in c.items():
                tot[k] = tot.get(k, 0) + v
        tot["excused_frac"] = tot["mismatches"] / tot["indices"]
        tot["in_band_unit_frac"] = tot["in_band_unit"] / tot["indices"]
        tot["in_band_std_frac"] = tot["in_band_std"] / tot["indices"]
        tot["ok"] = tot["outside_band"] == 0 and tot["excused_frac"] <= 1e-4 and \
            tot.get("qjl_outside_band", 0) == 0
        out["keys" if which == "k" else "values"] = tot
    n = sum(x[0].shape[0] for x in xs.values())
    out["sample"] = (f"{n} K and {n} V vectors: tokens [0, {n // len(xs)}) of (sequence, kv head) "
                     f"{', '.join(str(k) for k in xs)}; band 1e-5 on the unit scale "
                     f"(standardized scale: 1e-5 / sqrt(d))")
    return out


def run_reference(args, w):
    """Reference arm: the fp64 CPU oracle on a bounded sample per step."""
    import numpy as np
    import tq_inputs
    from oracle import tq_oracle as o
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    G = w["Hq"] // w["Hkv"]
    sample_T = 2048
    tab = o.make_tables(w["d"], w["bits_k"], w["bits_v"], w["m"], 0)
    K = tq_inputs.outlier_kv(1, 1, sample_T, w["d"], seed=1)[0, 0].double().numpy()
    V = tq_inputs.outlier_kv(1, 1, sample_T, w["d"], seed=2)[0, 0].double().numpy()
    zk = o.quantize(K, tab, "k")
    zv = o.quantize(V, tab, "v")
    r = lambda a: None if a is None else a[None, None]
    kh = {"codes": r(zk.codes), "qjl": r(zk.qjl), "norm": r(zk.norm), "rnorm": r(zk.rnorm)}
    vh = {"codes": r(zv.codes), "norm": r(zv.norm)}
    qs = [tq_inputs.iid((1, G, w["d"]), seed=100 + i).double().numpy() for i in range(4)]
    knew = tq_inputs.outlier_kv(1, 1, 1, w["d"], seed=3)[0, 0].double().numpy()

    def step(i):
        # quantize the newest K/V token, then attend over the sample
        o.quantize(knew, tab, "k")
        o.quantize(knew, tab, "v")
        oracle_decode_sample(w, kh, vh, qs[i % 4], tab)

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(i)
    dt = (time.perf_counter() - t0) / max(args.steps, 1)
    tokens_equiv = sample_T / w["Hkv"]
    value = tokens_equiv / dt
    cores = len(os.sched_getaffinity(0))
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": config_of(args, w),
        "impl": "reference",
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"per step: quantize one K and one V token, then fp64 oracle "
                                   f"attention of {G} query heads over one (sequence, kv head) slice "
                                   f"of {sample_T} tokens; counted as {sample_T}/{w['Hkv']} KV tokens"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def config_of(args, w):
    return {"workload": args.workload, "batch": w["B"], "q_heads": w["Hq"], "kv_heads": w["Hkv"],
            "head_dim": w["d"], "context": w["T"],
            "kv_format": f"k{w['bits_k']}v{w['bits_v']} (keys {w['bits_k'] - 1} Lloyd-Max bits + 1 QJL bit, "
                         f"m={w['m']}; values {w['bits_v']} bits)",
            "inputs": "bf16 K/V with log-normal per-channel scales and 1% x20 outlier channels; bf16 N(0,1) queries",
            "l2": "no flush: the packed cache read each step is larger than L2",
            "parallelism": f"replicas x{args.gpus} (no exchange)"}


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------
def quantize_sweep(tq, tq_inputs, torch, dev, hbm_peak, steps=10, warmup=3):
    s = QUANT_SWEEP
    X = tq_inputs.outlier_kv(1, s["heads"], s["tokens"], s["d"], seed=31, device=dev)[0].reshape(-1, s["d"])
    Y = tq_inputs.outlier_kv(1, s["heads"], s["tokens"], s["d"], seed=32, device=dev)[0].reshape(-1, s["d"])
    n = X.shape[0]
    points = []
    for bits in s["bits"]:
        for qjl in (True, False):
            ctx = tq.Context(s["d"], bits, bits, s["d"] if qjl else 0, 0)
            pk = ctx.empty_packed(tq.TQ_KEY, (n,), device=dev)
            pv = ctx.empty_packed(tq.TQ_VALUE, (n,), device=dev)
            for _ in range(warmup):
                ctx.quantize_into(X, tq.TQ_KEY, pk)
                ctx.quantize_into(Y, tq.TQ_VALUE, pv)
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(steps):
                ctx.quantize_into(X, tq.TQ_KEY, pk)
                ctx.quantize_into(Y, tq.TQ_VALUE, pv)
            e1.record()
            torch.cuda.synchronize()
            t = e0.elapsed_time(e1) / 1e3 / steps
            byts = 2 * n * s["d"] * 2 + n * (ctx.key_layout["bytes_per_vector"] + ctx.value_layout["bytes_per_vector"])
            points.append({"bits": bits, "qjl": qjl, "mvec_per_s": 2 * n / t / 1e6,
                           "gbs": byts / t / 1e9, "frac_hbm": byts / t / 1e9 / hbm_peak})
            ctx.close()
            del pk, pv
    del X, Y
    torch.cuda.empty_cache()
    head = next(p for p in points if p["bits"] == 3 and p["qjl"])
    return {"config": f"{s['tokens']} tokens x {s['heads']} kv heads x d={s['d']} bf16 K and V "
                      f"(outlier channels); K and V quantized each iteration; Mvec counts K+V vectors",
            "value": head["mvec_per_s"], "unit": "Mvec/s", "point": "bits=3 with QJL",
            "frac_hbm": head["frac_hbm"], "sweep": points}


VSEARCH = dict(n=1_000_000, nq=10_000, k=10, d=200, bits_k=4, m=200)


def vector_search(tq, tq_inputs, torch, dev, sm_mhz_max, steps=3, warmup=1):
    """Inner-product top-k over a compressed database (3 Lloyd-Max bits + QJL,
    m = d = 200): 1e6 mixture vectors, 1e4 queries, top-10 per query."""
    s = VSEARCH
    ctx = tq.Context(s["d"], s["bits_k"], 3, s["m"], 0)
    X = tq_inputs.mixture(s["n"], s["d"], seed=21, device=dev)
    Q = tq_inputs.mixture(s["nq"], s["d"], seed=22, means_seed=21, device=dev)
    db = ctx.quantize(X, tq.TQ_KEY)
    # The database build itself (fp32 input, d = 200: the CUDA-core quantizer), timed once warm.
    qa, qb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    qa.record()
    ctx.quantize_into(X, tq.TQ_KEY, db)
    qb.record()
    torch.cuda.synchronize()
    db_ms = qa.elapsed_time(qb)
    del X
    ws = torch.empty(ctx.topk_workspace_bytes(s["nq"], s["n"], s["k"]), dtype=torch.uint8, device=dev)
    for _ in range(warmup):
        ctx.topk(Q, db, s["k"], workspace=ws)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        ctx.topk(Q, db, s["k"], workspace=ws)
    e1.record()
    torch.cuda.synchronize()
    t = e0.elapsed_time(e1) / 1e3 / steps
    flop = 2.0 * s["nq"] * s["n"] * (s["d"] + s["m"])   # <q', c[idx]> over d, <s, sigma> over m
    # The scores are an fp16 tensor-core contraction: its peak is the measured
    # dense bf16 rate (fp16 has the same nominal rate).
    peak, peak_src = tensor_peak()
    ctx.close()
    del db, Q, ws
    torch.cuda.empty_cache()
    return {"config": f"{s['n']} db vectors x d={s['d']} (Gaussian mixture), {s['nq']} queries, "
                      f"top-{s['k']}; keys 3 Lloyd-Max bits + QJL (m={s['m']})",
            "value": s["nq"] / t, "unit": "queries/s", "ms_per_call": t * 1e3,
            "roofline": {"bound": "tensor", "achieved": flop / t / 1e12, "peak": peak, "unit": "TFLOP/s",
                         "frac": flop / t / 1e12 / peak, "peak_source": peak_src},
            "db_quantize": {"ms": db_ms, "mvec_per_s": s["n"] / db_ms / 1e3,
                            "note": "one warm tq_quantize of the fp32 database (fp32 CUDA-core kernel at d = 200)"}}


def variant_decode(tq, tq_inputs, torch, dev, hbm_peak, shape, steps=20, warmup=3):
    """tq_attn_decode for each format of FORMAT_VARIANTS on one decode shape."""
    B, Hq, Hkv, d, T = shape["B"], shape["Hq"], shape["Hkv"], shape["d"], shape["T"]
    out = {}
    runs = [(name, False) for name in FORMAT_VARIANTS] + [(name, True) for name in FORMAT_VARIANTS]
    for name, f16 in runs:
        label = name + ("+fp16norms" if f16 else "")
        try:
            out[label] = _variant_once(tq, tq_inputs, torch, dev, hbm_peak, shape, name, f16, steps, warmup)
        except Exception as e:   # a failed extra must not cost the headline line
            out[label] = {"error": f"{type(e).__name__}: {e}"}
    torch.cuda.empty_cache()
    return out


def decode_70b(tq, tq_inputs, torch, dev, hbm_peak, steps=20, warmup=3):
    """The 70B-shaped long-context decode (B=4, Hq=64, Hkv=8, T=131072,
    GQA 8) in both of its formats: the attention call (pre-rotate, split-K
    attention, merge) timed like the headline's."""
    out = {}
    for name in ("70b-decode-k3v4", "70b-decode-k4v4"):
        w = WORKLOADS[name]
        try:
            ctx = tq.Context(w["d"], w["bits_k"], w["bits_v"], w["m"], 0)
            res = _decode_call(tq, tq_inputs, torch, dev, hbm_peak, w, ctx, steps, warmup)
            res["kv_format"] = (f"k{w['bits_k']}v{w['bits_v']}: keys {w['bits_k'] - 1} Lloyd-Max bits + 1 QJL "
                                f"bit (m={w['m']}), values {w['bits_v']} bits")
            out[name] = res
        except Exception as e:   # a failed extra must not cost the headline line
            out[name] = {"error": f"{type(e).__name__}: {e}"}
    torch.cuda.empty_cache()
    return out


def _decode_call(tq, tq_inputs, torch, dev, hbm_peak, shape, ctx, steps, warmup):
    """Cache build (untimed), then CUDA-event timing of tq_attn_decode graph
    replays; returns ms per call, KV tokens/s and the fraction of measured HBM
    bandwidth on the algorithmic bytes (packed cache + queries + output)."""
    B, Hq, Hkv, d, T = shape["B"], shape["Hq"], shape["Hkv"], shape["d"], shape["T"]
    kc = ctx.empty_packed(tq.TQ_KEY, (B, Hkv, T), device=dev)
    vc = ctx.empty_packed(tq.TQ_VALUE, (B, Hkv, T), device=dev)
    for b in range(B):
        K = tq_inputs.outlier_kv(1, Hkv, T, d, seed=1000 + b, device=dev, scale_seed=1)[0]
        V = tq_inputs.outlier_kv(1, Hkv, T, d, seed=2000 + b, device=dev, scale_seed=2)[0]
        ctx.quantize_into(K, tq.TQ_KEY, {k: (None if v is None else v[b]) for k, v in kc.items()})
        ctx.quantize_into(V, tq.TQ_VALUE, {k: (None if v is None else v[b]) for k, v in vc.items()})
        del K, V
    q = tq_inputs.iid((B, Hq, d), seed=10, device=dev, dtype=torch.bfloat16)
    lens = torch.full((B,), T, dtype=torch.int32, device=dev)
    o = torch.empty(B, Hq, d, dtype=torch.float32, device=dev)
    ws = torch.empty(ctx.attn_workspace_bytes(B, Hq, T), dtype=torch.uint8, device=dev)
    for _ in range(warmup):
        ctx.attn_decode(q, kc, vc, lens, out=o, workspace=ws)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        ctx.attn_decode(q, kc, vc, lens, out=o, workspace=ws)
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    kb, vb = ctx.key_layout["bytes_per_vector"], ctx.value_layout["bytes_per_vector"]
    alg = B * Hkv * T * (kb + vb) + B * Hq * d * 2 + B * Hq * d * 4
    del g, kc, vc, ws
    ctx.close()
    return {"attn_ms": ms, "kv_tokens_per_s": B * T / (ms / 1e3),
            "hbm_frac": alg / (ms / 1e3) / 1e9 / hbm_peak, "algorithmic_bytes": alg,
            "shape": f"B={B} Hq={Hq} Hkv={Hkv} d={d} T={T}", "timing": f"{steps} CUDA-graph replays"}


def _variant_once(tq, tq_inputs, torch, dev, hbm_peak, shape, name, f16, steps, warmup):
    """One format: cache build (untimed), then graph replays of tq_attn_decode."""
    B, Hq, Hkv, d, T = shape["B"], shape["Hq"], shape["Hkv"], shape["d"], shape["T"]
    ctx = tq.Context.variant(name, d, 0, norm_f16=f16)
    kc = ctx.empty_packed(tq.TQ_KEY, (B, Hkv, T), device=dev)
    vc = ctx.empty_packed(tq.TQ_VALUE, (B, Hkv, T), device=dev)
    # The cache build's quantize calls of sequences 1.. are timed (sequence 0 warms up).
    qa, qb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    q_ms = 0.0
    for b in range(B):
        K = tq_inputs.outlier_kv(1, Hkv, T, d, seed=1000 + b, device=dev, scale_seed=1)[0]
        V = tq_inputs.outlier_kv(1, Hkv, T, d, seed=2000 + b, device=dev, scale_seed=2)[0]
        if b > 0:
            qa.record()
        ctx.quantize_into(K, tq.TQ_KEY, {k: (None if v is None else v[b]) for k, v in kc.items()})
        ctx.quantize_into(V, tq.TQ_VALUE, {k: (None if v is None else v[b]) for k, v in vc.items()})
        if b > 0:
            qb.record()
            torch.cuda.synchronize()
            q_ms += qa.elapsed_time(qb)
        del K, V
    q = tq_inputs.iid((B, Hq, d), seed=10, device=dev, dtype=torch.bfloat16)
    lens = torch.full((B,), T, dtype=torch.int32, device=dev)
    o = torch.empty(B, Hq, d, dtype=torch.float32, device=dev)
    ws = torch.empty(ctx.attn_workspace_bytes(B, Hq, T), dtype=torch.uint8, device=dev)
    for _ in range(warmup):
        ctx.attn_decode(q, kc, vc, lens, out=o, workspace=ws)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        ctx.attn_decode(q, kc, vc, lens, out=o, workspace=ws)
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    kb, vb = ctx.key_layout["bytes_per_vector"], ctx.value_layout["bytes_per_vector"]
    alg = B * Hkv * T * (kb + vb) + B * Hq * d * 2 + B * Hq * d * 4
    bits_k, bits_v, _, nc = tq.VARIANTS[name]
    res = {"kv_format": f"keys {bits_k} Lloyd-Max bits, values {bits_v} bits, MSE only"
                        f"{', norm-corrected' if nc else ''}{', binary16 norms' if f16 else ''}; "
                        f"{kb + vb} B per token-head",
           "attn_ms": ms, "kv_tokens_per_s": B * T / (ms / 1e3),
           "hbm_frac": alg / (ms / 1e3) / 1e9 / hbm_peak}
    if B > 1 and q_ms > 0:
        res["quantize_mvec_per_s"] = 2 * (B - 1) * Hkv * T / (q_ms / 1e3) / 1e6
        res["quantize_sample"] = (f"cache build of sequences 1..{B - 1}: {Hkv * T} bf16 K and {Hkv * T} "
                                  f"bf16 V vectors per sequence, CUDA events around the quantize calls")
    del g, kc, vc, ws
    ctx.close()
    return res


def small_case(tq, tq_inputs, torch, dev, reps=50):
    """Latency of the smallest workload: quantize 1024 K and 1024 V (fp32,
    d = 128, k3v4), then attention of 8 query heads over them (one kv head)."""
    ctx = tq.Context(128, 3, 4, 128, 0)
    K = tq_inputs.iid((1, 1, 1024, 128), seed=0, device=dev)
    V = tq_inputs.iid((1, 1, 1024, 128), seed=1, device=dev)
    q = tq_inputs.iid((1, 8, 128), seed=2, device=dev)
    kc = ctx.empty_packed(tq.TQ_KEY, (1, 1, 1024), device=dev)
    vc = ctx.empty_packed(tq.TQ_VALUE, (1, 1, 1024), device=dev)
    lens = torch.full((1,), 1024, dtype=torch.int32, device=dev)
    out = torch.empty(1, 8, 128, device=dev)
    ws = torch.empty(ctx.attn_workspace_bytes(1, 8, 1024), dtype=torch.uint8, device=dev)

    def quant():
        ctx.quantize_into(K, tq.TQ_KEY, kc)
        ctx.quantize_into(V, tq.TQ_VALUE, vc)

    def attend():
        ctx.attn_decode(q, kc, vc, lens, out=out, workspace=ws)

    res = {}
    for name, fn in (("quantize_kv_us", quant), ("attn_decode_us", attend)):
        fn()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(10):
                fn()
        g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            g.replay()
        e1.record()
        torch.cuda.synchronize()
        res[name] = e0.elapsed_time(e1) * 1e3 / (reps * 10)
        del g
    ctx.close()
    res["config"] = "1024 K + 1024 V fp32 N(0,1), d=128, k3v4; 8 query heads over one kv head"
    res["timing"] = "CUDA-graph replays of 10 calls, device time per call"
    return res


def run_gpu(args, w):
    import torch
    import torch.distributed as dist
    import compressed_decode_attention_quantize_b200 as tq
    import tq_inputs

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    hbm_peak, peak_src = peaks()

    B, Hq, Hkv, d, T = w["B"], w["Hq"], w["Hkv"], w["d"], w["T"]
    ctx = tq.Context(d, w["bits_k"], w["bits_v"], w["m"], 0)
    # Build the packed cache (setup, not timed): bf16 K/V with outlier channels.
    kc = ctx.empty_packed(tq.TQ_KEY, (B, Hkv, T), device=dev)
    vc = ctx.empty_packed(tq.TQ_VALUE, (B, Hkv, T), device=dev)
    # Inputs of two sampled (sequence, kv head) slices stay on the host for the
    # oracle's code check (tokens below T - 1, which the timed steps rewrite).
    nsample = min(16384, T - 1)
    keep = {(0, 0): None, (B - 1, Hkv - 1): None}
    for b in range(B):
        K = tq_inputs.outlier_kv(1, Hkv, T, d, seed=1000 + b, device=dev, scale_seed=1)[0]
        V = tq_inputs.outlier_kv(1, Hkv, T, d, seed=2000 + b, device=dev, scale_seed=2)[0]
        ctx.quantize_into(K, tq.TQ_KEY, {k: (None if v is None else v[b]) for k, v in kc.items()})
        ctx.quantize_into(V, tq.TQ_VALUE, {k: (None if v is None else v[b]) for k, v in vc.items()})
        for (kb, kh) in keep:
            if kb == b:
                keep[(kb, kh)] = (K[kh, :nsample].float().cpu().numpy(), V[kh, :nsample].float().cpu().numpy())
        del K, V
    torch.cuda.synchronize()
    POOL = 8  # distinct step inputs, reused round-robin
    qs = [tq_inputs.iid((B, Hq, d), seed=10 + i, device=dev, dtype=torch.bfloat16) for i in range(POOL)]
    kn = [tq_inputs.outlier_kv(B, Hkv, 1, d, seed=20 + i, device=dev, scale_seed=1)[:, :, 0].contiguous()
          for i in range(POOL)]
    vn = [tq_inputs.outlier_kv(B, Hkv, 1, d, seed=40 + i, device=dev, scale_seed=2)[:, :, 0].contiguous()
          for i in range(POOL)]
    pos = torch.full((B,), T - 1, dtype=torch.int32, device=dev)
    lens = torch.full((B,), T, dtype=torch.int32, device=dev)
    out = torch.empty(B, Hq, d, dtype=torch.float32, device=dev)
    ws = torch.empty(ctx.attn_workspace_bytes(B, Hq, T), dtype=torch.uint8, device=dev)
    launches_per_step = 3  # append + pre-rotate, attention, merge (tq_decode_step)

    # Each step replays one CUDA graph of tq_decode_step (append the new K/V
    # token at slot T-1, then attend over all T tokens), so host launch latency
    # is not timed.  The attention call alone (pre-rotate + attention + merge,
    # tq_attn_decode) is timed in a second loop over the same inputs, with
    # events around every replay, for the roofline.
    def step_body(j):
        ctx.decode_step(qs[j], kn[j], vn[j], kc, vc, pos, out=out, workspace=ws)

    def attend(j):
        ctx.attn_decode(qs[j], kc, vc, lens, out=out, workspace=ws)

    for j in range(POOL):           # eager warm-up before capture
        step_body(j)
        attend(j)
    torch.cuda.synchronize()
    g_step, g_att = [], []
    for j in range(POOL):
        ga, gb = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(ga):
            step_body(j)
        with torch.cuda.graph(gb):
            attend(j)
        g_step.append(ga)
        g_att.append(gb)
    torch.cuda.synchronize()

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    sampler = ClockSampler(local)
    sampler.start()
    for i in range(args.warmup):
        g_step[i % POOL].replay()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    w0 = time.time()
    torch.cuda.nvtx.range_push("tq:decode_steps")
    e0.record()
    for i in range(args.steps):
        g_step[i % POOL].replay()
    e1.record()
    torch.cuda.nvtx.range_pop()
    barrier()
    sampler.mark(w0, time.time())
    t_ms = e0.elapsed_time(e1) / args.steps

    for i in range(args.warmup):
        g_att[i % POOL].replay()
    barrier()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    w0 = time.time()
    torch.cuda.nvtx.range_push("tq:attention_calls")
    for i in range(args.steps):
        evs[i][0].record()
        g_att[i % POOL].replay()
        evs[i][1].record()
    torch.cuda.nvtx.range_pop()
    barrier()
    sampler.mark(w0, time.time())
    attn_ms = sum(a.elapsed_time(b) for a, b in evs) / args.steps

    # End to end through the public API with host buffers: every step copies
    # its inputs from pinned host memory and reads its output back, inside the
    # timed region.  The copies run on a side stream beside the kernels (two
    # buffer sets): the graph of step j copies step j+1's inputs in and step
    # j-1's output out while step j attends; graphs replay in order, so each
    # buffer is free when it is reused.
    hq = [x.cpu().pin_memory() for x in qs]
    hk = [x.cpu().pin_memory() for x in kn]
    hv = [x.cpu().pin_memory() for x in vn]
    hout = [torch.empty(B, Hq, d, dtype=torch.float32).pin_memory() for _ in range(POOL)]
    dq = [torch.empty_like(qs[0]) for _ in range(2)]
    dk = [torch.empty_like(kn[0]) for _ in range(2)]
    dv = [torch.empty_like(vn[0]) for _ in range(2)]
    dout = [torch.empty(B, Hq, d, dtype=torch.float32, device=dev) for _ in range(2)]
    side = torch.cuda.Stream(device=dev)

    def e2e_body(j):
        cur = torch.cuda.current_stream()
        side.wait_stream(cur)
        with torch.cuda.stream(side):
            n, nb, pb = (j + 1) % POOL, (j + 1) % 2, (j - 1) % 2
            dq[nb].copy_(hq[n], non_blocking=True)
            dk[nb].copy_(hk[n], non_blocking=True)
            dv[nb].copy_(hv[n], non_blocking=True)
            hout[(j - 1) % POOL].copy_(dout[pb], non_blocking=True)
        ctx.decode_step(dq[j % 2], dk[j % 2], dv[j % 2], kc, vc, pos, out=dout[j % 2], workspace=ws)
        cur.wait_stream(side)

    dq[0].copy_(hq[0])
    dk[0].copy_(hk[0])
    dv[0].copy_(hv[0])
    torch.cuda.synchronize()
    g_e2e = []
    for j in range(POOL):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            e2e_body(j)
        g_e2e.append(g)
    for i in range(args.warmup):
        g_e2e[i % POOL].replay()
    barrier()
    w0 = time.time()
    e0.record()
    for i in range(args.warmup, args.warmup + args.steps):
        g_e2e[i % POOL].replay()
    last = args.warmup + args.steps - 1
    hout[last % POOL].copy_(dout[last % 2], non_blocking=True)   # the last step's output
    e1.record()
    barrier()
    sampler.mark(w0, time.time())
    e2e_ms = e0.elapsed_time(e1) / args.steps
    h2d = hq[0].numel() * hq[0].element_size() + 2 * hk[0].numel() * hk[0].element_size()
    d2h = hout[0].numel() * hout[0].element_size()
    del g_step, g_att, g_e2e

    torch.cuda.nvtx.range_push("tq:quantize_sweep")
    quant = quantize_sweep(tq, tq_inputs, torch, dev, hbm_peak)
    torch.cuda.nvtx.range_pop()
    clocks = sampler.stop()
    vsearch = small = variants = d70 = None
    if not args.skip_extra:
        torch.cuda.nvtx.range_push("tq:vector_search")
        vsearch = vector_search(tq, tq_inputs, torch, dev, clocks.get("sm_max_mhz") or 1965.0)
        torch.cuda.nvtx.range_pop()
        small = small_case(tq, tq_inputs, torch, dev)
        variants = variant_decode(tq, tq_inputs, torch, dev, hbm_peak, WORKLOADS["llama3-8b-decode"])
        d70 = decode_70b(tq, tq_inputs, torch, dev, hbm_peak)

    t_ms, attn_ms, e2e_ms = max_over_ranks([t_ms, attn_ms, e2e_ms], world, dev)

    cpu = parity = None
    if rank == 0 and world == 1:
        ctx.attn_decode(qs[0], kc, vc, lens, out=out, workspace=ws)
        gpu_out = out.cpu().numpy()
        cpu, attn_parity = cpu_baseline_from_device(w, ctx, kc, vc, qs[0], gpu_out)
        parity = code_parity(w, kc, vc, keep)
        parity["attention"] = attn_parity

    if rank == 0:
        kvb = kv_bytes(w, ctx)
        alg = kvb + B * Hq * d * 2 + B * Hq * d * 4  # packed cache + bf16 queries + fp32 output
        achieved = alg / (attn_ms / 1e3) / 1e9
        traffic = recorded_traffic(args.workload)
        line = {
            "metric": METRIC, "value": whole_job_rate(B * T, world, t_ms), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": t_ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": "int8 key-bit x 4-limb query MMA + fp16 value MMA, fp32 accumulate and softmax",
            "data": "synthetic",
            "config": config_of(args, w),
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                         "frac": achieved / hbm_peak, "traffic": traffic,
                         "kernel": "tq_attn_decode (pre-rotate + split-K attention + merge), "
                                   "timed in its own loop of K graph replays",
                         "algorithmic_bytes_per_launch": alg, "launch_ms": attn_ms,
                         "peak_source": f"{peak_src} hbm_gbs (copy bandwidth)",
                         "frac_of_nominal_8tbs": achieved / 8000.0},
            "e2e": {"value": whole_job_rate(B * T, world, e2e_ms), "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                    "copies": "pinned host <-> device on a side stream, overlapped with the previous / next "
                              "step's kernels (two buffer sets), all inside the timed region"},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clocks,
            "quantize": quant,
        }
        if vsearch is not None:
            line["vector_search"] = vsearch
            line["small_case"] = small
            line["format_variants_decode"] = variants
            line["decode_70b"] = d70
        if cpu is not None:
            line["cpu_baseline"] = cpu
            line["parity"] = parity
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_case(args):
    """One library call on a synthetic case, repeated (for profilers: a small
    case of one kernel).  Prints the mean CUDA-event time per call and the
    algorithmic bytes per call."""
    import torch
    import compressed_decode_attention_quantize_b200 as tq
    import tq_inputs

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(args.steps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / args.steps

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    if args.case == "decode":
        w = dict(WORKLOADS[args.workload])
        for k in ("B", "T"):
            if getattr(args, k) is not None:
                w[k] = getattr(args, k)
        B, Hq, Hkv, d, T = w["B"], w["Hq"], w["Hkv"], w["d"], w["T"]
        ctx = tq.Context(d, w["bits_k"], w["bits_v"], w["m"], 0)
        kc = ctx.empty_packed(tq.TQ_KEY, (B, Hkv, T), device=dev)
        vc = ctx.empty_packed(tq.TQ_VALUE, (B, Hkv, T), device=dev)
        for b in range(B):
            K = tq_inputs.outlier_kv(1, Hkv, T, d, seed=1000 + b, device=dev, scale_seed=1)[0]
            V = tq_inputs.outlier_kv(1, Hkv, T, d, seed=2000 + b, device=dev, scale_seed=2)[0]
            ctx.quantize_into(K, tq.TQ_KEY, {k: (None if v is None else v[b]) for k, v in kc.items()})
            ctx.quantize_into(V, tq.TQ_VALUE, {k: (None if v is None else v[b]) for k, v in vc.items()})
            del K, V
        q = tq_inputs.iid((B, Hq, d), seed=10, device=dev, dtype=torch.bfloat16)
        lens = torch.full((B,), T, dtype=torch.int32, device=dev)
        out = torch.empty(B, Hq, d, device=dev)
        ws = torch.empty(ctx.attn_workspace_bytes(B, Hq, T), dtype=torch.uint8, device=dev)
        ms = timed(lambda: ctx.attn_decode(q, kc, vc, lens, out=out, workspace=ws))
        byts = kv_bytes(w, ctx)
        desc = f"{args.workload} B={B} T={T}"
    elif args.case == "quantize":
        n = args.n or (1 << 20)
        m = args.d if args.qjl else 0
        ctx = tq.Context(args.d, args.bits, args.bits, m, 0)
        if args.d == 128:
            X = tq_inputs.outlier_kv(1, 8, n // 8, args.d, seed=31, device=dev)[0].reshape(-1, args.d)
        else:
            X = tq_inputs.mixture(n, args.d, seed=21, device=dev)
        pk = ctx.empty_packed(tq.TQ_KEY, (X.shape[0],), device=dev)
        ms = timed(lambda: ctx.quantize_into(X, tq.TQ_KEY, pk))
        byts = X.shape[0] * (args.d * X.element_size() + ctx.key_layout["bytes_per_vector"])
        desc = f"n={X.shape[0]} d={args.d} bits={args.bits} qjl={args.qjl}"
    else:
        s = VSEARCH
        n = args.n or s["n"]
        ctx = tq.Context(s["d"], s["bits_k"], 3, s["m"], 0)
        X = tq_inputs.mixture(n, s["d"], seed=21, device=dev)
        Q = tq_inputs.mixture(args.nq, s["d"], seed=22, means_seed=21, device=dev)
        db = ctx.quantize(X, tq.TQ_KEY)
        ws = torch.empty(ctx.topk_workspace_bytes(args.nq, n, s["k"]), dtype=torch.uint8, device=dev)
        ms = timed(lambda: ctx.topk(Q, db, s["k"], workspace=ws))
        byts = n * ctx.key_layout["bytes_per_vector"]
        desc = f"n={n} nq={args.nq} d={s['d']} k={s['k']}"
    print(json.dumps({"case": args.case, "config": desc, "ms_per_call": ms, "bytes_per_call": byts,
                      "gbs": byts / (ms / 1e3) / 1e9}), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=int(os.environ.get("WORLD_SIZE", "1")))
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="llama3-8b-decode", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="tq", choices=["tq", "reference"])
    ap.add_argument("--skip-extra", dest="skip_extra", action="store_true",
                    help="omit the vector-search and small-case measurements")
    ap.add_argument("--case", choices=["decode", "quantize", "topk"],
                    help="profiling case: one library call repeated (--steps times after --warmup), "
                         "no JSON bench line")
    ap.add_argument("--B", type=int, help="--case decode: batch (default: the workload's)")
    ap.add_argument("--T", type=int, help="--case decode: context (default: the workload's)")
    ap.add_argument("--n", type=int, help="--case quantize / topk: vectors")
    ap.add_argument("--nq", type=int, default=1000, help="--case topk: queries")
    ap.add_argument("--d", type=int, default=128, help="--case quantize: dimension")
    ap.add_argument("--bits", type=int, default=3, help="--case quantize: bits (keys count the QJL bit)")
    ap.add_argument("--qjl", type=int, default=1, help="--case quantize: QJL stage (m = d) on/off")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    w = WORKLOADS[args.workload]
    if args.case:
        return run_case(args)
    if args.impl == "reference":
        return run_reference(args, w)
    return run_gpu(args, w)


if __name__ == "__main__":
    sys.exit(main())
