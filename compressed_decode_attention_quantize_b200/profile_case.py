"""Run one libtq operation on a synthetic case a few times (for profilers).

  python -m compressed_decode_attention_quantize_b200.profile_case decode --B 4 --T 32768
  python -m compressed_decode_attention_quantize_b200.profile_case quantize --n 1048576 --bits 3
  python -m compressed_decode_attention_quantize_b200.profile_case topk --n 1000000 --nq 1000

Prints the mean CUDA-event time per call and the algorithmic bytes per call.
"""
from __future__ import annotations

import argparse
import json
import sys
from pathlib import Path

import torch

sys.path.insert(0, str(Path(__file__).resolve().parent.parent))

import compressed_decode_attention_quantize_b200 as tq  # noqa: E402
import tq_inputs  # noqa: E402


def timed(fn, iters, warmup):
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(iters):
        fn()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / iters


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("op", choices=["decode", "quantize", "topk"])
    ap.add_argument("--B", type=int, default=4)
    ap.add_argument("--Hq", type=int, default=32)
    ap.add_argument("--Hkv", type=int, default=8)
    ap.add_argument("--T", type=int, default=32768)
    ap.add_argument("--d", type=int, default=128)
    ap.add_argument("--bits_k", type=int, default=3)
    ap.add_argument("--bits_v", type=int, default=4)
    ap.add_argument("--m", type=int, default=128)
    ap.add_argument("--n", type=int, default=1 << 20)
    ap.add_argument("--nq", type=int, default=1000)
    ap.add_argument("--bits", type=int, default=3)
    ap.add_argument("--qjl", type=int, default=1)
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=3)
    a = ap.parse_args()
    dev = torch.device("cuda", 0)
    if a.op == "decode":
        ctx = tq.Context(a.d, a.bits_k, a.bits_v, a.m, 0)
        kc = ctx.empty_packed(tq.TQ_KEY, (a.B, a.Hkv, a.T), device=dev)
        vc = ctx.empty_packed(tq.TQ_VALUE, (a.B, a.Hkv, a.T), device=dev)
        for b in range(a.B):
            K = tq_inputs.outlier_kv(1, a.Hkv, a.T, a.d, seed=1000 + b, device=dev, scale_seed=1)[0]
            V = tq_inputs.outlier_kv(1, a.Hkv, a.T, a.d, seed=2000 + b, device=dev, scale_seed=2)[0]
            ctx.quantize_into(K, tq.TQ_KEY, {k: (None if v is None else v[b]) for k, v in kc.items()})
            ctx.quantize_into(V, tq.TQ_VALUE, {k: (None if v is None else v[b]) for k, v in vc.items()})
            del K, V
        q = tq_inputs.iid((a.B, a.Hq, a.d), seed=10, device=dev, dtype=torch.bfloat16)
        lens = torch.full((a.B,), a.T, dtype=torch.int32, device=dev)
        out = torch.empty(a.B, a.Hq, a.d, device=dev)
        ws = torch.empty(ctx.attn_workspace_bytes(a.B, a.Hq, a.T), dtype=torch.uint8, device=dev)
        ms = timed(lambda: ctx.attn_decode(q, kc, vc, lens, out=out, workspace=ws), a.iters, a.warmup)
        byts = a.B * a.Hkv * a.T * (ctx.key_layout["bytes_per_vector"] + ctx.value_layout["bytes_per_vector"])
    elif a.op == "quantize":
        m = a.d if a.qjl else 0
        ctx = tq.Context(a.d, a.bits, a.bits, m, 0)
        X = tq_inputs.outlier_kv(1, 8, a.n // 8, a.d, seed=31, device=dev)[0].reshape(-1, a.d)
        pk = ctx.empty_packed(tq.TQ_KEY, (X.shape[0],), device=dev)
        ms = timed(lambda: ctx.quantize_into(X, tq.TQ_KEY, pk), a.iters, a.warmup)
        byts = X.shape[0] * (a.d * 2 + ctx.key_layout["bytes_per_vector"])
    else:
        ctx = tq.Context(a.d if a.d != 128 else 200, 4, 3, a.d if a.d != 128 else 200, 0)
        dd = ctx.d
        X = tq_inputs.mixture(a.n, dd, seed=21, device=dev)
        Q = tq_inputs.mixture(a.nq, dd, seed=22, means_seed=21, device=dev)
        db = ctx.quantize(X, tq.TQ_KEY)
        ws = torch.empty(ctx.topk_workspace_bytes(a.nq, a.n, 10), dtype=torch.uint8, device=dev)
        ms = timed(lambda: ctx.topk(Q, db, 10, workspace=ws), a.iters, a.warmup)
        byts = a.n * ctx.key_layout["bytes_per_vector"]
    print(json.dumps({"op": a.op, "ms_per_call": ms, "bytes_per_call": byts,
                      "gbs": byts / (ms / 1e3) / 1e9}))


if __name__ == "__main__":
    main()
