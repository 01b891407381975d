"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module holds no part of the quantization or attention arithmetic: it only
draws random tensors with the shapes and value distributions of the workloads.
Generation runs on the device the caller names (torch's generator for that
device), so the same call on CPU and on CUDA gives different, but each
reproducible, numbers; a comparison always hands both sides copies of the same
tensor.

Recipes:
  iid         N(0,1) entries (single-head cases).
  outlier_kv  K/V shaped [B, H, T, d]: N(0,1) entries times a per-(head,
              channel) scale exp(N(0,1)); each (head, channel) is an outlier
              channel with probability 0.01 and then scaled by 20 more;
              rounded to bf16.  This stands in for LLM K/V activations with
              heavy channels, the workload of the vLLM study of TurboQuant.
  mixture     unit-norm points of a Gaussian mixture: `components` means drawn
              N(0, I_d), points = mean + 0.5 N(0, I_d), uniform weights, then
              normalised; a stand-in for the GloVe d=200 vector-search set.
"""
from __future__ import annotations

import torch


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def iid(shape, seed: int, device="cpu", dtype=torch.float32) -> torch.Tensor:
    g = _gen(seed, device)
    return torch.randn(*shape, generator=g, device=device, dtype=torch.float32).to(dtype)


def outlier_kv(B: int, H: int, T: int, d: int, seed: int, device="cpu",
               outlier_p: float = 0.01, outlier_scale: float = 20.0,
               scale_seed: int | None = None) -> torch.Tensor:
    """`scale_seed` fixes the per-(head, channel) scales independently of
    `seed`, so that several calls (e.g. one per sequence) share them."""
    g = _gen(seed, device)
    gs = g if scale_seed is None else _gen(scale_seed, device)
    scale = torch.exp(torch.randn(H, d, generator=gs, device=device))
    heavy = torch.rand(H, d, generator=gs, device=device) < outlier_p
    scale = torch.where(heavy, scale * outlier_scale, scale)
    out = torch.empty(B, H, T, d, device=device, dtype=torch.bfloat16)
    # Draw per (b, h) slice to bound the fp32 temporary.
    for b in range(B):
        for h in range(H):
            x = torch.randn(T, d, generator=g, device=device)
            out[b, h] = (x * scale[h]).to(torch.bfloat16)
    return out


def mixture(n: int, d: int, seed: int, components: int = 256, spread: float = 0.5,
            device="cpu", means_seed: int | None = None, chunk: int = 1 << 18) -> torch.Tensor:
    """Unit-norm mixture points.  `means_seed` fixes the component means so
    that a database and its queries share them while the points differ."""
    gm = _gen(seed if means_seed is None else means_seed, device)
    means = torch.randn(components, d, generator=gm, device=device)
    g = _gen(seed + 0x5EED, device)
    out = torch.empty(n, d, device=device, dtype=torch.float32)
    for s in range(0, n, chunk):
        e = min(n, s + chunk)
        comp = torch.randint(0, components, (e - s,), generator=g, device=device)
        x = means[comp] + spread * torch.randn(e - s, d, generator=g, device=device)
        out[s:e] = x / torch.linalg.vector_norm(x, dim=1, keepdim=True)
    return out


def seq_lens(B: int, max_T: int, seed: int, mode: str = "full") -> torch.Tensor:
    """Per-sequence lengths: 'full' = all max_T; 'ragged' = uniform in [1, max_T]
    with the first sequence empty and the last full (edge cases)."""
    if mode == "full":
        return torch.full((B,), max_T, dtype=torch.int32)
    g = _gen(seed, "cpu")
    lens = torch.randint(1, max_T + 1, (B,), generator=g, dtype=torch.int32)
    if B > 1:
        lens[0] = 0
        lens[-1] = max_T
    return lens
