"""Decode attention through tq_attn_decode_static, the entry point for callers
that cannot allocate device memory on the call path (its scratch is a static
device array inside the library).  Its output must match tq_attn_decode with
a caller workspace, on two calls in a row (the shared scratch keeps the
previous call's contents).  Kept in a file of its own that runs last."""
import numpy as np
import pytest
import torch

import compressed_decode_attention_quantize_b200 as tq
import tq_inputs

pytestmark = pytest.mark.gpu

ATTN_RTOL = 2e-3  # relative L2 per (sequence, head), as in the oracle parity tests


def _rel(a, b):
    a, b = a.double().cpu().numpy(), b.double().cpu().numpy()
    num = np.linalg.norm(a - b, axis=-1)
    den = np.linalg.norm(b, axis=-1)
    return np.where(den > 0, num / np.where(den > 0, den, 1), num)


@pytest.mark.parametrize("d,bk,bv,m,Hq,Hkv,T", [(128, 3, 4, 128, 8, 2, 700), (64, 2, 2, 0, 4, 4, 333)])
def test_static_scratch_matches_workspace_path(cuda, d, bk, bv, m, Hq, Hkv, T):
    c = tq.Context(d, bk, bv, m, 3)
    B = 3
    K = tq_inputs.outlier_kv(B, Hkv, T, d, seed=5).to(cuda)
    V = tq_inputs.outlier_kv(B, Hkv, T, d, seed=6).to(cuda)
    kc, vc = c.quantize(K, tq.TQ_KEY), c.quantize(V, tq.TQ_VALUE)
    lens = torch.tensor([T, 1, T // 2], dtype=torch.int32, device=cuda)
    q1 = tq_inputs.iid((B, Hq, d), seed=7, device=cuda)
    q2 = tq_inputs.iid((B, Hq, d), seed=8, device=cuda)
    ref1 = c.attn_decode(q1, kc, vc, lens)
    ref2 = c.attn_decode(q2, kc, vc, lens)
    got1 = c.attn_decode_static(q1, kc, vc, lens)
    got2 = c.attn_decode_static(q2, kc, vc, lens)
    torch.cuda.synchronize()
    assert np.all(_rel(got1, ref1) <= ATTN_RTOL)
    assert np.all(_rel(got2, ref2) <= ATTN_RTOL)


def test_static_scratch_rejects_oversized(cuda):
    c = tq.Context(128, 3, 4, 128, 0)
    limit = tq._lib.tq_attn_static_scratch_bytes()
    assert limit == 32 << 20
    B, Hq, Hkv, T = 64, 64, 8, 131072
    assert c.attn_workspace_bytes(B, Hq, T) > limit
    # The size check comes before any launch, so placeholder arrays suffice.
    tiny_i = torch.empty(1, dtype=torch.int32, device=cuda)
    norms = torch.empty(1, device=cuda).expand(B, Hkv, T)
    kc = {"codes": tiny_i, "qjl": tiny_i, "norm": norms, "rnorm": norms}
    vc = {"codes": tiny_i, "norm": norms}
    with pytest.raises(tq.TQError) as e:
        c.attn_decode_static(torch.zeros(B, Hq, 128, device=cuda), kc, vc,
                             torch.full((B,), T, dtype=torch.int32, device=cuda))
    assert e.value.status == tq.TQ_ERR_WORKSPACE
