"""CUDA path vs the fp64 oracle, through the C ABI (libtq via its binding).

Small cases run the oracle on every output; the full-size workloads (decode
attention shaped like Llama-3-8B and a 70B model, the vector-search top-k)
check sampled outputs.  Rules are in tests/_parity.py."""
import math

import numpy as np
import pytest
import torch

import compressed_decode_attention_quantize_b200 as tq
import tq_inputs
from oracle import tq_oracle as o
import _parity as P

pytestmark = pytest.mark.gpu


def _ctx(d, bk, bv, m, seed=0):
    return tq.Context(d, bk, bv, m, seed)


def _flat(p, n):
    return {k: (None if v is None else v.reshape(n, -1) if v.ndim > 1 else v) for k, v in P.packed_np(p).items()}


# --- layout and tables ------------------------------------------------------
def test_layout_bytes(cuda):
    c = _ctx(128, 3, 4, 128)
    assert c.key_layout["bytes_per_vector"] == 56      # 2-bit fields 32 B + 16 B QJL + |k| + gamma
    assert c.value_layout["bytes_per_vector"] == 68    # 4-bit fields 64 B + |v|
    c2 = _ctx(200, 4, 3, 200)
    assert c2.key_layout["words"] == 13 + 7 and c2.key_layout["qjl_words"] == 7  # 3-bit: 2-bit + 1-bit streams


def test_device_context_tables_match_oracle(cuda):
    c = _ctx(128, 3, 4, 128, seed=42)
    t = c.tables()
    ot = o.make_tables(128, 3, 4, 128, 42)
    assert np.abs(t["Pi"] - ot.Pi).max() < 1e-12
    assert np.array_equal(t["S"], ot.S)
    assert np.abs(t["ck"] - ot.cb_k.centroids).max() < 1e-12
    assert np.abs(t["cv"] - ot.cb_v.centroids).max() < 1e-12


# --- quantize ------------------------------------------------------------------
def test_quantize_single_head_fp32(cuda):
    """1024 keys + 1024 values, d=128, fp32 N(0,1), seed 0; k3 (2+1, m=128), v4."""
    c = _ctx(128, 3, 4, 128, seed=0)
    tab = P.oracle_tables(c)
    K = tq_inputs.iid((1024, 128), seed=0)
    V = tq_inputs.iid((1024, 128), seed=1)
    pk = c.quantize(K.to(cuda), tq.TQ_KEY)
    pv = c.quantize(V.to(cuda), tq.TQ_VALUE)
    torch.cuda.synchronize()
    P.check_quantized(tab, "k", K.double().numpy(), _flat(pk, 1024))
    P.check_quantized(tab, "v", V.double().numpy(), _flat(pv, 1024))


@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("qjl", [True, False])
def test_quantize_bit_sweep_outlier_bf16(cuda, bits, qjl):
    """Prefill-style quantization sweep on bf16 K/V with outlier channels
    (8 heads x 1031 tokens, a ragged count)."""
    m = 128 if qjl else 0
    c = _ctx(128, bits, bits, m, seed=3)
    tab = P.oracle_tables(c)
    X = tq_inputs.outlier_kv(1, 8, 1031, 128, seed=bits * 10 + qjl)[0].reshape(-1, 128)
    n = X.shape[0]
    pk = c.quantize(X.to(cuda), tq.TQ_KEY)
    pv = c.quantize(X.to(cuda), tq.TQ_VALUE)
    torch.cuda.synchronize()
    x = X.double().numpy()
    P.check_quantized(tab, "k", x, _flat(pk, n))
    P.check_quantized(tab, "v", x, _flat(pv, n))


@pytest.mark.parametrize("bits,qjl", [(3, True), (4, False)])
def test_quantize_prefill_full_size_sampled(cuda, bits, qjl):
    """The bench's quantize launch at full size: 131072 tokens x 8 kv heads of
    bf16 K (1,048,576 vectors, the tensor-core path), the oracle on 6144
    sampled vectors (first, middle and last 2048)."""
    m = 128 if qjl else 0
    c = _ctx(128, bits, bits, m, seed=12)
    tab = P.oracle_tables(c)
    X = tq_inputs.outlier_kv(1, 8, 131072, 128, seed=90 + bits, device=cuda)[0].reshape(-1, 128)
    n = X.shape[0]
    pk = c.quantize(X, tq.TQ_KEY)
    torch.cuda.synchronize()
    for s0 in (0, n // 2 - 1024, n - 2048):
        sl = slice(s0, s0 + 2048)
        P.check_quantized(tab, "k", P.to_np(X[sl]), _flat({k: (None if v is None else v[sl]) for k, v in pk.items()}, 2048))
    del X, pk
    torch.cuda.empty_cache()


def test_quantize_d200_mixture(cuda):
    """d=200 (7 words per plane), 3-bit Lloyd-Max + QJL with m=200, unit-norm mixture."""
    c = _ctx(200, 4, 3, 200, seed=5)
    tab = P.oracle_tables(c)
    X = tq_inputs.mixture(3000, 200, seed=1)
    pk = c.quantize(X.to(cuda), tq.TQ_KEY)
    torch.cuda.synchronize()
    P.check_quantized(tab, "k", X.double().numpy(), _flat(pk, 3000))


def test_quantize_edge_cases(cuda):
    c = _ctx(64, 3, 2, 64, seed=8)
    tab = P.oracle_tables(c)
    # n = 0 is a no-op
    empty = torch.empty(0, 64, device=cuda)
    c.quantize(empty, tq.TQ_KEY)
    # zero vectors, a single vector, fp16 input, and a strided (ld > d) view
    X = tq_inputs.iid((37, 64), seed=4)
    X[0] = 0
    X[5] = 0
    big = torch.zeros(37, 80)
    big[:, :64] = X
    for src in (X.to(cuda), X.half().to(cuda), big.to(cuda)[:, :64]):
        pk = c.quantize(src, tq.TQ_KEY) if src.stride(0) == 64 else None
        if pk is None:
            pk = c.empty_packed(tq.TQ_KEY, (37,))
            c.quantize_into(src, tq.TQ_KEY, pk)
        torch.cuda.synchronize()
        x = src.double().cpu().numpy()
        P.check_quantized(tab, "k", x, _flat(pk, 37))
        g = P.packed_np(pk)
        assert g["norm"][0] == 0 and g["rnorm"][0] == 0
        assert np.all(o.unpack_codes(g["codes"][0], 2, 64) == 2)


# --- dequantize / logits ---------------------------------------------------------
def test_dequantize_matches_oracle(cuda):
    c = _ctx(128, 3, 4, 128, seed=0)
    tab = P.oracle_tables(c)
    K = tq_inputs.iid((500, 128), seed=2) * 3
    for which, wch in ((tq.TQ_KEY, "k"), (tq.TQ_VALUE, "v")):
        p = c.quantize(K.to(cuda), which)
        xh = c.dequantize(which, p)
        torch.cuda.synchronize()
        g = _flat(p, 500)
        ref = o.dequantize(tab, wch, g["codes"], g["norm"], g["qjl"], g["rnorm"])
        err = np.linalg.norm(xh.cpu().double().numpy() - ref, axis=1) / np.linalg.norm(ref, axis=1)
        assert err.max() < 1e-5


def test_logits_single_head(cuda):
    """Logits of 8 N(0,1) queries against the 1024 packed keys, from codes."""
    c = _ctx(128, 3, 4, 128, seed=0)
    tab = P.oracle_tables(c)
    K = tq_inputs.iid((1024, 128), seed=0)
    Q = tq_inputs.iid((8, 128), seed=2)
    pk = c.quantize(K.to(cuda), tq.TQ_KEY)
    lg = c.logits(Q.to(cuda), pk)
    torch.cuda.synchronize()
    P.check_logits(tab, Q.double().numpy(), _flat(pk, 1024), lg.cpu().double().numpy())


# --- decode attention ---------------------------------------------------------
def _cache(c, K, V, cuda):
    return c.quantize(K.to(cuda), tq.TQ_KEY), c.quantize(V.to(cuda), tq.TQ_VALUE)


def test_attention_single_head(cuda):
    """8 queries over 1024 keys/values of one KV head (softmax . V)."""
    c = _ctx(128, 3, 4, 128, seed=0)
    tab = P.oracle_tables(c)
    K = tq_inputs.iid((1, 1, 1024, 128), seed=0)
    V = tq_inputs.iid((1, 1, 1024, 128), seed=1)
    Q = tq_inputs.iid((1, 8, 128), seed=2)
    kc, vc = _cache(c, K, V, cuda)
    lens = torch.tensor([1024], dtype=torch.int32)
    out = c.attn_decode(Q.to(cuda), kc, vc, lens.to(cuda))
    torch.cuda.synchronize()
    P.check_attention(tab, Q.double().numpy(), P.packed_np(kc), P.packed_np(vc), lens.numpy(), 1,
                      out.cpu().numpy())


@pytest.mark.parametrize("d,Hq,Hkv,bk,bv,m,T", [
    (128, 8, 2, 3, 4, 128, 1100),   # tensor-core path, group 4
    (128, 4, 4, 3, 4, 128, 1100),   # tensor-core path, group 1
    (128, 4, 2, 3, 4, 128, 1100),   # tensor-core path, group 2
    (128, 16, 2, 3, 4, 128, 1100),  # tensor-core path, group 8
    (128, 8, 2, 3, 4, 128, 1002),   # max_T % 4 != 0: generic path
    (128, 16, 2, 4, 4, 128, 1000),  # 3-bit keys: tensor-core path, group 8
    (128, 8, 2, 4, 4, 128, 1000),   # 3-bit keys: tensor-core path, group 4
    (128, 8, 2, 4, 4, 128, 998),    # 3-bit keys, max_T % 4 != 0: generic path
    (128, 4, 4, 4, 4, 128, 1000),   # 3-bit keys, group 1: tensor-core path
    (128, 4, 2, 4, 4, 128, 1000),   # 3-bit keys, group 2: tensor-core path
    (200, 6, 3, 4, 3, 200, 1000), (64, 4, 4, 2, 2, 0, 1000),
    (128, 8, 2, 8, 4, 0, 1000),     # 8-bit keys (k8v4): tensor-core path, group 4
    (128, 16, 2, 8, 4, 0, 998),     # 8-bit keys, max_T % 4 != 0: generic path
    (256, 4, 2, 8, 8, 0, 300)])     # 8-bit keys and values at d = 256 (64 code words)
def test_attention_ragged_outlier(cuda, d, Hq, Hkv, bk, bv, m, T):
    """Ragged lengths (0, 1, odd, chunk edges, full), GQA groups 1-8, d=64/128/200."""
    c = _ctx(d, bk, bv, m, seed=7)
    tab = P.oracle_tables(c)
    B = 6
    K = tq_inputs.outlier_kv(B, Hkv, T, d, seed=1)
    V = tq_inputs.outlier_kv(B, Hkv, T, d, seed=2)
    Q = tq_inputs.iid((B, Hq, d), seed=3, dtype=torch.bfloat16)
    kc, vc = _cache(c, K, V, cuda)
    lens = torch.tensor([0, 1, 129, 513, 777, T], dtype=torch.int32)
    out = c.attn_decode(Q.to(cuda), kc, vc, lens.to(cuda))
    torch.cuda.synchronize()
    P.check_attention(tab, Q.double().numpy(), P.packed_np(kc), P.packed_np(vc), lens.numpy(), Hkv,
                      out.cpu().numpy())


@pytest.mark.parametrize("Hq,Hkv,lens_kind,bk", [
    (8, 2, "mixed", 3), (16, 2, "mixed", 3), (4, 4, "mixed", 3), (2, 1, "mixed", 3),
    (8, 2, "tiny", 3), (16, 2, "tiny", 3), (16, 2, "mixed", 4), (16, 2, "tiny", 4)])
def test_attention_many_short_rows(cuda, Hq, Hkv, lens_kind, bk):
    """Tensor-core paths with many short sequences: the balanced tile ranges
    cross many (sequence, kv head) rows, and with tiny lengths there are
    fewer tiles than warps."""
    c = _ctx(128, bk, 4, 128, seed=5)
    tab = P.oracle_tables(c)
    B, T = 37, 256
    g = torch.Generator().manual_seed(11)
    if lens_kind == "mixed":
        lens = torch.randint(0, T + 1, (B,), generator=g, dtype=torch.int32)
        lens[:4] = torch.tensor([0, T, 16, 17], dtype=torch.int32)
    else:
        lens = torch.randint(0, 3, (B,), generator=g, dtype=torch.int32)
    K = tq_inputs.outlier_kv(B, Hkv, T, 128, seed=21)
    V = tq_inputs.outlier_kv(B, Hkv, T, 128, seed=22)
    Q = tq_inputs.iid((B, Hq, 128), seed=23, dtype=torch.bfloat16)
    kc, vc = _cache(c, K, V, cuda)
    out = c.attn_decode(Q.to(cuda), kc, vc, lens.to(cuda))
    torch.cuda.synchronize()
    P.check_attention(tab, Q.double().numpy(), P.packed_np(kc), P.packed_np(vc), lens.numpy(), Hkv,
                      out.cpu().numpy())


def _slice_pairs(kc, vc, pairs, Hq, Hkv):
    """Host copies of the (b, kv-head) slices the sampled (b, h) pairs read."""
    G = Hq // Hkv
    out = []
    for b, h in pairs:
        g = h // G
        sl = lambda t: None if t is None else P.to_np(t[b:b + 1, g:g + 1])
        out.append(({k: sl(v) for k, v in kc.items()}, {k: sl(v) for k, v in vc.items()}))
    return out


def _full_size(cuda, B, Hq, Hkv, T, bk, bv, pairs, seed):
    c = _ctx(128, bk, bv, 128, seed=0)
    tab = P.oracle_tables(c)
    K = tq_inputs.outlier_kv(B, Hkv, T, 128, seed=seed, device=cuda)
    V = tq_inputs.outlier_kv(B, Hkv, T, 128, seed=seed + 1, device=cuda)
    Q = tq_inputs.iid((B, Hq, 128), seed=seed + 2, device=cuda, dtype=torch.bfloat16)
    kc, vc = c.quantize(K, tq.TQ_KEY), c.quantize(V, tq.TQ_VALUE)
    # quantize parity on one sampled slice of each
    n = 4096
    P.check_quantized(tab, "k", P.to_np(K[0, 0, :n]), _flat({k: (None if v is None else v[0, 0, :n]) for k, v in kc.items()}, n))
    P.check_quantized(tab, "v", P.to_np(V[B - 1, Hkv - 1, -n:]), _flat({k: (None if v is None else v[B - 1, Hkv - 1, -n:]) for k, v in vc.items()}, n))
    del K, V
    lens = torch.full((B,), T, dtype=torch.int32, device=cuda)
    out = c.attn_decode(Q, kc, vc, lens)
    torch.cuda.synchronize()
    qn = P.to_np(Q)
    G = Hq // Hkv
    for (b, h), (ks, vs) in zip(pairs, _slice_pairs(kc, vc, pairs, Hq, Hkv)):
        P.check_attention(tab, qn[b:b + 1, h:h + 1], ks, vs, np.array([T]), 1,
                          P.to_np(out[b:b + 1, h:h + 1]))
    del kc, vc
    torch.cuda.empty_cache()


def test_attention_llama8b_shape_sampled(cuda):
    """B=16, Hq=32, Hkv=8 (GQA 4), d=128, T=32768, bf16 outlier K/V, k3v4."""
    _full_size(cuda, 16, 32, 8, 32768, 3, 4, [(0, 0), (7, 13), (15, 31)], seed=100)


@pytest.mark.parametrize("bk", [3, 4])
def test_attention_70b_shape_sampled(cuda, bk):
    """B=4, Hq=64, Hkv=8 (GQA 8), d=128, T=131072, bf16 outlier K/V, k3v4 / k4v4."""
    _full_size(cuda, 4, 64, 8, 131072, bk, 4, [(0, 5), (3, 63)], seed=200 + bk)


# --- top-k --------------------------------------------------------------------
def _oracle_topk_chunked(tab, q, g, k, chunk=25_000):
    n = g["norm"].size
    best_v = np.full((q.shape[0], 0), -np.inf)
    best_i = np.zeros((q.shape[0], 0), dtype=np.int64)
    for s in range(0, n, chunk):
        e = min(n, s + chunk)
        qj = None if g["qjl"] is None else g["qjl"][s:e].reshape(e - s, -1)
        rn = None if g["rnorm"] is None else g["rnorm"][s:e]
        sc = o.logits(tab, q, g["codes"][s:e], g["norm"][s:e], qj, rn)
        best_v = np.concatenate([best_v, sc], axis=1)
        best_i = np.concatenate([best_i, np.broadcast_to(np.arange(s, e), sc.shape)], axis=1)
        order = np.lexsort((best_i, -best_v), axis=1)[:, :k]
        best_v = np.take_along_axis(best_v, order, 1)
        best_i = np.take_along_axis(best_i, order, 1)
    return best_i, best_v


def _check_topk(tab, q, g, idx, score, k):
    ref_i, ref_v = _oracle_topk_chunked(tab, q, g, k)
    qn = np.linalg.norm(q, axis=1)
    for r in range(q.shape[0]):
        tol = P.LOGIT_TOL * qn[r] * max(1.0, float(np.max(g["norm"])))
        assert np.all(np.abs(score[r] - ref_v[r]) <= tol)
        if list(idx[r]) != list(ref_i[r]):
            # near-ties may swap: any differing member must score within tol of the k-th
            diff = set(idx[r]) ^ set(ref_i[r])
            kth = ref_v[r, -1]
            for j in diff:
                qj = None if g["qjl"] is None else g["qjl"][j:j + 1].reshape(1, -1)
                rn = None if g["rnorm"] is None else g["rnorm"][j:j + 1]
                sc = o.logits(tab, q[r:r + 1], g["codes"][j:j + 1], g["norm"][j:j + 1], qj, rn)[0, 0]
                assert abs(sc - kth) <= 2 * tol, (r, j, sc, kth)


def test_topk_small_with_ties_and_short_db(cuda):
    c = _ctx(200, 4, 3, 200, seed=5)
    tab = P.oracle_tables(c)
    X = tq_inputs.mixture(5000, 200, seed=3)
    X[17] = X[4]
    Q = tq_inputs.mixture(40, 200, seed=4, means_seed=3)
    db = c.quantize(X.to(cuda), tq.TQ_KEY)
    idx, score = c.topk(Q.to(cuda), db, 10)
    torch.cuda.synchronize()
    g = _flat(db, 5000)
    _check_topk(tab, Q.double().numpy(), g, idx.cpu().numpy(), score.cpu().numpy(), 10)
    # fewer database vectors than k: the rest is (-1, -inf)
    small = {k: (None if v is None else v[:5]) for k, v in db.items()}
    idx2, score2 = c.topk(Q[:3].to(cuda), small, 10)
    torch.cuda.synchronize()
    assert np.all(idx2.cpu().numpy()[:, 5:] == -1) and np.all(np.isneginf(score2.cpu().numpy()[:, 5:]))
    assert sorted(idx2.cpu().numpy()[0, :5].tolist()) == [0, 1, 2, 3, 4]
    # an empty database: every slot is (-1, -inf)
    empty = {k: (None if v is None else v[:0]) for k, v in db.items()}
    idx3, score3 = c.topk(Q[:3].to(cuda), empty, 4)
    torch.cuda.synchronize()
    assert np.all(idx3.cpu().numpy() == -1) and np.all(np.isneginf(score3.cpu().numpy()))


@pytest.mark.parametrize("d,bk,m,k", [(128, 3, 128, 32), (64, 2, 0, 1), (200, 5, 200, 16), (96, 2, 64, 12)])
def test_topk_code_widths_and_k(cuda, d, bk, m, k):
    """Every packed width (1 to 4 Lloyd-Max bits, with and without QJL),
    k from 1 to 32 (both query-block sizes of the tensor-core scorer), and
    more queries than one block with a ragged last block."""
    c = _ctx(d, bk, 3, m, seed=13)
    tab = P.oracle_tables(c)
    X = tq_inputs.mixture(3000, d, seed=31)
    Q = tq_inputs.mixture(150, d, seed=32, means_seed=31)
    db = c.quantize(X.to(cuda), tq.TQ_KEY)
    idx, score = c.topk(Q.to(cuda), db, k)
    torch.cuda.synchronize()
    g = _flat(db, 3000)
    _check_topk(tab, Q.double().numpy(), g, idx.cpu().numpy(), score.cpu().numpy(), k)


def test_bounded_wait_expiry_sets_fault_and_recovers(cuda):
    """The tensor-core quantize and top-k kernels with their main bounded
    waits cut to one non-blocking poll (tq_set_wait_limit): on an ordinary
    launch the first wait gives up, the kernel waits with the full limit for
    the MMAs and copies it issued, sets its tq_device_fault bit (1 quantize,
    2 top-k) and returns; the next launch with the full limit is correct."""
    c = _ctx(128, 3, 4, 128, seed=2)
    tab = P.oracle_tables(c)
    n = 8192   # above the small-batch bound: the tensor-core quantize
    X = tq_inputs.outlier_kv(1, 1, n, 128, seed=12)[0, 0].to(torch.bfloat16)
    xd = X.to(cuda)
    assert tq.tq_device_fault() == 0
    c.set_wait_limit(1)
    c.quantize(xd, tq.TQ_KEY)
    assert tq.tq_device_fault() == 1
    c.set_wait_limit(0)
    pk = c.quantize(xd, tq.TQ_KEY)
    torch.cuda.synchronize()
    assert tq.tq_device_fault() == 0
    P.check_quantized(tab, "k", X.double().numpy(), _flat(pk, n))

    ct = _ctx(96, 3, 3, 64, seed=23)
    tabt = P.oracle_tables(ct)
    nq, nd, k = 129, 129, 5   # a ragged query block and tile on the tcgen05 scorer
    Xd = tq_inputs.mixture(nd, 96, seed=51)
    Q = tq_inputs.mixture(nq, 96, seed=52, means_seed=51)
    db = ct.quantize(Xd.to(cuda), tq.TQ_KEY)
    ct.set_wait_limit(1)
    ct.topk(Q.to(cuda), db, k)
    assert tq.tq_device_fault() == 2
    ct.set_wait_limit(0)
    idx, score = ct.topk(Q.to(cuda), db, k)
    torch.cuda.synchronize()
    assert tq.tq_device_fault() == 0
    _check_topk(tabt, Q.double().numpy(), _flat(db, nd), idx.cpu().numpy(), score.cpu().numpy(), k)


@pytest.mark.parametrize("d,bk,m,nq,n,k", [
    (64, 2, 64, 1, 127, 12),      # one query, a database shorter than one 128-row tile
    (96, 3, 64, 129, 129, 5),     # ragged query block and tile, K padded to 16s
    (256, 4, 256, 40, 1000, 3),   # eight 64-wide K blocks (the largest query operand)
    (256, 2, 0, 200, 700, 12),    # MSE-only keys (no sign accumulator), k at the register-list limit
])
def test_topk_tensor_core_edges(cuda, d, bk, m, nq, n, k):
    """Edge shapes of the tcgen05 scorer: partial tiles and query blocks,
    the widest query operand, MSE-only keys; no device fault is raised."""
    c = _ctx(d, bk, 3, m, seed=23)
    tab = P.oracle_tables(c)
    X = tq_inputs.mixture(n, d, seed=51)
    Q = tq_inputs.mixture(nq, d, seed=52, means_seed=51)
    db = c.quantize(X.to(cuda), tq.TQ_KEY)
    idx, score = c.topk(Q.to(cuda), db, k)
    torch.cuda.synchronize()
    assert tq.tq_device_fault() == 0
    g = _flat(db, n)
    _check_topk(tab, Q.double().numpy(), g, idx.cpu().numpy(), score.cpu().numpy(), k)


def test_topk_sample_bar_pass(cuda):
    """A database large enough for the two-pass scorer (the k-th best of a
    leading sample bars every list): exact duplicates inside the sample (equal
    scores, broken by index), a query whose best match sits past the sample,
    and k larger than the number of duplicates."""
    n, d = 150_000, 64
    c = _ctx(d, 2, 3, 64, seed=17)
    tab = P.oracle_tables(c)
    X = tq_inputs.mixture(n, d, seed=41)
    Q = tq_inputs.mixture(64, d, seed=42, means_seed=41)
    # queries 0 and 1 point away from every mixture component, so their own
    # copies are their best matches by a wide margin
    Q[0:2] = tq_inputs.iid((2, d), seed=43)
    Q[0:2] /= torch.linalg.vector_norm(Q[0:2], dim=1, keepdim=True)
    X[0:5] = Q[0]
    X[n - 7] = Q[1]
    X[n - 3] = Q[1]
    db = c.quantize(X.to(cuda), tq.TQ_KEY)
    idx, score = c.topk(Q.to(cuda), db, 16)
    torch.cuda.synchronize()
    g = _flat(db, n)
    idx, score = idx.cpu().numpy(), score.cpu().numpy()
    _check_topk(tab, Q.double().numpy(), g, idx, score, 16)
    assert idx[0, :5].tolist() == [0, 1, 2, 3, 4]
    assert idx[1, :2].tolist() == [n - 7, n - 3]
    assert np.all(np.diff(score, axis=1) <= 0)
    for r in range(idx.shape[0]):
        assert len(set(idx[r].tolist())) == 16


def test_topk_vector_search_full(cuda):
    """1e6 unit-norm d=200 mixture vectors, 1e4 queries, 3-bit + QJL, top-10;
    the oracle checks the first 32 queries on the same codes."""
    c = _ctx(200, 4, 3, 200, seed=11)
    tab = P.oracle_tables(c)
    X = tq_inputs.mixture(1_000_000, 200, seed=21, device=cuda)
    Q = tq_inputs.mixture(10_000, 200, seed=22, means_seed=21, device=cuda)
    db = c.quantize(X, tq.TQ_KEY)
    n = 8192
    P.check_quantized(tab, "k", P.to_np(X[:n]), _flat({k: v[:n] for k, v in db.items()}, n))
    idx, score = c.topk(Q, db, 10)
    torch.cuda.synchronize()
    g = _flat(db, 1_000_000)
    _check_topk(tab, P.to_np(Q[:32]), g, idx[:32].cpu().numpy(), score[:32].cpu().numpy(), 10)
    assert np.all(np.diff(score.cpu().numpy(), axis=1) <= 0)
    assert tq.tq_device_fault() == 0


# --- error reporting through the C ABI ----------------------------------------------
def test_errors_are_reported(cuda):
    c = _ctx(128, 3, 4, 128)
    K = torch.randn(4, 1, 16, 128, device=cuda)
    kc, vc = _cache(c, K, K, cuda)
    q = torch.randn(4, 8, 128, device=cuda)
    lens = torch.full((4,), 16, dtype=torch.int32, device=cuda)
    small = torch.empty(16, dtype=torch.uint8, device=cuda)
    with pytest.raises(tq.TQError) as e:
        c.attn_decode(q, kc, vc, lens, workspace=small)
    assert e.value.status == tq.TQ_ERR_WORKSPACE
    with pytest.raises(tq.TQError) as e:
        c.attn_decode(torch.randn(4, 34, 128, device=cuda), kc, vc, lens)
    assert e.value.status == tq.TQ_ERR_UNSUPPORTED
    with pytest.raises(tq.TQError) as e:
        tq._check(tq._lib.tq_quantize(c.ptr, 7, None, 0, 1, 128, None, None, None, None, None))
    assert e.value.status == tq.TQ_ERR_ARG


def test_norm_dtype_mismatch_is_refused(cuda):
    """Norms reach the C ABI as untyped pointers, so the binding refuses a norm
    array of the wrong type (binary16 for an fp32-norm context, and the
    reverse) before any launch."""
    c = _ctx(128, 3, 4, 128)
    K = torch.randn(2, 1, 16, 128, device=cuda)
    kc, vc = _cache(c, K, K, cuda)
    q = torch.randn(2, 4, 128, device=cuda)
    lens = torch.full((2,), 16, dtype=torch.int32, device=cuda)
    bad = dict(kc, norm=kc["norm"].half())
    for call in (lambda: c.attn_decode(q, bad, vc, lens), lambda: c.logits(q[0], bad),
                 lambda: c.dequantize(tq.TQ_KEY, bad), lambda: c.quantize_into(K, tq.TQ_KEY, bad)):
        with pytest.raises(tq.TQError) as e:
            call()
        assert e.value.status == tq.TQ_ERR_ARG
    c16 = tq.Context.variant("4bit_nc", 128, norm_f16=True)
    vc16 = c16.quantize(K, tq.TQ_VALUE)
    with pytest.raises(tq.TQError) as e:
        c16.dequantize(tq.TQ_VALUE, dict(vc16, norm=vc16["norm"].float()))
    assert e.value.status == tq.TQ_ERR_ARG


def test_context_of_another_device_is_refused(cuda):
    """A context's tables live on the device current at tq_init; a compute
    call with another device current is refused before any launch."""
    if torch.cuda.device_count() < 2:
        pytest.skip("needs two GPUs")
    c = _ctx(128, 3, 4, 128)
    x = torch.randn(4, 128, device="cuda:1")
    pk = {k: (None if v is None else v.to("cuda:1")) for k, v in c.empty_packed(tq.TQ_KEY, (4,)).items()}
    with torch.cuda.device(1):
        with pytest.raises(tq.TQError) as e:
            c.quantize_into(x, tq.TQ_KEY, pk)
    assert e.value.status == tq.TQ_ERR_ARG and "device" in str(e.value)


def test_quantize_append_writes_addressed_slots(cuda):
    """Only slot pos[b] of each sequence is written; a pos outside [0, T)
    writes nothing."""
    c = _ctx(128, 3, 4, 128, seed=0)
    B, H, T = 5, 2, 50
    x = tq_inputs.outlier_kv(B, H, 1, 128, seed=9)[:, :, 0].contiguous().to(cuda)
    pos = torch.tensor([0, 49, 17, -1, 50], dtype=torch.int32, device=cuda)
    for which in (tq.TQ_KEY, tq.TQ_VALUE):
        cache = c.empty_packed(which, (B, H, T), device=cuda)
        for v in cache.values():
            if v is not None:
                v.fill_(-7)
        c.quantize_append(x, which, cache, pos)
        ref = c.quantize(x.reshape(B * H, 128), which)
        torch.cuda.synchronize()
        for k, v in cache.items():
            if v is None:
                continue
            got = v.cpu()
            want = ref[k].cpu().reshape((B, H) + tuple(v.shape[3:]))
            for b in range(B):
                p = int(pos[b])
                mask = torch.ones(T, dtype=torch.bool)
                if 0 <= p < T:
                    assert torch.equal(got[b, :, p], want[b]), (k, b)
                    mask[p] = False
                assert torch.all(got[b][:, mask] == -7), (k, b)


def test_quantize_tensor_core_fp16_strided(cuda):
    """More than 4096 vectors of fp16 input with a row pitch of 136 elements
    (the tensor-core path), including zero rows and a ragged last tile."""
    c = _ctx(128, 3, 4, 128, seed=2)
    tab = P.oracle_tables(c)
    n = 5000
    X = tq_inputs.outlier_kv(1, 1, n, 128, seed=12)[0, 0].half()
    X[7] = 0
    big = torch.zeros(n, 136, dtype=torch.float16)
    big[:, :128] = X
    src = big.to(cuda)[:, :128]
    for which, wch in ((tq.TQ_KEY, "k"), (tq.TQ_VALUE, "v")):
        pk = c.empty_packed(which, (n,))
        c.quantize_into(src, which, pk)
        torch.cuda.synchronize()
        assert tq.tq_device_fault() == 0
        P.check_quantized(tab, wch, X.double().numpy(), _flat(pk, n))


def test_quantize_append_large_batch(cuda):
    """Appending 8192 (sequence, head) rows at per-sequence slots (tensor-core
    path with cache placement)."""
    c = _ctx(128, 3, 4, 128, seed=0)
    B, H, T = 64, 128, 6
    x = tq_inputs.outlier_kv(B, H, 1, 128, seed=19)[:, :, 0].contiguous().to(cuda)
    pos = torch.randint(0, T, (B,), generator=torch.Generator().manual_seed(3), dtype=torch.int32)
    pos[5], pos[40] = -1, T          # skipped: nothing written for these sequences
    pos = pos.to(cuda)
    ok = (pos >= 0) & (pos < T)
    for which in (tq.TQ_KEY, tq.TQ_VALUE):
        cache = c.empty_packed(which, (B, H, T), device=cuda)
        for v in cache.values():
            if v is not None:
                v.fill_(-7)
        c.quantize_append(x, which, cache, pos)
        ref = c.quantize(x.reshape(B * H, 128), which)
        torch.cuda.synchronize()
        for k, v in cache.items():
            if v is None:
                continue
            want = ref[k].reshape((B, H) + tuple(v.shape[3:]))
            bs = torch.arange(B, device=cuda)[ok]
            got = v[bs, :, pos[ok].long()]
            assert torch.equal(got, want[ok]), k
            assert torch.all(v[~ok] == -7), k


@pytest.mark.parametrize("Hq,Hkv,bk,max_T", [
    (8, 2, 3, 300),     # tensor-core decode, group 4
    (16, 2, 3, 300),    # group 8
    (16, 2, 4, 300),    # 3-bit keys, group 8
    (8, 2, 4, 300),     # 3-bit keys, group 4
    (8, 2, 3, 302),     # max_T % 4 != 0: generic decode
])
def test_decode_step_equals_append_then_decode(cuda, Hq, Hkv, bk, max_T):
    """tq_decode_step = quantize_append (K, V) + attn_decode over pos + 1
    tokens: identical caches and outputs, and the outputs match the oracle.
    Positions cover the first slot, the middle, the last slot, a skipped
    negative position (empty context) and one past the end (no write, full
    context)."""
    c = _ctx(128, bk, 4, 128, seed=4)
    tab = P.oracle_tables(c)
    B, d = 6, 128
    K = tq_inputs.outlier_kv(B, Hkv, max_T, d, seed=31).to(cuda)
    V = tq_inputs.outlier_kv(B, Hkv, max_T, d, seed=32).to(cuda)
    kA, vA = c.quantize(K, tq.TQ_KEY), c.quantize(V, tq.TQ_VALUE)
    kB = {k: (None if v is None else v.clone()) for k, v in kA.items()}
    vB = {k: (None if v is None else v.clone()) for k, v in vA.items()}
    q = tq_inputs.iid((B, Hq, d), seed=33, dtype=torch.bfloat16).to(cuda)
    kn = tq_inputs.outlier_kv(B, Hkv, 1, d, seed=34)[:, :, 0].contiguous().to(cuda)
    vn = tq_inputs.outlier_kv(B, Hkv, 1, d, seed=35)[:, :, 0].contiguous().to(cuda)
    pos = torch.tensor([0, 17, 160, max_T - 1, -1, max_T], dtype=torch.int32, device=cuda)
    outA = c.decode_step(q, kn, vn, kA, vA, pos)
    c.quantize_append(kn, tq.TQ_KEY, kB, pos)
    c.quantize_append(vn, tq.TQ_VALUE, vB, pos)
    lens = torch.clamp(pos.long() + 1, 0, max_T).to(torch.int32)
    outB = c.attn_decode(q, kB, vB, lens)
    torch.cuda.synchronize()
    for name, a_, b_ in (("k", kA, kB), ("v", vA, vB)):
        for k in a_:
            if a_[k] is not None:
                assert torch.equal(a_[k], b_[k]), (name, k)
    assert torch.equal(outA, outB)
    P.check_attention(tab, q.double().cpu().numpy(), P.packed_np(kA), P.packed_np(vA),
                      lens.cpu().numpy(), Hkv, outA.cpu().numpy())


@pytest.mark.parametrize("fmt,Hq", [("k3v4", 8), ("k3v4", 16), ("k3v4", 2), ("k4v4", 8), ("k4v4", 4),
                                    ("k3v4_nc", 8), ("4bit_nc", 2), ("3bit_nc", 16), ("k8v4", 8)])
def test_decode_logit_precision(cuda, fmt, Hq):
    """Two keys whose logits are large but differ by 1/100 of their size,
    the query scaled so the difference is one unit: the softmax weights then
    expose logit errors 100x magnified.  The tensor-core decode carries ~22
    bits (fp16 head + tail of both operands), so the output stays within
    the attention bound; a dropped tail term (~11 bits, ~6e-3 here) would
    not."""
    c = tq.Context.variant(fmt, 128, seed=31)
    tab = P.oracle_tables(c)
    B, Hkv, d = 4, 2, 128
    G = Hq // Hkv
    pool = tq_inputs.iid((2048, d), seed=71)
    pk = c.quantize(pool.to(cuda), tq.TQ_KEY)
    torch.cuda.synchronize()
    g = _flat(pk, 2048)
    q0 = tq_inputs.iid((B, Hkv, d), seed=72).double().numpy()
    Q = np.zeros((B, Hq, d))
    pick = np.zeros((B, Hkv, 2), dtype=np.int64)
    for b in range(B):
        for h in range(Hkv):
            lg = o.logits(tab, q0[b, h][None], g["codes"], g["norm"], g.get("qjl"), g.get("rnorm"))[0]
            order = np.argsort(lg)
            gaps = np.diff(lg[order])
            size = np.maximum(np.abs(lg[order][:-1]), np.abs(lg[order][1:]))
            r = np.argmin(np.abs(np.log(np.maximum(gaps, 1e-30) * 100.0 / np.maximum(size, 1e-30))))
            i, j = order[r], order[r + 1]
            pick[b, h] = (i, j)
            f = 1.0 / (lg[j] - lg[i]) * math.sqrt(d)   # scaled logit difference of one
            Q[b, h * G:(h + 1) * G] = q0[b, h] * f
    kc = {k: (None if v is None else v[torch.as_tensor(pick).reshape(-1).to(cuda)].reshape(
        (B, Hkv, 2) + tuple(v.shape[1:]))) for k, v in pk.items()}
    kc = {k: (None if v is None else torch.cat([v, v], dim=2).contiguous()) for k, v in kc.items()}   # max_T 4
    V = tq_inputs.outlier_kv(B, Hkv, 4, d, seed=73)
    vc = c.quantize(V.to(cuda), tq.TQ_VALUE)
    lens = torch.full((B,), 2, dtype=torch.int32)
    Qt = torch.from_numpy(Q).float()
    out = c.attn_decode(Qt.to(cuda), kc, vc, lens.to(cuda))
    torch.cuda.synchronize()
    P.check_attention(tab, Qt.double().numpy(), P.packed_np(kc), P.packed_np(vc), lens.numpy(), Hkv,
                      out.cpu().numpy())


# --- norm-corrected cache formats -------------------------------------------------
@pytest.mark.parametrize("name,Hq", [("k3v4_nc", 8), ("k3v4_nc", 16), ("4bit_nc", 8), ("4bit_nc", 16),
                                     ("3bit_nc", 8), ("3bit_nc", 16), ("4bit_nc", 2), ("3bit_nc", 4)])
def test_norm_corrected_variants(cuda, name, Hq):
    """The MSE-only _nc formats: quantize through the bulk and the small-batch
    kernels (stored norm n / |c[idx]|), logits, ragged decode attention, and
    the fused decode step (equal to append + decode), all against the oracle
    with the same reading of norm correction."""
    c = tq.Context.variant(name, 128, seed=8)
    assert c.nc_k and c.nc_v and c.qjl_m == 0
    tab = P.oracle_tables(c)
    B, Hkv, T, d = 4, 2, 1100, 128
    K = tq_inputs.outlier_kv(B, Hkv, T, d, seed=61)
    V = tq_inputs.outlier_kv(B, Hkv, T, d, seed=62)
    kc, vc = _cache(c, K, V, cuda)
    n = B * Hkv * T
    P.check_quantized(tab, "k", P.to_np(K.reshape(n, d)), _flat(kc, n))
    P.check_quantized(tab, "v", P.to_np(V.reshape(n, d)), _flat(vc, n))
    small = K[0, 0, :300].contiguous()
    ks = c.quantize(small.to(cuda), tq.TQ_KEY)
    P.check_quantized(tab, "k", P.to_np(small), _flat(ks, 300))
    Q = tq_inputs.iid((B, Hq, d), seed=63, dtype=torch.bfloat16)
    lg = c.logits(Q[0].to(cuda), ks)
    torch.cuda.synchronize()
    P.check_logits(tab, Q[0].double().numpy(), _flat(ks, 300), lg.cpu().double().numpy())
    lens = torch.tensor([0, 1, 517, T], dtype=torch.int32)
    out = c.attn_decode(Q.to(cuda), kc, vc, lens.to(cuda))
    torch.cuda.synchronize()
    P.check_attention(tab, Q.double().numpy(), P.packed_np(kc), P.packed_np(vc), lens.numpy(), Hkv,
                      out.cpu().numpy())
    # fused step vs append + decode on copies of the same cache
    kB = {k: (None if v is None else v.clone()) for k, v in kc.items()}
    vB = {k: (None if v is None else v.clone()) for k, v in vc.items()}
    kn = tq_inputs.outlier_kv(B, Hkv, 1, d, seed=64)[:, :, 0].contiguous().to(cuda)
    vn = tq_inputs.outlier_kv(B, Hkv, 1, d, seed=65)[:, :, 0].contiguous().to(cuda)
    pos = torch.tensor([0, 600, T - 1, -1], dtype=torch.int32, device=cuda)
    q = Q.to(cuda)
    outA = c.decode_step(q, kn, vn, kc, vc, pos)
    c.quantize_append(kn, tq.TQ_KEY, kB, pos)
    c.quantize_append(vn, tq.TQ_VALUE, vB, pos)
    lens2 = torch.clamp(pos.long() + 1, 0, T).to(torch.int32)
    outB = c.attn_decode(q, kB, vB, lens2)
    torch.cuda.synchronize()
    for a_, b_ in ((kc, kB), (vc, vB)):
        for k in a_:
            if a_[k] is not None:
                assert torch.equal(a_[k], b_[k]), k
    assert torch.equal(outA, outB)
    P.check_attention(tab, Q.double().numpy(), P.packed_np(kc), P.packed_np(vc), lens2.cpu().numpy(), Hkv,
                      outA.cpu().numpy())


@pytest.mark.parametrize("Hq", [8, 16, 2])
def test_eight_bit_keys(cuda, Hq):
    """k8v4: 8-bit Lloyd-Max keys (MSE only), 4-bit values.  Quantize through
    the bulk and the small-batch kernels, logits, ragged decode and the fused
    step against the oracle; top-k declines 8-bit keys."""
    c = tq.Context.variant("k8v4", 128, seed=9)
    assert c.key_layout["bits"] == 8 and c.key_layout["bytes_per_vector"] == 132
    tab = P.oracle_tables(c)
    B, Hkv, T, d = 3, 2, 700, 128
    K = tq_inputs.outlier_kv(B, Hkv, T, d, seed=71)
    V = tq_inputs.outlier_kv(B, Hkv, T, d, seed=72)
    kc, vc = _cache(c, K, V, cuda)
    n = B * Hkv * T
    P.check_quantized(tab, "k", P.to_np(K.reshape(n, d)), _flat(kc, n))
    small = K[1, 1, :200].contiguous()
    ks = c.quantize(small.to(cuda), tq.TQ_KEY)
    P.check_quantized(tab, "k", P.to_np(small), _flat(ks, 200))
    Q = tq_inputs.iid((B, Hq, d), seed=73, dtype=torch.bfloat16)
    lg = c.logits(Q[0].to(cuda), ks)
    torch.cuda.synchronize()
    P.check_logits(tab, Q[0].double().numpy(), _flat(ks, 200), lg.cpu().double().numpy())
    lens = torch.tensor([1, 333, T], dtype=torch.int32)
    out = c.attn_decode(Q.to(cuda), kc, vc, lens.to(cuda))
    torch.cuda.synchronize()
    P.check_attention(tab, Q.double().numpy(), P.packed_np(kc), P.packed_np(vc), lens.numpy(), Hkv,
                      out.cpu().numpy())
    kB = {k: (None if v is None else v.clone()) for k, v in kc.items()}
    vB = {k: (None if v is None else v.clone()) for k, v in vc.items()}
    kn = tq_inputs.outlier_kv(B, Hkv, 1, d, seed=74)[:, :, 0].contiguous().to(cuda)
    vn = tq_inputs.outlier_kv(B, Hkv, 1, d, seed=75)[:, :, 0].contiguous().to(cuda)
    pos = torch.tensor([5, T - 1, 400], dtype=torch.int32, device=cuda)
    q = Q.to(cuda)
    outA = c.decode_step(q, kn, vn, kc, vc, pos)
    c.quantize_append(kn, tq.TQ_KEY, kB, pos)
    c.quantize_append(vn, tq.TQ_VALUE, vB, pos)
    outB = c.attn_decode(q, kB, vB, (pos + 1).to(torch.int32))
    torch.cuda.synchronize()
    for a_, b_ in ((kc, kB), (vc, vB)):
        for k in a_:
            if a_[k] is not None:
                assert torch.equal(a_[k], b_[k]), k
    assert torch.equal(outA, outB)
    with pytest.raises(tq.TQError) as e:
        c.topk(Q[0].to(cuda), ks, 4)
    assert e.value.status == tq.TQ_ERR_UNSUPPORTED


@pytest.mark.parametrize("name,Hq", [("k3v4_nc", 8), ("4bit_nc", 4), ("3bit_nc", 16), ("k8v4", 8)])
def test_binary16_norm_variants(cuda, name, Hq):
    """The MSE-only formats with binary16 norms: layout, quantize (bulk and
    small batch), logits, dequantize, decode on the tensor-core path
    (max_T % 8 == 0) and the generic path, the fused step, paged caches and
    (for keys of at most 4 bits) top-k, all against the oracle."""
    c = tq.Context.variant(name, 128, seed=14, norm_f16=True)
    assert c.key_layout["norm_bytes"] == 2 and c.value_layout["norm_bytes"] == 2
    tab = P.oracle_tables(c)
    B, Hkv, T, d = 4, 2, 1104, 128
    K = tq_inputs.outlier_kv(B, Hkv, T, d, seed=81)
    V = tq_inputs.outlier_kv(B, Hkv, T, d, seed=82)
    kc, vc = _cache(c, K, V, cuda)
    assert kc["norm"].dtype == torch.float16
    n = B * Hkv * T
    P.check_quantized(tab, "k", P.to_np(K.reshape(n, d)), _flat(kc, n))
    P.check_quantized(tab, "v", P.to_np(V.reshape(n, d)), _flat(vc, n))
    small = V[1, 0, :300].contiguous()
    vs = c.quantize(small.to(cuda), tq.TQ_VALUE)
    P.check_quantized(tab, "v", P.to_np(small), _flat(vs, 300))
    Q = tq_inputs.iid((B, Hq, d), seed=83, dtype=torch.bfloat16)
    ks = {k: (None if v is None else v[0, 0, :256].contiguous()) for k, v in kc.items()}
    lg = c.logits(Q[0].to(cuda), ks)
    xh = c.dequantize(tq.TQ_VALUE, vs)
    torch.cuda.synchronize()
    P.check_logits(tab, Q[0].double().numpy(), _flat(ks, 256), lg.cpu().double().numpy())
    g = _flat(vs, 300)
    ref = o.dequantize(tab, "v", g["codes"], g["norm"])
    assert np.abs(xh.cpu().double().numpy() - ref).max() <= 1e-5 * np.abs(ref).max()
    lens = torch.tensor([0, 1, 517, T], dtype=torch.int32)
    out = c.attn_decode(Q.to(cuda), kc, vc, lens.to(cuda))
    kg = {k: (None if v is None else v[:, :, :T - 2].contiguous()) for k, v in kc.items()}   # generic path
    vg = {k: (None if v is None else v[:, :, :T - 2].contiguous()) for k, v in vc.items()}
    lens_g = torch.tensor([0, 1, 517, T - 2], dtype=torch.int32)
    outg = c.attn_decode(Q.to(cuda), kg, vg, lens_g.to(cuda))
    torch.cuda.synchronize()
    P.check_attention(tab, Q.double().numpy(), P.packed_np(kc), P.packed_np(vc), lens.numpy(), Hkv,
                      out.cpu().numpy())
    P.check_attention(tab, Q.double().numpy(), P.packed_np(kg), P.packed_np(vg), lens_g.numpy(), Hkv,
                      outg.cpu().numpy())
    # fused step vs append + decode
    kB = {k: (None if v is None else v.clone()) for k, v in kc.items()}
    vB = {k: (None if v is None else v.clone()) for k, v in vc.items()}
    kn = tq_inputs.outlier_kv(B, Hkv, 1, d, seed=84)[:, :, 0].contiguous().to(cuda)
    vn = tq_inputs.outlier_kv(B, Hkv, 1, d, seed=85)[:, :, 0].contiguous().to(cuda)
    pos = torch.tensor([3, 700, T - 1, 64], dtype=torch.int32, device=cuda)
    q = Q.to(cuda)
    outA = c.decode_step(q, kn, vn, kc, vc, pos)
    c.quantize_append(kn, tq.TQ_KEY, kB, pos)
    c.quantize_append(vn, tq.TQ_VALUE, vB, pos)
    outB = c.attn_decode(q, kB, vB, (pos + 1).to(torch.int32))
    torch.cuda.synchronize()
    for a_, b_ in ((kc, kB), (vc, vB)):
        for k in a_:
            if a_[k] is not None:
                assert torch.equal(a_[k], b_[k]), k
    assert torch.equal(outA, outB)
    # paged: the same records through a shuffled block table
    bs, mb = 16, T // 16
    perm = torch.randperm(B * mb, generator=torch.Generator().manual_seed(3)).to(torch.int32)
    kp, vp = _to_paged(kc, B, Hkv, T, bs, perm), _to_paged(vc, B, Hkv, T, bs, perm)
    got = c.attn_decode_paged(q, kp, vp, perm.reshape(B, mb).to(cuda), lens.to(cuda))
    ref_c = c.attn_decode(q, kc, vc, lens.to(cuda))
    torch.cuda.synchronize()
    assert torch.equal(got, ref_c)
    if c.key_layout["bits"] <= 4:
        X = tq_inputs.mixture(3000, d, seed=86)
        Qs = tq_inputs.mixture(60, d, seed=87, means_seed=86)
        db = c.quantize(X.to(cuda), tq.TQ_KEY)
        idx, score = c.topk(Qs.to(cuda), db, 8)
        torch.cuda.synchronize()
        assert tq.tq_device_fault() == 0
        _check_topk(tab, Qs.double().numpy(), _flat(db, 3000), idx.cpu().numpy(), score.cpu().numpy(), 8)


# --- paged caches ---------------------------------------------------------------
def _to_paged(cache, B, Hkv, max_T, bs, perm):
    """Scatter a contiguous [B, Hkv, max_T, ...] cache into blocks
    [num_blocks, Hkv, bs, ...]; block i of sequence b is perm[b * mb + i]."""
    mb = max_T // bs
    nb = int(perm.max()) + 1
    out = {}
    for k, v in cache.items():
        if v is None:
            out[k] = None
            continue
        tail = tuple(v.shape[3:])
        pv = torch.full((nb, Hkv, bs) + tail, -3, dtype=v.dtype, device=v.device)
        blocks = v.reshape((B, Hkv, mb, bs) + tail).transpose(1, 2).reshape((B * mb, Hkv, bs) + tail)
        pv[perm.long().to(v.device)] = blocks
        out[k] = pv
    return out


@pytest.mark.parametrize("Hq,Hkv,bk,bs,variant", [
    (8, 2, 3, 32, None), (16, 2, 3, 16, None), (16, 2, 4, 48, None), (4, 4, 3, 16, None),
    (8, 2, 4, 16, None), (8, 2, None, 32, "4bit_nc"), (16, 2, None, 16, "k3v4_nc"),
    (8, 2, None, 16, "3bit_nc"), (16, 2, None, 48, "3bit_nc"), (8, 2, None, 32, "k8v4"),
    (16, 2, None, 16, "k8v4"), (4, 2, None, 16, "k3v4_nc"), (2, 2, 4, 32, None)])
def test_paged_decode_equals_contiguous(cuda, Hq, Hkv, bk, bs, variant):
    """The paged decode reads the same records through the block table, so it
    must reproduce the contiguous decode bit for bit (ragged lengths,
    partial last blocks, an empty sequence, blocks in shuffled order)."""
    c = tq.Context.variant(variant, 128, seed=6) if variant else _ctx(128, bk, 4, 128, seed=6)
    B, d, max_T = 5, 128, 288
    K = tq_inputs.outlier_kv(B, Hkv, max_T, d, seed=41).to(cuda)
    V = tq_inputs.outlier_kv(B, Hkv, max_T, d, seed=42).to(cuda)
    kc, vc = c.quantize(K, tq.TQ_KEY), c.quantize(V, tq.TQ_VALUE)
    mb = max_T // bs
    perm = torch.randperm(B * mb + 7, generator=torch.Generator().manual_seed(5))[:B * mb].to(torch.int32)
    kp, vp = _to_paged(kc, B, Hkv, max_T, bs, perm), _to_paged(vc, B, Hkv, max_T, bs, perm)
    table = perm.reshape(B, mb).to(cuda)
    q = tq_inputs.iid((B, Hq, d), seed=43, dtype=torch.bfloat16).to(cuda)
    lens = torch.tensor([0, 1, bs + 3, 200, max_T], dtype=torch.int32, device=cuda)
    ref = c.attn_decode(q, kc, vc, lens)
    got = c.attn_decode_paged(q, kp, vp, table, lens)
    torch.cuda.synchronize()
    assert torch.equal(got, ref)


@pytest.mark.parametrize("Hq,Hkv,bk", [(8, 2, 3), (16, 2, 4)])
def test_paged_decode_step_equals_contiguous(cuda, Hq, Hkv, bk):
    """decode_step_paged writes the new token into its block slot and attends
    like decode_step on the equivalent contiguous cache; a sequence whose
    block id is invalid gets nothing written."""
    c = _ctx(128, bk, 4, 128, seed=8)
    B, d, max_T, bs = 4, 128, 128, 32
    K = tq_inputs.outlier_kv(B, Hkv, max_T, d, seed=51).to(cuda)
    V = tq_inputs.outlier_kv(B, Hkv, max_T, d, seed=52).to(cuda)
    kc, vc = c.quantize(K, tq.TQ_KEY), c.quantize(V, tq.TQ_VALUE)
    mb = max_T // bs
    perm = torch.randperm(B * mb, generator=torch.Generator().manual_seed(9)).to(torch.int32)
    kp, vp = _to_paged(kc, B, Hkv, max_T, bs, perm), _to_paged(vc, B, Hkv, max_T, bs, perm)
    table = perm.reshape(B, mb).to(cuda)
    q = tq_inputs.iid((B, Hq, d), seed=53, dtype=torch.bfloat16).to(cuda)
    kn = tq_inputs.outlier_kv(B, Hkv, 1, d, seed=54)[:, :, 0].contiguous().to(cuda)
    vn = tq_inputs.outlier_kv(B, Hkv, 1, d, seed=55)[:, :, 0].contiguous().to(cuda)
    pos = torch.tensor([0, 40, 95, 127], dtype=torch.int32, device=cuda)
    ref = c.decode_step(q, kn, vn, kc, vc, pos)
    got = c.decode_step_paged(q, kn, vn, kp, vp, table, pos)
    torch.cuda.synchronize()
    assert torch.equal(got, ref)
    kp2, vp2 = _to_paged(kc, B, Hkv, max_T, bs, perm), _to_paged(vc, B, Hkv, max_T, bs, perm)
    for a_, b_ in ((kp, kp2), (vp, vp2)):
        for k in a_:
            if a_[k] is not None:
                assert torch.equal(a_[k], b_[k]), k
    # an invalid block id: the append is skipped
    bad = table.clone()
    bad[1, 40 // bs] = -1
    before = {k: (None if v is None else v.clone()) for k, v in kp.items()}
    c.quantize_append_paged(kn, tq.TQ_KEY, kp, bad, pos)
    torch.cuda.synchronize()
    blk = int(table[1, 40 // bs])
    for k, v in kp.items():
        if v is not None:
            assert torch.equal(v[blk], before[k][blk]), k


def _from_paged(cache_np, table, B, bs):
    """Host copy of a paged cache [blocks, Hkv, bs, ...] as a contiguous
    [B, Hkv, max_blocks * bs, ...] cache through the block table (invalid ids
    give zero records, which the callers never read)."""
    mb = table.shape[1]
    out = {}
    for k, v in cache_np.items():
        if v is None:
            out[k] = None
            continue
        rows = []
        for b in range(B):
            blocks = [v[int(i)] if 0 <= int(i) < v.shape[0] else np.zeros_like(v[0]) for i in table[b]]
            rows.append(np.concatenate(blocks, axis=1))
        out[k] = np.stack(rows)
    return out


def _drop_tokens(cache_np, b, lo, hi):
    """Sequence b's records with tokens [lo, hi) removed (softmax . V is
    invariant to the order of the (key, value) pairs, so a masked block is the
    same as a shorter context without it)."""
    return {k: (None if v is None else np.delete(v[b:b + 1], np.s_[lo:hi], axis=2)) for k, v in cache_np.items()}


@pytest.mark.parametrize("fmt,Hq,bs", [("k3v4", 8, 32), ("k3v4", 16, 16), ("k3v4", 2, 16), ("k4v4", 8, 16),
                                       ("k4v4", 16, 48), ("4bit_nc", 8, 32), ("3bit_nc", 16, 16)])
def test_paged_decode_matches_oracle(cuda, fmt, Hq, bs):
    """The paged decode against the fp64 oracle on the same codes: shuffled
    blocks, ragged lengths (empty, one token, a partial last block, full), an
    invalid block id inside a sequence (its tokens are masked: the reference
    is the context without them) and one past a sequence's length (no
    effect)."""
    c = tq.Context.variant(fmt, 128, seed=6)
    tab = P.oracle_tables(c)
    B, Hkv, d, max_T = 5, 2, 128, 288
    K = tq_inputs.outlier_kv(B, Hkv, max_T, d, seed=41)
    V = tq_inputs.outlier_kv(B, Hkv, max_T, d, seed=42)
    kc, vc = c.quantize(K.to(cuda), tq.TQ_KEY), c.quantize(V.to(cuda), tq.TQ_VALUE)
    mb = max_T // bs
    perm = torch.randperm(B * mb + 7, generator=torch.Generator().manual_seed(5))[:B * mb].to(torch.int32)
    kp, vp = _to_paged(kc, B, Hkv, max_T, bs, perm), _to_paged(vc, B, Hkv, max_T, bs, perm)
    table = perm.reshape(B, mb).clone()
    lens = torch.tensor([0, 1, bs + 3, 200, max_T], dtype=torch.int32)
    table[4, 1] = -1          # inside sequence 4: tokens [bs, 2 bs) masked
    table[2, mb - 1] = 10**6  # past sequence 2's length: never read
    q = tq_inputs.iid((B, Hq, d), seed=43, dtype=torch.bfloat16)
    got = c.attn_decode_paged(q.to(cuda), kp, vp, table.to(cuda), lens.to(cuda))
    torch.cuda.synchronize()
    kh, vh = P.packed_np(kc), P.packed_np(vc)
    qn, gn = q.double().numpy(), got.cpu().numpy()
    for b in range(B):
        L = int(lens[b])
        if b == 4:
            kb, vb, L = _drop_tokens(kh, b, bs, 2 * bs), _drop_tokens(vh, b, bs, 2 * bs), L - bs
        else:
            kb = {k: (None if v is None else v[b:b + 1]) for k, v in kh.items()}
            vb = {k: (None if v is None else v[b:b + 1]) for k, v in vh.items()}
        P.check_attention(tab, qn[b:b + 1], kb, vb, np.array([L]), Hkv, gn[b:b + 1])


@pytest.mark.parametrize("fmt,Hq", [("k3v4", 32), ("k3v4", 64), ("k4v4", 32)])
def test_paged_decode_long_pieces_mask_only_invalid_tiles(cuda, fmt, Hq):
    """Pieces of more than 32 tiles per warp (1 x 8 heads x 131072 tokens):
    an invalid first block masks its own tiles only.  The kernels keep one
    mask bit per tile modulo 32, so tile k + 32 of the same warp reuses tile
    k's bit; value vectors 1000x larger at the tokens of those later tiles
    (tiles 32-35 and 128-131 of the first piece) make a stale bit visible."""
    c = tq.Context.variant(fmt, 128, seed=12)
    tab = P.oracle_tables(c)
    B, Hkv, d, T, bs = 1, 8, 128, 131072, 64
    K = tq_inputs.outlier_kv(B, Hkv, T, d, seed=61).to(cuda)
    V = tq_inputs.outlier_kv(B, Hkv, T, d, seed=62).to(cuda)
    V[0, 0, 512:576] *= 1000
    V[0, 0, 2048:2112] *= 1000
    kc, vc = c.quantize(K, tq.TQ_KEY), c.quantize(V, tq.TQ_VALUE)
    del K, V
    mb = T // bs
    perm = torch.randperm(B * mb, generator=torch.Generator().manual_seed(13)).to(torch.int32)
    kp, vp = _to_paged(kc, B, Hkv, T, bs, perm), _to_paged(vc, B, Hkv, T, bs, perm)
    table = perm.reshape(B, mb).clone()
    table[0, 0] = -1   # tokens [0, 64) masked
    lens = torch.tensor([T], dtype=torch.int32)
    q = tq_inputs.iid((B, Hq, d), seed=63, dtype=torch.bfloat16)
    got = c.attn_decode_paged(q.to(cuda), kp, vp, table.to(cuda), lens.to(cuda))
    torch.cuda.synchronize()
    G = Hq // Hkv
    kh = _drop_tokens(P.packed_np({k: (None if v is None else v[:, :1]) for k, v in kc.items()}), 0, 0, bs)
    vh = _drop_tokens(P.packed_np({k: (None if v is None else v[:, :1]) for k, v in vc.items()}), 0, 0, bs)
    P.check_attention(tab, q[:, :G].double().numpy(), kh, vh, np.array([T - bs]), 1,
                      got[:, :G].cpu().numpy())


@pytest.mark.parametrize("fmt,Hq", [("k3v4", 8), ("k4v4", 16), ("k3v4_nc", 8)])
def test_paged_decode_step_matches_oracle(cuda, fmt, Hq):
    """decode_step_paged against the oracle: the appended tokens are read back
    from the paged cache, which is gathered into contiguous order on the host,
    and the attention over [0, pos] is checked on the same codes."""
    c = tq.Context.variant(fmt, 128, seed=8)
    tab = P.oracle_tables(c)
    B, Hkv, d, max_T, bs = 4, 2, 128, 128, 32
    K = tq_inputs.outlier_kv(B, Hkv, max_T, d, seed=51).to(cuda)
    V = tq_inputs.outlier_kv(B, Hkv, max_T, d, seed=52).to(cuda)
    kc, vc = c.quantize(K, tq.TQ_KEY), c.quantize(V, tq.TQ_VALUE)
    mb = max_T // bs
    perm = torch.randperm(B * mb, generator=torch.Generator().manual_seed(9)).to(torch.int32)
    kp, vp = _to_paged(kc, B, Hkv, max_T, bs, perm), _to_paged(vc, B, Hkv, max_T, bs, perm)
    table = perm.reshape(B, mb)
    q = tq_inputs.iid((B, Hq, d), seed=53, dtype=torch.bfloat16).to(cuda)
    kn = tq_inputs.outlier_kv(B, Hkv, 1, d, seed=54)[:, :, 0].contiguous().to(cuda)
    vn = tq_inputs.outlier_kv(B, Hkv, 1, d, seed=55)[:, :, 0].contiguous().to(cuda)
    pos = torch.tensor([0, 40, 95, 127], dtype=torch.int32, device=cuda)
    got = c.decode_step_paged(q, kn, vn, kp, vp, table.to(cuda), pos)
    torch.cuda.synchronize()
    tn = table.numpy()
    kh = _from_paged(P.packed_np(kp), tn, B, bs)
    vh = _from_paged(P.packed_np(vp), tn, B, bs)
    # the appended records are the oracle's quantization of the new tokens
    for which, x, h in (("k", kn, kh), ("v", vn, vh)):
        recs = {k: (None if v is None else np.stack([v[b, :, int(pos[b])] for b in range(B)]).reshape(B * Hkv, -1)
                    if v.ndim > 3 else np.stack([v[b, :, int(pos[b])] for b in range(B)]).reshape(B * Hkv))
                for k, v in h.items()}
        P.check_quantized(tab, which, P.to_np(x.reshape(B * Hkv, d)), recs)
    lens = (pos + 1).cpu().numpy()
    P.check_attention(tab, q.double().cpu().numpy(), kh, vh, lens, Hkv, got.cpu().numpy())


def test_paged_rejections(cuda):
    c = _ctx(64, 2, 2, 0)
    q = torch.zeros(1, 2, 64, dtype=torch.bfloat16, device=cuda)
    kp = c.empty_packed(tq.TQ_KEY, (2, 1, 16), device=cuda)
    vp = c.empty_packed(tq.TQ_VALUE, (2, 1, 16), device=cuda)
    table = torch.zeros(1, 2, dtype=torch.int32, device=cuda)
    lens = torch.ones(1, dtype=torch.int32, device=cuda)
    with pytest.raises(tq.TQError) as e:
        c.attn_decode_paged(q, kp, vp, table, lens)
    assert e.value.status == tq.TQ_ERR_UNSUPPORTED
    c2 = _ctx(128, 3, 4, 128)
    q2 = torch.zeros(1, 4, 128, dtype=torch.bfloat16, device=cuda)
    kp2 = c2.empty_packed(tq.TQ_KEY, (2, 1, 24), device=cuda)
    vp2 = c2.empty_packed(tq.TQ_VALUE, (2, 1, 24), device=cuda)
    with pytest.raises(tq.TQError) as e:
        c2.attn_decode_paged(q2, kp2, vp2, table, lens)
    assert e.value.status == tq.TQ_ERR_ARG


@pytest.mark.parametrize("fmt,Hq,f16", [("k3v4", 8, False), ("k3v4", 16, False), ("k4v4", 8, False),
                                        ("k3v4_nc", 8, False), ("4bit_nc", 4, True)])
def test_decode_ignores_records_past_seq_len(cuda, fmt, Hq, f16):
    """Records at or past seq_lens[b] are not data: filled with NaN norms and
    all-ones codes they leave the output bit-identical to a clean cache.  The
    lengths are not multiples of 4 (or 8), so 16-byte norm copies reach past
    the end of each row.  Value norms spanning 2^-e .. 2^e inside a row
    exercise the fp16 scale of the value product (e = 13, or 5 where the
    norms are binary16, whose largest finite value is 65504)."""
    c = tq.Context.variant(fmt, 128, seed=17, norm_f16=f16)
    tab = P.oracle_tables(c)
    B, Hkv, T, d = 4, 2, 1104, 128
    K = tq_inputs.outlier_kv(B, Hkv, T, d, seed=91)
    V = tq_inputs.outlier_kv(B, Hkv, T, d, seed=92)
    e = 5 if f16 else 13
    V[:, :, :40] *= 2.0 ** -e
    V[:, :, 600:660] *= 2.0 ** e
    V[:, :, 900:905] *= 2.0 ** 6
    kc, vc = _cache(c, K, V, cuda)
    lens = torch.tensor([1101, 0, 619, 3], dtype=torch.int32)
    kp = {k: (None if v is None else v.clone()) for k, v in kc.items()}
    vp = {k: (None if v is None else v.clone()) for k, v in vc.items()}
    for cache in (kp, vp):
        for k, v in cache.items():
            if v is None:
                continue
            for b in range(B):
                if v.is_floating_point():
                    v[b, :, int(lens[b]):] = float("nan")
                else:
                    v[b, :, int(lens[b]):] = 0xFF
    Q = tq_inputs.iid((B, Hq, d), seed=93, dtype=torch.bfloat16)
    out = c.attn_decode(Q.to(cuda), kc, vc, lens.to(cuda))
    outp = c.attn_decode(Q.to(cuda), kp, vp, lens.to(cuda))
    torch.cuda.synchronize()
    assert torch.isfinite(outp).all()
    assert torch.equal(out, outp)
    P.check_attention(tab, Q.double().numpy(), P.packed_np(kc), P.packed_np(vc), lens.numpy(), Hkv,
                      out.cpu().numpy())


@pytest.mark.parametrize("name,f16,dtype", [("k3v4_nc", False, torch.bfloat16), ("k3v4_nc", True, torch.float16),
                                            ("4bit_nc", True, torch.float16), ("3bit_nc", False, torch.bfloat16),
                                            ("k8v4", True, torch.bfloat16), ("k8v4", False, torch.float16)])
def test_quantize_tensor_core_norm_variants(cuda, name, f16, dtype):
    """Norm-corrected formats and binary16 norms on the tensor-core quantize
    (16-bit input, more than 4096 vectors, row pitch 136, a zero row, a
    ragged last tile): codes and stored norms against the oracle; an append
    of 6144 rows at per-sequence slots equals the bulk call on the same rows
    and leaves the other slots alone.  k8v4 keys take the 8-bit codes of the
    same kernel (thresholds in a breadth-first search tree)."""
    c = tq.Context.variant(name, 128, seed=23, norm_f16=f16)
    tab = P.oracle_tables(c)
    n = 6000
    X = tq_inputs.outlier_kv(1, 1, n, 128, seed=24)[0, 0].to(dtype)
    X[11] = 0
    big = torch.zeros(n, 136, dtype=dtype)
    big[:, :128] = X
    src = big.to(cuda)[:, :128]
    for which, wch in ((tq.TQ_KEY, "k"), (tq.TQ_VALUE, "v")):
        pk = c.empty_packed(which, (n,))
        c.quantize_into(src, which, pk)
        torch.cuda.synchronize()
        assert tq.tq_device_fault() == 0
        assert pk["norm"].dtype == (torch.float16 if f16 else torch.float32)
        P.check_quantized(tab, wch, X.double().numpy(), _flat(pk, n))
    B, H, T = 64, 96, 5
    x = tq_inputs.outlier_kv(B, H, 1, 128, seed=25)[:, :, 0].to(dtype).contiguous().to(cuda)
    pos = torch.randint(0, T, (B,), generator=torch.Generator().manual_seed(4), dtype=torch.int32)
    pos[3], pos[50] = -1, T
    pos = pos.to(cuda)
    ok = (pos >= 0) & (pos < T)
    for which in (tq.TQ_KEY, tq.TQ_VALUE):
        cache = c.empty_packed(which, (B, H, T), device=cuda)
        for v in cache.values():
            if v is not None:
                v.fill_(-7)
        c.quantize_append(x, which, cache, pos)
        ref = c.quantize(x.reshape(B * H, 128), which)
        torch.cuda.synchronize()
        for k, v in cache.items():
            if v is None:
                continue
            want = ref[k].reshape((B, H) + tuple(v.shape[3:]))
            bs = torch.arange(B, device=cuda)[ok]
            assert torch.equal(v[bs, :, pos[ok].long()], want[ok]), k
            assert torch.all(v[~ok] == -7), k
