"""Comparison rules between the CUDA path and the fp64 oracle (tests only).

Rules (stated tolerances of the method's specification):
  * Lloyd-Max indices and QJL bits are bit-exact, except indices whose rotated
    unit-vector coordinate lies within BAND = 1e-5 of a decision boundary and
    QJL bits whose |(S r)_i| is within BAND * |r| of 0; such mismatches are
    counted and must be at most 1e-4 of all indices (of all bits).
  * The packed words are exactly the canonical packing of the indices (layout
    and zero padding).
  * |x| agrees to a relative 1e-6.  gamma = |x| |r| agrees to a relative 1e-5
    (against the oracle's sketch rebuilt from the CUDA path's indices): gamma
    only scales the QJL logit term sqrt(pi/2)/m * gamma * <S q', sigma>, whose
    size is at most ~|q| |x| |r|, so a 1e-5 relative error moves a logit by
    < 1e-5 |q| |k|, two orders inside the 1e-3 |q| |k| logit tolerance.  The
    residual norm |r| is small (0.1-0.35) and the rotation is accumulated on
    tensor cores with ~1e-6 absolute error per coordinate.
  * Logits agree to |d| <= 1e-3 |q| |k| given identical codes.
  * Attention outputs agree to relative L2 <= 2e-3 per (sequence, head).
"""
import numpy as np
import torch

from oracle import tq_oracle as o

BAND = 1e-5
MAX_EXCUSED_FRAC = 1e-4
NORM_RTOL = 1e-6
RNORM_RTOL = 1e-5
LOGIT_TOL = 1e-3
ATTN_RTOL = 2e-3


def to_np(t):
    if t is None:
        return None
    a = t.detach().cpu()
    if a.dtype == torch.int32:
        return a.numpy().view(np.uint32)
    if a.dtype == torch.bfloat16 or a.dtype == torch.float16:
        return a.float().numpy().astype(np.float64)
    return a.numpy()


def packed_np(p):
    return {k: to_np(v) for k, v in p.items()}


def oracle_tables(ctx):
    return o.make_tables(ctx.d, ctx.bits_k, ctx.bits_v, ctx.qjl_m, ctx.seed,
                         nc_k=getattr(ctx, "nc_k", False), nc_v=getattr(ctx, "nc_v", False),
                         norm_f16=getattr(ctx, "norm_f16", False))


def check_quantized(tab, which, x, gpu, report=None):
    """x: fp64 [n, d] (the exact input values); gpu: numpy dict of the CUDA
    outputs flattened to [n, ...]."""
    d = tab.d
    cb = tab.cb_k if which == "k" else tab.cb_v
    n = x.shape[0]
    q = o.quantize(x, tab, which)
    codes = gpu["codes"].reshape(n, -1)
    assert codes.shape[1] == o.code_words(d, cb.bits)
    gidx = o.unpack_codes(codes, cb.bits, d)
    assert np.array_equal(codes, o.pack_codes(gidx, cb.bits)), "non-canonical packing"
    mism = gidx != q.idx
    band = o.boundary_distance(q.y, cb) < BAND
    assert not np.any(mism & ~band), f"{int(np.sum(mism & ~band))} index mismatches outside the band"
    n_exc = int(mism.sum())
    assert n_exc <= MAX_EXCUSED_FRAC * mism.size, f"{n_exc} excused indices"
    gnorm = gpu["norm"].reshape(n).astype(np.float64)
    onorm = np.sqrt(np.sum(x * x, axis=1))
    # R13: under norm correction the stored scalar is n / |c[idx]|, taken on
    # the CUDA path's own indices (an excused index changes |c[idx]|)
    want = o.corrected_norm(onorm, gidx, cb) if (tab.nc_k if which == "k" else tab.nc_v) else onorm
    if tab.norm_f16:
        # binary16: the CUDA path rounds its fp32 value, the oracle its fp64 value; they agree to
        # one binary16 step (2^-10 relative), and both are representable binary16 values
        assert np.array_equal(gnorm, gnorm.astype(np.float16).astype(np.float64)), "norm not binary16"
        assert np.all(np.abs(gnorm - want) <= 2.0 ** -10 * want + 1e-30), "norm"
    else:
        assert np.all(np.abs(gnorm - want) <= NORM_RTOL * want + 1e-30), "norm"
    dist = o.boundary_distance(q.y, cb)
    band_std = dist < BAND / np.sqrt(d)
    stats = {"indices": int(mism.size), "excused": n_exc, "band": int(band.sum()),
             "band_std": int(band_std.sum()), "excused_outside_std_band": int(np.sum(mism & ~band_std))}
    if which == "k" and tab.qjl_m > 0:
        o.sketch_from_indices(q, tab, idx=gidx)
        gbits = o.unpack_bits(gpu["qjl"].reshape(n, -1), tab.qjl_m)
        assert np.array_equal(gpu["qjl"].reshape(n, -1), o.pack_bits(gbits)), "non-canonical QJL packing"
        qm = gbits != q.qjl_bits
        qband = np.abs(q.proj) < BAND * q.rho[:, None]
        assert not np.any(qm & ~qband), f"{int(np.sum(qm & ~qband))} QJL mismatches outside the band"
        assert int(qm.sum()) <= MAX_EXCUSED_FRAC * qm.size
        orn = onorm * q.rho
        grn = gpu["rnorm"].reshape(n).astype(np.float64)
        assert np.all(np.abs(grn - orn) <= RNORM_RTOL * orn + 1e-30), "rnorm"
        stats.update(qjl_bits=int(qm.size), qjl_excused=int(qm.sum()))
    if report is not None:
        report.append(stats)
    return stats


def check_logits(tab, q, gpu_keys, gpu_logits):
    """q: fp64 [nq, d]; gpu_keys: numpy dict [nk, ...]; gpu_logits [nq, nk]."""
    nk = gpu_keys["norm"].size
    ref = o.logits(tab, q, gpu_keys["codes"].reshape(nk, -1),
                   gpu_keys["norm"].reshape(nk),
                   None if gpu_keys.get("qjl") is None else gpu_keys["qjl"].reshape(nk, -1),
                   None if gpu_keys.get("rnorm") is None else gpu_keys["rnorm"].reshape(nk))
    bound = LOGIT_TOL * np.linalg.norm(q, axis=1)[:, None] * gpu_keys["norm"].reshape(1, nk)
    err = np.abs(gpu_logits - ref)
    assert np.all(err <= bound + 1e-30), float((err / (bound + 1e-30)).max())
    return ref


def check_attention(tab, q, kc, vc, lens, Hkv, gpu_out, scale=None, pairs=None):
    """kc / vc: numpy dicts of [B, Hkv, T, ...] arrays from the CUDA path."""
    B, Hq, d = q.shape
    pairs = [(b, h) for b in range(B) for h in range(Hq)] if pairs is None else pairs
    worst = 0.0
    for b, h in pairs:
        ref = o.attention(tab, q, kc["codes"], kc.get("qjl"), kc["norm"], kc.get("rnorm"),
                          vc["codes"], vc["norm"], lens, Hkv, scale=scale,
                          batches=[b], heads=[h])[b, h]
        got = gpu_out[b, h].astype(np.float64)
        if lens[b] == 0:
            assert np.all(got == 0), (b, h)
            continue
        rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
        worst = max(worst, rel)
        assert rel <= ATTN_RTOL, (b, h, rel)
    return worst
