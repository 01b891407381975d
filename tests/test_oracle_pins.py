"""Pins of the fp64 oracle to facts fixed outside itself: published test
vectors and tables, closed forms, the probability laws the method rests on,
invariants, and brute force on tiny inputs.  CPU only."""
import math
from pathlib import Path

import numpy as np
import pytest
from scipy import integrate, stats
from scipy.special import gammaln

from oracle import tq_oracle as o

GOLDEN = Path(__file__).resolve().parent / "golden"


def _golden_lines(name):
    return [ln.split() for ln in (GOLDEN / name).read_text().splitlines()
            if ln.strip() and not ln.startswith("#")]


# --- R9: random numbers ------------------------------------------------------
def test_splitmix64_published_vector():
    want = [int(t[0]) for t in _golden_lines("splitmix64_seed1234567.txt")]
    got = [int(v) for v in o.splitmix64_sequence(1234567, 5)]
    assert got == want


def test_normals_are_standard_normal():
    z = o.stream_normals(123, 0, 200_000)
    assert abs(z.mean()) < 4 / math.sqrt(z.size)
    assert abs(z.var() - 1) < 4 * math.sqrt(2 / z.size)
    assert stats.kstest(z, "norm").pvalue > 1e-3


def test_streams_differ_and_repeat():
    a = o.stream_draws(5, 0, 64)
    assert np.array_equal(a, o.stream_draws(5, 0, 64))
    assert not np.array_equal(a, o.stream_draws(5, 1, 64))
    assert not np.array_equal(a, o.stream_draws(6, 0, 64))


# --- R8: rotation -------------------------------------------------------------
@pytest.mark.parametrize("d", [8, 64, 128, 200])
def test_rotation_orthogonal_and_sign_convention(d):
    Pi = o.rotation(d, 11)
    assert np.abs(Pi.T @ Pi - np.eye(d)).max() < 1e-12
    assert abs(abs(np.linalg.det(Pi)) - 1) < 1e-10
    # G = Pi R with R upper triangular and a positive diagonal.
    R = Pi.T @ o.gaussian_matrix(d, 11)
    assert np.abs(np.tril(R, -1)).max() < 1e-10
    assert np.all(np.diag(R) > 0)


def test_rotation_is_applied_as_pi_times_x():
    d = 32
    tab = o.make_tables(d, 3, 3, 32, 3)
    # x = row j of Pi = Pi^T e_j must rotate to y = e_j exactly (up to rounding).
    q = o.quantize(tab.Pi[:5] * 3.0, tab, "v")
    assert np.allclose(q.y, np.eye(d)[:5], atol=1e-12)
    assert np.allclose(q.norm, 3.0)
    top = len(tab.cb_v.centroids) - 1
    for j in range(5):
        assert q.idx[j, j] == top
        # the other coordinates are 0 up to rounding: the two cells around 0
        assert np.all(np.abs(np.delete(q.idx[j], j) - len(tab.cb_v.centroids) / 2 + 0.5) == 0.5)


# --- R2: the Beta law of rotated coordinates --------------------------------
@pytest.mark.parametrize("d", [16, 128])
def test_rotated_coordinates_follow_beta_law(d):
    rng = np.random.default_rng(0)
    tab = o.make_tables(d, 2, 2, 0, 9)
    # Uniformly random directions (isotropic Gaussian rows) rotated by Pi.
    u = rng.standard_normal((100_000, d))
    y = o.quantize(u, tab, "v").y[:, 3]
    a = (d - 1) / 2
    assert stats.kstest(y, lambda t: stats.beta.cdf((1 + t) / 2, a, a)).pvalue > 1e-3
    assert abs(np.var(y) * d - 1) < 0.02
    # The density helper integrates to 1 and matches the histogram.
    assert abs(integrate.quad(lambda t: o.beta_density(np.array([t]), d)[0], -1, 1)[0] - 1) < 1e-10


# --- R2 / Lloyd-Max codebook ------------------------------------------------
@pytest.mark.parametrize("d,bits", [(128, 1), (128, 2), (128, 3), (128, 4), (200, 3), (37, 2), (128, 8)])
def test_lloyd_max_fixed_point(d, bits):
    cb = o.lloyd_max(d, bits)
    L = 1 << bits
    assert len(cb.centroids) == L and len(cb.boundaries) == L - 1
    assert np.allclose(cb.centroids, -cb.centroids[::-1], atol=0)
    assert np.all(np.diff(cb.centroids) > 0)
    assert np.allclose(cb.boundaries, 0.5 * (cb.centroids[:-1] + cb.centroids[1:]), atol=1e-15)
    # Centroid condition checked with an independent quadrature of f_d.
    f = lambda t: o.beta_density(np.array([t]), d)[0]
    edges = np.concatenate([[-1.0], cb.boundaries, [1.0]])
    s = 1 / math.sqrt(d)
    for i in range(L):
        lo, hi = edges[i], edges[i + 1]
        pts = [p for p in (-5 * s, 0.0, 5 * s) if lo < p < hi]
        m0 = integrate.quad(f, lo, hi, points=pts or None, epsabs=1e-15, epsrel=1e-13, limit=400)[0]
        m1 = integrate.quad(lambda t: t * f(t), lo, hi, points=pts or None, epsabs=1e-16,
                            epsrel=1e-13, limit=400)[0]
        assert abs(m1 / m0 - cb.centroids[i]) < 1e-11 * max(1.0, abs(cb.centroids[i]) * math.sqrt(d))


@pytest.mark.parametrize("d", [16, 128, 200])
def test_one_bit_closed_form(d):
    want = math.exp(gammaln(d / 2) - gammaln((d + 1) / 2)) / math.sqrt(math.pi)  # E|T|
    assert abs(o.lloyd_max(d, 1).centroids[1] - want) < 1e-14


def test_large_d_limit_is_max_gaussian_table():
    d = 20001
    for row in _golden_lines("max1960_gaussian.txt"):
        levels = int(row[0])
        outs = np.array([float(t) for t in row[1:-1]])
        mse = float(row[-1])
        cb = o.lloyd_max(d, int(math.log2(levels)), max_iter=5000)
        got = cb.centroids[levels // 2:] * math.sqrt(d)
        assert np.allclose(got, outs, atol=2e-3), (levels, got, outs)
        assert abs(o.distortion(d, cb) - mse) < 2e-3 * mse + 5e-5


@pytest.mark.parametrize("bits", [1, 2, 3, 4, 8])
def test_empirical_mse_within_two_percent(bits):
    d = 128
    tab = o.make_tables(d, bits, bits, 0, 21)
    rng = np.random.default_rng(bits)
    x = rng.standard_normal((40_000, d)) * 3.7
    q = o.quantize(x, tab, "v")
    emp = d * np.mean((q.y - tab.cb_v.centroids[q.idx]) ** 2)
    ref = o.distortion(d, tab.cb_v)
    assert abs(emp / ref - 1) < 0.02


# --- R13: norm correction ------------------------------------------------------
@pytest.mark.parametrize("d", [64, 128])
def test_norm_correction_one_bit_closed_form(d):
    """At 1 bit every rotated coordinate maps to +-c1 with c1 = E|T| (closed
    form), so |c[idx]| = sqrt(d) c1 for every vector and the stored norm is
    n / (sqrt(d) c1)."""
    c1 = math.exp(gammaln(d / 2) - gammaln((d + 1) / 2)) / math.sqrt(math.pi)
    tab = o.make_tables(d, 1, 1, 0, 5, nc_k=True, nc_v=True)
    x = np.random.default_rng(3).standard_normal((500, d)) * 2.5
    n = np.linalg.norm(x, axis=1)
    for which in ("k", "v"):
        q = o.quantize(x, tab, which)
        want = n / (math.sqrt(d) * c1)
        assert np.all(np.abs(q.norm - want) <= 1e-7 * want)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_norm_correction_keeps_the_norm(bits):
    """Under norm correction the dequantized vector has the input's norm
    (up to the fp32 rounding of the stored scalar); the codes are unchanged."""
    d = 128
    x = np.random.default_rng(bits).standard_normal((2000, d)) * 0.3
    x[7] = 0.0
    n = np.linalg.norm(x, axis=1)
    tab = o.make_tables(d, bits, bits, 0, 9, nc_k=True, nc_v=True)
    plain = o.make_tables(d, bits, bits, 0, 9)
    for which in ("k", "v"):
        q = o.quantize(x, tab, which)
        xh = o.dequantize(tab, which, q.codes, q.norm)
        assert np.all(np.abs(np.linalg.norm(xh, axis=1) - n) <= 2e-7 * n)
        assert q.norm[7] == 0.0 and np.all(xh[7] == 0.0)
        qp = o.quantize(x, plain, which)
        assert np.array_equal(qp.codes, q.codes)


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_norm_correction_mean_square_is_one_minus_distortion(bits):
    """Lloyd-Max centroids are cell means, so E|c[idx]|^2 = E|y|^2 - E|y - c|^2
    = 1 - D_b: the mean of (n / stored)^2 over uniform directions must match
    the codebook's distortion."""
    d = 128
    tab = o.make_tables(d, bits, bits, 0, 13, nc_v=True)
    x = np.random.default_rng(40 + bits).standard_normal((40_000, d))
    q = o.quantize(x, tab, "v")
    ratio2 = (np.linalg.norm(x, axis=1) / q.norm.astype(np.float64)) ** 2
    assert abs(ratio2.mean() - (1.0 - o.distortion(d, tab.cb_v))) < 3e-3


@pytest.mark.parametrize("bits", [3, 4])
def test_binary16_norms(bits):
    """Binary16 norms: the stored scalar is the fp64 value rounded to the
    nearest binary16, so the dequantized vector keeps the corrected norm to
    half a binary16 step (2^-11 relative), and QJL keys are refused."""
    d = 128
    x = np.random.default_rng(bits + 60).standard_normal((3000, d)) * 7.0
    n = np.linalg.norm(x, axis=1)
    tab = o.make_tables(d, bits, bits, 0, 4, nc_k=True, nc_v=True, norm_f16=True)
    for which in ("k", "v"):
        q = o.quantize(x, tab, which)
        assert q.norm.dtype == np.float16
        xh = o.dequantize(tab, which, q.codes, q.norm)
        assert np.all(np.abs(np.linalg.norm(xh, axis=1) - n) <= 2.0 ** -11 * n * (1 + 1e-9))
    with pytest.raises(ValueError):
        o.make_tables(d, bits, bits, 64, 4, norm_f16=True)


def test_norm_correction_needs_mse_only_keys():
    with pytest.raises(ValueError):
        o.make_tables(64, 3, 4, 64, 1, nc_k=True)


@pytest.mark.parametrize("d", [128, 200])
def test_eight_bit_distortion_near_panter_dite(d):
    """High-resolution theory (Panter & Dite 1951): with L levels the least
    mean-square distortion tends to (int f^(1/3))^3 / (12 L^2).  At 256 levels
    the 8-bit codebook must sit just below it (within 1.5 %), and the 4-bit
    one visibly further below (the bound is asymptotic)."""
    f3 = integrate.quad(lambda t: o.beta_density(np.array([t]), d)[0] ** (1 / 3), -1, 1, points=[0],
                        limit=400, epsabs=1e-14)[0]
    for bits, lo, hi in ((8, -0.015, 0.0), (4, -0.15, -0.05)):
        pd = d * f3 ** 3 / (12 * (1 << bits) ** 2)
        ratio = o.distortion(d, o.lloyd_max(d, bits)) / pd - 1
        assert lo < ratio < hi, (bits, ratio)


def test_printed_three_bit_cosine():
    want = float(_golden_lines("page_claims.txt")[0][1])
    d = 128
    cb = o.lloyd_max(d, 3)
    assert abs(math.sqrt(1 - o.distortion(d, cb)) - want) < 1e-3
    tab = o.make_tables(d, 3, 3, 0, 2)
    x = np.random.default_rng(7).standard_normal((20_000, d))
    q = o.quantize(x, tab, "v")
    xh = o.dequantize(tab, "v", q.codes, q.norm)
    cos = np.sum(x * xh, axis=1) / (np.linalg.norm(x, axis=1) * np.linalg.norm(xh, axis=1))
    assert abs(cos.mean() - want) < 1e-3


# --- packing ---------------------------------------------------------------
def test_packing_worked_example():
    rows = {r[0]: [int(t, 16) for t in r[1:]] for r in _golden_lines("packing_fields.txt")}
    for bits in (1, 2, 3, 4):
        idx = (np.arange(40) % (1 << bits))[None, :]
        codes = o.pack_codes(idx, bits)
        assert codes.dtype == np.uint32 and codes.shape == (1, o.code_words(40, bits))
        assert list(codes[0]) == rows[f"b{bits}"], bits
        assert np.array_equal(o.unpack_codes(codes, bits, 40), idx)
    # 8-bit codes (the k8v4 format): one byte per coordinate, LSB first
    idx = (np.arange(40) ^ 0xA0)[None, :]
    codes = o.pack_codes(idx, 8)
    assert codes.dtype == np.uint32 and codes.shape == (1, o.code_words(40, 8)) == (1, 10)
    assert list(codes[0]) == rows["b8"]
    assert np.array_equal(o.unpack_codes(codes, 8, 40), idx)


def test_pack_roundtrip_random():
    rng = np.random.default_rng(1)
    for bits in (1, 2, 3, 4, 8):
        for d in (200, 128, 8, 36):
            idx = rng.integers(0, 1 << bits, size=(50, d))
            assert np.array_equal(o.unpack_codes(o.pack_codes(idx, bits), bits, d), idx)
    bits = rng.integers(0, 2, size=(50, 72))
    w = o.pack_bits(bits)
    assert w.shape == (50, 3) and np.all(w[:, 2] >> np.uint32(8) == 0)
    assert np.array_equal(o.unpack_bits(w, 72), bits)


# --- agreement counts used to report excused indices -----------------------------
def test_code_agreement_counts():
    """The counting helper: identical codes give no mismatch, a planted
    mismatch far from every boundary is a real disagreement, and the in-band
    counts over uniform directions match the integrated density at the
    boundaries, sum_i 2 band f_d(beta_i) per coordinate, on the unit scale and
    sqrt(d) times fewer on the standardized scale."""
    d = 128
    tab = o.make_tables(d, 3, 2, d, 5)   # keys: 2 Lloyd-Max bits + QJL (m = d); values: 2 bits
    rng = np.random.default_rng(7)
    x = rng.standard_normal((20000, d))
    q = o.quantize(x, tab, "k")
    c = o.code_agreement(tab, "k", x, q.codes, q.qjl)
    assert c["indices"] == x.size and c["mismatches"] == 0 and c["outside_band"] == 0
    assert c["qjl_bits"] == x.size and c["qjl_mismatches"] == 0
    idx = q.idx.copy()
    far = int(np.argmax(o.boundary_distance(q.y, tab.cb_k).ravel()))
    r, j = divmod(far, d)
    idx[r, j] ^= 1
    c2 = o.code_agreement(tab, "k", x, o.pack_codes(idx, 2))
    assert (c2["mismatches"], c2["outside_band"], c2["mismatches_outside_std_band"]) == (1, 1, 1)
    band = 1e-5
    expect = x.size * float(np.sum(2 * band * o.beta_density(tab.cb_k.boundaries, d)))
    for got, mean in ((c["in_band_unit"], expect), (c["in_band_std"], expect / math.sqrt(d))):
        assert abs(got - mean) <= 5 * math.sqrt(mean), (got, mean)


# --- R14: zero vector ---------------------------------------------------------
def test_zero_vector():
    tab = o.make_tables(64, 3, 2, 64, 4)
    q = o.quantize(np.zeros((2, 64)), tab, "k")
    assert np.all(q.idx == 2) and np.all(q.norm == 0) and np.all(q.rnorm == 0)
    l = o.logits(tab, np.ones((1, 64)), q.codes, q.norm, q.qjl, q.rnorm)
    assert np.all(l == 0)


# --- QJL: unbiased inner products (stage 2) -----------------------------------
def test_qjl_estimator_is_unbiased_and_mse_stage_is_not():
    d = m = 64
    seeds, per = 1000, 100  # 1e5 pairs; S and Pi redrawn per seed
    cb = o.lloyd_max(d, 2)
    rng = np.random.default_rng(3)
    err_q, err_mse = [], []
    for sd in range(seeds):
        tab = o.Tables(d, 2, 2, m, sd, o.rotation(d, sd), o.qjl_matrix(m, d, sd), cb, cb)
        k = rng.standard_normal((per, d)) * rng.uniform(0.5, 2.0, size=(per, 1))
        qv = k + 0.3 * rng.standard_normal((per, d))          # correlated query
        z = o.quantize(k, tab, "k")
        est = np.einsum("ij,ij->i", np.eye(per), o.logits(tab, qv, z.codes, z.norm, z.qjl, z.rnorm))
        mse_only = np.einsum("ij,ij->i", np.eye(per),
                             o.logits(o.Tables(d, 2, 2, 0, sd, tab.Pi, None, cb, cb), qv, z.codes, z.norm))
        true = np.sum(qv * k, axis=1)
        err_q.append(np.mean(est - true))
        err_mse.append(np.mean(mse_only - true))
    err_q, err_mse = np.array(err_q), np.array(err_mse)
    se = err_q.std(ddof=1) / math.sqrt(seeds)
    assert abs(err_q.mean()) < 3 * se
    # The MSE stage alone under-estimates <q, k> (the bias QJL removes).
    assert err_mse.mean() < -10 * err_mse.std(ddof=1) / math.sqrt(seeds)


# --- logits from codes = dot with the dequantized key ----------------------
def test_logits_equal_dot_with_dequantized_keys():
    tab = o.make_tables(128, 3, 4, 128, 0)
    rng = np.random.default_rng(2)
    k = rng.standard_normal((300, 128)) * 2
    qv = rng.standard_normal((5, 128))
    z = o.quantize(k, tab, "k")
    kh = o.dequantize(tab, "k", z.codes, z.norm, z.qjl, z.rnorm)
    l = o.logits(tab, qv, z.codes, z.norm, z.qjl, z.rnorm)
    assert np.abs(l - qv @ kh.T).max() < 1e-11 * np.abs(l).max()


# --- attention: brute force and special cases ----------------------------------
def _cache(tab, B, Hkv, T, rng):
    k = rng.standard_normal((B, Hkv, T, tab.d))
    v = rng.standard_normal((B, Hkv, T, tab.d))
    zk = o.quantize(k.reshape(-1, tab.d), tab, "k")
    zv = o.quantize(v.reshape(-1, tab.d), tab, "v")
    r = lambda a, *tail: None if a is None else a.reshape((B, Hkv, T) + tail)
    mw = (tab.qjl_m + 31) // 32
    return (r(zk.codes, o.code_words(tab.d, tab.bits_k_lm)), r(zk.qjl, mw), r(zk.norm), r(zk.rnorm),
            r(zv.codes, o.code_words(tab.d, tab.bits_v)), r(zv.norm))


def test_attention_brute_force_tiny():
    tab = o.make_tables(16, 3, 2, 16, 5)
    rng = np.random.default_rng(4)
    B, Hq, Hkv, T = 2, 4, 2, 7
    kc, kq, kn, kr, vc, vn = _cache(tab, B, Hkv, T, rng)
    q = rng.standard_normal((B, Hq, 16))
    lens = np.array([7, 3])
    out = o.attention(tab, q, kc, kq, kn, kr, vc, vn, lens, Hkv, scale=0.7)
    for b in range(B):
        for h in range(Hq):
            g = h // (Hq // Hkv)
            K = o.dequantize(tab, "k", kc[b, g, :lens[b]], kn[b, g, :lens[b]], kq[b, g, :lens[b]], kr[b, g, :lens[b]])
            V = o.dequantize(tab, "v", vc[b, g, :lens[b]], vn[b, g, :lens[b]])
            s = 0.7 * (K @ q[b, h])
            w = np.exp(s) / np.exp(s).sum()
            assert np.allclose(out[b, h], w @ V, rtol=1e-12, atol=1e-12)


def test_attention_special_cases():
    tab = o.make_tables(16, 2, 3, 0, 6)
    rng = np.random.default_rng(8)
    kc, kq, kn, kr, vc, vn = _cache(tab, 3, 1, 5, rng)
    q = rng.standard_normal((3, 2, 16))
    out = o.attention(tab, q, kc, kq, kn, kr, vc, vn, np.array([0, 1, 5]), 1)
    assert np.all(out[0] == 0)                                     # empty context
    v0 = o.dequantize(tab, "v", vc[1, 0, :1], vn[1, 0, :1])[0]
    assert np.allclose(out[1], v0[None, :], atol=1e-13)            # one token: o = v_hat
    out0 = o.attention(tab, q, kc, kq, kn, kr, vc, vn, np.array([0, 1, 5]), 1, scale=0.0)
    V = o.dequantize(tab, "v", vc[2, 0], vn[2, 0])
    assert np.allclose(out0[2], V.mean(axis=0)[None, :], atol=1e-13)   # scale 0: uniform weights


# --- top-k ---------------------------------------------------------------------
def test_topk_brute_force_and_tie_order():
    tab = o.make_tables(24, 3, 3, 24, 1)
    rng = np.random.default_rng(5)
    x = rng.standard_normal((60, 24))
    x[10] = x[3]  # duplicate -> equal scores, lower index first
    z = o.quantize(x, tab, "k")
    qv = rng.standard_normal((4, 24))
    idx, val, scores = o.topk(tab, qv, z.codes, z.norm, z.qjl, z.rnorm, 12)
    for i in range(4):
        pairs = sorted(range(60), key=lambda j: (-scores[i, j], j))[:12]
        assert list(idx[i]) == pairs
        assert np.all(np.diff(val[i]) <= 0)
        if 3 in idx[i] and 10 in idx[i]:
            assert list(idx[i]).index(3) < list(idx[i]).index(10)
