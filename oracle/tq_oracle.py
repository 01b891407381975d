"""Plain fp64 CPU oracle for TurboQuant-style K/V quantization and decode attention.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
execute this module: only the tests, the smoke check and the benchmark's
CPU-baseline arm use it.  It shares no code with the CUDA library (no tables,
no helpers); both sides implement the same published definitions
independently.  Every step is written the slow, obvious way in float64 with
numpy; library primitives (matmul, QR, the regularised incomplete beta
function) serve as single steps.

Sources, by page title and section (the pages are web articles):
  [WHAT]  a2a-mcp.org, "什么是TurboQuant？谷歌突破性AI压缩技术实现6倍KV缓存缩减和8倍推理加速"
          ("What is TurboQuant?"), section "TurboQuant 工作原理：技术深度解析"
          ("How TurboQuant works"): stage 1 step 1 (random orthogonal rotation,
          Beta law of rotated coordinates), stage 1 step 2 (normalisation and
          the Lloyd-Max quantizer for the Beta law), stage 2 (1-bit QJL
          residual correction), and the closing paragraph of that section
          (attention logits straight from compressed indices); section
          "如何实现 TurboQuant：分步指南" ("How to implement"), part 1
          (per-dimension Lloyd-Max codebooks; the fused kernel pre-rotates the
          query once and takes dot products from the indices).
  [VLLM]  papercache.org, "A First Comprehensive Study of TurboQuant: Accuracy
          and Performance", sections A2 and A3 (the KV cache is dequantized
          for the attention over values).

Where the pages leave a step open, the reading taken is named R<k> below:
  R2  Beta((d-1)/2,(d-1)/2) on [-1,1] is the affine image of Beta(a,a) on
      [0,1]: density proportional to (1-t^2)^((d-3)/2), the exact law of one
      coordinate of a uniform unit vector.
  R3  Key bit budget counts the QJL bit: k3 = 2 Lloyd-Max bits + 1 QJL bit.
  R4  The per-vector norm is stored (fp32); "zero overhead" on [WHAT] means no
      per-block scale or zero point.
  R5  S is m x d with i.i.d. N(0,1) entries, drawn on its own RNG stream and
      rounded to fp16 (round to nearest even); the rounded values are the
      definition of S.  It acts on the rotated residual.
  R6  sign(0) = +1; a stored QJL bit 1 means +1.
  R7  A coordinate exactly on a boundary goes to the upper cell (y >= beta).
  R8  Pi = Q diag(sgn(diag R)) from the Householder QR of G (sgn(0)=+1), so
      Pi^T G is upper triangular with a positive diagonal; y = Pi x.
  R9  RNG: SplitMix64 (Steele, Lea & Flood 2014).  Stream s of seed has
      state0 = mix(seed + (s+1)*gamma); draw i is mix(state0 + (i+1)*gamma).
      uniform = ((z >> 11) + 0.5) * 2^-53; normal = sqrt(-2 ln u1) cos(2 pi u2)
      (Box-Muller, two draws per normal).  Stream 0 fills G, stream 1 fills S,
      row-major.
  R11 Logits returned by `logits` are the unscaled <q,k>; attention scales
      them by `scale` (1/sqrt(d) by default).
  R12 Values are MSE-stage only; key dequantization includes the QJL
      back-projection, so logits(q, codes) = <q, dequantize(codes)>.
  R13 "Norm correction" (the _nc variants named in [VLLM] A3) is not
      defined on the pages.  Reading: the stored norm becomes n / |c[idx]|,
      so the dequantized vector n Pi^T c[idx] / |c[idx]| keeps the input's
      norm exactly.  It applies to MSE-only vectors: values, and keys without
      the QJL stage (the variants name no QJL bit).
  R14 A zero vector has n = 0, u = 0, every index L/2, gamma = 0.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
from scipy.linalg import solve_banded
from scipy.special import betaincc, gammaln

# ----------------------------------------------------------------------------
# R9: SplitMix64 counter generator, uniforms and Box-Muller normals.
# ----------------------------------------------------------------------------
_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)


def splitmix64_mix(z: np.ndarray) -> np.ndarray:
    """The SplitMix64 output function applied elementwise to uint64 values."""
    z = np.asarray(z, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def splitmix64_sequence(state: int, count: int) -> np.ndarray:
    """Outputs 1..count of the plain SplitMix64 generator started at `state`
    (each call adds gamma to the state, then mixes)."""
    i = np.arange(1, count + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return splitmix64_mix(np.uint64(state) + i * _GAMMA)


def stream_draws(seed: int, stream: int, count: int) -> np.ndarray:
    """R9: `count` raw 64-bit draws of stream `stream` of `seed`."""
    state0 = int(splitmix64_sequence(seed, stream + 1)[stream])
    return splitmix64_sequence(state0, count)


def stream_uniforms(seed: int, stream: int, count: int) -> np.ndarray:
    z = stream_draws(seed, stream, count)
    return ((z >> np.uint64(11)).astype(np.float64) + 0.5) * 2.0 ** -53


def stream_normals(seed: int, stream: int, count: int) -> np.ndarray:
    u = stream_uniforms(seed, stream, 2 * count)
    u1, u2 = u[0::2], u[1::2]
    return np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * math.pi * u2)


# ----------------------------------------------------------------------------
# [WHAT] stage 1 step 1: random orthogonal rotation from the QR of a Gaussian
# matrix (R8), and the QJL projection matrix (R5).
# ----------------------------------------------------------------------------
def gaussian_matrix(d: int, seed: int) -> np.ndarray:
    return stream_normals(seed, 0, d * d).reshape(d, d)


def rotation(d: int, seed: int) -> np.ndarray:
    """Pi = Q diag(sgn(diag R)) where G = QR (Householder, LAPACK) - R8."""
    G = gaussian_matrix(d, seed)
    Q, R = np.linalg.qr(G)
    s = np.where(np.diag(R) >= 0.0, 1.0, -1.0)
    return Q * s[None, :]


def qjl_matrix(m: int, d: int, seed: int) -> np.ndarray:
    """S: m x d, N(0,1) entries from stream 1, rounded to fp16 (R5)."""
    g = stream_normals(seed, 1, m * d).reshape(m, d)
    return g.astype(np.float16).astype(np.float64)


# ----------------------------------------------------------------------------
# [WHAT] stage 1 step 1 (Beta law) and step 2 (Lloyd-Max for that law), R2.
# ----------------------------------------------------------------------------
def beta_log_norm(d: int) -> float:
    """log of Gamma(d/2) / (sqrt(pi) Gamma((d-1)/2)), the density constant."""
    return gammaln(d / 2.0) - 0.5 * math.log(math.pi) - gammaln((d - 1) / 2.0)


def beta_density(t: np.ndarray, d: int) -> np.ndarray:
    """f_d(t) = K (1 - t^2)^((d-3)/2) on [-1, 1]: the law of one coordinate of a
    uniformly random unit vector in R^d (R2)."""
    t = np.asarray(t, dtype=np.float64)
    out = np.zeros_like(t)
    inside = np.abs(t) < 1.0
    out[inside] = np.exp(beta_log_norm(d) + 0.5 * (d - 3) * np.log1p(-t[inside] ** 2))
    return out


def _upper_tail(t: np.ndarray, d: int) -> np.ndarray:
    """P(T >= t) for T ~ f_d, via the regularised incomplete beta function."""
    a = 0.5 * (d - 1)
    return betaincc(a, a, 0.5 * (1.0 + np.asarray(t, dtype=np.float64)))


def _first_moment(lo: np.ndarray, hi: np.ndarray, d: int) -> np.ndarray:
    """int_lo^hi t f_d(t) dt in closed form: K [-(1-t^2)^((d-1)/2) / (d-1)]."""
    K = math.exp(beta_log_norm(d))
    p = 0.5 * (d - 1)
    return K * ((1.0 - lo ** 2) ** p - (1.0 - hi ** 2) ** p) / (d - 1)


@dataclass(frozen=True)
class Codebook:
    bits: int
    centroids: np.ndarray   # L values, increasing
    boundaries: np.ndarray  # L-1 interior decision boundaries, increasing
    iterations: int


def _lloyd_update(c: np.ndarray, d: int):
    """One Lloyd-Max step on the upper-half centroids c (boundary 0 in the
    middle): boundaries at the midpoints, then each centroid the mean of its
    cell.  Also returns the cells' edges and masses."""
    edges = np.concatenate([[0.0], 0.5 * (c[:-1] + c[1:]), [1.0]])
    lo, hi = edges[:-1], edges[1:]
    mass = _upper_tail(lo, d) - _upper_tail(hi, d)
    return _first_moment(lo, hi, d) / mass, lo, hi, mass


def lloyd_max(d: int, bits: int, tol: float = 1e-15, max_iter: int = 100000) -> Codebook:
    """Lloyd-Max quantizer for f_d with L = 2^bits levels ([WHAT] stage 1
    step 2; "per hidden dimension and bit width" in "How to implement").

    Alternates the two optimality conditions: each boundary is the midpoint of
    its neighbouring centroids, each centroid is the conditional mean of its
    cell.  f_d is symmetric, so the iteration runs on the upper half
    (boundary 0 in the middle) and the lower half is mirrored.  For bits = 1
    this is one step: c = E[T | T > 0].

    The plain alternation converges slowly when there are many levels (an
    8-bit codebook), so once its steps fall below 1e-7 (or after 4000 of
    them) the same fixed point c = U(c) of the update U is finished by Newton
    steps on c - U(c).  U_i depends on c_{i-1}, c_i, c_{i+1} through the two
    midpoints, and d U_i / d hi = f(hi) (hi - U_i) / P_i, d U_i / d lo =
    f(lo) (U_i - lo) / P_i (P_i the cell's mass), so each step is one
    tridiagonal solve.  Newton stops at tol or, after eight steps, once its
    steps are below 1e-12 (the rounding floor of the cell masses for 8 bits).
    """
    L = 1 << bits
    half = L // 2
    c = (np.arange(half) + 0.5) / half * 3.0 / math.sqrt(d)
    it = 0
    delta = math.inf
    for it in range(1, max_iter + 1):
        c_new = _lloyd_update(c, d)[0]
        delta = float(np.max(np.abs(c_new - c)))
        c = c_new
        if delta < tol or (delta < 1e-7 and half > 1) or it >= 4000:
            break
    newton = 0
    while delta >= tol and half > 1 and it < max_iter:
        it += 1
        newton += 1
        u, lo, hi, mass = _lloyd_update(c, d)
        r = u - c
        du_hi = beta_density(hi, d) * (hi - u) / mass
        du_lo = beta_density(lo, d) * (u - lo) / mass
        du_hi[-1] = 0.0                    # the last edge is 1, fixed
        du_lo[0] = 0.0                     # the first edge is 0, fixed
        # (I - J) step = r with J_{i,i-1} = du_lo/2, J_{i,i} = (du_lo + du_hi)/2, J_{i,i+1} = du_hi/2
        ab = np.zeros((3, half))
        ab[0, 1:] = -0.5 * du_hi[:-1]
        ab[1, :] = 1.0 - 0.5 * (du_lo + du_hi)
        ab[2, :-1] = -0.5 * du_lo[1:]
        step = solve_banded((1, 1), ab, r)
        scale = 1.0
        while True:                        # keep the centroids increasing inside (0, 1)
            cand = c + scale * step
            if np.all(np.diff(cand) > 0) and cand[0] > 0 and cand[-1] < 1:
                break
            scale *= 0.5
        c = cand
        delta = float(np.max(np.abs(scale * step)))
        if newton >= 8 and delta < 1e-12:
            break                          # at the floor set by rounding in the cell masses
    centroids = np.concatenate([-c[::-1], c])
    inner = 0.5 * (c[:-1] + c[1:])
    boundaries = np.concatenate([-inner[::-1], [0.0], inner])
    return Codebook(bits, centroids, boundaries, it)


def distortion(d: int, cb: Codebook) -> float:
    """d * E[(T - c(T))^2] for T ~ f_d, integrated cell by cell."""
    edges = np.concatenate([[-1.0], cb.boundaries, [1.0]])
    lo, hi = edges[:-1], edges[1:]
    mass = _upper_tail(lo, d) - _upper_tail(hi, d)
    m1 = _first_moment(lo, hi, d)
    # E[T^2] over the whole line is 1/d; per cell, sum(c^2 mass - 2 c m1) + 1/d.
    return d * (1.0 / d + float(np.sum(cb.centroids ** 2 * mass - 2.0 * cb.centroids * m1)))


# ----------------------------------------------------------------------------
# Per-context tables.
# ----------------------------------------------------------------------------
@dataclass
class Tables:
    d: int
    bits_k_lm: int
    bits_v: int
    qjl_m: int
    seed: int
    Pi: np.ndarray
    S: np.ndarray | None
    cb_k: Codebook
    cb_v: Codebook
    nc_k: bool = False     # R13 norm correction of keys
    nc_v: bool = False     # R13 norm correction of values
    norm_f16: bool = False # norms stored as binary16 (MSE-only keys)


def make_tables(d: int, bits_k: int, bits_v: int, qjl_m: int, seed: int,
                nc_k: bool = False, nc_v: bool = False, norm_f16: bool = False) -> Tables:
    """bits_k counts the QJL bit when qjl_m > 0 (R3).  nc_k / nc_v turn on
    the R13 norm correction (keys only without QJL); norm_f16 stores the
    per-vector norms as binary16 (MSE-only keys)."""
    if nc_k and qjl_m > 0:
        raise ValueError("key norm correction applies to MSE-only keys (qjl_m = 0)")
    if norm_f16 and qjl_m > 0:
        raise ValueError("binary16 norms apply to MSE-only keys (qjl_m = 0)")
    bits_k_lm = bits_k - 1 if qjl_m > 0 else bits_k
    Pi = rotation(d, seed)
    S = qjl_matrix(qjl_m, d, seed) if qjl_m > 0 else None
    return Tables(d, bits_k_lm, bits_v, qjl_m, seed, Pi, S,
                  lloyd_max(d, bits_k_lm), lloyd_max(d, bits_v), nc_k, nc_v, norm_f16)


# ----------------------------------------------------------------------------
# Bit packing (the library's own layout; the pages only say the fused kernel
# reads the indices directly).  A vector's Lloyd-Max indices are packed as
# b-bit fields, LSB first, 32/b fields per uint32 word, for b in {1, 2, 4, 8}:
# coordinate j sits in word j // (32/b) at bit b * (j % (32/b)).  For b = 3
# the low two bits of every index form a 2-bit field stream and the top bit a
# 1-bit stream that follows it.  Padding bits are zero.  QJL bits form a 1-bit
# stream (bit i set when sigma_i = +1).
# ----------------------------------------------------------------------------
def field_words(n: int, b: int) -> int:
    per = 32 // b
    return (n + per - 1) // per


def code_words(d: int, bits: int) -> int:
    if bits == 3:
        return field_words(d, 2) + field_words(d, 1)
    return field_words(d, bits)


def pack_fields(vals: np.ndarray, b: int) -> np.ndarray:
    """vals: [..., n] integers in [0, 2^b) -> uint32 [..., ceil(n*b/32)]."""
    vals = np.asarray(vals, dtype=np.uint64)
    n = vals.shape[-1]
    per = 32 // b
    W = field_words(n, b)
    pad = np.zeros(vals.shape[:-1] + (W * per - n,), dtype=np.uint64)
    v = np.concatenate([vals, pad], axis=-1).reshape(vals.shape[:-1] + (W, per))
    shifts = (np.uint64(b) * np.arange(per, dtype=np.uint64))
    return (v << shifts).sum(axis=-1).astype(np.uint32)


def unpack_fields(words: np.ndarray, n: int, b: int) -> np.ndarray:
    words = np.asarray(words, dtype=np.uint32).astype(np.uint64)
    per = 32 // b
    shifts = np.uint64(b) * np.arange(per, dtype=np.uint64)
    v = (words[..., :, None] >> shifts) & np.uint64((1 << b) - 1)
    return v.reshape(words.shape[:-1] + (-1,))[..., :n].astype(np.int64)


def pack_bits(bits: np.ndarray) -> np.ndarray:
    """bits: [..., n] of 0/1 -> uint32 [..., ceil(n/32)], LSB first."""
    return pack_fields(bits, 1)


def unpack_bits(words: np.ndarray, n: int) -> np.ndarray:
    return unpack_fields(words, n, 1)


def pack_codes(idx: np.ndarray, bits: int) -> np.ndarray:
    idx = np.asarray(idx, dtype=np.int64)
    if bits == 3:
        return np.concatenate([pack_fields(idx & 3, 2), pack_fields(idx >> 2, 1)], axis=-1)
    return pack_fields(idx, bits)


def unpack_codes(codes: np.ndarray, bits: int, d: int) -> np.ndarray:
    codes = np.asarray(codes, dtype=np.uint32)
    if bits == 3:
        w2 = field_words(d, 2)
        return unpack_fields(codes[..., :w2], d, 2) | (unpack_fields(codes[..., w2:], d, 1) << 2)
    return unpack_fields(codes, d, bits)


# ----------------------------------------------------------------------------
# [WHAT] stage 1 (normalise, rotate, Lloyd-Max index) and stage 2 (QJL sign
# sketch of the residual), one vector per row.
# ----------------------------------------------------------------------------
def lloyd_max_index(y: np.ndarray, cb: Codebook) -> np.ndarray:
    """idx = number of boundaries at or below y (R7: ties go up)."""
    return (y[..., None] >= cb.boundaries).sum(axis=-1).astype(np.int64)


@dataclass
class Quantized:
    idx: np.ndarray        # [N, d] int64 Lloyd-Max indices
    codes: np.ndarray      # [N, code_words(d, b)] uint32
    norm: np.ndarray       # [N] fp32 (R4)
    y: np.ndarray          # [N, d] rotated unit vectors (fp64), for band checks
    qjl_bits: np.ndarray | None = None   # [N, m] 0/1
    qjl: np.ndarray | None = None        # [N, ceil(m/32)] uint32
    rnorm: np.ndarray | None = None      # [N] fp32 gamma = n * |r|
    proj: np.ndarray | None = None       # [N, m] S r (fp64), for band checks
    rho: np.ndarray | None = None        # [N] |r| (fp64)


def quantize(x: np.ndarray, tab: Tables, which: str) -> Quantized:
    """Quantize rows of x (any float dtype; converted exactly to fp64).

    which = "k": Lloyd-Max with bits_k_lm bits, plus the QJL sketch when
    qjl_m > 0.  which = "v": Lloyd-Max with bits_v bits only (R12).
    """
    x = np.asarray(x, dtype=np.float64)
    cb = tab.cb_k if which == "k" else tab.cb_v
    n = np.sqrt(np.sum(x * x, axis=-1))
    safe = np.where(n > 0.0, n, 1.0)
    u = np.where((n > 0.0)[:, None], x / safe[:, None], 0.0)
    y = u @ tab.Pi.T
    idx = lloyd_max_index(y, cb)
    nc = tab.nc_k if which == "k" else tab.nc_v
    stored = corrected_norm(n, idx, cb) if nc else n
    # The stored scalar: fp32 (R4), or binary16 rounded to nearest even.
    q = Quantized(idx=idx, codes=pack_codes(idx, cb.bits),
                  norm=stored.astype(np.float16 if tab.norm_f16 else np.float32), y=y)
    if which == "k" and tab.qjl_m > 0:
        sketch_from_indices(q, tab)
    return q


def corrected_norm(n: np.ndarray, idx: np.ndarray, cb: Codebook) -> np.ndarray:
    """R13: n / |c[idx]| (fp64), the norm stored under norm correction.  The
    codebook has no zero centroid, so |c[idx]| > 0."""
    chat = cb.centroids[idx]
    return np.asarray(n, dtype=np.float64) / np.sqrt(np.sum(chat * chat, axis=-1))


def sketch_from_indices(q: Quantized, tab: Tables, idx: np.ndarray | None = None) -> None:
    """[WHAT] stage 2: residual r = y - c[idx], rho = |r|, sigma = sign(S r)
    with sign(0) = +1 (R6, stored as bit 1), gamma = n rho.  `idx` overrides the indices (used to rebuild the sketch
    for codes produced elsewhere)."""
    idx = q.idx if idx is None else idx
    r = q.y - tab.cb_k.centroids[idx]
    rho = np.sqrt(np.sum(r * r, axis=-1))
    q.proj = r @ tab.S.T
    q.qjl_bits = (q.proj >= 0.0).astype(np.int64)
    q.qjl = pack_bits(q.qjl_bits)
    q.rho = rho
    q.rnorm = (q.norm.astype(np.float64) * rho).astype(np.float32)


def boundary_distance(y: np.ndarray, cb: Codebook) -> np.ndarray:
    """|y - nearest decision boundary| on the rotated unit-vector scale."""
    return np.min(np.abs(y[..., None] - cb.boundaries), axis=-1)


# ----------------------------------------------------------------------------
# Agreement counts: another implementation's codes against this oracle.
# "Within 1e-5 of a decision boundary" is read on the rotated unit-vector
# scale (the scale on which the Beta law and the boundaries live): an index
# may differ from the oracle's only when |y_j - beta_i| < band.  The counts
# also give the in-band fraction on the standardized scale sqrt(d) * y, where
# the same band is sqrt(d) times narrower.
# ----------------------------------------------------------------------------
def code_agreement(tab: Tables, which: str, x: np.ndarray, codes: np.ndarray,
                   qjl: np.ndarray | None = None, band: float = 1e-5) -> dict:
    """Counts for codes (and QJL words) produced elsewhere from the rows of x.

    Returns indices, mismatches, mismatches outside the unit-scale band (a
    real disagreement), in-band counts on the unit and standardized scales,
    mismatches outside the standardized band, and for keys with QJL the same
    for the sign bits (band |(S r)_i| < band * |r|, with the sketch rebuilt
    from the other side's indices).
    """
    x = np.asarray(x, dtype=np.float64)
    cb = tab.cb_k if which == "k" else tab.cb_v
    n = x.shape[0]
    q = quantize(x, tab, which)
    gidx = unpack_codes(np.asarray(codes).reshape(n, -1), cb.bits, tab.d)
    dist = boundary_distance(q.y, cb)
    mism = gidx != q.idx
    in_unit = dist < band
    in_std = dist < band / math.sqrt(tab.d)
    out = {"indices": int(mism.size), "mismatches": int(mism.sum()),
           "outside_band": int(np.sum(mism & ~in_unit)),
           "in_band_unit": int(in_unit.sum()), "in_band_std": int(in_std.sum()),
           "mismatches_outside_std_band": int(np.sum(mism & ~in_std))}
    if which == "k" and tab.qjl_m > 0 and qjl is not None:
        sketch_from_indices(q, tab, idx=gidx)
        gbits = unpack_bits(np.asarray(qjl).reshape(n, -1), tab.qjl_m)
        qm = gbits != q.qjl_bits
        qband = np.abs(q.proj) < band * q.rho[:, None]
        out.update(qjl_bits=int(qm.size), qjl_mismatches=int(qm.sum()),
                   qjl_outside_band=int(np.sum(qm & ~qband)), qjl_in_band=int(qband.sum()))
    return out


# ----------------------------------------------------------------------------
# Dequantization and logits (closing paragraph of "How TurboQuant works";
# "How to implement" part 1: pre-rotate the query once).
# ----------------------------------------------------------------------------
def qjl_constant(m: int) -> float:
    """sqrt(pi/2)/m: E[sign(<s,r>) <s,q>] = sqrt(2/pi) <q,r>/|r| for s ~ N(0,I)."""
    return math.sqrt(math.pi / 2.0) / m


def dequantize(tab: Tables, which: str, codes, norm, qjl=None, rnorm=None) -> np.ndarray:
    """x_hat = n Pi^T c[idx]  (+ C gamma Pi^T S^T sigma for keys with QJL, R12)."""
    cb = tab.cb_k if which == "k" else tab.cb_v
    idx = unpack_codes(codes, cb.bits, tab.d)
    rot = cb.centroids[idx] * np.asarray(norm, dtype=np.float64)[:, None]
    if which == "k" and tab.qjl_m > 0:
        sigma = 2.0 * unpack_bits(qjl, tab.qjl_m) - 1.0
        rot = rot + qjl_constant(tab.qjl_m) * np.asarray(rnorm, dtype=np.float64)[:, None] * (sigma @ tab.S)
    return rot @ tab.Pi


def logits(tab: Tables, q: np.ndarray, codes, norm, qjl=None, rnorm=None) -> np.ndarray:
    """l = n <Pi q, c[idx]> + C gamma <S Pi q, sigma>, unscaled (R11).
    q: [nq, d]; codes etc. for nk keys; returns [nq, nk]."""
    q = np.asarray(q, dtype=np.float64)
    qr = q @ tab.Pi.T                       # pre-rotated query
    idx = unpack_codes(codes, tab.cb_k.bits, tab.d)
    chat = tab.cb_k.centroids[idx]          # [nk, d]
    out = (qr @ chat.T) * np.asarray(norm, dtype=np.float64)[None, :]
    if tab.qjl_m > 0:
        s = qr @ tab.S.T                    # S Pi q
        sigma = 2.0 * unpack_bits(qjl, tab.qjl_m) - 1.0
        out = out + qjl_constant(tab.qjl_m) * (s @ sigma.T) * np.asarray(rnorm, dtype=np.float64)[None, :]
    return out


# ----------------------------------------------------------------------------
# Decode attention over the packed cache ([WHAT] closing paragraph of "How
# TurboQuant works"; [VLLM] A2: values are dequantized for softmax . V).
# Cache arrays are [B, Hkv, T, ...]; query head h reads kv head h*Hkv//Hq.
# ----------------------------------------------------------------------------
def attention(tab: Tables, q, kcodes, kqjl, knorm, krnorm, vcodes, vnorm,
              seq_lens, Hkv: int, scale: float | None = None,
              batches=None, heads=None) -> np.ndarray:
    """Returns out [B, Hq, d] (or the selected (b, h) rows) in fp64.

    For each (b, h): s_i = scale * l_i for i < seq_len_b, p = softmax(s)
    (max-subtracted), o = sum_i p_i * vhat_i with each vhat_i dequantized on
    its own.  seq_len 0 gives o = 0.
    """
    q = np.asarray(q, dtype=np.float64)
    B, Hq, d = q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    batches = range(B) if batches is None else batches
    heads = range(Hq) if heads is None else heads
    out = np.zeros((B, Hq, d))
    for b in batches:
        T = int(seq_lens[b])
        if T == 0:
            continue
        for h in heads:
            kv = h * Hkv // Hq
            l = logits(tab, q[b, h][None, :], kcodes[b, kv, :T],
                       knorm[b, kv, :T],
                       None if kqjl is None else kqjl[b, kv, :T],
                       None if krnorm is None else krnorm[b, kv, :T])[0]
            s = scale * l
            p = np.exp(s - np.max(s))
            p /= np.sum(p)
            vhat = dequantize(tab, "v", vcodes[b, kv, :T], vnorm[b, kv, :T])
            out[b, h] = p @ vhat
    return out


# ----------------------------------------------------------------------------
# Inner-product top-k over compressed database vectors ([WHAT] section
# "基准测试与实际性能表现" ("Benchmarks"): top-k recall on d=200 vectors).
# ----------------------------------------------------------------------------
def topk(tab: Tables, q, codes, norm, qjl, rnorm, k: int):
    """Exact top-k of the compressed scores, ordered by (score desc, index asc)."""
    scores = logits(tab, q, codes, norm, qjl, rnorm)
    n = scores.shape[1]
    idx = np.empty((scores.shape[0], k), dtype=np.int64)
    val = np.empty((scores.shape[0], k))
    order_key = np.arange(n)
    for i in range(scores.shape[0]):
        order = np.lexsort((order_key, -scores[i]))[:k]
        idx[i] = order
        val[i] = scores[i, order]
    return idx, val, scores
