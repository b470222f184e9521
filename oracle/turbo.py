"""Float64 oracle for the TurboQuant-prod key quantizer and its decode.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module.  It shares no code with the CUDA library in ``bit_jl_key_b200``.

Source: "The Geometry of Forgetting: How Three Papers Cracked KV Cache
Quantization", sections
  * "Random rotation, and what high dimensions do to your intuitions": the
    rotation Pi comes from orthogonalising a Gaussian matrix; each coordinate
    of Pi x, x a unit vector, has the density
        f(x) = Gamma(d/2) / (sqrt(pi) Gamma((d-1)/2)) * (1 - x^2)^((d-3)/2)
    on [-1, 1];
  * "TurboQuant: bridging MSE and inner product, in two stages": stage one
    quantizes every rotated coordinate with the Lloyd-Max codebook of f
    (centroids minimising the expected squared error, cells bounded by the
    midpoints of neighbouring centroids), b - 1 bits; stage two spends one
    bit per coordinate on QJL applied to the stage-one residual; the sum of
    the two estimates is unbiased, with D_prod <= sqrt(3) pi^2 ||y||^2 /
    (d 4^b) for a unit key.

Readings where the pages leave a step open:
  * Both stages act on the unit vector x = k / ||k|| (x = 0 when k = 0); the
    key norm is stored beside the code as binary16, as in the QJL path.
  * Pi = Q of the QR factorisation G = Q R with R's diagonal positive (the
    unique such Q), G[i][j] the standard normal of element i*d + j of the
    sketch generator with the rotation's own seed.  Pi is stored in bfloat16
    (Pit below); the key side uses Pit: y = Pit x.
  * The cell of coordinate y_i is that of the nearest centroid; a value
    exactly on a boundary goes to the cell nearer zero (so the quantizer is
    odd-symmetric; 0 goes to the cell just below it); yhat_i = c[cell].  The
    (b-1)-bit cell index is stored as b-1 bit planes, plane p holding bit p
    of every coordinate's index, each plane d bits LSB-first.
  * Stage two works in the rotated frame on the residual r = y - yhat: its
    code is sign(S rt) with rt = r rounded to bfloat16 (the precision of the
    contraction's input; bit 1 for >= 0) and an m x d Gaussian sketch S, and
    its norm ||r|| (of the residual itself) is stored as binary16.  For
    an exactly orthogonal Pi this is the pages' construction in distribution:
    S r = (S Pi^T)(Pi r) and S Pi^T is again an i.i.d. Gaussian matrix.
  * The query is mapped with the inverse transpose of the stored rotation,
    w = Pit^{-T} q, so that <w, y> = <q, x> holds exactly whatever rounding
    did to Pit; the estimate of <q, k> is
        ||k|| * ( <w, yhat> + sqrt(pi/2)/m * ||r|| * <S w, sign(S rt)> ),
    whose expectation over S is ||k|| <w, yhat + rt ||r|| / ||rt||>, i.e.
    <q, k> up to the bfloat16 rounding of the residual and the binary16 norms.
"""
from __future__ import annotations

import math

import numpy as np
import scipy.special

from . import _c, bf16_bits_to_f64, f64_to_bf16_bits_array, fp16_round_bits, gauss

SQRT_HALF_PI = math.sqrt(math.pi / 2.0)


# --------------------------------------------------------------------------
# the coordinate density of a rotated unit vector

def _log_const(d: int) -> float:
    return (scipy.special.gammaln(d / 2) - 0.5 * math.log(math.pi)
            - scipy.special.gammaln((d - 1) / 2))


def coord_density(x, d: int):
    """f(x) on [-1, 1] (0 outside)."""
    x = np.asarray(x, dtype=np.float64)
    body = np.power(np.clip(1 - x * x, 0.0, None), (d - 3) / 2)
    return np.where(np.abs(x) <= 1, math.exp(_log_const(d)) * body, 0.0)


def coord_cdf(x, d: int):
    """P(X <= x).  X = 2B - 1 with B ~ Beta((d-1)/2, (d-1)/2), whose density
    is f after the change of variable, so this is the regularised incomplete
    Beta function at (x + 1)/2."""
    a = (d - 1) / 2
    u = (np.clip(np.asarray(x, dtype=np.float64), -1, 1) + 1) / 2
    return scipy.special.betainc(a, a, u)


def partial_mean(lo, hi, d: int):
    """int_lo^hi x f(x) dx, from the antiderivative of x (1 - x^2)^((d-3)/2),
    which is -(1 - x^2)^((d-1)/2) / (d - 1)."""
    F = lambda x: -np.power(np.clip(1 - np.asarray(x) ** 2, 0.0, None), (d - 1) / 2) / (d - 1)
    return math.exp(_log_const(d)) * (F(hi) - F(lo))


# --------------------------------------------------------------------------
# stage one: the Lloyd-Max codebook

def lloyd_max(d: int, bits: int, tol: float = 1e-15, max_iter: int = 100000):
    """Centroids c_0 < ... < c_{L-1} (L = 2^bits) of the Lloyd-Max quantizer
    of f: alternate (i) boundaries at the midpoints of neighbouring centroids
    and (ii) each centroid at the mean of f over its cell, until the
    centroids move by less than tol.  Starts from the conditional means of
    L equal-probability cells.  Returns float64 [L]."""
    L = 1 << bits
    a = (d - 1) / 2
    edges = 2 * scipy.special.betaincinv(a, a, np.linspace(0, 1, L + 1)) - 1
    edges[0], edges[-1] = -1.0, 1.0
    c = partial_mean(edges[:-1], edges[1:], d) / np.diff(coord_cdf(edges, d))
    for _ in range(max_iter):
        t = np.concatenate([[-1.0], (c[:-1] + c[1:]) / 2, [1.0]])
        c_new = partial_mean(t[:-1], t[1:], d) / np.diff(coord_cdf(t, d))
        done = np.max(np.abs(c_new - c)) <= tol
        c = c_new
        if done:
            break
    # the density is even: make the symmetry exact, so the middle boundary of
    # an even number of cells is exactly 0
    return (c - c[::-1]) / 2


def cell_of(Y, c):
    """Cell of every value: the cell of the nearest centroid; a value exactly
    on a boundary goes to the cell nearer zero (0 goes to the cell just below
    it), which keeps the quantizer odd-symmetric.  With L cells and the
    positive boundaries t_+:  y > 0 -> L/2 + #{t in t_+ : t < y},
    y <= 0 -> L/2 - 1 - #{t in t_+ : t < -y}."""
    t = boundaries(c)
    L = len(c)
    tpos = t[L // 2:]
    Y = np.asarray(Y, dtype=np.float64)
    outer = np.sum(np.abs(Y)[..., None] > tpos, axis=-1)
    return np.where(Y > 0, L // 2 + outer, L // 2 - 1 - outer).astype(np.uint8)


def boundaries(c):
    """Cell boundaries: midpoints of neighbouring centroids, float64 [L-1]."""
    c = np.asarray(c, dtype=np.float64)
    return (c[:-1] + c[1:]) / 2


def codebook_mse(c, d: int, nodes: int = 400) -> float:
    """Expected squared error per coordinate, sum_i int_cell_i (x - c_i)^2 f,
    by Gauss-Legendre quadrature on each cell."""
    c = np.asarray(c, dtype=np.float64)
    t = np.concatenate([[-1.0], boundaries(c), [1.0]])
    xs, ws = np.polynomial.legendre.leggauss(nodes)
    total = 0.0
    for i in range(len(c)):
        lo, hi = t[i], t[i + 1]
        x = (hi - lo) / 2 * xs + (hi + lo) / 2
        total += (hi - lo) / 2 * float(np.sum(ws * (x - c[i]) ** 2 * coord_density(x, d)))
    return total


# --------------------------------------------------------------------------
# the rotation

def gaussian_matrix(d: int, seed: int) -> np.ndarray:
    """G[i][j] = standard normal of element i*d + j of the sketch generator."""
    return np.array([[gauss(seed, i * d + j) for j in range(d)] for i in range(d)])


def rotation(d: int, seed: int) -> np.ndarray:
    """Pi = Q of G = Q R with diag(R) > 0, float64 (library QR, then the
    column signs that make R's diagonal positive)."""
    Q, R = np.linalg.qr(gaussian_matrix(d, seed))
    return Q * np.sign(np.diag(R))[None, :]


def rotation_bf16_bits(d: int, seed: int) -> np.ndarray:
    """Pit: Pi rounded to bfloat16 (nearest, ties to even), row-major codes."""
    return f64_to_bf16_bits_array(rotation(d, seed))


def rotation_stored(d: int, seed: int) -> np.ndarray:
    """Pit as float64 values."""
    return bf16_bits_to_f64(rotation_bf16_bits(d, seed))


def query_map(Pit) -> np.ndarray:
    """Pit^{-T} (float64, library inverse)."""
    return np.linalg.inv(np.asarray(Pit, dtype=np.float64)).T


# --------------------------------------------------------------------------
# quantizer

def _bf16_round(x) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 (ties to even)."""
    return bf16_bits_to_f64(f64_to_bf16_bits_array(x))


def _bf16_ulp(x) -> np.ndarray:
    a = np.abs(np.asarray(x, dtype=np.float64))
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, 2.0 ** (e - 7), 2.0 ** -133)


def quantize(K, Pit, c, S, round_residual: bool = True, band_abs: float = 0.0,
             band_rel: float = 0.0):
    """TurboQuant-prod code of each row of K.

    K [n, d]; Pit [d, d] and S [m, d] float64 values of the stored matrices;
    c the stage-one centroids (float64 [L]).  Returns a dict:
      cell    uint8  [n, d]  stage-one cell of every rotated coordinate
      y       f64    [n, d]  the rotated unit key
      r, rt   f64    [n, d]  residual y - c[cell], and as given to QJL
      signs   uint32 [n, m/32]  sign(S rt), LSB-first (bit 1 for >= 0)
      proj    f64    [n, m]  S rt
      norm, rnorm  f64 [n]   ||k||, ||r|| (exact)
      norm16, rnorm16 uint16 [n]  their binary16 codes
    With band_abs > 0 also:
      cell_band bool [n, d]  y within band_abs of a boundary
      r_amb     bool [n, d]  r within band_abs of a bfloat16 rounding midpoint
      sign_allow f64 [n, m]  |(S rt)_i| below which bit i may differ:
                 band_rel ||rt|| + sum over r_amb coordinates j of
                 |S_ij| * ulp(r_j)
    """
    K = _c(K, np.float64)
    Pit = np.asarray(Pit, dtype=np.float64)
    S = np.asarray(S, dtype=np.float64)
    c = np.asarray(c, dtype=np.float64)
    n, d = K.shape
    norm = np.sqrt(np.sum(K * K, axis=1))
    X = K / np.where(norm > 0, norm, 1.0)[:, None]
    Y = X @ Pit.T
    t = boundaries(c)
    cell = cell_of(Y, c)
    R = Y - c[cell]
    Rt = _bf16_round(R) if round_residual else R
    P = Rt @ S.T
    m = S.shape[0]
    bits = (P >= 0).astype(np.uint64)
    signs = np.zeros((n, m // 32), dtype=np.uint64)
    for i in range(m):
        signs[:, i // 32] |= bits[:, i] << np.uint64(i % 32)
    rnorm = np.sqrt(np.sum(R * R, axis=1))
    out = {"cell": cell, "y": Y, "r": R, "rt": Rt, "signs": signs.astype(np.uint32),
           "proj": P, "norm": norm, "rnorm": rnorm,
           "norm16": fp16_round_bits(norm), "rnorm16": fp16_round_bits(rnorm)}
    if band_abs > 0:
        out["cell_band"] = np.min(np.abs(Y[:, :, None] - t[None, None, :]), axis=2) < band_abs
        ulp = _bf16_ulp(R)
        # distance of r to the nearest midpoint between bfloat16 neighbours
        frac = np.abs(R - Rt)
        amb = np.abs(ulp / 2 - frac) < band_abs
        out["r_amb"] = amb
        out["sign_allow"] = band_rel * rnorm[:, None] + (amb * ulp) @ np.abs(S).T
    return out


def pack_planes(cell, bits: int) -> np.ndarray:
    """Cell indices [n, d] as bit planes: uint32 [n, bits * d/32], plane p
    (words p*d/32 ...) holding bit p of each index, coordinate i at bit i%32
    of word i/32 of the plane."""
    cell = np.asarray(cell, dtype=np.uint64)
    n, d = cell.shape
    out = np.zeros((n, bits * d // 32), dtype=np.uint64)
    for p in range(bits):
        for i in range(d):
            out[:, p * d // 32 + i // 32] |= ((cell[:, i] >> np.uint64(p)) & np.uint64(1)) << np.uint64(i % 32)
    return out.astype(np.uint32)


def unpack_planes(words, d: int, bits: int) -> np.ndarray:
    w = np.asarray(words, dtype=np.uint64)
    cell = np.zeros((w.shape[0], d), dtype=np.uint64)
    for p in range(bits):
        for i in range(d):
            cell[:, i] |= ((w[:, p * d // 32 + i // 32] >> np.uint64(i % 32)) & np.uint64(1)) << np.uint64(p)
    return cell.astype(np.uint8)


# --------------------------------------------------------------------------
# estimator and decode

def scores(Q, Pit, S, c, cell, signs, norms, rnorms):
    """Estimates of <q, k>, float64 [nq, n].  norms / rnorms are the float64
    values of the stored norms (or exact ones)."""
    Q = _c(Q, np.float64)
    W = Q @ query_map(Pit).T                  # rows w = Pit^{-T} q
    c = np.asarray(c, dtype=np.float64)
    mse = W @ c[np.asarray(cell)].T           # <w, yhat>
    U = W @ np.asarray(S, dtype=np.float64).T  # S w
    m = U.shape[1]
    sg = np.asarray(signs, dtype=np.uint64)
    z = np.empty((sg.shape[0], m))
    for i in range(m):
        z[:, i] = 2.0 * ((sg[:, i // 32] >> np.uint64(i % 32)) & np.uint64(1)).astype(np.float64) - 1.0
    qjl = (SQRT_HALF_PI / m) * (U @ z.T) * np.asarray(rnorms, dtype=np.float64)[None, :]
    return np.asarray(norms, dtype=np.float64)[None, :] * (mse + qjl)


def dequantize(cell, signs, norms, rnorms, Pit, S, c):
    """Q_prod^-1 of each code, float64 [n, d]: stage one's reconstruction plus
    the QJL dequantizer of the residual code ("TurboQuant: bridging MSE and
    inner product, in two stages": the QJL estimate is added back to xhat),
    taken in the rotated frame and mapped back with the inverse of the
    stored rotation, then scaled by the key norm:
        khat = ||k|| * Pit^{-1} ( c[cell] + sqrt(pi/2)/m * ||r|| * S^T z ),
    z_i = +1 where code bit i is set, else -1.  For every q,
    <q, khat> = ||k|| (<w, c[cell]> + sqrt(pi/2)/m ||r|| <S w, z>) with
    w = Pit^{-T} q, the estimate `scores` gives.

    cell uint8 [n, d]; signs uint32 [n, m/32]; norms, rnorms [n] (float64
    values of the stored norms or exact ones); Pit [d, d]; S [m, d]; c the
    centroids."""
    cell = np.asarray(cell)
    sg = np.asarray(signs, dtype=np.uint64)
    S = np.asarray(S, dtype=np.float64)
    c = np.asarray(c, dtype=np.float64)
    m, d = S.shape
    n = cell.shape[0]
    assert cell.shape == (n, d) and sg.shape == (n, m // 32)
    z = np.empty((n, m))
    for i in range(m):
        z[:, i] = 2.0 * ((sg[:, i // 32] >> np.uint64(i % 32)) & np.uint64(1)).astype(np.float64) - 1.0
    rn = np.asarray(rnorms, dtype=np.float64).reshape(n)
    nk = np.asarray(norms, dtype=np.float64).reshape(n)
    yrec = c[cell] + (SQRT_HALF_PI / m) * rn[:, None] * (z @ S)   # rows c[cell] + a S^T z
    Pinv = np.linalg.inv(np.asarray(Pit, dtype=np.float64))
    return nk[:, None] * (yrec @ Pinv.T)


def decode(Q, Pit, S, c, cell, signs, norms, rnorms, V, softmax_scale: float,
           want_scores=False):
    """Decode attention with TurboQuant-prod scores.

    Q [B, Hq, d]; cell [B, Hkv, T, d]; signs [B, Hkv, T, m/32]; norms, rnorms
    [B, Hkv, T]; V [B, Hkv, T, d].  Query head h reads kv head h // (Hq/Hkv);
    logits = softmax_scale * score, softmax with the maximum subtracted, and
    the probability-weighted sum of the values.  Returns (out [B, Hq, d],
    scores [B, Hq, T] or None)."""
    Q = _c(Q, np.float64)
    V = np.asarray(V, dtype=np.float64)
    B, Hq, d = Q.shape
    Hkv, T = cell.shape[1], cell.shape[2]
    G = Hq // Hkv
    out = np.empty((B, Hq, d))
    sc_all = np.empty((B, Hq, T)) if want_scores else None
    for b in range(B):
        for h in range(Hkv):
            sc = scores(Q[b, h * G:(h + 1) * G], Pit, S, c, cell[b, h], signs[b, h],
                        norms[b, h], rnorms[b, h])
            lg = sc * softmax_scale
            p = np.exp(lg - lg.max(axis=1, keepdims=True))
            p /= p.sum(axis=1, keepdims=True)
            out[b, h * G:(h + 1) * G] = p @ V[b, h]
            if want_scores:
                sc_all[b, h * G:(h + 1) * G] = sc
    return out, sc_all


def prod_bits_per_coordinate(mse_bits: int, m: int, d: int, norm_bits: int = 16) -> float:
    """Stored bits per key coordinate: mse_bits planes of d bits, m QJL bits
    and two norms."""
    return (mse_bits * d + m + 2 * norm_bits) / d
