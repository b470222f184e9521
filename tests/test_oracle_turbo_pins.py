"""Pins for the TurboQuant-prod oracle (oracle/turbo.py).

Each test checks the oracle against something other than itself: closed
forms (the d = 3 density is uniform, so its Lloyd-Max quantizer is the
uniform one; the 1-bit centroid is E|X|), the Gaussian Lloyd-Max table that
the codebook must approach as d grows (Max, "Quantizing for minimum
distortion", 1960), independent quadrature, the defining properties of the
QR factor, the sampled distribution of a rotated coordinate, brute force on
tiny inputs, and the statistics the pages state for the estimator
(unbiasedness, the QJL variance on the residual, the D_prod bound).
"""
import math

import numpy as np
import pytest
import scipy.special
import scipy.stats

import oracle
from oracle import turbo as tq


def _gl(lo, hi, fn, nodes=400):
    xs, ws = np.polynomial.legendre.leggauss(nodes)
    x = (hi - lo) / 2 * xs + (hi + lo) / 2
    return (hi - lo) / 2 * float(np.sum(ws * fn(x)))


# --------------------------------------------------------------------------
# density

@pytest.mark.parametrize("d", [3, 5, 64, 128])
def test_density_is_normalised_with_variance_one_over_d(d):
    f = lambda x: tq.coord_density(x, d)
    assert _gl(-1, 1, f) == pytest.approx(1.0, abs=1e-12)
    assert _gl(-1, 1, lambda x: x * x * f(x)) == pytest.approx(1.0 / d, rel=1e-10)
    assert _gl(-1, 1, lambda x: x * f(x)) == pytest.approx(0.0, abs=1e-14)


@pytest.mark.parametrize("d", [5, 128])
def test_cdf_and_partial_mean_match_quadrature(d):
    for lo, hi in [(-1.0, -0.3), (-0.2, 0.05), (0.01, 0.2), (0.3, 1.0)]:
        p = float(tq.coord_cdf(hi, d) - tq.coord_cdf(lo, d))
        assert p == pytest.approx(_gl(lo, hi, lambda x: tq.coord_density(x, d)), abs=1e-13)
        pm = float(tq.partial_mean(lo, hi, d))
        assert pm == pytest.approx(_gl(lo, hi, lambda x: x * tq.coord_density(x, d)), abs=1e-13)


# --------------------------------------------------------------------------
# codebook

@pytest.mark.parametrize("bits", [1, 2, 3])
def test_d3_codebook_is_the_uniform_quantizer(bits):
    # d = 3: f = 1/2 on [-1, 1]; the optimal L-level quantizer of a uniform
    # variable has equal cells, centroids at their midpoints, MSE (2/L)^2/12
    L = 1 << bits
    c = tq.lloyd_max(3, bits)
    assert np.allclose(c, -1 + (2 * np.arange(L) + 1) / L, atol=1e-12)
    assert tq.codebook_mse(c, 3) == pytest.approx((2.0 / L) ** 2 / 12, rel=1e-9)


@pytest.mark.parametrize("d", [4, 64, 128, 256])
def test_one_bit_centroid_is_mean_absolute_coordinate(d):
    # E|X| = 2 int_0^1 x f(x) dx = Gamma(d/2) / (sqrt(pi) Gamma((d+1)/2))
    want = math.exp(scipy.special.gammaln(d / 2) - 0.5 * math.log(math.pi)
                    - scipy.special.gammaln((d + 1) / 2))
    c = tq.lloyd_max(d, 1)
    assert c == pytest.approx([-want, want], rel=1e-12)


# Max (1960), Table I: optimum quantizer of a unit Gaussian, output levels
# (positive half) and mean squared error
MAX_TABLE = {1: ([0.7979], 0.3634), 2: ([0.4528, 1.510], 0.1175),
             3: ([0.2451, 0.7560, 1.344, 2.152], 0.03454)}


@pytest.mark.parametrize("bits", [1, 2, 3])
def test_codebook_approaches_gaussian_lloyd_max_table(bits):
    # as d grows sqrt(d) X tends to N(0, 1), so sqrt(d) c -> Max's levels
    d = 100000
    c = tq.lloyd_max(d, bits)
    L = 1 << bits
    levels, mse = MAX_TABLE[bits]
    assert np.allclose(c[L // 2:] * math.sqrt(d), levels, atol=1.5e-3)
    assert tq.codebook_mse(c, d) * d == pytest.approx(mse, rel=2e-3)


@pytest.mark.parametrize("d,bits", [(5, 2), (64, 3), (128, 2), (128, 3)])
def test_codebook_is_stationary_and_locally_optimal(d, bits):
    c = tq.lloyd_max(d, bits)
    t = np.concatenate([[-1.0], tq.boundaries(c), [1.0]])
    f = lambda x: tq.coord_density(x, d)
    for i in range(len(c)):
        mass = _gl(t[i], t[i + 1], f)
        mean = _gl(t[i], t[i + 1], lambda x: x * f(x)) / mass
        assert c[i] == pytest.approx(mean, abs=1e-12)
    # symmetric (the density is even)
    assert np.allclose(c, -c[::-1], atol=1e-14)
    base = tq.codebook_mse(c, d)
    for i in range(len(c)):
        for eps in (-1e-3, 1e-3):
            cc = c.copy()
            cc[i] += eps / math.sqrt(d)
            assert tq.codebook_mse(cc, d) > base


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_codebook_mse_between_shannon_and_stated_bound(bits):
    # per unit vector: D_mse = d * (per-coordinate error), between 1/4^b and
    # sqrt(3) pi / 2 / 4^b
    for d in (64, 128):
        c = tq.lloyd_max(d, bits)
        D = d * tq.codebook_mse(c, d)
        assert 4.0 ** -bits < D <= math.sqrt(3) * math.pi / 2 * 4.0 ** -bits


# --------------------------------------------------------------------------
# rotation

def test_rotation_is_the_positive_diagonal_qr_factor():
    d = 48
    G = tq.gaussian_matrix(d, 5)
    P = tq.rotation(d, 5)
    assert np.abs(P.T @ P - np.eye(d)).max() < 1e-12
    R = P.T @ G
    assert np.abs(np.tril(R, -1)).max() < 1e-10
    assert np.all(np.diag(R) > 0)
    # G is the sketch generator's output with m = d
    Sb = oracle.sketch_bf16_bits(d, d, 5)
    assert np.array_equal(Sb, np.array([[oracle.f64_to_bf16_bits(v) for v in row] for row in G],
                                       dtype=np.uint16))


def test_rotated_coordinate_follows_the_density():
    d = 12
    x = np.arange(1.0, d + 1)
    x /= np.linalg.norm(x)
    y = np.array([tq.rotation(d, 1000 + s) @ x for s in range(600)])
    # every coordinate is distributed as f; coordinates of different seeds
    # are independent
    for i in (0, 5, 11):
        ks = scipy.stats.kstest(y[:, i], lambda v: tq.coord_cdf(v, d))
        assert ks.pvalue > 1e-3
    assert np.mean(y * y) == pytest.approx(1.0 / d, rel=0.05)


def test_stored_rotation_and_query_map():
    d = 32
    Pit = tq.rotation_stored(d, 9)
    P = tq.rotation(d, 9)
    assert np.abs(Pit - P).max() <= np.abs(P).max() * 2.0 ** -8
    W = tq.query_map(Pit)
    assert np.abs(W.T @ Pit - np.eye(d)).max() < 1e-12


# --------------------------------------------------------------------------
# quantizer

def test_cells_are_nearest_centroids_brute_force():
    rng = np.random.default_rng(3)
    d, bits = 8, 2
    c = tq.lloyd_max(d, bits)
    Pit = tq.rotation_stored(d, 4)
    S = oracle.sketch(32, d, 6)
    K = rng.standard_normal((20, d))
    # one key whose first rotated coordinate sits on a boundary exactly is
    # hard to build; instead check the tie rule on the cell function itself
    q = tq.quantize(K, Pit, c, S)
    for n in range(K.shape[0]):
        x = K[n] / np.linalg.norm(K[n])
        y = [sum(Pit[i][j] * x[j] for j in range(d)) for i in range(d)]
        for i in range(d):
            dist = [abs(y[i] - cj) for cj in c]
            best = min(range(len(c)), key=lambda j: (dist[j], j))
            assert q["cell"][n, i] == best
            assert q["r"][n, i] == pytest.approx(y[i] - c[best], abs=1e-15)
    # exactly on a boundary -> the cell nearer zero; 0 -> the cell below it;
    # the quantizer is odd-symmetric
    t = tq.boundaries(c)
    Y = np.array([[t[0], t[1], t[2], c[0], c[3], -1.0, 1.0, 0.0]])
    assert t[1] == 0.0
    assert list(tq.cell_of(Y, c)[0]) == [1, 1, 2, 0, 3, 0, 3, 1]
    c3 = tq.lloyd_max(d, 3)
    t3 = tq.boundaries(c3)
    Y3 = np.concatenate([t3, -t3, c3, np.linspace(-0.9, 0.9, 37)])
    cells = tq.cell_of(Y3, c3)
    assert np.array_equal(c3[tq.cell_of(-Y3[Y3 != 0], c3)], -c3[cells[Y3 != 0]])
    assert list(tq.cell_of(t3, c3)) == [1, 2, 3, 3, 4, 5, 6]


def test_residual_code_is_qjl_of_the_rounded_residual():
    rng = np.random.default_rng(8)
    d, m = 16, 64
    c = tq.lloyd_max(d, 2)
    Pit = tq.rotation_stored(d, 2)
    S = oracle.sketch(m, d, 3)
    K = rng.standard_normal((6, d))
    q = tq.quantize(K, Pit, c, S)
    # the residual handed to QJL is exactly bfloat16
    codes = np.array([[oracle.f64_to_bf16_bits(v) for v in row] for row in q["rt"]], dtype=np.uint16)
    assert np.array_equal(oracle.bf16_bits_to_f64(codes), q["rt"])
    assert np.abs(q["rt"] - q["r"]).max() <= np.abs(q["r"]).max() * 2.0 ** -8
    signs, norms, _, _ = oracle.quantize(q["rt"], S)
    assert np.array_equal(signs, q["signs"])
    assert np.allclose(np.linalg.norm(q["r"], axis=1), q["rnorm"], rtol=1e-15)
    assert np.allclose(q["norm"], np.linalg.norm(K, axis=1), rtol=1e-15)


def test_zero_key_has_zero_score():
    d, m = 16, 32
    c = tq.lloyd_max(d, 2)
    Pit = tq.rotation_stored(d, 2)
    S = oracle.sketch(m, d, 3)
    q = tq.quantize(np.zeros((1, d)), Pit, c, S)
    assert q["norm"][0] == 0.0
    sc = tq.scores(np.ones((1, d)), Pit, S, c, q["cell"], q["signs"], q["norm"], q["rnorm"])
    assert sc[0, 0] == 0.0


@pytest.mark.parametrize("bits", [1, 2, 3])
def test_plane_packing_round_trip_and_layout(bits):
    rng = np.random.default_rng(bits)
    d = 64
    cell = rng.integers(0, 1 << bits, size=(5, d)).astype(np.uint8)
    w = tq.pack_planes(cell, bits)
    assert w.shape == (5, bits * d // 32)
    assert np.array_equal(tq.unpack_planes(w, d, bits), cell)
    # coordinate 33's bit p sits at bit 1 of word p*d/32 + 1
    for p in range(bits):
        assert ((w[:, p * d // 32 + 1] >> 1) & 1).tolist() == ((cell[:, 33] >> p) & 1).tolist()


def test_bits_per_coordinate():
    # two stage-one bits, one QJL bit per coordinate (m = d) and two norms
    assert tq.prod_bits_per_coordinate(2, 128, 128) == pytest.approx(3.25)
    assert tq.prod_bits_per_coordinate(1, 64, 64) == pytest.approx(2.5)


# --------------------------------------------------------------------------
# estimator

def _sketches(m, d, count, base):
    return [oracle.sketch(m, d, base + s) for s in range(count)]


def test_prod_estimator_unbiased_over_sketches():
    rng = np.random.default_rng(11)
    d = m = 32
    c = tq.lloyd_max(d, 2)
    Pit = tq.rotation_stored(d, 21)
    k = rng.standard_normal(d) * 0.7
    qv = rng.standard_normal(d)
    exact = float(qv @ k)
    est = []
    for S in _sketches(m, d, 3000, 5000):
        q = tq.quantize(k[None, :], Pit, c, S, round_residual=False)
        est.append(tq.scores(qv[None, :], Pit, S, c, q["cell"], q["signs"], q["norm"],
                             q["rnorm"])[0, 0])
    est = np.array(est)
    assert abs(est.mean() - exact) < 4 * est.std() / math.sqrt(est.size)


def test_prod_variance_is_qjl_variance_of_the_residual():
    # over sketches, Var = (||k|| ||r|| / ||rt||)^2 ((pi/2) ||w||^2 ||rt||^2 - <w, rt>^2) / m
    rng = np.random.default_rng(12)
    d, m = 24, 64
    c = tq.lloyd_max(d, 1)
    Pit = tq.rotation_stored(d, 22)
    k = rng.standard_normal(d)
    qv = rng.standard_normal(d)
    w = tq.query_map(Pit) @ qv
    est = []
    q0 = None
    for S in _sketches(m, d, 3000, 9000):
        q = tq.quantize(k[None, :], Pit, c, S)
        q0 = q
        est.append(tq.scores(qv[None, :], Pit, S, c, q["cell"], q["signs"], q["norm"],
                             q["rnorm"])[0, 0])
    est = np.array(est)
    rt = q0["rt"][0]
    nk = q0["norm"][0]
    # the code is QJL of rt scaled by ||r|| (the residual's own norm)
    sc = q0["rnorm"][0] / math.sqrt(rt @ rt)
    var = (nk * sc) ** 2 * ((math.pi / 2) * (w @ w) * (rt @ rt) - (w @ rt) ** 2) / m
    n = est.size
    lo = scipy.stats.chi2.ppf(1e-4, n - 1) / (n - 1)
    hi = scipy.stats.chi2.ppf(1 - 1e-4, n - 1) / (n - 1)
    assert lo * var < est.var(ddof=1) < hi * var
    # the mean is ||k|| <w, yhat + rt ||r|| / ||rt||>
    yhat = c[q0["cell"][0]]
    mean = nk * (w @ (yhat + sc * rt))
    assert abs(est.mean() - mean) < 4 * math.sqrt(var / n)


@pytest.mark.parametrize("mse_bits", [1, 2, 3])
def test_prod_error_within_stated_bound(mse_bits):
    # D_prod = E |<y, x> - estimate|^2 over rotations and sketches, unit x,
    # b = mse_bits + 1 bits per coordinate (m = d), below
    # sqrt(3) pi^2 ||y||^2 / (d 4^b); the measured value also follows the
    # QJL variance of the residual averaged over rotations
    d = m = 64
    b = mse_bits + 1
    c = tq.lloyd_max(d, mse_bits)
    rng = np.random.default_rng(30 + mse_bits)
    x = rng.standard_normal(d)
    x /= np.linalg.norm(x)
    yv = rng.standard_normal(d)
    err2, pred = [], []
    for r in range(60):
        P = tq.rotation(d, 700 + r)
        for S in _sketches(m, d, 40, 20000 + 40 * r):
            q = tq.quantize(x[None, :], P, c, S, round_residual=False)
            est = tq.scores(yv[None, :], P, S, c, q["cell"], q["signs"], q["norm"], q["rnorm"])[0, 0]
            err2.append((est - yv @ x) ** 2)
        rt = q["rt"][0]
        w = P @ yv
        pred.append(((math.pi / 2) * (w @ w) * (rt @ rt) - (w @ rt) ** 2) / m)
    D = float(np.mean(err2))
    bound = math.sqrt(3) * math.pi ** 2 * (yv @ yv) / (d * 4.0 ** b)
    assert D < bound
    assert D == pytest.approx(float(np.mean(pred)), rel=0.1)


def test_scores_equal_dequantized_inner_product():
    # <w, yhat> + sqrt(pi/2)/m ||rt|| <S w, z> computed the other way round:
    # reconstruct the rotated key yhat + sqrt(pi/2)/m ||rt|| S^T z, map it
    # back with Pit^{-1} and take the plain inner product with q
    rng = np.random.default_rng(13)
    d, m = 16, 32
    c = tq.lloyd_max(d, 2)
    Pit = tq.rotation_stored(d, 7)
    S = oracle.sketch(m, d, 8)
    K = rng.standard_normal((5, d))
    Qm = rng.standard_normal((3, d))
    q = tq.quantize(K, Pit, c, S)
    sc = tq.scores(Qm, Pit, S, c, q["cell"], q["signs"], q["norm16"].view(np.float16).astype(np.float64),
                   q["rnorm16"].view(np.float16).astype(np.float64))
    Pinv = np.linalg.inv(Pit)
    for n in range(K.shape[0]):
        z = np.array([1.0 if (q["signs"][n, i // 32] >> (i % 32)) & 1 else -1.0 for i in range(m)])
        nk = float(oracle.fp16_bits_to_f64(q["norm16"][n]))
        nr = float(oracle.fp16_bits_to_f64(q["rnorm16"][n]))
        yrec = c[q["cell"][n]] + math.sqrt(math.pi / 2) / m * nr * (S.T @ z)
        krec = nk * (Pinv @ yrec)
        for j in range(Qm.shape[0]):
            assert sc[j, n] == pytest.approx(Qm[j] @ krec, rel=1e-12, abs=1e-12)


# --------------------------------------------------------------------------
# the prod dequantizer

@pytest.mark.parametrize("d,m,bits", [(16, 32, 1), (24, 64, 2), (32, 32, 3)])
def test_dequantized_inner_product_is_the_estimator(d, m, bits):
    # <q, Q_prod^-1(code)> is the estimate of <q, k> that scores() computes
    # the other way round (query mapped, centroids and sketch products)
    rng = np.random.default_rng(40 + bits)
    c = tq.lloyd_max(d, bits)
    Pit = tq.rotation_stored(d, 17)
    S = oracle.sketch(m, d, 18)
    K = rng.standard_normal((7, d)) * 1.3
    Qm = rng.standard_normal((4, d))
    q = tq.quantize(K, Pit, c, S)
    nk = oracle.fp16_bits_to_f64(q["norm16"])
    nr = oracle.fp16_bits_to_f64(q["rnorm16"])
    khat = tq.dequantize(q["cell"], q["signs"], nk, nr, Pit, S, c)
    assert khat.shape == K.shape
    sc = tq.scores(Qm, Pit, S, c, q["cell"], q["signs"], nk, nr)
    assert np.allclose(Qm @ khat.T, sc, rtol=1e-11, atol=1e-12)


def test_dequantized_residual_part_is_the_qjl_dequantizer():
    # khat / ||k|| mapped into the rotated frame is c[cell] plus the QJL
    # dequantizer (the C oracle) of the residual code with the norm ||r||
    rng = np.random.default_rng(41)
    d, m = 32, 64
    c = tq.lloyd_max(d, 2)
    Pit = tq.rotation_stored(d, 19)
    S = oracle.sketch(m, d, 20)
    K = rng.standard_normal((6, d))
    q = tq.quantize(K, Pit, c, S)
    nk, nr = q["norm"], q["rnorm"]
    khat = tq.dequantize(q["cell"], q["signs"], nk, nr, Pit, S, c)
    qjl = oracle.dequantize(q["signs"], nr, S)
    want = nk[:, None] * np.linalg.solve(Pit, (c[q["cell"]] + qjl).T).T
    assert np.allclose(khat, want, rtol=1e-11, atol=1e-13)


def test_dequantized_key_is_unbiased_over_sketches():
    # E_S[khat] = k (exact residual, exact norms), coordinate by coordinate
    rng = np.random.default_rng(42)
    d = m = 32
    c = tq.lloyd_max(d, 2)
    Pit = tq.rotation_stored(d, 23)
    k = rng.standard_normal(d) * 0.8
    est = []
    for S in _sketches(m, d, 3000, 31000):
        q = tq.quantize(k[None, :], Pit, c, S, round_residual=False)
        est.append(tq.dequantize(q["cell"], q["signs"], q["norm"], q["rnorm"], Pit, S, c)[0])
    est = np.array(est)
    se = est.std(axis=0, ddof=1) / math.sqrt(est.shape[0])
    assert np.all(np.abs(est.mean(axis=0) - k) < 4.5 * se)
    # stage one alone is biased: the mean is not c[cell] mapped back
    q = tq.quantize(k[None, :], Pit, c, _sketches(m, d, 1, 31000)[0], round_residual=False)
    mse_only = q["norm"][0] * np.linalg.solve(Pit, c[q["cell"][0]])
    assert np.max(np.abs(mse_only - k) / se) > 10


def test_dequantized_error_is_the_qjl_distortion_of_the_residual():
    # exact rotation P: E_S ||k - khat||^2 = ||k||^2 ||r||^2 ((pi/2) d - 1) / m,
    # the QJL reconstruction error of the residual (r does not depend on S)
    rng = np.random.default_rng(43)
    d, m = 16, 64
    c = tq.lloyd_max(d, 1)
    P = tq.rotation(d, 24)
    k = rng.standard_normal(d) * 2.0
    err2 = []
    r2 = None
    for S in _sketches(m, d, 3000, 41000):
        q = tq.quantize(k[None, :], P, c, S, round_residual=False)
        khat = tq.dequantize(q["cell"], q["signs"], q["norm"], q["rnorm"], P, S, c)[0]
        err2.append(float(np.sum((k - khat) ** 2)))
        r2 = float(q["rnorm"][0] ** 2)
    err2 = np.array(err2)
    pred = float(k @ k) * r2 * ((math.pi / 2) * d - 1) / m
    assert abs(err2.mean() - pred) < 4.5 * err2.std(ddof=1) / math.sqrt(err2.size)


def test_dequantized_zero_key_and_norm_scaling():
    d, m = 16, 32
    c = tq.lloyd_max(d, 2)
    Pit = tq.rotation_stored(d, 25)
    S = oracle.sketch(m, d, 26)
    K = np.zeros((2, d))
    K[1] = np.linspace(-1, 1, d)
    q = tq.quantize(K, Pit, c, S)
    khat = tq.dequantize(q["cell"], q["signs"], q["norm"], q["rnorm"], Pit, S, c)
    assert np.all(khat[0] == 0)
    # the code of 5 k is the code of k; khat scales with the norm
    q5 = tq.quantize(5 * K[1:], Pit, c, S)
    assert np.array_equal(q5["cell"], q["cell"][1:]) and np.array_equal(q5["signs"], q["signs"][1:])
    k5 = tq.dequantize(q5["cell"], q5["signs"], q5["norm"], q5["rnorm"], Pit, S, c)
    assert np.allclose(k5[0], 5 * khat[1], rtol=1e-12)


def test_decode_invariants():
    rng = np.random.default_rng(14)
    d, m = 16, 32
    c = tq.lloyd_max(d, 2)
    Pit = tq.rotation_stored(d, 7)
    S = oracle.sketch(m, d, 8)
    B, Hq, Hkv, T = 1, 4, 2, 5
    K = rng.standard_normal((B, Hkv, T, d))
    V = rng.standard_normal((B, Hkv, T, d))
    Qm = rng.standard_normal((B, Hq, d))
    q = tq.quantize(K.reshape(-1, d), Pit, c, S)
    cell = q["cell"].reshape(B, Hkv, T, d)
    signs = q["signs"].reshape(B, Hkv, T, -1)
    nk = q["norm"].reshape(B, Hkv, T)
    nr = q["rnorm"].reshape(B, Hkv, T)
    out, sc = tq.decode(Qm, Pit, S, c, cell, signs, nk, nr, V, 0.25, want_scores=True)
    # scores of head h come from kv head h // 2
    for h in range(Hq):
        want = tq.scores(Qm[0, h][None, :], Pit, S, c, cell[0, h // 2], signs[0, h // 2],
                         nk[0, h // 2], nr[0, h // 2])[0]
        assert np.allclose(sc[0, h], want, rtol=1e-13)
        p = scipy.special.softmax(0.25 * want)
        assert np.allclose(out[0, h], p @ V[0, h // 2], rtol=1e-12, atol=1e-13)
    # a single key returns its value
    out1, _ = tq.decode(Qm, Pit, S, c, cell[:, :, :1], signs[:, :, :1], nk[:, :, :1],
                        nr[:, :, :1], V[:, :, :1], 0.25)
    for h in range(Hq):
        assert np.allclose(out1[0, h], V[0, h // 2, 0], rtol=1e-14)
