"""Pins for the float64 oracle against what the pages and mathematics fix.

Each test checks the oracle against something other than itself: values the
pages print, closed forms, exact quadrature, hand-derived fixtures, library
routines (numpy float16, scipy softmax / KS test) and brute force on tiny
inputs.  A plausible slip in the oracle (dropped constant, flipped sign,
transposed sketch, wrong bit order, wrong head mapping) fails at least one.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import scipy.special
import scipy.stats

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# --------------------------------------------------------------------------
# generator

def test_splitmix64_published_outputs():
    g = _golden("splitmix64_seed0.json")
    got = [oracle.splitmix64(g["seed"], n) for n in range(3)]
    assert got == [int(h, 16) for h in g["outputs_hex"]]


def test_uniform_is_open_interval():
    L = oracle.lib()
    assert L.jlo_uniform(0) > 0.0
    assert L.jlo_uniform((1 << 64) - 1) < 1.0
    assert L.jlo_uniform(1 << 63) == pytest.approx(0.5, abs=1e-15)
    assert L.jlo_uniform(0) == 2.0 ** -53


def test_gauss_is_standard_normal():
    x = np.array([oracle.gauss(7, e) for e in range(40000)])
    assert abs(x.mean()) < 4.0 / math.sqrt(x.size)
    assert abs(x.var() - 1.0) < 4.0 * math.sqrt(2.0 / x.size)
    ks = scipy.stats.kstest(x, "norm")
    assert ks.pvalue > 1e-3
    # consecutive elements are uncorrelated
    assert abs(np.corrcoef(x[:-1], x[1:])[0, 1]) < 4.0 / math.sqrt(x.size)


def _bf16_value(code):
    return Fraction(float(oracle.bf16_bits_to_f64(np.uint16(code))))


def _bf16_brute(x: float) -> int:
    """Nearest bfloat16 by exhaustive comparison over all finite codes of the
    right sign near x (exact rational arithmetic, ties to the even code)."""
    fx = Fraction(x)
    sign = 0x8000 if x < 0 or (x == 0 and math.copysign(1, x) < 0) else 0
    best, best_err = None, None
    # candidates: the 65536 codes are monotone in magnitude for one sign, so a
    # window around the truncated code holds the nearest two
    trunc = int(np.float64(abs(x)).astype(np.float32).view(np.uint32)) >> 16
    for c in range(max(0, trunc - 2), min(0x7F80, trunc + 3)):
        err = abs(abs(fx) - _bf16_value(c))
        if best is None or err < best_err or (err == best_err and c % 2 == 0):
            best, best_err = c, err
    return best | sign


def test_bf16_rounding_brute_force():
    rng = np.random.default_rng(3)
    vals = list(rng.normal(size=300)) + list(rng.normal(size=100) * 1e-30)
    # exact ties and near-ties, including the float32 double-rounding trap
    vals += [1 + 2 ** -8, 1 + 3 * 2 ** -8, 1 + 2 ** -8 + 2 ** -40,
             1 + 2 ** -8 - 2 ** -40, -(1 + 2 ** -8), 3.0, -0.75, 2 ** -130,
             3 * 2 ** -134, 5 * 2 ** -134]
    for x in vals:
        assert oracle.f64_to_bf16_bits(x) == _bf16_brute(float(x)), x


def test_fp16_norm_rounding_is_direct_rne():
    # 1 + 2^-11 + 2^-40 rounds up to 1 + 2^-10 when rounded directly; a
    # float32 intermediate would land on the tie and round to even (1.0)
    assert int(oracle.fp16_round_bits([1 + 2 ** -11 + 2 ** -40])[0]) == 0x3C01
    assert int(oracle.fp16_round_bits([1 + 2 ** -11])[0]) == 0x3C00
    assert int(oracle.fp16_round_bits([1 + 3 * 2 ** -11])[0]) == 0x3C02


def test_sketch_layout_and_statistics():
    m, d, seed = 64, 32, 11
    bits = oracle.sketch_bf16_bits(m, d, seed)
    for (i, j) in [(0, 0), (0, 31), (1, 0), (63, 31), (17, 5)]:
        assert bits[i, j] == oracle.f64_to_bf16_bits(oracle.gauss(seed, i * d + j))
    S = oracle.sketch(256, 128, 0)
    assert abs(S.mean()) < 4.0 / math.sqrt(S.size)
    assert abs(S.var() - 1.0) < 0.02
    assert scipy.stats.kstest(S.ravel(), "norm").pvalue > 1e-4
    assert not np.array_equal(oracle.sketch(8, 8, 0), oracle.sketch(8, 8, 1))


# --------------------------------------------------------------------------
# quantizer

def test_quantizer_hand_fixture():
    g = _golden("qjl_hand_fixture.json")
    S = np.array(g["S"], dtype=np.float64)
    k = np.array(g["k"], dtype=np.float64)
    np.testing.assert_array_equal(S @ k, np.array(g["y"], dtype=np.float64))
    signs, norms, n16, band = oracle.quantize(k[None, :], S, band_rel=1e-5,
                                              want_band=True)
    word = sum(b << i for i, b in enumerate(g["bits"]))  # LSB-first
    assert int(signs[0, 0]) == word
    assert norms[0] == pytest.approx(math.sqrt(5.0), rel=1e-15)
    assert int(n16[0]) == int(g["norm_fp16_hex"], 16)
    zero_rows = [i for i, y in enumerate(g["y"]) if y == 0]
    assert list(np.nonzero(band[0])[0]) == zero_rows


def test_quantizer_word_layout_multiword():
    # row i of S is +-e_{i mod d}; the code of k = (1, 1, ..., 1) has bit i set
    # iff row i is +e: pins word order for m = 128 (4 words)
    d, m = 8, 128
    sgn = np.array([1 if (i * 7) % 3 else -1 for i in range(m)], dtype=np.float64)
    S = np.zeros((m, d))
    S[np.arange(m), np.arange(m) % d] = sgn
    signs, _, _, _ = oracle.quantize(np.ones((1, d)), S)
    for i in range(m):
        assert ((int(signs[0, i // 32]) >> (i % 32)) & 1) == (1 if sgn[i] > 0 else 0)


# --------------------------------------------------------------------------
# estimator: constant, unbiasedness, variance

def _ring_sketch(m):
    """Rows c (cos phi_i, sin phi_i), phi_i on a uniform midpoint grid, with
    c = E|r| = sqrt(pi/2) for the Rayleigh radius of a 2-D standard normal.
    The estimator is linear in each row's radius, so its expectation over a
    Gaussian sketch equals this deterministic quadrature in the limit."""
    phi = 2 * np.pi * (np.arange(m) + 0.5) / m
    return math.sqrt(math.pi / 2) * np.stack([np.cos(phi), np.sin(phi)], 1)


@pytest.mark.parametrize("q,k", [((1.0, 0.3), (2.0, -1.0)),
                                 ((-0.7, 2.0), (0.5, 0.5)),
                                 ((1.0, 1.0), (1.0, -1.0)),   # orthogonal
                                 ((3.0, -4.0), (-1.5, 2.0))])  # anti-parallel
def test_estimator_constant_by_quadrature(q, k):
    # E[(s.q) sign(s.k)] = sqrt(2/pi) <q,k>/||k||; the dequantizer's
    # sqrt(pi/2) must undo it exactly.
    S = _ring_sketch(1 << 16)
    q, k = np.array(q), np.array(k)
    est = oracle.estimate(q, k, S)
    assert est == pytest.approx(float(q @ k), abs=1e-4 * np.linalg.norm(q) * np.linalg.norm(k))


def _sketch_estimates(q, k, m, R, seed):
    rng = np.random.default_rng(seed)
    d = q.size
    est = np.empty(R)
    for r in range(R):
        S = rng.standard_normal((m, d))
        est[r] = oracle.estimate(q, k, S)
    return est


def _closed_form_var(q, k, m):
    # sign^2 = 1 and E[(s.q)^2] = ||q||^2, so E[X^2] = (pi/2)||q||^2||k||^2/m
    # for the estimator X; the mean is <q,k>.
    return (math.pi / 2 * (q @ q) * (k @ k) - (q @ k) ** 2) / m


@pytest.mark.parametrize("seed", [1, 2])
def test_estimator_unbiased(seed):
    rng = np.random.default_rng(100 + seed)
    d, m, R = 16, 64, 3000
    q = rng.standard_normal(d)
    k = q * 0.8 + 0.6 * rng.standard_normal(d)   # correlated pair
    est = _sketch_estimates(q, k, m, R, seed)
    sem = est.std(ddof=1) / math.sqrt(R)
    assert abs(est.mean() - q @ k) < 4 * sem


def test_estimator_variance_closed_form_and_bound():
    rng = np.random.default_rng(5)
    d, m, R = 12, 32, 4000
    q = rng.standard_normal(d)
    k = rng.standard_normal(d) + 0.5 * q
    est = _sketch_estimates(q, k, m, R, 9)
    v = est.var(ddof=1)
    v_cf = _closed_form_var(q, k, m)
    assert v == pytest.approx(v_cf, rel=0.12)
    # property 2 (m rows): variance <= pi/(2m) ||q||^2 ||k||^2
    assert v_cf <= math.pi / (2 * m) * (q @ q) * (k @ k)


def test_estimator_variance_scales_as_one_over_m():
    rng = np.random.default_rng(6)
    d = 8
    q = rng.standard_normal(d)
    k = rng.standard_normal(d)
    ms = [32, 128, 512, 2048]
    vs = [_sketch_estimates(q, k, m, 600, 20 + m).var(ddof=1) for m in ms]
    slope = np.polyfit(np.log(ms), np.log(vs), 1)[0]
    assert slope == pytest.approx(-1.0, abs=0.12)


def test_recovery_on_tiny_case():
    rng = np.random.default_rng(8)
    q = np.array([0.3, -1.2, 0.7])
    k = np.array([1.1, 0.4, -0.9])
    errs = []
    for m in [1 << 8, 1 << 12, 1 << 16]:
        S = rng.standard_normal((m, 3))
        errs.append(abs(oracle.estimate(q, k, S) - q @ k)
                    / (np.linalg.norm(q) * np.linalg.norm(k)))
    assert errs[-1] < 5 * math.sqrt(math.pi / 2 / (1 << 16))
    assert errs[-1] < errs[0]


@pytest.mark.parametrize("m,d", [(64, 64), (256, 128), (512, 64)])
def test_normalised_error_matches_closed_form(m, d):
    # rms over independent Gaussian (q, k) of (est - <q,k>)/(||q|| ||k||) is
    # sqrt((pi/2 - E cos^2)/m) with E cos^2 = 1/d
    rng = np.random.default_rng(m + d)
    S = rng.standard_normal((m, d))
    n = 4000
    Q = rng.standard_normal((n, d))
    K = rng.standard_normal((n, d))
    signs, norms, _, _ = oracle.quantize(K, S)
    U = oracle.project(Q, S)
    est = np.array([oracle.scores(U[i], signs[i:i + 1], norms[i:i + 1])[0]
                    for i in range(n)])
    exact = np.einsum("ij,ij->i", Q, K)
    err = (est - exact) / (np.linalg.norm(Q, axis=1) * np.linalg.norm(K, axis=1))
    pred = math.sqrt((math.pi / 2 - 1.0 / d) / m)
    assert np.sqrt(np.mean(err ** 2)) == pytest.approx(pred, rel=0.06)


# --------------------------------------------------------------------------
# attention stage

def _identity_sketch(d):
    return np.eye(d)


def test_decode_reduces_to_softmax_of_known_scores():
    # S = I (m = d = 32): u = q, score_t = sqrt(pi/2)/32 * n_t * sum_i q_i sigma_ti
    rng = np.random.default_rng(2)
    d = m = 32
    T = 7
    q = np.zeros(d)
    q[3] = 2.0
    codes = rng.integers(0, 2 ** 32, size=T, dtype=np.uint64).astype(np.uint32)
    norms = rng.uniform(0.5, 3.0, size=T)
    sigma3 = np.where((codes >> 3) & 1, 1.0, -1.0)
    s = math.sqrt(math.pi / 2) / m * norms * 2.0 * sigma3
    V = rng.standard_normal((T, d))
    scale = 0.37
    out, sc = oracle.decode(q[None, None, :], _identity_sketch(d),
                            codes.reshape(1, 1, T, 1), norms[None, None, :],
                            V[None, None], scale, want_scores=True)
    np.testing.assert_allclose(sc[0, 0], s, rtol=1e-13, atol=1e-14)
    p = scipy.special.softmax(s * scale)
    np.testing.assert_allclose(out[0, 0], p @ V, rtol=1e-12, atol=1e-13)


def test_decode_single_key_returns_its_value():
    rng = np.random.default_rng(4)
    d, m = 16, 32
    S = rng.standard_normal((m, d))
    K = rng.standard_normal((1, d))
    signs, norms, _, _ = oracle.quantize(K, S)
    V = rng.standard_normal((1, 1, 1, d))
    out, _ = oracle.decode(rng.standard_normal((1, 1, d)), S,
                           signs.reshape(1, 1, 1, 1), norms.reshape(1, 1, 1),
                           V, 0.25)
    np.testing.assert_allclose(out[0, 0], V[0, 0, 0], rtol=1e-14)


def test_decode_identical_keys_average_values():
    rng = np.random.default_rng(5)
    d, m, T = 16, 64, 9
    S = rng.standard_normal((m, d))
    k = rng.standard_normal((1, d))
    signs, norms, _, _ = oracle.quantize(np.repeat(k, T, 0), S)
    V = rng.standard_normal((1, 1, T, d))
    out, _ = oracle.decode(rng.standard_normal((1, 1, d)), S,
                           signs.reshape(1, 1, T, 2), norms.reshape(1, 1, T),
                           V, 1.0)
    np.testing.assert_allclose(out[0, 0], V[0, 0].mean(0), rtol=1e-12, atol=1e-14)


def test_decode_state_of_known_scores():
    # S = I as above: the part's lse2 is log2 of the library's sum of exps of
    # the known logits, and its output is the plain decode of the part
    rng = np.random.default_rng(21)
    d = m = 32
    T = 11
    q = rng.standard_normal(d) * 3.0
    codes = rng.integers(0, 2 ** 32, size=T, dtype=np.uint64).astype(np.uint32)
    norms = rng.uniform(0.5, 3.0, size=T)
    bits = (codes[:, None] >> np.arange(32)[None, :]) & 1
    s = math.sqrt(math.pi / 2) / m * norms * (np.where(bits, 1.0, -1.0) @ q)
    V = rng.standard_normal((T, d))
    scale = 0.61
    out, lse2 = oracle.decode_state(q[None, None, :], _identity_sketch(d),
                                    codes.reshape(1, 1, T, 1), norms[None, None, :],
                                    V[None, None], scale)
    assert lse2.shape == (1, 1)
    np.testing.assert_allclose(lse2[0, 0], scipy.special.logsumexp(scale * s) / math.log(2),
                               rtol=1e-13)
    np.testing.assert_allclose(out[0, 0], scipy.special.softmax(scale * s) @ V, rtol=1e-12,
                               atol=1e-13)


@pytest.mark.parametrize("cuts", [(1,), (20, 21), (5, 17, 30, 39), (40,)])
def test_merge_of_split_states_equals_whole_decode(cuts):
    # softmax over a union of disjoint key sets: merging the parts' states
    # must give the C decode over the whole context (GQA, peaked logits)
    rng = np.random.default_rng(22)
    B, Hq, Hkv, T, m, d = 2, 4, 2, 41, 64, 16
    S = rng.standard_normal((m, d))
    K = rng.standard_normal((B * Hkv * T, d)) * 2.0
    signs, norms, _, _ = oracle.quantize(K, S)
    signs = signs.reshape(B, Hkv, T, m // 32)
    norms = norms.reshape(B, Hkv, T)
    V = rng.standard_normal((B, Hkv, T, d))
    Q = rng.standard_normal((B, Hq, d)) * 2.0
    scale = 0.9
    whole, _ = oracle.decode(Q, S, signs, norms, V, scale)
    edges = (0,) + tuple(cuts) + (T,)
    parts = [oracle.decode_state(Q, S, signs[:, :, a:b], norms[:, :, a:b], V[:, :, a:b],
                                 scale) for a, b in zip(edges[:-1], edges[1:])]
    merged = oracle.merge_states([p[0] for p in parts], [p[1] for p in parts])
    np.testing.assert_allclose(merged, whole, rtol=1e-11, atol=1e-12)
    # the parts' softmax masses add up to the whole's
    _, lse_whole = oracle.decode_state(Q, S, signs, norms, V, scale)
    tot = np.log2(sum(np.exp2(p[1]) for p in parts))
    np.testing.assert_allclose(tot, lse_whole, rtol=1e-12)


def test_decode_grouped_query_head_mapping():
    # Hq = 6, Hkv = 2: heads 0..2 read KV head 0, heads 3..5 read KV head 1
    rng = np.random.default_rng(6)
    d, m, B = 8, 32, 2
    S = rng.standard_normal((m, d))
    K = rng.standard_normal((B * 2, d))
    signs, norms, _, _ = oracle.quantize(K, S)
    V = rng.standard_normal((B, 2, 1, d))
    out, _ = oracle.decode(rng.standard_normal((B, 6, d)), S,
                           signs.reshape(B, 2, 1, 1), norms.reshape(B, 2, 1),
                           V, 1.0)
    for b in range(B):
        for h in range(6):
            np.testing.assert_allclose(out[b, h], V[b, h // 3, 0], rtol=1e-14)


def test_decode_scores_equal_estimator():
    rng = np.random.default_rng(7)
    d, m, T = 16, 64, 20
    S = rng.standard_normal((m, d))
    K = rng.standard_normal((T, d))
    q = rng.standard_normal(d)
    signs, norms, _, _ = oracle.quantize(K, S)
    _, sc = oracle.decode(q[None, None], S, signs.reshape(1, 1, T, 2),
                          norms.reshape(1, 1, T), rng.standard_normal((1, 1, T, d)),
                          1.0, want_scores=True)
    for t in range(T):
        assert sc[0, 0, t] == pytest.approx(oracle.estimate(q, K[t], S), rel=1e-12)


def test_exact_attention_matches_library_softmax():
    rng = np.random.default_rng(9)
    d, T = 8, 11
    Q = rng.standard_normal((1, 1, d))
    K = rng.standard_normal((1, 1, T, d))
    V = rng.standard_normal((1, 1, T, d))
    out, sc = oracle.exact_attention(Q, K, V, 0.5, want_scores=True)
    s = K[0, 0] @ Q[0, 0]
    np.testing.assert_allclose(sc[0, 0], s, rtol=1e-13)
    np.testing.assert_allclose(out[0, 0], scipy.special.softmax(0.5 * s) @ V[0, 0],
                               rtol=1e-12)


# --------------------------------------------------------------------------
# storage arithmetic printed on the pages

def test_block_overhead_worked_example():
    g = _golden("block_overhead_example.json")
    for c in g["cases"]:
        eff = oracle.block_effective_bits(c["bits"], c["block"], g["const_bits"])
        assert eff == pytest.approx(c["effective_bits"], abs=0)
        if "overhead_fraction_of_budget" in c:
            assert (eff - c["bits"]) / c["bits"] == c["overhead_fraction_of_budget"]


def test_qjl_code_has_no_block_constants():
    # one norm per vector, not per block: m = d = 128 with a 16-bit norm costs
    # 1 + 16/128 bits per coordinate, independent of any block size
    assert oracle.qjl_bits_per_coordinate(128, 128, 16) == 1.125
    assert oracle.qjl_bits_per_coordinate(256, 128, 16) == 2.125


# --------------------------------------------------------------------------
# dequantizer Q^-1 ("The Geometry of Forgetting ...", QJL section), with m
# rows and the stored norm: khat = sqrt(pi/2)/m * ||k|| * S^T sign(S k)

def test_dequantizer_hand_fixture():
    fx = _golden("qjl_dequant_fixture.json")
    d, m = fx["d"], fx["m"]
    S = np.zeros((m, d))
    S[:2] = np.array(fx["S_rows_0_1"], dtype=np.float64)
    for key in fx["keys"]:
        k = np.array(key["k"], dtype=np.float64)
        signs, norms, _, _ = oracle.quantize(k[None], S)
        assert int(signs[0, 0]) == key["code"]
        assert norms[0] ** 2 == pytest.approx(key["norm_sq"], rel=1e-15)
        khat = oracle.dequantize(signs, norms, S)[0]
        want = math.sqrt(math.pi / 2) / m * math.sqrt(key["norm_sq"]) * np.array(key["StZ"])
        assert np.allclose(khat, want, rtol=1e-14, atol=1e-15)


def test_dequantizer_inner_product_equals_estimator():
    # <y, Q^-1(Q(k))> is the asymmetric estimator, whatever y is: this ties
    # the dequantizer's orientation (S^T z, not S z) and constant to the
    # estimator, which is pinned on its own above
    rng = np.random.default_rng(31)
    d, m, n = 24, 96, 40
    S = rng.standard_normal((m, d))
    K = rng.standard_normal((n, d))
    Y = rng.standard_normal((n, d)) * 3
    signs, norms, _, _ = oracle.quantize(K, S)
    khat = oracle.dequantize(signs, norms, S)
    U = oracle.project(Y, S)
    for i in range(n):
        est = oracle.scores(U[i], signs[i:i + 1], norms[i:i + 1])[0]
        assert Y[i] @ khat[i] == pytest.approx(est, rel=1e-12, abs=1e-12)


def _reconstructions(k, m, R, seed):
    rng = np.random.default_rng(seed)
    d = k.shape[0]
    out = np.empty((R, d))
    for r in range(R):
        S = rng.standard_normal((m, d))
        signs, norms, _, _ = oracle.quantize(k[None], S)
        out[r] = oracle.dequantize(signs, norms, S)[0]
    return out


def test_dequantizer_unbiased():
    # E_S[khat] = sqrt(pi/2)/m ||k|| * m * E[s sign(s.k)] = k
    rng = np.random.default_rng(40)
    d, m, R = 10, 64, 4000
    k = rng.standard_normal(d) * 2
    rec = _reconstructions(k, m, R, 41)
    sem = rec.std(axis=0, ddof=1) / math.sqrt(R)
    assert np.all(np.abs(rec.mean(axis=0) - k) < 5 * sem)


@pytest.mark.parametrize("m", [32, 128, 512])
def test_reconstruction_mse_closed_form(m):
    # D_mse of the page, for this quantizer: E||k - khat||^2 =
    # ||k||^2 ((pi/2) d - 1) / m  (E||khat||^2 = ||k||^2 ((pi/2) d/m + (m-1)/m)
    # for i.i.d. N(0,1) rows, minus ||k||^2 since khat is unbiased)
    rng = np.random.default_rng(50 + m)
    d, R = 16, 1500
    k = rng.standard_normal(d)
    rec = _reconstructions(k, m, R, 60 + m)
    err = np.sum((rec - k) ** 2, axis=1) / (k @ k)
    pred = (math.pi / 2 * d - 1) / m
    sem = err.std(ddof=1) / math.sqrt(R)
    assert abs(err.mean() - pred) < 5 * sem
    assert err.mean() == pytest.approx(pred, rel=0.08)


# --------------------------------------------------------------------------
# inner-product search over a compressed index (the final section of "The
# Geometry of Forgetting ...": the same quantizer for any store of vectors
# read through inner products)

def test_search_topk_brute_force_tiny():
    rng = np.random.default_rng(70)
    d, m, N, nq, k = 8, 32, 40, 5, 6
    S = rng.standard_normal((m, d))
    X = rng.standard_normal((N, d))
    X[7] = X[3]                                   # an exact tie
    Q = rng.standard_normal((nq, d))
    signs, norms, _, _ = oracle.quantize(X, S)
    idx, sc, _ = oracle.search_topk(Q, S, signs, norms, k)
    for i in range(nq):
        est = [oracle.estimate(Q[i], X[j], S) for j in range(N)]
        want = sorted(range(N), key=lambda j: (-est[j], j))[:k]
        assert list(idx[i]) == want
        assert np.allclose(sc[i], [est[j] for j in want], rtol=1e-12)


def test_search_recovers_exact_top1_with_many_rows():
    # the estimator concentrates as m grows, so the estimated best match of a
    # planted near-duplicate is the exact best match
    rng = np.random.default_rng(71)
    d, N = 32, 300
    X = rng.standard_normal((N, d))
    Q = X[[11, 200, 57]] * 1.0 + 0.05 * rng.standard_normal((3, d))
    exact = np.argmax(Q @ X.T, axis=1)
    S = rng.standard_normal((4096, d))
    signs, norms, _, _ = oracle.quantize(X, S)
    idx, _, _ = oracle.search_topk(Q, S, signs, norms, 1)
    assert list(idx[:, 0]) == list(exact)
