"""Parity at the workloads' full sizes, on sampled outputs.

The GPU quantizes the whole cache and decodes it in the same launch
configuration the bench times.  The oracle recomputes a sample: whole
(b, kv-head) units for the decode workloads, and random keys for the prefill
workload.  Each sampled unit is checked twice: the GPU chain (the GPU's own
codes decoded on the GPU; scores compared on every key whose code and norm
equal the oracle's, outputs whole), then with the oracle's codes written into
the GPU cache (every score and output).
"""
import math

import numpy as np
import pytest
import torch

import bit_jl_key_b200 as jl
import oracle
import workloads
from tests import helpers as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    jl.load()
    torch.cuda.set_device(0)
    yield
    torch.cuda.empty_cache()
    assert jl.jl_device_error() == 0


def _decode_workload_check(w, units, q_scale=1.0):
    dev = "cuda"
    S = jl.jl_sketch_init(w.m, w.d, w.sketch_seed)
    S64 = oracle.sketch(w.m, w.d, w.sketch_seed)
    K = workloads.keys(w, dev)
    V = workloads.values(w, dev)
    Q = workloads.queries(w, dev, q_scale)
    W = w.m // 32
    signs, norms = jl.jl_quantize_keys(K.view(-1, w.d), S)
    signs = signs.view(w.B, w.Hkv, w.T, W)
    norms = norms.view(w.B, w.Hkv, w.T)
    # 1) the GPU chain: decode the GPU's own codes and norms
    out, sc = jl.jl_decode_attention(Q, S, signs, norms, V,
                                     softmax_scale=w.softmax_scale,
                                     want_scores=True)
    torch.cuda.synchronize()
    chain = {}
    for (b, hk) in units:
        hqs = list(range(hk * w.G, (hk + 1) * w.G))
        chain[(b, hk)] = (H.f64(sc[b, hqs])[None], H.f64(out[b, hqs])[None])
    del out, sc
    # 2) the oracle's codes for the sampled units: compared with the GPU's
    # (band rule), then written into the cache for an all-keys decode check
    report, refs = [], {}
    for (b, hk) in units:
        Kf = H.f64(K[b, hk])
        rsig, _, rn16, band = oracle.quantize(Kf, S64, band_rel=H.BAND_REL,
                                              want_band=True)
        g_words, g_norm = H.u32(signs[b, hk]), H.fp16_bits(norms[b, hk])
        out_band, in_band = H.compare_codes(g_words, rsig, band, w.m)
        assert out_band == 0, (b, hk, out_band)
        ulp = H.fp16_ulp_diff(g_norm, rn16)
        assert ulp.max() <= 1
        mask = H.key_match_mask(g_words, rsig, g_norm, rn16)
        refs[(b, hk)] = mask
        report.append((b, hk, in_band, int((ulp > 0).sum()), int((~mask).sum())))
        signs[b, hk] = torch.from_numpy(rsig.view(np.int32)).to(dev)
        norms[b, hk] = torch.from_numpy(rn16.view(np.float16)).to(dev)
    del K
    out, sc = jl.jl_decode_attention(Q, S, signs, norms, V,
                                     softmax_scale=w.softmax_scale,
                                     want_scores=True)
    torch.cuda.synchronize()
    for (b, hk) in units:
        hqs = list(range(hk * w.G, (hk + 1) * w.G))
        Qs = H.f64(Q[b, hqs])[None]
        rsig = H.u32(signs[b, hk])[None, None]
        rn = H.f64(norms[b, hk])[None, None]
        Vs = H.f64(V[b, hk])[None, None]
        ref_out, ref_sc = oracle.decode(Qs, S64, rsig, rn, Vs, w.softmax_scale,
                                        want_scores=True)
        # planted codes: every score and output
        g_sc = H.f64(sc[b, hqs])[None]
        g_out = H.f64(out[b, hqs])[None]
        assert H.score_violations(g_sc, ref_sc) == 0, (b, hk)
        mabs, rel = H.output_errors(g_out, ref_out)
        assert mabs <= H.OUT_ABS and rel <= 1e-2, (b, hk, mabs, rel)
        # GPU chain: scores of the keys whose code and norm match the
        # oracle's exactly; outputs of the whole chain
        c_sc, c_out = chain[(b, hk)]
        mask = refs[(b, hk)]
        assert int((~mask).sum()) <= max(4, w.T // 100), (b, hk)
        assert H.masked_score_violations(c_sc, ref_sc, mask) == 0, (b, hk)
        mabs, _ = H.output_errors(c_out, ref_out)
        assert mabs <= H.OUT_ABS, (b, hk, mabs)
    print(f"{w.name} m={w.m} d={w.d}: units (b, hkv, in-band flips, norm ulps, "
          f"keys left out of the chain's score check) {report}")


def test_gqa_full_size():
    w = workloads.GQA
    _decode_workload_check(w, [(0, 0), (7, 7), (3, 5)])


def test_long_context_full_size():
    w = workloads.LONG
    _decode_workload_check(w, [(0, 0), (0, 31)])


@pytest.mark.parametrize("w", workloads.sweep_points(), ids=lambda w: f"m{w.m}d{w.d}")
def test_sweep_full_size(w):
    _decode_workload_check(w, [(15, 31)])


def test_prefill_full_size_sampled_keys():
    w = workloads.PREFILL
    S = jl.jl_sketch_init(w.m, w.d, w.sketch_seed)
    S64 = oracle.sketch(w.m, w.d, w.sketch_seed)
    K = workloads.keys(w, "cuda").view(-1, w.d)
    signs, norms = jl.jl_quantize_keys(K, S)
    rng = np.random.default_rng(4)
    idx = np.unique(np.concatenate([rng.integers(0, K.shape[0], 8192),
                                    [0, K.shape[0] - 1]]))
    it = torch.from_numpy(idx).cuda()
    Ks = H.f64(K[it])
    rsig, _, rn16, band = oracle.quantize(Ks, S64, band_rel=H.BAND_REL,
                                          want_band=True)
    out_band, in_band = H.compare_codes(H.u32(signs[it]), rsig, band, w.m)
    assert out_band == 0
    ulp = H.fp16_ulp_diff(H.fp16_bits(norms[it]), rn16)
    assert ulp.max() <= 1
    print(f"prefill: {len(idx)} sampled keys, {in_band} in-band flips, "
          f"{int((ulp > 0).sum())} norms 1 ulp off")
