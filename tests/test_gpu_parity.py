"""GPU vs oracle parity at sizes the oracle finishes in seconds.

Every GPU result is produced through the C ABI (the ctypes binding) and
compared element by element with the float64 oracle on the same seeded
inputs.  Decode comparisons feed both sides the oracle's codes and norms, so
they isolate the decode kernels from the quantizer's near-zero band; the
end-to-end test chains the GPU quantizer into the GPU decode.
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

ALL_MD = [(m, d) for d in (64, 128) for m in (64, 128, 256, 512)]


@pytest.fixture(scope="module", autouse=True)
def _device():
    jl.load()
    torch.cuda.set_device(0)
    yield
    assert jl.jl_device_error() == 0


def _oracle_codes(K: torch.Tensor, S_f64: np.ndarray, band=True):
    Kf = H.f64(K.reshape(-1, K.shape[-1]))
    return oracle.quantize(Kf, S_f64, band_rel=H.BAND_REL, want_band=band)


# --------------------------------------------------------------------------
# sketch

@pytest.mark.parametrize("m,d", ALL_MD)
@pytest.mark.parametrize("seed", [0, 12345, 2 ** 63 + 7])
def test_sketch_bit_exact(m, d, seed):
    S = jl.jl_sketch_init(m, d, seed)
    ref = oracle.sketch_bf16_bits(m, d, seed)
    got = S.cpu().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, ref)


# --------------------------------------------------------------------------
# quantizer

QUANT_CASES = [
    # (n, m, d, dtype)
    (1024, 256, 128, torch.float32),     # the single-head workload's keys
    (1, 256, 128, torch.bfloat16),
    (31, 64, 64, torch.bfloat16),
    (1000, 128, 128, torch.bfloat16),
    (4099, 256, 128, torch.bfloat16),
    (777, 512, 128, torch.bfloat16),
    (2050, 512, 64, torch.bfloat16),
    (513, 128, 64, torch.float32),
    (300, 64, 128, torch.bfloat16),
]


def _check_quantize(fn, K, S_gpu, S_f64, m):
    signs, norms = fn(K, S_gpu)
    rsig, _, rn16, band = _oracle_codes(K, S_f64)
    out_band, in_band = H.compare_codes(H.u32(signs), rsig, band, m)
    assert out_band == 0, f"{out_band} code bits differ outside the band"
    ulp = H.fp16_ulp_diff(H.fp16_bits(norms), rn16)
    assert ulp.max() <= 1
    return in_band, int(np.count_nonzero(ulp))


@pytest.mark.parametrize("impl", ["jl_quantize_keys", "jl_quantize_keys_simt"])
@pytest.mark.parametrize("n,m,d,dtype", QUANT_CASES)
def test_quantize_matches_oracle(impl, n, m, d, dtype):
    S = jl.jl_sketch_init(m, d, 0)
    S64 = oracle.sketch(m, d, 0)
    K = workloads.random_keys(n, d, seed=n + m + d, dtype=dtype).cuda()
    in_band, ulp1 = _check_quantize(getattr(jl, impl), K, S, S64, m)
    print(f"{impl} n={n} m={m} d={d}: {in_band} in-band flips, {ulp1} norms 1 ulp off")


@pytest.mark.parametrize("impl", ["jl_quantize_keys", "jl_quantize_keys_simt"])
def test_quantize_strided_keys(impl):
    m, d, n = 256, 128, 600
    S = jl.jl_sketch_init(m, d, 3)
    S64 = oracle.sketch(m, d, 3)
    big = workloads.random_keys(n, 3 * d, seed=5).cuda()
    K = big[:, d:2 * d]                      # row stride 3d, offset d
    assert K.stride(0) == 3 * d
    _check_quantize(getattr(jl, impl), K, S, S64, m)


@pytest.mark.parametrize("impl", ["jl_quantize_keys", "jl_quantize_keys_simt"])
def test_quantize_degenerate_keys(impl):
    # zero keys: every projection is exactly 0 -> code all ones (sign(0)=+1),
    # norm 0; huge and tiny keys keep their codes and round their norms
    m, d = 256, 128
    S = jl.jl_sketch_init(m, d, 0)
    S64 = oracle.sketch(m, d, 0)
    K = torch.zeros((5, d), dtype=torch.bfloat16)
    K[1] = workloads.random_keys(1, d, 1)[0] * 1000.0
    K[2] = workloads.random_keys(1, d, 2)[0] * 1e-3
    K[3, 7] = 1.0                               # one-hot key
    signs, norms = getattr(jl, impl)(K.cuda(), S)
    rsig, _, rn16, band = _oracle_codes(K, S64)
    assert np.all(H.u32(signs)[0] == 0xFFFFFFFF)
    assert H.fp16_bits(norms)[0] == 0
    out_band, _ = H.compare_codes(H.u32(signs), rsig, band, m)
    assert out_band == 0
    assert H.fp16_ulp_diff(H.fp16_bits(norms), rn16).max() <= 1


def test_quantize_empty_is_noop():
    S = jl.jl_sketch_init(256, 128, 0)
    signs, norms = jl.jl_quantize_keys(torch.empty((0, 128), dtype=torch.bfloat16,
                                                   device="cuda"), S)
    assert signs.numel() == 0 and norms.numel() == 0


# --------------------------------------------------------------------------
# decode

DECODE_CASES = [
    # (B, Hq, Hkv, T, m, d, qdtype, q_scale)
    (1, 1, 1, 1024, 256, 128, torch.float32, 1.0),   # single-head workload
    (2, 8, 2, 1000, 256, 128, torch.bfloat16, 1.0),  # GQA, ragged context
    (1, 4, 4, 33, 128, 64, torch.bfloat16, 3.0),     # MHA, one key past a block
    (1, 2, 1, 1, 256, 128, torch.bfloat16, 1.0),     # a single key
    (2, 16, 1, 300, 64, 64, torch.bfloat16, 2.0),    # 16 heads per KV head
    (1, 5, 1, 257, 512, 128, torch.bfloat16, 1.0),   # 5 heads, m = 512
    (1, 3, 3, 4096, 512, 64, torch.bfloat16, 4.0),   # peaked softmax
    (3, 6, 2, 2049, 128, 128, torch.float32, 1.0),
    (1, 8, 8, 8192, 64, 128, torch.bfloat16, 1.0),
    # head groups of 8 on the bulk-tensor copy path (T % 8 == 0)
    (1, 16, 1, 1024, 256, 128, torch.bfloat16, 2.0),
    (2, 12, 1, 512, 128, 64, torch.bfloat16, 1.0),
    # int8 scoring (one head per KV head, or m = 512) on both copy paths
    (1, 4, 4, 2048, 256, 128, torch.bfloat16, 3.0),
    (1, 4, 4, 1001, 128, 64, torch.bfloat16, 1.0),
    (1, 2, 2, 512, 512, 128, torch.bfloat16, 2.0),
    (2, 4, 1, 777, 512, 64, torch.bfloat16, 1.0),
    # one head per KV head with m >= 4d: keys as the int8 MMA's rows
    (2, 3, 3, 999, 256, 64, torch.float32, 2.0),
    (1, 2, 2, 4097, 512, 128, torch.bfloat16, 3.0),
    # two to four heads per KV head, keys as rows (m >= 4d, or d = 64)
    (2, 8, 2, 1500, 256, 64, torch.bfloat16, 2.0),
    (1, 6, 2, 700, 128, 64, torch.float32, 1.0),
    (2, 8, 4, 1000, 512, 128, torch.bfloat16, 3.0),
    (1, 12, 4, 4096, 512, 64, torch.bfloat16, 1.0),
]


def _decode_inputs(B, Hq, Hkv, T, m, d, qdtype, q_scale, seed):
    kd = torch.float32 if qdtype == torch.float32 else torch.bfloat16
    K = workloads.random_keys(B * Hkv * T, d, seed, dtype=kd).reshape(B, Hkv, T, d)
    V = workloads.random_keys(B * Hkv * T, d, seed + 1).reshape(B, Hkv, T, d)
    Q = workloads.random_keys(B * Hq, d, seed + 2, dtype=qdtype,
                              scale=q_scale).reshape(B, Hq, d)
    return K, V, Q


def _run_decode_case(B, Hq, Hkv, T, m, d, qdtype, q_scale, seed=11):
    S = jl.jl_sketch_init(m, d, 0)
    S64 = oracle.sketch(m, d, 0)
    K, V, Q = _decode_inputs(B, Hq, Hkv, T, m, d, qdtype, q_scale, seed)
    rsig, _, rn16, _ = _oracle_codes(K, S64, band=False)
    signs = torch.from_numpy(rsig.view(np.int32).reshape(B, Hkv, T, m // 32)).cuda()
    norms = torch.from_numpy(rn16.view(np.float16).reshape(B, Hkv, T)).cuda()
    scale = 1.0 / math.sqrt(d)
    out, sc = jl.jl_decode_attention(Q.cuda(), S, signs, norms, V.cuda(),
                                     softmax_scale=scale, want_scores=True)
    ref_out, ref_sc = oracle.decode(H.f64(Q), S64, rsig.reshape(B, Hkv, T, m // 32),
                                    oracle.fp16_bits_to_f64(rn16).reshape(B, Hkv, T),
                                    H.f64(V), scale, want_scores=True)
    return H.f64(out), H.f64(sc), ref_out, ref_sc


@pytest.mark.parametrize("case", DECODE_CASES)
def test_decode_matches_oracle(case):
    out, sc, ref_out, ref_sc = _run_decode_case(*case)
    assert H.score_violations(sc, ref_sc) == 0
    mabs, rel = H.output_errors(out, ref_out)
    print(f"decode {case}: max|dout|={mabs:.3e} max rel={rel:.3e}")
    assert mabs <= H.OUT_ABS
    assert rel <= 1e-2


def test_decode_zero_keys_average_values():
    B, Hq, Hkv, T, m, d = 1, 4, 2, 100, 256, 128
    S = jl.jl_sketch_init(m, d, 0)
    signs = torch.full((B, Hkv, T, m // 32), -1, dtype=torch.int32, device="cuda")
    norms = torch.zeros((B, Hkv, T), dtype=torch.float16, device="cuda")
    V = workloads.random_keys(B * Hkv * T, d, 9).reshape(B, Hkv, T, d).cuda()
    Q = workloads.random_keys(B * Hq, d, 10).reshape(B, Hq, d).cuda()
    out, sc = jl.jl_decode_attention(Q, S, signs, norms, V, want_scores=True)
    assert torch.count_nonzero(sc) == 0
    ref = H.f64(V).mean(axis=2)              # [B, Hkv, d]
    for h in range(Hq):
        np.testing.assert_allclose(H.f64(out)[0, h], ref[0, h // 2], atol=4e-3)


def test_decode_is_deterministic():
    case = (2, 8, 2, 1000, 256, 128, torch.bfloat16, 1.0)
    a = _run_decode_case(*case, seed=3)
    b = _run_decode_case(*case, seed=3)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_decode_empty_batch_is_noop():
    S = jl.jl_sketch_init(256, 128, 0)
    e = torch.empty
    out = jl.jl_decode_attention(
        e((0, 8, 128), dtype=torch.bfloat16, device="cuda"), S,
        e((0, 2, 16, 8), dtype=torch.int32, device="cuda"),
        e((0, 2, 16), dtype=torch.float16, device="cuda"),
        e((0, 2, 16, 128), dtype=torch.bfloat16, device="cuda"))
    assert out.shape == (0, 8, 128)


# --------------------------------------------------------------------------
# end to end: GPU quantizer feeding GPU decode

E2E_CASES = [(1, 1, 1, 1024, 256, 128, torch.float32, 1.0),
             (2, 8, 2, 3000, 256, 128, torch.bfloat16, 2.0),
             (1, 4, 4, 2048, 512, 64, torch.bfloat16, 3.0),
             (2, 6, 2, 1001, 64, 128, torch.bfloat16, 1.0)]


@pytest.mark.parametrize("case", E2E_CASES)
def test_end_to_end(case):
    """The GPU quantizer's codes and norms go straight into the GPU decode.
    The oracle runs its own chain (its codes, its norms, its estimator).  Every
    score of a key whose GPU code and norm equal the oracle's bit for bit must
    match the oracle's score; the keys left out (codes that differ inside the
    near-zero band, norms one binary16 step apart) are counted and must be
    few.  Outputs of the two chains are compared whole."""
    B, Hq, Hkv, T, m, d, qdtype, q_scale = case
    G = Hq // Hkv
    S = jl.jl_sketch_init(m, d, 0)
    S64 = oracle.sketch(m, d, 0)
    K, V, Q = _decode_inputs(B, Hq, Hkv, T, m, d, qdtype, q_scale, 21)
    signs, norms = jl.jl_quantize_keys(K.cuda().reshape(-1, d), S)
    out, sc = jl.jl_decode_attention(Q.cuda(), S, signs.reshape(B, Hkv, T, m // 32),
                                     norms.reshape(B, Hkv, T), V.cuda(),
                                     want_scores=True)
    rsig, _, rn16, band = _oracle_codes(K, S64)
    out_band, in_band = H.compare_codes(H.u32(signs), rsig, band, m)
    assert out_band == 0
    ulp = H.fp16_ulp_diff(H.fp16_bits(norms), rn16)
    assert ulp.max() <= 1
    ref_out, ref_sc = oracle.decode(H.f64(Q), S64, rsig.reshape(B, Hkv, T, m // 32),
                                    oracle.fp16_bits_to_f64(rn16).reshape(B, Hkv, T),
                                    H.f64(V), 1.0 / math.sqrt(d), want_scores=True)
    mask = H.key_match_mask(H.u32(signs), rsig, H.fp16_bits(norms), rn16)
    mask = mask.reshape(B, Hkv, 1, T).repeat(G, axis=2).reshape(B, Hq, T)
    left_out = int(np.count_nonzero(~mask[:, ::G]))
    assert left_out <= max(4, B * Hkv * T // 100), left_out
    assert H.masked_score_violations(H.f64(sc), ref_sc, mask) == 0
    mabs, rel = H.output_errors(H.f64(out), ref_out)
    print(f"e2e {case}: {in_band} in-band flips, {int((ulp > 0).sum())} norm ulps, "
          f"{left_out} of {B * Hkv * T} keys left out of the score check, "
          f"max|dout|={mabs:.3e}")
    assert mabs <= H.OUT_ABS
