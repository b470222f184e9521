"""Explicit dequantizer khat = sqrt(pi/2)/m * ||k|| * S^T z against the oracle.

The codes and norms fed to the GPU come from the oracle's quantization of
seeded keys (or are random bits); each bf16 output must be within one bf16
step of the oracle's float64 value rounded to bf16 (the GPU accumulates the
exact +-1 x bf16 products in fp32, scales in fp32 and rounds once).
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

MD = [(m, d) for d in (64, 128) for m in (64, 128, 256, 512)]


def _bf16_ordered(bits):
    b = bits.astype(np.int64)
    return np.where(b & 0x8000, -(b & 0x7FFF), b)


def _ref_bf16_bits(x):
    flat = x.reshape(-1)
    return np.array([oracle.f64_to_bf16_bits(float(v)) for v in flat], dtype=np.uint16).reshape(x.shape)


def _check(gpu_out, ref64):
    g = gpu_out.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    r = _ref_bf16_bits(ref64)
    ulp = np.abs(_bf16_ordered(g) - _bf16_ordered(r))
    assert ulp.max() <= 1, (int(ulp.max()), int(np.count_nonzero(ulp)))
    return int(np.count_nonzero(ulp))


@pytest.mark.parametrize("m,d", MD)
def test_dequantize_matches_oracle(m, d):
    torch.cuda.set_device(0)
    n = 300                                   # two full tiles and a ragged 44
    S = jl.jl_sketch_init(m, d, 0)
    S64 = oracle.sketch(m, d, 0)
    K = workloads.random_keys(n, d, 70 + m + d, scale=1.5)
    signs, _, n16, _ = oracle.quantize(H.f64(K), S64)
    sg = torch.from_numpy(signs.view(np.int32)).cuda()
    nr = torch.from_numpy(n16.view(np.float16)).cuda()
    out = jl.jl_dequantize_keys(sg, nr, S)
    torch.cuda.synchronize()
    assert jl.jl_device_error() == 0
    ref = oracle.dequantize(signs, oracle.fp16_bits_to_f64(n16), S64)
    _check(out, ref)


def test_dequantize_single_key_and_random_bits():
    torch.cuda.set_device(0)
    m, d = 256, 128
    S = jl.jl_sketch_init(m, d, 0)
    S64 = oracle.sketch(m, d, 0)
    rng = np.random.default_rng(5)
    for n in (1, 129):
        signs = rng.integers(0, 2 ** 32, size=(n, m // 32), dtype=np.uint64).astype(np.uint32)
        n16 = rng.uniform(0.01, 40.0, size=n).astype(np.float16).view(np.uint16)
        out = jl.jl_dequantize_keys(torch.from_numpy(signs.view(np.int32)).cuda(),
                                    torch.from_numpy(n16.view(np.float16)).cuda(), S)
        ref = oracle.dequantize(signs, oracle.fp16_bits_to_f64(n16), S64)
        _check(out, ref)


def test_dequantize_fullsize_sampled_rows():
    # the gqa cache size: 2.1 M codes, sampled rows against the oracle
    torch.cuda.set_device(0)
    m, d, n = 256, 128, 2097152
    S = jl.jl_sketch_init(m, d, 0)
    S64 = oracle.sketch(m, d, 0)
    g = torch.Generator(device="cuda")
    g.manual_seed(77)
    sg = torch.randint(-2 ** 31, 2 ** 31 - 1, (n, m // 32), dtype=torch.int32, device="cuda",
                       generator=g)
    nr = (torch.rand((n,), device="cuda", generator=g) * 20 + 0.1).half()
    out = jl.jl_dequantize_keys(sg, nr, S)
    torch.cuda.synchronize()
    assert jl.jl_device_error() == 0
    rows = np.unique(np.concatenate([np.arange(0, n, 65537), [0, 127, 128, n - 1]]))
    idx = torch.from_numpy(rows).cuda()
    signs = sg[idx].cpu().numpy().view(np.uint32)
    n16 = nr[idx].cpu().numpy().view(np.uint16)
    ref = oracle.dequantize(signs, oracle.fp16_bits_to_f64(n16), S64)
    _check(out[idx], ref)


@pytest.mark.parametrize("m,d", [(64, 128), (256, 128), (512, 64)])
def test_reconstruction_error_matches_closed_form(m, d):
    # property at any size: E||k - khat||^2 / ||k||^2 = ((pi/2) d - 1) / m,
    # an expectation over Gaussian S; one sketch can sit a few percent off it,
    # so the mean is taken over 8 seeded bf16 sketches (GPU quantize +
    # dequantize end to end, 16384 Gaussian keys each)
    torch.cuda.set_device(0)
    n = 16384
    means = []
    for seed in range(8):
        S = jl.jl_sketch_init(m, d, 100 + seed)
        K = workloads.random_keys(n, d, 90 + m + seed, device="cuda")
        sg, nr = jl.jl_quantize_keys(K, S)
        khat = jl.jl_dequantize_keys(sg, nr, S).float()
        k = K.float()
        means.append((((khat - k) ** 2).sum(1) / (k * k).sum(1)).mean().item())
    pred = (math.pi / 2 * d - 1) / m
    assert float(np.mean(means)) == pytest.approx(pred, rel=0.04)
