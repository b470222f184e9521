"""jl_decode_attention_noalloc: decode attention without a caller workspace.

Some callers cannot allocate device memory where they call this library
(plugins inside an engine that owns all device memory, latency-critical
paths), so the library offers a variant whose scratch is a static device
array.  This file checks, through the C ABI, that the variant returns what
jl_decode_attention returns with a caller-allocated workspace, on two calls
in a row (the second call reuses the array the first one left behind), and
that shapes too large for the array are refused before anything runs.  One
more case compares the variant straight with the float64 oracle, with an fp32
query.  It is named so that pytest collects it last.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

import bit_jl_key_b200 as jl
import oracle
import workloads
from tests import helpers as H

pytestmark = pytest.mark.gpu


def _inputs(B, Hq, Hkv, T, m, d, seed):
    S = jl.jl_sketch_init(m, d, 0)
    K = workloads.random_keys(B * Hkv * T, d, seed).cuda()
    V = workloads.random_keys(B * Hkv * T, d, seed + 1).reshape(B, Hkv, T, d).cuda()
    Q = workloads.random_keys(B * Hq, d, seed + 2, scale=2.0).reshape(B, Hq, d).cuda()
    signs, norms = jl.jl_quantize_keys(K, S)
    return (Q, S, signs.reshape(B, Hkv, T, m // 32), norms.reshape(B, Hkv, T), V)


def _compare(args):
    d = args[0].shape[-1]
    ref_out, ref_sc = jl.jl_decode_attention(*args, softmax_scale=1 / math.sqrt(d),
                                             want_scores=True)
    out, sc = jl.jl_decode_attention_noalloc(*args, softmax_scale=1 / math.sqrt(d),
                                             want_scores=True)
    torch.cuda.synchronize()
    assert H.score_violations(H.f64(sc), H.f64(ref_sc)) == 0
    mabs, rel = H.output_errors(H.f64(out), H.f64(ref_out))
    assert mabs <= H.OUT_ABS and rel <= 1e-2
    return torch.equal(out, ref_out)


def test_noalloc_matches_workspace_path_twice():
    torch.cuda.set_device(0)
    # two calls in a row with different shapes: the second one reads nothing
    # the first one left in the shared scratch
    first = _inputs(8, 32, 8, 4096, 256, 128, seed=40)
    second = _inputs(2, 8, 2, 1000, 128, 64, seed=50)
    same1 = _compare(first)
    same2 = _compare(second)
    print(f"noalloc bitwise equal to workspace path: {same1}, {same2}")
    assert jl.jl_device_error() == 0


def test_noalloc_refuses_shapes_beyond_its_scratch():
    torch.cuda.set_device(0)
    B, Hq, Hkv, T, m, d = 256, 32, 32, 64, 512, 128
    assert jl.jl_decode_workspace_bytes(B, Hq, Hkv, T, m, d) > jl.DECODE_STATIC_SCRATCH_BYTES
    fake = ctypes.c_void_p(1 << 20)
    st = jl.load().jl_decode_attention_noalloc(
        fake, jl.JL_BF16, fake, fake, fake, fake, B, Hq, Hkv, T, m, d,
        ctypes.c_float(0.1), fake, ctypes.c_void_p(0), ctypes.c_void_p(0))
    assert st == jl.JL_ERR_SCRATCH_LIMIT
    assert "static decode scratch" in jl.status_string(st)


def test_noalloc_matches_oracle_fp32_query():
    # the oracle's own codes and norms feed both sides, so the comparison
    # covers the decode alone (scores and outputs by the parity tests' rules)
    torch.cuda.set_device(0)
    B, Hq, Hkv, T, m, d = 2, 8, 2, 777, 256, 128
    S = jl.jl_sketch_init(m, d, 0)
    S64 = oracle.sketch(m, d, 0)
    K = workloads.random_keys(B * Hkv * T, d, 60, dtype=torch.float32)
    V = workloads.random_keys(B * Hkv * T, d, 61).reshape(B, Hkv, T, d)
    Q = workloads.random_keys(B * Hq, d, 62, dtype=torch.float32, scale=2.0).reshape(B, Hq, d)
    rsig, _, rn16, _ = oracle.quantize(H.f64(K), S64)
    signs = torch.from_numpy(rsig.view(np.int32).reshape(B, Hkv, T, m // 32)).cuda()
    norms = torch.from_numpy(rn16.view(np.float16).reshape(B, Hkv, T)).cuda()
    scale = 1.0 / math.sqrt(d)
    for _ in range(2):
        out, sc = jl.jl_decode_attention_noalloc(Q.cuda(), S, signs, norms, V.cuda(),
                                                 softmax_scale=scale, want_scores=True)
        torch.cuda.synchronize()
        ref_out, ref_sc = oracle.decode(H.f64(Q), S64, rsig.reshape(B, Hkv, T, m // 32),
                                        oracle.fp16_bits_to_f64(rn16).reshape(B, Hkv, T),
                                        H.f64(V), scale, want_scores=True)
        assert H.score_violations(H.f64(sc), ref_sc) == 0
        mabs, rel = H.output_errors(H.f64(out), ref_out)
        assert mabs <= H.OUT_ABS and rel <= 1e-2
    assert jl.jl_device_error() == 0
