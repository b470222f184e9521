"""Failure detection on the GPU without a GPU fault.

Every wait inside the library's kernels is bounded.  When one runs out, the
kernel records a code in the device error word, lets the copies it started
land, frees its tensor memory and returns, so the context stays usable.  The
test hook jl_test_drop_copies makes the next launches start no copy at all
(the message that never arrives), with a 1 ms bound on the waits: the
consumers' waits then run out.  Each test checks that the call returns well
before the default 2 s bound, that jl_device_error reports the kernel's
timeout code, and that a normal call right after it gives the oracle's
results (for the tensor-core quantizer this also shows its tensor memory was
freed: the next launch allocates it again).
"""
import math
import time

import numpy as np
import pytest
import torch

import bit_jl_key_b200 as jl
import oracle
import workloads
from tests import helpers as H

pytestmark = pytest.mark.gpu

LIMIT_NS = 1_000_000          # 1 ms per wait


@pytest.fixture(autouse=True)
def _device():
    jl.load()
    torch.cuda.set_device(0)
    assert jl.jl_device_error() == 0
    yield
    jl.jl_test_drop_copies(False, 0)
    assert jl.jl_device_error() == 0


def _timed_failing_call(fn):
    """Run fn with every copy dropped; returns (device error code, seconds)."""
    torch.cuda.synchronize()
    jl.jl_test_drop_copies(True, LIMIT_NS)
    try:
        t0 = time.perf_counter()
        fn()
        code = jl.jl_device_error()           # synchronises
        dt = time.perf_counter() - t0
    finally:
        jl.jl_test_drop_copies(False, 0)
    return code, dt


@pytest.mark.parametrize("m,d", [(256, 128), (512, 64)])
def test_quantizer_wait_runs_out_then_recovers(m, d):
    n = 50_000                                 # several tiles per CTA
    S = jl.jl_sketch_init(m, d, 0)
    S64 = oracle.sketch(m, d, 0)
    K = workloads.random_keys(n, d, seed=71).cuda()
    jl.jl_quantize_keys(K, S)                  # module loaded, maps encoded
    torch.cuda.synchronize()

    code, dt = _timed_failing_call(lambda: jl.jl_quantize_keys(K, S))
    assert code == jl.JL_DERR_TC_WAIT_TIMEOUT
    assert dt < 1.0, dt                        # the 1 ms bound, not the 2 s default

    signs, norms = jl.jl_quantize_keys(K, S)   # a normal call right after
    rsig, _, rn16, band = oracle.quantize(H.f64(K), S64, band_rel=H.BAND_REL, want_band=True)
    out_band, _ = H.compare_codes(H.u32(signs), rsig, band, m)
    assert out_band == 0
    assert H.fp16_ulp_diff(H.fp16_bits(norms), rn16).max() <= 1


def test_decode_wait_runs_out_then_recovers():
    B, Hq, Hkv, T, m, d = 2, 8, 2, 3000, 256, 128
    S = jl.jl_sketch_init(m, d, 0)
    S64 = oracle.sketch(m, d, 0)
    K = workloads.random_keys(B * Hkv * T, d, 81)
    V = workloads.random_keys(B * Hkv * T, d, 82).reshape(B, Hkv, T, d).cuda()
    Q = workloads.random_keys(B * Hq, d, 83, scale=2.0).reshape(B, Hq, d).cuda()
    rsig, _, rn16, _ = oracle.quantize(H.f64(K), S64)
    signs = torch.from_numpy(rsig.view(np.int32).reshape(B, Hkv, T, m // 32)).cuda()
    norms = torch.from_numpy(rn16.view(np.float16).reshape(B, Hkv, T)).cuda()
    scale = 1.0 / math.sqrt(d)
    jl.jl_decode_attention(Q, S, signs, norms, V, softmax_scale=scale)
    torch.cuda.synchronize()

    code, dt = _timed_failing_call(
        lambda: jl.jl_decode_attention(Q, S, signs, norms, V, softmax_scale=scale))
    assert code == jl.JL_DERR_DECODE_WAIT_TIMEOUT
    assert dt < 1.0, dt

    out, sc = jl.jl_decode_attention(Q, S, signs, norms, V, softmax_scale=scale,
                                     want_scores=True)
    ref_out, ref_sc = oracle.decode(H.f64(Q), S64, rsig.reshape(B, Hkv, T, m // 32),
                                    oracle.fp16_bits_to_f64(rn16).reshape(B, Hkv, T),
                                    H.f64(V), scale, want_scores=True)
    assert H.score_violations(H.f64(sc), ref_sc) == 0
    mabs, rel = H.output_errors(H.f64(out), ref_out)
    assert mabs <= H.OUT_ABS and rel <= 1e-2

