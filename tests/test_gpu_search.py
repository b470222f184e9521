"""Top-k inner-product search over a compressed index against the oracle.

Where several answers are correct (near-ties), the test compares what is
unique: the GPU's scores must match the oracle's scores of the same indices,
and the returned set must be a valid top-k under the oracle's scores (it may
differ from the oracle's own set only by vectors scoring within tolerance of
the k-th best).
"""
import numpy as np
import pytest
import torch

import bit_jl_key_b200 as jl
import oracle
import workloads
from tests import helpers as H

pytestmark = pytest.mark.gpu


def _index(N, d, m, seed, S64):
    X = workloads.random_keys(N, d, seed, scale=1.0)
    # spread the norms so that the norm factor matters
    X = (X.float() * torch.linspace(0.5, 2.0, N)[:, None]).bfloat16()
    signs, _, n16, _ = oracle.quantize(H.f64(X), S64)
    return signs, n16


def _check(gi, gs, allsc, k):
    nq, N = allsc.shape
    rms = np.sqrt(np.mean(allsc ** 2, axis=1))
    for q in range(nq):
        tol = H.SCORE_REL * rms[q]
        valid = gi[q] >= 0
        nv = min(k, N)
        assert valid.sum() == nv
        idx = gi[q][:nv]
        assert len(set(idx.tolist())) == nv and idx.min() >= 0 and idx.max() < N
        ref = allsc[q, idx]
        assert np.all(np.abs(gs[q][:nv] - ref) <= tol + H.SCORE_REL * np.abs(ref)), q
        assert np.all(np.diff(gs[q][:nv]) <= tol), q            # best first
        kth = np.sort(allsc[q])[::-1][nv - 1]
        assert np.all(ref >= kth - 2 * tol), q                   # a valid top-k
        if nv < k:
            assert np.all(gi[q][nv:] == -1) and np.all(np.isneginf(gs[q][nv:]))


@pytest.mark.parametrize("m,d,N,nq", [(256, 128, 20000, 200), (64, 64, 3001, 7),
                                      (512, 64, 4096, 130), (128, 128, 999, 128)])
def test_search_matches_oracle(m, d, N, nq):
    torch.cuda.set_device(0)
    k = 10
    S = jl.jl_sketch_init(m, d, 0)
    S64 = oracle.sketch(m, d, 0)
    signs, n16 = _index(N, d, m, 500 + m + N, S64)
    Q = workloads.random_keys(nq, d, 600 + m, scale=2.0)
    gi, gs = jl.jl_search_topk(Q.cuda(), S, torch.from_numpy(signs.view(np.int32)).cuda(),
                               torch.from_numpy(n16.view(np.float16)).cuda(), k)
    torch.cuda.synchronize()
    assert jl.jl_device_error() == 0
    _, _, allsc = oracle.search_topk(H.f64(Q), S64, signs, oracle.fp16_bits_to_f64(n16), k)
    _check(gi.cpu().numpy(), gs.cpu().numpy(), allsc, k)


@pytest.mark.parametrize("m,d,N,nq,k", [(256, 128, 50000, 40, 1), (256, 128, 50000, 40, 16),
                                        (512, 128, 9000, 3, 1), (512, 128, 9000, 3, 16)])
def test_search_k_extremes(m, d, N, nq, k):
    # k = 1 and the largest k, on both operand paths (U in shared memory for
    # m <= 256, in tensor memory for m = 512)
    torch.cuda.set_device(0)
    S = jl.jl_sketch_init(m, d, 0)
    S64 = oracle.sketch(m, d, 0)
    signs, n16 = _index(N, d, m, 800 + m + k, S64)
    Q = workloads.random_keys(nq, d, 900 + k, scale=2.0)
    gi, gs = jl.jl_search_topk(Q.cuda(), S, torch.from_numpy(signs.view(np.int32)).cuda(),
                               torch.from_numpy(n16.view(np.float16)).cuda(), k)
    torch.cuda.synchronize()
    assert jl.jl_device_error() == 0
    assert gi.shape == (nq, k)
    _, _, allsc = oracle.search_topk(H.f64(Q), S64, signs, oracle.fp16_bits_to_f64(n16), k)
    _check(gi.cpu().numpy(), gs.cpu().numpy(), allsc, k)


def test_search_fp32_queries_duplicates_and_small_index():
    torch.cuda.set_device(0)
    m, d = 256, 128
    S = jl.jl_sketch_init(m, d, 0)
    S64 = oracle.sketch(m, d, 0)
    N = 70000                                    # several CTAs' worth of tiles
    signs, n16 = _index(N, d, m, 77, S64)
    Q = workloads.random_keys(5, d, 78, dtype=torch.float32, scale=1.5)
    # plant a strong match for query 0 twice, far apart: a tie won by the lower index
    q0 = Q[0].double().numpy()
    s_dup, _, n_dup, _ = oracle.quantize(q0[None] * 3.0, S64)
    for pos in (123, 65001):
        signs[pos] = s_dup[0]
        n16[pos] = n_dup[0]
    gi, gs = jl.jl_search_topk(Q.cuda(), S, torch.from_numpy(signs.view(np.int32)).cuda(),
                               torch.from_numpy(n16.view(np.float16)).cuda(), 4)
    gi, gs = gi.cpu().numpy(), gs.cpu().numpy()
    assert gi[0][0] == 123 and gi[0][1] == 65001 and gs[0][0] == gs[0][1]
    _, _, allsc = oracle.search_topk(Q.double().numpy(), S64, signs,
                                     oracle.fp16_bits_to_f64(n16), 4)
    _check(gi, gs, allsc, 4)
    # fewer vectors than k: the tail is (-1, -inf)
    gi2, gs2 = jl.jl_search_topk(Q.cuda(), S, torch.from_numpy(signs[:3].view(np.int32)).cuda(),
                                 torch.from_numpy(n16[:3].view(np.float16)).cuda(), 8)
    _, _, allsc2 = oracle.search_topk(Q.double().numpy(), S64, signs[:3],
                                      oracle.fp16_bits_to_f64(n16[:3]), 8)
    _check(gi2.cpu().numpy(), gs2.cpu().numpy(), allsc2, 8)


def test_search_fullsize_sampled_queries():
    # the search workload's index size (8,388,608 vectors), two queries checked
    torch.cuda.set_device(0)
    m, d, N, nq, k = 256, 128, 8388608, 128, 10
    S = jl.jl_sketch_init(m, d, 0)
    g = torch.Generator(device="cuda")
    g.manual_seed(91)
    signs = torch.randint(-2 ** 31, 2 ** 31 - 1, (N, m // 32), dtype=torch.int32, device="cuda",
                          generator=g)
    norms = (torch.rand((N,), device="cuda", generator=g) * 2 + 0.5).half()
    Q = workloads.random_keys(nq, d, 92, device="cuda")
    gi, gs = jl.jl_search_topk(Q, S, signs, norms, k)
    torch.cuda.synchronize()
    assert jl.jl_device_error() == 0
    S64 = oracle.sketch(m, d, 0)
    sg = signs.cpu().numpy().view(np.uint32)
    n64 = oracle.fp16_bits_to_f64(norms.cpu().numpy().view(np.uint16))
    for q in (0, 127):
        _, _, allsc = oracle.search_topk(Q[q:q + 1].double().cpu().numpy(), S64, sg, n64, k)
        _check(gi[q:q + 1].cpu().numpy(), gs[q:q + 1].cpu().numpy(), allsc, k)


def test_search_with_warm_start_bound():
    # 409,600 vectors = 1600 tiles: large enough that the search first scores
    # a spread sample of tiles and starts the full pass from its bound
    torch.cuda.set_device(0)
    m, d, N, k = 256, 128, 409600, 16
    S = jl.jl_sketch_init(m, d, 0)
    S64 = oracle.sketch(m, d, 0)
    g = torch.Generator(device="cuda")
    g.manual_seed(93)
    signs = torch.randint(-2 ** 31, 2 ** 31 - 1, (N, m // 32), dtype=torch.int32, device="cuda",
                          generator=g)
    norms = (torch.rand((N,), device="cuda", generator=g) * 2 + 0.5).half()
    Q = workloads.random_keys(40, d, 94, device="cuda", scale=3.0)
    gi, gs = jl.jl_search_topk(Q, S, signs, norms, k)
    torch.cuda.synchronize()
    assert jl.jl_device_error() == 0
    sg = signs.cpu().numpy().view(np.uint32)
    n64 = oracle.fp16_bits_to_f64(norms.cpu().numpy().view(np.uint16))
    for q in (0, 13, 39):
        _, _, allsc = oracle.search_topk(Q[q:q + 1].double().cpu().numpy(), S64, sg, n64, k)
        _check(gi[q:q + 1].cpu().numpy(), gs[q:q + 1].cpu().numpy(), allsc, k)
