"""Context-split decode on the GPU against the oracle.

A context is cut into parts; each part is decoded to softmax states by
``jl_decode_attention_state`` and the states are merged by
``jl_merge_attention_states``.  Both sides take the oracle's codes and norms.
Checked per part: the part's output acc / l and its log-sum-exp mx + log2(l)
(the two quantities a state fixes) against ``oracle.decode_state``, and its
scores; after the merge: the output against the oracle's decode over the
whole context and against one ``jl_decode_attention`` call.  The parts run
one after another on one GPU; the exchange between ranks is tested on the
host (gloo) and, with one rank, through NCCL here.
"""
import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import bit_jl_key_b200 as jl
import oracle
import workloads
from bit_jl_key_b200 import context_parallel as cp
from tests import helpers as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    jl.load()
    torch.cuda.set_device(0)
    yield
    assert jl.jl_device_error() == 0


CASES = [
    # (B, Hq, Hkv, T, m, d, qdtype, q_scale, cut points)
    (1, 32, 32, 4096, 256, 128, torch.bfloat16, 1.0, (1000, 1001, 3000)),  # MHA, a 1-key part
    (2, 8, 2, 1000, 256, 128, torch.bfloat16, 1.0, (504,)),                 # GQA
    (1, 4, 1, 777, 512, 64, torch.bfloat16, 2.0, (13, 400)),                # int8 scoring
    (2, 8, 2, 1500, 256, 64, torch.float32, 2.0, (700,)),                   # keys as rows
    (1, 3, 3, 2048, 128, 128, torch.bfloat16, 4.0, (256, 512, 1024)),       # peaked softmax
]


def _inputs(B, Hq, Hkv, T, m, d, qdtype, q_scale, seed=17):
    kd = torch.float32 if qdtype == torch.float32 else torch.bfloat16
    K = workloads.random_keys(B * Hkv * T, d, seed, dtype=kd).reshape(B, Hkv, T, d)
    V = workloads.random_keys(B * Hkv * T, d, seed + 1).reshape(B, Hkv, T, d)
    Q = workloads.random_keys(B * Hq, d, seed + 2, dtype=qdtype,
                              scale=q_scale).reshape(B, Hq, d)
    S64 = oracle.sketch(m, d, 0)
    rsig, _, rn16, _ = oracle.quantize(H.f64(K.reshape(-1, d)), S64)
    signs = rsig.reshape(B, Hkv, T, m // 32)
    norms = oracle.fp16_bits_to_f64(rn16).reshape(B, Hkv, T)
    gsigns = torch.from_numpy(rsig.view(np.int32).reshape(B, Hkv, T, m // 32)).cuda()
    gnorms = torch.from_numpy(rn16.view(np.float16).reshape(B, Hkv, T)).cuda()
    return Q, V, S64, signs, norms, gsigns, gnorms


def _state_parts(states):
    """(acc / l, mx + log2 l) of GPU states [..., d + 2]."""
    st = H.f64(states)
    acc, mx, l = st[..., :-2], st[..., -2], st[..., -1]
    return acc / l[..., None], mx + np.log2(l)


@pytest.mark.parametrize("case", CASES)
def test_split_decode_matches_oracle(case):
    B, Hq, Hkv, T, m, d, qdtype, q_scale, cuts = case
    Q, V, S64, signs, norms, gsigns, gnorms = _inputs(B, Hq, Hkv, T, m, d, qdtype, q_scale)
    S = jl.jl_sketch_init(m, d, 0)
    Qg, Vg = Q.cuda(), V.cuda()
    scale = 1.0 / math.sqrt(d)
    edges = (0,) + tuple(cuts) + (T,)
    states = []
    for a, b in zip(edges[:-1], edges[1:]):
        # clone: a slice that is already contiguous (one KV head) would keep
        # its offset, and the library wants 16-byte aligned norms
        st, sc = jl.jl_decode_attention_state(Qg, S, gsigns[:, :, a:b].clone(),
                                              gnorms[:, :, a:b].clone(),
                                              Vg[:, :, a:b].clone(), scale,
                                              want_scores=True)
        ref_o, ref_lse = oracle.decode_state(H.f64(Q), S64, signs[:, :, a:b], norms[:, :, a:b],
                                             H.f64(V)[:, :, a:b], scale)
        _, ref_sc = oracle.decode(H.f64(Q), S64, signs[:, :, a:b], norms[:, :, a:b],
                                  H.f64(V)[:, :, a:b], scale, want_scores=True)
        o, lse = _state_parts(st)
        assert H.score_violations(H.f64(sc), ref_sc) == 0
        assert np.max(np.abs(o - ref_o)) <= H.OUT_ABS
        # a score error of 1e-3 of the score scale moves lse2 by about that
        # much times softmax_scale * log2(e)
        lse_tol = 2e-3 * np.maximum(1.0, np.abs(ref_lse))
        assert np.all(np.abs(lse - ref_lse) <= lse_tol), np.max(np.abs(lse - ref_lse))
        states.append(st)
    merged = jl.jl_merge_attention_states(torch.stack(states))
    whole_ref, _ = oracle.decode(H.f64(Q), S64, signs, norms, H.f64(V), scale)
    mabs, rel = H.output_errors(H.f64(merged), whole_ref)
    print(f"split decode {case[:6]} parts={len(states)}: max|dout|={mabs:.3e} rel={rel:.3e}")
    assert mabs <= H.OUT_ABS and rel <= 1e-2
    whole = jl.jl_decode_attention(Qg, S, gsigns, gnorms, Vg, scale)
    assert np.max(np.abs(H.f64(merged) - H.f64(whole))) <= 1e-2


def test_one_part_state_reproduces_decode():
    B, Hq, Hkv, T, m, d = 2, 8, 2, 1000, 256, 128
    Q, V, _, _, _, gsigns, gnorms = _inputs(B, Hq, Hkv, T, m, d, torch.bfloat16, 1.0)
    S = jl.jl_sketch_init(m, d, 0)
    st = jl.jl_decode_attention_state(Q.cuda(), S, gsigns, gnorms, V.cuda())
    out = jl.jl_decode_attention(Q.cuda(), S, gsigns, gnorms, V.cuda())
    merged = jl.jl_merge_attention_states(st[None])
    # acc / l against acc * (1 / l): at most one bf16 step apart
    diff = np.abs(H.f64(merged) - H.f64(out))
    assert np.max(diff) <= 2.0 ** -7 * max(1.0, float(np.max(np.abs(H.f64(out)))))


def test_merge_ignores_empty_parts_and_zeroes_empty_rows():
    rows, d = 6, 64
    g = torch.Generator().manual_seed(5)
    acc = torch.randn((2, rows, d), generator=g)
    mx = torch.randn((2, rows), generator=g) * 4
    l = torch.rand((2, rows), generator=g) + 0.5
    parts = torch.cat([acc, mx[..., None], l[..., None]], dim=-1).cuda()
    empty = torch.zeros((1, rows, d + 2))
    empty[..., d] = -math.inf
    ref = jl.jl_merge_attention_states(parts)
    with_empty = jl.jl_merge_attention_states(torch.cat([empty.cuda(), parts, empty.cuda()]))
    assert torch.equal(ref, with_empty)
    # the merge itself against the plain formula in float64
    a, m_, l_ = (x.double() for x in (acc, mx, l))
    top = m_.max(dim=0).values
    w = torch.exp2(m_ - top)
    want = (w[..., None] * a).sum(0) / (w * l_).sum(0)[..., None]
    np.testing.assert_allclose(H.f64(ref), want.numpy(), atol=2e-2, rtol=1e-2)
    assert torch.count_nonzero(jl.jl_merge_attention_states(empty.repeat(3, 1, 1).cuda())) == 0


def test_merge_rejects_bad_arguments():
    with pytest.raises(jl.JLError):
        jl.jl_merge_attention_states(torch.zeros((2, 4, 98), device="cuda"))    # d = 96
    with pytest.raises(jl.JLError):
        jl.jl_merge_attention_states(torch.zeros((0, 4, 130), device="cuda"))   # no part
    with pytest.raises(ValueError):
        jl.jl_merge_attention_states(torch.zeros((2, 4, 130), device="cuda",
                                                 dtype=torch.float64))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_decode_context_parallel_one_rank_nccl():
    B, Hq, Hkv, T, m, d = 1, 8, 8, 512, 256, 128
    Q, V, S64, signs, norms, gsigns, gnorms = _inputs(B, Hq, Hkv, T, m, d, torch.bfloat16, 1.0)
    S = jl.jl_sketch_init(m, d, 0)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(_free_port())
    dist.init_process_group("nccl", rank=0, world_size=1,
                            device_id=torch.device("cuda", 0))
    try:
        t0, t1 = cp.context_range(T, 1, 0)
        out = cp.decode_context_parallel(Q.cuda(), S, gsigns[:, :, t0:t1].clone(),
                                         gnorms[:, :, t0:t1].clone(),
                                         V.cuda()[:, :, t0:t1].clone())
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    ref, _ = oracle.decode(H.f64(Q), S64, signs, norms, H.f64(V), 1.0 / math.sqrt(d))
    mabs, _ = H.output_errors(H.f64(out), ref)
    assert mabs <= H.OUT_ABS
