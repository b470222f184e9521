"""Paged, ragged decode over TurboQuant-prod keys, with the new key appended.

As the QJL paged test: a shuffled pool of fixed-size pages whose unused slots
hold garbage (random code words, random norms, NaN values).  The oracle
quantizes every key (the cache and the appended one) itself, and decodes each
sequence over its own keys; the GPU result comes through
jl_turbo_decode_attention_paged.  The appended key, quantized on the GPU by
fp32 SIMT products, is checked against the oracle with the band rules of the
quantizer tests.
"""
import numpy as np
import pytest
import torch

import bit_jl_key_b200 as jl
import oracle
import workloads
from oracle import turbo as tq
from tests import helpers as H

pytestmark = pytest.mark.gpu

D = M = 128
BAND_Y = 2e-6
BAND_SIGN = 1e-5


def _bf16_tensor(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def _codes(ref, bits):
    return np.concatenate([tq.pack_planes(ref["cell"], bits), ref["signs"]], axis=1)


@pytest.mark.parametrize("cfg", [
    # B, Hq, Hkv, P, lens, append, bits, query and new-key dtype, d = m
    (4, 8, 2, 32, [0, 31, 100, 257], True, 2, torch.bfloat16, 128),
    (3, 4, 4, 64, [1, 64, 130], True, 3, torch.bfloat16, 128),
    (2, 16, 1, 128, [500, 33], True, 1, torch.bfloat16, 128),
    (3, 8, 2, 32, [40, 0, 96], False, 2, torch.bfloat16, 128),
    (3, 8, 2, 64, [70, 1, 200], True, 2, torch.float32, 128),
    (4, 8, 2, 32, [0, 31, 100, 257], True, 2, torch.bfloat16, 64),
    (3, 4, 4, 64, [1, 64, 130], True, 3, torch.bfloat16, 64),
    (2, 16, 1, 64, [500, 33], True, 1, torch.float32, 64),
])
def test_turbo_paged_append_decode_matches_oracle(cfg):
    torch.cuda.set_device(0)
    B, Hq, Hkv, P, lens, append, bits, dt, D = cfg
    M = D
    rng = np.random.default_rng(B * 100 + P + bits)
    max_len = max(lens) + 1 + 7
    c = tq.lloyd_max(D, bits)
    pit_bits = tq.rotation_bf16_bits(D, 1)
    Pit = oracle.bf16_bits_to_f64(pit_bits)
    S64 = oracle.sketch(M, D, 0)
    S = jl.jl_sketch_init(M, D, 0)
    Pi = _bf16_tensor(pit_bits)
    Pinv = torch.from_numpy(np.linalg.inv(Pit).astype(np.float32)).cuda()
    words = jl.turbo_code_words(bits, M, D)
    pages_per_seq = [max(1, -(-(L + 1) // P)) for L in lens]
    max_pages = -(-max_len // P)
    num_pages = sum(pages_per_seq) + 3
    perm = rng.permutation(num_pages)
    table = np.full((B, max_pages), -1, dtype=np.int32)
    k = 0
    for b in range(B):
        table[b, :pages_per_seq[b]] = perm[k:k + pages_per_seq[b]]
        k += pages_per_seq[b]
    code_pool = rng.integers(-2 ** 31, 2 ** 31 - 1, size=(num_pages, Hkv, P, words),
                             dtype=np.int64).astype(np.int32)
    norm_pool = rng.uniform(0, 5, size=(num_pages, Hkv, P, 2)).astype(np.float16)
    val_pool = np.full((num_pages, Hkv, P, D), np.nan, dtype=np.float32)
    keys, vals = [], []
    for b in range(B):
        K = workloads.random_keys(Hkv * lens[b], D, 300 + b).reshape(Hkv, lens[b], D)
        V = workloads.random_keys(Hkv * lens[b], D, 400 + b).reshape(Hkv, lens[b], D)
        keys.append(K)
        vals.append(V)
        for h in range(Hkv):
            if lens[b] == 0:
                continue
            ref = tq.quantize(H.f64(K[h]), Pit, c, S64)
            cw = _codes(ref, bits)
            for t in range(lens[b]):
                pg, sl = table[b, t // P], t % P
                code_pool[pg, h, sl] = cw[t].view(np.int32)
                norm_pool[pg, h, sl, 0] = ref["norm16"][t:t + 1].view(np.float16)[0]
                norm_pool[pg, h, sl, 1] = ref["rnorm16"][t:t + 1].view(np.float16)[0]
                val_pool[pg, h, sl] = H.f64(V[h, t])
    cp = torch.from_numpy(code_pool).cuda()
    npg = torch.from_numpy(norm_pool).cuda()
    vp = torch.from_numpy(val_pool).to(torch.bfloat16).cuda()
    Q = workloads.random_keys(B * Hq, D, 55, dtype=dt, scale=2.0).reshape(B, Hq, D)
    Kn = workloads.random_keys(B * Hkv, D, 56, dtype=dt).reshape(B, Hkv, D)
    Vn = workloads.random_keys(B * Hkv, D, 57).reshape(B, Hkv, D)
    seq = torch.tensor(lens, dtype=torch.int32, device="cuda")
    out, sc = jl.jl_turbo_decode_attention_paged(
        Q.cuda(), Pinv, S, cp, npg, vp, torch.from_numpy(table).cuda(), seq, max_len, bits,
        Pi=Pi if append else None, K_new=Kn.cuda() if append else None,
        V_new=Vn.cuda() if append else None, want_scores=True)
    torch.cuda.synchronize()
    assert jl.jl_device_error() == 0
    cp_h = H.u32(cp)
    np_h = H.fp16_bits(npg)
    vp_h = vp.cpu()
    scale = 1.0 / np.sqrt(D)
    G = Hq // Hkv
    for b in range(B):
        T = lens[b] + (1 if append else 0)
        K, V = keys[b], vals[b]
        same = True
        if append:
            K = torch.cat([K.to(Kn.dtype), Kn[b][:, None, :]], dim=1)
            V = torch.cat([V, Vn[b][:, None, :]], dim=1)
            # the appended key: cells and signs within the bands, norms 1 step,
            # value bitwise
            pg, sl = table[b, lens[b] // P], lens[b] % P
            ref = tq.quantize(H.f64(Kn[b]), Pit, c, S64, band_abs=BAND_Y, band_rel=BAND_SIGN)
            gw = cp_h[pg, :, sl]
            gcell = tq.unpack_planes(gw[:, :bits * D // 32], D, bits)
            cdiff = gcell != ref["cell"]
            assert not np.any(cdiff & ~ref["cell_band"]), b
            ok = ~cdiff.any(axis=1)
            sdiff = (H.code_bits(gw[:, bits * D // 32:], M) != H.code_bits(ref["signs"], M))
            sdiff &= ok[:, None]
            assert not np.any(sdiff & ~(np.abs(ref["proj"]) < ref["sign_allow"])), b
            gn = np_h[pg, :, sl]
            assert H.fp16_ulp_diff(gn[:, 0], ref["norm16"]).max() <= 1
            assert H.fp16_ulp_diff(gn[:, 1], ref["rnorm16"])[ok].max(initial=0) <= 1
            assert torch.equal(vp_h[pg, :, sl], Vn[b])
            same = (np.array_equal(gw, _codes(ref, bits)) and
                    np.array_equal(gn[:, 0], ref["norm16"]) and
                    np.array_equal(gn[:, 1], ref["rnorm16"]))
        if T == 0:
            assert torch.count_nonzero(out[b]) == 0
            continue
        for h in range(Hkv):
            ref = tq.quantize(H.f64(K[h]), Pit, c, S64)
            hqs = list(range(h * G, (h + 1) * G))
            ref_out, ref_sc = tq.decode(
                H.f64(Q[b, hqs])[None], Pit, S64, c, ref["cell"][None, None],
                ref["signs"][None, None], oracle.fp16_bits_to_f64(ref["norm16"])[None, None],
                oracle.fp16_bits_to_f64(ref["rnorm16"])[None, None], H.f64(V[h])[None, None],
                scale, want_scores=True)
            upto = T if same else T - 1
            g_sc = H.f64(sc[b, hqs, :T])[None]
            assert H.score_violations(g_sc[..., :upto], ref_sc[..., :upto]) == 0, (b, h)
            mabs, rel = H.output_errors(H.f64(out[b, hqs])[None], ref_out)
            assert mabs <= H.OUT_ABS and rel <= 1e-2, (b, h, mabs, rel)


def test_turbo_paged_bad_length_is_reported():
    # a sequence length past the bound: device error 3, clipped, and the next
    # call runs clean
    torch.cuda.set_device(0)
    bits, B, Hq, Hkv, P = 2, 2, 4, 2, 32
    max_len = 64
    words = jl.turbo_code_words(bits, M, D)
    cp = torch.zeros((4, Hkv, P, words), dtype=torch.int32, device="cuda")
    npg = torch.zeros((4, Hkv, P, 2), dtype=torch.float16, device="cuda")
    vp = torch.zeros((4, Hkv, P, D), dtype=torch.bfloat16, device="cuda")
    tab = torch.tensor([[0, 1], [2, 3]], dtype=torch.int32, device="cuda")
    Pi, Pinv = jl.jl_turbo_rotation_init(D, 1)
    S = jl.jl_sketch_init(M, D, 0)
    Q = workloads.random_keys(B * Hq, D, 5, device="cuda").reshape(B, Hq, D)
    bad = torch.tensor([10, 500], dtype=torch.int32, device="cuda")
    jl.jl_turbo_decode_attention_paged(Q, Pinv, S, cp, npg, vp, tab, bad, max_len, bits)
    assert jl.jl_device_error() == 3
    assert jl.jl_device_error() == 0
    good = torch.tensor([10, 20], dtype=torch.int32, device="cuda")
    jl.jl_turbo_decode_attention_paged(Q, Pinv, S, cp, npg, vp, tab, good, max_len, bits)
    assert jl.jl_device_error() == 0
