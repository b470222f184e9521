"""Paged, ragged decode with the new key appended in the same step.

A batch of sequences of different lengths keeps its compressed cache in a
shuffled pool of fixed-size pages; unused slots hold garbage (random codes,
NaN values) that must never reach a result.  The oracle quantizes every key
(including the appended one) itself and decodes each sequence over its own
gathered keys; the GPU result comes through jl_decode_attention_paged.
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


def _setup(B, Hq, Hkv, d, m, P, lens, max_len, seed, garbage=True):
    rng = np.random.default_rng(seed)
    W = m // 32
    pages_per_seq = [max(1, -(-(L + 1) // P)) for L in lens]
    max_pages = -(-max_len // P)
    num_pages = sum(pages_per_seq) + 3
    perm = rng.permutation(num_pages)
    table = np.full((B, max_pages), -1, dtype=np.int32)
    k = 0
    for b in range(B):
        table[b, :pages_per_seq[b]] = perm[k:k + pages_per_seq[b]]
        k += pages_per_seq[b]
    S = jl.jl_sketch_init(m, d, 0)
    S64 = oracle.sketch(m, d, 0)
    # pools full of garbage: random code words, random norms, NaN values
    sign_pool = rng.integers(-2 ** 31, 2 ** 31 - 1, size=(num_pages, Hkv, P, W), dtype=np.int64).astype(np.int32)
    norm_pool = rng.uniform(0, 5, size=(num_pages, Hkv, P)).astype(np.float16)
    val_pool = np.full((num_pages, Hkv, P, d), np.nan if garbage else 0.0, dtype=np.float32)
    keys, vals = [], []
    for b in range(B):
        K = workloads.random_keys(Hkv * lens[b], d, seed + 10 + b).reshape(Hkv, lens[b], d)
        V = workloads.random_keys(Hkv * lens[b], d, seed + 100 + b).reshape(Hkv, lens[b], d)
        keys.append(K)
        vals.append(V)
        for h in range(Hkv):
            if lens[b] == 0:
                continue
            sig, _, n16, _ = oracle.quantize(H.f64(K[h]), S64)
            for t in range(lens[b]):
                pg, sl = table[b, t // P], t % P
                sign_pool[pg, h, sl] = sig[t].view(np.int32)
                norm_pool[pg, h, sl] = n16[t:t + 1].view(np.float16)[0]
                val_pool[pg, h, sl] = H.f64(V[h, t])
    dev = "cuda"
    pools = (torch.from_numpy(sign_pool).to(dev), torch.from_numpy(norm_pool).to(dev),
             torch.from_numpy(val_pool).to(torch.bfloat16).to(dev))
    return S, S64, table, pools, keys, vals


@pytest.mark.parametrize("cfg", [
    # B, Hq, Hkv, d, m, P, lens, append, query and new-key dtype
    (4, 8, 2, 128, 256, 32, [0, 31, 100, 257], True, torch.bfloat16),  # GQA, page = 1 block
    (3, 4, 4, 64, 128, 64, [1, 64, 130], True, torch.bfloat16),        # MHA (int8), 2 blocks/page
    (2, 16, 1, 128, 256, 128, [500, 33], True, torch.bfloat16),        # two head groups
    (3, 2, 2, 128, 512, 32, [40, 0, 96], False, torch.bfloat16),       # no append, one empty
    (3, 8, 2, 128, 256, 64, [70, 1, 200], True, torch.float32),        # fp32 query and new key
    (2, 2, 2, 64, 256, 32, [95, 31], True, torch.bfloat16),            # MHA, m = 4d: keys as MMA rows
    (3, 8, 2, 64, 256, 64, [300, 0, 77], True, torch.bfloat16),        # GQA, keys as MMA rows
    (2, 8, 4, 128, 512, 32, [129, 64], True, torch.float32),           # 2 heads/KV head, m = 4d
])
def test_paged_append_decode_matches_oracle(cfg):
    torch.cuda.set_device(0)
    B, Hq, Hkv, d, m, P, lens, append, dt = cfg
    max_len = max(lens) + 1 + 7
    S, S64, table, (sp, npg, vp), keys, vals = _setup(B, Hq, Hkv, d, m, P, lens, max_len, 7)
    Q = workloads.random_keys(B * Hq, d, 55, dtype=dt, scale=2.0).reshape(B, Hq, d)
    Kn = workloads.random_keys(B * Hkv, d, 56, dtype=dt).reshape(B, Hkv, d)
    Vn = workloads.random_keys(B * Hkv, d, 57).reshape(B, Hkv, d)
    seq = torch.tensor(lens, dtype=torch.int32, device="cuda")
    out, sc = jl.jl_decode_attention_paged(
        Q.cuda(), S, sp, npg, vp, torch.from_numpy(table).cuda(), seq, max_len,
        K_new=Kn.cuda() if append else None, V_new=Vn.cuda() if append else None,
        want_scores=True)
    torch.cuda.synchronize()
    assert jl.jl_device_error() == 0
    sp_h, np_h, vp_h = H.u32(sp), H.fp16_bits(npg), vp.cpu()
    scale = 1.0 / math.sqrt(d)
    for b in range(B):
        T = lens[b] + (1 if append else 0)
        K = keys[b]
        V = vals[b]
        if append:
            K = torch.cat([K.to(Kn.dtype), Kn[b][:, None, :]], dim=1)
            V = torch.cat([V, Vn[b][:, None, :]], dim=1)
            # the appended key: code (band rule), norm (1 ulp), value (bitwise)
            pg, sl = table[b, lens[b] // P], lens[b] % P
            rsig, _, rn16, band = oracle.quantize(H.f64(Kn[b]), S64, band_rel=H.BAND_REL,
                                                  want_band=True)
            out_band, _ = H.compare_codes(sp_h[pg, :, sl], rsig, band, m)
            assert out_band == 0
            assert H.fp16_ulp_diff(np_h[pg, :, sl], rn16).max() <= 1
            assert torch.equal(vp_h[pg, :, sl], Vn[b])
        if T == 0:
            assert torch.count_nonzero(out[b]) == 0
            continue
        # the oracle decodes its own codes of the sequence's keys (the pool's
        # cache part holds exactly those; the GPU's appended code was checked
        # above against the oracle's within the band)
        pos = np.arange(T)
        pg, sl = table[b, pos // P], pos % P
        ref = [oracle.quantize(H.f64(K[h]), S64) for h in range(Hkv)]
        sig = np.stack([r[0] for r in ref])
        n16 = np.stack([r[2] for r in ref])
        if lens[b]:
            pool_sig = np.stack([sp_h[pg, h, sl] for h in range(Hkv)])
            assert np.array_equal(pool_sig[:, :lens[b]], sig[:, :lens[b]])
        ref_out, ref_sc = oracle.decode(H.f64(Q[b])[None], S64, sig[None],
                                        oracle.fp16_bits_to_f64(n16)[None], H.f64(V)[None],
                                        scale, want_scores=True)
        g_sc = H.f64(sc[b, :, :T])[None]
        # the appended key's score only when its GPU code and norm equal the
        # oracle's (an in-band flip or a 1-ulp norm moves that one score)
        same = True
        if append:
            pa, sa = table[b, lens[b] // P], lens[b] % P
            same = (np.array_equal(sp_h[pa, :, sa], sig[:, -1])
                    and np.array_equal(np_h[pa, :, sa], n16[:, -1]))
        upto = T if same else T - 1
        assert H.score_violations(g_sc[..., :upto], ref_sc[..., :upto]) == 0, b
        mabs, rel = H.output_errors(H.f64(out[b])[None], ref_out)
        assert mabs <= H.OUT_ABS and rel <= 1e-2, (b, mabs, rel)


def test_paged_equals_contiguous_decode():
    # one page per sequence holding the whole context: the paged call must give
    # what jl_decode_attention gives on the same contiguous cache
    torch.cuda.set_device(0)
    B, Hq, Hkv, T, m, d = 2, 8, 2, 1024, 256, 128
    S = jl.jl_sketch_init(m, d, 0)
    K = workloads.random_keys(B * Hkv * T, d, 3).cuda()
    V = workloads.random_keys(B * Hkv * T, d, 4).reshape(B, Hkv, T, d).cuda()
    Q = workloads.random_keys(B * Hq, d, 5).reshape(B, Hq, d).cuda()
    signs, norms = jl.jl_quantize_keys(K, S)
    signs = signs.reshape(B, Hkv, T, m // 32)
    norms = norms.reshape(B, Hkv, T)
    ref = jl.jl_decode_attention(Q, S, signs, norms, V)
    table = torch.arange(B, dtype=torch.int32, device="cuda").reshape(B, 1)
    seq = torch.full((B,), T, dtype=torch.int32, device="cuda")
    out = jl.jl_decode_attention_paged(Q, S, signs.contiguous(), norms.contiguous(),
                                       V.contiguous(), table, seq, T)
    mabs, rel = H.output_errors(H.f64(out), H.f64(ref))
    assert mabs <= 1e-2 and rel <= 1e-2


def test_paged_length_past_bound_reports_error_and_recovers():
    # a length at the bound with a key to append cannot fit: the kernels clip
    # the sequence, skip the write and record an error; the next valid call
    # is unaffected
    torch.cuda.set_device(0)
    B, Hq, Hkv, d, m, P = 2, 4, 2, 128, 256, 32
    lens = [64, 10]
    max_len = 65
    S, S64, table, (sp, npg, vp), keys, vals = _setup(B, Hq, Hkv, d, m, P, lens, max_len, 11,
                                                      garbage=False)
    Q = workloads.random_keys(B * Hq, d, 60).reshape(B, Hq, d).cuda()
    Kn = workloads.random_keys(B * Hkv, d, 61).reshape(B, Hkv, d).cuda()
    Vn = workloads.random_keys(B * Hkv, d, 62).reshape(B, Hkv, d).cuda()
    tab = torch.from_numpy(table).cuda()
    assert jl.jl_device_error() == 0
    bad = torch.tensor([65, 10], dtype=torch.int32, device="cuda")
    jl.jl_decode_attention_paged(Q, S, sp, npg, vp, tab, bad, max_len, K_new=Kn, V_new=Vn)
    assert jl.jl_device_error() == 3          # inconsistent work split / bound
    assert jl.jl_device_error() == 0          # reading clears it
    good = torch.tensor(lens, dtype=torch.int32, device="cuda")
    out = jl.jl_decode_attention_paged(Q, S, sp, npg, vp, tab, good, max_len)
    torch.cuda.synchronize()
    assert jl.jl_device_error() == 0
    scale = 1.0 / math.sqrt(d)
    for b in range(B):
        sig = np.stack([oracle.quantize(H.f64(keys[b][h]), S64)[0] for h in range(Hkv)])
        n16 = np.stack([oracle.quantize(H.f64(keys[b][h]), S64)[2] for h in range(Hkv)])
        ref_out, _ = oracle.decode(H.f64(Q[b].cpu())[None], S64, sig[None],
                                   oracle.fp16_bits_to_f64(n16)[None], H.f64(vals[b])[None], scale)
        mabs, rel = H.output_errors(H.f64(out[b])[None], ref_out)
        assert mabs <= H.OUT_ABS and rel <= 1e-2, (b, mabs, rel)
