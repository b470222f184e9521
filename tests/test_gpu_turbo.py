"""TurboQuant-prod keys on the GPU against the float64 oracle (oracle/turbo.py).

Tolerances, from the arithmetic of the two sides:
  * rotation: bf16 Pi bit-exact, except an element whose float64 value lies
    within 1e-12 of a bf16 rounding midpoint (both sides orthogonalise in
    float64, by different algorithms); Pinv within 1e-6 (fp32 rounding of a
    float64 inverse).
  * codebook: the library's float centroids equal the oracle's rounded to
    float.
  * cells: exact, except a coordinate whose float64 y lies within BAND_Y of a
    boundary (the GPU forms y in fp32 from exact bf16 products, then scales).
  * residual signs, for keys whose cells all agree: exact, except a sign
    whose float64 projection is below the oracle's allowance: 1e-5 ||rt||
    plus |S_ij| ulp(r_j) for every residual coordinate within BAND_Y of a
    bf16 rounding midpoint.
  * norms: ||k||, and ||r|| for keys whose cells agree, within 1 binary16
    step (fp32 against float64 sums before the rounding).
  * decode (the oracle's codes fed to both sides): scores within
    1e-3 max(|ref|, rms of the row); outputs within 2e-2.
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


def _setup(bits, rot_seed=1, sk_seed=0, d=D):
    c = tq.lloyd_max(d, bits)
    pit_bits = tq.rotation_bf16_bits(d, rot_seed)
    Pit = oracle.bf16_bits_to_f64(pit_bits)
    s_bits = oracle.sketch_bf16_bits(d, d, sk_seed)
    S64 = oracle.bf16_bits_to_f64(s_bits)
    return c, pit_bits, Pit, s_bits, S64


@pytest.mark.parametrize("d,seed", [(64, 3), (128, 1), (128, 77)])
def test_rotation_matches_oracle(d, seed):
    torch.cuda.set_device(0)
    Pi, Pinv = jl.jl_turbo_rotation_init(d, seed)
    torch.cuda.synchronize()
    g = Pi.view(torch.int16).cpu().numpy().view(np.uint16)
    r = tq.rotation_bf16_bits(d, seed)
    P = tq.rotation(d, seed)
    Pr = oracle.bf16_bits_to_f64(r)
    ulp = np.abs(P - Pr)
    a = np.abs(P)
    half = 2.0 ** (np.floor(np.log2(np.where(a > 0, a, 1.0))) - 8)
    amb = np.abs(ulp - half) < 1e-12
    diff = g != r
    assert not np.any(diff & ~amb), int(np.count_nonzero(diff & ~amb))
    inv = np.linalg.inv(oracle.bf16_bits_to_f64(g))
    err = np.abs(H.f64(Pinv) - inv).max()
    assert err < 1e-6, err
    print(f"rotation d={d} seed={seed}: {int(diff.sum())} midpoint flips, Pinv err {err:.2e}")


@pytest.mark.parametrize("bits", [1, 2, 3])
def test_codebook_matches_oracle(bits):
    for d in (64, 128):
        g = np.array(jl.jl_turbo_codebook(d, bits), dtype=np.float32)
        assert np.array_equal(g, tq.lloyd_max(d, bits).astype(np.float32))


def _quantize_case(bits, K, rot_seed=1):
    d = m = K.shape[1]
    c, pit_bits, Pit, s_bits, S64 = _setup(bits, rot_seed, d=d)
    n = K.shape[0]
    codes, norms = jl.jl_turbo_quantize_keys(K.cuda(), _bf16_tensor(pit_bits), _bf16_tensor(s_bits),
                                             bits)
    torch.cuda.synchronize()
    assert jl.jl_device_error() == 0
    ref = tq.quantize(H.f64(K), Pit, c, S64, band_abs=BAND_Y, band_rel=BAND_SIGN)
    gw = H.u32(codes).reshape(n, -1)
    pw = bits * d // 32
    gcell = tq.unpack_planes(gw[:, :pw], d, bits)
    cdiff = gcell != ref["cell"]
    assert not np.any(cdiff & ~ref["cell_band"]), int(np.count_nonzero(cdiff & ~ref["cell_band"]))
    ok = ~cdiff.any(axis=1)
    gz = H.code_bits(gw[:, pw:], m)
    rz = H.code_bits(ref["signs"], m)
    sdiff = (gz != rz) & ok[:, None]
    allowed = np.abs(ref["proj"]) < ref["sign_allow"]
    assert not np.any(sdiff & ~allowed), int(np.count_nonzero(sdiff & ~allowed))
    gn = H.fp16_bits(norms).reshape(n, 2)
    assert H.fp16_ulp_diff(gn[:, 0], ref["norm16"]).max() <= 1
    assert H.fp16_ulp_diff(gn[:, 1], ref["rnorm16"])[ok].max(initial=0) <= 1
    return int(cdiff.sum()), int(sdiff.sum()), int((~ok).sum())


@pytest.mark.parametrize("d", [128, 64])
@pytest.mark.parametrize("bits", [1, 2, 3])
@pytest.mark.parametrize("n", [1, 300, 4099])
def test_quantize_matches_oracle(bits, n, d):
    torch.cuda.set_device(0)
    K = workloads.random_keys(n, d, 900 + n + bits + d, scale=1.3)
    cf, sf, kf = _quantize_case(bits, K)
    print(f"turbo quantize d={d} bits={bits} n={n}: {cf} in-band cells, {sf} allowed sign "
          f"flips, {kf} keys skipped for the residual check")


@pytest.mark.parametrize("d", [128, 64])
def test_quantize_edge_keys(d):
    # a zero key (norm 0, y = 0: every coordinate in the cell just below 0),
    # huge and tiny keys, outlier channels
    torch.cuda.set_device(0)
    K = workloads.random_keys(256, d, 31)
    K[0] = 0
    K[1] *= 3000
    K[2] *= 1e-3
    K[3, :4] *= 50
    for bits in (1, 2, 3):
        _quantize_case(bits, K)


def test_quantize_gqa_keys_sampled():
    # keys of the turbo-gqa cache (outlier channels), a 64K-key slice
    torch.cuda.set_device(0)
    w = workloads.TURBO_GQA.with_(B=1, Hkv=2)
    K = workloads.keys(w).reshape(-1, D)[:65536]
    cf, sf, kf = _quantize_case(workloads.TURBO_MSE_BITS, K, workloads.TURBO_ROTATION_SEED)
    print(f"turbo-gqa keys: {cf} in-band cells, {sf} allowed sign flips, {kf} keys skipped")


def _decode_inputs(bits, B, Hq, Hkv, T, seed, qdtype=torch.bfloat16, d=D):
    c, pit_bits, Pit, s_bits, S64 = _setup(bits, d=d)
    K = workloads.random_keys(B * Hkv * T, d, seed, scale=1.0)
    V = workloads.random_keys(B * Hkv * T, d, seed + 1).reshape(B, Hkv, T, d)
    Q = workloads.random_keys(B * Hq, d, seed + 2, dtype=qdtype).reshape(B, Hq, d)
    ref = tq.quantize(H.f64(K), Pit, c, S64)
    planes = tq.pack_planes(ref["cell"], bits)
    codes = np.concatenate([planes, ref["signs"]], axis=1).reshape(B, Hkv, T, -1)
    norms = np.stack([ref["norm16"], ref["rnorm16"]], axis=1).reshape(B, Hkv, T, 2)
    nk = oracle.fp16_bits_to_f64(ref["norm16"]).reshape(B, Hkv, T)
    nr = oracle.fp16_bits_to_f64(ref["rnorm16"]).reshape(B, Hkv, T)
    want = tq.decode(H.f64(Q), Pit, S64, c, ref["cell"].reshape(B, Hkv, T, d),
                     ref["signs"].reshape(B, Hkv, T, -1), nk, nr, H.f64(V), 1 / np.sqrt(d),
                     want_scores=True)
    gpu_in = dict(Q=Q.cuda(),
                  Pinv=torch.from_numpy(np.linalg.inv(Pit).astype(np.float32)).cuda(),
                  S=_bf16_tensor(s_bits),
                  codes=torch.from_numpy(np.ascontiguousarray(codes).view(np.int32)).cuda(),
                  norms=torch.from_numpy(np.ascontiguousarray(norms).view(np.float16)).cuda(),
                  V=V.cuda())
    return gpu_in, want


@pytest.mark.parametrize("bits", [1, 2, 3])
@pytest.mark.parametrize("B,Hq,Hkv,T,d", [(2, 8, 2, 300, 128), (1, 4, 4, 1, 128),
                                          (2, 32, 8, 4096, 128), (1, 8, 1, 1001, 128),
                                          (2, 8, 2, 300, 64), (1, 4, 4, 1, 64),
                                          (2, 16, 4, 2048, 64), (1, 8, 1, 1001, 64),
                                          # three heads per KV head (keys as MMA rows)
                                          (2, 6, 2, 777, 128), (1, 9, 3, 1500, 64)])
def test_decode_matches_oracle(bits, B, Hq, Hkv, T, d):
    torch.cuda.set_device(0)
    gi, (ref_out, ref_sc) = _decode_inputs(bits, B, Hq, Hkv, T, 4000 + T + B + d, d=d)
    out, sc = jl.jl_turbo_decode_attention(gi["Q"], gi["Pinv"], gi["S"], gi["codes"], gi["norms"],
                                           gi["V"], bits, want_scores=True)
    torch.cuda.synchronize()
    assert jl.jl_device_error() == 0
    assert H.score_violations(H.f64(sc), ref_sc) == 0
    mabs, rel = H.output_errors(H.f64(out), ref_out)
    assert mabs <= H.OUT_ABS, mabs
    print(f"turbo decode d={d} bits={bits} {B}x{Hq}/{Hkv}x{T}: out err {mabs:.2e} "
          f"(rel {rel:.2e})")


@pytest.mark.parametrize("d", [128, 64])
def test_decode_fp32_queries(d):
    torch.cuda.set_device(0)
    gi, (ref_out, ref_sc) = _decode_inputs(2, 1, 8, 2, 640, 77 + d, qdtype=torch.float32, d=d)
    out, sc = jl.jl_turbo_decode_attention(gi["Q"], gi["Pinv"], gi["S"], gi["codes"], gi["norms"],
                                           gi["V"], 2, want_scores=True)
    torch.cuda.synchronize()
    assert H.score_violations(H.f64(sc), ref_sc) == 0
    assert H.output_errors(H.f64(out), ref_out)[0] <= H.OUT_ABS


@pytest.mark.parametrize("d", [128, 64])
def test_end_to_end_library_rotation_and_codes(d):
    # rotation, quantization and decode all from the library; the oracle
    # decodes its own codes of the same keys
    torch.cuda.set_device(0)
    bits, B, Hq, Hkv, T = 2, 2, 8, 2, 2048
    c, pit_bits, Pit, s_bits, S64 = _setup(bits, rot_seed=5, d=d)
    Pi, Pinv = jl.jl_turbo_rotation_init(d, 5)
    S = jl.jl_sketch_init(d, d, 0)
    K = workloads.random_keys(B * Hkv * T, d, 123)
    V = workloads.random_keys(B * Hkv * T, d, 124).reshape(B, Hkv, T, d)
    Q = workloads.random_keys(B * Hq, d, 125).reshape(B, Hq, d)
    codes, norms = jl.jl_turbo_quantize_keys(K.cuda(), Pi, S, bits)
    out = jl.jl_turbo_decode_attention(Q.cuda(), Pinv, S, codes.reshape(B, Hkv, T, -1),
                                       norms.reshape(B, Hkv, T, 2), V.cuda(), bits)
    torch.cuda.synchronize()
    assert jl.jl_device_error() == 0
    ref = tq.quantize(H.f64(K), Pit, c, S64)
    ref_out, _ = tq.decode(H.f64(Q), Pit, S64, c, ref["cell"].reshape(B, Hkv, T, d),
                           ref["signs"].reshape(B, Hkv, T, -1),
                           oracle.fp16_bits_to_f64(ref["norm16"]).reshape(B, Hkv, T),
                           oracle.fp16_bits_to_f64(ref["rnorm16"]).reshape(B, Hkv, T),
                           H.f64(V), 1 / np.sqrt(d))
    mabs, rel = H.output_errors(H.f64(out), ref_out)
    assert mabs <= H.OUT_ABS, mabs


def test_decode_rejects_bad_arguments():
    torch.cuda.set_device(0)
    L = jl.load()
    assert jl.jl_turbo_decode_workspace_bytes(1, 8, 2, 64, 128, 128, 4) == 0
    assert jl.jl_turbo_decode_workspace_bytes(1, 8, 2, 64, 256, 128, 2) == 0
    assert jl.jl_turbo_decode_workspace_bytes(1, 8, 2, 64, 128, 128, 2) > 0
    assert jl.jl_turbo_decode_workspace_bytes(1, 8, 2, 64, 64, 64, 2) > 0
    assert jl.jl_turbo_decode_workspace_bytes(1, 8, 2, 64, 128, 64, 2) == 0   # m = d only
    st = L.jl_turbo_quantize_keys(None, jl.JL_F32, 4, 128, None, None, 128, 128, 2, None, None,
                                  None)
    assert st == jl.JL_ERR_UNSUPPORTED


def test_turbo_gqa_full_size_sampled_units():
    # the turbo-gqa cache at full size, in the bench's launch configuration:
    # library rotation, sketch and quantizer over all 2,097,152 keys, then one
    # decode.  Sampled (b, kv-head) units: their codes are checked against the
    # oracle's, then the oracle's codes are planted in the GPU cache so that
    # the sampled heads' scores and outputs compare exactly-defined quantities.
    torch.cuda.set_device(0)
    w = workloads.TURBO_GQA
    bits = workloads.TURBO_MSE_BITS
    dev = "cuda"
    Pi, Pinv = jl.jl_turbo_rotation_init(w.d, workloads.TURBO_ROTATION_SEED)
    S = jl.jl_sketch_init(w.m, w.d, w.sketch_seed)
    pit_bits = tq.rotation_bf16_bits(w.d, workloads.TURBO_ROTATION_SEED)
    assert np.array_equal(Pi.cpu().view(torch.int16).numpy().view(np.uint16), pit_bits)
    Pit = oracle.bf16_bits_to_f64(pit_bits)
    S64 = oracle.sketch(w.m, w.d, w.sketch_seed)
    c = tq.lloyd_max(w.d, bits)
    K = workloads.keys(w, dev)
    V = workloads.values(w, dev)
    Q = workloads.queries(w, dev)
    codes, norms = jl.jl_turbo_quantize_keys(K.view(-1, w.d), Pi, S, bits)
    codes = codes.view(w.B, w.Hkv, w.T, -1)
    norms = norms.view(w.B, w.Hkv, w.T, 2)
    torch.cuda.synchronize()
    assert jl.jl_device_error() == 0
    units = [(0, 0), (7, 7), (3, 5)]
    refs = {}
    for (b, hk) in units:
        ref = tq.quantize(H.f64(K[b, hk]), Pit, c, S64, band_abs=BAND_Y, band_rel=BAND_SIGN)
        gw = H.u32(codes[b, hk])
        gcell = tq.unpack_planes(gw[:, :bits * D // 32], D, bits)
        cdiff = gcell != ref["cell"]
        assert not np.any(cdiff & ~ref["cell_band"]), (b, hk)
        ok = ~cdiff.any(axis=1)
        sdiff = (H.code_bits(gw[:, bits * D // 32:], M) != H.code_bits(ref["signs"], M)) & ok[:, None]
        assert not np.any(sdiff & ~(np.abs(ref["proj"]) < ref["sign_allow"])), (b, hk)
        gn = H.fp16_bits(norms[b, hk])
        assert H.fp16_ulp_diff(gn[:, 0], ref["norm16"]).max() <= 1
        assert H.fp16_ulp_diff(gn[:, 1], ref["rnorm16"])[ok].max(initial=0) <= 1
        rc = np.concatenate([tq.pack_planes(ref["cell"], bits), ref["signs"]], axis=1)
        codes[b, hk] = torch.from_numpy(rc.view(np.int32)).to(dev)
        norms[b, hk] = torch.from_numpy(
            np.stack([ref["norm16"], ref["rnorm16"]], axis=1).view(np.float16)).to(dev)
        refs[(b, hk)] = ref
        print(f"turbo-gqa unit {(b, hk)}: {int(cdiff.sum())} in-band cells, "
              f"{int(sdiff.sum())} allowed sign flips")
    del K
    out, sc = jl.jl_turbo_decode_attention(Q, Pinv, S, codes, norms, V, bits,
                                           softmax_scale=w.softmax_scale, want_scores=True)
    torch.cuda.synchronize()
    assert jl.jl_device_error() == 0
    for (b, hk) in units:
        ref = refs[(b, hk)]
        hqs = list(range(hk * w.G, (hk + 1) * w.G))
        ref_out, ref_sc = tq.decode(H.f64(Q[b, hqs])[None], Pit, S64, c,
                                    ref["cell"].reshape(1, 1, w.T, D),
                                    ref["signs"].reshape(1, 1, w.T, -1),
                                    oracle.fp16_bits_to_f64(ref["norm16"]).reshape(1, 1, w.T),
                                    oracle.fp16_bits_to_f64(ref["rnorm16"]).reshape(1, 1, w.T),
                                    H.f64(V[b, hk])[None, None], w.softmax_scale,
                                    want_scores=True)
        assert H.score_violations(H.f64(sc[b, hqs])[None], ref_sc) == 0, (b, hk)
        mabs, rel = H.output_errors(H.f64(out[b, hqs])[None], ref_out)
        assert mabs <= H.OUT_ABS and rel <= 1e-2, (b, hk, mabs, rel)
