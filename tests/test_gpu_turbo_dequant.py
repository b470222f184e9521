"""TurboQuant-prod dequantizer on the GPU against the float64 oracle.

khat = ||k|| * Pi^{-1} (c[cell] + sqrt(pi/2)/m ||r|| S^T z)  (tq.dequantize).

The GPU computes khat_j = bf16( ||k|| * sum_K R16[j][K] a16[K] ) with the
reconstruction matrix R = [Pinv | Pinv S^T] rounded to binary16
(jl_turbo_dequant_basis, fp32 products) and a = [fp16(c[cell]);
fp16(alpha) z], alpha = sqrt(pi/2)/m ||r||, accumulated in fp32.  The
tolerance of every output element follows from that arithmetic:
  * binary16 rounding of R and of a: relative 2^-11 each, so 2^-10 (+ 2^-21)
    of S1 + S2, where S1 = sum_i |Pinv_ji| |c_i| and
    S2 = alpha sum_l |(Pinv S^T)_jl| are the absolute sums of the two parts;
  * a subnormal binary16 alpha (||r|| below about 6e-3): absolute 2^-25 per
    sign term, 2^-25 sum_l |(Pinv S^T)_jl|;
  * the fp32 sums: 2^-16 (S1 + S2) for the 256-term accumulation, and
    128 * 2^-24 alpha sum_l sum_i |Pinv_ji| |S_li| for R's own sums;
  * the query map: the tests feed the oracle's inverse of Pit rounded to
    fp32 (relative 2^-24), or the library's (within EPS_PINV absolute of the
    exact inverse, the rotation test's bound): EPS_PINV (sum_i |c_i| +
    alpha sum_l sum_i |S_li|);
  * the final bf16 rounding: 2^-8 of |value|.
All of it scaled by ||k||; the bound is checked element by element.  The
basis is checked on its own: within half a binary16 step (plus the fp32
sum's error) of the float64 product.
"""
import math

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
SQRT_HALF_PI = math.sqrt(math.pi / 2)
EPS_PINV = 1e-6


def _bf16_tensor(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def _setup(bits, rot_seed=1, sk_seed=0, d=D):
    c = tq.lloyd_max(d, bits)
    pit_bits = tq.rotation_bf16_bits(d, rot_seed)
    Pit = oracle.bf16_bits_to_f64(pit_bits)
    s_bits = oracle.sketch_bf16_bits(d, d, sk_seed)
    S64 = oracle.bf16_bits_to_f64(s_bits)
    return c, pit_bits, Pit, s_bits, S64


def _oracle_pinv32(Pit):
    return np.linalg.inv(Pit).astype(np.float32)


def _tolerance(cell, signs, norms, rnorms, Pinv, S64, c, ref, eps_pinv=0.0):
    """Element-wise bound on |gpu - ref| (see the module docstring)."""
    n = cell.shape[0]
    m, d = S64.shape
    nk = np.asarray(norms, dtype=np.float64)[:, None]
    alpha = (SQRT_HALF_PI / m) * np.asarray(rnorms, dtype=np.float64)[:, None]
    aP = np.abs(Pinv)
    PS = Pinv @ S64.T                                    # d x m
    s1 = np.abs(c[cell]) @ aP.T                          # [n, d]
    sps = np.abs(PS).sum(axis=1)[None, :]                # sum_l |(Pinv S^T)_jl|
    s2 = alpha * sps
    s2b = alpha * (aP @ np.abs(S64).T).sum(axis=1)[None, :]
    sc = np.abs(c[cell]).sum(axis=1)[:, None]
    ss = np.abs(S64).sum()
    e = nk * ((2.0 ** -10 + 2.0 ** -20) * (s1 + s2) + 2.0 ** -25 * sps + 2.0 ** -16 * (s1 + s2)
              + d * 2.0 ** -24 * s2b + eps_pinv * (sc + alpha * ss))
    assert e.shape == (n, d)
    return e + 2.0 ** -8 * (np.abs(ref) + e) + 1e-30


def _check(out, ref, tol):
    g = H.f64(out)
    err = np.abs(g - ref)
    bad = err > tol
    assert not np.any(bad), (int(bad.sum()), float((err / tol).max()))
    return float((err / tol).max())


def _oracle_case(bits, K, rot_seed=1, sk_seed=0):
    c, pit_bits, Pit, s_bits, S64 = _setup(bits, rot_seed, sk_seed, d=K.shape[1])
    ref = tq.quantize(H.f64(K), Pit, c, S64)
    codes = np.concatenate([tq.pack_planes(ref["cell"], bits), ref["signs"]], axis=1)
    norms = np.stack([ref["norm16"], ref["rnorm16"]], axis=1)
    nk = oracle.fp16_bits_to_f64(ref["norm16"])
    nr = oracle.fp16_bits_to_f64(ref["rnorm16"])
    return c, Pit, s_bits, S64, ref, codes, norms, nk, nr


def test_basis_matches_oracle():
    torch.cuda.set_device(0)
    c, pit_bits, Pit, s_bits, S64 = _setup(2)
    P32 = _oracle_pinv32(Pit)
    R = jl.jl_turbo_dequant_basis(torch.from_numpy(P32).cuda(), _bf16_tensor(s_bits))
    torch.cuda.synchronize()
    assert jl.jl_device_error() == 0
    assert R.shape == (D, D + M) and R.dtype == torch.float16
    g = R.cpu().numpy().astype(np.float64)
    P = P32.astype(np.float64)
    want = np.concatenate([P, P @ S64.T], axis=1)
    dot_err = np.concatenate([np.zeros((D, D)), 128 * 2.0 ** -24 * (np.abs(P) @ np.abs(S64).T)],
                             axis=1)
    tol = 2.0 ** -11 * (np.abs(want) + dot_err) + dot_err + 2.0 ** -25
    assert np.all(np.abs(g - want) <= tol)
    # the Pinv block is exactly the binary16 rounding of the fp32 input
    assert np.array_equal(R[:, :D].cpu().numpy(), P32.astype(np.float16))


@pytest.mark.parametrize("d", [128, 64])
@pytest.mark.parametrize("bits", [1, 2, 3])
@pytest.mark.parametrize("n", [1, 300, 4099])
def test_dequantize_matches_oracle(bits, n, d):
    # oracle codes of seeded keys; n = 300 is two full tiles and a ragged 44,
    # 4099 spans 33 tiles (several per CTA) with a ragged 3
    torch.cuda.set_device(0)
    K = workloads.random_keys(n, d, 1300 + n + bits + d, scale=1.4)
    c, Pit, s_bits, S64, ref, codes, norms, nk, nr = _oracle_case(bits, K)
    P32 = _oracle_pinv32(Pit)
    R = jl.jl_turbo_dequant_basis(torch.from_numpy(P32).cuda(), _bf16_tensor(s_bits))
    out = jl.jl_turbo_dequantize_keys(torch.from_numpy(codes.view(np.int32)).cuda(),
                                      torch.from_numpy(norms.view(np.float16)).cuda(), R, bits)
    torch.cuda.synchronize()
    assert jl.jl_device_error() == 0
    want = tq.dequantize(ref["cell"], ref["signs"], nk, nr, Pit, S64, c)
    tol = _tolerance(ref["cell"], ref["signs"], nk, nr, np.linalg.inv(Pit), S64, c, want)
    worst = _check(out, want, tol)
    print(f"turbo dequantize d={d} bits={bits} n={n}: worst error {worst:.3f} of the bound")


@pytest.mark.parametrize("d", [128, 64])
def test_dequantize_random_codes_and_edge_norms(d):
    # random code bits and norms, zero norms (a zero key), a tiny ||r|| whose
    # binary16 alpha is subnormal, and large ||k||
    torch.cuda.set_device(0)
    rng = np.random.default_rng(8 + d)
    for bits in (1, 2, 3):
        c, pit_bits, Pit, s_bits, S64 = _setup(bits, rot_seed=3, sk_seed=4, d=d)
        n = 260
        words = (bits * d + d) // 32
        codes = rng.integers(0, 2 ** 32, size=(n, words), dtype=np.uint64).astype(np.uint32)
        nk16 = rng.uniform(0.01, 60.0, size=n).astype(np.float16)
        nr16 = rng.uniform(0.0, 0.6, size=n).astype(np.float16)
        nk16[0], nr16[0] = 0.0, 0.0
        nr16[1] = np.float16(2e-4)
        nr16[2] = np.float16(1e-7)
        nk16[3] = np.float16(6e4)
        norms = np.stack([nk16, nr16], axis=1)
        P32 = _oracle_pinv32(Pit)
        R = jl.jl_turbo_dequant_basis(torch.from_numpy(P32).cuda(), _bf16_tensor(s_bits))
        out = jl.jl_turbo_dequantize_keys(torch.from_numpy(codes.view(np.int32)).cuda(),
                                          torch.from_numpy(norms).cuda(), R, bits)
        torch.cuda.synchronize()
        assert jl.jl_device_error() == 0
        cell = tq.unpack_planes(codes[:, :bits * d // 32], d, bits)
        signs = codes[:, bits * d // 32:]
        nk = nk16.astype(np.float64)
        nr = nr16.astype(np.float64)
        want = tq.dequantize(cell, signs, nk, nr, Pit, S64, c)
        tol = _tolerance(cell, signs, nk, nr, np.linalg.inv(Pit), S64, c, want)
        _check(out, want, tol)
        assert torch.all(out[0] == 0)


def test_dequantize_empty_and_bad_arguments():
    torch.cuda.set_device(0)
    L = jl.load()
    c, pit_bits, Pit, s_bits, S64 = _setup(2)
    R = jl.jl_turbo_dequant_basis(torch.from_numpy(_oracle_pinv32(Pit)).cuda(),
                                  _bf16_tensor(s_bits))
    codes = torch.zeros((0, 12), dtype=torch.int32, device="cuda")
    norms = torch.zeros((0, 2), dtype=torch.float16, device="cuda")
    out = jl.jl_turbo_dequantize_keys(codes, norms, R, 2)
    assert out.shape == (0, D)
    assert L.jl_turbo_dequantize_keys(None, None, 0, None, 128, 128, 2, None, None) == jl.JL_OK
    assert L.jl_turbo_dequantize_keys(None, None, -1, None, 128, 128, 2, None, None) == \
        jl.JL_ERR_INVALID_ARG
    assert L.jl_turbo_dequantize_keys(None, None, 4, None, 128, 128, 4, None, None) == \
        jl.JL_ERR_UNSUPPORTED
    assert L.jl_turbo_dequantize_keys(None, None, 4, None, 256, 128, 2, None, None) == \
        jl.JL_ERR_UNSUPPORTED
    assert L.jl_turbo_dequantize_keys(None, None, 4, None, 128, 128, 2, None, None) == \
        jl.JL_ERR_INVALID_ARG
    c2 = torch.zeros((4, 12), dtype=torch.int32, device="cuda")
    n2 = torch.zeros((4, 2), dtype=torch.float16, device="cuda")
    o2 = torch.zeros((4, D), dtype=torch.bfloat16, device="cuda")
    st = L.jl_turbo_dequantize_keys(c2.data_ptr() + 4, n2.data_ptr(), 4, R.data_ptr(), 128, 128,
                                    2, o2.data_ptr(), None)
    assert st == jl.JL_ERR_INVALID_ARG                      # misaligned codes
    assert L.jl_turbo_dequant_basis(None, None, 128, 128, None, None) == jl.JL_ERR_INVALID_ARG
    assert L.jl_turbo_dequant_basis(None, None, 128, 64, None, None) == jl.JL_ERR_UNSUPPORTED


@pytest.mark.parametrize("d", [128, 64])
def test_end_to_end_library_rotation_quantizer_and_basis(d):
    # rotation, sketch, codes and basis all from the library; compared with
    # the oracle's dequantization of its own codes for the keys whose codes
    # and norms agree bit for bit (the others differ only within the
    # quantizer's stated bands, which its own tests check)
    torch.cuda.set_device(0)
    bits, n = 2, 4096
    c, pit_bits, Pit, s_bits, S64 = _setup(bits, rot_seed=5, d=d)
    Pi, Pinv = jl.jl_turbo_rotation_init(d, 5)
    S = jl.jl_sketch_init(d, d, 0)
    K = workloads.random_keys(n, d, 321)
    codes, norms = jl.jl_turbo_quantize_keys(K.cuda(), Pi, S, bits)
    R = jl.jl_turbo_dequant_basis(Pinv, S)
    out = jl.jl_turbo_dequantize_keys(codes, norms, R, bits)
    torch.cuda.synchronize()
    assert jl.jl_device_error() == 0
    ref = tq.quantize(H.f64(K), Pit, c, S64)
    rc = np.concatenate([tq.pack_planes(ref["cell"], bits), ref["signs"]], axis=1)
    rn = np.stack([ref["norm16"], ref["rnorm16"]], axis=1)
    same = np.all(H.u32(codes).reshape(n, -1) == rc, axis=1) & \
        np.all(H.fp16_bits(norms).reshape(n, 2) == rn, axis=1)
    assert same.mean() > 0.9, same.mean()
    nk = oracle.fp16_bits_to_f64(ref["norm16"])
    nr = oracle.fp16_bits_to_f64(ref["rnorm16"])
    want = tq.dequantize(ref["cell"], ref["signs"], nk, nr, Pit, S64, c)
    tol = _tolerance(ref["cell"], ref["signs"], nk, nr, np.linalg.inv(Pit), S64, c, want,
                     eps_pinv=EPS_PINV)
    _check(out[torch.from_numpy(np.nonzero(same)[0]).cuda()], want[same], tol[same])


def test_reconstruction_error_matches_qjl_distortion_of_residual():
    # property at any size: E_S ||k - khat||^2 = ||k||^2 ||r||^2 ((pi/2) d - 1) / m
    # (the QJL error of the residual); averaged over 16384 keys and 8 seeded
    # bf16 sketches, GPU quantize + dequantize end to end, the ratio of the
    # measured to the predicted mean error is 1 within a few percent
    torch.cuda.set_device(0)
    bits, n = 2, 16384
    Pi, Pinv = jl.jl_turbo_rotation_init(D, 9)
    ratios = []
    for seed in range(8):
        S = jl.jl_sketch_init(M, D, 300 + seed)
        K = workloads.random_keys(n, D, 500 + seed, device="cuda")
        codes, norms = jl.jl_turbo_quantize_keys(K, Pi, S, bits)
        khat = jl.jl_turbo_dequantize_keys(codes, norms, jl.jl_turbo_dequant_basis(Pinv, S),
                                           bits).double()
        k = K.double()
        nk = norms[:, 0].double()
        nr = norms[:, 1].double()
        meas = ((khat - k) ** 2).sum(1).mean().item()
        pred = ((nk * nr) ** 2).mean().item() * ((math.pi / 2) * D - 1) / M
        ratios.append(meas / pred)
    assert float(np.mean(ratios)) == pytest.approx(1.0, rel=0.04), ratios


def test_turbo_dequant_full_size_sampled_rows():
    # the turbo-gqa cache size (2,097,152 codes) in the bench's launch
    # configuration: random codes and norms, sampled rows against the oracle
    torch.cuda.set_device(0)
    bits = workloads.TURBO_MSE_BITS
    n = workloads.TURBO_GQA.B * workloads.TURBO_GQA.Hkv * workloads.TURBO_GQA.T
    words = (bits * D + M) // 32
    c, pit_bits, Pit, s_bits, S64 = _setup(bits, rot_seed=workloads.TURBO_ROTATION_SEED)
    g = torch.Generator(device="cuda")
    g.manual_seed(78)
    codes = torch.randint(-2 ** 31, 2 ** 31 - 1, (n, words), dtype=torch.int32, device="cuda",
                          generator=g)
    norms = torch.stack([torch.rand((n,), device="cuda", generator=g) * 20 + 0.1,
                         torch.rand((n,), device="cuda", generator=g) * 0.5], dim=1).half()
    P32 = _oracle_pinv32(Pit)
    R = jl.jl_turbo_dequant_basis(torch.from_numpy(P32).cuda(), _bf16_tensor(s_bits))
    out = jl.jl_turbo_dequantize_keys(codes, norms, R, bits)
    torch.cuda.synchronize()
    assert jl.jl_device_error() == 0
    rows = np.unique(np.concatenate([np.arange(0, n, 65537), [0, 127, 128, n - 1]]))
    idx = torch.from_numpy(rows).cuda()
    cw = H.u32(codes[idx]).reshape(len(rows), -1)
    cell = tq.unpack_planes(cw[:, :bits * D // 32], D, bits)
    signs = cw[:, bits * D // 32:]
    nn = norms[idx].cpu().numpy().astype(np.float64)
    want = tq.dequantize(cell, signs, nn[:, 0], nn[:, 1], Pit, S64, c)
    tol = _tolerance(cell, signs, nn[:, 0], nn[:, 1], np.linalg.inv(Pit), S64, c, want)
    _check(out[idx], want, tol)
