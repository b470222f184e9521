"""Host-side checks of libjlkey that need no GPU.

The library must load, export every entry point include/jlkey.h declares, and
reject bad arguments before launching anything.  The host copy of the
sketch's bf16 rounding is compared with the oracle's rounding.
"""
import ctypes
import os
import re

import numpy as np
import pytest

import bit_jl_key_b200 as jl
import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"JL_API\s+[\w\s\*]*?\b(jl_\w+)\s*\(", src)
    return names


@pytest.fixture(scope="module")
def lib():
    from bit_jl_key_b200 import build
    build.build()
    return jl.load()


def test_every_declared_symbol_is_exported(lib):
    names = _declared_symbols()
    assert len(names) >= 8
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(jl.EXPORTED)


def test_status_strings(lib):
    for st in (jl.JL_OK, jl.JL_ERR_INVALID_ARG, jl.JL_ERR_UNSUPPORTED,
               jl.JL_ERR_WORKSPACE, jl.JL_ERR_CUDA, jl.JL_ERR_DEVICE):
        s = jl.status_string(st)
        assert s and s != "unknown status"
    assert jl.status_string(12345) == "unknown status"


def test_host_bf16_rounding_matches_oracle(lib):
    rng = np.random.default_rng(0)
    vals = list(rng.normal(size=2000)) + list(rng.normal(size=200) * 1e-38)
    vals += [1 + 2 ** -8, 1 + 3 * 2 ** -8, 1 + 2 ** -8 + 2 ** -40, -(1 + 2 ** -8),
             0.0, -0.0, 3e38, -3.5e38, 2 ** -133, 2 ** -134, 3 * 2 ** -134, 1e-300]
    for x in vals:
        assert jl.jl_bf16_from_f64(float(x)) == oracle.f64_to_bf16_bits(float(x)), x


def test_workspace_query(lib):
    f = jl.jl_decode_workspace_bytes
    assert f(8, 32, 8, 32768, 256, 128) > 8 * 32 * 256 * 4
    assert f(1, 1, 1, 1024, 256, 128) > 0
    assert f(0, 32, 8, 1024, 256, 128) == 0        # nothing to do
    assert f(1, 6, 4, 1024, 256, 128) == 0         # Hq not a multiple of Hkv
    assert f(1, 1, 1, 1024, 96, 128) == 0          # unsupported m
    assert f(1, 1, 1, 1024, 256, 96) == 0          # unsupported d
    assert f(1, 1, 1, 0, 256, 128) == 0            # empty context
    # depends on shapes only
    assert f(2, 16, 4, 777, 128, 64) == f(2, 16, 4, 777, 128, 64)


NULL = ctypes.c_void_p(0)
FAKE = ctypes.c_void_p(1 << 20)          # 16-byte aligned, never dereferenced
MISALIGNED = ctypes.c_void_p((1 << 20) + 2)


def test_sketch_argument_errors(lib):
    assert lib.jl_sketch_init(NULL, 256, 128, 0, NULL) == jl.JL_ERR_INVALID_ARG
    assert lib.jl_sketch_init(MISALIGNED, 256, 128, 0, NULL) == jl.JL_ERR_INVALID_ARG
    assert lib.jl_sketch_init(FAKE, 100, 128, 0, NULL) == jl.JL_ERR_UNSUPPORTED
    assert lib.jl_sketch_init(FAKE, 256, 32, 0, NULL) == jl.JL_ERR_UNSUPPORTED


@pytest.mark.parametrize("name", ["jl_quantize_keys", "jl_quantize_keys_simt"])
def test_quantize_argument_errors(lib, name):
    f = getattr(lib, name)
    ok = dict(K=FAKE, kt=jl.JL_BF16, n=10, ldk=128, S=FAKE, m=256, d=128,
              signs=FAKE, norms=FAKE)

    def call(**kw):
        a = dict(ok, **kw)
        return f(a["K"], a["kt"], a["n"], a["ldk"], a["S"], a["m"], a["d"],
                 a["signs"], a["norms"], NULL)

    assert call(n=0) == jl.JL_OK                     # empty: no-op
    assert call(n=-1) == jl.JL_ERR_INVALID_ARG
    assert call(K=NULL) == jl.JL_ERR_INVALID_ARG
    assert call(S=NULL) == jl.JL_ERR_INVALID_ARG
    assert call(signs=NULL) == jl.JL_ERR_INVALID_ARG
    assert call(norms=NULL) == jl.JL_ERR_INVALID_ARG
    assert call(K=MISALIGNED) == jl.JL_ERR_INVALID_ARG
    assert call(ldk=100) == jl.JL_ERR_INVALID_ARG     # < d
    assert call(ldk=130) == jl.JL_ERR_INVALID_ARG     # 260 B not a 16 B multiple
    assert call(kt=7) == jl.JL_ERR_INVALID_ARG
    assert call(m=96) == jl.JL_ERR_UNSUPPORTED
    assert call(d=80, ldk=80) == jl.JL_ERR_UNSUPPORTED


def test_decode_argument_errors(lib):
    f = lib.jl_decode_attention
    ok = dict(Q=FAKE, qt=jl.JL_BF16, S=FAKE, signs=FAKE, norms=FAKE, V=FAKE,
              B=2, Hq=8, Hkv=2, T=100, m=256, d=128, scale=0.1, out=FAKE,
              scores=NULL, ws=FAKE, wsb=1 << 40)

    def call(**kw):
        a = dict(ok, **kw)
        return f(a["Q"], a["qt"], a["S"], a["signs"], a["norms"], a["V"],
                 a["B"], a["Hq"], a["Hkv"], a["T"], a["m"], a["d"],
                 ctypes.c_float(a["scale"]), a["out"], a["scores"], a["ws"],
                 a["wsb"], NULL)

    assert call(B=0) == jl.JL_OK                     # empty batch: no-op
    assert call(T=0) == jl.JL_ERR_INVALID_ARG        # empty context
    assert call(Hq=6, Hkv=4) == jl.JL_ERR_INVALID_ARG
    assert call(Hkv=0) == jl.JL_ERR_INVALID_ARG
    assert call(qt=5) == jl.JL_ERR_INVALID_ARG
    assert call(m=48) == jl.JL_ERR_UNSUPPORTED
    assert call(d=256) == jl.JL_ERR_UNSUPPORTED
    for k in ("Q", "S", "signs", "norms", "V", "out"):
        assert call(**{k: NULL}) == jl.JL_ERR_INVALID_ARG, k
    assert call(V=MISALIGNED) == jl.JL_ERR_INVALID_ARG
    assert call(signs=MISALIGNED) == jl.JL_ERR_INVALID_ARG
    assert call(norms=ctypes.c_void_p((1 << 20) + 8)) == jl.JL_ERR_INVALID_ARG
    assert call(scale=float("nan")) == jl.JL_ERR_INVALID_ARG
    assert call(ws=NULL) == jl.JL_ERR_WORKSPACE
    need = jl.jl_decode_workspace_bytes(2, 8, 2, 100, 256, 128)
    assert call(wsb=need - 1) == jl.JL_ERR_WORKSPACE
    assert call(ws=ctypes.c_void_p((1 << 20) + 16)) == jl.JL_ERR_WORKSPACE


def test_noalloc_argument_errors_match_decode(lib):
    # the no-alloc variant shares jl_decode_attention's checks (minus the
    # workspace): every argument error gets the same status from both
    f = lib.jl_decode_attention_noalloc
    g = lib.jl_decode_attention
    ok = dict(Q=FAKE, qt=jl.JL_BF16, S=FAKE, signs=FAKE, norms=FAKE, V=FAKE,
              B=2, Hq=8, Hkv=2, T=100, m=256, d=128, scale=0.1, out=FAKE,
              scores=NULL)

    def both(**kw):
        a = dict(ok, **kw)
        args = (a["Q"], a["qt"], a["S"], a["signs"], a["norms"], a["V"], a["B"], a["Hq"],
                a["Hkv"], a["T"], a["m"], a["d"], ctypes.c_float(a["scale"]), a["out"],
                a["scores"])
        return f(*args, NULL), g(*args, FAKE, 1 << 40, NULL)

    cases = [dict(B=0), dict(T=0), dict(Hq=6, Hkv=4), dict(Hkv=0), dict(qt=5), dict(m=48),
             dict(d=256), dict(V=MISALIGNED), dict(signs=MISALIGNED),
             dict(norms=ctypes.c_void_p((1 << 20) + 8)), dict(scale=float("nan")),
             dict(scores=ctypes.c_void_p((1 << 20) + 2))]
    cases += [{k: NULL} for k in ("Q", "S", "signs", "norms", "V", "out")]
    for kw in cases:
        na, ws = both(**kw)
        assert na == ws, (kw, na, ws)
        assert (na == jl.JL_OK) == (kw == dict(B=0)), kw


def test_state_decode_argument_errors_match_decode(lib):
    # the state variant takes jl_decode_attention's checks, the state buffer
    # standing in for the output
    f = lib.jl_decode_attention_state
    g = lib.jl_decode_attention
    ok = dict(Q=FAKE, qt=jl.JL_BF16, S=FAKE, signs=FAKE, norms=FAKE, V=FAKE,
              B=2, Hq=8, Hkv=2, T=100, m=256, d=128, scale=0.1, out=FAKE,
              scores=NULL, ws=FAKE, wsb=1 << 40)

    def both(**kw):
        a = dict(ok, **kw)
        args = (a["Q"], a["qt"], a["S"], a["signs"], a["norms"], a["V"], a["B"], a["Hq"],
                a["Hkv"], a["T"], a["m"], a["d"], ctypes.c_float(a["scale"]), a["out"],
                a["scores"], a["ws"], a["wsb"], NULL)
        return f(*args), g(*args)

    cases = [dict(B=0), dict(T=0), dict(Hq=6, Hkv=4), dict(Hkv=0), dict(qt=5), dict(m=48),
             dict(d=256), dict(V=MISALIGNED), dict(signs=MISALIGNED),
             dict(out=ctypes.c_void_p((1 << 20) + 2)), dict(scale=float("nan")),
             dict(ws=NULL), dict(wsb=jl.jl_decode_workspace_bytes(2, 8, 2, 100, 256, 128) - 1)]
    cases += [{k: NULL} for k in ("Q", "S", "signs", "norms", "V", "out")]
    for kw in cases:
        st, dec = both(**kw)
        assert st == dec, (kw, st, dec)
        assert (st == jl.JL_OK) == (kw == dict(B=0)), kw


def test_merge_states_argument_errors(lib):
    f = lib.jl_merge_attention_states

    def call(states=FAKE, R=2, rows=16, d=128, out=FAKE):
        return f(states, R, rows, d, out, NULL)

    assert call(rows=0) == jl.JL_OK                   # nothing to merge
    assert call(R=0) == jl.JL_ERR_INVALID_ARG
    assert call(R=65537) == jl.JL_ERR_INVALID_ARG
    assert call(rows=-1) == jl.JL_ERR_INVALID_ARG
    assert call(rows=1 << 31) == jl.JL_ERR_INVALID_ARG
    assert call(d=96) == jl.JL_ERR_UNSUPPORTED
    assert call(states=NULL) == jl.JL_ERR_INVALID_ARG
    assert call(out=NULL) == jl.JL_ERR_INVALID_ARG
    assert call(states=ctypes.c_void_p((1 << 20) + 2)) == jl.JL_ERR_INVALID_ARG
    assert call(out=ctypes.c_void_p((1 << 20) + 2)) == jl.JL_ERR_INVALID_ARG


def test_state_wrappers_refuse_bad_tensors(lib):
    import torch
    with pytest.raises(ValueError):             # well-formed, but on the host
        jl.jl_merge_attention_states(torch.zeros(2, 4, 130))
    with pytest.raises(ValueError):
        jl.jl_merge_attention_states(torch.zeros(2, 4, 130, dtype=torch.float64))
    with pytest.raises(ValueError):
        jl.jl_merge_attention_states(torch.zeros(2, 4, 130),
                                     out=torch.zeros(4, 64, dtype=torch.bfloat16))
    B, Hq, Hkv, T, m, d = 1, 4, 2, 64, 256, 128
    args = (torch.zeros(B, Hq, d, dtype=torch.bfloat16), torch.zeros(m, d, dtype=torch.bfloat16),
            torch.zeros(B, Hkv, T, m // 32, dtype=torch.int32),
            torch.zeros(B, Hkv, T, dtype=torch.float16),
            torch.zeros(B, Hkv, T, d, dtype=torch.bfloat16))
    with pytest.raises(ValueError):             # state of the wrong width
        jl.jl_decode_attention_state(*args, state=torch.zeros(B, Hq, d))
    with pytest.raises(ValueError):
        jl.jl_decode_attention_state(*args)


@pytest.mark.parametrize("fn", ["jl_decode_attention", "jl_decode_attention_noalloc"])
def test_decode_wrappers_check_shapes_and_dtypes(lib, fn):
    # the library sizes its copies from the shapes, so the binding must refuse
    # tensors that do not hold what those shapes say (checked before any
    # device test: these tensors are on the host)
    import torch
    B, Hq, Hkv, T, m, d = 2, 8, 2, 64, 256, 128
    Q = torch.zeros(B, Hq, d, dtype=torch.bfloat16)
    S = torch.zeros(m, d, dtype=torch.bfloat16)
    signs = torch.zeros(B, Hkv, T, m // 32, dtype=torch.int32)
    norms = torch.zeros(B, Hkv, T, dtype=torch.float16)
    V = torch.zeros(B, Hkv, T, d, dtype=torch.bfloat16)
    call = getattr(jl, fn)
    bad = [
        dict(signs=torch.zeros(B, Hkv, T - 1, m // 32, dtype=torch.int32)),
        dict(signs=torch.zeros(B, Hkv, T, m // 64, dtype=torch.int32)),
        dict(signs=signs.float()),
        dict(norms=torch.zeros(B, Hkv, T - 1, dtype=torch.float16)),
        dict(norms=norms.float()),
        dict(V=V.half()),
        dict(V=torch.zeros(B, Hkv, T, 64, dtype=torch.bfloat16)),
        dict(S=torch.zeros(m, 64, dtype=torch.bfloat16)),
        dict(S=S.float()),
    ]
    for kw in bad:
        a = dict(Q=Q, S=S, signs=signs, norms=norms, V=V)
        a.update(kw)
        with pytest.raises(ValueError):
            call(a["Q"], a["S"], a["signs"], a["norms"], a["V"])
    with pytest.raises(TypeError):
        call(Q.half(), S, signs, norms, V)
    with pytest.raises(ValueError):          # well-formed, but on the host
        call(Q, S, signs, norms, V)


def test_drop_copies_hook_arguments(lib):
    f = lib.jl_test_drop_copies
    assert f(0, 0) == jl.JL_OK
    assert f(1, 1_000_000) == jl.JL_OK
    assert f(1, 0) == jl.JL_OK                 # default bound
    assert f(2, 0) == jl.JL_ERR_INVALID_ARG
    assert f(1, 999) == jl.JL_ERR_INVALID_ARG   # below 1 us
    assert f(1, 2_000_000_001) == jl.JL_ERR_INVALID_ARG
    assert f(0, 0) == jl.JL_OK                 # left off for the other tests


def test_binding_refuses_cpu_tensors(lib):
    import torch
    with pytest.raises(ValueError):
        jl.jl_quantize_keys(torch.zeros(4, 128, dtype=torch.bfloat16),
                            torch.zeros(256, 128, dtype=torch.bfloat16))


def test_paged_workspace_query(lib):
    f = jl.jl_decode_paged_workspace_bytes
    assert f(4, 32, 8, 4096, 256, 128) > 4 * 32 * 256 * 4
    assert f(0, 32, 8, 4096, 256, 128) == 0
    assert f(1, 6, 4, 4096, 256, 128) == 0
    assert f(1, 1, 1, 0, 256, 128) == 0
    # sized by the bound, so never below the contiguous plan at that length
    assert f(4, 32, 8, 4096, 256, 128) >= jl.jl_decode_workspace_bytes(4, 32, 8, 4096, 256, 128)


def test_paged_decode_argument_errors(lib):
    f = lib.jl_decode_attention_paged
    ok = dict(Q=FAKE, qt=jl.JL_BF16, Kn=FAKE, kt=jl.JL_BF16, Vn=FAKE, S=FAKE,
              sp=FAKE, np_=FAKE, vp=FAKE, npages=16, P=64, table=FAKE, maxp=4,
              lens=FAKE, B=2, Hq=8, Hkv=2, max_len=256, m=256, d=128, scale=0.1,
              out=FAKE, scores=NULL, ws=FAKE, wsb=1 << 40)

    def call(**kw):
        a = dict(ok, **kw)
        return f(a["Q"], a["qt"], a["Kn"], a["kt"], a["Vn"], a["S"], a["sp"], a["np_"],
                 a["vp"], a["npages"], a["P"], a["table"], a["maxp"], a["lens"], a["B"],
                 a["Hq"], a["Hkv"], a["max_len"], a["m"], a["d"],
                 ctypes.c_float(a["scale"]), a["out"], a["scores"], a["ws"], a["wsb"], NULL)

    assert call(B=0) == jl.JL_OK
    assert call(P=48) == jl.JL_ERR_INVALID_ARG          # page not a whole number of 32-key blocks
    assert call(P=0) == jl.JL_ERR_INVALID_ARG
    assert call(maxp=3) == jl.JL_ERR_INVALID_ARG        # 3 * 64 < max_len
    assert call(npages=0) == jl.JL_ERR_INVALID_ARG
    assert call(max_len=0) == jl.JL_ERR_INVALID_ARG
    assert call(Hq=6, Hkv=4) == jl.JL_ERR_INVALID_ARG
    assert call(kt=9) == jl.JL_ERR_INVALID_ARG
    assert call(Vn=NULL) == jl.JL_ERR_INVALID_ARG        # key without its value
    assert call(m=96) == jl.JL_ERR_UNSUPPORTED
    for k in ("Q", "S", "sp", "np_", "vp", "table", "lens", "out"):
        assert call(**{k: NULL}) == jl.JL_ERR_INVALID_ARG, k
    assert call(vp=MISALIGNED) == jl.JL_ERR_INVALID_ARG
    assert call(Kn=MISALIGNED) == jl.JL_ERR_INVALID_ARG
    assert call(lens=ctypes.c_void_p((1 << 20) + 2)) == jl.JL_ERR_INVALID_ARG
    assert call(ws=NULL) == jl.JL_ERR_WORKSPACE
    need = jl.jl_decode_paged_workspace_bytes(2, 8, 2, 256, 256, 128)
    assert call(wsb=need - 1) == jl.JL_ERR_WORKSPACE
    # without a new key, the key dtype is not looked at
    assert call(Kn=NULL, Vn=NULL, kt=9, ws=NULL) == jl.JL_ERR_WORKSPACE


def test_dequantize_argument_errors(lib):
    f = lib.jl_dequantize_keys
    ok = dict(signs=FAKE, norms=FAKE, n=10, S=FAKE, m=256, d=128, out=FAKE)

    def call(**kw):
        a = dict(ok, **kw)
        return f(a["signs"], a["norms"], a["n"], a["S"], a["m"], a["d"], a["out"], NULL)

    assert call(n=0) == jl.JL_OK
    assert call(n=-1) == jl.JL_ERR_INVALID_ARG
    assert call(m=96) == jl.JL_ERR_UNSUPPORTED
    assert call(d=32) == jl.JL_ERR_UNSUPPORTED
    for k in ("signs", "norms", "S", "out"):
        assert call(**{k: NULL}) == jl.JL_ERR_INVALID_ARG, k
    assert call(signs=MISALIGNED) == jl.JL_ERR_INVALID_ARG
    assert call(out=ctypes.c_void_p((1 << 20) + 8)) == jl.JL_ERR_INVALID_ARG
    assert call(norms=ctypes.c_void_p((1 << 20) + 1)) == jl.JL_ERR_INVALID_ARG


def test_search_argument_errors(lib):
    f = lib.jl_search_topk
    ok = dict(Q=FAKE, qt=jl.JL_BF16, nq=4, S=FAKE, m=256, d=128, signs=FAKE, norms=FAKE,
              N=1000, k=10, oi=FAKE, os=FAKE, ws=FAKE, wsb=1 << 40)

    def call(**kw):
        a = dict(ok, **kw)
        return f(a["Q"], a["qt"], a["nq"], a["S"], a["m"], a["d"], a["signs"], a["norms"],
                 a["N"], a["k"], a["oi"], a["os"], a["ws"], a["wsb"], NULL)

    assert call(nq=0) == jl.JL_OK
    assert call(nq=-1) == jl.JL_ERR_INVALID_ARG
    assert call(N=0) == jl.JL_ERR_INVALID_ARG
    assert call(k=0) == jl.JL_ERR_INVALID_ARG
    assert call(k=17) == jl.JL_ERR_INVALID_ARG
    assert call(qt=3) == jl.JL_ERR_INVALID_ARG
    assert call(m=100) == jl.JL_ERR_UNSUPPORTED
    for key in ("Q", "S", "signs", "norms", "oi", "os"):
        assert call(**{key: NULL}) == jl.JL_ERR_INVALID_ARG, key
    assert call(signs=MISALIGNED) == jl.JL_ERR_INVALID_ARG
    assert call(ws=NULL) == jl.JL_ERR_WORKSPACE
    need = jl.jl_search_workspace_bytes(4, 256, 128, 10)
    assert need > 0 and call(wsb=need - 1) == jl.JL_ERR_WORKSPACE
    assert jl.jl_search_workspace_bytes(4, 256, 128, 17) == 0


# --------------------------------------------------------------------------
# TurboQuant-prod entry points

@pytest.mark.parametrize("bits", [1, 2, 3])
def test_turbo_codebook_matches_oracle_on_host(lib, bits):
    # the library computes its codebook on the host (its own quadrature); it
    # must equal the oracle's Lloyd-Max centroids rounded to float
    from oracle import turbo as tq
    for d in (3, 64, 128, 1000):
        got = np.array(jl.jl_turbo_codebook(d, bits), dtype=np.float32)
        assert np.array_equal(got, tq.lloyd_max(d, bits).astype(np.float32)), d


def test_turbo_codebook_argument_errors(lib):
    buf = (ctypes.c_float * 8)()
    p = ctypes.cast(buf, ctypes.c_void_p)
    assert lib.jl_turbo_codebook(128, 2, NULL) == jl.JL_ERR_INVALID_ARG
    assert lib.jl_turbo_codebook(2, 2, p) == jl.JL_ERR_UNSUPPORTED
    assert lib.jl_turbo_codebook(128, 0, p) == jl.JL_ERR_UNSUPPORTED
    assert lib.jl_turbo_codebook(128, 4, p) == jl.JL_ERR_UNSUPPORTED
    assert lib.jl_turbo_codebook(128, 3, p) == jl.JL_OK


def test_turbo_rotation_argument_errors(lib):
    f = lib.jl_turbo_rotation_init
    need = jl.jl_turbo_rotation_workspace_bytes(128)
    assert need == 4 * 128 * 128 * 8
    assert jl.jl_turbo_rotation_workspace_bytes(96) == 0
    assert f(FAKE, FAKE, 96, 1, FAKE, need, NULL) == jl.JL_ERR_UNSUPPORTED
    assert f(NULL, FAKE, 128, 1, FAKE, need, NULL) == jl.JL_ERR_INVALID_ARG
    assert f(FAKE, MISALIGNED, 128, 1, FAKE, need, NULL) == jl.JL_ERR_INVALID_ARG
    assert f(FAKE, FAKE, 128, 1, NULL, need, NULL) == jl.JL_ERR_WORKSPACE
    assert f(FAKE, FAKE, 128, 1, FAKE, need - 1, NULL) == jl.JL_ERR_WORKSPACE


def test_turbo_quantize_argument_errors(lib):
    f = lib.jl_turbo_quantize_keys
    ok = dict(K=FAKE, kt=jl.JL_BF16, n=10, ld=128, Pi=FAKE, S=FAKE, m=128, d=128, bits=2,
              codes=FAKE, norms=FAKE)

    def call(**kw):
        a = dict(ok, **kw)
        return f(a["K"], a["kt"], a["n"], a["ld"], a["Pi"], a["S"], a["m"], a["d"], a["bits"],
                 a["codes"], a["norms"], NULL)

    assert call(n=0) == jl.JL_OK
    assert call(n=-1) == jl.JL_ERR_INVALID_ARG
    assert call(kt=jl.JL_F32) == jl.JL_ERR_UNSUPPORTED
    assert call(m=256) == jl.JL_ERR_UNSUPPORTED
    assert call(d=64) == jl.JL_ERR_UNSUPPORTED
    assert call(bits=0) == jl.JL_ERR_UNSUPPORTED
    assert call(bits=4) == jl.JL_ERR_UNSUPPORTED
    for k in ("K", "Pi", "S", "codes", "norms"):
        assert call(**{k: NULL}) == jl.JL_ERR_INVALID_ARG, k
    assert call(ld=100) == jl.JL_ERR_INVALID_ARG
    assert call(ld=132) == jl.JL_ERR_INVALID_ARG          # 264-byte rows: not 16-byte multiples
    assert call(K=MISALIGNED) == jl.JL_ERR_INVALID_ARG
    assert call(norms=ctypes.c_void_p((1 << 20) + 2)) == jl.JL_ERR_INVALID_ARG


def test_turbo_decode_argument_errors(lib):
    f = lib.jl_turbo_decode_attention
    need = jl.jl_turbo_decode_workspace_bytes(2, 8, 2, 64, 128, 128, 2)
    assert need > 0
    assert jl.jl_turbo_decode_workspace_bytes(2, 8, 2, 64, 128, 128, 4) == 0
    assert jl.jl_turbo_decode_workspace_bytes(2, 8, 2, 64, 128, 128, 3) > need
    assert jl.jl_turbo_decode_workspace_bytes(2, 8, 2, 64, 256, 128, 2) == 0
    ok = dict(Q=FAKE, qt=jl.JL_BF16, Pinv=FAKE, S=FAKE, codes=FAKE, norms=FAKE, V=FAKE, B=2,
              Hq=8, Hkv=2, T=64, m=128, d=128, bits=2, scale=0.088, out=FAKE, sc=NULL, ws=FAKE,
              wsb=need)

    def call(**kw):
        a = dict(ok, **kw)
        return f(a["Q"], a["qt"], a["Pinv"], a["S"], a["codes"], a["norms"], a["V"], a["B"],
                 a["Hq"], a["Hkv"], a["T"], a["m"], a["d"], a["bits"],
                 ctypes.c_float(a["scale"]), a["out"], a["sc"], a["ws"], a["wsb"], NULL)

    assert call(B=0) == jl.JL_OK
    assert call(B=-1) == jl.JL_ERR_INVALID_ARG
    assert call(T=0) == jl.JL_ERR_INVALID_ARG
    assert call(Hq=6, Hkv=4) == jl.JL_ERR_INVALID_ARG
    assert call(bits=4) == jl.JL_ERR_UNSUPPORTED
    assert call(m=256) == jl.JL_ERR_UNSUPPORTED
    assert call(scale=float("nan")) == jl.JL_ERR_INVALID_ARG
    for k in ("Q", "Pinv", "S", "codes", "norms", "V", "out"):
        assert call(**{k: NULL}) == jl.JL_ERR_INVALID_ARG, k
    assert call(codes=MISALIGNED) == jl.JL_ERR_INVALID_ARG
    assert call(ws=NULL) == jl.JL_ERR_WORKSPACE
    assert call(wsb=need - 1) == jl.JL_ERR_WORKSPACE


def test_turbo_paged_argument_errors(lib):
    f = lib.jl_turbo_decode_attention_paged
    need = jl.jl_turbo_decode_paged_workspace_bytes(2, 8, 2, 256, 128, 128, 2)
    assert need > 0
    assert jl.jl_turbo_decode_paged_workspace_bytes(2, 8, 2, 256, 128, 128, 4) == 0
    ok = dict(Q=FAKE, qt=jl.JL_BF16, K=FAKE, kt=jl.JL_BF16, V=FAKE, Pi=FAKE, Pinv=FAKE, S=FAKE,
              cp=FAKE, np_=FAKE, vp=FAKE, npages=20, P=64, tab=FAKE, maxp=4, lens=FAKE, B=2, Hq=8,
              Hkv=2, max_len=256, m=128, d=128, bits=2, scale=0.088, out=FAKE, sc=NULL, ws=FAKE,
              wsb=need)

    def call(**kw):
        a = dict(ok, **kw)
        return f(a["Q"], a["qt"], a["K"], a["kt"], a["V"], a["Pi"], a["Pinv"], a["S"], a["cp"],
                 a["np_"], a["vp"], a["npages"], a["P"], a["tab"], a["maxp"], a["lens"], a["B"],
                 a["Hq"], a["Hkv"], a["max_len"], a["m"], a["d"], a["bits"],
                 ctypes.c_float(a["scale"]), a["out"], a["sc"], a["ws"], a["wsb"], NULL)

    assert call(B=0) == jl.JL_OK
    assert call(P=48) == jl.JL_ERR_INVALID_ARG            # not a multiple of 32
    assert call(maxp=3) == jl.JL_ERR_INVALID_ARG          # pages cannot hold max_len
    assert call(bits=4) == jl.JL_ERR_UNSUPPORTED
    assert call(m=256) == jl.JL_ERR_UNSUPPORTED
    assert call(Pi=NULL) == jl.JL_ERR_INVALID_ARG         # appending needs the rotation
    assert call(V=NULL) == jl.JL_ERR_INVALID_ARG          # key without its value
    assert call(kt=9) == jl.JL_ERR_INVALID_ARG
    assert call(Hq=6, Hkv=4) == jl.JL_ERR_INVALID_ARG
    # without a new key neither the rotation nor the key dtype is looked at
    assert call(K=NULL, V=NULL, Pi=NULL, kt=9, ws=NULL) == jl.JL_ERR_WORKSPACE
    for k in ("Q", "Pinv", "S", "cp", "np_", "vp", "tab", "lens", "out"):
        assert call(**{k: NULL}) == jl.JL_ERR_INVALID_ARG, k
    assert call(cp=MISALIGNED) == jl.JL_ERR_INVALID_ARG
    assert call(ws=NULL) == jl.JL_ERR_WORKSPACE
    assert call(wsb=need - 1) == jl.JL_ERR_WORKSPACE


def test_missing_library_fails_loudly(tmp_path):
    # no fallback: with the library absent, loading it raises instead of
    # quietly running something else
    import subprocess
    import sys
    env = dict(os.environ, JLKEY_LIBRARY=str(tmp_path / "absent" / "libjlkey.so"))
    r = subprocess.run([sys.executable, "-c", "import bit_jl_key_b200 as jl; jl.load()"],
                       cwd=os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode != 0
    assert "libjlkey" in (r.stderr + r.stdout)
