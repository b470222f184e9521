"""Float64 CPU oracle for QJL sign-bit key compression and decode attention.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  It shares no code with the CUDA library in ``bit_jl_key_b200``; the
two meet only through the seeded input generators in ``workloads.py``.

The arithmetic lives in ``jl_oracle.c`` (plain C, float64, OpenMP over
independent keys / heads).  This module marshals numpy arrays through ctypes
and applies the one storage rounding the C code leaves to the caller: the key
norm is stored as IEEE binary16 (numpy's float64 -> float16 cast, which rounds
to nearest-even directly from float64).

Sources, cited by page title and section:
  * "QJL: 1-Bit Quantized JL Transform for KV Cache Quantization with Zero
    Overhead", Abstract -- JL transform + sign bits; asymmetric estimator.
  * "The Geometry of Forgetting: How Three Papers Cracked KV Cache
    Quantization", section "QJL: one bit, zero parameters, unbiased inner
    products" -- Gaussian S from a seed, Q(x) = sign(Sx),
    Q^-1(z) = sqrt(pi/2)/d S^T z, unbiasedness, variance bound.
  * same page, section "The overhead nobody tells you about" -- the
    effective-bits equation of a block quantizer.
"""
import ctypes
import math
import os

import numpy as np

from . import build as _build

_LIB = None

_f64p = ctypes.POINTER(ctypes.c_double)
_u32p = ctypes.POINTER(ctypes.c_uint32)
_u16p = ctypes.POINTER(ctypes.c_uint16)
_u8p = ctypes.POINTER(ctypes.c_uint8)


def lib():
    """Load (building on first use) the oracle shared library."""
    global _LIB
    if _LIB is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        L.jlo_splitmix64.restype = ctypes.c_uint64
        L.jlo_splitmix64.argtypes = [ctypes.c_uint64, ctypes.c_uint64]
        L.jlo_uniform.restype = ctypes.c_double
        L.jlo_uniform.argtypes = [ctypes.c_uint64]
        L.jlo_gauss.restype = ctypes.c_double
        L.jlo_gauss.argtypes = [ctypes.c_uint64, ctypes.c_uint64]
        L.jlo_f64_to_bf16.restype = ctypes.c_uint16
        L.jlo_f64_to_bf16.argtypes = [ctypes.c_double]
        L.jlo_f64_to_bf16_array.restype = None
        L.jlo_f64_to_bf16_array.argtypes = [ctypes.c_long, _f64p, _u16p]
        L.jlo_bf16_to_f64.restype = ctypes.c_double
        L.jlo_bf16_to_f64.argtypes = [ctypes.c_uint16]
        L.jlo_sketch_bf16.restype = None
        L.jlo_sketch_bf16.argtypes = [ctypes.c_int, ctypes.c_int,
                                      ctypes.c_uint64, _u16p]
        L.jlo_quantize.restype = None
        L.jlo_quantize.argtypes = [ctypes.c_long, ctypes.c_int, ctypes.c_int,
                                   _f64p, ctypes.c_long, _f64p, _u32p, _f64p,
                                   ctypes.c_double, _u8p]
        L.jlo_project.restype = None
        L.jlo_project.argtypes = [ctypes.c_long, ctypes.c_int, ctypes.c_int,
                                  _f64p, _f64p, _f64p]
        L.jlo_estimate_one.restype = ctypes.c_double
        L.jlo_estimate_one.argtypes = [ctypes.c_int, _f64p, _u32p,
                                       ctypes.c_double]
        L.jlo_scores.restype = None
        L.jlo_scores.argtypes = [ctypes.c_long, ctypes.c_int, _f64p, _u32p,
                                 _f64p, _f64p]
        L.jlo_dequantize.restype = None
        L.jlo_dequantize.argtypes = [ctypes.c_long, ctypes.c_int, ctypes.c_int,
                                     _u32p, _f64p, _f64p, _f64p]
        L.jlo_decode.restype = None
        L.jlo_decode.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                 ctypes.c_long, ctypes.c_int, ctypes.c_int,
                                 _f64p, _f64p, _u32p, _f64p, _f64p,
                                 ctypes.c_double, _f64p, _f64p]
        L.jlo_exact_attention.restype = None
        L.jlo_exact_attention.argtypes = [ctypes.c_int, ctypes.c_int,
                                          ctypes.c_int, ctypes.c_long,
                                          ctypes.c_int, _f64p, _f64p, _f64p,
                                          ctypes.c_double, _f64p, _f64p]
        L.jlo_block_effective_bits.restype = ctypes.c_double
        L.jlo_block_effective_bits.argtypes = [ctypes.c_double] * 3
        L.jlo_qjl_bits_per_coordinate.restype = ctypes.c_double
        L.jlo_qjl_bits_per_coordinate.argtypes = [ctypes.c_int] * 3
        L.jlo_max_threads.restype = ctypes.c_int
        L.jlo_max_threads.argtypes = []
        _LIB = L
    return _LIB


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _ptr(a, ptype):
    return a.ctypes.data_as(ptype)


# --------------------------------------------------------------------------
# generator and roundings

def splitmix64(seed: int, n: int) -> int:
    """n-th output (0-based) of SplitMix64 started from state ``seed``."""
    return int(lib().jlo_splitmix64(seed, n))


def gauss(seed: int, e: int) -> float:
    """Standard normal drawn for sketch element e (Box-Muller, cosine)."""
    return float(lib().jlo_gauss(seed, e))


def f64_to_bf16_bits(x: float) -> int:
    return int(lib().jlo_f64_to_bf16(float(x)))


def f64_to_bf16_bits_array(x) -> np.ndarray:
    """Elementwise f64_to_bf16_bits of an array (same C rounding)."""
    x = _c(x, np.float64)
    out = np.empty(x.shape, dtype=np.uint16)
    lib().jlo_f64_to_bf16_array(x.size, _ptr(x, _f64p), _ptr(out, _u16p))
    return out


def bf16_bits_to_f64(bits) -> np.ndarray:
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def fp16_round_bits(x) -> np.ndarray:
    """IEEE binary16 codes of float64 values (round to nearest, ties even)."""
    return np.asarray(x, dtype=np.float64).astype(np.float16).view(np.uint16)


def fp16_bits_to_f64(bits) -> np.ndarray:
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


# --------------------------------------------------------------------------
# the method

def sketch_bf16_bits(m: int, d: int, seed: int) -> np.ndarray:
    """S as an (m, d) array of bfloat16 codes."""
    out = np.empty((m, d), dtype=np.uint16)
    lib().jlo_sketch_bf16(m, d, seed, _ptr(out, _u16p))
    return out


def sketch(m: int, d: int, seed: int) -> np.ndarray:
    """S as float64 values (each exactly a bfloat16)."""
    return bf16_bits_to_f64(sketch_bf16_bits(m, d, seed))


def quantize(K, S, band_rel: float = 0.0, want_band: bool = False):
    """Q(k) = sign(S k) packed LSB-first, and ||k||.

    Returns (signs uint32 [n, m/32], norms float64 [n], norms_fp16 uint16 [n],
    band uint8 [n, m] or None).  ``band`` marks |(S k)_i| < band_rel*||k||.
    """
    K = _c(K, np.float64)
    S = _c(S, np.float64)
    n, d = K.shape
    m = S.shape[0]
    assert S.shape[1] == d and m % 32 == 0
    signs = np.empty((n, m // 32), dtype=np.uint32)
    norms = np.empty(n, dtype=np.float64)
    band = np.empty((n, m), dtype=np.uint8) if want_band else None
    lib().jlo_quantize(n, d, m, _ptr(K, _f64p), d, _ptr(S, _f64p),
                       _ptr(signs, _u32p), _ptr(norms, _f64p), band_rel,
                       _ptr(band, _u8p) if want_band else None)
    return signs, norms, fp16_round_bits(norms), band


def project(Q, S) -> np.ndarray:
    """u = S q for every row of Q."""
    Q = _c(Q, np.float64)
    S = _c(S, np.float64)
    n, d = Q.shape
    m = S.shape[0]
    U = np.empty((n, m), dtype=np.float64)
    lib().jlo_project(n, d, m, _ptr(Q, _f64p), _ptr(S, _f64p), _ptr(U, _f64p))
    return U


def scores(u, signs, norms) -> np.ndarray:
    """Estimator sqrt(pi/2)/m * norm_t * <u, sign_t> for every key t."""
    u = _c(u, np.float64)
    signs = _c(signs, np.uint32)
    norms = _c(norms, np.float64)
    T = signs.shape[0]
    m = u.shape[0]
    assert signs.shape[1] * 32 == m
    out = np.empty(T, dtype=np.float64)
    lib().jlo_scores(T, m, _ptr(u, _f64p), _ptr(signs, _u32p),
                     _ptr(norms, _f64p), _ptr(out, _f64p))
    return out


def estimate(q, k, S) -> float:
    """Asymmetric estimate of <q, k> with sketch S (exact float64 norm)."""
    signs, norms, _, _ = quantize(np.asarray(k, np.float64)[None, :], S)
    u = project(np.asarray(q, np.float64)[None, :], S)[0]
    return float(scores(u, signs, norms)[0])


def dequantize(signs, norms, S) -> np.ndarray:
    """Q^-1: khat = sqrt(pi/2)/m * ||k|| * S^T z for each code.

    signs uint32 [n, m/32]; norms [n] (float64 values of the stored norms);
    S [m, d].  Returns float64 [n, d].
    """
    signs = _c(signs, np.uint32)
    norms = _c(norms, np.float64).reshape(-1)
    S = _c(S, np.float64)
    m, d = S.shape
    n = signs.shape[0]
    assert signs.shape == (n, m // 32) and norms.shape == (n,)
    out = np.empty((n, d), dtype=np.float64)
    lib().jlo_dequantize(n, d, m, _ptr(signs, _u32p), _ptr(norms, _f64p),
                         _ptr(S, _f64p), _ptr(out, _f64p))
    return out


def search_topk(Q, S, signs, norms, k: int):
    """Inner-product search over a QJL-compressed index: for each query q,
    the k index vectors with the largest estimated <q, x> (the asymmetric
    estimator, as in decode), best first; ties go to the lower index.

    Q [nq, d]; signs [N, m/32]; norms [N] (float64 values of the stored
    norms).  Returns (idx int64 [nq, k], scores float64 [nq, k], all scores
    float64 [nq, N]).  The ordering step is a library sort.
    """
    Q = _c(Q, np.float64)
    U = project(Q, S)
    N = signs.shape[0]
    allsc = np.stack([scores(U[i], signs, norms) for i in range(U.shape[0])])
    # descending by score, ascending by index among equal scores
    order = np.lexsort((np.broadcast_to(np.arange(N), allsc.shape), -allsc), axis=-1)
    idx = order[:, :k]
    return idx, np.take_along_axis(allsc, idx, axis=1), allsc


def decode(Q, S, signs, norms, V, softmax_scale: float, want_scores=False):
    """Decode attention over compressed keys.

    Q [B,Hq,d]; signs [B,Hkv,T,m/32]; norms [B,Hkv,T] (float64 values of the
    stored norms); V [B,Hkv,T,d].  Returns (out [B,Hq,d], scores [B,Hq,T] or
    None), scores being the estimator before softmax_scale.
    """
    Q = _c(Q, np.float64)
    S = _c(S, np.float64)
    signs = _c(signs, np.uint32)
    norms = _c(norms, np.float64)
    V = _c(V, np.float64)
    B, Hq, d = Q.shape
    _, Hkv, T, W = signs.shape
    m = S.shape[0]
    assert W * 32 == m and Hq % Hkv == 0 and V.shape == (B, Hkv, T, d)
    out = np.empty((B, Hq, d), dtype=np.float64)
    sc = np.empty((B, Hq, T), dtype=np.float64) if want_scores else None
    lib().jlo_decode(B, Hq, Hkv, T, m, d, _ptr(Q, _f64p), _ptr(S, _f64p),
                     _ptr(signs, _u32p), _ptr(norms, _f64p), _ptr(V, _f64p),
                     softmax_scale, _ptr(out, _f64p),
                     _ptr(sc, _f64p) if want_scores else None)
    return out, sc


def decode_state(Q, S, signs, norms, V, softmax_scale: float):
    """Softmax state of decode attention over one part of a context.

    The pages say nothing about splitting a context; this is the plain
    algebra of the softmax.  For a part holding keys t, with logits
    x_t = softmax_scale * s_t (s the estimator, as in ``decode``), returns
    (out [B,Hq,d], lse2 [B,Hq]): the part's own attention output and
    lse2 = log2 sum_t exp(x_t).  Both are unique, whatever running maximum
    an implementation keeps.
    """
    out, sc = decode(Q, S, signs, norms, V, softmax_scale, want_scores=True)
    x = softmax_scale * sc                                  # [B,Hq,T]
    mx = x.max(axis=-1, keepdims=True)
    lse2 = (mx[..., 0] + np.log(np.exp(x - mx).sum(axis=-1))) / math.log(2.0)
    return out, lse2


def merge_states(outs, lse2s):
    """Attention output of a context split into R parts from the parts'
    states (``decode_state``): each part's output weighted by its share
    2^lse2_r / sum_r 2^lse2_r of the softmax mass.  outs [R,...,d],
    lse2s [R,...]."""
    outs = np.asarray(outs, dtype=np.float64)
    lse2s = np.asarray(lse2s, dtype=np.float64)
    top = lse2s.max(axis=0, keepdims=True)
    w = np.exp2(lse2s - top)                                # [R,...]
    return (w[..., None] * outs).sum(axis=0) / w.sum(axis=0)[..., None]


def exact_attention(Q, K, V, softmax_scale: float, want_scores=False):
    """Attention with the unquantized keys (context only)."""
    Q = _c(Q, np.float64)
    K = _c(K, np.float64)
    V = _c(V, np.float64)
    B, Hq, d = Q.shape
    _, Hkv, T, _ = K.shape
    out = np.empty((B, Hq, d), dtype=np.float64)
    sc = np.empty((B, Hq, T), dtype=np.float64) if want_scores else None
    lib().jlo_exact_attention(B, Hq, Hkv, T, d, _ptr(Q, _f64p),
                              _ptr(K, _f64p), _ptr(V, _f64p), softmax_scale,
                              _ptr(out, _f64p),
                              _ptr(sc, _f64p) if want_scores else None)
    return out, sc


# --------------------------------------------------------------------------
# storage arithmetic

def block_effective_bits(b: float, block: float, const_bits: float = 64.0):
    """Bits per number of a block quantizer with per-block constants."""
    return float(lib().jlo_block_effective_bits(b, block, const_bits))


def qjl_bits_per_coordinate(m: int, d: int, norm_bits: int = 16) -> float:
    """Bits per key coordinate of a QJL code: m sign bits + one norm."""
    return float(lib().jlo_qjl_bits_per_coordinate(m, d, norm_bits))


def max_threads() -> int:
    return int(lib().jlo_max_threads())


SQRT_HALF_PI = math.sqrt(math.pi / 2.0)
