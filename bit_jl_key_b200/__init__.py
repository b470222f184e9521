"""bit_jl_key_b200 -- QJL sign-bit key compression and compressed-key decode
attention on NVIDIA B200 (sm_100a).

This module is a thin ctypes binding over ``libjlkey.so`` (C ABI in
``include/jlkey.h``).  It only marshals torch tensors into pointers, sizes and
the current CUDA stream; every step of the computation runs in the library's
CUDA kernels.  There is no CPU fallback: if the library is missing or a call
fails, an exception is raised.

Functions (same names as the C entry points):
  jl_sketch_init(m, d, seed)            -> S  (bf16 [m, d])
  jl_quantize_keys(K, S)                -> (signs int32 [n, m/32], norms fp16 [n])
  jl_quantize_keys_simt(K, S)           -> same, SIMT-core kernel
  jl_decode_workspace_bytes(B, Hq, Hkv, T, m, d) -> int
  jl_decode_attention(Q, S, signs, norms, V, ...) -> out bf16 [B, Hq, d]
  jl_device_error()                     -> int (0 = no device fault reported)
  jl_turbo_codebook(d, mse_bits)        -> centroids (list of float)
  jl_turbo_rotation_init(d, seed)       -> (Pi bf16 [d, d], Pinv fp32 [d, d])
  jl_turbo_quantize_keys(K, Pi, S, mse_bits) -> (codes int32 [n, words], norms fp16 [n, 2])
  jl_turbo_decode_attention(Q, Pinv, S, codes, norms, V, mse_bits, ...) -> out bf16

Sign codes are returned as torch.int32 tensors holding the uint32 words bit
for bit (torch has no general uint32 arithmetic); word w of a key holds sketch
rows 32w..32w+31, LSB first, bit = 1 iff (S k)_i >= 0.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# JLKEY_LIBRARY may name another build of the same library (e.g. to compare
# two builds of a kernel); by default the in-tree build is loaded.
LIB_PATH = os.environ.get("JLKEY_LIBRARY") or os.path.join(_HERE, "libjlkey.so")

JL_BF16 = 0
JL_F32 = 1
JL_OK = 0
JL_ERR_INVALID_ARG = -1
JL_ERR_UNSUPPORTED = -2
JL_ERR_WORKSPACE = -3
JL_ERR_CUDA = -4
JL_ERR_DEVICE = -5
JL_ERR_SCRATCH_LIMIT = -6
DECODE_STATIC_SCRATCH_BYTES = 16 << 20

EXPORTED = ("jl_status_string", "jl_sketch_init", "jl_quantize_keys",
            "jl_quantize_keys_simt", "jl_decode_workspace_bytes",
            "jl_decode_attention", "jl_device_error", "jl_bf16_from_f64",
            "jl_decode_attention_noalloc", "jl_decode_paged_workspace_bytes",
            "jl_decode_attention_paged", "jl_dequantize_keys", "jl_search_workspace_bytes",
            "jl_search_topk", "jl_turbo_codebook", "jl_turbo_rotation_workspace_bytes",
            "jl_turbo_rotation_init", "jl_turbo_quantize_keys", "jl_turbo_decode_workspace_bytes",
            "jl_turbo_decode_attention", "jl_turbo_decode_paged_workspace_bytes",
            "jl_turbo_decode_attention_paged", "jl_turbo_dequant_basis",
            "jl_turbo_dequantize_keys", "jl_test_drop_copies", "jl_build_flags",
            "jl_decode_attention_state", "jl_merge_attention_states")

# device error codes (jl_device_error)
JL_DERR_TC_WAIT_TIMEOUT = 1
JL_DERR_DECODE_PLAN = 3
JL_DERR_DECODE_WAIT_TIMEOUT = 4
JL_DERR_INDEX = 5
JL_BUILD_INDEX_CHECKS = 1

_lib = None


class JLError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: status {status} ({status_string(status)})")


def load():
    """Load libjlkey.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is missing: build it with `python -m bit_jl_key_b200.build` "
            "(there is no CPU fallback)")
    L = ctypes.CDLL(LIB_PATH)
    vp, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
    L.jl_status_string.restype = ctypes.c_char_p
    L.jl_status_string.argtypes = [i32]
    L.jl_sketch_init.restype = i32
    L.jl_sketch_init.argtypes = [vp, i32, i32, ctypes.c_uint64, vp]
    for name in ("jl_quantize_keys", "jl_quantize_keys_simt"):
        f = getattr(L, name)
        f.restype = i32
        f.argtypes = [vp, i32, i64, i64, vp, i32, i32, vp, vp, vp]
    L.jl_decode_workspace_bytes.restype = sz
    L.jl_decode_workspace_bytes.argtypes = [i32, i32, i32, i64, i32, i32]
    L.jl_decode_attention.restype = i32
    L.jl_decode_attention.argtypes = [vp, i32, vp, vp, vp, vp, i32, i32, i32,
                                      i64, i32, i32, ctypes.c_float, vp, vp,
                                      vp, sz, vp]
    L.jl_decode_attention_state.restype = i32
    L.jl_decode_attention_state.argtypes = list(L.jl_decode_attention.argtypes)
    L.jl_merge_attention_states.restype = i32
    L.jl_merge_attention_states.argtypes = [vp, i32, i64, i32, vp, vp]
    L.jl_decode_attention_noalloc.restype = i32
    L.jl_decode_attention_noalloc.argtypes = [vp, i32, vp, vp, vp, vp, i32, i32,
                                              i32, i64, i32, i32, ctypes.c_float,
                                              vp, vp, vp]
    L.jl_search_workspace_bytes.restype = sz
    L.jl_search_workspace_bytes.argtypes = [i32, i32, i32, i32]
    L.jl_search_topk.restype = i32
    L.jl_search_topk.argtypes = [vp, i32, i32, vp, i32, i32, vp, vp, i64, i32, vp, vp, vp, sz,
                                 vp]
    L.jl_dequantize_keys.restype = i32
    L.jl_dequantize_keys.argtypes = [vp, vp, i64, vp, i32, i32, vp, vp]
    L.jl_decode_paged_workspace_bytes.restype = sz
    L.jl_decode_paged_workspace_bytes.argtypes = [i32, i32, i32, i64, i32, i32]
    L.jl_decode_attention_paged.restype = i32
    L.jl_decode_attention_paged.argtypes = [vp, i32, vp, i32, vp, vp, vp, vp, vp, i32, i32,
                                            vp, i32, vp, i32, i32, i32, i64, i32, i32,
                                            ctypes.c_float, vp, vp, vp, sz, vp]
    L.jl_turbo_codebook.restype = i32
    L.jl_turbo_codebook.argtypes = [i32, i32, vp]
    L.jl_turbo_rotation_workspace_bytes.restype = sz
    L.jl_turbo_rotation_workspace_bytes.argtypes = [i32]
    L.jl_turbo_rotation_init.restype = i32
    L.jl_turbo_rotation_init.argtypes = [vp, vp, i32, ctypes.c_uint64, vp, sz, vp]
    L.jl_turbo_quantize_keys.restype = i32
    L.jl_turbo_quantize_keys.argtypes = [vp, i32, i64, i64, vp, vp, i32, i32, i32, vp, vp, vp]
    L.jl_turbo_decode_workspace_bytes.restype = sz
    L.jl_turbo_decode_workspace_bytes.argtypes = [i32, i32, i32, i64, i32, i32, i32]
    L.jl_turbo_decode_attention.restype = i32
    L.jl_turbo_decode_attention.argtypes = [vp, i32, vp, vp, vp, vp, vp, i32, i32, i32, i64,
                                            i32, i32, i32, ctypes.c_float, vp, vp, vp, sz, vp]
    L.jl_turbo_decode_paged_workspace_bytes.restype = sz
    L.jl_turbo_decode_paged_workspace_bytes.argtypes = [i32, i32, i32, i64, i32, i32, i32]
    L.jl_turbo_decode_attention_paged.restype = i32
    L.jl_turbo_decode_attention_paged.argtypes = [vp, i32, vp, i32, vp, vp, vp, vp, vp, vp, vp, i32,
                                                  i32, vp, i32, vp, i32, i32, i32, i64, i32, i32,
                                                  i32, ctypes.c_float, vp, vp, vp, sz, vp]
    L.jl_turbo_dequant_basis.restype = i32
    L.jl_turbo_dequant_basis.argtypes = [vp, vp, i32, i32, vp, vp]
    L.jl_turbo_dequantize_keys.restype = i32
    L.jl_turbo_dequantize_keys.argtypes = [vp, vp, i64, vp, i32, i32, i32, vp, vp]
    L.jl_device_error.restype = i32
    L.jl_device_error.argtypes = [ctypes.POINTER(i32), vp]
    L.jl_build_flags.restype = i32
    L.jl_build_flags.argtypes = []
    L.jl_test_drop_copies.restype = i32
    L.jl_test_drop_copies.argtypes = [i32, ctypes.c_uint64]
    L.jl_bf16_from_f64.restype = ctypes.c_uint16
    L.jl_bf16_from_f64.argtypes = [ctypes.c_double]
    _lib = L
    return L


def status_string(status: int) -> str:
    return load().jl_status_string(int(status)).decode()


def _check(status: int, where: str):
    if status != JL_OK:
        raise JLError(status, where)


def _stream(t: torch.Tensor | None = None, stream=None):
    if stream is not None:
        return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))
    dev = t.device if t is not None else torch.device("cuda")
    return ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)


def _ptr(t: torch.Tensor | None):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _need_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("libjlkey works on CUDA tensors only (no CPU fallback)")


# --------------------------------------------------------------------------

def jl_sketch_init(m: int, d: int, seed: int = 0, device=None, out=None,
                   stream=None) -> torch.Tensor:
    """The m x d bf16 Gaussian sketch regenerated from ``seed``."""
    if out is None:
        out = torch.empty((m, d), dtype=torch.bfloat16,
                          device=device if device is not None else "cuda")
    _need_cuda(out)
    assert out.dtype == torch.bfloat16 and out.is_contiguous() and out.shape == (m, d)
    _check(load().jl_sketch_init(_ptr(out), m, d, ctypes.c_uint64(seed),
                                 _stream(out, stream)), "jl_sketch_init")
    return out


def _quantize(name, K, S, signs, norms, stream):
    L = load()
    if K.dim() != 2:
        K = K.reshape(-1, K.shape[-1])
    n, d = K.shape
    m = S.shape[0]
    _need_cuda(K, S)
    if K.stride(1) != 1:
        raise ValueError("keys must have unit stride along d")
    if K.dtype == torch.bfloat16:
        kt = JL_BF16
    elif K.dtype == torch.float32:
        kt = JL_F32
    else:
        raise TypeError(f"unsupported key dtype {K.dtype}")
    assert S.dtype == torch.bfloat16 and S.is_contiguous() and S.shape[1] == d
    if signs is None:
        signs = torch.empty((n, m // 32), dtype=torch.int32, device=K.device)
    if norms is None:
        norms = torch.empty((n,), dtype=torch.float16, device=K.device)
    assert signs.dtype == torch.int32 and signs.is_contiguous() and signs.numel() == n * (m // 32)
    assert norms.dtype == torch.float16 and norms.is_contiguous() and norms.numel() == n
    _check(getattr(L, name)(_ptr(K), kt, n, K.stride(0) if n > 0 else d, _ptr(S),
                            m, d, _ptr(signs), _ptr(norms), _stream(K, stream)),
           name)
    return signs, norms


def jl_quantize_keys(K, S, signs=None, norms=None, stream=None):
    """Sign codes and fp16 norms of the rows of K ([..., d], bf16 or fp32)."""
    return _quantize("jl_quantize_keys", K, S, signs, norms, stream)


def jl_quantize_keys_simt(K, S, signs=None, norms=None, stream=None):
    """Same as jl_quantize_keys, computed on the SIMT cores."""
    return _quantize("jl_quantize_keys_simt", K, S, signs, norms, stream)


def jl_dequantize_keys(signs, norms, S, out=None, stream=None):
    """khat = sqrt(pi/2)/m * ||k|| * S^T z for each code: [n, d] bf16."""
    L = load()
    m, d = S.shape
    _need_cuda(signs, norms, S, out)
    assert signs.dtype == torch.int32 and signs.shape[-1] == m // 32
    assert norms.dtype == torch.float16 and S.dtype == torch.bfloat16
    signs2 = signs.reshape(-1, m // 32)
    n = signs2.shape[0]
    assert norms.numel() == n
    for t in (signs2, norms, S):
        if not t.is_contiguous():
            raise ValueError("dequantize inputs must be contiguous")
    if out is None:
        out = torch.empty((n, d), dtype=torch.bfloat16, device=signs.device)
    assert out.dtype == torch.bfloat16 and out.numel() == n * d and out.is_contiguous()
    _check(L.jl_dequantize_keys(_ptr(signs2), _ptr(norms), n, _ptr(S), m, d, _ptr(out),
                                _stream(signs, stream)), "jl_dequantize_keys")
    return out


def jl_search_workspace_bytes(n_queries, m, d, k) -> int:
    return int(load().jl_search_workspace_bytes(n_queries, m, d, k))


def jl_search_topk(Q, S, signs, norms, k, out_index=None, out_scores=None, workspace=None,
                   stream=None):
    """Top-k inner-product search of the queries Q [nq, d] over the index
    (signs [N, m/32] int32, norms [N] fp16).  Returns (index int32 [nq, k],
    scores fp32 [nq, k]), best first."""
    L = load()
    m, d = S.shape
    nq = Q.shape[0]
    _need_cuda(Q, S, signs, norms)
    assert Q.dim() == 2 and Q.shape[1] == d
    assert signs.dtype == torch.int32 and signs.shape[1] == m // 32
    assert norms.dtype == torch.float16 and norms.numel() == signs.shape[0]
    for t in (Q, S, signs, norms):
        if not t.is_contiguous():
            raise ValueError("search inputs must be contiguous")
    qt = JL_F32 if Q.dtype == torch.float32 else JL_BF16
    if out_index is None:
        out_index = torch.empty((nq, k), dtype=torch.int32, device=Q.device)
    if out_scores is None:
        out_scores = torch.empty((nq, k), dtype=torch.float32, device=Q.device)
    need = jl_search_workspace_bytes(nq, m, d, k)
    if workspace is None:
        workspace = torch.empty((max(need, 1),), dtype=torch.uint8, device=Q.device)
    _check(L.jl_search_topk(_ptr(Q), qt, nq, _ptr(S), m, d, _ptr(signs), _ptr(norms),
                            signs.shape[0], k, _ptr(out_index), _ptr(out_scores),
                            _ptr(workspace), workspace.numel(), _stream(Q, stream)),
           "jl_search_topk")
    return out_index, out_scores


def jl_decode_workspace_bytes(B, Hq, Hkv, T, m, d) -> int:
    return int(load().jl_decode_workspace_bytes(B, Hq, Hkv, T, m, d))


def _decode_shapes(Q, S, signs, norms, V, out, scores):
    """Shape, dtype and layout checks shared by the two decode wrappers: the
    library sizes its copies from (B, Hq, Hkv, T, m, d), so a tensor shorter
    than those shapes say would be read past its end.  Returns
    (B, Hq, Hkv, T, m, d, query dtype code)."""
    if Q.dim() != 3 or V.dim() != 4 or S.dim() != 2:
        raise ValueError("Q must be [B, Hq, d], V [B, Hkv, T, d] and S [m, d]")
    B, Hq, d = Q.shape
    Bv, Hkv, T, dv = V.shape
    m = S.shape[0]
    if Q.dtype == torch.float32:
        qt = JL_F32
    elif Q.dtype == torch.bfloat16:
        qt = JL_BF16
    else:
        raise TypeError(f"unsupported query dtype {Q.dtype}")
    if Bv != B or dv != d:
        raise ValueError(f"V {tuple(V.shape)} does not match Q {tuple(Q.shape)}")
    if S.shape != (m, d) or S.dtype != torch.bfloat16:
        raise ValueError(f"S must be bf16 [m, {d}], got {S.dtype} {tuple(S.shape)}")
    if signs.shape != (B, Hkv, T, m // 32) or signs.dtype != torch.int32:
        raise ValueError(f"signs must be int32 {(B, Hkv, T, m // 32)}, got "
                         f"{signs.dtype} {tuple(signs.shape)}")
    if norms.shape != (B, Hkv, T) or norms.dtype != torch.float16:
        raise ValueError(f"norms must be float16 {(B, Hkv, T)}, got "
                         f"{norms.dtype} {tuple(norms.shape)}")
    if V.dtype != torch.bfloat16:
        raise ValueError(f"V must be bf16, got {V.dtype}")
    if out is not None and (out.shape != (B, Hq, d) or out.dtype != torch.bfloat16
                            or not out.is_contiguous()):
        raise ValueError(f"out must be a contiguous bf16 {(B, Hq, d)} tensor")
    if scores is not None and (scores.shape != (B, Hq, T) or scores.dtype != torch.float32
                               or not scores.is_contiguous()):
        raise ValueError(f"scores must be a contiguous float32 {(B, Hq, T)} tensor")
    for t in (Q, S, signs, norms, V):
        if not t.is_contiguous():
            raise ValueError("decode inputs must be contiguous")
    _need_cuda(Q, S, signs, norms, V, out, scores)
    return B, Hq, Hkv, T, m, d, qt


def jl_decode_attention(Q, S, signs, norms, V, softmax_scale=None, out=None,
                        scores=None, want_scores=False, workspace=None,
                        stream=None):
    """One decode step over compressed keys.

    Q [B, Hq, d] (bf16/fp32); signs [B, Hkv, T, m/32] int32; norms [B, Hkv, T]
    fp16; V [B, Hkv, T, d] bf16.  Returns out [B, Hq, d] bf16, or
    (out, scores [B, Hq, T] fp32) when ``want_scores`` (or ``scores`` given).
    """
    L = load()
    B, Hq, Hkv, T, m, d, qt = _decode_shapes(Q, S, signs, norms, V, out, scores)
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.bfloat16, device=Q.device)
    if want_scores and scores is None:
        scores = torch.empty((B, Hq, T), dtype=torch.float32, device=Q.device)
    need = jl_decode_workspace_bytes(B, Hq, Hkv, T, m, d)
    if workspace is None:
        workspace = torch.empty((max(need, 1),), dtype=torch.uint8, device=Q.device)
    _check(L.jl_decode_attention(_ptr(Q), qt, _ptr(S), _ptr(signs), _ptr(norms),
                                 _ptr(V), B, Hq, Hkv, T, m, d,
                                 ctypes.c_float(softmax_scale), _ptr(out),
                                 _ptr(scores), _ptr(workspace),
                                 workspace.numel() * workspace.element_size(),
                                 _stream(Q, stream)),
           "jl_decode_attention")
    if scores is not None:
        return out, scores
    return out


def jl_decode_attention_state(Q, S, signs, norms, V, softmax_scale=None, state=None,
                              scores=None, want_scores=False, workspace=None,
                              stream=None):
    """jl_decode_attention over one part of a context, returning the softmax
    state of every (b, query head) instead of the output: state [B, Hq, d + 2]
    fp32 holding (acc[d], max, sum), for jl_merge_attention_states.  Returns
    state, or (state, scores [B, Hq, T]) when ``want_scores``."""
    L = load()
    B, Hq, Hkv, T, m, d, qt = _decode_shapes(Q, S, signs, norms, V, None, scores)
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(d)
    if state is None:
        state = torch.empty((B, Hq, d + 2), dtype=torch.float32, device=Q.device)
    elif (state.shape != (B, Hq, d + 2) or state.dtype != torch.float32
          or not state.is_contiguous()):
        raise ValueError(f"state must be a contiguous float32 {(B, Hq, d + 2)} tensor")
    _need_cuda(state)
    if want_scores and scores is None:
        scores = torch.empty((B, Hq, T), dtype=torch.float32, device=Q.device)
    need = jl_decode_workspace_bytes(B, Hq, Hkv, T, m, d)
    if workspace is None:
        workspace = torch.empty((max(need, 1),), dtype=torch.uint8, device=Q.device)
    _check(L.jl_decode_attention_state(_ptr(Q), qt, _ptr(S), _ptr(signs), _ptr(norms),
                                       _ptr(V), B, Hq, Hkv, T, m, d,
                                       ctypes.c_float(softmax_scale), _ptr(state),
                                       _ptr(scores), _ptr(workspace),
                                       workspace.numel() * workspace.element_size(),
                                       _stream(Q, stream)),
           "jl_decode_attention_state")
    if scores is not None:
        return state, scores
    return state


def jl_merge_attention_states(states, out=None, stream=None):
    """Attention output [..., d] bf16 from the states [R, ..., d + 2] fp32 of R
    disjoint parts of each row's context (jl_decode_attention_state)."""
    L = load()
    if states.dim() < 2 or states.dtype != torch.float32 or not states.is_contiguous():
        raise ValueError("states must be a contiguous float32 [R, ..., d + 2] tensor")
    R = states.shape[0]
    d = states.shape[-1] - 2
    lead = tuple(states.shape[1:-1])
    rows = 1
    for n in lead:
        rows *= n
    if out is None:
        out = torch.empty(lead + (d,), dtype=torch.bfloat16, device=states.device)
    elif (tuple(out.shape) != lead + (d,) or out.dtype != torch.bfloat16
          or not out.is_contiguous()):
        raise ValueError(f"out must be a contiguous bf16 {lead + (d,)} tensor")
    _need_cuda(states, out)
    _check(L.jl_merge_attention_states(_ptr(states), R, rows, d, _ptr(out),
                                       _stream(states, stream)),
           "jl_merge_attention_states")
    return out


def jl_decode_attention_noalloc(Q, S, signs, norms, V, softmax_scale=None,
                                out=None, scores=None, want_scores=False,
                                stream=None):
    """jl_decode_attention without a workspace, for callers that cannot
    allocate device memory where they call it (plugins inside an engine that
    owns all device memory, latency-critical paths).  The library's static
    device scratch (DECODE_STATIC_SCRATCH_BYTES, held by every GPU that loads
    the library) replaces the workspace; calls must not overlap on a GPU, and
    shapes needing more scratch raise JLError(JL_ERR_SCRATCH_LIMIT).  Output
    tensors passed in are used as given; when ``out``/``scores`` are None this
    wrapper creates them with torch, as it would for any caller."""
    L = load()
    B, Hq, Hkv, T, m, d, qt = _decode_shapes(Q, S, signs, norms, V, out, scores)
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.bfloat16, device=Q.device)
    if want_scores and scores is None:
        scores = torch.empty((B, Hq, T), dtype=torch.float32, device=Q.device)
    _check(L.jl_decode_attention_noalloc(_ptr(Q), qt, _ptr(S), _ptr(signs),
                                         _ptr(norms), _ptr(V), B, Hq, Hkv, T,
                                         m, d, ctypes.c_float(softmax_scale),
                                         _ptr(out), _ptr(scores),
                                         _stream(Q, stream)),
           "jl_decode_attention_noalloc")
    if scores is not None:
        return out, scores
    return out


def jl_decode_paged_workspace_bytes(B, Hq, Hkv, max_len, m, d) -> int:
    return int(load().jl_decode_paged_workspace_bytes(B, Hq, Hkv, max_len, m, d))


def jl_decode_attention_paged(Q, S, sign_pages, norm_pages, value_pages, block_table,
                              seq_lens, max_len, K_new=None, V_new=None,
                              softmax_scale=None, out=None, scores=None,
                              want_scores=False, workspace=None, stream=None):
    """One decode step over a paged compressed cache of ragged sequences.

    Q [B, Hq, d]; pools sign_pages int32 [P_n, Hkv, P, m/32], norm_pages fp16
    [P_n, Hkv, P], value_pages bf16 [P_n, Hkv, P, d]; block_table int32
    [B, max_pages]; seq_lens int32 [B] (device, not modified).  With K_new
    [B, Hkv, d] and V_new [B, Hkv, d] the new key of every sequence is
    quantized and stored at position seq_lens[b] first, and attention covers
    seq_lens[b] + 1 keys.  Returns out [B, Hq, d] (and scores [B, Hq, max_len]).
    """
    L = load()
    B, Hq, d = Q.shape
    num_pages, Hkv, P, W = sign_pages.shape
    m = W * 32
    _need_cuda(Q, S, sign_pages, norm_pages, value_pages, block_table, seq_lens, K_new, V_new)
    assert S.shape == (m, d) and S.dtype == torch.bfloat16
    assert norm_pages.shape == (num_pages, Hkv, P) and norm_pages.dtype == torch.float16
    assert value_pages.shape == (num_pages, Hkv, P, d) and value_pages.dtype == torch.bfloat16
    assert block_table.dtype == torch.int32 and block_table.dim() == 2 and block_table.shape[0] == B
    assert seq_lens.dtype == torch.int32 and seq_lens.shape == (B,)
    for t in (Q, S, sign_pages, norm_pages, value_pages, block_table, seq_lens, K_new, V_new):
        if t is not None and not t.is_contiguous():
            raise ValueError("paged decode inputs must be contiguous")
    qt = JL_F32 if Q.dtype == torch.float32 else JL_BF16
    kt = JL_BF16
    if K_new is not None:
        assert K_new.shape == (B, Hkv, d) and V_new is not None and V_new.shape == (B, Hkv, d)
        kt = JL_F32 if K_new.dtype == torch.float32 else JL_BF16
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.bfloat16, device=Q.device)
    if want_scores and scores is None:
        scores = torch.empty((B, Hq, max_len), dtype=torch.float32, device=Q.device)
    need = jl_decode_paged_workspace_bytes(B, Hq, Hkv, max_len, m, d)
    if workspace is None:
        workspace = torch.empty((max(need, 1),), dtype=torch.uint8, device=Q.device)
    _check(L.jl_decode_attention_paged(
        _ptr(Q), qt, _ptr(K_new), kt, _ptr(V_new), _ptr(S), _ptr(sign_pages),
        _ptr(norm_pages), _ptr(value_pages), num_pages, P, _ptr(block_table),
        block_table.shape[1], _ptr(seq_lens), B, Hq, Hkv, max_len, m, d,
        ctypes.c_float(softmax_scale), _ptr(out), _ptr(scores), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(Q, stream)),
        "jl_decode_attention_paged")
    if scores is not None:
        return out, scores
    return out


def jl_device_error(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device error word."""
    code = ctypes.c_int(0)
    st = load().jl_device_error(ctypes.byref(code), _stream(None, stream))
    if st not in (JL_OK, JL_ERR_DEVICE):
        raise JLError(st, "jl_device_error")
    return int(code.value)


def jl_test_drop_copies(enable: bool, wait_limit_ns: int = 0):
    """Test hook: make the quantizer's and decode scorer's next launches start
    no copy, with every wait bounded by ``wait_limit_ns`` (0 = default), so
    that their bounded waits run out; ``jl_test_drop_copies(False)`` restores
    normal operation.  See include/jlkey.h."""
    _check(load().jl_test_drop_copies(1 if enable else 0, ctypes.c_uint64(wait_limit_ns)),
           "jl_test_drop_copies")


def jl_build_flags() -> int:
    """JL_BUILD_* bits of the loaded library (JL_BUILD_INDEX_CHECKS for the
    index-checking debug build)."""
    return int(load().jl_build_flags())


def jl_bf16_from_f64(x: float) -> int:
    return int(load().jl_bf16_from_f64(float(x)))


# --------------------------------------------------------------------------
# TurboQuant-prod keys

def turbo_code_words(mse_bits: int, m: int, d: int) -> int:
    """uint32 words of one key's code: mse_bits cell planes of d bits, then m
    residual sign bits."""
    return (mse_bits * d + m) // 32


def jl_turbo_codebook(d: int, mse_bits: int):
    """The 2^mse_bits Lloyd-Max centroids of the rotated-coordinate density
    (ascending, as float), computed by the library on the host."""
    L = load()
    buf = (ctypes.c_float * (1 << mse_bits))()
    _check(L.jl_turbo_codebook(d, mse_bits, ctypes.cast(buf, ctypes.c_void_p)),
           "jl_turbo_codebook")
    return [float(v) for v in buf]


def jl_turbo_rotation_workspace_bytes(d: int) -> int:
    return int(load().jl_turbo_rotation_workspace_bytes(d))


def jl_turbo_rotation_init(d: int, seed: int, device=None, stream=None):
    """(Pi bf16 [d, d], Pinv fp32 [d, d]) regenerated from ``seed``."""
    L = load()
    dev = device if device is not None else "cuda"
    Pi = torch.empty((d, d), dtype=torch.bfloat16, device=dev)
    Pinv = torch.empty((d, d), dtype=torch.float32, device=dev)
    ws = torch.empty((max(jl_turbo_rotation_workspace_bytes(d), 1),), dtype=torch.uint8,
                     device=dev)
    _check(L.jl_turbo_rotation_init(_ptr(Pi), _ptr(Pinv), d, ctypes.c_uint64(seed), _ptr(ws),
                                    ws.numel(), _stream(Pi, stream)), "jl_turbo_rotation_init")
    return Pi, Pinv


def jl_turbo_quantize_keys(K, Pi, S, mse_bits: int, codes=None, norms=None, stream=None):
    """TurboQuant-prod codes (int32 [n, words]) and norms (fp16 [n, 2]:
    ||k||, ||rt||) of the rows of K ([..., d] bf16)."""
    L = load()
    if K.dim() != 2:
        K = K.reshape(-1, K.shape[-1])
    n, d = K.shape
    m = S.shape[0]
    _need_cuda(K, Pi, S)
    if K.stride(1) != 1:
        raise ValueError("keys must have unit stride along d")
    if K.dtype != torch.bfloat16:
        raise TypeError("the TurboQuant quantizer takes bf16 keys")
    assert Pi.dtype == torch.bfloat16 and Pi.is_contiguous() and Pi.shape == (d, d)
    assert S.dtype == torch.bfloat16 and S.is_contiguous() and S.shape[1] == d
    words = turbo_code_words(mse_bits, m, d)
    if codes is None:
        codes = torch.empty((n, words), dtype=torch.int32, device=K.device)
    if norms is None:
        norms = torch.empty((n, 2), dtype=torch.float16, device=K.device)
    assert codes.dtype == torch.int32 and codes.is_contiguous() and codes.numel() == n * words
    assert norms.dtype == torch.float16 and norms.is_contiguous() and norms.numel() == 2 * n
    _check(L.jl_turbo_quantize_keys(_ptr(K), JL_BF16, n, K.stride(0) if n > 0 else d, _ptr(Pi),
                                    _ptr(S), m, d, mse_bits, _ptr(codes), _ptr(norms),
                                    _stream(K, stream)), "jl_turbo_quantize_keys")
    return codes, norms


def jl_turbo_dequant_basis(Pinv, S, out=None, stream=None):
    """R = [Pinv | Pinv S^T] as binary16 [d, d + m]: the reconstruction matrix
    of jl_turbo_dequantize_keys."""
    L = load()
    m, d = S.shape
    _need_cuda(Pinv, S, out)
    assert Pinv.dtype == torch.float32 and Pinv.shape == (d, d) and Pinv.is_contiguous()
    assert S.dtype == torch.bfloat16 and S.is_contiguous()
    if out is None:
        out = torch.empty((d, d + m), dtype=torch.float16, device=S.device)
    assert out.dtype == torch.float16 and out.shape == (d, d + m) and out.is_contiguous()
    _check(L.jl_turbo_dequant_basis(_ptr(Pinv), _ptr(S), m, d, _ptr(out), _stream(S, stream)),
           "jl_turbo_dequant_basis")
    return out


def jl_turbo_dequantize_keys(codes, norms, basis, mse_bits: int, out=None, stream=None):
    """khat = ||k|| Pi^{-1} (c[cell] + sqrt(pi/2)/m ||r|| S^T z) for each
    TurboQuant-prod code (codes int32 [..., words], norms fp16 [..., 2],
    basis from jl_turbo_dequant_basis): [n, d] bf16."""
    L = load()
    d = basis.shape[0]
    m = basis.shape[1] - d
    words = turbo_code_words(mse_bits, m, d)
    _need_cuda(codes, norms, basis, out)
    assert codes.dtype == torch.int32 and codes.shape[-1] == words
    assert norms.dtype == torch.float16 and norms.shape[-1] == 2
    assert basis.dtype == torch.float16
    codes2 = codes.reshape(-1, words)
    n = codes2.shape[0]
    assert norms.numel() == 2 * n
    for t in (codes2, norms, basis):
        if not t.is_contiguous():
            raise ValueError("dequantize inputs must be contiguous")
    if out is None:
        out = torch.empty((n, d), dtype=torch.bfloat16, device=codes.device)
    assert out.dtype == torch.bfloat16 and out.numel() == n * d and out.is_contiguous()
    _check(L.jl_turbo_dequantize_keys(_ptr(codes2), _ptr(norms), n, _ptr(basis), m, d, mse_bits,
                                      _ptr(out), _stream(codes, stream)),
           "jl_turbo_dequantize_keys")
    return out


def jl_turbo_decode_workspace_bytes(B, Hq, Hkv, T, m, d, mse_bits) -> int:
    return int(load().jl_turbo_decode_workspace_bytes(B, Hq, Hkv, T, m, d, mse_bits))


def jl_turbo_decode_attention(Q, Pinv, S, codes, norms, V, mse_bits, softmax_scale=None,
                              out=None, scores=None, want_scores=False, workspace=None,
                              stream=None):
    """One decode step over TurboQuant-prod keys.

    Q [B, Hq, d] (bf16/fp32); codes [B, Hkv, T, words] int32; norms
    [B, Hkv, T, 2] fp16; V [B, Hkv, T, d] bf16.  Returns out [B, Hq, d] bf16,
    or (out, scores [B, Hq, T] fp32) when ``want_scores`` (or ``scores``)."""
    L = load()
    B, Hq, d = Q.shape
    m = S.shape[0]
    Hkv, T = V.shape[1], V.shape[2]
    words = turbo_code_words(mse_bits, m, d)
    _need_cuda(Q, Pinv, S, codes, norms, V, out, scores)
    assert codes.dtype == torch.int32 and codes.shape == (B, Hkv, T, words)
    assert norms.dtype == torch.float16 and norms.shape == (B, Hkv, T, 2)
    assert V.dtype == torch.bfloat16 and V.shape == (B, Hkv, T, d)
    assert Pinv.dtype == torch.float32 and Pinv.shape == (d, d)
    for t in (Q, Pinv, S, codes, norms, V):
        if not t.is_contiguous():
            raise ValueError("decode inputs must be contiguous")
    qt = JL_F32 if Q.dtype == torch.float32 else JL_BF16
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.bfloat16, device=Q.device)
    if want_scores and scores is None:
        scores = torch.empty((B, Hq, T), dtype=torch.float32, device=Q.device)
    need = jl_turbo_decode_workspace_bytes(B, Hq, Hkv, T, m, d, mse_bits)
    if workspace is None:
        workspace = torch.empty((max(need, 1),), dtype=torch.uint8, device=Q.device)
    _check(L.jl_turbo_decode_attention(_ptr(Q), qt, _ptr(Pinv), _ptr(S), _ptr(codes),
                                       _ptr(norms), _ptr(V), B, Hq, Hkv, T, m, d, mse_bits,
                                       ctypes.c_float(softmax_scale), _ptr(out), _ptr(scores),
                                       _ptr(workspace), workspace.numel(), _stream(Q, stream)),
           "jl_turbo_decode_attention")
    return (out, scores) if scores is not None else out


def jl_turbo_decode_paged_workspace_bytes(B, Hq, Hkv, max_len, m, d, mse_bits) -> int:
    return int(load().jl_turbo_decode_paged_workspace_bytes(B, Hq, Hkv, max_len, m, d, mse_bits))


def jl_turbo_decode_attention_paged(Q, Pinv, S, code_pages, norm_pages, value_pages, block_table,
                                    seq_lens, max_len, mse_bits, Pi=None, K_new=None, V_new=None,
                                    softmax_scale=None, out=None, scores=None, want_scores=False,
                                    workspace=None, stream=None):
    """One decode step over a paged TurboQuant-prod cache of ragged sequences.

    Pools: code_pages int32 [P_n, Hkv, P, words], norm_pages fp16 [P_n, Hkv,
    P, 2], value_pages bf16 [P_n, Hkv, P, d].  With K_new / V_new [B, Hkv, d]
    (and the rotation Pi) the new key of every sequence is quantized and stored
    at position seq_lens[b] first.  Returns out [B, Hq, d] (and scores)."""
    L = load()
    B, Hq, d = Q.shape
    num_pages, Hkv, P, words = code_pages.shape
    m = S.shape[0]
    assert words == turbo_code_words(mse_bits, m, d)
    _need_cuda(Q, Pinv, S, code_pages, norm_pages, value_pages, block_table, seq_lens, K_new,
               V_new, Pi)
    assert norm_pages.shape == (num_pages, Hkv, P, 2) and norm_pages.dtype == torch.float16
    assert value_pages.shape == (num_pages, Hkv, P, d) and value_pages.dtype == torch.bfloat16
    assert block_table.dtype == torch.int32 and block_table.dim() == 2 and block_table.shape[0] == B
    assert seq_lens.dtype == torch.int32 and seq_lens.shape == (B,)
    for t in (Q, Pinv, S, code_pages, norm_pages, value_pages, block_table, seq_lens, K_new, V_new,
              Pi):
        if t is not None and not t.is_contiguous():
            raise ValueError("paged decode inputs must be contiguous")
    qt = JL_F32 if Q.dtype == torch.float32 else JL_BF16
    kt = JL_BF16
    if K_new is not None:
        assert K_new.shape == (B, Hkv, d) and V_new is not None and V_new.shape == (B, Hkv, d)
        assert Pi is not None and Pi.shape == (d, d) and Pi.dtype == torch.bfloat16
        kt = JL_F32 if K_new.dtype == torch.float32 else JL_BF16
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.bfloat16, device=Q.device)
    if want_scores and scores is None:
        scores = torch.empty((B, Hq, max_len), dtype=torch.float32, device=Q.device)
    need = jl_turbo_decode_paged_workspace_bytes(B, Hq, Hkv, max_len, m, d, mse_bits)
    if workspace is None:
        workspace = torch.empty((max(need, 1),), dtype=torch.uint8, device=Q.device)
    _check(L.jl_turbo_decode_attention_paged(
        _ptr(Q), qt, _ptr(K_new), kt, _ptr(V_new), _ptr(Pi), _ptr(Pinv), _ptr(S),
        _ptr(code_pages), _ptr(norm_pages), _ptr(value_pages), num_pages, P, _ptr(block_table),
        block_table.shape[1], _ptr(seq_lens), B, Hq, Hkv, max_len, m, d, mse_bits,
        ctypes.c_float(softmax_scale), _ptr(out), _ptr(scores), _ptr(workspace),
        workspace.numel(), _stream(Q, stream)), "jl_turbo_decode_attention_paged")
    return (out, scores) if scores is not None else out
