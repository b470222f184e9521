"""Conversions and comparison rules shared by the parity tests.

Tolerances (each derived from the arithmetic of the two sides):
  * sketch, sign codes: bit-exact; a code bit may differ only where the float64
    projection satisfies |(S k)_i| < 1e-5 * ||k|| (the GPU accumulates exact
    bf16 x bf16 products in fp32, whose error is far below that band); such
    coordinates are counted and reported.
  * norms: binary16 within 1 ulp (the GPU sums squares in fp32 before rounding
    to binary16, the oracle in float64; the two roundings can straddle a
    binary16 rounding boundary, by at most one step).
  * scores: |gpu - ref| <= 1e-3 * max(|ref|, rms of that head's scores).
  * outputs: |gpu - ref| <= 2e-2 absolute (bf16 outputs), and a tighter
    relative check on each output vector.
"""
import math

import numpy as np
import torch

BAND_REL = 1e-5
SCORE_REL = 1e-3
OUT_ABS = 2e-2


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def u32(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().numpy().view(np.uint32)


def fp16_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().numpy().view(np.uint16)


def code_bits(words: np.ndarray, m: int) -> np.ndarray:
    """[..., m/32] uint32 -> [..., m] 0/1 (LSB first)."""
    w = words.astype(np.uint64)[..., :, None]
    bits = (w >> np.arange(32, dtype=np.uint64)) & 1
    return bits.reshape(*words.shape[:-1], m).astype(np.uint8)


def compare_codes(gpu_words: np.ndarray, ref_words: np.ndarray, band: np.ndarray, m: int):
    """Returns (#differing bits outside the band, #differing bits inside it)."""
    g = code_bits(gpu_words, m)
    r = code_bits(ref_words, m)
    diff = g != r
    inband = band.reshape(diff.shape).astype(bool)
    return int(np.count_nonzero(diff & ~inband)), int(np.count_nonzero(diff & inband))


def fp16_ulp_diff(a_bits: np.ndarray, b_bits: np.ndarray) -> np.ndarray:
    """Distance in binary16 steps between two arrays of non-negative codes."""
    return np.abs(a_bits.astype(np.int64) - b_bits.astype(np.int64))


def score_violations(gpu: np.ndarray, ref: np.ndarray) -> int:
    """Count of scores outside 1e-3 * max(|ref|, rms over the last axis)."""
    rms = np.sqrt(np.mean(ref ** 2, axis=-1, keepdims=True))
    tol = SCORE_REL * np.maximum(np.abs(ref), rms)
    return int(np.count_nonzero(np.abs(gpu - ref) > tol))


def key_match_mask(gpu_words: np.ndarray, ref_words: np.ndarray,
                   gpu_norm_bits: np.ndarray, ref_norm_bits: np.ndarray) -> np.ndarray:
    """[...] bool: keys whose GPU code and binary16 norm equal the oracle's
    bit for bit (code words on the last axis)."""
    same_code = np.all(gpu_words.astype(np.uint32) == ref_words.astype(np.uint32), axis=-1)
    return same_code & (gpu_norm_bits.astype(np.uint16) == ref_norm_bits.astype(np.uint16))


def masked_score_violations(gpu: np.ndarray, ref: np.ndarray, mask: np.ndarray) -> int:
    """score_violations restricted to the entries where ``mask`` is set (the
    rms that scales the tolerance still runs over every key of the row)."""
    rms = np.sqrt(np.mean(ref ** 2, axis=-1, keepdims=True))
    tol = SCORE_REL * np.maximum(np.abs(ref), rms)
    bad = (np.abs(gpu - ref) > tol) & np.broadcast_to(mask, ref.shape)
    return int(np.count_nonzero(bad))


def output_errors(gpu: np.ndarray, ref: np.ndarray):
    """(max abs error, max over vectors of ||err|| / ||ref||)."""
    err = gpu - ref
    mabs = float(np.max(np.abs(err))) if err.size else 0.0
    nrm = np.linalg.norm(ref, axis=-1)
    rel = np.linalg.norm(err, axis=-1) / np.maximum(nrm, 1e-30)
    return mabs, float(np.max(rel)) if rel.size else 0.0


def cuda_available() -> bool:
    return torch.cuda.is_available()


def softmax_scale(d: int) -> float:
    return 1.0 / math.sqrt(d)
