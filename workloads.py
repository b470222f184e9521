"""Seeded synthetic inputs for the QJL key-compression workloads.

This module is shared by the tests, the smoke check and the bench, and is the
only thing the CUDA path and the CPU oracle have in common.  It holds no step
of the method: it only draws keys, values and queries with the shapes and
distributions of the five workloads below and records how it drew them.

Workloads (keys/values/queries are synthetic; there are no model weights):
  single   1 head, d=128, m=256, 1024 fp32 keys and 1 fp32 query N(0,1);
           values N(0,1) stored as bf16; quantize + one decode step.
  gqa      GQA decode: batch 8, 32 query heads / 8 KV heads, d=128, m=256,
           context 32768; bf16 keys N(0,1) with 4 outlier channels x10;
           bf16 values N(0,1); one query token per sequence.
  long     MHA decode: batch 1, 32 heads, d=128, m=256, context 131072; bf16
           keys k_t = r_t g_t with g_t ~ N(0, I) and r_t ~ lognormal(0, 0.5);
           bf16 values N(0,1).
  prefill  quantization of 65536 tokens x 32 layers x 8 KV heads, d=128,
           m=256; bf16 keys N(0,1) with 4 outlier channels x10.
  sweep    m in {64,128,256,512} x d in {64,128}; batch 16, 32 heads MHA,
           context 16384; bf16 keys and values N(0,1).
  paged-gqa  serving step of the gqa shapes over a paged cache: batch 8,
           32 / 8 heads, d=128, m=256; sequence lengths uniform in
           [16384, 32767) plus the appended key (bound 32768); pages of 64
           tokens assigned in a shuffled order; cache contents drawn as for
           gqa.
  dequant-gqa  the gqa cache's 2,097,152 codes (m=256) and norms turned back
           into bf16 keys of d=128 (codes made from gqa's keys).
  search   top-10 inner-product search of 128 bf16 N(0,1) queries over an index
           of 8,388,608 N(0,1) vectors (d=128) kept as QJL codes (m=256).
  turbo-gqa  the gqa decode step with TurboQuant-prod keys: 2-bit cells of
           the rotated key (rotation seed 1) plus QJL on the residual with a
           128-row sketch (3 bits per coordinate plus two binary16 norms).
  turbo-paged-gqa  the paged-gqa serving step with TurboQuant-prod keys.
  turbo-dequant-gqa  the turbo-gqa cache's 2,097,152 TurboQuant-prod codes
           (2-bit cells, m=128) and norm pairs turned back into bf16 keys.
  turbo-gqa-d64  turbo-gqa with 64-dimension heads: d = m = 64 (keys drawn
           as gqa's, with d = 64).

Recipe details that the workload descriptions leave open:
  * the sketch seed is 0 for every workload;
  * data seeds: workload index i and sequence g (the position of a batch
    row in the global batch) give torch generator seeds
    1000*i + k + 1000003*g with k in {0: keys, 1: values, 2: queries,
    4: per-token norms, 5: sequence length, 7: appended key, 8: appended
    value}; k = 3 (outlier channels) and k = 6 (page order) are drawn once
    per workload (page order: per rank's pool);
  * sharding: under data parallelism rank r holds sequences
    [r*B, (r+1)*B) of the global batch (``shard``), so the ranks' batches
    are distinct and together are exactly the global batch of B*world
    sequences;
  * outlier channels: the first 4 entries of a seeded permutation of range(d);
  * queries are N(0,1) in the key dtype, scaled by ``q_scale`` (default 1);
  * softmax scale 1/sqrt(d).
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    index: int              # selects the data seeds
    B: int                  # batch
    Hq: int                 # query heads
    Hkv: int                # KV heads
    T: int                  # context length (keys per (b, kv-head))
    d: int                  # head dimension
    m: int                  # sketch rows
    key_dtype: torch.dtype  # dtype keys and queries are stored in
    outliers: int = 0       # number of outlier channels scaled by 10
    lognormal_sigma: float = 0.0  # per-token norm spread (0 = none)
    sketch_seed: int = 0
    first_seq: int = 0      # global index of this batch's first sequence

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def n_keys(self) -> int:
        return self.B * self.Hkv * self.T

    @property
    def softmax_scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


SINGLE = Workload("single", 1, 1, 1, 1, 1024, 128, 256, torch.float32)
GQA = Workload("gqa", 2, 8, 32, 8, 32768, 128, 256, torch.bfloat16, outliers=4)
LONG = Workload("long", 3, 1, 32, 32, 131072, 128, 256, torch.bfloat16,
                lognormal_sigma=0.5)
# prefill: 65536 tokens x 32 layers x 8 KV heads, laid out as B=32 layers,
# Hkv=8 heads, T=65536 tokens (no queries; quantization only)
PREFILL = Workload("prefill", 4, 32, 8, 8, 65536, 128, 256, torch.bfloat16,
                   outliers=4)
SWEEP_BASE = Workload("sweep", 5, 16, 32, 32, 16384, 128, 256, torch.bfloat16)
SWEEP_M = (64, 128, 256, 512)
SWEEP_D = (64, 128)

# paged-gqa: T is the length bound (max_len) of the paged cache
PAGED_GQA = Workload("paged-gqa", 6, 8, 32, 8, 32768, 128, 256, torch.bfloat16,
                     outliers=4)
PAGE_TOKENS = 64

# dequant-gqa: the codes of the gqa cache turned back into bf16 keys
DEQUANT_GQA = GQA.with_(name="dequant-gqa")

# search: 128 queries against an index of 8,388,608 vectors (as keys of one
# sequence: B = Hkv = 1, T = index size; Hq = queries)
SEARCH = Workload("search", 7, 1, 128, 1, 8388608, 128, 256, torch.bfloat16)
# TurboQuant-prod decode over the gqa cache: the same keys, values and
# queries, cells of 2 bits per rotated coordinate, a 128-row residual sketch
# (seed 0) and the rotation of seed TURBO_ROTATION_SEED
TURBO_GQA = GQA.with_(name="turbo-gqa", m=128)
TURBO_MSE_BITS = 2
TURBO_ROTATION_SEED = 1
# the paged serving step of paged-gqa with TurboQuant-prod keys (same data)
TURBO_PAGED_GQA = PAGED_GQA.with_(name="turbo-paged-gqa", m=128)
# the turbo-gqa cache's codes turned back into bf16 keys (same data)
TURBO_DEQUANT_GQA = TURBO_GQA.with_(name="turbo-dequant-gqa")
# turbo-gqa with 64-dimension heads (one residual bit per coordinate: m = d)
TURBO_GQA_D64 = TURBO_GQA.with_(name="turbo-gqa-d64", d=64, m=64)
SEARCH_K = 10

ALL = {w.name: w for w in (SINGLE, GQA, LONG, PREFILL, SWEEP_BASE, PAGED_GQA, DEQUANT_GQA,
                           SEARCH, TURBO_GQA, TURBO_PAGED_GQA, TURBO_DEQUANT_GQA,
                           TURBO_GQA_D64)}


def sweep_points():
    return [SWEEP_BASE.with_(m=m, d=d) for d in SWEEP_D for m in SWEEP_M]


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


SEQ_SEED_STRIDE = 1000003


def _seq_gen(w: Workload, kind: int, b: int, device) -> torch.Generator:
    """Generator of draw ``kind`` for batch row b (global sequence
    w.first_seq + b)."""
    return _gen(device, 1000 * w.index + kind + SEQ_SEED_STRIDE * (w.first_seq + b))


def shard(w: Workload, rank: int) -> Workload:
    """Rank ``rank``'s batch under data parallelism: the B sequences starting
    at global sequence rank*B (weak scaling: every rank holds B sequences)."""
    return w.with_(first_seq=w.first_seq + rank * w.B)


def outlier_channels(w: Workload) -> torch.Tensor:
    if w.outliers == 0:
        return torch.empty(0, dtype=torch.long)
    perm = torch.randperm(w.d, generator=_gen("cpu", 1000 * w.index + 3))
    return perm[: w.outliers].sort().values


def _fill_normal(out: torch.Tensor, gen: torch.Generator, rows_per_chunk: int,
                 scale_cols: torch.Tensor | None, row_scale=None):
    """Fill a [rows, d] view with N(0,1) draws chunk by chunk (bounded temp)."""
    rows, d = out.shape
    for r0 in range(0, rows, rows_per_chunk):
        r1 = min(rows, r0 + rows_per_chunk)
        x = torch.randn((r1 - r0, d), generator=gen, device=out.device,
                        dtype=torch.float32)
        if scale_cols is not None and scale_cols.numel():
            x[:, scale_cols.to(out.device)] *= 10.0
        if row_scale is not None:
            x *= row_scale[r0:r1, None].to(out.device)
        out[r0:r1].copy_(x)


def keys(w: Workload, device="cpu", rows_per_chunk: int = 1 << 20):
    """Keys [B, Hkv, T, d] in w.key_dtype (each sequence from its own seed)."""
    K = torch.empty((w.B, w.Hkv, w.T, w.d), dtype=w.key_dtype, device=device)
    cols = outlier_channels(w)
    for b in range(w.B):
        flat = K[b].view(-1, w.d)
        row_scale = None
        if w.lognormal_sigma > 0:
            z = torch.randn(flat.shape[0], generator=_seq_gen(w, 4, b, device),
                            device=device, dtype=torch.float32)
            row_scale = torch.exp(w.lognormal_sigma * z)
        _fill_normal(flat, _seq_gen(w, 0, b, device), rows_per_chunk, cols, row_scale)
    return K


def values(w: Workload, device="cpu", rows_per_chunk: int = 1 << 20):
    """Values [B, Hkv, T, d] in bf16 (fp32 draws rounded to bf16)."""
    V = torch.empty((w.B, w.Hkv, w.T, w.d), dtype=torch.bfloat16, device=device)
    for b in range(w.B):
        _fill_normal(V[b].view(-1, w.d), _seq_gen(w, 1, b, device), rows_per_chunk, None)
    return V


def queries(w: Workload, device="cpu", q_scale: float = 1.0):
    """One query token per (b, query head): [B, Hq, d] in w.key_dtype."""
    Q = torch.empty((w.B, w.Hq, w.d), dtype=w.key_dtype, device=device)
    for b in range(w.B):
        q = torch.randn((w.Hq, w.d), generator=_seq_gen(w, 2, b, device), device=device,
                        dtype=torch.float32) * q_scale
        Q[b].copy_(q)
    return Q


def random_keys(n: int, d: int, seed: int, dtype=torch.bfloat16, device="cpu",
                scale: float = 1.0):
    """Plain N(0, scale^2) keys [n, d] for edge-case tests."""
    x = torch.randn((n, d), generator=_gen(device, seed), device=device,
                    dtype=torch.float32) * scale
    return x.to(dtype)


def paged_layout(w: Workload, page_tokens: int = PAGE_TOKENS, spare_pages: int = 16):
    """Sequence lengths and a shuffled block table for a paged cache.

    Lengths are uniform in [T/2, T-1) so that the appended key still fits the
    bound T (sequence g's length from its own seed); sequence b owns
    ceil((len_b + 1) / page_tokens) pages, taken from a seeded permutation of
    the pool.  Returns (lens int32 [B], block_table int32 [B, max_pages] with
    -1 in unused entries, num_pages).
    """
    lens = torch.cat([torch.randint(w.T // 2, w.T - 1, (1,), generator=_seq_gen(w, 5, b, "cpu"),
                                    dtype=torch.int64) for b in range(w.B)])
    per_seq = [-(-(int(L) + 1) // page_tokens) for L in lens]
    max_pages = -(-w.T // page_tokens)
    num_pages = sum(per_seq) + spare_pages
    perm = torch.randperm(num_pages, generator=_gen("cpu", 1000 * w.index + 6 +
                                                     SEQ_SEED_STRIDE * w.first_seq))
    table = torch.full((w.B, max_pages), -1, dtype=torch.int32)
    k = 0
    for b, n in enumerate(per_seq):
        table[b, :n] = perm[k:k + n].to(torch.int32)
        k += n
    return lens.to(torch.int32), table, num_pages


def new_tokens(w: Workload, device="cpu"):
    """The key and value each sequence appends in a decode step: [B, Hkv, d]
    each, drawn like the cache's keys (outlier channels included) and values."""
    K = torch.empty((w.B, w.Hkv, w.d), dtype=w.key_dtype, device=device)
    V = torch.empty((w.B, w.Hkv, w.d), dtype=torch.bfloat16, device=device)
    cols = outlier_channels(w)
    for b in range(w.B):
        _fill_normal(K[b], _seq_gen(w, 7, b, device), 1 << 20, cols)
        _fill_normal(V[b], _seq_gen(w, 8, b, device), 1 << 20, None)
    return K, V
