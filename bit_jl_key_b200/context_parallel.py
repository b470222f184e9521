"""Decode attention over a context split across ranks (one process per GPU).

Every rank holds a contiguous slice of each sequence's keys (its codes, norms
and values, quantized where they live) and the same queries.  A decode step
is then:

1. ``jl_decode_attention_state`` over the local slice: one softmax state
   (acc[d], max, sum) per (sequence, query head), B x Hq x (d + 2) fp32;
2. one all-gather of those states (16.6 KB per rank for one sequence of 32
   heads at d = 128);
3. ``jl_merge_attention_states`` on every rank: the log-sum-exp merge of the
   ranks' states into the bf16 output.

Softmax over a union of disjoint key sets is exactly the merge of the sets'
states, so the result does not depend on how the keys are split.  The
exchange is a few kilobytes, bound by launch latency rather than by NVLink
bandwidth, so it goes through the process group's all-gather (NCCL on GPUs,
gloo on the host) and is not fused into the kernels.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import jl_decode_attention_state, jl_merge_attention_states


def context_range(T: int, world: int, rank: int) -> tuple[int, int]:
    """Keys [t0, t1) of a T-key context that rank ``rank`` of ``world`` holds:
    contiguous slices whose sizes differ by at most one, in rank order.  Every
    rank needs at least one key (a softmax over no keys is undefined)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a world of {world}")
    if T < world:
        raise ValueError(f"a context of {T} keys cannot give each of {world} ranks a key")
    base, extra = divmod(T, world)
    t0 = rank * base + min(rank, extra)
    return t0, t0 + base + (1 if rank < extra else 0)


def gather_states(state: torch.Tensor, group=None) -> torch.Tensor:
    """All ranks' states stacked in rank order: [world, *state.shape].  Every
    rank of ``group`` must call it with a state of the same shape.  Without
    an initialised process group the caller is the only rank."""
    if not (dist.is_available() and dist.is_initialized()):
        return state.unsqueeze(0)
    world = dist.get_world_size(group)
    flat = state.contiguous().reshape(-1)
    out = torch.empty((world * flat.numel(),), dtype=state.dtype, device=state.device)
    dist.all_gather_into_tensor(out, flat, group=group)
    return out.view((world,) + tuple(state.shape))


def decode_context_parallel(Q, S, signs, norms, V, softmax_scale=None, group=None,
                            out=None, workspace=None, stream=None):
    """One decode step over a context split across the ranks of ``group``.

    Q [B, Hq, d] and S are the same on every rank; signs [B, Hkv, T_r, m/32],
    norms [B, Hkv, T_r] and V [B, Hkv, T_r, d] hold this rank's slice
    (T_r >= 1, may differ between ranks).  Returns out [B, Hq, d] bf16, the
    same on every rank."""
    state = jl_decode_attention_state(Q, S, signs, norms, V, softmax_scale,
                                      workspace=workspace, stream=stream)
    return jl_merge_attention_states(gather_states(state, group), out=out, stream=stream)
