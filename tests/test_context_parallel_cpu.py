"""Host logic of the context-split decode on CPU (gloo).

With a context split across ranks, each rank decodes its own slice of every
sequence to softmax states and the ranks all-gather them before the merge.
Here the ranks compute their slices' states with the oracle, exchange them
through ``context_parallel.gather_states`` over gloo, merge them with the
oracle's merge, and must reproduce the oracle's decode over the whole
context: that checks the slicing (disjoint, covering, in rank order) and the
gather's rank order.  The GPU kernels of the same steps are tested in
``test_gpu_context_parallel.py``.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from bit_jl_key_b200.context_parallel import context_range

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("T", [1, 2, 3, 7, 8, 100, 131072, 131075])
@pytest.mark.parametrize("world", [1, 2, 3, 8])
def test_context_range_covers_in_rank_order(T, world):
    if T < world:
        with pytest.raises(ValueError):
            context_range(T, world, 0)
        return
    ranges = [context_range(T, world, r) for r in range(world)]
    assert ranges[0][0] == 0 and ranges[-1][1] == T
    for (a0, a1), (b0, b1) in zip(ranges[:-1], ranges[1:]):
        assert a1 == b0
    sizes = [b - a for a, b in ranges]
    assert min(sizes) >= 1 and max(sizes) - min(sizes) <= 1


def test_context_range_rejects_bad_rank():
    with pytest.raises(ValueError):
        context_range(10, 2, 2)
    with pytest.raises(ValueError):
        context_range(10, 0, 0)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(B, Hq, Hkv, T, m, d):
    import oracle
    rng = np.random.default_rng(31)
    S = rng.standard_normal((m, d))
    K = rng.standard_normal((B * Hkv * T, d)) * 1.5
    signs, norms, _, _ = oracle.quantize(K, S)
    V = rng.standard_normal((B, Hkv, T, d))
    Q = rng.standard_normal((B, Hq, d)) * 2.0
    return Q, S, signs.reshape(B, Hkv, T, m // 32), norms.reshape(B, Hkv, T), V


SHAPE = (2, 4, 2, 37, 64, 16)   # B, Hq, Hkv, T (ragged over 2 or 3 ranks), m, d
SCALE = 0.8


def _worker(rank, world, port, out_q):
    sys.path.insert(0, ROOT)
    import oracle
    from bit_jl_key_b200.context_parallel import gather_states
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        Q, S, signs, norms, V = _inputs(*SHAPE)
        t0, t1 = context_range(SHAPE[3], world, rank)
        o, lse2 = oracle.decode_state(Q, S, signs[:, :, t0:t1], norms[:, :, t0:t1],
                                      V[:, :, t0:t1], SCALE)
        st = torch.from_numpy(np.concatenate([o, lse2[..., None]], axis=-1))
        allst = gather_states(st).numpy()
        merged = oracle.merge_states(allst[..., :-1], allst[..., -1])
        whole, _ = oracle.decode(Q, S, signs, norms, V, SCALE)
        # the merge does not see the order, so check it apart: entry r is the
        # state of rank r's slice
        order_err = 0.0
        for r in range(world):
            a, b = context_range(SHAPE[3], world, r)
            o_r, l_r = oracle.decode_state(Q, S, signs[:, :, a:b], norms[:, :, a:b],
                                           V[:, :, a:b], SCALE)
            order_err = max(order_err, float(np.max(np.abs(allst[r, ..., :-1] - o_r))),
                            float(np.max(np.abs(allst[r, ..., -1] - l_r))))
        out_q.put((rank, allst.shape, float(np.max(np.abs(merged - whole))), order_err))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_split_context_states_merge_to_whole_decode(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=180) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    B, Hq, d = SHAPE[0], SHAPE[1], SHAPE[5]
    for rank, shape, err, order_err in res:
        assert shape == (world, B, Hq, d + 1)
        assert err < 1e-12, (rank, err)
        assert order_err == 0.0, (rank, order_err)
