"""Multi-rank host logic of the bench on CPU (gloo, world size 2).

The decode and quantize path shards by independent (batch, kv-head) units, so
ranks run independent batches and the only collective is the max over ranks
of the step time.  This checks that reduction and the whole-job rate, that
the ranks' seeded batches are distinct and together are exactly the global
batch the rate counts, and that the reference arm prints on rank 0 only.
"""
import os
import socket
import subprocess
import sys
import types

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, times, out_q):
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = bench.reduce_max_over_ranks(times[rank], world, torch.device("cpu"))
        rate = bench.whole_job_rate(1000, world, ms)
        out_q.put((rank, ms, rate))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_rate():
    world = 2
    times = [3.0, 5.0]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, times, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, rate in res:
        assert ms == 5.0
        assert rate == pytest.approx(2 * 1000 / 5e-3)


def _shard_worker(rank, world, port, out_q):
    sys.path.insert(0, ROOT)
    import bench
    import workloads
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        args = types.SimpleNamespace(workload="gqa", batch=2)
        w = bench.rank_workload(args, rank).with_(T=96)
        mine = {"K": workloads.keys(w).float(), "V": workloads.values(w).float(),
                "Q": workloads.queries(w).float(),
                "lens": workloads.paged_layout(w.with_(T=4096))[0].float(),
                "Kn": workloads.new_tokens(w)[0].float()}
        gathered = {}
        for name, t in mine.items():
            parts = [torch.empty_like(t) for _ in range(world)]
            dist.all_gather(parts, t)
            gathered[name] = parts
        ms = bench.reduce_max_over_ranks([4.0, 2.0][rank], world, torch.device("cpu"))
        rate = bench.whole_job_rate(w.n_keys, world, ms)
        # numpy arrays travel through the queue by value (torch tensors would
        # be shared through file descriptors that die with this process)
        out_q.put((rank, w.first_seq, w.n_keys, rate,
                   {k: [p.numpy().copy() for p in v] for k, v in gathered.items()}
                   if rank == 0 else None))
    finally:
        dist.destroy_process_group()


def test_ranks_hold_distinct_shards_of_the_global_batch():
    import workloads
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted([q.get(timeout=300) for _ in range(world)], key=lambda r: r[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [0, 2]          # first global sequence per rank
    glob = workloads.GQA.with_(B=2 * world, T=96)
    want = {"K": workloads.keys(glob).float(), "V": workloads.values(glob).float(),
            "Q": workloads.queries(glob).float(),
            "lens": workloads.paged_layout(glob.with_(T=4096))[0].float(),
            "Kn": workloads.new_tokens(glob)[0].float()}
    parts = {k: [torch.from_numpy(a) for a in v] for k, v in res[0][4].items()}
    for name, full in want.items():
        assert not torch.equal(parts[name][0], parts[name][1]), name
        assert torch.equal(torch.cat(parts[name]), full), name
    # the whole-job rate counts the keys of the global batch over the
    # slowest rank's time
    for r in res:
        assert r[2] * world == glob.n_keys
        assert r[3] == pytest.approx(glob.n_keys / 4e-3)


def test_single_rank_rate_is_plain():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max_over_ranks(2.5, 1, torch.device("cpu")) == 2.5
    assert bench.whole_job_rate(500, 1, 2.0) == pytest.approx(250000.0)


def test_reference_arm_prints_on_rank_zero_only():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "0", "--workload", "single"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0
    assert r.stdout.strip() == ""
