"""The N>1 path of bench.py on CPU: two gloo ranks, each with its own replica
timing; the job takes the slowest rank's time and every rank's bytes."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    from top_kv_span_b200 import workloads as wl

    def reduce_max(vals):
        t = torch.tensor(vals, dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return [float(v) for v in t.tolist()]

    # rank-dependent times: rank 1 is the slow one
    total, e2e, scan = 10.0 + rank, 12.0 + 3 * rank, 5.0 - rank
    agg = bench.aggregate(world, 1_000_000, 10, total, e2e, scan, reduce_max)
    # replicas draw different sequences (seed offset per rank)
    w = wl.WORKLOADS["tiny_f32_4k"].replace(T=64, seed=wl.WORKLOADS["tiny_f32_4k"].seed + 1000 * rank)
    x = wl.make_inputs(w)
    digest = torch.tensor([float(x["k_cache"].double().sum())])
    all_d = [torch.zeros(1) for _ in range(world)]
    dist.all_gather(all_d, digest)
    q.put((rank, agg, [float(v) for v in all_d]))
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_aggregation():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, agg, digests in res:
        assert agg["total_ms"] == 11.0 and agg["e2e_ms"] == 15.0 and agg["scan_ms"] == 5.0
        assert agg["value"] == pytest.approx(2 * 1_000_000 * 10 / 11e-3 / 1e9)
        assert digests[0] != digests[1]
