"""The N>1 path of bench.py on CPU: two gloo ranks, each with its own replica
timing; the job takes the slowest rank's time and every rank's bytes."""
import json
import os
import socket
import subprocess
import sys

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


def test_bench_launches_its_own_ranks():
    """`bench.py --gpus 2` without a launcher starts two ranks itself (under
    torch.distributed.run, rendezvous on 127.0.0.1) and rank 0 alone prints
    the job line: the same launch path as a GPU run, with gloo ranks and no
    GPU work (--launch-check)."""
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items()
           if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "2",
                        "--launch-check", "--steps", "7"], capture_output=True, text=True,
                       timeout=300, env=env, cwd=root)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(ln) for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    line = lines[0]
    assert line["n_gpus"] == 2 and line["steps"] == 7
    # rank 1 is the slower one in every timing: the job takes its times
    assert line["total_ms"] == 11.0 and line["e2e_ms"] == 15.0 and line["scan_ms"] == 5.0
    assert line["value"] == pytest.approx(2 * 1_000_000 * 7 / 11e-3 / 1e9)


def _shard_rank(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        from tests.shard_fake import FakeShardOps
        from top_kv_span_b200 import reatt as R
        from top_kv_span_b200 import workloads as wl
        from top_kv_span_b200.sharded import ShardedStep, dist_all_gather, shard_rows

        oracle.build()
        w = wl.WORKLOADS["tiny_f32_4k"].replace(T=700, G=4, L=64, S=16, k=6, Hq=4, Hkv=2,
                                                B=1, n_needles=1, seed=91)
        x = wl.make_inputs(w)   # every rank draws the same sequence, keeps its rows
        d = R.dims_of(w)
        shards = R.reatt_shard_plan(d, world)
        sh = shards[rank]
        step = ShardedStep(d, sh, world, device="cpu", ops=FakeShardOps(oracle))
        out = torch.empty((w.B, w.Hq, w.C, w.d), dtype=torch.float32)
        step(x["q"], shard_rows(x["k_cache"], sh), shard_rows(x["v_cache"], sh), x["k_cur"],
             x["v_cur"], out, dist_all_gather())
        names = ("q", "k_cache", "v_cache", "k_cur", "v_cur")
        ref = oracle.step(**{n: wl.to_oracle(x[n]) for n in names}, G=w.G, L=w.L, S=w.S, k=w.k,
                          rope_base=w.rope_base)
        q.put((rank, (sh.t_begin, sh.t_end, sh.owns_current), step.sel.numpy().tolist(),
               ref["sel"].tolist(), float(abs(out.double().numpy() - ref["out"]).max())))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_sharded_step_on_cpu():
    """The sharded step's call order and exchanges on two gloo ranks, each
    holding half of one sequence's cache (the library's shard plan), with
    the kernels replaced by an oracle-built CPU stand-in: both ranks select
    the oracle's spans and produce the oracle's output for the whole
    sequence."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=300) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, sh0, sel0, ref0, err0), (r1, sh1, sel1, ref1, err1) = res
    assert sh0[0] == 0 and sh0[1] == sh1[0] and sh1[2] == 1 and sh0[2] == 0
    assert sel0 == sel1 == ref0
    assert err0 <= 1e-6 and err1 <= 1e-6
