"""Multi-rank host logic of bench.py with world-size-2 gloo ranks on CPU.

Each rank is an independent replica (tokens sharded by rank, weights replicated,
no data-path collective); the only collectives are the timing barrier and the
max-over-ranks reduction, which these tests exercise.
"""
import os
import socket

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    import workloads as W
    ms = 10.0 + 5.0 * rank                       # the slower rank decides
    dist.barrier()
    mx = bench.reduce_max(ms, torch.device("cpu"))
    tput = bench.job_throughput(world, 4096, 20, mx)
    # each replica draws its own tokens; the weights are the same on every rank
    spec = W.tiny_spec(T=8, D=16, E=4, k=2, F=16, dtype="bf16")
    x = W.make_layer(spec, seed=rank, with_experts=False)["x"]
    wg = W.make_experts(spec, seed=0)["w_gate"]
    q.put((rank, mx, tput, x.tobytes(), wg.tobytes()))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_max_and_throughput():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, mx0, t0, x0, w0), (r1, mx1, t1, x1, w1) = res
    assert mx0 == mx1 == 15.0
    assert t0 == t1 == pytest.approx(2 * 4096 * 20 / 0.015)
    assert x0 != x1          # different tokens per replica
    assert w0 == w1          # replicated weights


def test_reference_arm_other_ranks_do_nothing(capsys):
    import bench

    class A:
        workload = "tiny_fp32"
        steps = 1
        warmup = 0

    assert bench.run_reference(A, rank=1, world=2) is None
    assert capsys.readouterr().out == ""


def test_reference_arm_line_on_rank0(capsys):
    import json

    import bench

    class A:
        workload = "tiny_fp32"
        steps = 2
        warmup = 1

    bench.run_reference(A, rank=0, world=1)
    line = json.loads(capsys.readouterr().out.strip())
    assert line["impl"] == "reference" and line["unit"] == "tokens/s" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
