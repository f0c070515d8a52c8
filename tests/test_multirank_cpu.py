"""Host logic of the multi-GPU bench path with world_size 2 over gloo on CPU:
replicas draw distinct batches, the step time is the max over ranks, the
whole-job throughput sums all ranks, and the reference arm prints on rank 0
only."""
import io
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = 10.0 + 5.0 * rank                  # rank 1 is the slower one
        ms = bench.max_over_ranks(local_ms, dist, "cpu")
        seeds = [None] * world
        dist.all_gather_object(seeds, bench.rank_input_seed(0, rank))
        q.put((rank, ms, seeds))
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_and_seeds():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, seeds in res:
        assert ms == 15.0                              # max over ranks, on every rank
        assert len(set(seeds)) == 2                    # distinct replica batches


def test_aggregate_is_whole_job():
    sys.path.insert(0, ROOT)
    import bench
    one = bench.aggregate_tokens_per_s(1, 512, 2048, 50.0)
    assert one == pytest.approx(512 * 2048 / 0.05)
    assert bench.aggregate_tokens_per_s(4, 512, 2048, 50.0) == pytest.approx(4 * one)


def test_reference_arm_prints_on_rank_zero_only(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    called = []
    monkeypatch.setattr(bench, "time_oracle", lambda *a, **k: called.append(1) or (1.0, 1.0))
    args = type("A", (), dict(workload="headline", steps=2, warmup=1, seed=0, schedule="blocked",
                             driver="graph"))()
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.run_reference(args, rank=1, world=2)
    assert buf.getvalue() == "" and not called
    with redirect_stdout(buf):
        bench.run_reference(args, rank=0, world=2)
    import json
    line = json.loads(buf.getvalue())
    assert line["impl"] == "reference" and line["e2e"]["h2d_bytes_per_step"] == 0
    assert line["cpu_baseline"]["kind"] == "oracle"
