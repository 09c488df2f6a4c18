"""Multi-process host logic of bench.py on CPU (gloo, world size 2): the max-over-ranks
timing reduction, the barrier, and the reference arm that only rank 0 runs and prints."""
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      LOCAL_RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.reduce_max(float(10 * rank + 3))
        bench.barrier()
        buf = io.StringIO()
        with redirect_stdout(buf):
            rc = bench.main(["--impl", "reference", "--workload", "tiny", "--steps", "1",
                             "--warmup", "0", "--gpus", str(world), "--cpu-seconds", "0.2"])
        q.put((rank, got, rc, buf.getvalue()))
    finally:
        dist.destroy_process_group()


def test_two_rank_reduction_and_reference_arm():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = [q.get(timeout=240) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    by_rank = {r[0]: r for r in results}
    for rank in (0, 1):
        _, got, rc, out = by_rank[rank]
        assert got == 13.0          # max over ranks of (3, 13)
        assert rc == 0
    line = json.loads(by_rank[0][3].strip())
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert by_rank[1][3].strip() == ""  # rank 1 does no work and prints nothing


def test_single_process_reduce_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max(2.5) == 2.5


def test_l2_flush_decision_per_gpu():
    sys.path.insert(0, ROOT)
    import bench
    from ulysses_attention_output_b200 import workloads as W
    video, mmdit = W.WORKLOADS["video"], W.WORKLOADS["mmdit"]
    assert "no flush" in bench.workload_config(video, 1)["l2"]        # 960 MiB
    assert "no flush" in bench.workload_config(video, 4)["l2"]        # 240 MiB per GPU
    assert "before every timed step" in bench.workload_config(video, 8)["l2"]  # 120 MiB per GPU
    assert "before every timed step" in bench.workload_config(mmdit, 1)["l2"]  # 81 MiB
