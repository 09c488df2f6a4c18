"""Ulysses rank plan (CPU): head and sequence ranges per rank, and -- across two gloo ranks --
that per-rank attention of the planned heads, assembled into the sequence shards by the
plan's offsets, reproduces the single-process oracle pipeline."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from ulysses_attention_output_b200 import ulysses

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_plan_ranges():
    plans = [ulysses.rank_plan(g, 4, 16, 1024) for g in range(4)]
    assert [p.head_offset for p in plans] == [0, 4, 8, 12]
    assert all(p.heads_local == 4 and p.seq_local == 256 for p in plans)
    assert [p.seq_offset for p in plans] == [0, 256, 512, 768]
    with pytest.raises(ValueError):
        ulysses.rank_plan(0, 3, 16, 1024)
    with pytest.raises(ValueError):
        ulysses.rank_plan(4, 4, 16, 1024)


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import oracle
    from ulysses_attention_output_b200 import ulysses as U
    from ulysses_attention_output_b200 import workloads as W
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, H, S, D = 1, 4, 64, 8
        qf, kf, vf = W.make_qkv(B, H, S, D, seed=3)
        plan = U.rank_plan(rank, world, H, S)
        hs = slice(plan.head_offset, plan.head_offset + plan.heads_local)
        o_local = torch.from_numpy(oracle.attention(qf[:, hs], kf[:, hs], vf[:, hs]))  # [B, Hl, S, D]
        # post-attention exchange by the plan: every rank sends rows of its heads to rank r
        slabs = torch.zeros((world, B, plan.seq_local, H, D), dtype=torch.float64)
        for r in range(world):
            pr = U.rank_plan(r, world, H, S)
            part = o_local[:, :, pr.seq_offset:pr.seq_offset + pr.seq_local]   # [B, Hl, Sl, D]
            slabs[r, :, :, hs] = part.permute(0, 2, 1, 3)
        dist.all_reduce(slabs)   # disjoint head columns: the sum assembles the slabs
        if rank == 0:
            ref = oracle.a2a_post(oracle.attention(qf, kf, vf), world)
            q.put(float(np.abs(slabs.numpy() - ref).max()))
    finally:
        dist.destroy_process_group()


def test_two_rank_plan_reproduces_oracle_pipeline():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    err = q.get(timeout=240)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert err < 1e-12
