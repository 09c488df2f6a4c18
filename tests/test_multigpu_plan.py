"""Multi-GPU Ulysses layer, host logic on the CPU (gloo ranks, no GPU): the plan of heads and
slabs per GPU, the table of slab addresses built from the exchanged IPC handles (a fake IPC
provider hands out recognisable addresses), unmapping when a mapping fails, and the serial
exchange (all-to-all of the packed pieces + unpack) against the oracle's post-attention
exchange."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from ulysses_attention_output_b200 import multigpu as M

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FAKE_BASE = 1 << 40     # fake mapped address of GPU g's allocation: FAKE_BASE * (g + 1)
FAKE_OFFSET = 4096      # every fake export reports its tensor this far into the allocation


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_gpu_plan():
    plans = [M.gpu_plan(g, 2, 40, 32768, 8) for g in range(2)]
    assert [(p.heads_local, p.head_offset, p.slabs_local, p.first_slab) for p in plans] == \
        [(20, 0, 4, 0), (20, 20, 4, 4)]
    p8 = M.gpu_plan(7, 8, 40, 32768, 8)
    assert (p8.heads_local, p8.head_offset, p8.slabs_local, p8.first_slab) == (5, 35, 1, 7)
    one = M.gpu_plan(0, 1, 40, 32768, 8)
    assert (one.heads_local, one.slabs_local) == (40, 8)
    with pytest.raises(ValueError):
        M.gpu_plan(0, 3, 40, 32768, 8)      # 3 does not divide P
    with pytest.raises(ValueError):
        M.gpu_plan(2, 2, 40, 32768, 8)      # rank outside the group
    with pytest.raises(ValueError):
        M.gpu_plan(0, 2, 12, 32768, 8)      # P does not divide H


def test_slab_table():
    plan = M.gpu_plan(1, 2, 8, 64, 4)
    assert M.slab_table(plan, [1000, 50000], 100) == [1000, 1100, 50000, 50100]
    plan4 = M.gpu_plan(0, 4, 8, 64, 4)
    assert M.slab_table(plan4, [10, 20, 30, 40], 7) == [10, 20, 30, 40]
    with pytest.raises(ValueError):
        M.slab_table(plan, [1000], 100)
    assert M.slab_bytes(1, 32768, 40, 128, 8) == 4096 * 40 * 128 * 2


class FakeIpc:
    """Handles name their GPU; opening GPU g's handle gives FAKE_BASE * (g + 1)."""

    def __init__(self, rank, fail_on=None):
        self.rank, self.fail_on = rank, fail_on
        self.opened, self.closed = [], []

    def export(self, t):
        return f"gpu{self.rank}".encode().ljust(64, b"\0"), FAKE_OFFSET

    def open(self, handle):
        g = int(handle.rstrip(b"\0").decode()[3:])
        if g == self.fail_on:
            raise RuntimeError(f"mapping of GPU {g} refused")
        base = FAKE_BASE * (g + 1)
        self.opened.append(base)
        return base

    def close(self, base):
        self.closed.append(base)


def _layer_worker(rank, world, port, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import oracle
    from ulysses_attention_output_b200 import multigpu as MM
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, H, S, D, P = 2, 4, 48, 8, 4
        ipc = FakeIpc(rank)
        layer = MM.UlyssesGpu(B, H, S, D, P, device="cpu", ipc=ipc)
        pl, nb = layer.plan, layer.slab_nbytes
        expect = []
        for r in range(P):
            g, i = divmod(r, pl.slabs_local)
            base = layer.slabs.data_ptr() if g == rank else FAKE_BASE * (g + 1) + FAKE_OFFSET
            expect.append(base + i * nb)
        table_ok = layer.dest == expect
        # arrival counters: right after each GPU's P/N slabs, 256 bytes apart
        cexp = []
        for r in range(P):
            g, i = divmod(r, pl.slabs_local)
            base = layer.slabs.data_ptr() if g == rank else FAKE_BASE * (g + 1) + FAKE_OFFSET
            cexp.append(base + pl.slabs_local * nb + 256 * i)
        table_ok = table_ok and layer.flag_table == cexp and \
            layer.counters.data_ptr() == layer.slabs.data_ptr() + pl.slabs_local * nb and \
            int(layer.counters.abs().sum()) == 0 and layer.rows_per_slab == B * (S // P) * H

        # serial exchange: pack this GPU's heads per rank, all-to-all, unpack
        rng = np.random.default_rng(11)
        o_full = rng.integers(-64, 64, size=(B, H, S, D)).astype(np.float64) / 8  # exact in bf16
        hs = slice(pl.head_offset, pl.head_offset + pl.heads_local)
        Sl = S // P
        out, send, recv = layer.alloc_exchange_buffers()
        o_mine = torch.from_numpy(o_full[:, hs]).to(torch.bfloat16)
        for r in range(P):   # send[r][b, s, h, :] = O_mine[b, h, r*Sl + s, :]
            send[r] = o_mine[:, :, r * Sl:(r + 1) * Sl].permute(0, 2, 1, 3)
        layer.slabs.fill_(float("nan"))
        layer.exchange_packed(send, recv)
        ref = oracle.a2a_post(o_full, P)[pl.first_slab:pl.first_slab + pl.slabs_local]
        diff = float(np.abs(layer.slabs.to(torch.float64).numpy() - ref).max())
        layer.complete()
        layer.close()
        out_q.put((rank, table_ok, diff, sorted(ipc.opened) == sorted(ipc.closed), len(ipc.opened)))
    finally:
        dist.destroy_process_group()


def _run(worker, world, *extra):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=worker, args=(r, world, port, q, *extra)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=180) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return sorted(res)


def test_two_gpu_layer_host_logic():
    res = _run(_layer_worker, 2)
    for rank, table_ok, diff, unmapped, n_opened in res:
        assert table_ok, f"slab table of rank {rank}"
        assert diff == 0.0, f"serial exchange of rank {rank} differs from the oracle by {diff}"
        assert unmapped and n_opened == 1


def _failing_worker(rank, world, port, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    from ulysses_attention_output_b200 import multigpu as MM
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ipc = FakeIpc(rank, fail_on=2 if rank != 2 else None)
        try:
            MM.UlyssesGpu(1, 6, 12, 8, 6, device="cpu", ipc=ipc)
            raised = False
        except RuntimeError:
            raised = True
        out_q.put((rank, raised, sorted(ipc.opened) == sorted(ipc.closed), len(ipc.opened)))
    finally:
        dist.destroy_process_group()


def test_failed_mapping_unmaps_what_was_mapped():
    res = _run(_failing_worker, 3)
    # ranks 0 and 1 map one peer, fail on GPU 2 and unmap the one they had; rank 2 maps both
    assert res[0][:3] == (0, True, True) and res[0][3] == 1
    assert res[1][:3] == (1, True, True) and res[1][3] == 1
    assert res[2][:2] == (2, False) and res[2][3] == 2
