"""Multi-process Ulysses layer on one GPU: two processes, each with its own heads and its own
sequence-shard slabs, map each other's slabs through CUDA IPC; the fused call of each
process stores its finished tiles into both processes' slabs.  The processes are ordered by
the host (stream synchronisation + a gloo barrier), so no kernel waits on another.

Checked bit for bit against the single-process fused call on all heads (itself checked
against the oracle by the parity tests): the fused multi-process step, the serial step
(attention, pack, all-to-all, unpack), the fused step with arrival counters (each
process's warps release-add their row counts to the owning process's counters through the
IPC mapping; the counts must come out exact), and the end-to-end step with pinned host
buffers (``LayerHostPipeline``: head groups on two compute streams, slabs copied out after
completion).  Every slab is filled with NaN bits first, so a
missing store fails the comparison.
"""
import os
import socket
import sys
from datetime import timedelta

import pytest
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# B, H, S, D, P; two processes.  S/P straddles 128-row tiles; 640 and 384 leave ragged items.
CASES = [(1, 4, 640, 128, 4), (2, 8, 384, 72, 8)]


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, case, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=120))
    try:
        out_q.put((rank, None, *_steps(case, dev)))
    except Exception as e:  # reported to the parent instead of leaving it waiting
        out_q.put((rank, repr(e), False, False, False, -1, 0))
        raise
    finally:
        dist.destroy_process_group()


def _steps(case, dev):
    import torch

    import ulysses_attention_output_b200 as xs
    from ulysses_attention_output_b200 import multigpu as MM
    from ulysses_attention_output_b200 import workloads as W
    B, H, S, D, P = case
    q, k, v = W.make_qkv(B, H, S, D, seed=700 + S + D)
    ref = xs.alloc_dest(B, H, S, D, P, device=dev)
    xs.attn_a2a_fused(q.to(dev), k.to(dev), v.to(dev), ref)
    layer = MM.UlyssesGpu(B, H, S, D, P, device=dev)
    pl = layer.plan
    hs = slice(pl.head_offset, pl.head_offset + pl.heads_local)
    ql, kl, vl = (t[:, hs].contiguous().to(dev) for t in (q, k, v))
    status = torch.zeros(1, dtype=torch.int32, device=dev)

    def matches():
        torch.cuda.synchronize(dev)
        return all(torch.equal(layer.slabs[i].view(torch.int16), ref[pl.first_slab + i].view(torch.int16))
                   for i in range(pl.slabs_local))

    layer.slabs.view(torch.int16).fill_(-1)   # NaN bits
    layer.complete()                          # every process's sentinel is in place
    layer.fused(ql, kl, vl, status=status)
    layer.complete()                          # every process's stores have landed
    fused_ok = matches()
    layer.complete()                          # both have read before the next writes

    out, send, recv = layer.alloc_exchange_buffers()
    layer.slabs.view(torch.int16).fill_(-1)
    layer.serial(ql, kl, vl, out, send, recv, status=status)
    layer.complete()
    serial_ok = matches()
    layer.complete()

    # arrival counters: each process's stores add to the owner's counters (IPC-mapped); the
    # host orders both processes' fused calls before either waits, so the waits find their
    # counts already there and no kernel spins while another on this GPU produces
    layer.slabs.view(torch.int16).fill_(-1)
    layer.complete()
    layer.fused_flags(ql, kl, vl, status=status)
    layer.complete()
    target = layer.wait_slabs(status=status)
    flags_ok = matches() and target == layer.rows_per_slab and \
        [int(c) for c in layer.counters.cpu()] == [layer.rows_per_slab] * pl.slabs_local
    st = int(status.item())
    layer.complete()

    # the end-to-end step with host buffers, two head groups on two compute streams, run
    # twice (the second run reuses every device buffer)
    pipe = MM.LayerHostPipeline(layer, chunks=2)
    qh, kh, vh = (t[:, hs].contiguous().pin_memory() for t in (q, k, v))
    slabs_h = torch.empty(layer.slabs.shape, dtype=torch.bfloat16).pin_memory()
    pipe_ok = True
    for _ in range(2):
        slabs_h.view(torch.int16).fill_(-1)
        layer.slabs.view(torch.int16).fill_(-1)
        layer.complete()
        pipe.run(qh, kh, vh, slabs_h)
        torch.cuda.synchronize(dev)
        pipe_ok = pipe_ok and all(torch.equal(slabs_h[i].view(torch.int16), ref[pl.first_slab + i].cpu().view(torch.int16))
                                  for i in range(pl.slabs_local))
    st = st or int(pipe.status.item())
    layer.complete()
    layer.close()
    return fused_ok, serial_ok and flags_ok, pipe_ok, st, len(layer.dest)


@pytest.mark.parametrize("case", CASES)
def test_two_process_fused_exchange_bit_exact(case, cuda_device):
    from ulysses_attention_output_b200 import build
    build.build()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, case, q)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        res = sorted(q.get(timeout=300) for _ in procs)
    finally:
        for p in procs:
            p.join(timeout=120)
    assert [p.exitcode for p in procs] == [0, 0]
    for rank, err, fused_ok, serial_ok, pipe_ok, st, n_dest in res:
        assert err is None, f"process {rank}: {err}"
        assert st == 0, f"device status {st} on process {rank}"
        assert n_dest == case[4]
        assert fused_ok, f"fused multi-process slabs of process {rank} differ from the single fused call"
        assert serial_ok, (f"serial (or flagged) multi-process slabs or arrival counts of process {rank} "
                           "differ from the single fused call")
        assert pipe_ok, f"host-buffer pipeline slabs of process {rank} differ from the single fused call"
