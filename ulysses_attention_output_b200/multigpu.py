"""Ulysses attention over the GPUs of one node, one process per GPU, with the post-attention
All-to-All fused into the attention kernel across GPUs.

Layout (N GPUs, P Ulysses ranks, N | P): GPU g holds
* the H/N heads ``[g*H/N, (g+1)*H/N)`` of Q, K, V over the full sequence, ``[B, H/N, S, D]``;
* the sequence-shard slabs of ranks ``[g*P/N, (g+1)*P/N)``, ``[P/N, B, S/P, H, D]``, in one
  allocation that every other GPU maps (CUDA IPC).

The fused step: every GPU runs ``xs_attn_a2a_fused_rank`` on its heads with a ``dest`` table
of all P slabs, its own and the mapped ones of the other GPUs, so each finished output tile
is stored by its owner straight into the slab of the rank that needs it, over NVLink, while
the owner goes on to its next tile (the X-Stage explainer, "FlashAttention-A2A
(Piggybacking)").  ``complete()`` then orders those stores before anything that reads the
slabs.  No kernel waits on another GPU: the ordering is a one-element collective enqueued
after the fused kernel.  Alternatively ``fused_flags()`` has every storing warp add its row
count to the owning slab's arrival counter with a system-scope release, and ``wait_slabs()``
waits (bounded) on this GPU's counters: a consumer of a slab can then start without the
collective.

The serial form (attention, then a separate exchange) packs the head-major output per
destination GPU with the library's exchange kernel, moves it with one all-to-all of the
process group and unpacks it into the slabs.
"""
from __future__ import annotations

import contextlib
from dataclasses import dataclass


@dataclass(frozen=True)
class GpuPlan:
    rank: int            # this GPU's index in the group
    world: int           # GPUs in the group (N)
    P: int               # Ulysses ranks (sequence shards)
    heads_total: int     # H
    heads_local: int     # H / N
    head_offset: int     # global index of this GPU's first head
    slabs_local: int     # P / N sequence shards held here
    first_slab: int      # global rank of this GPU's first slab


def gpu_plan(rank: int, world: int, heads_total: int, seq_len: int, P: int) -> GpuPlan:
    """Heads and slabs of GPU ``rank`` of ``world``.  Needs N | P, P | H and P | S."""
    if world <= 0 or not 0 <= rank < world:
        raise ValueError("rank must lie in [0, world)")
    if P % world:
        raise ValueError(f"the GPU count {world} must divide the Ulysses rank count P={P}")
    if heads_total % P or seq_len % P:
        raise ValueError("Ulysses sharding needs H % P == 0 and S % P == 0")
    hl, sl = heads_total // world, P // world
    return GpuPlan(rank, world, P, heads_total, hl, rank * hl, sl, rank * sl)


def slab_bytes(B: int, S: int, H: int, D: int, P: int) -> int:
    """Bytes of one sequence-shard slab [B, S/P, H, D] of bf16."""
    return B * (S // P) * H * D * 2


def slab_table(plan: GpuPlan, bases: list[int], nbytes: int) -> list[int]:
    """Address, in this process, of every rank's slab: rank r lives on GPU r // (P/N) as that
    GPU's slab r % (P/N); ``bases[g]`` is the address here of GPU g's first slab."""
    if len(bases) != plan.world:
        raise ValueError(f"need one base per GPU ({plan.world}), got {len(bases)}")
    return [bases[r // plan.slabs_local] + (r % plan.slabs_local) * nbytes for r in range(plan.P)]


COUNTER_STRIDE = 256  # bytes between two slabs' arrival counters


def counter_table(plan: GpuPlan, bases: list[int], slabs_nbytes: int) -> list[int]:
    """Address, in this process, of every rank's arrival counter: GPU g keeps the counters of
    its P/N slabs right after them (``slabs_nbytes`` = P/N slabs), COUNTER_STRIDE apart."""
    if len(bases) != plan.world:
        raise ValueError(f"need one base per GPU ({plan.world}), got {len(bases)}")
    return [bases[r // plan.slabs_local] + slabs_nbytes + (r % plan.slabs_local) * COUNTER_STRIDE
            for r in range(plan.P)]


class XsIpc:
    """CUDA IPC through libxs (``xs_ipc_export`` / ``xs_ipc_open`` / ``xs_ipc_close``)."""

    def export(self, t):
        import ulysses_attention_output_b200 as xs
        return xs.ipc_export(t)

    def open(self, handle: bytes) -> int:
        import ulysses_attention_output_b200 as xs
        return xs.ipc_open(handle)

    def close(self, base: int) -> None:
        import ulysses_attention_output_b200 as xs
        xs.ipc_close(base)


class UlyssesGpu:
    """This process's GPU in a Ulysses layer over the process group ``group`` (default: the
    world).  Collective: every process of the group constructs it with the same shape, in the
    same order, and calls ``close()``.

    ``slabs``  -- this GPU's sequence-shard slabs, ``[P/N, B, S/P, H, D]`` bf16 (rank
                  ``plan.first_slab + i`` is ``slabs[i]``);
    ``dest``   -- the address of every rank's slab as seen here (own and mapped), the ``dest``
                  table of the fused call.
    ``ipc``    -- the export/open/close provider (``XsIpc`` unless a test substitutes one).
    """

    def __init__(self, B: int, H: int, S: int, D: int, P: int, device=None, group=None, ipc=None):
        import torch
        import torch.distributed as dist

        self.group = group
        self.rank, self.world = dist.get_rank(group), dist.get_world_size(group)
        self.B, self.H, self.S, self.D, self.P = B, H, S, D, P
        self.plan = gpu_plan(self.rank, self.world, H, S, P)
        self.device = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
        self.ipc = ipc if ipc is not None else XsIpc()
        self.backend = dist.get_backend(group)
        self.slab_nbytes = slab_bytes(B, S, H, D, P)
        # One allocation: this GPU's slabs, then one arrival counter per slab (256 bytes apart),
        # exported together so that the other GPUs map both.
        nb_slabs = self.plan.slabs_local * self.slab_nbytes
        self._buf = torch.empty(nb_slabs + COUNTER_STRIDE * self.plan.slabs_local, dtype=torch.uint8,
                                device=self.device)
        self.slabs = self._buf[:nb_slabs].view(torch.bfloat16).view(self.plan.slabs_local, B, S // P, H, D)
        self.counters = self._buf[nb_slabs:].view(torch.int32)[::COUNTER_STRIDE // 4]
        self.counters.zero_()
        self._steps_flagged = 0
        handle, offset = self.ipc.export(self._buf)
        infos = [None] * self.world
        dist.all_gather_object(infos, (self.rank, handle, offset), group=group)
        self._mapped: list[int] = []
        bases = []
        try:
            for g, (rank_g, handle_g, offset_g) in enumerate(infos):
                if rank_g != g:
                    raise RuntimeError(f"slab handle of GPU {rank_g} arrived in slot {g}")
                if g == self.rank:
                    bases.append(self.slabs.data_ptr())
                else:
                    base = self.ipc.open(handle_g)
                    self._mapped.append(base)
                    bases.append(base + offset_g)
        except Exception:
            self._unmap()
            raise
        self.dest = slab_table(self.plan, bases, self.slab_nbytes)
        self.flag_table = counter_table(self.plan, bases, nb_slabs)
        self._token = torch.zeros(1, dtype=torch.float32, device=self.device)
        self._closed = False

    # ------------------------------------------------------------ the fused step
    def fused(self, q, k, v, scale=None, stream=None, status=None):
        """Attention on this GPU's heads ``q, k, v`` [B, H/N, S, D], every finished tile
        stored into its rank's slab wherever that lives.  Enqueued on ``stream``; call
        ``complete()`` before reading the slabs."""
        import ulysses_attention_output_b200 as xs
        xs.attn_a2a_fused_rank(q, k, v, self.dest, heads_total=self.H, head_offset=self.plan.head_offset,
                               scale=scale, stream=stream, status=status)

    def fused_flags(self, q, k, v, scale=None, stream=None, status=None):
        """:meth:`fused` that also adds each slab's stored rows to that slab's arrival counter
        (on the GPU that owns the slab) with a system-scope release; one step adds
        ``rows_per_slab`` to every counter once all GPUs' calls have run."""
        import ulysses_attention_output_b200 as xs
        xs.attn_a2a_fused_flags(q, k, v, self.dest, self.flag_table, heads_total=self.H,
                                head_offset=self.plan.head_offset, scale=scale, stream=stream, status=status)
        self._steps_flagged += 1

    @property
    def rows_per_slab(self) -> int:
        """Rows (one head of one sequence position) that one step stores into each slab."""
        return self.B * (self.S // self.P) * self.H

    def wait_slabs(self, stream=None, status=None, limit_ns: int = 2_000_000_000):
        """Enqueue on ``stream`` a bounded wait until this GPU's slabs hold every row of every
        flagged step so far (each counter reaches steps x ``rows_per_slab``): the consumer of
        a slab may then start on it without a collective.  The waits run on this GPU after its
        own fused call (stream order) and wait only for the other GPUs' stores; ``status``
        (int32 CUDA tensor) receives XS_ERR_TIMEOUT if a count is still short after
        ``limit_ns``.  Overwriting a slab that another GPU still reads is not covered: call
        ``complete()`` between the last read and the next fused call."""
        import torch

        import ulysses_attention_output_b200 as xs
        if status is None:
            raise ValueError("wait_slabs needs a status tensor")
        target = self._steps_flagged * self.rows_per_slab
        for i in range(self.plan.slabs_local):
            xs.slab_wait(self.counters[i:i + 1], target, limit_ns, status, stream=stream)
        return target

    def complete(self, stream=None):
        """Order every GPU's slab stores enqueued so far before the later work on ``stream``.

        With NCCL: a one-element all-reduce enqueued after the fused kernel.  Each GPU's
        all-reduce starts after its own fused kernel has finished (stream order) and ends
        only after every GPU's has started, hence after every GPU's fused kernel has
        finished, and a finished kernel's stores, peer stores included, are visible.  No host
        synchronisation.  Call it again after the last read of the slabs and before the next
        fused call, so that no GPU overwrites a slab another GPU is still reading.
        With another backend (gloo: the single-GPU multi-process tests): synchronise
        ``stream``, then a barrier of the group."""
        import torch
        import torch.distributed as dist
        if self.backend == "nccl":
            if stream is None:
                dist.all_reduce(self._token, group=self.group)
            else:
                with torch.cuda.stream(stream):
                    dist.all_reduce(self._token, group=self.group)
        else:
            if self.device.type == "cuda":
                (stream or torch.cuda.current_stream(self.device)).synchronize()
            dist.barrier(group=self.group)

    # ------------------------------------------------------------ the serial step
    def alloc_exchange_buffers(self):
        """Head-major output ``[B, H/N, S, D]`` of this GPU's heads and the packed send /
        receive buffers ``[P, B, S/P, H/N, D]`` of the serial exchange."""
        import torch
        pl = self.plan
        out = torch.empty((self.B, pl.heads_local, self.S, self.D), dtype=torch.bfloat16, device=self.device)
        shape = (self.P, self.B, self.S // self.P, pl.heads_local, self.D)
        send = torch.empty(shape, dtype=torch.bfloat16, device=self.device)
        recv = torch.empty(shape, dtype=torch.bfloat16, device=self.device)
        return out, send, recv

    def serial(self, q, k, v, out, send, recv, scale=None, stream=None, status=None):
        """Attention into ``out`` (head-major), then the separate exchange into the slabs."""
        import ulysses_attention_output_b200 as xs
        xs.attn(q, k, v, out, scale=scale, stream=stream, status=status)
        xs.a2a_relayout(out, [send[r] for r in range(self.P)], stream=stream)
        self.exchange_packed(send, recv, stream=stream)

    def exchange_packed(self, send, recv, stream=None):
        """All-to-all of the packed per-rank pieces, then unpack into the slabs.

        ``send[r]`` = ``[B, S/P, H/N, D]``: this GPU's heads of rank r's sequence shard.  The
        ranks of GPU j are contiguous in ``send``, so one all-to-all with equal splits gives
        ``recv`` = ``[N (source GPU), P/N (local slab), B, S/P, H/N, D]``; source GPU g's
        heads go to columns ``[g*H/N, (g+1)*H/N)`` of every local slab."""
        import torch
        import torch.distributed as dist
        pl = self.plan
        ctx = torch.cuda.stream(stream) if stream is not None else contextlib.nullcontext()
        with ctx:
            if self.backend == "nccl" or not send.is_cuda:
                dist.all_to_all_single(recv, send, group=self.group)
            else:  # gloo moves host tensors only
                if stream is not None:
                    stream.synchronize()
                r_host = torch.empty(recv.shape, dtype=recv.dtype)
                dist.all_to_all_single(r_host, send.cpu(), group=self.group)
                recv.copy_(r_host)
            src = recv.view(pl.world, pl.slabs_local, self.B, self.S // self.P, pl.heads_local, self.D)
            dst = self.slabs.view(pl.slabs_local, self.B, self.S // self.P, pl.world, pl.heads_local, self.D)
            dst.copy_(src.permute(1, 2, 3, 0, 4, 5))

    # ------------------------------------------------------------ teardown
    def _unmap(self):
        while self._mapped:
            self.ipc.close(self._mapped.pop())

    def close(self):
        """Collective: wait until no GPU can still store into a mapping, unmap the other
        GPUs' slabs, and wait until every GPU has unmapped this one's before it may be freed."""
        import torch.distributed as dist
        if getattr(self, "_closed", True):
            return
        if self.device.type == "cuda":
            import torch
            torch.cuda.synchronize(self.device)
        dist.barrier(group=self.group)
        self._unmap()
        dist.barrier(group=self.group)
        self._closed = True


class LayerHostPipeline:
    """End-to-end step of one GPU of the layer with host buffers: this GPU's heads' q, k, v
    [B, H/N, S, D] from pinned host memory in, this GPU's slabs [P/N, B, S/P, H, D] to pinned
    host memory out.

    The local heads are split into ``chunks`` groups: the host-to-device copies of a group's
    q, k, v (input-copy stream) overlap the fused calls of the groups before it (the caller's
    stream for even groups, a second compute stream for odd ones), each call storing its
    heads' rows into every GPU's slabs.  After the last group: ``complete()``, the copy of
    this GPU's slabs to the host, and ``complete()`` again, so that no GPU's next fused call
    overwrites a slab that is still being copied out.  The slabs cannot be copied out per
    group as on one GPU: their rows come from every GPU's heads, and only ``complete()``
    orders the other GPUs' stores.  ``chunks=1`` runs copies, calls and copies in sequence.
    """

    def __init__(self, layer: UlyssesGpu, chunks: int | None = None, scale=None):
        import torch
        self.layer = layer
        self.scale = scale
        pl = layer.plan
        B, S, D = layer.B, layer.S, layer.D
        hl = pl.heads_local
        if chunks is None:
            # about one wave of 256-row work items per group, at most 20 groups (as on one GPU)
            sms = torch.cuda.get_device_properties(layer.device).multi_processor_count
            items_per_head = B * ((S + 255) // 256)
            chunks = max(1, min(20, hl, (hl * items_per_head) // sms))
        self.chunks = int(chunks)
        hc = (hl + self.chunks - 1) // self.chunks
        self.groups = [(h0, min(hl, h0 + hc)) for h0 in range(0, hl, hc)]
        dev = layer.device
        self.q = [torch.empty((B, h1 - h0, S, D), dtype=torch.bfloat16, device=dev) for h0, h1 in self.groups]
        self.k = [torch.empty_like(t) for t in self.q]
        self.v = [torch.empty_like(t) for t in self.q]
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.s_in = torch.cuda.Stream(device=dev)
        self.s_k2 = torch.cuda.Stream(device=dev)   # calls of the odd groups
        self.ev_in = [torch.cuda.Event() for _ in self.groups]     # group's inputs on the device
        self.ev_kern = [torch.cuda.Event() for _ in self.groups]   # group's call done
        self._started = False

    @property
    def in_shape(self):
        pl = self.layer.plan
        return (self.layer.B, pl.heads_local, self.layer.S, self.layer.D)

    @property
    def h2d_bytes(self) -> int:
        return 3 * sum(t.numel() for t in self.q) * 2

    @property
    def d2h_bytes(self) -> int:
        return self.layer.slabs.numel() * 2

    def run(self, q_host, k_host, v_host, slabs_host, stream=None):
        """Enqueue one step (collective: every GPU of the layer calls it).  ``slabs_host`` is
        ready once the caller's stream has reached the point where ``run`` returned."""
        import torch

        import ulysses_attention_output_b200 as xs
        layer = self.layer
        s = stream or torch.cuda.current_stream(layer.device)
        for name, t in (("q_host", q_host), ("k_host", k_host), ("v_host", v_host)):
            if tuple(t.shape) != self.in_shape or t.dtype != torch.bfloat16 or t.is_cuda \
                    or not t.is_contiguous() or not t.is_pinned():
                raise ValueError(f"{name} must be a contiguous pinned CPU bf16 tensor of shape {self.in_shape}")
        if tuple(slabs_host.shape) != tuple(layer.slabs.shape) or slabs_host.dtype != torch.bfloat16 \
                or slabs_host.is_cuda or not slabs_host.is_contiguous() or not slabs_host.is_pinned():
            raise ValueError(f"slabs_host must be a contiguous pinned CPU bf16 tensor of shape "
                             f"{tuple(layer.slabs.shape)}")
        start = torch.cuda.Event()
        start.record(s)
        self.s_in.wait_event(start)
        self.s_k2.wait_event(start)
        pl = layer.plan
        for g, (h0, h1) in enumerate(self.groups):
            with torch.cuda.stream(self.s_in):
                if self._started:
                    self.s_in.wait_event(self.ev_kern[g])   # the group's buffers are free
                for b in range(layer.B):   # one contiguous host range per batch entry
                    self.q[g][b].copy_(q_host[b, h0:h1], non_blocking=True)
                    self.k[g][b].copy_(k_host[b, h0:h1], non_blocking=True)
                    self.v[g][b].copy_(v_host[b, h0:h1], non_blocking=True)
                self.ev_in[g].record(self.s_in)
            ks = s if g % 2 == 0 else self.s_k2
            ks.wait_event(self.ev_in[g])
            xs.attn_a2a_fused_rank(self.q[g], self.k[g], self.v[g], layer.dest, heads_total=layer.H,
                                   head_offset=pl.head_offset + h0, scale=self.scale, stream=ks,
                                   status=self.status)
            self.ev_kern[g].record(ks)
        self._started = True
        for g in range(len(self.groups)):
            s.wait_event(self.ev_kern[g])
        layer.complete(s)
        with torch.cuda.stream(s):
            slabs_host.copy_(layer.slabs, non_blocking=True)
        layer.complete(s)
