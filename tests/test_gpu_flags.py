"""Per-slab arrival counters of the fused exchange (xs_attn_a2a_fused_flags, xs_slab_wait).

The storing warps add each slab's row count to its counter with a system-scope release after
their stores.  Checked here on one GPU, in one process:

* the counters end at exactly B * S/P * H rows per slab (per call), also when a warp's 32 rows
  straddle several slabs (P = 16, 6-row slabs) or run past a ragged S;
* the slabs are bit-identical to those of the fused call without counters;
* per-rank calls (the emulated ranks of one layer) add up to the layer's count, and the
  counters keep growing across steps;
* a consumer's bounded wait on a second stream, ordered after the producer by an event, ends
  with status 0, and one whose target is never reached reports XS_ERR_TIMEOUT and returns.

The wait is always ordered after the producing call: on one GPU a kernel that spins on a
counter and the kernel that would raise it are not guaranteed to run at the same time.
"""
import pytest
import torch

import ulysses_attention_output_b200 as xs
from ulysses_attention_output_b200 import workloads as W

from _parity import run_fused, to_gpu

pytestmark = pytest.mark.gpu

LIMIT_NS = 2_000_000_000


@pytest.fixture(scope="module", autouse=True)
def _built(cuda_device):
    from ulysses_attention_output_b200 import build
    build.build()
    xs.load()


def _counters(P):
    # one allocation, counters 256 bytes apart (distinct, never inside a slab)
    buf = torch.zeros(P * 64, dtype=torch.int32, device="cuda")
    return buf, [buf[64 * r:64 * r + 1] for r in range(P)]


@pytest.mark.parametrize("B,H,S,D,P", [(1, 4, 256, 64, 2), (1, 8, 200, 128, 2), (2, 16, 96, 128, 16),
                                       (2, 16, 1024, 72, 4)])
def test_counters_exact_and_slabs_identical(B, H, S, D, P):
    q, k, v = to_gpu(*W.make_qkv(B, H, S, D, seed=31 + S))
    ref, st = run_fused(q, k, v, P)
    assert st == 0
    dest = xs.alloc_dest(B, H, S, D, P, device="cuda", fill=float("nan"))
    buf, flags = _counters(P)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    xs.attn_a2a_fused_flags(q, k, v, dest, flags, status=status)
    done = torch.cuda.Event()
    done.record()
    consumer = torch.cuda.Stream()
    consumer.wait_event(done)
    per_slab = B * (S // P) * H
    for r in range(P):
        xs.slab_wait(flags[r], per_slab, LIMIT_NS, status, stream=consumer)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert [int(f.item()) for f in flags] == [per_slab] * P
    for a, b in zip(dest, ref):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_rank_calls_add_up_and_grow_across_steps():
    B, H, S, D, P = 1, 8, 512, 128, 4
    q, k, v = to_gpu(*W.make_qkv(B, H, S, D, seed=5))
    ref, _ = run_fused(q, k, v, P)
    dest = xs.alloc_dest(B, H, S, D, P, device="cuda")
    buf, flags = _counters(P)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    hr = H // P
    per_slab = B * (S // P) * H
    consumer = torch.cuda.Stream()
    for step in (1, 2):
        for g in range(P):
            sl = slice(g * hr, (g + 1) * hr)
            xs.attn_a2a_fused_flags(q[:, sl].contiguous(), k[:, sl].contiguous(), v[:, sl].contiguous(),
                                    dest, flags, heads_total=H, head_offset=g * hr, status=status)
        ev = torch.cuda.Event()
        ev.record()
        consumer.wait_event(ev)
        for r in range(P):
            xs.slab_wait(flags[r], step * per_slab, LIMIT_NS, status, stream=consumer)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert [int(f.item()) for f in flags] == [step * per_slab] * P
    for a, b in zip(dest, ref):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_wait_for_a_count_never_reached_times_out():
    B, H, S, D, P = 1, 2, 256, 64, 2
    q, k, v = to_gpu(*W.make_qkv(B, H, S, D, seed=8))
    dest = xs.alloc_dest(B, H, S, D, P, device="cuda")
    buf, flags = _counters(P)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    xs.attn_a2a_fused_flags(q, k, v, dest, flags, status=status)
    torch.cuda.synchronize()
    per_slab = B * (S // P) * H
    xs.slab_wait(flags[0], per_slab + 1, 2_000_000, status)  # 2 ms, one row short forever
    torch.cuda.synchronize()
    assert int(status.item()) == xs.XS_ERR_TIMEOUT
    # the context is intact: a wait whose count is there passes
    status.zero_()
    xs.slab_wait(flags[1], per_slab, LIMIT_NS, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0


def test_wait_compares_modulo_two_to_the_32():
    """Counters wrap: a target just past the wrap is reached by a counter that wrapped."""
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    c = torch.tensor([5], dtype=torch.int32, device="cuda")  # 2^32 + 5 after a wrap
    xs.slab_wait(c, 0xFFFFFFF0, LIMIT_NS, status)               # 21 below the counter
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    xs.slab_wait(c, 6, 2_000_000, status)
    torch.cuda.synchronize()
    assert int(status.item()) == xs.XS_ERR_TIMEOUT
