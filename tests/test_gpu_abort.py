"""The attention kernel's own abort path, on the GPU, without a fault.

``xs_selftest_attn_abort`` runs the head-major attention kernel with a short wait limit and
with every CTA's TMA producer stopping before one of its fills, as if that copy never
arrived.  The waits that depend on it run out: the kernel must report XS_ERR_TIMEOUT in the
status word and return (no hang, no trap), each CTA first letting its own copies and MMAs in
flight finish and freeing its tensor memory.  A normal call in the same process afterwards
must still match the oracle: the context and every SM's tensor memory are intact.

Stall points: before any fill (the MMA thread's first Q wait runs out), in the middle of the
key loop (MMAs and copies in flight when the abort is raised), and at the first fill of a
CTA's second work item (the first item's epilogue completed, the next one never starts).
"""
import pytest
import torch

import oracle
import ulysses_attention_output_b200 as xs
from ulysses_attention_output_b200 import workloads as W

from _parity import assert_close, run_attn, to_gpu

pytestmark = pytest.mark.gpu

LIMIT_NS = 2_000_000  # 2 ms


@pytest.fixture(scope="module", autouse=True)
def _built(cuda_device):
    from ulysses_attention_output_b200 import build
    build.build()
    xs.load()


def _sm_count() -> int:
    return torch.cuda.get_device_properties(0).multi_processor_count


def _cases():
    # (B, H, S, D, stall_fill): fills of one CTA are Q0, Q1, then K_j, V_j per key tile.
    return [
        (1, 2, 256, 64, 0),    # nothing issued at all
        (1, 2, 1024, 128, 5),  # Q0 Q1 K0 V0 K1 issued, V1 never comes: stall inside the key loop
        (1, 2, 1024, 72, 9),   # later in the key loop, padded head dim
        (1, None, 256, 64, 6),  # first fill of the second item (H set so that items > SMs)
    ]


@pytest.mark.parametrize("B,H,S,D,stall", _cases())
def test_abort_reports_timeout_and_next_call_is_exact(B, H, S, D, stall):
    if H is None:
        H = _sm_count() + 2  # one item per (b, h) at S = 256: two CTAs get a second item
    q, k, v = W.make_qkv(B, H, S, D, seed=900 + S + D + stall)
    qg, kg, vg = to_gpu(q, k, v)
    out = torch.full_like(qg, float("nan"))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    xs.selftest_attn_abort(qg, kg, vg, out, status, stall_fill=stall, limit_ns=LIMIT_NS)
    torch.cuda.synchronize()
    assert int(status.item()) == xs.XS_ERR_TIMEOUT
    # the same process, a normal call: exact against the oracle (sampled heads keep it quick)
    got, st = run_attn(qg, kg, vg)
    assert st == 0
    hs = sorted({0, H // 2, H - 1})
    ref = oracle.attention(q[:, hs], k[:, hs], v[:, hs])
    assert_close(got[:, hs].double().cpu().numpy(), ref, f"after abort {B, H, S, D}")


def test_stall_past_the_last_fill_completes_normally():
    """A stall point no CTA reaches changes nothing: status stays 0 and the output is exact."""
    B, H, S, D = 1, 2, 384, 64
    q, k, v = W.make_qkv(B, H, S, D, seed=77)
    qg, kg, vg = to_gpu(q, k, v)
    out = torch.full_like(qg, float("nan"))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    xs.selftest_attn_abort(qg, kg, vg, out, status, stall_fill=10_000, limit_ns=LIMIT_NS)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert_close(out.double().cpu().numpy(), oracle.attention(q, k, v), "no stall")
