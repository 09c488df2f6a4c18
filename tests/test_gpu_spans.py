"""GPU: the fused call that records store-issue spans (``xs_attn_a2a_fused_spans``) writes the
same slabs as ``xs_attn_a2a_fused`` bit for bit, and its stamps are complete and ordered."""
import numpy as np
import pytest
import torch

import ulysses_attention_output_b200 as xs
from ulysses_attention_output_b200 import burst_gap as bg
from ulysses_attention_output_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built(cuda_device):
    from ulysses_attention_output_b200 import build
    build.build()
    xs.load()


@pytest.mark.parametrize("B,H,S,D,P", [(1, 4, 256, 64, 2), (2, 16, 1024, 72, 4), (1, 8, 4608, 128, 8), (1, 3, 300, 128, 3)])
def test_spans_call_matches_fused_and_stamps_are_ordered(B, H, S, D, P):
    q, k, v = (t.cuda() for t in W.make_qkv(B, H, S, D, seed=S + D))
    d0 = xs.alloc_dest(B, H, S, D, P, device="cuda", fill=float("nan"))
    d1 = xs.alloc_dest(B, H, S, D, P, device="cuda", fill=float("nan"))
    xs.attn_a2a_fused(q, k, v, d0)
    spans = xs.attn_a2a_fused_spans(q, k, v, d1)
    torch.cuda.synchronize()
    for a, b in zip(d0, d1):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    st = spans.cpu().numpy()
    n_items = B * H * ((S + 255) // 256)
    assert st.shape == (n_items, 2, 4, 3)
    assert (st[..., 0] > 0).all() and (st[..., 2] > 0).all()
    assert (st[..., 1] >= st[..., 0]).all()
    r = bg.span_stats(st, min(n_items, torch.cuda.get_device_properties(0).multi_processor_count), ghz=1.9)
    assert r["tiles"] == 2 * n_items and r["span_ns"]["p50"] > 0


def test_spans_buffer_too_small_is_rejected():
    q, k, v = (t.cuda() for t in W.make_qkv(1, 2, 256, 64, seed=1))
    dest = xs.alloc_dest(1, 2, 256, 64, 2, device="cuda")
    small = torch.zeros(10, dtype=torch.int64, device="cuda")
    with pytest.raises(xs.XsError):
        xs.attn_a2a_fused_spans(q, k, v, dest, spans=small)
