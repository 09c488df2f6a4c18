"""GPU: the fused call can be captured in a CUDA graph (after one eager call on the device,
which sets the kernel's shared-memory attribute) and replayed with new inputs copied into the
captured buffers; every replay equals the eager call bit for bit."""
import pytest
import torch

import ulysses_attention_output_b200 as xs
from ulysses_attention_output_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built(cuda_device):
    from ulysses_attention_output_b200 import build
    build.build()
    xs.load()


@pytest.mark.parametrize("B,H,S,D,P", [(1, 4, 256, 64, 2), (1, 8, 1024, 128, 4), (2, 16, 1024, 72, 4)])
def test_fused_call_replays_from_a_cuda_graph(B, H, S, D, P):
    q = torch.empty((B, H, S, D), dtype=torch.bfloat16, device="cuda")
    k, v = torch.empty_like(q), torch.empty_like(q)
    dest = xs.alloc_dest(B, H, S, D, P, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    qi, ki, vi = W.make_qkv(B, H, S, D, seed=5)
    q.copy_(qi); k.copy_(ki); v.copy_(vi)
    xs.attn_a2a_fused(q, k, v, dest, status=status)  # eager first: per-device setup
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            xs.attn_a2a_fused(q, k, v, dest, stream=s, status=status)
    torch.cuda.synchronize()
    for seed in (11, 12):
        qi, ki, vi = W.make_qkv(B, H, S, D, seed=seed)
        q.copy_(qi); k.copy_(ki); v.copy_(vi)
        for d in dest:
            d.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        ref = xs.alloc_dest(B, H, S, D, P, device="cuda")
        xs.attn_a2a_fused(q, k, v, ref)
        torch.cuda.synchronize()
        for a, b in zip(dest, ref):
            assert torch.equal(a.view(torch.int16), b.view(torch.int16))
