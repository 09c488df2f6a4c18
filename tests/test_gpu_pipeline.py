"""GPU: the end-to-end HostPipeline (pinned host buffers in and out, head groups overlapped
across copy and compute streams) returns exactly the slabs of the on-device fused call."""
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


@pytest.mark.parametrize("B,H,S,D,P,chunks", [(1, 8, 1024, 128, 4, None), (2, 8, 768, 64, 4, 3),
                                              (1, 6, 300, 72, 3, 1), (2, 4, 512, 128, 2, 4)])
def test_pipeline_matches_device_call(B, H, S, D, P, chunks):
    pipe = xs.HostPipeline(B, H, S, D, P, device="cuda", chunks=chunks)
    dest_h = [torch.full(d.shape, float("nan"), dtype=torch.bfloat16).pin_memory() for d in pipe.dest]
    s = torch.cuda.Stream()
    for step in range(2):  # the second step reuses every buffer
        q, k, v = W.make_qkv(B, H, S, D, seed=100 * step + S)
        qp, kp, vp = (t.pin_memory() for t in (q, k, v))
        pipe.run(qp, kp, vp, dest_h, stream=s)
        s.synchronize()
        assert int(pipe.status.item()) == 0
        ref = xs.alloc_dest(B, H, S, D, P, device="cuda")
        xs.attn_a2a_fused(q.cuda(), k.cuda(), v.cuda(), ref)
        torch.cuda.synchronize()
        for r in range(P):
            assert torch.equal(dest_h[r].view(torch.int16), ref[r].cpu().view(torch.int16)), (step, r)
