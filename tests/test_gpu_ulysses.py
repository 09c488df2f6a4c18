"""Ulysses layer pieces on one GPU (ranks emulated), against the CPU oracle.

* the pre-attention exchange moves every word to the oracle's slot (bit-exact), for all
  heads and for one rank's head range;
* P per-rank fused calls (each rank its heads, writing into all P slabs) produce exactly the
  single fused call's slabs, and leave no slot unwritten;
* a whole layer (pre-exchange per rank -> fused attention + post-exchange per rank) from
  sequence-sharded inputs matches the oracle pipeline a2a_pre -> attention -> a2a_post.
"""
import numpy as np
import pytest
import torch

import oracle
import ulysses_attention_output_b200 as xs
from ulysses_attention_output_b200 import ulysses
from ulysses_attention_output_b200 import workloads as W

from _parity import assert_close, slabs_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built(cuda_device):
    from ulysses_attention_output_b200 import build
    build.build()
    xs.load()


def random_slabs(B, H, S, D, P, seed):
    g = torch.Generator().manual_seed(seed)
    bits = torch.randint(-2**15, 2**15, (P, B, S // P, H, D), generator=g, dtype=torch.int32).to(torch.int16)
    return bits, [bits[r].cuda().contiguous().view(torch.bfloat16) for r in range(P)]


@pytest.mark.parametrize("B,H,S,D,P", [(1, 8, 256, 64, 2), (2, 16, 1024, 72, 4), (1, 24, 4608, 128, 8)])
def test_pre_exchange_bit_exact(B, H, S, D, P):
    bits, slabs = random_slabs(B, H, S, D, P, seed=S + D)
    expect = oracle.a2a_pre(bits.numpy())          # [B, H, S, D]
    full = torch.full((B, H, S, D), -1, dtype=torch.int16, device="cuda").view(torch.bfloat16)
    xs.a2a_pre(slabs, full)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(full.view(torch.int16).cpu().numpy(), expect)
    hl = H // P
    for g in (0, P - 1):
        part = torch.full((B, hl, S, D), -1, dtype=torch.int16, device="cuda").view(torch.bfloat16)
        xs.a2a_pre(slabs, part, heads_local=hl, head_offset=g * hl)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(part.view(torch.int16).cpu().numpy(), expect[:, g * hl:(g + 1) * hl])


@pytest.mark.parametrize("B,H,S,D,P", [(1, 8, 512, 128, 2), (2, 16, 1024, 72, 4), (1, 8, 1000, 64, 8)])
def test_rank_calls_compose_to_the_fused_call(B, H, S, D, P):
    q, k, v = (t.cuda() for t in W.make_qkv(B, H, S, D, seed=21 + S))
    ref = xs.alloc_dest(B, H, S, D, P, device="cuda", fill=float("nan"))
    xs.attn_a2a_fused(q, k, v, ref)
    got = xs.alloc_dest(B, H, S, D, P, device="cuda", fill=float("nan"))
    hl = H // P
    for g in range(P):
        sl = slice(g * hl, (g + 1) * hl)
        xs.attn_a2a_fused_rank(q[:, sl].contiguous(), k[:, sl].contiguous(), v[:, sl].contiguous(), got,
                               heads_total=H, head_offset=g * hl)
    torch.cuda.synchronize()
    for a, b in zip(ref, got):
        assert torch.isfinite(b.float()).all(), "a slot was left unwritten"
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))


@pytest.mark.parametrize("B,H,S,D,P", [(1, 8, 512, 128, 4), (2, 16, 1024, 72, 4)])
def test_whole_layer_matches_oracle(B, H, S, D, P):
    q, k, v = W.make_qkv(B, H, S, D, seed=5 + D)
    # sequence-sharded inputs, as the layer receives them: slab r = rows [r S/P, (r+1) S/P)
    shard = lambda x: [t.cuda().contiguous() for t in torch.from_numpy(
        oracle.a2a_post(x.view(torch.int16).numpy(), P)).view(torch.bfloat16)]
    qs, ks, vs = shard(q), shard(k), shard(v)
    out = xs.alloc_dest(B, H, S, D, P, device="cuda", fill=float("nan"))
    ulysses.layer_on_one_gpu(qs, ks, vs, out)
    torch.cuda.synchronize()
    # oracle pipeline: a2a_pre of the shards (= the original head-major tensors), attention,
    # a2a_post
    q_hm = oracle.a2a_pre(np.stack([t.view(torch.int16).cpu().numpy() for t in qs]))
    assert (q_hm == q.view(torch.int16).numpy()).all()
    ref = oracle.a2a_post(oracle.attention(q, k, v), P)
    assert_close(slabs_f64(out), ref, "Ulysses layer")
