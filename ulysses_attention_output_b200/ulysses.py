"""Host-side plan of a Ulysses sequence-parallel attention layer over P ranks.

Before the layer, rank g holds the sequence shard s in [g*S/P, (g+1)*S/P) of Q, K and V for
all H heads ([B, S/P, H, D]).  The pre-attention exchange gives rank g all S rows of its
H/P heads ([B, H/P, S, D]); attention runs per head; the post-attention exchange (fused into
the attention kernel's epilogue here) returns every rank its sequence shard of all heads.
This module holds only the index plan; the data movement and arithmetic are in libxs.so
(``a2a_pre``, ``attn_a2a_fused_rank``).
"""
from __future__ import annotations

from dataclasses import dataclass


@dataclass(frozen=True)
class RankPlan:
    rank: int
    world: int
    heads_total: int
    head_offset: int
    heads_local: int
    seq_offset: int
    seq_local: int


def rank_plan(rank: int, world: int, heads_total: int, seq_len: int) -> RankPlan:
    """Heads and sequence rows owned by ``rank`` (Ulysses needs H % P == 0, S % P == 0)."""
    if world <= 0 or not 0 <= rank < world:
        raise ValueError("rank must lie in [0, world)")
    if heads_total % world or seq_len % world:
        raise ValueError("Ulysses sharding needs H % P == 0 and S % P == 0")
    hl, sl = heads_total // world, seq_len // world
    return RankPlan(rank, world, heads_total, rank * hl, hl, rank * sl, sl)


def layer_on_one_gpu(q_slabs, k_slabs, v_slabs, out_slabs, scale=None, stream=None):
    """Run a whole Ulysses layer with the P ranks emulated on one GPU: per rank, the
    pre-attention exchange of its heads, then its fused attention + post-attention exchange
    into the shared output slabs.  All inputs and outputs are lists of P slabs
    [B, S/P, H, D] (bf16); the per-rank head-major buffers are allocated here."""
    import torch

    import ulysses_attention_output_b200 as xs
    P = len(q_slabs)
    B, Sl, H, D = (int(x) for x in q_slabs[0].shape)
    S = Sl * P
    for g in range(P):
        plan = rank_plan(g, P, H, S)
        qkv = []
        for slabs in (q_slabs, k_slabs, v_slabs):
            t = torch.empty((B, plan.heads_local, S, D), dtype=torch.bfloat16, device=slabs[0].device)
            xs.a2a_pre(slabs, t, heads_local=plan.heads_local, head_offset=plan.head_offset,
                       stream=stream)
            qkv.append(t)
        xs.attn_a2a_fused_rank(*qkv, out_slabs, heads_total=H, head_offset=plan.head_offset,
                               scale=scale, stream=stream)
