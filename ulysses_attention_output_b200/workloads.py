"""Seeded synthetic workloads for DiT self-attention + Ulysses post-attention All-to-All.

This module only draws inputs: it holds none of the attention or exchange arithmetic, so
both the CUDA path and the CPU oracle consume the very same arrays.

Every tensor is drawn on the CPU with a ``torch.Generator`` seeded per workload, as fp32
N(0, 1) in the [B, H, S, D] layout, in the order Q, K, V, and then rounded to bf16
(round-to-nearest-even).  Structure is added per workload:

* ``qknorm``   -- Q and K rows RMS-normalised over D (epsilon 1e-6) and multiplied by a
                  per-head gain vector gamma_h in R^D drawn iid N(1, 0.1^2), separately for
                  Q and K (the QK-norm used by MMDiT-style joint image+text models).
* ``outliers`` -- after the bf16 cast, floor(0.01 * S) key rows per (b, h), drawn uniformly
                  without replacement, are multiplied by 8 (exact in bf16: a power of two),
                  stressing the softmax running-max tracking.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    S: int
    D: int
    P: int
    structure: str = "iid"          # "iid" | "qknorm" | "outliers"
    seed: int = 0
    sampled_rows: int = 0           # 0: every query row is checked against the oracle
    description: str = field(default="", compare=False)

    @property
    def flops(self) -> int:
        """Algorithmic FLOPs of one attention pass: 4 * B * H * S^2 * D (true D)."""
        return 4 * self.B * self.H * self.S * self.S * self.D

    @property
    def qkv_bytes(self) -> int:
        return 3 * self.B * self.H * self.S * self.D * 2

    @property
    def out_bytes(self) -> int:
        return self.B * self.H * self.S * self.D * 2

    def shape(self) -> tuple[int, int, int, int]:
        return (self.B, self.H, self.S, self.D)


# The five workloads: the tiny check, a DiT-XL/2 (512 px) layer, an MMDiT joint
# image+text layer with QK-norm, a long-sequence image DiT layer with outlier keys and a
# video-DiT-scale layer.
WORKLOADS: dict[str, Workload] = {
    "tiny": Workload("tiny", 1, 4, 256, 64, 2, "iid", 1000, 0,
                     "tiny check: B=1 H=4 S=256 D=64, 2 virtual ranks"),
    "ditxl": Workload("ditxl", 2, 16, 1024, 72, 4, "iid", 1001, 0,
                      "DiT-XL/2 512px-like: B=2 H=16 S=1024 D=72 (hidden 1152), 4 ranks"),
    "mmdit": Workload("mmdit", 1, 24, 4608, 128, 8, "qknorm", 1002, 0,
                      "MMDiT-like joint image+text: B=1 H=24 S=4608 (4096+512) D=128, QK-norm, 8 ranks"),
    "long": Workload("long", 1, 24, 16384, 128, 8, "outliers", 1003, 256,
                     "long-sequence image DiT: B=1 H=24 S=16384 D=128, 1% keys x8, 8 ranks"),
    "video": Workload("video", 1, 40, 32768, 128, 8, "iid", 1004, 256,
                      "video-DiT-scale: B=1 H=40 S=32768 D=128, 8 ranks"),
}
ORDER = ["tiny", "ditxl", "mmdit", "long", "video"]


def _to_bf16(x: torch.Tensor) -> torch.Tensor:
    return x.to(torch.bfloat16)


def make_qkv(B: int, H: int, S: int, D: int, seed: int, structure: str = "iid"):
    """Draw (q, k, v) as contiguous bf16 CPU tensors of shape [B, H, S, D]."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    shape = (B, H, S, D)
    q = torch.randn(shape, generator=g, dtype=torch.float32)
    k = torch.randn(shape, generator=g, dtype=torch.float32)
    v = torch.randn(shape, generator=g, dtype=torch.float32)
    if structure == "qknorm":
        gamma_q = 1.0 + 0.1 * torch.randn((H, D), generator=g, dtype=torch.float32)
        gamma_k = 1.0 + 0.1 * torch.randn((H, D), generator=g, dtype=torch.float32)
        q = q * torch.rsqrt(q.pow(2).mean(dim=-1, keepdim=True) + 1e-6) * gamma_q[None, :, None, :]
        k = k * torch.rsqrt(k.pow(2).mean(dim=-1, keepdim=True) + 1e-6) * gamma_k[None, :, None, :]
    q, k, v = _to_bf16(q), _to_bf16(k), _to_bf16(v)
    if structure == "outliers":
        n_out = (S * 1) // 100
        if n_out > 0:
            for b in range(B):
                for h in range(H):
                    idx = torch.randperm(S, generator=g)[:n_out]
                    k[b, h, idx, :] = k[b, h, idx, :] * 8
    elif structure not in ("iid", "qknorm"):
        raise ValueError(f"unknown input structure {structure!r}")
    return q.contiguous(), k.contiguous(), v.contiguous()


def make_inputs(w: Workload):
    """(q, k, v) of a named workload."""
    return make_qkv(w.B, w.H, w.S, w.D, w.seed, w.structure)


def sample_rows(w: Workload, n: int | None = None, seed: int | None = None) -> torch.Tensor:
    """Query rows to check per (b, h): int32 [B, H, n], sorted.

    Drawn uniformly without replacement per (b, h) from a generator seeded with
    1234 + the workload's index, and always containing row 0, row S-1 and both rows at
    every rank boundary (r*S/P - 1 and r*S/P).
    """
    n = w.sampled_rows if n is None else n
    if seed is None:
        seed = 1234 + (ORDER.index(w.name) if w.name in ORDER else 0)
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    Sl = w.S // w.P
    forced = {0, w.S - 1}
    for r in range(1, w.P):
        forced.add(r * Sl - 1)
        forced.add(r * Sl)
    forced = sorted(forced)
    n = max(n, len(forced))
    out = torch.empty((w.B, w.H, n), dtype=torch.int32)
    for b in range(w.B):
        for h in range(w.H):
            perm = torch.randperm(w.S, generator=g)
            chosen = list(forced)
            seen = set(chosen)
            for i in perm.tolist():
                if len(chosen) >= n:
                    break
                if i not in seen:
                    chosen.append(i)
                    seen.add(i)
            out[b, h] = torch.tensor(sorted(chosen), dtype=torch.int32)
    return out


# ----------------------------------------------------------------------------- Route workloads
@dataclass(frozen=True)
class RouteWorkload:
    """Partial attention of routed query rows over KV shards held by several owners, merged by
    online softmax (the Route primitive).  ``shards`` lists each owner's key count."""
    name: str
    B: int
    H: int
    Sq: int
    shards: tuple
    D: int
    seed: int = 0
    sampled_rows: int = 0           # 0: every query row is checked against the oracle
    description: str = field(default="", compare=False)

    @property
    def S_kv(self) -> int:
        return int(sum(self.shards))

    @property
    def flops(self) -> int:
        """Algorithmic FLOPs of the partial attentions: 4 * B * H * Sq * S_kv * D."""
        return 4 * self.B * self.H * self.Sq * self.S_kv * self.D

    @property
    def merge_bytes(self) -> int:
        """Algorithmic bytes of the merge: every part's fp32 O and lse read, bf16 O and fp32
        lse written."""
        rows = self.B * self.H * self.Sq
        return len(self.shards) * rows * (4 * self.D + 4) + rows * (2 * self.D + 4)


ROUTE_WORKLOADS: dict[str, RouteWorkload] = {
    "route_tiny": RouteWorkload("route_tiny", 1, 2, 300, (256, 0, 411, 333), 128, 1005, 0,
                                "Route check: 300 query rows, 4 owners (one empty), ragged shards"),
    "route": RouteWorkload("route", 1, 32, 1024, (8192, 8192, 8192, 8192), 128, 1006, 64,
                           "Route batched dispatch: B=1 H=32, 1024 query rows per head, "
                           "4 owners x 8192 keys, D=128"),
}


def make_route_inputs(w: RouteWorkload):
    """(q, [k_t], [v_t]) as contiguous bf16 CPU tensors: q [B, H, Sq, D], then per shard t
    k_t and v_t [B, H, shards[t], D], all drawn fp32 N(0, 1) in that order and rounded."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(w.seed))
    q = torch.randn((w.B, w.H, w.Sq, w.D), generator=g, dtype=torch.float32).to(torch.bfloat16)
    ks, vs = [], []
    for n in w.shards:
        ks.append(torch.randn((w.B, w.H, n, w.D), generator=g, dtype=torch.float32).to(torch.bfloat16))
        vs.append(torch.randn((w.B, w.H, n, w.D), generator=g, dtype=torch.float32).to(torch.bfloat16))
    return q.contiguous(), ks, vs


def sample_route_rows(w: RouteWorkload, n: int | None = None, seed: int = 4321) -> torch.Tensor:
    """Query rows to check per (b, h): int32 [B, H, n], sorted, always with rows 0 and Sq-1."""
    n = max(2, w.sampled_rows if n is None else n)
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    out = torch.empty((w.B, w.H, n), dtype=torch.int32)
    for b in range(w.B):
        for h in range(w.H):
            rest = [i for i in torch.randperm(w.Sq, generator=g).tolist() if i not in (0, w.Sq - 1)]
            out[b, h] = torch.tensor(sorted([0, w.Sq - 1] + rest[:n - 2]), dtype=torch.int32)
    return out
