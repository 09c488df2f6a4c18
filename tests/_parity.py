"""Helpers shared by the GPU parity tests: run the CUDA path, run the oracle, compare.

Tolerances for bf16 attention outputs against the fp64 oracle: max-abs 2e-2 and relative
L2 5e-3 over every compared element (the bar the workload definition states).  Placement
by the exchange is compared bit for bit.
"""
import numpy as np
import torch

import oracle
import ulysses_attention_output_b200 as xs
from ulysses_attention_output_b200 import workloads as W

TOL_MAX_ABS = 2e-2
TOL_REL_L2 = 5e-3


def errors(got: np.ndarray, ref: np.ndarray) -> tuple[float, float]:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    diff = got - ref
    max_abs = float(np.abs(diff).max()) if diff.size else 0.0
    denom = float(np.linalg.norm(ref))
    rel = float(np.linalg.norm(diff)) / denom if denom > 0 else float(np.linalg.norm(diff))
    return max_abs, rel


def assert_close(got, ref, what=""):
    max_abs, rel = errors(got, ref)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    assert max_abs <= TOL_MAX_ABS and rel <= TOL_REL_L2, (
        f"{what}: max-abs {max_abs:.3e} (tol {TOL_MAX_ABS}), rel-L2 {rel:.3e} (tol {TOL_REL_L2})")
    return max_abs, rel


def to_gpu(*ts):
    return [t.cuda().contiguous() for t in ts]


def run_fused(q, k, v, P, scale=None):
    """q, k, v on the GPU; returns (list of P slabs, status)."""
    B, H, S, D = q.shape
    dest = xs.alloc_dest(B, H, S, D, P, device=q.device, fill=float("nan"))
    status = torch.zeros(1, dtype=torch.int32, device=q.device)
    xs.attn_a2a_fused(q, k, v, dest, scale=scale, status=status)
    torch.cuda.synchronize()
    return dest, int(status.item())


def run_attn(q, k, v, scale=None):
    out = torch.full_like(q, float("nan"))
    status = torch.zeros(1, dtype=torch.int32, device=q.device)
    xs.attn(q, k, v, out, scale=scale, status=status)
    torch.cuda.synchronize()
    return out, int(status.item())


def run_serial(q, k, v, P, scale=None):
    out, st = run_attn(q, k, v, scale)
    B, H, S, D = q.shape
    dest = xs.alloc_dest(B, H, S, D, P, device=q.device, fill=float("nan"))
    xs.a2a_relayout(out, dest)
    torch.cuda.synchronize()
    return dest, out, st


def slabs_f64(dest) -> np.ndarray:
    return torch.stack(dest).double().cpu().numpy()


def gather_rows_from_slabs(dest, w_shape, rows: np.ndarray) -> np.ndarray:
    """Read output rows (b, h, rows[b, h, i]) out of the GPU slabs, at the slots the oracle's
    exchange definition assigns them.  Returns [B, H, n, D] float64."""
    B, H, S, D, P = w_shape
    n = rows.shape[2]
    flat = [d.reshape(-1) for d in dest]
    idx_by_rank = [[] for _ in range(P)]
    where = []
    for b in range(B):
        for h in range(H):
            for i in range(n):
                r, off = oracle.dest_slot(B, H, S, D, P, b, h, int(rows[b, h, i]))
                where.append((r, len(idx_by_rank[r])))
                idx_by_rank[r].append(off)
    pieces = []
    for r in range(P):
        if idx_by_rank[r]:
            base = torch.tensor(idx_by_rank[r], dtype=torch.int64, device=flat[r].device)
            cols = torch.arange(D, device=flat[r].device)
            pieces.append(flat[r][base[:, None] + cols[None, :]].double().cpu().numpy())
        else:
            pieces.append(np.empty((0, D)))
    out = np.empty((B * H * n, D))
    for t, (r, j) in enumerate(where):
        out[t] = pieces[r][j]
    return out.reshape(B, H, n, D)


def workload_inputs(name):
    w = W.WORKLOADS[name]
    return w, W.make_inputs(w)


def rising_scores(B, H, S, D, seed, steps=(0.0, 1.23, 4.7)):
    """Q > 0 and key tile j offset by steps[j]: every row's maximum grows by 18-22 (exp2
    domain, D = 64, S = 384) at the second key tile, below the lazy-rescale threshold of 32
    (P up to ~2^22, no rescale), and the third tile's maximum lies 70-82 above the kept one,
    which rescales O and l."""
    g = torch.Generator().manual_seed(seed)
    q = (1.0 + 0.5 * torch.randn((B, H, S, D), generator=g).abs()).to(torch.bfloat16)
    k = 0.1 * torch.randn((B, H, S, D), generator=g)
    for j, c in enumerate(steps):
        k[:, :, 128 * j:128 * (j + 1)] += c
    k = k.to(torch.bfloat16)
    v = torch.randn((B, H, S, D), generator=g).to(torch.bfloat16)
    return q, k, v
