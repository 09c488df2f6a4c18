"""GPU parity of partial attention with log-sum-exp and of the online-softmax merge (the
Route primitive) against the CPU oracle (B200, sm_100a).

* partial attention over one key/value shard (any key count, ragged, or none) matches the
  oracle's O within the attention tolerances and its lse within LSE_TOL;
* over the full key set its fp32 output, rounded to bf16, equals ``xs_attn`` bit for bit;
* the merge kernel matches the oracle's merge on seeded synthetic parts (empty parts, rows
  whose parts are all empty, up to 16 parts) within one bf16 rounding;
* partial attention per owner + merge equals attention over the union of the shards, every
  row of a small ragged case and sampled rows of the batched-dispatch workload.

LSE_TOL: the kernel sums the probabilities after rounding them to bf16 (relative error
at most 2^-9 each, so at most 2^-9 on their sum) and evaluates exp2 with MUFU or a
polynomial of relative error 1.0e-4; fp32 rounding of the scores adds ~1e-6.  So
|lse_gpu - lse| <= 2^-9 + 1e-4 + 1e-6 ~= 2.1e-3; the bound used is 4e-3.
"""
import numpy as np
import pytest
import torch

import oracle
import ulysses_attention_output_b200 as xs
from ulysses_attention_output_b200 import workloads as W

from _parity import assert_close, errors, rising_scores, run_attn

pytestmark = pytest.mark.gpu

LSE_TOL = 4e-3


@pytest.fixture(scope="module", autouse=True)
def _built(cuda_device):
    from ulysses_attention_output_b200 import build
    build.build()
    xs.load()


def _draw(shape, g):
    return torch.randn(shape, generator=g, dtype=torch.float32).to(torch.bfloat16)


def _partial_gpu(q, k, v, scale=None):
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o = torch.full(tuple(q.shape), float("nan"), dtype=torch.float32, device="cuda")
    lse = torch.full(tuple(q.shape[:3]), float("nan"), dtype=torch.float32, device="cuda")
    xs.attn_partial(q.cuda(), k.cuda(), v.cuda(), o, lse, scale=scale, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return o.cpu().double().numpy(), lse.cpu().double().numpy()


def _check_lse(got, ref, what):
    assert np.isfinite(got).all(), f"{what}: non-finite lse"
    err = float(np.abs(got - ref).max())
    assert err <= LSE_TOL, f"{what}: lse max-abs error {err:.3e} (tol {LSE_TOL})"


# ----------------------------------------------------------------------------- partial
@pytest.mark.parametrize("B,H,Sq,Skv,D,scale", [
    (1, 2, 256, 384, 64, None),     # whole tiles
    (1, 2, 200, 333, 72, None),     # ragged queries and keys, padded D
    (2, 1, 130, 1, 128, None),      # a single key
    (1, 3, 64, 129, 128, 0.2),      # one key past a tile, custom scale
    (1, 2, 300, 1000, 128, None),   # several key tiles, ragged
])
def test_partial_matches_oracle(B, H, Sq, Skv, D, scale):
    g = torch.Generator().manual_seed(Sq * 7 + Skv)
    q, k, v = _draw((B, H, Sq, D), g), _draw((B, H, Skv, D), g), _draw((B, H, Skv, D), g)
    o, lse = _partial_gpu(q, k, v, scale)
    ro, rl = oracle.attention_partial(q, k, v, scale=scale)
    assert_close(o, ro, f"partial O {B, H, Sq, Skv, D}")
    _check_lse(lse, rl, f"partial lse {B, H, Sq, Skv, D}")


def test_partial_with_rescale_matches_oracle():
    """Partial attention whose row maxima move below, then above the lazy-rescale threshold
    (``rising_scores``): O and the lse match the oracle."""
    q, k, v = rising_scores(1, 2, 384, 64, seed=33)
    ref_o, ref_l = oracle.attention_partial(q, k, v)
    o, lse = _partial_gpu(q, k, v)
    assert_close(o, ref_o, "partial rescale O")
    _check_lse(lse, ref_l, "partial rescale")


def test_partial_empty_shard():
    g = torch.Generator().manual_seed(5)
    q = _draw((1, 2, 70, 64), g)
    empty = torch.empty((1, 2, 0, 64), dtype=torch.bfloat16)
    o, lse = _partial_gpu(q, empty, empty)
    assert (o == 0).all() and np.isneginf(lse).all()


def test_partial_over_all_keys_equals_attn_bits():
    g = torch.Generator().manual_seed(9)
    q, k, v = (_draw((1, 3, 333, 128), g) for _ in range(3))
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    o, _ = xs.attn_partial(qc, kc, vc)
    ref, st = run_attn(qc, kc, vc)
    assert st == 0
    torch.cuda.synchronize()
    assert torch.equal(o.to(torch.bfloat16).view(torch.int16), ref.view(torch.int16))


# ----------------------------------------------------------------------------- merge
@pytest.mark.parametrize("n,rows,D", [(1, 1000, 128), (3, 777, 72), (16, 300, 8), (4, 4096, 128)])
def test_merge_matches_oracle(n, rows, D):
    g = torch.Generator().manual_seed(n * 100 + D)
    o = torch.randn((n, rows, D), generator=g, dtype=torch.float32)
    lse = torch.randn((n, rows), generator=g, dtype=torch.float32) * 3
    empty = torch.rand((n, rows), generator=g) < 0.2
    lse[empty] = float("-inf")
    lse[:, 5] = float("-inf")  # a row whose parts are all empty
    o[empty] = 0.0
    ro, rl = oracle.lse_merge(o.double().numpy(), lse.double().numpy())
    parts = [o[t].cuda() for t in range(n)]
    lparts = [lse[t].cuda() for t in range(n)]
    out, lse_out = xs.lse_merge(parts, lparts)
    torch.cuda.synchronize()
    got = out.double().cpu().numpy()
    # one bf16 rounding (half an ulp, <= 2^-8 relative) of an fp32 result whose own error is
    # a few fp32 roundings of the weighted sum of magnitudes sum_t w_t |o_t| / W (terms of
    # opposite sign cancel, so that error is not relative to |O|); the magnitude sum is the
    # oracle's merge of |o_t|.
    mag, _ = oracle.lse_merge(np.abs(o.double().numpy()), lse.double().numpy())
    bound = 2.0 ** -8 * np.abs(ro) + (n + 4) * 2.0 ** -23 * mag
    assert (np.abs(got - ro) <= bound).all(), f"merge O: worst {np.max(np.abs(got - ro) - bound):.3e} over"
    gl = lse_out.double().cpu().numpy()
    fin = np.isfinite(rl)
    assert (np.isneginf(gl) == ~fin).all()
    assert np.abs(gl[fin] - rl[fin]).max() <= 1e-5 * (1 + np.abs(rl[fin])).max()
    assert (got[5] == 0).all()
    # an empty part's O is ignored whatever it holds (NaN here): same bits as with zeros
    parts_nan = [p.clone() for p in parts]
    for t in range(n):
        parts_nan[t][empty[t].cuda()] = float("nan")
    out2, _ = xs.lse_merge(parts_nan, lparts, lse_out=False)
    torch.cuda.synchronize()
    assert torch.equal(out2.view(torch.int16), out.view(torch.int16))


# ----------------------------------------------------------------------------- route
def _route_gpu(w):
    q, ks, vs = W.make_route_inputs(w)
    qc = q.cuda()
    parts = [xs.attn_partial(qc, k.cuda(), v.cuda()) for k, v in zip(ks, vs)]
    out, lse = xs.lse_merge([p[0] for p in parts], [p[1] for p in parts])
    torch.cuda.synchronize()
    return q, ks, vs, out, lse


def test_route_tiny_every_row():
    w = W.ROUTE_WORKLOADS["route_tiny"]
    q, ks, vs, out, lse = _route_gpu(w)
    k_all, v_all = torch.cat(ks, dim=2), torch.cat(vs, dim=2)
    ro, rl = oracle.attention_partial(q, k_all, v_all)
    assert_close(out.double().cpu().numpy(), ro, "route_tiny merged O")
    _check_lse(lse.double().cpu().numpy(), rl, "route_tiny merged lse")


def test_route_sampled_full_size():
    w = W.ROUTE_WORKLOADS["route"]
    q, ks, vs, out, lse = _route_gpu(w)
    rows = W.sample_route_rows(w).numpy()
    k_all, v_all = torch.cat(ks, dim=2), torch.cat(vs, dim=2)
    ro, rl = oracle.attention_partial(q, k_all, v_all, rows=rows)
    got = out.double().cpu().numpy()
    gl = lse.double().cpu().numpy()
    got_rows = np.take_along_axis(got, rows[..., None].astype(np.int64), axis=2)
    gl_rows = np.take_along_axis(gl, rows.astype(np.int64), axis=2)
    max_abs, rel = assert_close(got_rows, ro, "route merged O (sampled rows)")
    _check_lse(gl_rows, rl, "route merged lse (sampled rows)")
    assert np.isfinite(got).all()
