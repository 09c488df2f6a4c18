"""Pins of the oracle's partial attention (with log-sum-exp) and of its merge (CPU only).

Partial attention of query rows over one key/value shard returns ``(O, lse)`` with
``lse = log sum_j exp(s_j)``; the merge combines the results of disjoint shards with an
online softmax (the Route primitive of "Move the Query, Not the Cache: Characterizing
Cross-Instance Latent Attention Redistribution Across GPU Fabrics", "Methodik" ->
"Primitiv-Vergleich").  The pins use closed forms (one key, Q = 0, equal scores, equal
weights), ``scipy.special.logsumexp`` and ``scipy.special.softmax`` as independent library
routines, and the identity that merging the parts of a key split gives attention over the
union of the keys.  ``test_planted_mistakes_are_caught`` compiles mutated copies of the oracle
source and requires the pins to reject each of them.
"""
import ctypes
import os
import subprocess
import tempfile

import numpy as np
import pytest
from scipy.special import logsumexp
from scipy.special import softmax as scipy_softmax

import oracle


def scipy_partial(q, k, v, scale):
    s = np.einsum("bhid,bhjd->bhij", q, k) * scale
    return np.einsum("bhij,bhjd->bhid", scipy_softmax(s, axis=-1), v), logsumexp(s, axis=-1)


def partial_pins(partial):
    """``partial(q, k, v, scale) -> (o, lse)``; raises AssertionError on a mismatch."""
    rng = np.random.default_rng(11)
    # 1. brute force against scipy, Sq != Skv, several heads and batches
    for (B, H, Sq, Skv, D) in [(1, 1, 1, 1, 1), (2, 3, 5, 9, 3), (1, 2, 7, 16, 8), (1, 1, 13, 4, 72)]:
        q = rng.standard_normal((B, H, Sq, D)) * 1.5
        k = rng.standard_normal((B, H, Skv, D)) * 1.5
        v = rng.standard_normal((B, H, Skv, D))
        o, lse = partial(q, k, v, None)
        eo, else_ = scipy_partial(q, k, v, 1.0 / np.sqrt(D))
        np.testing.assert_allclose(o, eo, atol=1e-12, rtol=0)
        np.testing.assert_allclose(lse, else_, atol=1e-12, rtol=1e-13)
    # 2. one key: lse = scale * q.k exactly, O = that value row
    q = rng.standard_normal((1, 2, 3, 4))
    k = rng.standard_normal((1, 2, 1, 4))
    v = rng.standard_normal((1, 2, 1, 4))
    o, lse = partial(q, k, v, 0.5)
    np.testing.assert_allclose(lse, 0.5 * np.einsum("bhid,bhjd->bhi", q, k), atol=1e-14, rtol=0)
    np.testing.assert_allclose(o, np.broadcast_to(v, o.shape), atol=1e-15, rtol=0)
    # 3. Q = 0: every score is 0, lse = log(Skv), O = mean of V
    q = np.zeros((1, 1, 2, 4))
    k = rng.standard_normal((1, 1, 10, 4))
    v = rng.standard_normal((1, 1, 10, 4))
    o, lse = partial(q, k, v, None)
    np.testing.assert_allclose(lse, np.log(10.0), atol=1e-15, rtol=0)
    np.testing.assert_allclose(o, np.broadcast_to(v.mean(axis=2, keepdims=True), o.shape), atol=1e-14)
    # 4. identical keys: lse = s + log(Skv) for the common score s (scale 1 here)
    q = rng.standard_normal((1, 1, 3, 5))
    k = np.broadcast_to(rng.standard_normal(5), (1, 1, 6, 5)).copy()
    v = rng.standard_normal((1, 1, 6, 5))
    o, lse = partial(q, k, v, 1.0)
    np.testing.assert_allclose(lse[0, 0], q[0, 0] @ k[0, 0, 0] + np.log(6.0), atol=1e-13, rtol=0)
    # 5. large scores (hundreds): no overflow, still scipy's values
    q = rng.standard_normal((1, 1, 4, 8)) * 30
    k = rng.standard_normal((1, 1, 9, 8)) * 30
    v = rng.standard_normal((1, 1, 9, 8))
    o, lse = partial(q, k, v, None)
    eo, else_ = scipy_partial(q, k, v, 1.0 / np.sqrt(8))
    assert np.isfinite(lse).all() and np.isfinite(o).all()
    np.testing.assert_allclose(o, eo, atol=1e-12, rtol=0)
    np.testing.assert_allclose(lse, else_, atol=0, rtol=1e-13)
    # 6. an empty shard: O = 0, lse = -inf
    o, lse = partial(rng.standard_normal((1, 2, 3, 4)), np.zeros((1, 2, 0, 4)), np.zeros((1, 2, 0, 4)), None)
    assert (o == 0).all() and np.isneginf(lse).all()


def merge_pins(merge, partial):
    """``merge(o_parts, lse_parts) -> (o, lse)``; uses ``partial`` for the split identity."""
    rng = np.random.default_rng(12)
    # 1. a key split (one shard empty) merged = attention over all keys (scipy)
    B, H, Sq, S, D = 1, 2, 6, 23, 8
    q = rng.standard_normal((B, H, Sq, D)) * 2
    k = rng.standard_normal((B, H, S, D)) * 2
    v = rng.standard_normal((B, H, S, D))
    cuts = [0, 5, 5, 17, S]  # shards [0,5), [5,5) empty, [5,17), [17,23)
    parts = [partial(q, k[:, :, a:b], v[:, :, a:b], None) for a, b in zip(cuts[:-1], cuts[1:])]
    o, lse = merge(np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]))
    eo, else_ = scipy_partial(q, k, v, 1.0 / np.sqrt(D))
    np.testing.assert_allclose(o, eo, atol=1e-12, rtol=0)
    np.testing.assert_allclose(lse, else_, atol=1e-12, rtol=0)
    # 2. one part: the identity
    o1 = rng.standard_normal((3, 4))
    l1 = rng.standard_normal(3) * 5
    o, lse = merge(o1[None], l1[None])
    np.testing.assert_allclose(o, o1, atol=1e-15, rtol=0)
    np.testing.assert_allclose(lse, l1, atol=1e-15, rtol=0)
    # 3. a part at -inf has no weight; all parts at -inf give O = 0, lse = -inf
    o2 = rng.standard_normal((3, 4))
    o, lse = merge(np.stack([o2, o1]), np.stack([np.full(3, -np.inf), l1]))
    np.testing.assert_allclose(o, o1, atol=1e-15, rtol=0)
    np.testing.assert_allclose(lse, l1, atol=1e-15, rtol=0)
    o, lse = merge(np.stack([o1, o2]), np.full((2, 3), -np.inf))
    assert (o == 0).all() and np.isneginf(lse).all()
    # 4. equal weights: the mean, lse + log 2; weights 1 : 1/3 at lse near 1000 (no overflow)
    o, lse = merge(np.stack([o1, o2]), np.stack([l1, l1]))
    np.testing.assert_allclose(o, (o1 + o2) / 2, atol=1e-15, rtol=0)
    np.testing.assert_allclose(lse, l1 + np.log(2.0), atol=1e-14, rtol=0)
    big = np.full(3, 1000.0)
    o, lse = merge(np.stack([o1, o2]), np.stack([big, big - np.log(3.0)]))
    # (1000 - log 3 is rounded at an ulp of 1.1e-13, hence the looser bound)
    np.testing.assert_allclose(o, (o1 + o2 / 3) / (4 / 3), atol=1e-12, rtol=0)
    np.testing.assert_allclose(lse, 1000.0 + np.log(4 / 3), atol=1e-12, rtol=0)
    # 5. the order of the parts does not matter
    o3 = rng.standard_normal((3, 4))
    l3 = rng.standard_normal(3)
    a = merge(np.stack([o1, o2, o3]), np.stack([l1, l1 - 1, l3]))
    b = merge(np.stack([o3, o1, o2]), np.stack([l3, l1, l1 - 1]))
    np.testing.assert_allclose(a[0], b[0], atol=1e-14, rtol=0)
    np.testing.assert_allclose(a[1], b[1], atol=1e-14, rtol=0)


def test_partial_pins():
    partial_pins(lambda q, k, v, s: oracle.attention_partial(q, k, v, scale=s))


def test_merge_pins():
    merge_pins(oracle.lse_merge, lambda q, k, v, s: oracle.attention_partial(q, k, v, scale=s))


def test_partial_rows_subset_and_full_shard():
    rng = np.random.default_rng(3)
    q = rng.standard_normal((2, 2, 9, 8))
    k = rng.standard_normal((2, 2, 9, 8))
    v = rng.standard_normal((2, 2, 9, 8))
    o, lse = oracle.attention_partial(q, k, v)
    # over the whole key set, O is the attention oracle's output
    np.testing.assert_array_equal(o, oracle.attention(q, k, v))
    rows = np.array([8, 0, 4])
    os_, ls = oracle.attention_partial(q, k, v, rows=rows)
    np.testing.assert_array_equal(os_, o[:, :, rows])
    np.testing.assert_array_equal(ls, lse[:, :, rows])


def test_partial_rejects_bad_shapes():
    with pytest.raises(ValueError):
        oracle.attention_partial(np.zeros((1, 1, 2, 4)), np.zeros((1, 1, 3, 5)), np.zeros((1, 1, 3, 5)))
    with pytest.raises(ValueError):
        oracle.lse_merge(np.zeros((2, 3, 4)), np.zeros((2, 4)))


# ----------------------------------------------------------------------------- mutants
MUTANTS = {
    # the row maximum left out of the log-sum-exp
    "lse_no_max": ("*lse = m + log(l);", "*lse = log(l);"),
    # a base-2 logarithm instead of the natural one
    "lse_log2": ("*lse = m + log(l);", "*lse = m + log2(l);"),
    # merge weights with the exponent's sign flipped
    "merge_sign": ("const double w = exp(lse_parts[(size_t)t * R + r] - M);",
                   "const double w = exp(M - lse_parts[(size_t)t * R + r]);"),
    # merged O not divided by the total weight
    "merge_no_norm": ("for (int d = 0; d < D; ++d) o[d] /= W;", ""),
    # merged lse without the maximum
    "merge_lse_no_max": ("if (lse_out) lse_out[r] = M + log(W);", "if (lse_out) lse_out[r] = log(W);"),
    # the last part skipped
    "merge_drop_part": ("for (int t = 0; t < n; ++t) {\n      const double w",
                        "for (int t = 0; t < n - 1; ++t) {\n      const double w"),
}


def _mutant_fns(so_path):
    lib = ctypes.CDLL(so_path)
    dp = ctypes.POINTER(ctypes.c_double)
    ci = ctypes.c_int
    lib.xs_oracle_attention_partial.argtypes = [dp, dp, dp, ci, ci, ci, ci, ci, ctypes.c_double,
                                                ctypes.POINTER(ctypes.c_int32), ci, dp, dp, ci]
    lib.xs_oracle_lse_merge.argtypes = [dp, dp, ci, ctypes.c_longlong, ci, dp, dp]
    p = lambda a: a.ctypes.data_as(dp)

    def partial(q, k, v, scale):
        q, k, v = (np.ascontiguousarray(x, dtype=np.float64) for x in (q, k, v))
        B, H, Sq, D = q.shape
        Skv = k.shape[2]
        scale = 1.0 / np.sqrt(D) if scale is None else scale
        out = np.empty_like(q)
        lse = np.empty((B, H, Sq))
        kk = k if Skv else np.zeros(1)
        vv = v if Skv else np.zeros(1)
        rc = lib.xs_oracle_attention_partial(p(q), p(kk), p(vv), B, H, Sq, Skv, D, float(scale),
                                             ctypes.POINTER(ctypes.c_int32)(), Sq, p(out), p(lse), 1)
        assert rc == 0
        return out, lse

    def merge(o_parts, lse_parts):
        o = np.ascontiguousarray(o_parts, dtype=np.float64)
        ls = np.ascontiguousarray(lse_parts, dtype=np.float64)
        n, D = o.shape[0], o.shape[-1]
        lead = o.shape[1:-1]
        R = int(np.prod(lead)) if lead else 1
        out = np.empty(lead + (D,))
        lse = np.empty(lead)
        assert lib.xs_oracle_lse_merge(p(o), p(ls), n, R, D, p(out), p(lse)) == 0
        return out, lse
    return partial, merge


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistakes_are_caught(name):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "xs_oracle.c")).read()
    old, new = MUTANTS[name]
    assert src.count(old) == 1, f"mutation site for {name} not unique"
    mutated = src.replace(old, new)
    with tempfile.TemporaryDirectory() as tmp:
        c_path = os.path.join(tmp, f"{name}.c")
        so_path = os.path.join(tmp, f"{name}.so")
        open(c_path, "w").write(mutated)
        subprocess.run(["gcc", "-O2", "-fPIC", "-shared", "-o", so_path, c_path, "-lm"], check=True)
        partial, merge = _mutant_fns(so_path)
        with pytest.raises(AssertionError):
            with np.errstate(all="ignore"):
                partial_pins(partial)
                merge_pins(merge, partial)
