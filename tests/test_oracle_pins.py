"""Pins of the CPU oracle to facts that do not come from the oracle itself (CPU only).

Each check below would fail for a plausible slip in ``oracle/xs_oracle.c`` (a dropped
term, a wrong sign, a transposed operand, a wrong index or scale).
``test_planted_mistakes_are_caught`` proves it: it compiles mutated copies of the oracle
source and requires the pins to reject every one.

Sources: closed forms and hand-derived fixtures in ``tests/golden/`` (softmax attention
definition; Ulysses post-attention exchange layout), invariants of softmax attention,
``scipy.special.softmax`` and ``numpy.transpose`` as independent library routines.
"""
import ctypes
import json
import os
import subprocess
import tempfile

import numpy as np
import pytest
from scipy.special import softmax as scipy_softmax

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------------------- helpers
def scipy_attention(q, k, v, scale):
    """Independent brute force: scores with einsum, scipy's softmax, weighted sum."""
    s = np.einsum("bhid,bhjd->bhij", q, k) * scale
    p = scipy_softmax(s, axis=-1)
    return np.einsum("bhij,bhjd->bhid", p, v)


def rng_qkv(rng, B, H, S, D, spread=1.0):
    q = rng.standard_normal((B, H, S, D)) * spread
    k = rng.standard_normal((B, H, S, D)) * spread
    v = rng.standard_normal((B, H, S, D))
    return q, k, v


def attention_pins(attn):
    """Run the attention pins against ``attn(q, k, v, scale=None)``; raise AssertionError."""
    # 1. hand-derived closed forms (golden fixtures)
    doc = json.load(open(os.path.join(GOLDEN, "attention_closed_forms.json")))
    for case in doc["cases"]:
        q = np.array(case["q"], dtype=np.float64)[None, None]
        k = np.array(case["k"], dtype=np.float64)[None, None]
        v = np.array(case["v"], dtype=np.float64)[None, None]
        # The oracle takes one [B,H,S,D] shape for q, k and v.  Zero columns appended to q
        # and k leave every score unchanged, zero columns appended to v only add zero
        # output columns, and zero query rows appended after the real ones are sliced off.
        # (Cases that rely on the default scale already share one D.)
        nq, S, Dv = q.shape[2], k.shape[2], v.shape[3]
        Dm = max(k.shape[3], Dv)
        qq = np.zeros((1, 1, S, Dm)); qq[:, :, :nq, :q.shape[3]] = q
        kk = np.zeros((1, 1, S, Dm)); kk[..., :k.shape[3]] = k
        vv = np.zeros((1, 1, S, Dm)); vv[..., :Dv] = v
        assert case["scale"] is not None or (k.shape[3] == Dv and nq <= S)
        out = attn(qq, kk, vv, case["scale"])[:, :, :nq, :Dv]
        exp = np.array(case["expected"], dtype=np.float64)[None, None]
        np.testing.assert_allclose(out, exp, atol=doc["tolerance_abs"], rtol=0, err_msg=case["name"])

    rng = np.random.default_rng(7)
    # 2. brute force against scipy on tiny shapes (non-square D/S, several heads and batches)
    for (B, H, S, D) in [(1, 1, 1, 1), (2, 3, 5, 3), (1, 2, 16, 8), (2, 1, 9, 7), (1, 2, 13, 72)]:
        q, k, v = rng_qkv(rng, B, H, S, D, spread=1.5)
        np.testing.assert_allclose(attn(q, k, v, None), scipy_attention(q, k, v, 1.0 / np.sqrt(D)),
                                   atol=1e-12, rtol=1e-12)
    # 3. constant value rows give that constant, whatever the scores
    q, k, _ = rng_qkv(rng, 2, 2, 11, 4, spread=3.0)
    c = rng.standard_normal(4)
    v = np.broadcast_to(c, q.shape).copy()
    np.testing.assert_allclose(attn(q, k, v, None), v, atol=1e-12, rtol=0)
    # 4. Q = 0 gives the mean of V over keys
    q0 = np.zeros_like(q)
    v = rng.standard_normal(q.shape)
    np.testing.assert_allclose(attn(q0, k, v, None),
                               np.broadcast_to(v.mean(axis=2, keepdims=True), v.shape),
                               atol=1e-12, rtol=0)
    # 5. one key: the output is that key's value row
    q, k, v = rng_qkv(rng, 1, 3, 1, 6)
    np.testing.assert_allclose(attn(q, k, v, None), v, atol=1e-15, rtol=0)
    # 6. permuting keys and values together leaves the output unchanged
    q, k, v = rng_qkv(rng, 1, 2, 12, 5, spread=2.0)
    perm = rng.permutation(12)
    np.testing.assert_allclose(attn(q, k[:, :, perm], v[:, :, perm], None), attn(q, k, v, None),
                               atol=1e-12, rtol=0)
    # 7. V = identity (S == D): the output rows are the softmax rows, which sum to 1
    q, k, _ = rng_qkv(rng, 1, 1, 6, 6, spread=2.0)
    eye = np.eye(6)[None, None]
    o = attn(q, k, eye, None)
    np.testing.assert_allclose(o.sum(axis=-1), 1.0, atol=1e-13, rtol=0)
    assert (o > 0).all()
    np.testing.assert_allclose(o[0, 0], scipy_softmax(q[0, 0] @ k[0, 0].T / np.sqrt(6), axis=-1),
                               atol=1e-13, rtol=0)


def oracle_attn(q, k, v, scale):
    return oracle.attention(q, k, v, scale=scale)


# ----------------------------------------------------------------------------- attention
def test_attention_pins():
    attention_pins(oracle_attn)


def test_softmax_row_sums_to_one():
    rng = np.random.default_rng(1)
    q, k, _ = rng_qkv(rng, 2, 3, 37, 5, spread=4.0)
    for (b, h, i) in [(0, 0, 0), (1, 2, 36), (0, 1, 17)]:
        p = oracle.softmax_row(q, k, b, h, i)
        assert abs(p.sum() - 1.0) < 1e-12
        assert (p >= 0).all()
        np.testing.assert_allclose(p, scipy_softmax(q[b, h, i] @ k[b, h].T / np.sqrt(5)),
                                   atol=1e-14, rtol=0)


def test_rows_subset_matches_full():
    rng = np.random.default_rng(2)
    q, k, v = rng_qkv(rng, 2, 2, 40, 8)
    full = oracle.attention(q, k, v)
    rows = np.array([[[0, 5, 39], [3, 4, 38]], [[39, 0, 1], [7, 8, 9]]], dtype=np.int32)
    sub = oracle.attention(q, k, v, rows=rows)
    for b in range(2):
        for h in range(2):
            np.testing.assert_array_equal(sub[b, h], full[b, h, rows[b, h]])


def test_threads_do_not_change_result():
    rng = np.random.default_rng(3)
    q, k, v = rng_qkv(rng, 1, 4, 64, 16)
    a = oracle.attention(q, k, v, nthreads=1)
    b = oracle.attention(q, k, v, nthreads=4)
    np.testing.assert_array_equal(a, b)


def test_bf16_inputs_widen_exactly():
    import torch
    g = torch.Generator().manual_seed(0)
    q = torch.randn((1, 1, 8, 8), generator=g).to(torch.bfloat16)
    out = oracle.attention(q, q, q)
    ref = scipy_attention(*(q.double().numpy(),) * 3, 1 / np.sqrt(8))
    np.testing.assert_allclose(out, ref, atol=1e-12, rtol=1e-12)


def test_attention_rejects_bad_shapes():
    q = np.zeros((1, 1, 4, 2))
    with pytest.raises(ValueError):
        oracle.attention(q, np.zeros((1, 1, 5, 2)), q)
    with pytest.raises(ValueError):
        oracle.attention(q, q, q, rows=np.array([4], dtype=np.int32))


# ----------------------------------------------------------------------------- exchange
def test_a2a_golden():
    doc = json.load(open(os.path.join(GOLDEN, "a2a_permutation.json")))
    for c in doc["cases"]:
        B, H, S, D, P = c["B"], c["H"], c["S"], c["D"], c["P"]
        b, h, s, d = np.meshgrid(np.arange(B), np.arange(H), np.arange(S), np.arange(D), indexing="ij")
        src = eval(c["encoding"].split("=", 1)[1], {}, dict(b=b, h=h, s=s, d=d)).astype(np.int64)
        dest = oracle.a2a_post(src, P)
        np.testing.assert_array_equal(dest.reshape(-1), np.array(c["expected_flat"]), err_msg=c["name"])


@pytest.mark.parametrize("B,H,S,D,P", [(1, 4, 256, 64, 2), (2, 16, 64, 72, 4), (1, 8, 72, 8, 8), (2, 3, 6, 2, 3)])
def test_a2a_bijection_and_roundtrip(B, H, S, D, P):
    src = np.arange(B * H * S * D, dtype=np.int64).reshape(B, H, S, D)
    dest = oracle.a2a_post(src, P)
    assert dest.shape == (P, B, S // P, H, D)
    # every source element lands exactly once
    np.testing.assert_array_equal(np.sort(dest.reshape(-1)), np.arange(src.size))
    # and comes back through the inverse
    np.testing.assert_array_equal(oracle.a2a_pre(dest), src)
    # each slab r holds exactly the sequence shard [r*S/P, (r+1)*S/P) of every head
    ss = (dest // D) % S
    hh = (dest // (D * S)) % H
    for r in range(P):
        assert ss[r].min() == r * (S // P) and ss[r].max() == (r + 1) * (S // P) - 1
        np.testing.assert_array_equal(hh[r], np.broadcast_to(np.arange(H)[None, None, :, None], hh[r].shape))


def test_a2a_single_rank_is_transpose():
    rng = np.random.default_rng(4)
    src = rng.standard_normal((2, 3, 10, 4))
    dest = oracle.a2a_post(src, 1)
    np.testing.assert_array_equal(dest[0], np.transpose(src, (0, 2, 1, 3)))


def test_a2a_moves_bits_exactly():
    rng = np.random.default_rng(5)
    src = rng.integers(0, 2**16, size=(1, 4, 8, 8), dtype=np.uint16)
    dest = oracle.a2a_post(src, 2)
    assert dest.dtype == np.uint16
    np.testing.assert_array_equal(oracle.a2a_pre(dest), src)


def test_dest_slot_agrees_with_exchange():
    B, H, S, D, P = 2, 4, 24, 3, 4
    src = np.arange(B * H * S * D, dtype=np.int64).reshape(B, H, S, D)
    dest = oracle.a2a_post(src, P)
    flat = dest.reshape(P, -1)
    for (b, h, s) in [(0, 0, 0), (1, 3, 23), (0, 2, 5), (1, 1, 6), (1, 0, 17)]:
        r, off = oracle.dest_slot(B, H, S, D, P, b, h, s)
        np.testing.assert_array_equal(flat[r, off:off + D], src[b, h, s])


def test_a2a_rejects_indivisible():
    with pytest.raises(ValueError):
        oracle.a2a_post(np.zeros((1, 4, 10, 2)), 4)
    with pytest.raises(ValueError):
        oracle.a2a_post(np.zeros((1, 3, 8, 2)), 2)


# ----------------------------------------------------------------------------- mutants
MUTANTS = {
    # a dropped scale factor
    "no_scale": ("work[j] = dot * scale;", "work[j] = dot;"),
    # a wrong sign in the exponent
    "sign": ("work[j] = exp(work[j] - m);", "work[j] = exp(m - work[j]);"),
    # a transposed operand (k read as [D, S])
    "transpose_k": ("dot += q_row[d] * k[(size_t)j * D + d];", "dot += q_row[d] * k[(size_t)d * S + j];"),
    # a dropped normalisation
    "no_norm": ("out_row[d] = acc / l;", "out_row[d] = acc;"),
    # the row maximum not subtracted (overflows for large scores)
    "no_max": ("work[j] = exp(work[j] - m);", "work[j] = exp(work[j]);"),
    # an off-by-one key range
    "drop_last_key": ("for (int j = 0; j < S; ++j) acc += work[j] * v[(size_t)j * D + d];",
                      "for (int j = 0; j < S - 1; ++j) acc += work[j] * v[(size_t)j * D + d];"),
}


def _build_mutant(src_text, name, tmpdir):
    c_path = os.path.join(tmpdir, f"{name}.c")
    so_path = os.path.join(tmpdir, f"{name}.so")
    open(c_path, "w").write(src_text)
    subprocess.run(["gcc", "-O2", "-fPIC", "-shared", "-o", so_path, c_path, "-lm"], check=True)
    lib = ctypes.CDLL(so_path)
    dp = ctypes.POINTER(ctypes.c_double)
    lib.xs_oracle_attention.argtypes = [dp, dp, dp] + [ctypes.c_int] * 4 + [
        ctypes.c_double, ctypes.POINTER(ctypes.c_int32), ctypes.c_int, dp, ctypes.c_int]
    lib.xs_oracle_attention.restype = ctypes.c_int

    def attn(q, k, v, scale):
        q, k, v = (np.ascontiguousarray(x, dtype=np.float64) for x in (q, k, v))
        B, H, S, D = q.shape
        if scale is None:
            scale = 1.0 / np.sqrt(D)
        out = np.empty_like(q)
        p = lambda a: a.ctypes.data_as(dp)
        rc = lib.xs_oracle_attention(p(q), p(k), p(v), B, H, S, D, float(scale),
                                     ctypes.POINTER(ctypes.c_int32)(), S, p(out), 1)
        assert rc == 0
        return out
    return attn


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistakes_are_caught(name):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "xs_oracle.c")).read()
    old, new = MUTANTS[name]
    assert src.count(old) >= 1, f"mutation site for {name} not found"
    mutated = src.replace(old, new, 1)
    with tempfile.TemporaryDirectory() as tmp:
        attn = _build_mutant(mutated, name, tmp)
        with pytest.raises(AssertionError):
            with np.errstate(all="ignore"):
                attention_pins(attn)
