"""CPU oracle for fused attention + Ulysses post-attention All-to-All.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may import this package.  The product (``ulysses_attention_output_b200``)
never imports it and shares no code with it.

The arithmetic lives in ``xs_oracle.c`` (plain C, fp64, naive loops, OpenMP over independent
query rows).  This module compiles it with gcc on first use if the shared object is missing
or older than the source, and marshals numpy arrays in and out.

What each function follows (page: "X-Stage: An Overlooked Pipeline Stage for
Communication-Computation Overlap in DiT Inference"; abstract, and the explainer's
"Technisches Resuemee" -> "Zentrale Beitraege" -> "FlashAttention-A2A (Piggybacking)"):

* :func:`attention`   -- non-causal softmax(Q K^T * scale) V, the definition written out.
* :func:`a2a_post`    -- the post-attention All-to-All into sequence shards
                         ``dest[r][b, s_local, h, d]`` (layout reading: see ``xs_oracle.c``).
* :func:`a2a_pre`     -- its inverse (sequence shards -> head-major).
* :func:`dest_slot`   -- where one output row lands.
* :func:`softmax_row` -- the normalised probabilities of one query row.

Partial attention and its merge follow the page "Move the Query, Not the Cache:
Characterizing Cross-Instance Latent Attention Redistribution Across GPU Fabrics" (explainer
"Technisches Resuemee: Den Query bewegen, nicht den Cache" -> "Methodik" -> "Primitiv-Vergleich",
the Route primitive, and "Korrektheitsverifizierung"):

* :func:`attention_partial` -- attention of the query rows over one key/value shard, with the
  row's log-sum-exp ``lse = log sum_j exp(s_j)``.
* :func:`lse_merge`         -- the online-softmax merge of partial results of disjoint shards.

All are pinned by ``tests/test_oracle_pins.py`` against closed forms, invariants, hand-made
fixtures under ``tests/golden/`` and an independent numpy brute force.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "xs_oracle.c")
_LIB = os.path.join(_HERE, "_xs_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ``xs_oracle.c`` into ``_xs_oracle.so`` (gcc, -O2, OpenMP, strict IEEE)."""
    stale = (not os.path.exists(_LIB)) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = _LIB + f".tmp{os.getpid()}"
        # -O2 without -ffast-math: the summation order stays the one written in the source.
        cmd = ["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-fno-fast-math",
               "-ffp-contract=off", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            dp = ctypes.POINTER(ctypes.c_double)
            ip = ctypes.POINTER(ctypes.c_int32)
            vp = ctypes.c_void_p
            c_int = ctypes.c_int
            lib.xs_oracle_attention.argtypes = [dp, dp, dp, c_int, c_int, c_int, c_int,
                                                ctypes.c_double, ip, c_int, dp, c_int]
            lib.xs_oracle_attention.restype = c_int
            lib.xs_oracle_softmax_row.argtypes = [dp, dp, c_int, c_int, c_int, c_int,
                                                  ctypes.c_double, c_int, c_int, c_int, dp]
            lib.xs_oracle_softmax_row.restype = c_int
            for name in ("xs_oracle_a2a_post", "xs_oracle_a2a_pre"):
                fn = getattr(lib, name)
                fn.argtypes = [vp, vp, c_int, c_int, c_int, c_int, c_int, c_int]
                fn.restype = c_int
            lib.xs_oracle_dest_slot.argtypes = [c_int] * 8 + [ctypes.POINTER(c_int),
                                                             ctypes.POINTER(ctypes.c_longlong)]
            lib.xs_oracle_dest_slot.restype = c_int
            lib.xs_oracle_max_threads.restype = c_int
            lib.xs_oracle_attention_partial.argtypes = [dp, dp, dp, c_int, c_int, c_int, c_int, c_int,
                                                        ctypes.c_double, ip, c_int, dp, dp, c_int]
            lib.xs_oracle_attention_partial.restype = c_int
            lib.xs_oracle_lse_merge.argtypes = [dp, dp, c_int, ctypes.c_longlong, c_int, dp, dp]
            lib.xs_oracle_lse_merge.restype = c_int
            _lib = lib
    return _lib


def _f64(x) -> np.ndarray:
    """numpy fp64 contiguous copy of an array-like (torch tensors go through .float64)."""
    if hasattr(x, "detach"):  # torch tensor: widen exactly (bf16/fp32 -> fp64 is exact)
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _dp(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def max_threads() -> int:
    """Threads the oracle's OpenMP loop uses by default on this host."""
    return int(_load().xs_oracle_max_threads())


def attention(q, k, v, scale: float | None = None, rows=None, nthreads: int = 0) -> np.ndarray:
    """fp64 attention output.

    q, k, v: [B, H, S, D].  ``scale`` defaults to 1/sqrt(D) with the true (unpadded) D.
    ``rows``: None for every row, else an int array [B, H, n] (or [n], shared by all heads)
    of query rows.  Returns [B, H, S or n, D] float64.
    """
    lib = _load()
    q, k, v = _f64(q), _f64(k), _f64(v)
    if q.ndim != 4 or k.shape != q.shape or v.shape != q.shape:
        raise ValueError(f"q, k, v must share one [B,H,S,D] shape, got {q.shape} {k.shape} {v.shape}")
    B, H, S, D = q.shape
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    if rows is None:
        n = S
        rows_arr = None
        rows_ptr = ctypes.POINTER(ctypes.c_int32)()
    else:
        rows_arr = np.asarray(rows, dtype=np.int32)
        if rows_arr.ndim == 1:
            rows_arr = np.broadcast_to(rows_arr, (B, H, rows_arr.shape[0]))
        rows_arr = np.ascontiguousarray(rows_arr.reshape(B, H, -1), dtype=np.int32)
        n = rows_arr.shape[2]
        rows_ptr = rows_arr.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
    out = np.empty((B, H, n, D), dtype=np.float64)
    rc = lib.xs_oracle_attention(_dp(q), _dp(k), _dp(v), B, H, S, D, float(scale), rows_ptr, n,
                                 _dp(out), int(nthreads))
    if rc != 0:
        raise ValueError(f"xs_oracle_attention rejected its arguments (rc={rc})")
    return out


def softmax_row(q, k, b: int, h: int, i: int, scale: float | None = None) -> np.ndarray:
    """Normalised softmax probabilities p_j / l of query row i of head (b, h): [S] float64."""
    lib = _load()
    q, k = _f64(q), _f64(k)
    B, H, S, D = q.shape
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    probs = np.empty(S, dtype=np.float64)
    rc = lib.xs_oracle_softmax_row(_dp(q), _dp(k), B, H, S, D, float(scale), b, h, i, _dp(probs))
    if rc != 0:
        raise ValueError("xs_oracle_softmax_row rejected its arguments")
    return probs


def a2a_post(src: np.ndarray, P: int) -> np.ndarray:
    """Post-attention All-to-All of a head-major [B,H,S,D] array into [P, B, S/P, H, D].

    Any fixed-size dtype is moved bit for bit (the oracle copies raw elements).
    """
    lib = _load()
    src = np.ascontiguousarray(src)
    B, H, S, D = src.shape
    if S % P or H % P:
        raise ValueError("Ulysses exchange needs S % P == 0 and H % P == 0")
    dest = np.empty((P, B, S // P, H, D), dtype=src.dtype)
    rc = lib.xs_oracle_a2a_post(src.ctypes.data, dest.ctypes.data, B, H, S, D, P, src.itemsize)
    if rc != 0:
        raise ValueError("xs_oracle_a2a_post rejected its arguments")
    return dest


def a2a_pre(slabs: np.ndarray) -> np.ndarray:
    """Inverse exchange: [P, B, S/P, H, D] sequence shards back to head-major [B, H, S, D]."""
    lib = _load()
    slabs = np.ascontiguousarray(slabs)
    P, B, Sl, H, D = slabs.shape
    S = Sl * P
    out = np.empty((B, H, S, D), dtype=slabs.dtype)
    rc = lib.xs_oracle_a2a_pre(slabs.ctypes.data, out.ctypes.data, B, H, S, D, P, slabs.itemsize)
    if rc != 0:
        raise ValueError("xs_oracle_a2a_pre rejected its arguments")
    return out


def dest_slot(B: int, H: int, S: int, D: int, P: int, b: int, h: int, s: int) -> tuple[int, int]:
    """(rank, element offset inside slab ``rank``) of output row (b, h, s)."""
    lib = _load()
    r = ctypes.c_int()
    off = ctypes.c_longlong()
    rc = lib.xs_oracle_dest_slot(B, H, S, D, P, b, h, s, ctypes.byref(r), ctypes.byref(off))
    if rc != 0:
        raise ValueError("xs_oracle_dest_slot rejected its arguments")
    return int(r.value), int(off.value)


def _rows_arg(rows, B: int, H: int):
    rows_arr = np.asarray(rows, dtype=np.int32)
    if rows_arr.ndim == 1:
        rows_arr = np.broadcast_to(rows_arr, (B, H, rows_arr.shape[0]))
    rows_arr = np.ascontiguousarray(rows_arr.reshape(B, H, -1), dtype=np.int32)
    return rows_arr, rows_arr.shape[2], rows_arr.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))


def attention_partial(q, k, v, scale: float | None = None, rows=None, nthreads: int = 0):
    """fp64 partial attention of q [B,H,Sq,D] over one key/value shard k, v [B,H,Skv,D].

    Returns ``(out [B,H,n,D], lse [B,H,n])`` with n = Sq or len(rows); lse is the natural-log
    log-sum-exp of the scaled scores.  Skv may be 0 (then out = 0 and lse = -inf).
    ``scale`` defaults to 1/sqrt(D).
    """
    lib = _load()
    q, k, v = _f64(q), _f64(k), _f64(v)
    if q.ndim != 4 or k.ndim != 4 or v.shape != k.shape or k.shape[:2] != q.shape[:2] \
            or k.shape[3] != q.shape[3]:
        raise ValueError(f"need q [B,H,Sq,D] and k, v [B,H,Skv,D]; got {q.shape} {k.shape} {v.shape}")
    B, H, Sq, D = q.shape
    Skv = k.shape[2]
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    if rows is None:
        n, rows_arr, rows_ptr = Sq, None, ctypes.POINTER(ctypes.c_int32)()
    else:
        rows_arr, n, rows_ptr = _rows_arg(rows, B, H)
    out = np.empty((B, H, n, D), dtype=np.float64)
    lse = np.empty((B, H, n), dtype=np.float64)
    kk = k if Skv > 0 else np.zeros(1)
    vv = v if Skv > 0 else np.zeros(1)
    rc = lib.xs_oracle_attention_partial(_dp(q), _dp(kk), _dp(vv), B, H, Sq, Skv, D, float(scale),
                                         rows_ptr, n, _dp(out), _dp(lse), int(nthreads))
    if rc != 0:
        raise ValueError(f"xs_oracle_attention_partial rejected its arguments (rc={rc})")
    return out, lse


def lse_merge(o_parts, lse_parts):
    """fp64 online-softmax merge of n partial results.

    o_parts: [n, ..., D]; lse_parts: [n, ...] (same leading shape; -inf marks an empty part).
    Returns ``(out [..., D], lse [...])``.
    """
    lib = _load()
    o = _f64(o_parts)
    lse = _f64(lse_parts)
    if o.ndim < 2 or lse.shape != o.shape[:-1]:
        raise ValueError(f"need o_parts [n, ..., D] and lse_parts [n, ...]; got {o.shape} {lse.shape}")
    n, D = o.shape[0], o.shape[-1]
    lead = o.shape[1:-1]
    R = int(np.prod(lead)) if lead else 1
    out = np.empty(lead + (D,), dtype=np.float64)
    lse_out = np.empty(lead, dtype=np.float64)
    rc = lib.xs_oracle_lse_merge(_dp(o), _dp(lse), n, R, D, _dp(out), _dp(lse_out))
    if rc != 0:
        raise ValueError("xs_oracle_lse_merge rejected its arguments")
    return out, lse_out
