"""The C-ABI library on the host (CPU only): it builds, loads, exports every symbol that
``include/xs.h`` declares, and rejects bad arguments with the documented codes before any
CUDA call.  No kernel is launched here.
"""
import ctypes
import os
import re

import pytest

import ulysses_attention_output_b200 as xs
from ulysses_attention_output_b200 import build as xs_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    xs_build.build()
    return xs.load()


def declared_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"XS_API\s+[\w\s\*]+?\b(xs_\w+)\s*\(", text)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert {"xs_attn_a2a_fused", "xs_attn", "xs_a2a_relayout", "xs_burst_probe"} <= set(names)
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/ but not exported by libxs.so"


def test_version_and_strings(lib):
    assert xs.version() == 100
    for code, name in [(0, b"XS_OK"), (1, b"XS_ERR_INVALID_ARG"), (2, b"XS_ERR_UNSUPPORTED"),
                       (3, b"XS_ERR_CUDA"), (4, b"XS_ERR_TIMEOUT")]:
        assert lib.xs_get_error_string(code) == name


FAKE = 0x7f0000000000  # never dereferenced: every call below fails validation first
MB = 1 << 20


def fused(lib, q, k, v, dests, shape, scale=0.0):
    arr = (ctypes.c_void_p * max(1, len(dests)))(*dests) if dests is not None else None
    return lib.xs_attn_a2a_fused(q, k, v, arr, xs.Shape(*shape), scale, None, None)


@pytest.mark.parametrize("shape,code", [
    ((1, 4, 256, 100, 2), xs.XS_ERR_UNSUPPORTED),   # D not a multiple of 8
    ((1, 4, 256, 136, 2), xs.XS_ERR_UNSUPPORTED),   # D > 128
    ((1, 3, 256, 64, 2), xs.XS_ERR_UNSUPPORTED),    # H % P != 0
    ((1, 4, 255, 64, 2), xs.XS_ERR_UNSUPPORTED),    # S % P != 0
    ((1, 32, 256, 64, 32), xs.XS_ERR_UNSUPPORTED),  # P > 16
    ((0, 4, 256, 64, 2), xs.XS_ERR_INVALID_ARG),    # empty batch
    ((1, 4, 256, 64, 0), xs.XS_ERR_INVALID_ARG),    # no ranks
])
def test_fused_rejects_shapes(lib, shape, code):
    dests = [FAKE + 100 * MB * (r + 1) for r in range(max(shape[4], 1))]
    assert fused(lib, FAKE, FAKE + 30 * MB, FAKE + 60 * MB, dests, shape) == code


def test_fused_rejects_pointers(lib):
    shape = (1, 4, 256, 64, 2)
    good = [FAKE + 100 * MB, FAKE + 200 * MB]
    assert fused(lib, 0, FAKE + 30 * MB, FAKE + 60 * MB, good, shape) == xs.XS_ERR_INVALID_ARG
    assert fused(lib, FAKE + 8, FAKE + 30 * MB, FAKE + 60 * MB, good, shape) == xs.XS_ERR_INVALID_ARG
    assert fused(lib, FAKE, FAKE + 30 * MB, FAKE + 60 * MB, None, shape) == xs.XS_ERR_INVALID_ARG
    assert fused(lib, FAKE, FAKE + 30 * MB, FAKE + 60 * MB, [good[0], 0], shape) == xs.XS_ERR_INVALID_ARG
    # overlapping slabs, slab overlapping an input
    assert fused(lib, FAKE, FAKE + 30 * MB, FAKE + 60 * MB, [good[0], good[0] + 1024], shape) == xs.XS_ERR_INVALID_ARG
    assert fused(lib, FAKE, FAKE + 30 * MB, FAKE + 60 * MB, [good[0], FAKE + 1024], shape) == xs.XS_ERR_INVALID_ARG
    detail = lib.xs_last_error_detail().decode()
    assert "overlaps" in detail


def test_flags_and_wait_reject(lib):
    shape = xs.Shape(1, 4, 256, 64, 2)
    q, k, v = FAKE, FAKE + 30 * MB, FAKE + 60 * MB
    dest = (ctypes.c_void_p * 2)(FAKE + 100 * MB, FAKE + 200 * MB)

    def call(flags, sh=shape, ht=4, off=0):
        arr = (ctypes.c_void_p * 2)(*flags) if flags is not None else None
        return lib.xs_attn_a2a_fused_flags(q, k, v, dest, arr, sh, ht, off, 0.0, None, None)

    assert call(None) == xs.XS_ERR_INVALID_ARG                                        # no array
    assert call([FAKE + 300 * MB, 0]) == xs.XS_ERR_INVALID_ARG                        # null counter
    assert call([FAKE + 300 * MB, FAKE + 300 * MB + 2]) == xs.XS_ERR_INVALID_ARG      # misaligned
    assert call([FAKE + 300 * MB, FAKE + 300 * MB]) == xs.XS_ERR_INVALID_ARG          # same counter
    assert call([FAKE + 300 * MB, FAKE + 100 * MB + 64]) == xs.XS_ERR_INVALID_ARG     # inside a slab
    assert "inside dest" in lib.xs_last_error_detail().decode()
    assert call([FAKE + 300 * MB, FAKE + 64]) == xs.XS_ERR_INVALID_ARG                # inside q
    assert call([FAKE + 300 * MB, FAKE + 301 * MB], off=2) == xs.XS_ERR_INVALID_ARG   # heads past the layer
    assert call([FAKE + 300 * MB, FAKE + 301 * MB], sh=xs.Shape(1, 4, 256, 60, 2)) == xs.XS_ERR_UNSUPPORTED
    st = FAKE + 400 * MB
    assert lib.xs_slab_wait(0, 1, 10 ** 6, None, st) == xs.XS_ERR_INVALID_ARG
    assert lib.xs_slab_wait(FAKE + 2, 1, 10 ** 6, None, st) == xs.XS_ERR_INVALID_ARG
    assert lib.xs_slab_wait(FAKE, 1, 10 ** 6, None, 0) == xs.XS_ERR_INVALID_ARG
    assert lib.xs_slab_wait(FAKE, 1, 10, None, st) == xs.XS_ERR_INVALID_ARG


def test_attn_and_relayout_reject(lib):
    sh = xs.Shape(1, 4, 256, 64, 2)
    assert lib.xs_attn(FAKE, FAKE + MB, FAKE + 2 * MB, 0, sh, 0.0, None, None) == xs.XS_ERR_INVALID_ARG
    assert lib.xs_attn(FAKE, FAKE + MB, FAKE + 2 * MB, FAKE, sh, 0.0, None, None) == xs.XS_ERR_INVALID_ARG
    arr = (ctypes.c_void_p * 2)(FAKE + 100 * MB, FAKE + 200 * MB)
    assert lib.xs_a2a_relayout(0, arr, sh, None) == xs.XS_ERR_INVALID_ARG
    assert lib.xs_a2a_relayout(FAKE, arr, xs.Shape(1, 4, 256, 60, 2), None) == xs.XS_ERR_UNSUPPORTED
    assert lib.xs_a2a_relayout(FAKE, arr, xs.Shape(1, 4, 250, 64, 4), None) == xs.XS_ERR_UNSUPPORTED  # S % P


def test_probe_and_selftest_reject(lib):
    cfg = xs.BurstCfg(4096, 4, 0, 8, 256)
    assert lib.xs_burst_probe(0, 1 << 20, cfg, FAKE, None) == xs.XS_ERR_INVALID_ARG
    assert lib.xs_burst_probe(FAKE, 1 << 20, xs.BurstCfg(4100, 4, 0, 8, 256), FAKE + 8 * MB, None) == xs.XS_ERR_INVALID_ARG
    assert lib.xs_burst_probe(FAKE, 1024, cfg, FAKE + 8 * MB, None) == xs.XS_ERR_INVALID_ARG
    assert lib.xs_burst_probe(FAKE, 1 << 20, xs.BurstCfg(4096, 4, 0, 8, 100), FAKE + 8 * MB, None) == xs.XS_ERR_INVALID_ARG
    assert lib.xs_selftest_bounded_wait(0, 10 ** 6, None) == xs.XS_ERR_INVALID_ARG
    assert lib.xs_selftest_bounded_wait(FAKE, 10, None) == xs.XS_ERR_INVALID_ARG
    sh = xs.Shape(1, 2, 256, 64, 1)
    q, k, v, out = FAKE, FAKE + MB, FAKE + 2 * MB, FAKE + 3 * MB
    # every bad argument is refused on the host, before anything is enqueued
    assert lib.xs_selftest_attn_abort(q, k, v, out, sh, 0, 10 ** 6, None, 0) == xs.XS_ERR_INVALID_ARG
    assert lib.xs_selftest_attn_abort(q, k, v, out, sh, -1, 10 ** 6, None, FAKE + 4 * MB) == xs.XS_ERR_INVALID_ARG
    assert lib.xs_selftest_attn_abort(q, k, v, out, sh, 0, 10, None, FAKE + 4 * MB) == xs.XS_ERR_INVALID_ARG
    assert lib.xs_selftest_attn_abort(q, k, v, q, sh, 0, 10 ** 6, None, FAKE + 4 * MB) == xs.XS_ERR_INVALID_ARG
    assert lib.xs_selftest_attn_abort(q, k, v, out, xs.Shape(1, 2, 256, 60, 1), 0, 10 ** 6, None,
                                      FAKE + 4 * MB) == xs.XS_ERR_UNSUPPORTED


def test_binding_has_no_fallback(monkeypatch, tmp_path):
    """With the library missing, the binding raises instead of computing anything else."""
    monkeypatch.setattr(xs, "_lib", None)
    monkeypatch.setenv("XS_LIBRARY", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="missing"):
        xs.load()
    monkeypatch.setattr(xs, "_lib", None)


def test_product_never_imports_oracle():
    pkg = os.path.join(ROOT, "ulysses_attention_output_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, fn)).read()
                assert "import oracle" not in text and "from oracle" not in text, fn
                assert "xs_oracle" not in text, fn


def test_partial_and_merge_reject(lib):
    sh = xs.Shape(1, 4, 256, 64, 1)
    q, k, v, o, l = FAKE, FAKE + MB, FAKE + 2 * MB, FAKE + 8 * MB, FAKE + 16 * MB
    P = lib.xs_attn_partial
    assert P(q, k, v, o, l, xs.Shape(1, 4, 256, 64, 2), 128, 0.0, None, None) == xs.XS_ERR_INVALID_ARG  # P != 1
    assert P(q, k, v, o, l, sh, -1, 0.0, None, None) == xs.XS_ERR_INVALID_ARG            # negative s_kv
    assert P(q, k, v, o, l, xs.Shape(1, 4, 256, 136, 1), 128, 0.0, None, None) == xs.XS_ERR_UNSUPPORTED
    assert P(q, 0, v, o, l, sh, 128, 0.0, None, None) == xs.XS_ERR_INVALID_ARG            # k missing
    assert P(q, k, v, o + 4, l, sh, 128, 0.0, None, None) == xs.XS_ERR_INVALID_ARG        # o misaligned
    assert P(q, k, v, o, o + 1024, sh, 128, 0.0, None, None) == xs.XS_ERR_INVALID_ARG     # lse inside o
    assert P(q, k, v, q + 1024, l, sh, 128, 0.0, None, None) == xs.XS_ERR_INVALID_ARG     # o overlaps q
    M = lib.xs_lse_merge
    op = (ctypes.c_void_p * 2)(FAKE, FAKE + 4 * MB)
    lp = (ctypes.c_void_p * 2)(FAKE + 8 * MB, FAKE + 9 * MB)
    out = FAKE + 16 * MB
    assert M(op, lp, 0, out, None, 1024, 128, None) == xs.XS_ERR_UNSUPPORTED              # no parts
    assert M(op, lp, 17, out, None, 1024, 128, None) == xs.XS_ERR_UNSUPPORTED             # too many
    assert M(op, lp, 2, out, None, 1024, 100, None) == xs.XS_ERR_UNSUPPORTED              # D % 8
    assert M(op, lp, 2, out, None, 0, 128, None) == xs.XS_ERR_INVALID_ARG                 # no rows
    assert M(op, lp, 2, FAKE + 1024, None, 1024, 128, None) == xs.XS_ERR_INVALID_ARG      # out inside part 0
    bad = (ctypes.c_void_p * 2)(FAKE + 4, FAKE + 4 * MB)
    assert M(bad, lp, 2, out, None, 1024, 128, None) == xs.XS_ERR_INVALID_ARG             # misaligned part


def test_ipc_calls_reject_null_arguments(lib):
    buf = ctypes.create_string_buffer(xs.IPC_HANDLE_BYTES)
    off = ctypes.c_longlong(0)
    base = ctypes.c_void_p(0)
    assert lib.xs_ipc_export(None, buf, ctypes.byref(off)) == xs.XS_ERR_INVALID_ARG
    assert lib.xs_ipc_export(FAKE, None, ctypes.byref(off)) == xs.XS_ERR_INVALID_ARG
    assert lib.xs_ipc_export(FAKE, buf, None) == xs.XS_ERR_INVALID_ARG
    assert lib.xs_ipc_open(None, ctypes.byref(base)) == xs.XS_ERR_INVALID_ARG
    assert lib.xs_ipc_open(buf, None) == xs.XS_ERR_INVALID_ARG
    assert lib.xs_ipc_close(None) == xs.XS_ERR_INVALID_ARG
    assert "non-null" in lib.xs_last_error_detail().decode()


def test_ipc_binding_checks_its_arguments():
    import torch
    with pytest.raises(ValueError):
        xs.ipc_export(torch.zeros(4))              # host tensor
    with pytest.raises(ValueError):
        xs.ipc_open(b"\0" * (xs.IPC_HANDLE_BYTES - 1))
    ptr_text = open(os.path.join(ROOT, "include", "xs.h")).read()
    assert re.search(r"#define XS_IPC_HANDLE_BYTES (\d+)", ptr_text).group(1) == str(xs.IPC_HANDLE_BYTES)
