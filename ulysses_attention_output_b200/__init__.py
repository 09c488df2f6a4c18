"""Python binding of libxs.so: fused DiT attention + Ulysses post-attention All-to-All (B200).

Argument marshalling only.  Every step of the computation runs in the CUDA kernels of
``libxs.so`` (declared in ``include/xs.h``); PyTorch only supplies device memory and streams.
There is no fallback: if the library is missing or a call fails, these functions raise.

Calls (same names as the C ABI, without the ``xs_`` prefix):

* :func:`attn_a2a_fused` -- attention fused with the post-attention exchange into P slabs.
* :func:`attn`           -- attention with a head-major output.
* :func:`a2a_relayout`   -- the exchange as a separate pass (serial baseline).
* :func:`attn_a2a_fused_rank` -- the fused call of one Ulysses rank (its heads, all slabs).
* :func:`attn_a2a_fused_spans` -- the fused call, also recording each tile's store-issue span.
* :func:`attn_a2a_fused_flags` -- the fused call, also publishing per-slab arrival counters.
* :func:`slab_wait`      -- bounded wait of a consumer until a slab's counter reaches a target.
* :func:`a2a_pre`        -- the pre-attention exchange (sequence shards -> head-major).
* :func:`attn_partial`   -- partial attention over one key/value shard, fp32 output + lse.
* :func:`lse_merge`      -- online-softmax merge of partial results (the Route primitive).
* :func:`burst_probe`    -- Burst-Gap store microbenchmark.
* :func:`burst_probe_static` -- the same, with no device allocation (fixed library scratch).
* :func:`selftest_bounded_wait` -- exercises the bounded on-device wait.
* :func:`selftest_attn_abort` -- makes the attention kernel's own waits run out (abort path).
"""
from __future__ import annotations

import ctypes
import os
import threading

__all__ = [
    "XsError", "XS_OK", "XS_ERR_INVALID_ARG", "XS_ERR_UNSUPPORTED", "XS_ERR_CUDA", "XS_ERR_TIMEOUT",
    "library_path", "load", "version", "attn_a2a_fused", "attn", "a2a_relayout", "burst_probe",
    "attn_a2a_fused_rank", "a2a_pre", "attn_partial", "lse_merge", "attn_a2a_fused_spans",
    "burst_probe_static", "selftest_bounded_wait", "selftest_attn_abort", "alloc_dest",
    "attn_a2a_fused_flags", "slab_wait", "HostPipeline", "attention_flops",
    "ipc_export", "ipc_open", "ipc_close", "IPC_HANDLE_BYTES",
]

XS_OK, XS_ERR_INVALID_ARG, XS_ERR_UNSUPPORTED, XS_ERR_CUDA, XS_ERR_TIMEOUT = 0, 1, 2, 3, 4
XS_MAX_RANKS = 16
IPC_HANDLE_BYTES = 64  # XS_IPC_HANDLE_BYTES

_HERE = os.path.dirname(os.path.abspath(__file__))
_lock = threading.Lock()
_lib = None


class XsError(RuntimeError):
    """A libxs call returned a non-zero status."""

    def __init__(self, status: int, detail: str):
        super().__init__(f"{_STATUS_NAMES.get(status, status)}: {detail}")
        self.status = status


_STATUS_NAMES = {0: "XS_OK", 1: "XS_ERR_INVALID_ARG", 2: "XS_ERR_UNSUPPORTED", 3: "XS_ERR_CUDA",
                 4: "XS_ERR_TIMEOUT"}


class Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("S", ctypes.c_int), ("D", ctypes.c_int),
                ("P", ctypes.c_int)]


class BurstCfg(ctypes.Structure):
    _fields_ = [("burst_bytes", ctypes.c_longlong), ("producers", ctypes.c_int),
                ("gap_cycles", ctypes.c_longlong), ("n_bursts", ctypes.c_int),
                ("threads_per_producer", ctypes.c_int)]


def library_path() -> str:
    return os.environ.get("XS_LIBRARY", os.path.join(_HERE, "libxs.so"))


def load():
    """Load libxs.so (once).  Raises if it has not been built: there is no other path."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        path = library_path()
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: build it with "
                               "`python -m ulysses_attention_output_b200.build`")
        lib = ctypes.CDLL(path)
        vp, c_int, c_float = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
        vpp = ctypes.POINTER(ctypes.c_void_p)
        ip = ctypes.c_void_p  # device int*
        lib.xs_attn_a2a_fused.argtypes = [vp, vp, vp, vpp, Shape, c_float, vp, ip]
        lib.xs_attn.argtypes = [vp, vp, vp, vp, Shape, c_float, vp, ip]
        lib.xs_attn_a2a_fused_rank.argtypes = [vp, vp, vp, vpp, Shape, c_int, c_int, c_float, vp, ip]
        lib.xs_a2a_pre.argtypes = [vpp, vp, Shape, c_int, c_int, vp]
        lib.xs_a2a_relayout.argtypes = [vp, vpp, Shape, vp]
        lib.xs_burst_probe.argtypes = [vp, ctypes.c_longlong, BurstCfg, vp, vp]
        lib.xs_burst_probe_static.argtypes = [BurstCfg, vp, vp]
        lib.xs_selftest_bounded_wait.argtypes = [ip, ctypes.c_longlong, vp]
        lib.xs_selftest_attn_abort.argtypes = [vp, vp, vp, vp, Shape, c_int, ctypes.c_longlong, vp, ip]
        lib.xs_attn_a2a_fused_flags.argtypes = [vp, vp, vp, vpp, vpp, Shape, c_int, c_int, c_float, vp, ip]
        lib.xs_slab_wait.argtypes = [vp, ctypes.c_uint, ctypes.c_longlong, vp, ip]
        lib.xs_attn_partial.argtypes = [vp, vp, vp, vp, vp, Shape, c_int, c_float, vp, ip]
        lib.xs_attn_a2a_fused_spans.argtypes = [vp, vp, vp, vpp, Shape, c_float, vp, ctypes.c_longlong, vp, ip]
        lib.xs_lse_merge.argtypes = [vpp, vpp, c_int, vp, vp, ctypes.c_longlong, c_int, vp]
        lib.xs_ipc_export.argtypes = [vp, ctypes.c_char_p, ctypes.POINTER(ctypes.c_longlong)]
        lib.xs_ipc_open.argtypes = [ctypes.c_char_p, ctypes.POINTER(ctypes.c_void_p)]
        lib.xs_ipc_close.argtypes = [vp]
        for fn in (lib.xs_attn_a2a_fused, lib.xs_attn, lib.xs_a2a_relayout, lib.xs_burst_probe,
                   lib.xs_burst_probe_static, lib.xs_selftest_bounded_wait, lib.xs_selftest_attn_abort,
                   lib.xs_attn_a2a_fused_flags, lib.xs_slab_wait,
                   lib.xs_attn_a2a_fused_rank, lib.xs_a2a_pre, lib.xs_attn_partial, lib.xs_lse_merge,
                   lib.xs_attn_a2a_fused_spans):
            fn.restype = c_int
        lib.xs_get_error_string.argtypes = [c_int]
        lib.xs_get_error_string.restype = ctypes.c_char_p
        lib.xs_last_error_detail.restype = ctypes.c_char_p
        lib.xs_version.restype = c_int
        _lib = lib
        return lib


def version() -> int:
    return int(load().xs_version())


def _check(rc: int):
    if rc != XS_OK:
        detail = load().xs_last_error_detail().decode(errors="replace")
        raise XsError(rc, detail)


# ------------------------------------------------------------------ marshalling helpers
def _stream_handle(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream or None
    if isinstance(stream, int):
        return stream or None
    return stream.cuda_stream or None


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _bf16_cuda(name: str, t, shape=None):
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype not in (torch.bfloat16, torch.int16, torch.uint16):
        raise TypeError(f"{name} must hold 16-bit words (bf16), got {t.dtype}")
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA tensor")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def _shape_of(q, P: int) -> Shape:
    if q.dim() != 4:
        raise ValueError("q must be [B, H, S, D]")
    B, H, S, D = (int(x) for x in q.shape)
    return Shape(B, H, S, D, int(P))


def _dest_array(dest, shp: Shape):
    if len(dest) != shp.P:
        raise ValueError(f"need {shp.P} destination slabs, got {len(dest)}")
    for r, d in enumerate(dest):
        _bf16_cuda(f"dest[{r}]", d, (shp.B, shp.S // max(shp.P, 1), shp.H, shp.D))
    arr = (ctypes.c_void_p * shp.P)(*[d.data_ptr() for d in dest])
    return arr


def attention_flops(B: int, H: int, S: int, D: int) -> int:
    """Algorithmic FLOPs of one attention pass, 4*B*H*S^2*D (two S x S x D contractions)."""
    return 4 * B * H * S * S * D


# ------------------------------------------------------------------ calls
def attn_a2a_fused(q, k, v, dest, scale: float | None = None, stream=None, status=None):
    """Attention + post-attention All-to-All: fills ``dest[r]`` ([B, S/P, H, D]) for r < P."""
    P = len(dest)
    shp = _shape_of(q, P)
    for n, t in (("q", q), ("k", k), ("v", v)):
        _bf16_cuda(n, t, tuple(q.shape))
    arr = _dest_array(dest, shp)
    _check(load().xs_attn_a2a_fused(q.data_ptr(), k.data_ptr(), v.data_ptr(), arr, shp,
                                    float(scale or 0.0), _stream_handle(stream), _ptr(status)))


def attn_a2a_fused_spans(q, k, v, dest, spans=None, scale: float | None = None, stream=None, status=None):
    """``attn_a2a_fused`` that also records, for every work item (256 query rows), tile and
    storing warp, the SM clock before its first store, the SM clock after its last store
    was issued, and the global timer (ns): returns ``spans`` int64 [n_items, 2, 4, 3]."""
    import torch
    P = len(dest)
    shp = _shape_of(q, P)
    for n, t in (("q", q), ("k", k), ("v", v)):
        _bf16_cuda(n, t, tuple(q.shape))
    arr = _dest_array(dest, shp)
    n_items = shp.B * shp.H * ((shp.S + 255) // 256)
    if spans is None:
        spans = torch.zeros((n_items, 2, 4, 3), dtype=torch.int64, device=q.device)
    if spans.dtype != torch.int64 or not spans.is_cuda or not spans.is_contiguous():
        raise ValueError("spans must be a contiguous int64 CUDA tensor")
    _check(load().xs_attn_a2a_fused_spans(q.data_ptr(), k.data_ptr(), v.data_ptr(), arr, shp,
                                          float(scale or 0.0), spans.data_ptr(), spans.numel(),
                                          _stream_handle(stream), _ptr(status)))
    return spans


def attn_a2a_fused_rank(q, k, v, dest, heads_total: int, head_offset: int, scale: float | None = None,
                        stream=None, status=None):
    """One Ulysses rank's fused call: its heads ``q, k, v`` [B, H_rank, S, D] scattered into
    every rank's slab ``dest[r]`` [B, S/P, heads_total, D] at heads head_offset .. +H_rank.

    An entry of ``dest`` is either a tensor on this GPU or an int: the address of a slab in
    another process's memory mapped here with ``ipc_open`` (the library checks it for null,
    alignment and overlap; its extent is the caller's to guarantee)."""
    P = len(dest)
    shp = _shape_of(q, P)
    for n, t in (("q", q), ("k", k), ("v", v)):
        _bf16_cuda(n, t, tuple(q.shape))
    ptrs = []
    for r, d in enumerate(dest):
        if isinstance(d, int):
            ptrs.append(d)
        else:
            _bf16_cuda(f"dest[{r}]", d, (shp.B, shp.S // P, int(heads_total), shp.D))
            ptrs.append(d.data_ptr())
    arr = (ctypes.c_void_p * P)(*ptrs)
    _check(load().xs_attn_a2a_fused_rank(q.data_ptr(), k.data_ptr(), v.data_ptr(), arr, shp,
                                         int(heads_total), int(head_offset), float(scale or 0.0),
                                         _stream_handle(stream), _ptr(status)))


def attn_a2a_fused_flags(q, k, v, dest, flags, heads_total: int | None = None, head_offset: int = 0,
                         scale: float | None = None, stream=None, status=None):
    """:func:`attn_a2a_fused_rank` that also adds, after storing, each slab's row count to its
    arrival counter ``flags[r]`` (an int32/uint32 CUDA tensor element, or an int address of a
    counter mapped from another process) with a system-scope release.  ``heads_total``
    defaults to this call's own head count (the single-GPU fused call)."""
    P = len(dest)
    if len(flags) != P:
        raise ValueError(f"{len(flags)} counters for {P} slabs")
    shp = _shape_of(q, P)
    ht = shp.H if heads_total is None else int(heads_total)
    for n, t in (("q", q), ("k", k), ("v", v)):
        _bf16_cuda(n, t, tuple(q.shape))
    ptrs = []
    for r, d in enumerate(dest):
        if isinstance(d, int):
            ptrs.append(d)
        else:
            _bf16_cuda(f"dest[{r}]", d, (shp.B, shp.S // P, ht, shp.D))
            ptrs.append(d.data_ptr())
    fptrs = [f if isinstance(f, int) else _counter_ptr(f"flags[{r}]", f) for r, f in enumerate(flags)]
    arr = (ctypes.c_void_p * P)(*ptrs)
    farr = (ctypes.c_void_p * P)(*fptrs)
    _check(load().xs_attn_a2a_fused_flags(q.data_ptr(), k.data_ptr(), v.data_ptr(), arr, farr, shp,
                                          ht, int(head_offset), float(scale or 0.0),
                                          _stream_handle(stream), _ptr(status)))


def _counter_ptr(name: str, t) -> int:
    import torch
    if not isinstance(t, torch.Tensor) or not t.is_cuda or t.dtype not in (torch.int32, torch.uint32):
        raise TypeError(f"{name} must be a 32-bit integer CUDA tensor (one element)")
    if t.numel() < 1:
        raise ValueError(f"{name} is empty")
    return t.data_ptr()


def slab_wait(flag, target: int, limit_ns: int, status, stream=None):
    """Enqueue a wait until the arrival counter ``flag`` reaches ``target`` (modulo 2^32);
    after ``limit_ns`` it gives up and ``status`` (int32 CUDA tensor) receives XS_ERR_TIMEOUT.
    On one GPU, order it after the producing call (stream or event)."""
    fp = flag if isinstance(flag, int) else _counter_ptr("flag", flag)
    _check(load().xs_slab_wait(fp, int(target) & 0xFFFFFFFF, int(limit_ns), _stream_handle(stream),
                               status.data_ptr()))


def ipc_export(t) -> tuple[bytes, int]:
    """CUDA IPC handle of the allocation holding tensor ``t`` (on a GPU), and ``t``'s byte
    offset in it: what another process of this node needs to map ``t`` with ``ipc_open``."""
    if not getattr(t, "is_cuda", False):
        raise ValueError("ipc_export needs a CUDA tensor")
    buf = ctypes.create_string_buffer(IPC_HANDLE_BYTES)
    off = ctypes.c_longlong(0)
    _check(load().xs_ipc_export(t.data_ptr(), buf, ctypes.byref(off)))
    return buf.raw, int(off.value)


def ipc_open(handle: bytes) -> int:
    """Map an allocation exported by another process; returns its base address here."""
    if len(handle) != IPC_HANDLE_BYTES:
        raise ValueError(f"an IPC handle has {IPC_HANDLE_BYTES} bytes, got {len(handle)}")
    base = ctypes.c_void_p(0)
    _check(load().xs_ipc_open(handle, ctypes.byref(base)))
    return int(base.value)


def ipc_close(base: int) -> None:
    """Unmap a base address returned by ``ipc_open``."""
    _check(load().xs_ipc_close(ctypes.c_void_p(base)))


def a2a_pre(src, dst, heads_local: int | None = None, head_offset: int = 0, stream=None):
    """Pre-attention exchange: P sequence-shard slabs ``src[r]`` [B, S/P, H, D] -> head-major
    ``dst`` [B, heads_local, S, D] holding heads head_offset .. head_offset + heads_local."""
    P = len(src)
    B, Sl, H, D = (int(x) for x in src[0].shape)
    heads_local = H if heads_local is None else int(heads_local)
    for r, t in enumerate(src):
        _bf16_cuda(f"src[{r}]", t, (B, Sl, H, D))
    _bf16_cuda("dst", dst, (B, heads_local, Sl * P, D))
    arr = (ctypes.c_void_p * P)(*[t.data_ptr() for t in src])
    _check(load().xs_a2a_pre(arr, dst.data_ptr(), Shape(B, H, Sl * P, D, P), heads_local,
                             int(head_offset), _stream_handle(stream)))


def attn(q, k, v, out, scale: float | None = None, stream=None, status=None, P: int = 1):
    """Attention with head-major output ``out`` [B, H, S, D]."""
    shp = _shape_of(q, P)
    for n, t in (("q", q), ("k", k), ("v", v), ("out", out)):
        _bf16_cuda(n, t, tuple(q.shape))
    _check(load().xs_attn(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), shp,
                          float(scale or 0.0), _stream_handle(stream), _ptr(status)))


def _f32_cuda(name: str, t, shape):
    import torch
    if not isinstance(t, torch.Tensor) or t.dtype != torch.float32:
        raise TypeError(f"{name} must be a float32 torch.Tensor")
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA tensor")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def attn_partial(q, k, v, o_part=None, lse=None, scale: float | None = None, stream=None, status=None):
    """Partial attention of ``q`` [B, H, S, D] over the key/value shard ``k, v`` [B, H, Skv, D].

    Returns ``(o_part, lse)``: fp32 [B, H, S, D] (normalised over the shard's keys) and fp32
    [B, H, S] (natural-log log-sum-exp of the scaled scores).  Outputs are allocated by
    PyTorch when not given.  Skv may be 0.
    """
    import torch
    shp = _shape_of(q, 1)
    _bf16_cuda("q", q)
    if k.dim() != 4 or tuple(k.shape[:2]) != (shp.B, shp.H) or int(k.shape[3]) != shp.D:
        raise ValueError(f"k must be [B, H, Skv, D] matching q; got {tuple(k.shape)}")
    s_kv = int(k.shape[2])
    if s_kv > 0:
        _bf16_cuda("k", k)
        _bf16_cuda("v", v, tuple(k.shape))
    if o_part is None:
        o_part = torch.empty(tuple(q.shape), dtype=torch.float32, device=q.device)
    if lse is None:
        lse = torch.empty(tuple(q.shape[:3]), dtype=torch.float32, device=q.device)
    _f32_cuda("o_part", o_part, tuple(q.shape))
    _f32_cuda("lse", lse, tuple(q.shape[:3]))
    kp = k.data_ptr() if s_kv > 0 else None
    vp_ = v.data_ptr() if s_kv > 0 else None
    _check(load().xs_attn_partial(q.data_ptr(), kp, vp_, o_part.data_ptr(), lse.data_ptr(), shp, s_kv,
                                  float(scale or 0.0), _stream_handle(stream), _ptr(status)))
    return o_part, lse


def lse_merge(o_parts, lse_parts, out=None, lse_out=None, stream=None):
    """Merge partial results: ``o_parts[t]`` fp32 [..., D], ``lse_parts[t]`` fp32 [...].

    Returns ``out`` (bf16 [..., D]) and ``lse_out`` (fp32 [...]; pass ``lse_out=False`` to skip it).
    """
    import torch
    n = len(o_parts)
    if n != len(lse_parts) or n < 1:
        raise ValueError("need as many lse parts as output parts, at least one")
    lead = tuple(o_parts[0].shape[:-1])
    D = int(o_parts[0].shape[-1])
    for t in range(n):
        _f32_cuda(f"o_parts[{t}]", o_parts[t], lead + (D,))
        _f32_cuda(f"lse_parts[{t}]", lse_parts[t], lead)
    if out is None:
        out = torch.empty(lead + (D,), dtype=torch.bfloat16, device=o_parts[0].device)
    _bf16_cuda("out", out, lead + (D,))
    if lse_out is None:
        lse_out = torch.empty(lead, dtype=torch.float32, device=o_parts[0].device)
    if lse_out is not False:
        _f32_cuda("lse_out", lse_out, lead)
    rows = 1
    for x in lead:
        rows *= int(x)
    op = (ctypes.c_void_p * n)(*[t.data_ptr() for t in o_parts])
    lp = (ctypes.c_void_p * n)(*[t.data_ptr() for t in lse_parts])
    _check(load().xs_lse_merge(op, lp, n, out.data_ptr(), None if lse_out is False else lse_out.data_ptr(),
                               rows, D, _stream_handle(stream)))
    return out, (None if lse_out is False else lse_out)


def a2a_relayout(src, dest, stream=None):
    """Post-attention All-to-All as its own pass: head-major ``src`` -> P slabs ``dest``."""
    P = len(dest)
    shp = _shape_of(src, P)
    _bf16_cuda("src", src)
    arr = _dest_array(dest, shp)
    _check(load().xs_a2a_relayout(src.data_ptr(), arr, shp, _stream_handle(stream)))


def burst_probe(scratch, stamps, burst_bytes: int, producers: int, gap_cycles: int,
                n_bursts: int, threads_per_producer: int = 256, stream=None):
    """Burst-Gap microbenchmark; ``stamps`` is a uint64/int64 CUDA tensor [producers, n_bursts, 4]."""
    import torch
    if not scratch.is_cuda or not stamps.is_cuda:
        raise ValueError("scratch and stamps must be CUDA tensors")
    if stamps.dtype not in (torch.int64, torch.uint64) or stamps.numel() < producers * n_bursts * 4:
        raise ValueError("stamps must be int64/uint64 with producers * n_bursts * 4 elements")
    cfg = BurstCfg(int(burst_bytes), int(producers), int(gap_cycles), int(n_bursts),
                   int(threads_per_producer))
    nbytes = scratch.numel() * scratch.element_size()
    _check(load().xs_burst_probe(scratch.data_ptr(), nbytes, cfg, stamps.data_ptr(),
                                 _stream_handle(stream)))


def burst_probe_static(stamps, burst_bytes: int, producers: int, gap_cycles: int, n_bursts: int,
                       threads_per_producer: int = 256, stream=None):
    """Burst-Gap microbenchmark that allocates nothing: the bursts go to the library's fixed
    32 MiB scratch array instead of a caller buffer (see ``xs_burst_probe_static``)."""
    import torch
    if not stamps.is_cuda or stamps.dtype not in (torch.int64, torch.uint64) or \
            stamps.numel() < producers * n_bursts * 4:
        raise ValueError("stamps must be an int64/uint64 CUDA tensor with producers * n_bursts * 4 elements")
    cfg = BurstCfg(int(burst_bytes), int(producers), int(gap_cycles), int(n_bursts),
                   int(threads_per_producer))
    _check(load().xs_burst_probe_static(cfg, stamps.data_ptr(), _stream_handle(stream)))


def selftest_bounded_wait(status, limit_ns: int, stream=None):
    """Launch the bounded-wait self-test; ``status`` (int32 CUDA tensor) receives XS_ERR_TIMEOUT."""
    _check(load().xs_selftest_bounded_wait(status.data_ptr(), int(limit_ns), _stream_handle(stream)))


def selftest_attn_abort(q, k, v, out, status, stall_fill: int, limit_ns: int, stream=None):
    """Head-major attention whose TMA producer stops before fill ``stall_fill`` of every CTA and
    whose waits give up after ``limit_ns``: ``status`` (int32 CUDA tensor, required) receives
    XS_ERR_TIMEOUT and the kernel returns; ``out`` is left partly written."""
    shp = _shape_of(q, 1)
    for n, t in (("q", q), ("k", k), ("v", v), ("out", out)):
        _bf16_cuda(n, t, tuple(q.shape))
    _check(load().xs_selftest_attn_abort(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                         shp, int(stall_fill), int(limit_ns),
                                         _stream_handle(stream), status.data_ptr()))


def alloc_dest(B: int, H: int, S: int, D: int, P: int, device=None, fill: float | None = None):
    """P separately allocated destination slabs [B, S/P, H, D] bf16 (caller-owned memory)."""
    import torch
    if S % P:
        raise ValueError("S must be divisible by P")
    out = []
    for _ in range(P):
        t = torch.empty((B, S // P, H, D), dtype=torch.bfloat16, device=device)
        if fill is not None:
            t.fill_(fill)
        out.append(t)
    return out


class HostPipeline:
    """End-to-end call with host buffers: pinned host q/k/v in, pinned host slabs out.

    The heads are split into ``chunks`` groups that flow through four streams: host-to-device
    copies of a group's q, k, v (input-copy stream), the fused per-rank call for that group's
    heads writing every slab at the group's head offset (the caller's stream for even groups,
    a second compute stream for odd ones), and device-to-host copies of those heads' columns
    of every slab (output-copy stream, one 2-D copy per slab).  The copies of one group
    overlap the kernels of the others; with two compute streams the next group's kernel takes
    each SM that the current one's last wave of work items leaves idle (one CTA of the kernel
    fits an SM, so the two never share one).  Events order each group's stages and, across
    calls, the reuse of its buffers.  ``run`` makes the
    caller's stream wait for every copy it started, so work timed on that stream covers the
    whole step.  ``chunks=1`` runs copies, kernel and copies in sequence on the caller's stream.
    Device buffers are allocated once, here, by PyTorch.
    """

    def __init__(self, B: int, H: int, S: int, D: int, P: int, device=None, scale=None,
                 chunks: int | None = None):
        import torch
        self.shape = (B, H, S, D)
        self.P = P
        self.scale = scale
        dev = device or torch.device("cuda")
        self.device = dev
        if chunks is None:
            # about one wave of 256-row work items per group, at most 20 groups (on the video
            # workload, with two compute streams: 20 groups 21.5-22.0 ms per step, 40 gave 21.6,
            # 10 gave 22.7, 8 gave 23.0; one compute stream and 20 groups 24.2; 1 group 43.0;
            # halving the first and last group, whose copies overlap no kernel, was 1-2% slower)
            sms = torch.cuda.get_device_properties(dev).multi_processor_count
            items_per_head = B * ((S + 255) // 256)
            chunks = max(1, min(20, H, (H * items_per_head) // sms))
        self.chunks = int(chunks)
        hc = (H + self.chunks - 1) // self.chunks
        self.groups = [(h0, min(H, h0 + hc)) for h0 in range(0, H, hc)]
        # per-group contiguous device inputs [B, Hc, S, D]
        self.q = [torch.empty((B, h1 - h0, S, D), dtype=torch.bfloat16, device=dev) for h0, h1 in self.groups]
        self.k = [torch.empty_like(t) for t in self.q]
        self.v = [torch.empty_like(t) for t in self.q]
        self.dest = alloc_dest(B, H, S, D, P, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.s_in = torch.cuda.Stream(device=dev)
        self.s_out = torch.cuda.Stream(device=dev)
        self.s_k2 = torch.cuda.Stream(device=dev)   # kernels of the odd groups
        n = len(self.groups)
        self.ev_in = [torch.cuda.Event() for _ in range(n)]     # group's inputs on the device
        self.ev_kern = [torch.cuda.Event() for _ in range(n)]   # group's kernel done
        self.ev_out = [torch.cuda.Event() for _ in range(n)]    # group's columns copied out
        self._started = False

    @property
    def h2d_bytes(self) -> int:
        return 3 * sum(t.numel() for t in self.q) * 2

    @property
    def d2h_bytes(self) -> int:
        return sum(d.numel() * 2 for d in self.dest)

    def run(self, q_host, k_host, v_host, dest_host, stream=None):
        """Enqueue one step: ``q_host, k_host, v_host`` pinned CPU bf16 [B, H, S, D] in,
        ``dest_host`` P pinned CPU bf16 slabs [B, S/P, H, D] out (ready after the caller's
        stream has reached the point where ``run`` returned)."""
        import torch
        from cuda.bindings import runtime as rt
        s = stream or torch.cuda.current_stream()
        B, H, S, D = self.shape
        for name, t in (("q_host", q_host), ("k_host", k_host), ("v_host", v_host)):
            if tuple(t.shape) != self.shape or t.dtype != torch.bfloat16 or t.is_cuda \
                    or not t.is_contiguous() or not t.is_pinned():
                raise ValueError(f"{name} must be a contiguous pinned CPU bf16 tensor of shape {self.shape}")
        if len(dest_host) != self.P:
            raise ValueError(f"need {self.P} host slabs, got {len(dest_host)}")
        for r, t in enumerate(dest_host):
            if tuple(t.shape) != tuple(self.dest[r].shape) or t.dtype != torch.bfloat16 or t.is_cuda \
                    or not t.is_contiguous() or not t.is_pinned():
                raise ValueError(f"dest_host[{r}] must be a contiguous pinned CPU bf16 tensor of shape "
                                 f"{tuple(self.dest[r].shape)}")
        Sl = S // self.P
        row_bytes = H * D * 2
        start = torch.cuda.Event()
        start.record(s)
        self.s_in.wait_event(start)
        self.s_out.wait_event(start)
        self.s_k2.wait_event(start)
        for g, (h0, h1) in enumerate(self.groups):
            # inputs: the group's buffers are free once its previous kernel is done
            with torch.cuda.stream(self.s_in):
                if self._started:
                    self.s_in.wait_event(self.ev_kern[g])
                for b in range(B):
                    self.q[g][b].copy_(q_host[b, h0:h1], non_blocking=True)
                    self.k[g][b].copy_(k_host[b, h0:h1], non_blocking=True)
                    self.v[g][b].copy_(v_host[b, h0:h1], non_blocking=True)
                self.ev_in[g].record(self.s_in)
            # kernel: its inputs have landed and its slab columns have been copied out
            ks = s if g % 2 == 0 else self.s_k2
            ks.wait_event(self.ev_in[g])
            if self._started:
                ks.wait_event(self.ev_out[g])
            attn_a2a_fused_rank(self.q[g], self.k[g], self.v[g], self.dest, heads_total=H,
                                head_offset=h0, scale=self.scale, stream=ks, status=self.status)
            self.ev_kern[g].record(ks)
            # outputs: the group's heads in every slab, one 2-D copy per slab
            self.s_out.wait_event(self.ev_kern[g])
            width = (h1 - h0) * D * 2
            for dh, dd in zip(dest_host, self.dest):
                err, = rt.cudaMemcpy2DAsync(dh.data_ptr() + h0 * D * 2, row_bytes, dd.data_ptr() + h0 * D * 2,
                                            row_bytes, width, B * Sl,
                                            rt.cudaMemcpyKind.cudaMemcpyDeviceToHost, self.s_out.cuda_stream)
                if err != rt.cudaError_t.cudaSuccess:
                    raise RuntimeError(f"output copy failed: {err}")
            self.ev_out[g].record(self.s_out)
        self._started = True
        # the caller's stream covers every copy of this step
        for g in range(len(self.groups)):
            s.wait_event(self.ev_out[g])
