"""The allocation-free Burst-Gap probe (``xs_burst_probe_static``) against the probe that uses
a caller-allocated scratch buffer (``xs_burst_probe``), both called through the C ABI.

It is for callers that cannot call cudaMalloc (e.g. a monitoring hook inside a serving
process whose device memory belongs to that process's caching allocator): the bursts go to
a fixed 32 MiB array inside the library.  Both entry points run the same kernel, so with
the same configuration and a scratch ring of the same size their stamps must agree: every
(producer, burst) record written and ordered, the compute-gap cycles within 10 % (a fixed
dependent FMA chain) and the median issue cycles within a factor of 3 (store issue timing
varies run to run).  Checked on two calls in a row.  The property the entry point exists
for is checked as well: across calls after the first, neither torch's allocator counters nor
the device's free memory (cudaMemGetInfo) move.  A burst of exactly the array's size, the
largest accepted and the edge of the cyclic walk, writes every stamp.  This file is
collected last.
"""
import ctypes

import pytest
import torch

import ulysses_attention_output_b200 as xs

pytestmark = pytest.mark.gpu

PRODUCERS, N_BURSTS, BURST, GAP, THREADS = 8, 24, 8 * 16384, 8000, 256
STATIC_BYTES = 32 << 20
GAP_RTOL = 0.10
ISSUE_FACTOR = 3.0


@pytest.fixture(scope="module")
def lib(cuda_device):
    from ulysses_attention_output_b200 import build
    build.build()
    return xs.load()


def summarize(stamps: torch.Tensor):
    st = stamps.cpu().to(torch.int64)
    assert (st[..., 0] > 0).all(), "a burst record was not written"
    assert (st[..., 1] >= st[..., 0]).all() and (st[..., 2] >= st[..., 1]).all()
    assert (st[:, 1:, 3] >= st[:, :-1, 3]).all()
    steady = st[:, 2:]  # the first bursts pay cold TLB / L2 misses
    issue = (steady[..., 1] - steady[..., 0]).double().median().item()
    gap = (steady[..., 2] - steady[..., 1]).double().median().item()
    return issue, gap


def run_allocating(lib):
    scratch = torch.empty(STATIC_BYTES, dtype=torch.uint8, device="cuda")
    stamps = torch.zeros((PRODUCERS, N_BURSTS, 4), dtype=torch.int64, device="cuda")
    cfg = xs.BurstCfg(BURST, PRODUCERS, GAP, N_BURSTS, THREADS)
    assert lib.xs_burst_probe(scratch.data_ptr(), STATIC_BYTES, cfg, stamps.data_ptr(), None) == xs.XS_OK
    torch.cuda.synchronize()
    return summarize(stamps)


def run_static(lib):
    stamps = torch.zeros((PRODUCERS, N_BURSTS, 4), dtype=torch.int64, device="cuda")
    cfg = xs.BurstCfg(BURST, PRODUCERS, GAP, N_BURSTS, THREADS)
    rc = lib.xs_burst_probe_static(cfg, stamps.data_ptr(), None)
    assert rc == xs.XS_OK, lib.xs_last_error_detail()
    torch.cuda.synchronize()
    return summarize(stamps)


def test_static_probe_matches_allocating_probe_twice(lib):
    ref_issue, ref_gap = run_allocating(lib)
    for call in range(2):
        issue, gap = run_static(lib)
        assert abs(gap - ref_gap) <= GAP_RTOL * ref_gap, (call, gap, ref_gap)
        assert ref_issue / ISSUE_FACTOR <= issue <= ref_issue * ISSUE_FACTOR, (call, issue, ref_issue)


def test_static_probe_rejects_oversize_burst(lib):
    stamps = torch.zeros((PRODUCERS, 1, 4), dtype=torch.int64, device="cuda")
    cfg = xs.BurstCfg(STATIC_BYTES + 16 * PRODUCERS, PRODUCERS, 0, 1, THREADS)
    assert lib.xs_burst_probe_static(cfg, stamps.data_ptr(), None) == xs.XS_ERR_UNSUPPORTED
    assert b"exceeds the fixed" in lib.xs_last_error_detail()
    torch.cuda.synchronize()
    assert (stamps == 0).all()  # nothing was launched


def test_static_probe_allocates_nothing(lib):
    """After a first call (which may load the library's device code), further calls change
    neither torch's allocation counters nor the device's free memory."""
    stamps = torch.zeros((PRODUCERS, N_BURSTS, 4), dtype=torch.int64, device="cuda")
    cfg = xs.BurstCfg(BURST, PRODUCERS, GAP, N_BURSTS, THREADS)
    assert lib.xs_burst_probe_static(cfg, stamps.data_ptr(), None) == xs.XS_OK
    torch.cuda.synchronize()
    stats0 = torch.cuda.memory_stats()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        assert lib.xs_burst_probe_static(cfg, stamps.data_ptr(), None) == xs.XS_OK
    torch.cuda.synchronize()
    stats1 = torch.cuda.memory_stats()
    free1, _ = torch.cuda.mem_get_info()
    for key in ("allocation.all.allocated", "segment.all.allocated", "reserved_bytes.all.current"):
        assert stats1.get(key, 0) == stats0.get(key, 0), key
    assert free1 == free0


def test_static_probe_burst_of_the_whole_array(lib):
    """burst_bytes == XS_BURST_STATIC_SCRATCH_BYTES: every producer's share fills its part of
    the array exactly once per burst; all records are written and ordered."""
    n = 3
    stamps = torch.zeros((PRODUCERS, n, 4), dtype=torch.int64, device="cuda")
    cfg = xs.BurstCfg(STATIC_BYTES, PRODUCERS, 0, n, THREADS)
    rc = lib.xs_burst_probe_static(cfg, stamps.data_ptr(), None)
    assert rc == xs.XS_OK, lib.xs_last_error_detail()
    torch.cuda.synchronize()
    st = stamps.cpu()
    assert (st[..., 0] > 0).all() and (st[..., 1] >= st[..., 0]).all() and (st[..., 2] >= st[..., 1]).all()
