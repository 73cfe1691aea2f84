"""The scan entry point that allocates nothing (mssm_selective_scan_fwd_noalloc).

It exists for callers that cannot allocate device memory while the scan runs:
an application whose device memory is wholly owned by its own allocator or a
pre-reserved pool, or a loop that cannot take cudaMalloc's device-wide
synchronisation.  Instead of the library's cudaMalloc'd carry workspace it uses
a fixed array in the library's device image, shared by every call.

This file is collected last so that a run stopping at the first failure has
already run every other test; it also passes on its own in a fresh process.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import TOL, dev_scan_inputs

pytestmark = pytest.mark.gpu


def _scan_both(inp, m):
    d = dev_scan_inputs(inp)
    outs = []
    for fn in (m.mssm_selective_scan_fwd, m.mssm_selective_scan_fwd_noalloc):
        out = torch.empty_like(d["u"])
        last = torch.empty(inp.batch, inp.dim, 16, device="cuda")
        fn(d["u"], d["delta"], d["A"], d["B"], d["C"], d["D"], d["z"], d["delta_bias"], inp.softplus, out, last)
        torch.cuda.synchronize()
        outs.append((out.float().cpu().numpy().astype(np.float64), last.cpu().numpy().astype(np.float64)))
    return outs


def _close(got, ref, io_dtype):
    tol = TOL[io_dtype]
    assert np.isfinite(got).all()
    err = np.abs(got - ref) / (1.0 + np.abs(ref))
    assert float(err.max()) <= tol, float(err.max())


def _check(inp, m, calls=2):
    """`calls` no-allocation scans in a row of one problem: each against the allocating scan and
    against the fp64 oracle (so a fault shared by both entry points, such as in the launch
    planning or the workspace layout, is caught too)."""
    y_o, h_o = oracle.scan_inputs(inp)
    for _ in range(calls):
        (y_ref, h_ref), (y_na, h_na) = _scan_both(inp, m)
        _close(y_na, y_ref, inp.io_dtype)
        _close(h_na, h_ref, inp.io_dtype)
        _close(y_na, y_o, inp.io_dtype)
        _close(h_na, h_o, inp.io_dtype)


def test_noalloc_matches_the_allocating_scan_on_two_calls_in_a_row(cuda_device):
    import selective_state_space_46_b200 as m
    m.mssm_set_option(m.MSSM_OPT_CHUNK_LEN, 0)
    try:
        # two different problems in a row, both split into chunks (so both use the
        # fixed scratch); the second finds the first one's leftovers in it
        first = synth.workload_inputs("scan_bf16_2x1536x2048", seed=3)
        plan = m.mssm_scan_plan(first.batch, first.dim, first.length)
        assert plan["n_chunks"] > 1
        second = synth.make_scan_inputs(3, 200, 1000, io_dtype="f32", seed=4, delta_range=(1e-4, 1e-2))
        for inp in (first, second):
            if inp is second:
                m.mssm_set_option(m.MSSM_OPT_CHUNK_LEN, 128)
            _check(inp, m, calls=1)
    finally:
        m.mssm_set_option(m.MSSM_OPT_CHUNK_LEN, 0)


def test_noalloc_rejects_problems_beyond_its_scratch(cuda_device):
    import selective_state_space_46_b200 as m
    inp = synth.make_scan_inputs(1, 4096, 64 * 40, io_dtype="bf16", seed=5)
    d = dev_scan_inputs(inp)
    out = torch.empty_like(d["u"])
    m.mssm_set_option(m.MSSM_OPT_CHUNK_LEN, 64)   # 39 chunk summaries x 4096 rows x 68 B > 8 MiB
    try:
        with pytest.raises(m.MssmError) as e:
            m.mssm_selective_scan_fwd_noalloc(d["u"], d["delta"], d["A"], d["B"], d["C"], d["D"], d["z"],
                                              d["delta_bias"], True, out, None)
        assert e.value.status == m.MSSM_ERR_UNSUPPORTED
        assert "scratch" in str(e.value)
    finally:
        m.mssm_set_option(m.MSSM_OPT_CHUNK_LEN, 0)


def test_noalloc_chained_schedule_matches(cuda_device):
    """A shape with many row tiles uses the chained schedule; its hand-over state
    also lives in the fixed scratch."""
    import selective_state_space_46_b200 as m
    m.mssm_set_option(m.MSSM_OPT_CHUNK_LEN, 0)
    inp = synth.make_scan_inputs(2, 9600, 1000, io_dtype="bf16", seed=6)
    assert m.mssm_scan_plan(inp.batch, inp.dim, inp.length)["schedule"] == "chained"
    _check(inp, m, calls=2)


@pytest.mark.parametrize("io", ["bf16", "f32"])
def test_noalloc_fused_schedule_two_calls(cuda_device, io):
    """The fused look-back schedule keeps the most in the fixed array: per-chunk flags, chunk
    sums, summaries and end states.  Forced, with short chunks, twice in a row: the second call
    finds the first call's published flags in the array and must clear them first."""
    import selective_state_space_46_b200 as m
    m.mssm_set_option(m.MSSM_OPT_SCHEDULE, m.SCHEDULES["fused"])
    m.mssm_set_option(m.MSSM_OPT_CHUNK_LEN, 64)
    try:
        inp = synth.make_scan_inputs(2, 100, 700, io_dtype=io, seed=8, delta_range=(1e-4, 1e-2))
        assert m.mssm_scan_plan(inp.batch, inp.dim, inp.length)["schedule"] == "fused"
        _check(inp, m, calls=2)
        m.mssm_get_error()   # no bounded look-back wait gave up
    finally:
        m.mssm_set_option(m.MSSM_OPT_SCHEDULE, 0)
        m.mssm_set_option(m.MSSM_OPT_CHUNK_LEN, 0)
