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
            (y_ref, h_ref), (y_na, h_na) = _scan_both(inp, m)
            _close(y_na, y_ref, inp.io_dtype)
            _close(h_na, h_ref, inp.io_dtype)
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
    for _ in range(2):
        (y_ref, h_ref), (y_na, h_na) = _scan_both(inp, m)
        _close(y_na, y_ref, inp.io_dtype)
        _close(h_na, h_ref, inp.io_dtype)
