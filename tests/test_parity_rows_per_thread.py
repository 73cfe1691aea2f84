"""GPU parity of every row-tile kind of the scan kernels against the fp64 oracle.

A row tile is `rows` channels handled by rows / rpt threads, each keeping `rpt` channels'
states in registers (two per thread share one read of each step's B and C).  Every kind
is forced through every schedule it supports (a single forward kernel, chunk summaries +
forward, the chained hand-over, the fused look-back and the split chunks; the last three
take one-warp tiles only), on ragged channel counts (partial last tiles), with structured and general A,
the zero-order hold, an initial state and packed sequences.
"""
import numpy as np
import pytest

import oracle
import synth
from gpu_util import check_close, run_scan, to_f64

pytestmark = pytest.mark.gpu

KINDS = [(32, 1), (64, 1), (64, 2), (128, 2)]
SCHEDULES = [("forward", 0), ("summaries+forward", 64), ("summaries+forward", 192), ("chained", 128),
             ("fused", 128), ("split", 256), ("split", 512)]


def _reset():
    import selective_state_space_46_b200 as m
    for opt in (m.MSSM_OPT_FORCE_GENERAL_A, m.MSSM_OPT_CHUNK_LEN, m.MSSM_OPT_SCHEDULE, m.MSSM_OPT_ROWS_PER_CTA,
                m.MSSM_OPT_ROWS_PER_THREAD):
        m.mssm_set_option(opt, 0)


@pytest.fixture(autouse=True)
def _defaults(cuda_device):
    _reset()
    yield
    _reset()


def _force(rows, rpt, schedule, chunk):
    import selective_state_space_46_b200 as m
    m.mssm_set_option(m.MSSM_OPT_ROWS_PER_CTA, rows)
    m.mssm_set_option(m.MSSM_OPT_ROWS_PER_THREAD, rpt)
    m.mssm_set_option(m.MSSM_OPT_SCHEDULE, m.SCHEDULES[schedule])
    m.mssm_set_option(m.MSSM_OPT_CHUNK_LEN, chunk)


def _supported(rows, rpt, schedule):
    return schedule not in ("chained", "fused", "split") or rows == 32 * rpt


def _random_A(dim, seed):
    rng = np.random.default_rng(seed)
    return (-np.exp(rng.uniform(-1.0, 1.5, size=(dim, 16)))).astype(np.float32)


def _plan_is(rows, rpt, schedule, Bt, D, L, io):
    import selective_state_space_46_b200 as m
    plan = m.mssm_scan_plan(Bt, D, L, io_dtype=io)
    assert (plan["rows_per_cta"], plan["rows_per_thread"], plan["schedule"]) == (rows, rpt, schedule), plan


@pytest.mark.parametrize("rows,rpt", KINDS)
@pytest.mark.parametrize("schedule,chunk", SCHEDULES)
@pytest.mark.parametrize("structured", [True, False])
def test_kinds_and_schedules(rows, rpt, schedule, chunk, structured):
    if not _supported(rows, rpt, schedule):
        pytest.skip("the persistent schedules take one-warp tiles")
    Bt, D, L = 2, 200, 1000
    _force(rows, rpt, schedule, chunk)
    _plan_is(rows, rpt, schedule, Bt, D, L, "bf16")
    inp = synth.make_scan_inputs(Bt, D, L, io_dtype="bf16", seed=rows + rpt + chunk,
                                 delta_range=(1e-4, 1e-2) if chunk else (1e-3, 1e-1))
    if not structured:
        inp.A = _random_A(D, rows)
    out, last = run_scan(inp)
    import selective_state_space_46_b200 as m
    m.mssm_get_error()
    y_ref, h_ref = oracle.scan_inputs(inp)
    check_close(to_f64(out), y_ref, "bf16", "y")
    check_close(to_f64(last), h_ref, "bf16", "last_state")


@pytest.mark.parametrize("rows,rpt", [(64, 2), (128, 2)])
@pytest.mark.parametrize("Bt,D,L", [(1, 1, 1), (2, 3, 7), (1, 65, 33), (3, 130, 257), (1, 129, 640)])
def test_two_rows_ragged_shapes(rows, rpt, Bt, D, L):
    """Channel counts below, at and past a tile (a thread's second row may be past D), and
    lengths below a block, a chunk and a B/C stage."""
    _force(rows, rpt, "forward", 0)
    inp = synth.make_scan_inputs(Bt, D, L, io_dtype="bf16", seed=D + L)
    out, last = run_scan(inp)
    y_ref, h_ref = oracle.scan_inputs(inp)
    check_close(to_f64(out), y_ref, "bf16", "y")
    check_close(to_f64(last), h_ref, "bf16", "last_state")


@pytest.mark.parametrize("rows,rpt", [(64, 2), (128, 2)])
@pytest.mark.parametrize("schedule,chunk", SCHEDULES)
@pytest.mark.parametrize("structured", [True, False])
def test_two_rows_zoh_and_h0(rows, rpt, schedule, chunk, structured):
    if not _supported(rows, rpt, schedule):
        pytest.skip("the persistent schedules take one-warp tiles")
    import selective_state_space_46_b200 as m
    _force(rows, rpt, schedule, chunk)
    inp = synth.make_scan_inputs(2, 150, 700, io_dtype="bf16", seed=17)
    if not structured:
        inp.A = _random_A(150, 17)
    h0 = np.random.default_rng(5).normal(0.0, 0.5, size=(2, 150, 16)).astype(np.float32)
    import torch
    from gpu_util import dev_scan_inputs
    dev = dev_scan_inputs(inp)
    out, last = m.selective_scan_fwd(dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"], dev["D"], dev["z"],
                                     dev["delta_bias"], inp.softplus, h0=torch.from_numpy(h0).cuda(), zoh=True)
    torch.cuda.synchronize()
    m.mssm_get_error()
    y_ref, h_ref = oracle.scan_inputs(inp, h0=h0.astype(np.float64), zoh=True)
    check_close(to_f64(out), y_ref, "bf16", "y")
    check_close(to_f64(last), h_ref, "bf16", "last_state")


@pytest.mark.parametrize("rows,rpt", [(64, 2), (128, 2)])
@pytest.mark.parametrize("schedule,chunk", [("forward", 0), ("summaries+forward", 64), ("summaries+forward", 128),
                                            ("chained", 64)])
def test_two_rows_packed_sequences(rows, rpt, schedule, chunk):
    """Packed sequences: chunks that start inside a 16-byte block (identity head steps)."""
    if not _supported(rows, rpt, schedule):
        pytest.skip("the persistent schedules take one-warp tiles")
    import torch
    import selective_state_space_46_b200 as m
    from gpu_util import dev_scan_inputs
    _force(rows, rpt, schedule, chunk)
    lengths = [1, 5, 64, 65, 130, 257, 3, 700]
    inp = synth.make_scan_inputs(1, 150, int(sum(lengths)), io_dtype="bf16", seed=23)
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    dev = dev_scan_inputs(inp)
    out, last = m.selective_scan_fwd(dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"], dev["D"], dev["z"],
                                     dev["delta_bias"], inp.softplus, cu_seqlens=torch.from_numpy(cu).cuda(),
                                     max_seqlen=max(lengths))
    torch.cuda.synchronize()
    m.mssm_get_error()
    y_ref, h_ref = oracle.scan_varlen(inp.f64("u"), inp.f64("delta"), inp.f64("A"), inp.f64("B"), inp.f64("C"),
                                      cu, inp.f64("D"), inp.f64("z"), inp.f64("delta_bias"), inp.softplus)
    check_close(to_f64(out), y_ref, "bf16", "y")
    check_close(to_f64(last), h_ref, "bf16", "last_state")


def test_f32_io_ignores_two_rows_per_thread():
    """Two rows per thread exist for bf16 I/O only: forcing them with fp32 I/O plans one."""
    import selective_state_space_46_b200 as m
    _force(0, 2, "forward", 0)
    plan = m.mssm_scan_plan(2, 100, 300, io_dtype="f32")
    assert plan["rows_per_thread"] == 1
    inp = synth.make_scan_inputs(2, 100, 300, io_dtype="f32", seed=2)
    out, last = run_scan(inp)
    y_ref, h_ref = oracle.scan_inputs(inp)
    check_close(to_f64(out), y_ref, "f32", "y")
    check_close(to_f64(last), h_ref, "f32", "last_state")


@pytest.mark.parametrize("rows,rpt", [(32, 1), (64, 2)])
@pytest.mark.parametrize("Bt,D,L,chunk", [(1, 40, 1000, 256), (2, 100, 3000, 512), (1, 70, 513, 256),
                                          (1, 70, 257, 256), (3, 33, 2100, 1024), (1, 64, 300, 256)])
@pytest.mark.parametrize("io", ["bf16", "f32"])
def test_split_chunks_ragged(rows, rpt, Bt, D, L, chunk, io):
    """The split-chunk schedule: lengths that end inside a chunk and inside a warp's
    sub-segment, chunks whose later sub-segments are empty, a single chunk, partial tiles."""
    if io == "f32" and rpt == 2:
        pytest.skip("two rows per thread exist for bf16 I/O only")
    import selective_state_space_46_b200 as m
    _force(rows, rpt, "split", chunk)
    _plan_is(rows, rpt, "split", Bt, D, L, io)
    inp = synth.make_scan_inputs(Bt, D, L, io_dtype=io, seed=L + D, delta_range=(1e-4, 1e-2))
    out, last = run_scan(inp)
    m.mssm_get_error()
    y_ref, h_ref = oracle.scan_inputs(inp)
    check_close(to_f64(out), y_ref, io, "y")
    check_close(to_f64(last), h_ref, io, "last_state")


def test_split_chunks_long_sequence():
    """Many chunks handed over one after another (1 x 512 x 32768, 64 chunks of 512)."""
    import selective_state_space_46_b200 as m
    _force(32, 1, "split", 512)
    inp = synth.make_scan_inputs(1, 512, 32768, io_dtype="bf16", seed=31, delta_range=(1e-4, 1e-2))
    out, last = run_scan(inp)
    m.mssm_get_error()
    y_ref, h_ref = oracle.scan_inputs(inp)
    check_close(to_f64(out), y_ref, "bf16", "y")
    check_close(to_f64(last), h_ref, "bf16", "last_state")
