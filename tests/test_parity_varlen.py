"""GPU parity of the packed variable-length scan (mssm_selective_scan_fwd_ex with
cu_seqlens) against the oracle's per-sequence definition: every sequence is its own scan
from zero (or from h0[s]) over its steps of the packed row, and its final state lands
in last_state[s].  Sequence starts are deliberately not 16-byte aligned."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import check_close, dev_scan_inputs, to_f64

pytestmark = pytest.mark.gpu

LENGTHS = [5, 0, 1, 8, 9, 63, 64, 65, 130, 700, 3, 257]


def _reset():
    import selective_state_space_46_b200 as m
    m.mssm_set_option(m.MSSM_OPT_FORCE_GENERAL_A, 0)
    m.mssm_set_option(m.MSSM_OPT_CHUNK_LEN, 0)
    m.mssm_set_option(m.MSSM_OPT_SCHEDULE, 0)
    m.mssm_set_option(m.MSSM_OPT_ROWS_PER_CTA, 0)


@pytest.fixture(autouse=True)
def _defaults(cuda_device):
    _reset()
    yield
    _reset()


def packed(lengths, D, io, seed, **kw):
    T = int(sum(lengths))
    inp = synth.make_scan_inputs(1, D, T, io_dtype=io, seed=seed, **kw)
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    return inp, cu


def run_varlen(inp, cu, h0=None, zoh=False, max_seqlen=None):
    import selective_state_space_46_b200 as m
    dev = dev_scan_inputs(inp)
    cu_d = torch.from_numpy(cu).cuda()
    h0_d = None if h0 is None else torch.from_numpy(np.ascontiguousarray(h0, np.float32)).cuda()
    out, last = m.selective_scan_fwd(dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"], dev["D"], dev["z"],
                                     dev["delta_bias"], inp.softplus, h0=h0_d, zoh=zoh, cu_seqlens=cu_d,
                                     max_seqlen=max_seqlen)
    torch.cuda.synchronize()
    m.mssm_get_error()
    return out, last


def oracle_varlen(inp, cu, h0=None, zoh=False):
    return oracle.scan_varlen(inp.f64("u"), inp.f64("delta"), inp.f64("A"), inp.f64("B"), inp.f64("C"), cu,
                              inp.f64("D"), inp.f64("z"), inp.f64("delta_bias"), inp.softplus,
                              h0=None if h0 is None else h0.astype(np.float64), zoh=zoh)


def random_A(dim, seed):
    rng = np.random.default_rng(seed)
    return (-np.exp(rng.uniform(-1.0, 1.5, size=(dim, 16)))).astype(np.float32)


@pytest.mark.parametrize("schedule,chunk", [("forward", 0), ("summaries+forward", 64),
                                            ("summaries+forward", 192), ("chained", 64), ("chained", 128)])
@pytest.mark.parametrize("structured", [True, False])
@pytest.mark.parametrize("io", ["bf16", "f32"])
def test_varlen_each_schedule(schedule, chunk, structured, io):
    import selective_state_space_46_b200 as m
    m.mssm_set_option(m.MSSM_OPT_SCHEDULE, m.SCHEDULES[schedule])
    if chunk:
        m.mssm_set_option(m.MSSM_OPT_CHUNK_LEN, chunk)
    inp, cu = packed(LENGTHS, 70, io, seed=3)
    if not structured:
        inp.A = random_A(70, 3)
    out, last = run_varlen(inp, cu)
    y_ref, h_ref = oracle_varlen(inp, cu)
    check_close(to_f64(out), y_ref, io, "y")
    check_close(to_f64(last), h_ref, io, "last_state")


@pytest.mark.parametrize("schedule,chunk", [("forward", 0), ("summaries+forward", 64),
                                            ("summaries+forward", 128)])
@pytest.mark.parametrize("structured", [True, False])
@pytest.mark.parametrize("io", ["bf16", "f32"])
def test_varlen_64_row_tiles(schedule, chunk, structured, io):
    import selective_state_space_46_b200 as m
    m.mssm_set_option(m.MSSM_OPT_ROWS_PER_CTA, 64)
    m.mssm_set_option(m.MSSM_OPT_SCHEDULE, m.SCHEDULES[schedule])
    if chunk:
        m.mssm_set_option(m.MSSM_OPT_CHUNK_LEN, chunk)
    inp, cu = packed(LENGTHS, 100, io, seed=4)
    if not structured:
        inp.A = random_A(100, 4)
    h0 = np.random.default_rng(4).standard_normal((len(LENGTHS), 100, 16)).astype(np.float32) * 0.3
    out, last = run_varlen(inp, cu, h0=h0)
    y_ref, h_ref = oracle_varlen(inp, cu, h0=h0)
    check_close(to_f64(out), y_ref, io, "y")
    check_close(to_f64(last), h_ref, io, "last_state")


@pytest.mark.parametrize("schedule", ["forward", "summaries+forward", "chained"])
@pytest.mark.parametrize("zoh", [False, True])
def test_varlen_with_h0_and_zoh(schedule, zoh):
    import selective_state_space_46_b200 as m
    m.mssm_set_option(m.MSSM_OPT_SCHEDULE, m.SCHEDULES[schedule])
    if schedule != "forward":
        m.mssm_set_option(m.MSSM_OPT_CHUNK_LEN, 64)
    inp, cu = packed(LENGTHS, 40, "f32", seed=4)
    h0 = np.random.default_rng(2).normal(0, 0.5, size=(len(LENGTHS), 40, 16)).astype(np.float32)
    out, last = run_varlen(inp, cu, h0=h0, zoh=zoh)
    y_ref, h_ref = oracle_varlen(inp, cu, h0=h0, zoh=zoh)
    check_close(to_f64(out), y_ref, "f32", "y")
    check_close(to_f64(last), h_ref, "f32", "last_state")


def test_varlen_many_sequences_automatic_plan():
    """24 sequences of 1..4096 steps (48 K steps packed) over 1536 channels, bf16."""
    rng = np.random.default_rng(7)
    lengths = [int(x) for x in rng.integers(1, 4097, size=24)]
    inp, cu = packed(lengths, 1536, "bf16", seed=7)
    out, last = run_varlen(inp, cu)
    y_ref, h_ref = oracle_varlen(inp, cu)
    check_close(to_f64(out), y_ref, "bf16", "y")
    check_close(to_f64(last), h_ref, "bf16", "last_state")


def test_varlen_single_sequence_equals_plain_scan():
    import selective_state_space_46_b200 as m
    inp = synth.make_scan_inputs(1, 64, 1000, io_dtype="f32", seed=9)
    dev = dev_scan_inputs(inp)
    y0, h0 = m.selective_scan_fwd(dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"], dev["D"], dev["z"],
                                  dev["delta_bias"], True)
    y1, h1 = run_varlen(inp, np.array([0, 1000], np.int32))
    # packed sequences summarise chunks by the forward sweep, the plain call by the backward
    # one: the same sums in another order, so equal to fp32 rounding, not bit for bit
    assert float(((y1 - y0).abs() / (1 + y0.abs())).max()) <= 2e-5
    assert float(((h1 - h0).abs() / (1 + h0.abs())).max()) <= 2e-5


def test_varlen_empty_sequences():
    inp, cu = packed([0, 0, 0], 32, "f32", seed=1)
    out, last = run_varlen(inp, cu, max_seqlen=0)
    assert out.numel() == 0 and float(last.abs().max()) == 0.0
    h0 = np.full((3, 32, 16), 0.25, np.float32)
    out, last = run_varlen(inp, cu, h0=h0, max_seqlen=0)
    assert float((last - 0.25).abs().max()) == 0.0


def test_varlen_inconsistent_offsets_are_reported():
    import selective_state_space_46_b200 as m
    inp, cu = packed([100, 300], 32, "f32", seed=2)
    with pytest.raises(m.MssmError) as err:
        run_varlen(inp, cu, max_seqlen=200)  # the second sequence is longer than max_seqlen
    assert err.value.status == m.MSSM_ERR_INVALID_ARG
    m.mssm_get_error()  # cleared; the context is still usable
    out, last = run_varlen(inp, cu)
    y_ref, h_ref = oracle_varlen(inp, cu)
    check_close(to_f64(out), y_ref, "f32", "y")
