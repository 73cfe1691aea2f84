"""GPU parity of the scan options of mssm_selective_scan_fwd_ex (initial state h0,
zero-order-hold discretisation) and of the zero-order-hold decode step, against the
fp64 oracle, under every schedule and both A paths.

The zero-order-hold input gain per state is (exp(delta A_n) - 1) / A_n ("Linear
Attention vs Softmax Attention ...", section Core Concepts, item 3; "State Space
Models in Large Language Models ...", section Discretization)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import check_close, check_scan_every_row, dev_scan_inputs, to_dev, to_f64

pytestmark = pytest.mark.gpu

SCHEDULES = ["forward", "summaries+forward", "chained", "fused"]


def _reset():
    import selective_state_space_46_b200 as m
    m.mssm_set_option(m.MSSM_OPT_FORCE_GENERAL_A, 0)
    m.mssm_set_option(m.MSSM_OPT_CHUNK_LEN, 0)
    m.mssm_set_option(m.MSSM_OPT_SCHEDULE, 0)
    m.mssm_set_option(m.MSSM_OPT_DECODE_PATH, 0)


@pytest.fixture(autouse=True)
def _defaults(cuda_device):
    _reset()
    yield
    _reset()


def random_A(dim, seed, zero_states=()):
    rng = np.random.default_rng(seed)
    A = (-np.exp(rng.uniform(-1.0, 1.5, size=(dim, 16)))).astype(np.float32)
    for n in zero_states:
        A[:, n] = 0.0
    return A


def _force(schedule, chunk=128):
    import selective_state_space_46_b200 as m
    m.mssm_set_option(m.MSSM_OPT_SCHEDULE, m.SCHEDULES[schedule])
    if schedule != "forward":
        m.mssm_set_option(m.MSSM_OPT_CHUNK_LEN, chunk)


def _run_ex(inp, h0=None, zoh=False):
    import selective_state_space_46_b200 as m
    dev = dev_scan_inputs(inp)
    h0_d = None if h0 is None else torch.from_numpy(np.ascontiguousarray(h0, np.float32)).cuda()
    out, last = m.selective_scan_fwd(dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"], dev["D"], dev["z"],
                                     dev["delta_bias"], inp.softplus, h0=h0_d, zoh=zoh)
    torch.cuda.synchronize()
    m.mssm_get_error()
    return out, last


def _h0(inp, seed):
    return np.random.default_rng(seed).normal(0.0, 0.5, size=(inp.batch, inp.dim, 16)).astype(np.float32)


@pytest.mark.parametrize("schedule", SCHEDULES)
@pytest.mark.parametrize("structured", [True, False])
@pytest.mark.parametrize("io", ["bf16", "f32"])
def test_initial_state(schedule, structured, io):
    _force(schedule)
    inp = synth.make_scan_inputs(2, 70, 600, io_dtype=io, seed=3)
    if not structured:
        inp.A = random_A(70, 3)
    h0 = _h0(inp, 9)
    out, last = _run_ex(inp, h0=h0)
    y_ref, h_ref = oracle.scan_inputs(inp, h0=h0.astype(np.float64))
    check_close(to_f64(out), y_ref, io, "y")
    check_close(to_f64(last), h_ref, io, "last_state")


@pytest.mark.parametrize("zoh", [False, True])
def test_resume_reproduces_whole_sequence(zoh):
    """Prefill in two pieces: the second piece starts from the first piece's last_state."""
    import selective_state_space_46_b200 as m
    inp = synth.make_scan_inputs(2, 96, 900, io_dtype="f32", seed=5)
    whole, last_whole = _run_ex(inp, zoh=zoh)
    dev = dev_scan_inputs(inp)
    cut = 413
    part = {k: (v[..., :cut].contiguous() if k in ("u", "delta", "B", "C", "z") else v) for k, v in dev.items()}
    rest = {k: (v[..., cut:].contiguous() if k in ("u", "delta", "B", "C", "z") else v) for k, v in dev.items()}
    y1, h1 = m.selective_scan_fwd(part["u"], part["delta"], part["A"], part["B"], part["C"], part["D"], part["z"],
                                  part["delta_bias"], True, zoh=zoh)
    y2, h2 = m.selective_scan_fwd(rest["u"], rest["delta"], rest["A"], rest["B"], rest["C"], rest["D"], rest["z"],
                                  rest["delta_bias"], True, h0=h1, zoh=zoh)
    torch.cuda.synchronize()
    y = torch.cat([y1, y2], dim=-1)
    assert float(((y - whole).abs() / (1 + whole.abs())).max()) <= 2e-5
    assert float(((h2 - last_whole).abs() / (1 + last_whole.abs())).max()) <= 2e-5


@pytest.mark.parametrize("schedule", SCHEDULES)
@pytest.mark.parametrize("structured", [True, False])
@pytest.mark.parametrize("io", ["bf16", "f32"])
def test_zoh_scan(schedule, structured, io):
    _force(schedule)
    inp = synth.make_scan_inputs(2, 70, 600, io_dtype=io, seed=4)
    if not structured:
        inp.A = random_A(70, 4)
    out, last = _run_ex(inp, zoh=True)
    y_ref, h_ref = oracle.scan_inputs(inp, zoh=True)
    check_close(to_f64(out), y_ref, io, "y")
    check_close(to_f64(last), h_ref, io, "last_state")


@pytest.mark.parametrize("delta_range", [(1e-4, 1e-2), (1e-1, 3.0)])
@pytest.mark.parametrize("structured", [True, False])
def test_zoh_small_and_large_steps(delta_range, structured):
    """Small steps take the series branch of the gain, large ones the exponential one."""
    _force("summaries+forward", 192)
    inp = synth.make_scan_inputs(1, 64, 1000, io_dtype="f32", seed=6, delta_range=delta_range)
    if not structured:
        inp.A = random_A(64, 6)
    out, last = _run_ex(inp, h0=_h0(inp, 2), zoh=True)
    y_ref, h_ref = oracle.scan_inputs(inp, h0=_h0(inp, 2).astype(np.float64), zoh=True)
    check_close(to_f64(out), y_ref, "f32", "y")
    check_close(to_f64(last), h_ref, "f32", "last_state")


@pytest.mark.parametrize("schedule", SCHEDULES)
def test_zoh_zero_A(schedule):
    """A = 0 exactly: the gain is its limit delta (all-zero A takes the structured path,
    a few zero states among others the general one)."""
    _force(schedule)
    for A in (np.zeros((48, 16), np.float32), random_A(48, 8, zero_states=(0, 5, 15))):
        inp = synth.make_scan_inputs(1, 48, 300, io_dtype="f32", seed=7)
        inp.A = A
        out, last = _run_ex(inp, zoh=True)
        y_ref, h_ref = oracle.scan_inputs(inp, zoh=True)
        check_close(to_f64(out), y_ref, "f32", "y")
        check_close(to_f64(last), h_ref, "f32", "last_state")


def test_zoh_full_size_every_row():
    """The 8 x 5120 x 4096 workload with the zero-order hold, every element against the oracle."""
    inp = synth.workload_inputs("scan_bf16_8x5120x4096")
    out, last = _run_ex(inp, zoh=True)
    check_scan_every_row(inp, out, last, zoh=True)


@pytest.mark.parametrize("path", ["stream", "bulk_tile", "per_row"])
@pytest.mark.parametrize("io", ["bf16", "f32"])
def test_zoh_decode(path, io):
    import selective_state_space_46_b200 as m
    m.mssm_set_option(m.MSSM_OPT_DECODE_PATH, m.DECODE_PATHS[path])
    inp = synth.make_decode_inputs(5, 256, io_dtype=io, seed=8, dt_bias=True)
    inp.A = random_A(256, 8, zero_states=(3,))
    st = to_dev(inp.state)
    dv = {k: to_dev(getattr(inp, k)) for k in ("x", "dt", "A", "B", "C", "D", "z", "dt_bias")}
    out = m.state_update(st, dv["x"], dv["dt"], dv["A"], dv["B"], dv["C"], dv["D"], dv["z"],
                         dt_bias=dv["dt_bias"], softplus=True, zoh=True)
    torch.cuda.synchronize()
    m.mssm_get_error()
    st_ref, y_ref = oracle.state_update_inputs(inp, zoh=True)
    check_close(to_f64(out), y_ref, io, "y")
    check_close(to_f64(st), st_ref, "f32", "state")


def test_zoh_decode_chain_reproduces_scan():
    import selective_state_space_46_b200 as m
    Bt, D, T = 2, 64, 20
    inp = synth.make_scan_inputs(Bt, D, T, io_dtype="f32", seed=13)
    dev = dev_scan_inputs(inp)
    y_scan, h_scan = _run_ex(inp, zoh=True)
    state = torch.zeros(Bt, D, 16, device="cuda")
    ys = []
    for t in range(T):
        ys.append(m.state_update(state, dev["u"][..., t], dev["delta"][..., t], dev["A"], dev["B"][..., t],
                                 dev["C"][..., t], dev["D"], dev["z"][..., t], dt_bias=dev["delta_bias"],
                                 softplus=True, zoh=True))
    torch.cuda.synchronize()
    y_dec = torch.stack(ys, dim=-1)
    assert float(((y_dec - y_scan).abs() / (1 + y_scan.abs())).max()) <= 1e-5
    assert float(((state - h_scan).abs() / (1 + h_scan.abs())).max()) <= 1e-5


def test_ext_validation():
    import selective_state_space_46_b200 as m
    inp = synth.make_scan_inputs(1, 8, 16, io_dtype="f32", seed=1)
    dev = dev_scan_inputs(inp)
    out = torch.empty_like(dev["u"])
    last = torch.empty(1, 8, 16, device="cuda")
    args = (dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"], dev["D"], dev["z"], dev["delta_bias"], 1, out, last)
    with pytest.raises(m.MssmError, match="discretization"):
        m.mssm_selective_scan_fwd_ex(*args, discretization=7)
    with pytest.raises(m.MssmError, match="h0"):
        m.mssm_selective_scan_fwd_ex(*args, h0=torch.zeros(1, 8, 15, device="cuda"))
    with pytest.raises(m.MssmError, match="alias"):
        m.mssm_selective_scan_fwd_ex(*args, h0=last)
