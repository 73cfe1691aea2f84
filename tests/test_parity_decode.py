"""GPU parity of the decode state update against the fp64 oracle, and the
recurrent-view identity: T decode steps reproduce the scan over T tokens."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import check_close, dev_scan_inputs, run_scan, to_dev, to_f64

pytestmark = pytest.mark.gpu


def dev_decode(inp):
    return dict(state=to_dev(inp.state), x=to_dev(inp.x), dt=to_dev(inp.dt), A=to_dev(inp.A),
                B=to_dev(inp.B), C=to_dev(inp.C), D=to_dev(inp.D), z=to_dev(inp.z),
                dt_bias=to_dev(inp.dt_bias))


PATHS = ["auto", "stream", "bulk_tile", "per_row"]


@pytest.fixture
def decode_path(request):
    """Force one state-update kernel for the test (MSSM_OPT_DECODE_PATH), restore automatic after."""
    import selective_state_space_46_b200 as m
    m.mssm_set_option(m.MSSM_OPT_DECODE_PATH, m.DECODE_PATHS.get(request.param, 0))
    yield request.param
    m.mssm_set_option(m.MSSM_OPT_DECODE_PATH, 0)


@pytest.mark.parametrize("decode_path", PATHS, indirect=True)
def test_decode_workload_one_step(cuda_device, decode_path):
    import selective_state_space_46_b200 as m
    inp = synth.workload_inputs("decode_bf16_256x5120")
    dv = dev_decode(inp)
    out = torch.empty_like(dv["x"])
    m.mssm_state_update(dv["state"], dv["x"], dv["dt"], dv["A"], dv["B"], dv["C"], dv["D"], dv["z"], out)
    torch.cuda.synchronize()
    st_ref, y_ref = oracle.state_update_inputs(inp)
    check_close(to_f64(out), y_ref, "bf16", "y")
    # the state is fp32 in and out: hold it to the fp32 bound
    check_close(to_f64(dv["state"]), st_ref, "f32", "state")


@pytest.mark.parametrize("decode_path", ["stream", "bulk_tile", "per_row"], indirect=True)
@pytest.mark.parametrize("Bt,D,io", [(3, 4999, "bf16"), (37, 5003, "bf16"), (131, 5003, "bf16"), (1, 1, "bf16"),
                                     (1, 255, "bf16"), (2, 128, "bf16"), (3, 5000, "bf16"), (131, 4104, "bf16"),
                                     (300, 8, "bf16"), (5, 1028, "f32"), (7, 130, "f32")])
def test_decode_ragged_tiles(cuda_device, decode_path, Bt, D, io):
    """Row counts that leave a partial last tile or channel block, one or several tiles per
    CTA, CTAs that go round the shared-memory ring more than once (131 x 4104: 22 batch
    groups of up to 6 batches; 131 x 5003: 2561 tiles of 256 rows), and shapes the streaming
    kernel cannot take (D not a multiple of 16 bytes), where the path falls back."""
    import selective_state_space_46_b200 as m
    inp = synth.make_decode_inputs(Bt, D, io_dtype=io, seed=Bt * 7 + D)
    dv = dev_decode(inp)
    out = torch.empty_like(dv["x"])
    m.mssm_state_update(dv["state"], dv["x"], dv["dt"], dv["A"], dv["B"], dv["C"], dv["D"], dv["z"], out)
    torch.cuda.synchronize()
    m.mssm_get_error()  # raises on a device-side timeout
    st_ref, y_ref = oracle.state_update_inputs(inp)
    check_close(to_f64(out), y_ref, io, "y")
    check_close(to_f64(dv["state"]), st_ref, "f32", "state")


@pytest.mark.parametrize("decode_path", ["stream", "bulk_tile", "per_row"], indirect=True)
def test_decode_64_distinct_steps(cuda_device, decode_path):
    import selective_state_space_46_b200 as m
    inp0 = synth.make_decode_inputs(16, 5120, seed=1, step_stream=0)
    state = to_dev(inp0.state)
    st_ref = inp0.state.astype(np.float64)
    for k in range(64):
        inp = synth.make_decode_inputs(16, 5120, seed=1, step_stream=k)
        dv = dev_decode(inp)
        out = torch.empty_like(dv["x"])
        m.mssm_state_update(state, dv["x"], dv["dt"], dv["A"], dv["B"], dv["C"], dv["D"], dv["z"], out)
        st_ref, y_ref = oracle.state_update_inputs(inp, state=st_ref)
        torch.cuda.synchronize()
        check_close(to_f64(out), y_ref, "bf16", f"y step {k}")
    check_close(to_f64(state), st_ref, "f32", "state after 64 steps")


@pytest.mark.parametrize("io", ["bf16", "f32"])
@pytest.mark.parametrize("with_z,with_D", [(True, True), (False, False)])
@pytest.mark.parametrize("dim", [77, 128])
def test_decode_variants(cuda_device, io, with_z, with_D, dim):
    """Optional gate, skip and bias on the automatic path (D = 128: streaming kernel; 77: not)."""
    import selective_state_space_46_b200 as m
    inp = synth.make_decode_inputs(3, dim, io_dtype=io, seed=4, with_z=with_z, with_D=with_D, dt_bias=True)
    dv = dev_decode(inp)
    out = m.state_update(dv["state"], dv["x"], dv["dt"], dv["A"], dv["B"], dv["C"], dv["D"], dv["z"],
                         dt_bias=dv["dt_bias"], softplus=True)
    torch.cuda.synchronize()
    st_ref, y_ref = oracle.state_update_inputs(inp)
    check_close(to_f64(out), y_ref, io, "y")
    check_close(to_f64(dv["state"]), st_ref, "f32", "state")


def test_decode_strided_state(cuda_device):
    import selective_state_space_46_b200 as m
    inp = synth.make_decode_inputs(2, 33, io_dtype="bf16", seed=6)
    dv = dev_decode(inp)
    big = torch.zeros(2, 33, 17, device="cuda")   # row stride 17 floats: not 16-byte aligned
    big[..., :16] = dv["state"]
    st = big[..., :16]
    out = torch.empty_like(dv["x"])
    m.mssm_state_update(st, dv["x"], dv["dt"], dv["A"], dv["B"], dv["C"], dv["D"], dv["z"], out)
    torch.cuda.synchronize()
    st_ref, y_ref = oracle.state_update_inputs(inp)
    check_close(to_f64(out), y_ref, "bf16", "y")
    check_close(to_f64(st), st_ref, "f32", "state")
    assert float(big[..., 16].abs().max()) == 0.0


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_decode_steps_reproduce_scan(cuda_device, io):
    """Recurrent view == scan: T decode steps from a zero state give the scan's y and last state."""
    import selective_state_space_46_b200 as m
    Bt, D, T = 2, 40, 24
    inp = synth.make_scan_inputs(Bt, D, T, io_dtype=io, seed=12)
    dev = dev_scan_inputs(inp)
    y_scan, h_scan = run_scan(inp, dev)
    state = torch.zeros(Bt, D, 16, device="cuda")
    ys = []
    for t in range(T):
        out = m.state_update(state, dev["u"][..., t], dev["delta"][..., t], dev["A"], dev["B"][..., t],
                             dev["C"][..., t], dev["D"], dev["z"][..., t], dt_bias=dev["delta_bias"],
                             softplus=True)
        ys.append(out)
    torch.cuda.synchronize()
    y_dec = torch.stack(ys, dim=-1)
    tol = 1e-5 if io == "f32" else 1e-2
    assert float(((y_dec.float() - y_scan.float()).abs() / (1 + y_scan.float().abs())).max()) <= tol
    assert float(((state - h_scan).abs() / (1 + h_scan.abs())).max()) <= 1e-5
    y_ref, h_ref = oracle.scan_inputs(inp)
    check_close(to_f64(y_dec), y_ref, io, "decode-chain y")
    check_close(to_f64(state), h_ref, "f32", "decode-chain state")


@pytest.mark.slow
@pytest.mark.parametrize("decode_path", ["auto"], indirect=True)
def test_decode_1000_successive_steps_downscaled(cuda_device, decode_path):
    """The decode workload is timed over 1000 successive in-place steps whose per-token inputs
    cycle through a ring of 8 draws.  The same 1000 steps on a copy with batch 4 (every channel
    and state of the full shape): the final state against the oracle's after the same 1000
    steps, and the outputs of the last ring's worth of steps."""
    import selective_state_space_46_b200 as m
    ring = [synth.workload_inputs("decode_bf16_256x5120", batch=4, step_stream=k) for k in range(8)]
    state = to_dev(ring[0].state)
    dring = [dev_decode(r) for r in ring]
    st_ref = ring[0].state.astype(np.float64)
    outs, refs = [], []
    for k in range(1000):
        r, dv = ring[k % 8], dring[k % 8]
        out = torch.empty_like(dv["x"])
        m.mssm_state_update(state, dv["x"], dv["dt"], dv["A"], dv["B"], dv["C"], dv["D"], dv["z"], out)
        st_ref, y_ref = oracle.state_update_inputs(r, state=st_ref)
        if k >= 992:
            outs.append(out)
            refs.append(y_ref)
    torch.cuda.synchronize()
    m.mssm_get_error()
    for k, (o, y_ref) in enumerate(zip(outs, refs)):
        check_close(to_f64(o), y_ref, "bf16", f"y step {992 + k}")
    check_close(to_f64(state), st_ref, "f32", "state after 1000 steps")
