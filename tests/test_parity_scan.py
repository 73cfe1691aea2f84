"""GPU parity of mssm_selective_scan_fwd against the fp64 oracle.

Every problem, the full-size prefill shapes included, is compared element by
element; the full-size shapes run whole on the GPU in the launch configuration
the benchmark uses, and the oracle checks them block by block of channels.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import check_close, check_scan_every_row, dev_scan_inputs, run_scan, to_dev, to_f64

pytestmark = pytest.mark.gpu


def _reset_options():
    import selective_state_space_46_b200 as m
    m.mssm_set_option(m.MSSM_OPT_FORCE_GENERAL_A, 0)
    m.mssm_set_option(m.MSSM_OPT_CHUNK_LEN, 0)
    m.mssm_set_option(m.MSSM_OPT_SCHEDULE, 0)
    m.mssm_set_option(m.MSSM_OPT_ROWS_PER_CTA, 0)


@pytest.fixture(autouse=True)
def _defaults(cuda_device):
    _reset_options()
    yield
    _reset_options()


def compare_full(inp, **kw):
    out, last = run_scan(inp, **kw)
    y_ref, h_ref = oracle.scan_inputs(inp)
    check_close(to_f64(out), y_ref, inp.io_dtype, "y")
    check_close(to_f64(last), h_ref, inp.io_dtype, "last_state")


SPLIT_SCHEDULES = ["summaries+forward", "chained", "fused"]


def random_A(dim, seed):
    rng = np.random.default_rng(seed)
    return (-np.exp(rng.uniform(-1.0, 1.5, size=(dim, 16)))).astype(np.float32)


# ---------------------------------------------------------------------------
# the named workloads
# ---------------------------------------------------------------------------

def test_workload_f32_1x64x256():
    compare_full(synth.workload_inputs("scan_f32_1x64x256"))


def test_workload_bf16_2x1536x2048():
    compare_full(synth.workload_inputs("scan_bf16_2x1536x2048"))


def test_workload_bf16_2x1536x2048_general_A_path():
    import selective_state_space_46_b200 as m
    m.mssm_set_option(m.MSSM_OPT_FORCE_GENERAL_A, 1)
    compare_full(synth.workload_inputs("scan_bf16_2x1536x2048"))


@pytest.mark.parametrize("schedule", ["forward"] + SPLIT_SCHEDULES)
def test_workload_bf16_2x1536x2048_each_schedule(schedule):
    import selective_state_space_46_b200 as m
    m.mssm_set_option(m.MSSM_OPT_SCHEDULE, m.SCHEDULES[schedule])
    compare_full(synth.workload_inputs("scan_bf16_2x1536x2048"))
    m.mssm_get_error()


@pytest.mark.slow
def test_workload_bf16_8x5120x4096_every_row():
    """The Mamba-2.8B-shaped prefill in the benchmark's launch configuration, every element of y
    and of the final state against the oracle."""
    inp = synth.workload_inputs("scan_bf16_8x5120x4096")
    out, last = run_scan(inp)
    check_scan_every_row(inp, out, last)


@pytest.mark.slow
def test_workload_bf16_1x2048x131072_every_row():
    """The long-context workload (the benchmark's default), every element against the oracle."""
    inp = synth.workload_inputs("scan_bf16_1x2048x131072")
    out, last = run_scan(inp)
    check_scan_every_row(inp, out, last)


# ---------------------------------------------------------------------------
# shapes: ragged lengths and channel counts, options on and off
# ---------------------------------------------------------------------------

SHAPES = [
    (1, 1, 1), (1, 3, 2), (2, 5, 7), (1, 64, 15), (1, 65, 16), (2, 63, 17), (1, 1, 31),
    (1, 130, 33), (2, 64, 64), (1, 7, 100), (3, 129, 257), (1, 64, 1000), (2, 200, 777),
]


@pytest.mark.parametrize("Bt,D,L", SHAPES)
@pytest.mark.parametrize("io", ["bf16", "f32"])
def test_shapes(Bt, D, L, io):
    inp = synth.make_scan_inputs(Bt, D, L, io_dtype=io, seed=L * 7 + D)
    compare_full(inp)


@pytest.mark.parametrize("with_z,with_D,with_bias,softplus", [
    (False, False, False, True), (True, False, True, False), (False, True, False, False),
    (True, True, True, True),
])
@pytest.mark.parametrize("io", ["bf16", "f32"])
def test_optional_inputs(with_z, with_D, with_bias, softplus, io):
    inp = synth.make_scan_inputs(2, 70, 300, io_dtype=io, seed=3, with_z=with_z, with_D=with_D,
                                 with_bias=with_bias, softplus=softplus)
    if not softplus:
        # keep the step positive and small without softplus: delta = |raw| * 0.05
        raw = synth.bf16_bits_to_f32(inp.delta) if io == "bf16" else inp.delta
        pos = np.abs(raw) * 0.05
        inp.delta = synth.f32_to_bf16_bits(pos) if io == "bf16" else pos.astype(np.float32)
        inp.delta_bias = None
    compare_full(inp)


@pytest.mark.parametrize("io", ["bf16", "f32"])
def test_general_A_values(io):
    inp = synth.make_scan_inputs(2, 96, 500, io_dtype=io, seed=11)
    inp.A = random_A(96, 5)
    compare_full(inp)


@pytest.mark.parametrize("io", ["bf16", "f32"])
@pytest.mark.parametrize("chunk", [0, 128])
def test_general_A_extreme_decay(io, chunk):
    """General A whose per-step decay exponents reach far below 2^-125 (steps up to about 5
    times A down to -60): the exponentials computed on the FP32 pipe clamp there, the SFU ones
    flush to zero; both must agree with the oracle as a decay factor of zero would,
    whole-sequence and across chunk summaries.  A stays below -0.3, so no state keeps a long
    memory: with steps this large, a decay factor within 1% of 1 held for hundreds of steps
    compounds the SFU exponential's own error past the fp32 tolerance."""
    import selective_state_space_46_b200 as m
    Bt, D, L = 2, 70, 600
    inp = synth.make_scan_inputs(Bt, D, L, io_dtype=io, seed=41)
    rng = np.random.default_rng(41)
    A = -np.exp(rng.uniform(np.log(0.3), np.log(60.0), size=(D, 16)))
    inp.A = A.astype(np.float32)
    inp.delta_bias = rng.uniform(-1.0, 4.0, size=D).astype(np.float32)
    if chunk:
        m.mssm_set_option(m.MSSM_OPT_CHUNK_LEN, chunk)
    compare_full(inp)


@pytest.mark.parametrize("n", [0, 5])
def test_general_A_nan_propagates(n):
    """A NaN in A reaches the outputs of its channel whichever unit computes that state's decay
    (state 0 is in the pair computed on the FP32 pipe, state 5 on the SFU); other channels stay
    finite."""
    inp = synth.make_scan_inputs(2, 40, 300, io_dtype="f32", seed=3)
    A = random_A(40, 3)
    A[7, n] = np.nan
    inp.A = A
    out, last = run_scan(inp)
    y, h = to_f64(out), to_f64(last)
    assert np.isnan(y[:, 7, :]).all() and np.isnan(h[:, 7, n]).all()
    others = np.ones(40, bool)
    others[7] = False
    assert np.isfinite(y[:, others, :]).all() and np.isfinite(h[:, others, :]).all()


# ---------------------------------------------------------------------------
# the length split and its carry
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("chunk", [64, 128, 192, 320])
@pytest.mark.parametrize("structured", [True, False])
@pytest.mark.parametrize("io", ["bf16", "f32"])
@pytest.mark.parametrize("schedule", SPLIT_SCHEDULES)
def test_chunked_carry(chunk, structured, io, schedule):
    import selective_state_space_46_b200 as m
    m.mssm_set_option(m.MSSM_OPT_SCHEDULE, m.SCHEDULES[schedule])
    m.mssm_set_option(m.MSSM_OPT_CHUNK_LEN, chunk)
    assert m.mssm_scan_plan(2, 80, 1000)["schedule"] == schedule
    inp = synth.make_scan_inputs(2, 80, 1000, io_dtype=io, seed=chunk, delta_range=(1e-4, 1e-2))
    if not structured:
        inp.A = random_A(80, chunk)
    compare_full(inp)


@pytest.mark.parametrize("Bt,D,L", [(1, 1, 1), (2, 5, 7), (1, 64, 15), (1, 65, 100), (2, 130, 257),
                                    (3, 129, 1000), (1, 200, 777)])
@pytest.mark.parametrize("schedule,chunk", [("forward", 0), ("summaries+forward", 64),
                                            ("summaries+forward", 192)])
@pytest.mark.parametrize("io", ["bf16", "f32"])
def test_64_row_tiles(Bt, D, L, schedule, chunk, io):
    """Plans forced to 64-channel row tiles (two warps per CTA)."""
    import selective_state_space_46_b200 as m
    m.mssm_set_option(m.MSSM_OPT_ROWS_PER_CTA, 64)
    m.mssm_set_option(m.MSSM_OPT_SCHEDULE, m.SCHEDULES[schedule])
    if chunk:
        m.mssm_set_option(m.MSSM_OPT_CHUNK_LEN, chunk)
    plan = m.mssm_scan_plan(Bt, D, L)
    assert plan["rows_per_cta"] == 64
    inp = synth.make_scan_inputs(Bt, D, L, io_dtype=io, seed=D * 3 + L)
    compare_full(inp)


@pytest.mark.parametrize("with_z,with_D,with_bias,softplus", [
    (False, False, False, False), (True, True, False, True), (False, True, True, True)])
@pytest.mark.parametrize("structured", [True, False])
def test_64_row_tiles_options(with_z, with_D, with_bias, softplus, structured):
    import selective_state_space_46_b200 as m
    m.mssm_set_option(m.MSSM_OPT_ROWS_PER_CTA, 64)
    m.mssm_set_option(m.MSSM_OPT_CHUNK_LEN, 128)
    inp = synth.make_scan_inputs(2, 100, 600, io_dtype="bf16", seed=11, with_z=with_z, with_D=with_D,
                                 with_bias=with_bias, softplus=softplus)
    if not softplus:  # a positive, small step without softplus (a negative one makes the states grow)
        pos = np.abs(synth.bf16_bits_to_f32(inp.delta)) * 0.05
        inp.delta = synth.f32_to_bf16_bits(pos)
        inp.delta_bias = None
    if not structured:
        inp.A = random_A(100, 5)
    compare_full(inp)


def test_64_row_tiles_default_workload():
    import selective_state_space_46_b200 as m
    m.mssm_set_option(m.MSSM_OPT_ROWS_PER_CTA, 64)
    inp = synth.workload_inputs("scan_bf16_2x1536x2048", seed=0)
    compare_full(inp)


def test_chunked_equals_unchunked_closely():
    # the split changes only the association order of fp32 sums
    import selective_state_space_46_b200 as m
    inp = synth.make_scan_inputs(1, 64, 2048, io_dtype="f32", seed=21, delta_range=(1e-4, 1e-2))
    dev = dev_scan_inputs(inp)
    m.mssm_set_option(m.MSSM_OPT_CHUNK_LEN, 4096)
    y1, h1 = run_scan(inp, dev)
    m.mssm_set_option(m.MSSM_OPT_CHUNK_LEN, 128)
    y2, h2 = run_scan(inp, dev)
    scale = 1 + y1.abs()
    assert float(((y1 - y2).abs() / scale).max()) < 1e-5
    assert float(((h1 - h2).abs() / (1 + h1.abs())).max()) < 1e-5


def test_workspace_reuse_across_tile_counts():
    """Split calls with different row-tile counts share the library's carry
    workspace: a call with few tiles writes chunk sums where a later call with
    more tiles keeps arrival counters, unless the counters have a region of
    their own.  Sequence: size the workspace, split 1 tile, split 96 tiles."""
    import selective_state_space_46_b200 as m
    m.mssm_set_option(m.MSSM_OPT_CHUNK_LEN, 64)
    big = synth.make_scan_inputs(2, 1536, 4096, io_dtype="bf16", seed=30)
    run_scan(big)
    for Bt, D, L, seed in [(1, 32, 4096, 31), (2, 1536, 2048, 32)]:
        compare_full(synth.make_scan_inputs(Bt, D, L, io_dtype="bf16", seed=seed))


@pytest.mark.parametrize("io,chunk,structured,L", [
    ("bf16", 0, True, 1000), ("bf16", 64, True, 777), ("f32", 128, False, 640), ("bf16", 256, False, 1024),
])
def test_chained_schedule(io, chunk, structured, L):
    """Many row tiles: the persistent kernel hands each tile's state from chunk to chunk."""
    import selective_state_space_46_b200 as m
    m.mssm_set_option(m.MSSM_OPT_CHUNK_LEN, chunk)
    Bt, D = 2, 9600                      # 600 tiles of 32 rows
    plan = m.mssm_scan_plan(Bt, D, L)
    assert plan["schedule"] == "chained", plan
    inp = synth.make_scan_inputs(Bt, D, L, io_dtype=io, seed=L + chunk, delta_range=(1e-4, 1e-2))
    if not structured:
        inp.A = random_A(D, 3)
    compare_full(inp)
    m.mssm_get_error()                   # no bounded wait gave up


def test_long_slow_decay_many_chunks():
    inp = synth.make_scan_inputs(1, 64, 16384, io_dtype="bf16", seed=5, delta_range=(1e-4, 1e-2))
    compare_full(inp)


@pytest.mark.parametrize("schedule", ["summaries+forward", "chained"])
def test_chunk_count_past_the_grid_limit(schedule):
    """4.2 M steps (8 channels) forced into 64-step chunks would need 65 553 chunks, past the 65 535 a grid
    dimension holds: the plan doubles the chunk length instead; every row against the oracle."""
    import selective_state_space_46_b200 as m
    Bt, D, L = 1, 8, (1 << 22) + 777
    m.mssm_set_option(m.MSSM_OPT_CHUNK_LEN, 64)
    m.mssm_set_option(m.MSSM_OPT_SCHEDULE, m.SCHEDULES[schedule])
    plan = m.mssm_scan_plan(Bt, D, L)
    assert plan["n_chunks"] <= 65535 and plan["chunk_len"] == 128 and plan["schedule"] == schedule, plan
    inp = synth.make_scan_inputs(Bt, D, L, io_dtype="bf16", seed=13, delta_range=(1e-4, 1e-2))
    out, last = run_scan(inp)
    m.mssm_get_error()
    check_scan_every_row(inp, out, last)


# ---------------------------------------------------------------------------
# layouts: strided and unaligned rows take the scalar path
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("io", ["bf16", "f32"])
def test_strided_unaligned_rows(io):
    Bt, D, L = 2, 70, 203
    inp = synth.make_scan_inputs(Bt, D, L, io_dtype=io, seed=9)
    dev = dev_scan_inputs(inp)

    def padded(t, pad):
        big = torch.zeros(*t.shape[:-1], t.shape[-1] + pad, dtype=t.dtype, device=t.device)
        big[..., 1:1 + t.shape[-1]] = t
        return big[..., 1:1 + t.shape[-1]]

    for k in ("u", "delta", "z", "B", "C"):
        dev[k] = padded(dev[k], 5)
        assert not dev[k].is_contiguous()
    out_big = torch.zeros(Bt, D, L + 3, dtype=dev["u"].dtype, device="cuda")
    out = out_big[..., :L]
    last = torch.empty(Bt, D, 16, device="cuda")
    import selective_state_space_46_b200 as m
    m.mssm_selective_scan_fwd(dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"], dev["D"], dev["z"],
                              dev["delta_bias"], True, out, last)
    torch.cuda.synchronize()
    y_ref, h_ref = oracle.scan_inputs(inp)
    check_close(to_f64(out), y_ref, io, "y")
    check_close(to_f64(last), h_ref, io, "last_state")
    assert float(out_big[..., L:].abs().max()) == 0.0   # nothing written past the view


# ---------------------------------------------------------------------------
# edge cases and API behaviour
# ---------------------------------------------------------------------------

def test_empty_and_zero_length():
    import selective_state_space_46_b200 as m
    inp = synth.make_scan_inputs(2, 9, 0, io_dtype="bf16", seed=1)
    dev = dev_scan_inputs(inp)
    last = torch.full((2, 9, 16), 7.0, device="cuda")
    out = torch.empty(2, 9, 0, dtype=torch.bfloat16, device="cuda")
    m.mssm_selective_scan_fwd(dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"], dev["D"], dev["z"],
                              dev["delta_bias"], True, out, last)
    torch.cuda.synchronize()
    assert float(last.abs().max()) == 0.0
    inp0 = synth.make_scan_inputs(0, 9, 10, io_dtype="bf16", seed=1)
    y, h = run_scan(inp0)
    assert y.numel() == 0 and h.numel() == 0


def test_output_only_no_last_state_and_determinism():
    inp = synth.make_scan_inputs(2, 100, 900, io_dtype="bf16", seed=4)
    dev = dev_scan_inputs(inp)
    y1, _ = run_scan(inp, dev, return_last_state=False)
    y2, _ = run_scan(inp, dev, return_last_state=False)
    assert torch.equal(y1, y2)
    y_ref, _ = oracle.scan_inputs(inp)
    check_close(to_f64(y1), y_ref, "bf16")


def test_side_stream():
    import selective_state_space_46_b200 as m
    inp = synth.make_scan_inputs(1, 64, 512, io_dtype="bf16", seed=8)
    dev = dev_scan_inputs(inp)
    s = torch.cuda.Stream()
    out = torch.empty_like(dev["u"])
    last = torch.empty(1, 64, 16, device="cuda")
    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        m.mssm_selective_scan_fwd(dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"], dev["D"],
                                  dev["z"], dev["delta_bias"], True, out, last, stream=s)
    m.mssm_get_error(s)
    y_ref, h_ref = oracle.scan_inputs(inp)
    check_close(to_f64(out), y_ref, "bf16")
    check_close(to_f64(last), h_ref, "bf16")


def test_invalid_arguments_raise():
    import selective_state_space_46_b200 as m
    inp = synth.make_scan_inputs(1, 8, 16, io_dtype="bf16", seed=2)
    dev = dev_scan_inputs(inp)
    with pytest.raises(m.MssmError) as e:
        m.selective_scan_fwd(dev["u"], dev["delta"].float(), dev["A"], dev["B"], dev["C"])
    assert e.value.status == m.MSSM_ERR_INVALID_ARG
    with pytest.raises(m.MssmError) as e:
        m.selective_scan_fwd(dev["u"], dev["delta"], dev["A"][:, :8].contiguous(), dev["B"][:, :8],
                             dev["C"][:, :8])
    assert e.value.status == m.MSSM_ERR_UNSUPPORTED
