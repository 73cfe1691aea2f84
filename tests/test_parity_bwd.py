"""GPU parity of the backward scan (mssm_selective_scan_bwd) against the fp64 oracle's
reverse-mode chain rule, which is itself pinned by finite differences."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import TOL, check_close, dev_scan_inputs, to_dev, to_f64

pytestmark = pytest.mark.gpu


def random_A(dim, seed):
    rng = np.random.default_rng(seed)
    return (-np.exp(rng.uniform(-1.0, 1.5, size=(dim, 16)))).astype(np.float32)


def run_bwd(inp, seed=0):
    import selective_state_space_46_b200 as m
    dev = dev_scan_inputs(inp)
    rng = np.random.default_rng(seed + 1000)
    dout = rng.standard_normal(inp.u.shape).astype(np.float32)
    if inp.io_dtype == "bf16":
        dout = synth.f32_to_bf16_bits(dout)
    g = m.selective_scan_bwd(dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"], dev["D"], dev["z"],
                             dev["delta_bias"], inp.softplus, to_dev(dout))
    torch.cuda.synchronize()
    m.mssm_get_error()
    ref = oracle.scan_bwd(inp.f64("u"), inp.f64("delta"), inp.f64("A"), inp.f64("B"), inp.f64("C"),
                          inp.f64("D"), inp.f64("z"), inp.f64("delta_bias"), inp.softplus,
                          synth.to_f64(dout, inp.io_dtype))
    return g, ref


def compare(g, ref, io):
    for k, v in ref.items():
        if v is None:
            assert g[k] is None
            continue
        got = to_f64(g[k])
        if k in ("dA", "dD", "ddelta_bias", "dB", "dC"):
            # sums over many steps (and channels): held to the tolerance relative to their scale
            scale = max(1.0, float(np.abs(v).max()))
            err = float(np.abs(got - v).max()) / scale
            assert err <= TOL[io], f"{k}: worst error {err:.3e} of scale {scale:.3g}"
        else:
            check_close(got, v, io, k)


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("structured", [True, False])
@pytest.mark.parametrize("L", [5, 64, 65, 300])
def test_bwd_matches_oracle(cuda_device, io, structured, L):
    inp = synth.make_scan_inputs(2, 70, L, io_dtype=io, seed=L)
    if not structured:
        inp.A = random_A(70, L)
    g, ref = run_bwd(inp, seed=L)
    compare(g, ref, io)


@pytest.mark.parametrize("with_z,with_D,with_bias,softplus", [(False, False, False, True),
                                                              (True, True, True, False)])
def test_bwd_optional_inputs(cuda_device, with_z, with_D, with_bias, softplus):
    inp = synth.make_scan_inputs(1, 40, 200, io_dtype="f32", seed=3, with_z=with_z, with_D=with_D,
                                 with_bias=with_bias, softplus=softplus)
    if not softplus:  # keep the step positive, as softplus would
        inp.delta = (np.abs(synth.to_f64(inp.delta, "f32")) * 0.05).astype(np.float32)
        if inp.delta_bias is not None:
            inp.delta_bias = np.full(inp.dim, 0.02, np.float32)
    g, ref = run_bwd(inp, seed=4)
    compare(g, ref, "f32")


@pytest.mark.parametrize("Bt,D,L", [(1, 40, 1000), (2, 33, 1096), (1, 40, 8192)])
def test_bwd_aligned_rows_ragged_chunks(cuda_device, Bt, D, L):
    """bf16 rows that start 16-byte aligned (the vector loads and the 16-byte B/C staging)
    with a last chunk of 40 or 8 steps, and 128 chunks folded both ways."""
    inp = synth.make_scan_inputs(Bt, D, L, io_dtype="bf16", seed=L + D)
    g, ref = run_bwd(inp, seed=L)
    compare(g, ref, "bf16")


@pytest.mark.parametrize("Bt,D,L", [(32, 1024, 300), (16, 2050, 97)])
def test_bwd_short_chunks_many_tiles(cuda_device, Bt, D, L):
    """From 1024 row tiles of 32 channels on, the backward runs in 32-step chunks: ragged
    lengths and a partial last tile per batch."""
    inp = synth.make_scan_inputs(Bt, D, L, io_dtype="bf16", seed=Bt + L)
    g, ref = run_bwd(inp, seed=L)
    compare(g, ref, "bf16")


def test_bwd_default_workload_shape(cuda_device):
    """2 x 512 x 2048 (a quarter of the default prefill's channels), bf16."""
    inp = synth.make_scan_inputs(2, 512, 2048, io_dtype="bf16", seed=9)
    g, ref = run_bwd(inp, seed=9)
    compare(g, ref, "bf16")


def test_bwd_validation(cuda_device):
    import selective_state_space_46_b200 as m
    inp = synth.make_scan_inputs(1, 8, 16, io_dtype="f32", seed=1)
    dev = dev_scan_inputs(inp)
    dout = torch.ones_like(dev["u"])
    with pytest.raises(m.MssmError, match="dz"):
        g = m.selective_scan_bwd(dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"], dev["D"], dev["z"],
                                 dev["delta_bias"], True, dout)
        m.mssm_selective_scan_bwd(dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"], dev["D"], dev["z"],
                                  dev["delta_bias"], True, dout, g["du"], g["ddelta"], g["dA"], g["dB"],
                                  g["dC"], g["dD"], None, g["ddelta_bias"])
