"""Helpers for the GPU parity tests: move synth inputs to the device, run the
library through its C ABI, compare with the oracle under the stated tolerance.

Tolerance: |gpu - ref| <= tol * (1 + |ref|) elementwise, with tol = 1e-4 for
fp32 I/O and 2e-2 for bf16 I/O, on both y and the final state.
"""
import numpy as np
import torch

TOL = {"f32": 1e-4, "bf16": 2e-2}


def to_dev(a, io_dtype=None):
    if a is None:
        return None
    if a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def to_f64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def check_close(gpu, ref, io_dtype, what="y"):
    tol = TOL[io_dtype]
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    assert gpu.shape == ref.shape, (what, gpu.shape, ref.shape)
    assert np.isfinite(gpu).all(), f"{what}: non-finite values from the GPU"
    err = np.abs(gpu - ref) / (1.0 + np.abs(ref))
    worst = float(err.max()) if err.size else 0.0
    if worst > tol:
        idx = np.unravel_index(int(err.argmax()), err.shape)
        raise AssertionError(f"{what}: worst scaled error {worst:.3e} > {tol:g} at {idx}: "
                             f"gpu={gpu[idx]!r} ref={ref[idx]!r}")
    return worst


def dev_scan_inputs(inp):
    """Device tensors of a synth.ScanInputs problem."""
    return dict(u=to_dev(inp.u), delta=to_dev(inp.delta), A=to_dev(inp.A), B=to_dev(inp.B),
                C=to_dev(inp.C), D=to_dev(inp.D), z=to_dev(inp.z), delta_bias=to_dev(inp.delta_bias))


def run_scan(inp, dev=None, **kw):
    import selective_state_space_46_b200 as m
    dev = dev or dev_scan_inputs(inp)
    out, last = m.selective_scan_fwd(dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"], dev["D"],
                                     dev["z"], dev["delta_bias"], inp.softplus, **kw)
    torch.cuda.synchronize()
    return out, last


def check_scan_every_row(inp, out, last, zoh=False, h0=None, elems_per_block=1 << 23):
    """Compare a whole GPU scan output with the oracle on every row, element by element.

    The oracle runs on blocks of channels of one batch at a time (``oracle.scan_block``), so the
    host holds only one block's fp64 inputs and outputs: a full-size problem costs its oracle time
    (a few seconds on the host cores) and little memory.  Returns the worst scaled error of y and
    of the final state."""
    import oracle
    block = max(1, min(inp.dim, elems_per_block // max(1, inp.length)))
    worst_y = worst_h = 0.0
    for b in range(inp.batch):
        for d0 in range(0, inp.dim, block):
            d1 = min(inp.dim, d0 + block)
            hb = None if h0 is None else np.asarray(h0[b:b + 1, d0:d1], np.float64)
            y_ref, h_ref = oracle.scan_block(inp, b, d0, d1, h0=hb, zoh=zoh)
            worst_y = max(worst_y, check_close(to_f64(out[b:b + 1, d0:d1]), y_ref, inp.io_dtype,
                                               f"y (batch {b}, channels {d0}..{d1 - 1})"))
            if last is not None:
                worst_h = max(worst_h, check_close(to_f64(last[b:b + 1, d0:d1]), h_ref, inp.io_dtype,
                                                   f"last_state (batch {b}, channels {d0}..{d1 - 1})"))
    return worst_y, worst_h
