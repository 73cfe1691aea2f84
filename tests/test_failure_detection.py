"""Failure detection on the GPU without a fault: a bounded device-side wait is made to
run out and the host reads the error status; the context stays usable.

The chained (and split-chunk) scan schedules hand each chunk's end state to the next
chunk through a flag that the next chunk waits for with an iteration limit (the fused
schedule's look-back waits the same way).  MSSM_OPT_TEST_HOOKS = 1 makes the kernels
publish no flags, so the waits give up (about half a second), the
kernel records bit 1 of its device error word and returns; mssm_get_error reports
MSSM_ERR_TIMEOUT and clears the word.  Nothing faults, traps or waits without bound."""
import pytest
import torch

import oracle
import synth
from gpu_util import check_close, dev_scan_inputs, to_f64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("schedule,L,chunk", [("chained", 128, 64), ("fused", 128, 64), ("split", 512, 256)])
def test_chained_wait_timeout_is_reported_and_recoverable(cuda_device, schedule, L, chunk):
    import selective_state_space_46_b200 as m
    inp = synth.make_scan_inputs(1, 32, L, io_dtype="f32", seed=3)
    dev = dev_scan_inputs(inp)
    m.mssm_set_option(m.MSSM_OPT_SCHEDULE, m.SCHEDULES[schedule])
    m.mssm_set_option(m.MSSM_OPT_CHUNK_LEN, chunk)  # two chunks: one bounded wait
    try:
        assert m.mssm_scan_plan(1, 32, L, io_dtype="f32")["schedule"] == schedule
        m.mssm_get_error()  # start from a clear error word
        m.mssm_set_option(m.MSSM_OPT_TEST_HOOKS, 1)
        m.selective_scan_fwd(dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"], dev["D"], dev["z"],
                             dev["delta_bias"], inp.softplus)
        with pytest.raises(m.MssmError) as err:
            m.mssm_get_error()
        assert err.value.status == m.MSSM_ERR_TIMEOUT
        m.mssm_get_error()  # the word was cleared by the read
        # the context is still usable and the normal schedule is exact again
        m.mssm_set_option(m.MSSM_OPT_TEST_HOOKS, 0)
        out, last = m.selective_scan_fwd(dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"], dev["D"],
                                         dev["z"], dev["delta_bias"], inp.softplus)
        torch.cuda.synchronize()
        m.mssm_get_error()
        y_ref, h_ref = oracle.scan_inputs(inp)
        check_close(to_f64(out), y_ref, "f32", "y")
        check_close(to_f64(last), h_ref, "f32", "last_state")
    finally:
        m.mssm_set_option(m.MSSM_OPT_TEST_HOOKS, 0)
        m.mssm_set_option(m.MSSM_OPT_SCHEDULE, 0)
        m.mssm_set_option(m.MSSM_OPT_CHUNK_LEN, 0)
