"""GPU parity of the causal depthwise conv1d + SiLU (prefill and decode step) against the
fp64 oracle; the conv is the listed layer's grouped Conv1d with padding K - 1 truncated to
L, then SiLU ("Linear Attention vs Softmax Attention ...", section Implementation)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import check_close, dev_scan_inputs, to_dev, to_f64

pytestmark = pytest.mark.gpu


def conv_inputs(Bt, D, L, K, io, seed, with_bias=True):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((Bt, D, L)).astype(np.float32)
    if io == "bf16":
        x = synth.f32_to_bf16_bits(x)
    w = (rng.standard_normal((D, K)) / np.sqrt(K)).astype(np.float32)
    b = rng.standard_normal(D).astype(np.float32) * 0.5 if with_bias else None
    return x, w, b


def ref_conv(x, w, b, io, silu=True, cu=None):
    xf = synth.to_f64(x, io)
    if cu is None:
        return oracle.causal_conv1d(xf, w.astype(np.float64), None if b is None else b.astype(np.float64), silu)
    return oracle.causal_conv1d_varlen(xf, w.astype(np.float64), cu, None if b is None else b.astype(np.float64),
                                       silu)


@pytest.mark.parametrize("K", [1, 2, 3, 4])
@pytest.mark.parametrize("io", ["bf16", "f32"])
@pytest.mark.parametrize("silu,with_bias", [(True, True), (False, False)])
def test_conv_matches_oracle(cuda_device, K, io, silu, with_bias):
    import selective_state_space_46_b200 as m
    x, w, b = conv_inputs(2, 96, 1000, K, io, seed=K)
    out = m.causal_conv1d(to_dev(x), to_dev(w), to_dev(b), silu=silu)
    torch.cuda.synchronize()
    check_close(to_f64(out), ref_conv(x, w, b, io, silu), io, "conv out")


@pytest.mark.parametrize("L", [1, 3, 7, 255, 256, 257, 2049, 4100])
@pytest.mark.parametrize("io", ["bf16", "f32"])
def test_conv_ragged_lengths(cuda_device, L, io):
    import selective_state_space_46_b200 as m
    x, w, b = conv_inputs(3, 40, L, 4, io, seed=L)
    out = m.causal_conv1d(to_dev(x), to_dev(w), to_dev(b))
    torch.cuda.synchronize()
    check_close(to_f64(out), ref_conv(x, w, b, io), io, "conv out")


def test_conv_workload_size(cuda_device):
    import selective_state_space_46_b200 as m
    x, w, b = conv_inputs(2, 1536, 2048, 4, "bf16", seed=5)
    out = m.causal_conv1d(to_dev(x), to_dev(w), to_dev(b))
    torch.cuda.synchronize()
    check_close(to_f64(out), ref_conv(x, w, b, "bf16"), "bf16", "conv out")


def test_conv_large_workload_every_row(cuda_device):
    """8 x 5120 x 4096 in the benchmark's launch configuration, every element against the
    oracle (batch by batch, to bound host memory)."""
    import selective_state_space_46_b200 as m
    inp = synth.workload_inputs("conv_bf16_8x5120x4096", seed=0)
    out = m.causal_conv1d(to_dev(inp.x), to_dev(inp.weight), to_dev(inp.bias))
    torch.cuda.synchronize()
    for b in range(inp.batch):
        check_close(to_f64(out[b:b + 1]), ref_conv(inp.x[b:b + 1], inp.weight, inp.bias, "bf16"), "bf16",
                    f"conv batch {b}")


def test_conv_unaligned_rows(cuda_device):
    """Rows that do not start on 16-byte boundaries take the element path."""
    import selective_state_space_46_b200 as m
    x, w, b = conv_inputs(2, 24, 301, 4, "bf16", seed=6)
    xd = to_dev(x)
    big = torch.zeros(2, 24, 305, dtype=torch.bfloat16, device="cuda")
    big[..., 1:302] = xd
    xs = big[..., 1:302]
    out = m.causal_conv1d(xs, to_dev(w), to_dev(b))
    torch.cuda.synchronize()
    check_close(to_f64(out), ref_conv(x, w, b, "bf16"), "bf16", "conv out")


def test_conv_packed_sequences(cuda_device):
    import selective_state_space_46_b200 as m
    lengths = [5, 0, 1, 8, 9, 63, 64, 65, 130, 700, 3, 257]
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    T = int(cu[-1])
    x, w, b = conv_inputs(1, 70, T + 11, 4, "bf16", seed=7)
    out = torch.full((1, 70, T + 11), 7.0, dtype=torch.bfloat16, device="cuda")
    m.causal_conv1d(to_dev(x), to_dev(w), to_dev(b), cu_seqlens=torch.from_numpy(cu).cuda(), out=out)
    torch.cuda.synchronize()
    m.mssm_get_error()
    got = to_f64(out)
    check_close(got[..., :T], ref_conv(x[..., :T], w, b, "bf16", cu=cu)[..., :T], "bf16", "conv out")
    assert np.all(got[..., T:] == 7.0)  # steps outside every sequence are not written


@pytest.mark.parametrize("K", [2, 3, 4])
@pytest.mark.parametrize("io", ["bf16", "f32"])
def test_conv_update_chain_matches_prefill(cuda_device, K, io):
    import selective_state_space_46_b200 as m
    Bt, D, L = 3, 64, 12
    x, w, b = conv_inputs(Bt, D, L, K, io, seed=10 + K)
    xd = to_dev(x)
    dtype = torch.bfloat16 if io == "bf16" else torch.float32
    state = torch.zeros(Bt, D, K - 1, dtype=dtype, device="cuda")
    ref = ref_conv(x, w, b, io)
    st_ref = np.zeros((Bt, D, K - 1))
    for t in range(L):
        out = m.causal_conv1d_update(state, xd[..., t].contiguous(), to_dev(w), to_dev(b))
        torch.cuda.synchronize()
        st_ref, o_ref = oracle.causal_conv1d_update(st_ref, synth.to_f64(x[..., t], io), w.astype(np.float64),
                                                    b.astype(np.float64))
        check_close(to_f64(out), o_ref, io, f"update out t={t}")
        check_close(to_f64(out), ref[..., t], io, f"update vs prefill t={t}")
    # the window holds the last K - 1 inputs exactly (they are stored in their own dtype)
    assert np.array_equal(to_f64(state), synth.to_f64(x[..., L - K + 1:], io))


def test_conv_feeds_the_scan(cuda_device):
    """x -> conv + SiLU -> u -> scan, against the oracle's conv followed by its scan."""
    import selective_state_space_46_b200 as m
    inp = synth.make_scan_inputs(2, 64, 700, io_dtype="f32", seed=21)
    x, w, b = conv_inputs(2, 64, 700, 4, "f32", seed=21)
    dev = dev_scan_inputs(inp)
    u = m.causal_conv1d(to_dev(x), to_dev(w), to_dev(b))
    out, last = m.selective_scan_fwd(u, dev["delta"], dev["A"], dev["B"], dev["C"], dev["D"], dev["z"],
                                     dev["delta_bias"], True)
    torch.cuda.synchronize()
    u_ref = ref_conv(x, w, b, "f32")
    y_ref, h_ref = oracle.scan(u_ref, inp.f64("delta"), inp.f64("A"), inp.f64("B"), inp.f64("C"), inp.f64("D"),
                               inp.f64("z"), inp.f64("delta_bias"), True)
    check_close(to_f64(out), y_ref, "f32", "y")
    check_close(to_f64(last), h_ref, "f32", "last_state")
