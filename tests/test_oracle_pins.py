"""Pins for the fp64 oracle: closed forms, limits, brute force and invariants.

Each test ties the oracle to something other than itself, so that a plausible
mistake in it (a dropped term, a wrong sign or index, a transposed operand,
an off-by-one in when the input enters the state) fails at least one of them.
``test_mutants_are_caught`` checks exactly that by compiling deliberately
wrong variants of the oracle and running the pins against them.

The method is the Mamba-1 selective scan as the pages define it:
"Linear Attention vs Softmax Attention: Can RWKV or Mamba Replace
Transformers?" (section Implementation: the sequential loop of the listed
SelectiveSSMLayer) and "State Space Models in Large Language Models ..."
(sections Discretization and Dynamic Parameterization).
"""
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
N = 16


def softplus_ref(x):
    # independent routine: log(exp(0) + exp(x))
    return np.logaddexp(0.0, x)


def sigmoid_ref(x):
    # independent formulation: 0.5 * (1 + tanh(x / 2))
    return 0.5 * (1.0 + np.tanh(0.5 * x))


def rand_problem(rng, Bt, D, L, *, structured=False, with_z=True, with_D=True,
                 with_bias=True):
    u = rng.standard_normal((Bt, D, L))
    delta = rng.standard_normal((Bt, D, L))
    if structured:
        A = -np.tile(np.arange(1, N + 1, dtype=np.float64), (D, 1))
    else:
        A = -np.exp(rng.uniform(-1.0, 1.5, size=(D, N)))
    B = rng.standard_normal((Bt, N, L))
    C = rng.standard_normal((Bt, N, L))
    Dv = rng.standard_normal(D) if with_D else None
    z = rng.standard_normal((Bt, D, L)) if with_z else None
    bias = rng.uniform(-4.0, -1.0, size=D) if with_bias else None
    return dict(u=u, delta=delta, A=A, B=B, C=C, D=Dv, z=z, delta_bias=bias)


def eff_delta(p, softplus=True):
    d = p["delta"] + (0.0 if p["delta_bias"] is None else p["delta_bias"][None, :, None])
    return softplus_ref(d) if softplus else d


def gate(y, z):
    return y if z is None else y * z * sigmoid_ref(z)


# ---------------------------------------------------------------------------
# 1. A = 0: A_bar = 1, the state is a running sum of dt * B * u
# ---------------------------------------------------------------------------

def test_A_zero_is_prefix_sum():
    rng = np.random.default_rng(1)
    p = rand_problem(rng, 2, 3, 37)
    p["A"] = np.zeros_like(p["A"])
    y, last = oracle.scan(**p, softplus=True)
    dt = eff_delta(p)
    # h[b, d, n, t] = cumsum_t dt[b,d,t] * B[b,n,t] * u[b,d,t]
    incr = dt[:, :, None, :] * p["B"][:, None, :, :] * p["u"][:, :, None, :]
    h = np.cumsum(incr, axis=-1)
    y_ref = np.einsum("bdnt,bnt->bdt", h, p["C"]) + p["D"][None, :, None] * p["u"]
    y_ref = gate(y_ref, p["z"])
    np.testing.assert_allclose(y, y_ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(last, h[..., -1], rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------------------
# 2. LTI case: constant dt, B, C -> causal convolution with K_k = sum_n C_n a_n^k dt B_n
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("softplus,with_bias", [(True, False), (False, False), (True, True), (False, True)])
def test_lti_equals_convolution(softplus, with_bias):
    rng = np.random.default_rng(2)
    D, L = 3, 50
    u = rng.standard_normal((1, D, L))
    A = -np.exp(rng.uniform(-2.0, 1.0, size=(D, N)))
    raw = rng.uniform(-3.0, 0.5, size=D)
    bias = rng.uniform(0.5, 1.5, size=D) if with_bias else None
    if with_bias and not softplus:
        raw = raw * 0.01       # keep raw + bias positive: a stable step
    delta = np.repeat(raw[None, :, None], L, axis=2)
    b = rng.standard_normal(N)
    c = rng.standard_normal(N)
    B = np.repeat(b[None, :, None], L, axis=2)
    C = np.repeat(c[None, :, None], L, axis=2)
    Dv = rng.standard_normal(D)
    y, _ = oracle.scan(u, delta, A, B, C, Dv, None, bias, softplus)
    pre = raw + (bias if with_bias else 0.0)
    dt = softplus_ref(pre) if softplus else pre
    for d in range(D):
        k = np.arange(L)
        a = np.exp(dt[d] * A[d])                       # [N]
        K = (c[None, :] * a[None, :] ** k[:, None] * dt[d] * b[None, :]).sum(1)
        y_ref = np.convolve(u[0, d], K)[:L] + Dv[d] * u[0, d]
        np.testing.assert_allclose(y[0, d], y_ref, rtol=1e-11, atol=1e-12)


def test_lti_step_input_closed_form():
    # u = 1 for all t: y_t = sum_n C_n dt B_n (1 - a_n^(t+1)) / (1 - a_n) + D
    D, L = 2, 40
    A = -np.tile(np.arange(1, N + 1, dtype=np.float64), (D, 1))
    dt = np.array([0.05, 0.7])
    b = np.linspace(-1, 1, N)
    c = np.cos(np.arange(N))
    u = np.ones((1, D, L))
    delta = np.repeat(dt[None, :, None], L, axis=2)
    B = np.repeat(b[None, :, None], L, axis=2)
    C = np.repeat(c[None, :, None], L, axis=2)
    y, last = oracle.scan(u, delta, A, B, C, np.full(D, 0.5), None, None, False)
    for d in range(D):
        a = np.exp(dt[d] * A[d])
        t = np.arange(L)[:, None]
        y_ref = (c * dt[d] * b * (1 - a ** (t + 1)) / (1 - a)).sum(1) + 0.5
        np.testing.assert_allclose(y[0, d], y_ref, rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(last[0, d], dt[d] * b * (1 - a ** L) / (1 - a), rtol=1e-12)


# ---------------------------------------------------------------------------
# 3. tiny inputs: the fully unrolled sum
#    y_t = sum_{s<=t} sum_n C_{t,n} (prod_{s<r<=t} A_bar_{r,n}) dt_s B_{s,n} u_s + D u_t
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("seed,L,D", [(3, 1, 1), (4, 5, 2), (5, 12, 3)])
def test_tiny_unrolled_sum(seed, L, D):
    rng = np.random.default_rng(seed)
    p = rand_problem(rng, 2, D, L)
    y, last = oracle.scan(**p, softplus=True)
    dt = eff_delta(p)
    for b in range(2):
        for d in range(D):
            abar = [[math.exp(dt[b, d, r] * p["A"][d, n]) for n in range(N)] for r in range(L)]
            for t in range(L):
                acc = 0.0
                for s in range(t + 1):
                    for n in range(N):
                        prod = 1.0
                        for r in range(s + 1, t + 1):
                            prod *= abar[r][n]
                        acc += p["C"][b, n, t] * prod * dt[b, d, s] * p["B"][b, n, s] * p["u"][b, d, s]
                acc += p["D"][d] * p["u"][b, d, t]
                z = p["z"][b, d, t]
                acc *= z * sigmoid_ref(z)
                assert abs(y[b, d, t] - acc) <= 1e-12 * (1 + abs(acc))
            for n in range(N):
                hs = 0.0
                for s in range(L):
                    prod = 1.0
                    for r in range(s + 1, L):
                        prod *= abar[r][n]
                    hs += prod * dt[b, d, s] * p["B"][b, n, s] * p["u"][b, d, s]
                assert abs(last[b, d, n] - hs) <= 1e-12 * (1 + abs(hs))


# ---------------------------------------------------------------------------
# 4. limits of the step size
# ---------------------------------------------------------------------------

def test_delta_to_zero_preserves_state():
    rng = np.random.default_rng(6)
    p = rand_problem(rng, 1, 4, 30, with_z=False, with_bias=False)
    p["delta"] = np.full_like(p["delta"], -60.0)     # softplus(-60) ~ 8.8e-27
    h0 = rng.standard_normal((1, 4, N))
    y, last = oracle.scan(**p, softplus=True, h0=h0)
    np.testing.assert_allclose(last, h0, rtol=1e-20, atol=1e-22)
    y_ref = np.einsum("bdn,bnt->bdt", h0, p["C"]) + p["D"][None, :, None] * p["u"]
    np.testing.assert_allclose(y, y_ref, rtol=1e-20, atol=1e-20)
    # from a zero state nothing enters
    y0, last0 = oracle.scan(**p, softplus=True)
    assert np.abs(last0).max() < 1e-24
    np.testing.assert_allclose(y0, p["D"][None, :, None] * p["u"], rtol=0, atol=1e-24)


def test_large_delta_resets_state():
    rng = np.random.default_rng(7)
    p = rand_problem(rng, 2, 3, 25, with_bias=False)
    p["delta"] = np.full_like(p["delta"], 1.0e3)     # exp(-1e3 * |A|) == 0 in fp64
    y, last = oracle.scan(**p, softplus=False)
    h = 1.0e3 * p["B"][:, None, :, :] * p["u"][:, :, None, :]   # [b, d, n, t]
    y_ref = np.einsum("bdnt,bnt->bdt", h, p["C"]) + p["D"][None, :, None] * p["u"]
    np.testing.assert_allclose(y, gate(y_ref, p["z"]), rtol=1e-13, atol=1e-10)
    np.testing.assert_allclose(last, h[..., -1], rtol=1e-13)


# ---------------------------------------------------------------------------
# 5. recurrent view == scan;  split scan == scan  (associativity of the
#    composition of the per-step affine maps h -> A_bar h + B_bar x)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("softplus", [True, False])
def test_decode_steps_reproduce_scan(softplus):
    rng = np.random.default_rng(8)
    p = rand_problem(rng, 2, 5, 20)
    if not softplus:
        # without softplus the step is raw + bias itself: keep it positive (a stable decay)
        p["delta"] = np.abs(p["delta"]) * 0.05
        p["delta_bias"] = rng.uniform(0.01, 0.1, size=5)
    y, last = oracle.scan(**p, softplus=softplus)
    state = np.zeros((2, 5, N))
    for t in range(20):
        state, yt = oracle.state_update(state, p["u"][..., t], p["delta"][..., t], p["A"],
                                        p["B"][..., t], p["C"][..., t], p["D"], p["z"][..., t],
                                        p["delta_bias"], softplus)
        np.testing.assert_allclose(yt, y[..., t], rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(state, last, rtol=1e-13, atol=1e-14)


@pytest.mark.parametrize("io", ["bf16", "f32"])
def test_scan_rows_and_blocks_equal_the_whole_problem(io):
    """oracle.scan_rows and oracle.scan_block (which slice rows' inputs and their batch's B/C and
    widen them) give
    exactly the rows of the whole-problem oracle: a wrong batch of B/C, a wrong channel of A, D
    or bias, or a wrong widening would show here."""
    import synth
    inp = synth.make_scan_inputs(3, 9, 37, io_dtype=io, seed=41)
    y, last = oracle.scan_inputs(inp)
    rows = [(0, 0), (0, 8), (1, 3), (2, 0), (2, 5), (2, 8), (1, 3)]
    ys, hs = oracle.scan_rows(inp, rows)
    for i, (b, d) in enumerate(rows):
        np.testing.assert_array_equal(ys[i], y[b, d])
        np.testing.assert_array_equal(hs[i], last[b, d])
    # oracle.scan_block: channel blocks of one batch, the same way
    for b, d0, d1 in [(0, 0, 9), (1, 2, 7), (2, 8, 9)]:
        yb, hb = oracle.scan_block(inp, b, d0, d1)
        np.testing.assert_array_equal(yb[0], y[b, d0:d1])
        np.testing.assert_array_equal(hb[0], last[b, d0:d1])
    y_z, last_z = oracle.scan_inputs(inp, zoh=True)
    yb, hb = oracle.scan_block(inp, 2, 1, 6, zoh=True)
    np.testing.assert_array_equal(yb[0], y_z[2, 1:6])
    np.testing.assert_array_equal(hb[0], last_z[2, 1:6])


@pytest.mark.parametrize("split", [1, 7, 19])
def test_split_scan_equals_scan(split):
    rng = np.random.default_rng(9)
    p = rand_problem(rng, 1, 3, 20)
    y, last = oracle.scan(**p, softplus=True)
    first = {k: (v[..., :split] if k in ("u", "delta", "B", "C", "z") else v) for k, v in p.items()}
    second = {k: (v[..., split:] if k in ("u", "delta", "B", "C", "z") else v) for k, v in p.items()}
    y1, h1 = oracle.scan(**first, softplus=True)
    y2, h2 = oracle.scan(**second, softplus=True, h0=h1)
    np.testing.assert_allclose(np.concatenate([y1, y2], -1), y, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(h2, last, rtol=1e-13, atol=1e-14)


def test_affine_composition_is_associative():
    # the per-step map (a, b): h -> a*h + b composes as (a1,b1) then (a2,b2) = (a2 a1, a2 b1 + b2)
    rng = np.random.default_rng(10)

    def comp(p, q):
        return (q[0] * p[0], q[0] * p[1] + q[1])

    for _ in range(100):
        p, q, r = [(rng.uniform(0, 1), rng.standard_normal()) for _ in range(3)]
        lhs = comp(comp(p, q), r)
        rhs = comp(p, comp(q, r))
        assert abs(lhs[0] - rhs[0]) < 1e-15 and abs(lhs[1] - rhs[1]) < 1e-14
    # and the oracle's one-row state after L steps equals the composed map applied to 0
    D, L = 1, 9
    p = rand_problem(rng, 1, D, L, with_z=False, with_bias=False)
    _, last = oracle.scan(**p, softplus=False)
    for n in range(N):
        acc = (1.0, 0.0)
        for t in range(L):
            dt = p["delta"][0, 0, t]
            acc = comp(acc, (math.exp(dt * p["A"][0, n]), dt * p["B"][0, n, t] * p["u"][0, 0, t]))
        assert abs(acc[1] - last[0, 0, n]) <= 1e-12 * (1 + abs(acc[1]))


# ---------------------------------------------------------------------------
# 6. linearity in u (fixed dt, B, C, no gate), constant state size
# ---------------------------------------------------------------------------

def test_linear_in_u():
    rng = np.random.default_rng(11)
    p = rand_problem(rng, 2, 3, 33, with_z=False)
    u1, u2 = rng.standard_normal(p["u"].shape), rng.standard_normal(p["u"].shape)
    ys = []
    for u in (u1, u2, 2.5 * u1 - 0.75 * u2):
        q = dict(p)
        q["u"] = u
        ys.append(oracle.scan(**q, softplus=True))
    np.testing.assert_allclose(ys[2][0], 2.5 * ys[0][0] - 0.75 * ys[1][0], rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(ys[2][1], 2.5 * ys[0][1] - 0.75 * ys[1][1], rtol=1e-11, atol=1e-12)


def test_state_size_independent_of_length():
    rng = np.random.default_rng(12)
    for L in (1, 10, 100):
        p = rand_problem(rng, 2, 3, L)
        y, last = oracle.scan(**p, softplus=True)
        assert last.shape == (2, 3, N) and y.shape == (2, 3, L)


# ---------------------------------------------------------------------------
# 7. spot values of softplus and silu
# ---------------------------------------------------------------------------

def test_softplus_and_silu_spot_values():
    one = np.ones((1, 1, 1))
    A = -np.ones((1, N))
    B = np.full((1, N, 1), 0.5)
    C = np.full((1, N, 1), 2.0)
    u = 3.0 * one
    # softplus(0) = ln 2: y = sum_n C * (ln2 * B * u) = 16 * 2 * ln2 * 0.5 * 3
    y, last = oracle.scan(u, 0 * one, A, B, C, None, None, None, True)
    assert abs(y[0, 0, 0] - 48 * math.log(2)) < 1e-13
    assert np.allclose(last, 1.5 * math.log(2), rtol=1e-15)
    # silu(0) = 0
    y, _ = oracle.scan(u, 0 * one, A, B, C, None, 0 * one, None, True)
    assert y[0, 0, 0] == 0.0
    # silu(40) = 40 / (1 + e^-40) ~ 40
    y, _ = oracle.scan(u, 0 * one, A, B, C, None, 40 * one, None, True)
    assert abs(y[0, 0, 0] - 40 * 48 * math.log(2)) < 1e-9
    # bias enters before the softplus: raw -1 + bias 1 == raw 0
    y2, _ = oracle.scan(u, -one, A, B, C, None, None, np.ones(1), True)
    assert abs(y2[0, 0, 0] - 48 * math.log(2)) < 1e-13
    # softplus of a large argument does not overflow: softplus(800) = 800
    y3, _ = oracle.scan(u, 800 * one, A, B, C, None, None, None, True)
    assert abs(y3[0, 0, 0] - 16 * 2 * 800 * 0.5 * 3) < 1e-9


# ---------------------------------------------------------------------------
# 7b. zero-order hold ("Linear Attention vs Softmax Attention ...", Core Concepts, item 3;
#     "State Space Models in Large Language Models ...", Discretization)
# ---------------------------------------------------------------------------

def test_zoh_constant_input_is_exact():
    """With the step, A, B and u held constant, the zero-order-hold recurrence is exact:
    after t steps of size dt the state equals the continuous solution of h' = A h + B u
    from h(0) = 0 at time t dt, (exp(A t dt) - 1) / A * B u, whatever dt is."""
    rng = np.random.default_rng(21)
    D, L = 3, 40
    A = -np.exp(rng.uniform(-2.0, 1.0, size=(D, N)))
    for dt in (0.01, 0.37):
        u = np.full((1, D, L), 0.8)
        delta = np.full((1, D, L), dt)
        Bv = rng.standard_normal(N)
        B = np.repeat(Bv[None, :, None], L, axis=2)
        C = np.ones((1, N, L))
        y, last = oracle.scan(u, delta, A, B, C, None, None, None, softplus=False, zoh=True)
        tt = dt * np.arange(1, L + 1)
        h = np.expm1(A[:, :, None] * tt[None, None, :]) / A[:, :, None] * Bv[None, :, None] * 0.8
        np.testing.assert_allclose(y[0], h.sum(axis=1), rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(last[0], h[:, :, -1], rtol=1e-12, atol=1e-13)


def test_zoh_small_A_is_euler():
    """As A -> 0, (exp(dt A) - 1) / A -> dt: the two discretisations agree to O(dt^2 A)."""
    rng = np.random.default_rng(22)
    p = rand_problem(rng, 1, 4, 30)
    p["A"] = np.full_like(p["A"], -1e-9)
    y_e, h_e = oracle.scan(**p, softplus=True)
    y_z, h_z = oracle.scan(**p, softplus=True, zoh=True)
    np.testing.assert_allclose(y_z, y_e, rtol=1e-7, atol=1e-9)
    np.testing.assert_allclose(h_z, h_e, rtol=1e-7, atol=1e-9)


def test_zoh_decode_steps_reproduce_scan():
    rng = np.random.default_rng(23)
    p = rand_problem(rng, 2, 5, 16)
    y, last = oracle.scan(**p, softplus=True, zoh=True)
    state = np.zeros((2, 5, N))
    for t in range(16):
        state, yt = oracle.state_update(state, p["u"][..., t], p["delta"][..., t], p["A"],
                                        p["B"][..., t], p["C"][..., t], p["D"], p["z"][..., t],
                                        p["delta_bias"], True, zoh=True)
        np.testing.assert_allclose(yt, y[..., t], rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(state, last, rtol=1e-13, atol=1e-14)


# ---------------------------------------------------------------------------
# 7c. causal depthwise conv1d + SiLU feeding the scan ("Linear Attention vs Softmax
#     Attention ...", section Implementation: grouped Conv1d, padding K - 1, truncated)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("silu", [False, True])
def test_conv1d_matches_numpy_convolve(silu):
    rng = np.random.default_rng(31)
    Bt, D, L, K = 2, 5, 23, 4
    x = rng.standard_normal((Bt, D, L))
    w = rng.standard_normal((D, K))
    b = rng.standard_normal(D)
    out = oracle.causal_conv1d(x, w, b, silu=silu)
    # cross-correlation with left zero padding == the first L outputs of a full convolution
    # with the reversed filter
    ref = np.stack([np.stack([np.convolve(x[i, d], w[d][::-1])[:L] + b[d] for d in range(D)])
                    for i in range(Bt)])
    if silu:
        ref = ref * sigmoid_ref(ref)
    np.testing.assert_allclose(out, ref, rtol=1e-13, atol=1e-14)


def test_conv1d_matches_torch_conv1d():
    import torch
    rng = np.random.default_rng(32)
    Bt, D, L, K = 3, 4, 17, 4
    x = rng.standard_normal((Bt, D, L))
    w = rng.standard_normal((D, K))
    b = rng.standard_normal(D)
    ref = torch.nn.functional.conv1d(torch.from_numpy(x), torch.from_numpy(w)[:, None, :],
                                     torch.from_numpy(b), padding=K - 1, groups=D)[..., :L]
    ref = torch.nn.functional.silu(ref).numpy()
    np.testing.assert_allclose(oracle.causal_conv1d(x, w, b, silu=True), ref, rtol=1e-13, atol=1e-14)


def test_conv1d_impulse_response():
    # a unit impulse at t0 comes out as the filter read backwards: out[t0 + m] = w[K - 1 - m]
    K, L, t0 = 4, 12, 3
    w = np.array([[0.5, -1.0, 2.0, 3.0]])
    x = np.zeros((1, 1, L))
    x[0, 0, t0] = 1.0
    out = oracle.causal_conv1d(x, w, None, silu=False)[0, 0]
    expect = np.zeros(L)
    for m in range(K):
        expect[t0 + m] = w[0, K - 1 - m]
    np.testing.assert_array_equal(out, expect)


def test_conv1d_update_chain_is_the_conv():
    """T decode steps of the conv from a zero window give the prefill conv, step by step."""
    rng = np.random.default_rng(33)
    Bt, D, L, K = 2, 3, 11, 4
    x = rng.standard_normal((Bt, D, L))
    w = rng.standard_normal((D, K))
    b = rng.standard_normal(D)
    full = oracle.causal_conv1d(x, w, b, silu=True)
    st = np.zeros((Bt, D, K - 1))
    for t in range(L):
        st, o = oracle.causal_conv1d_update(st, x[..., t], w, b, silu=True)
        np.testing.assert_allclose(o, full[..., t], rtol=1e-14, atol=1e-15)
    np.testing.assert_array_equal(st, x[..., L - K + 1:])


def test_conv1d_varlen_restarts_at_boundaries():
    rng = np.random.default_rng(34)
    D, K = 3, 4
    cu = [0, 2, 2, 9, 15]
    x = rng.standard_normal((1, D, 15))
    w = rng.standard_normal((D, K))
    out = oracle.causal_conv1d_varlen(x, w, cu, None, silu=False)
    # the third sequence alone, from zeros: its first outputs see only its own inputs
    np.testing.assert_allclose(out[..., 9:], oracle.causal_conv1d(x[..., 9:], w, None, silu=False), rtol=1e-15)
    np.testing.assert_allclose(out[0, :, 9], w[:, K - 1] * x[0, :, 9], rtol=1e-15)


# ---------------------------------------------------------------------------
# 7d. packed variable-length sequences: the state restarts at every boundary
# ---------------------------------------------------------------------------

def test_varlen_single_sequence_is_the_scan():
    rng = np.random.default_rng(41)
    p = rand_problem(rng, 1, 3, 25)
    y, last = oracle.scan(**p, softplus=True)
    yv, lv = oracle.scan_varlen(p["u"], p["delta"], p["A"], p["B"], p["C"], [0, 25], p["D"], p["z"],
                                p["delta_bias"], True)
    np.testing.assert_array_equal(yv, y)
    np.testing.assert_array_equal(lv, last)


def test_varlen_sequences_are_isolated():
    rng = np.random.default_rng(42)
    p = rand_problem(rng, 1, 3, 40)
    cu = [0, 9, 9, 30, 40]  # includes an empty sequence
    h0 = rng.standard_normal((4, 3, N))
    y, last = oracle.scan_varlen(p["u"], p["delta"], p["A"], p["B"], p["C"], cu, p["D"], p["z"],
                                 p["delta_bias"], True, h0=h0)
    # perturbing sequence 0 changes nothing in sequences 2 and 3
    q = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in p.items()}
    q["u"][..., :9] += 1.0
    q["B"][..., :9] -= 0.5
    y2, last2 = oracle.scan_varlen(q["u"], q["delta"], q["A"], q["B"], q["C"], cu, q["D"], q["z"],
                                   q["delta_bias"], True, h0=h0)
    np.testing.assert_array_equal(y2[..., 9:], y[..., 9:])
    np.testing.assert_array_equal(last2[1:], last[1:])
    assert np.abs(y2[..., :9] - y[..., :9]).max() > 1e-3
    # the empty sequence hands back its initial state
    np.testing.assert_array_equal(last[1], h0[1])
    # with zero initial states, the scan of sequence 3 alone is the same
    y0, _ = oracle.scan_varlen(p["u"], p["delta"], p["A"], p["B"], p["C"], cu, p["D"], p["z"],
                               p["delta_bias"], True)
    sl = {k: (v[..., 30:] if k in ("u", "delta", "B", "C", "z") else v) for k, v in p.items()}
    ys, _ = oracle.scan(**sl, softplus=True)
    np.testing.assert_array_equal(y0[..., 30:], ys)


# ---------------------------------------------------------------------------
# 7e. backward: every gradient against central finite differences of the forward
# ---------------------------------------------------------------------------

def _fd_check_bwd(softplus, with_z, with_D, seed, n_probe=24):
    rng = np.random.default_rng(seed)
    p = rand_problem(rng, 2, 3, 7, with_z=with_z, with_D=with_D)
    if not softplus:  # keep the raw step positive, as softplus would
        p["delta"] = 0.2 * np.abs(p["delta"])
        p["delta_bias"] = rng.uniform(0.01, 0.1, size=p["delta_bias"].shape)
    dout = rng.standard_normal(p["u"].shape)
    g = oracle.scan_bwd(**p, softplus=softplus, dout=dout)

    def loss(q):
        return float((oracle.scan(**q, softplus=softplus)[0] * dout).sum())

    eps = 1e-6
    for name in ("u", "delta", "A", "B", "C", "D", "z", "delta_bias"):
        if p[name] is None:
            assert g.get("d" + name) is None
            continue
        grad = g["d" + name]
        idxs = list(np.ndindex(p[name].shape))
        pick = rng.choice(len(idxs), size=min(n_probe, len(idxs)), replace=False)
        for i in pick:
            idx = idxs[i]
            q = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in p.items()}
            q[name][idx] += eps
            lp = loss(q)
            q[name][idx] -= 2 * eps
            lm = loss(q)
            fd = (lp - lm) / (2 * eps)
            assert abs(fd - grad[idx]) <= 1e-6 * (1 + abs(fd)), (name, idx, fd, grad[idx])


def test_backward_matches_finite_differences():
    _fd_check_bwd(True, True, True, seed=51)


def test_backward_without_softplus_gate_or_skip():
    _fd_check_bwd(False, False, False, seed=52)


# ---------------------------------------------------------------------------
# 8. hand-derived worked example (tests/golden/halving_decay.txt)
# ---------------------------------------------------------------------------

def test_golden_halving_decay():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "halving_decay.txt"))
            if l.strip() and not l.startswith("#")]
    L = len(rows)
    u = np.array([float(r[1]) for r in rows]).reshape(1, 1, L)
    y_exp = np.array([float(r[2]) for r in rows])
    A = -np.arange(1, N + 1, dtype=np.float64).reshape(1, N)
    delta = np.full((1, 1, L), math.log(2))
    Bm = np.ones((1, N, L))
    Cm = np.ones((1, N, L))
    y, last = oracle.scan(u, delta, A, Bm, Cm, None, None, None, False)
    np.testing.assert_allclose(y[0, 0], y_exp, rtol=1e-14)
    ln2 = math.log(2)
    np.testing.assert_allclose(last[0, 0], 8.0 ** -(np.arange(N) + 1) * ln2 + 2 * ln2, rtol=1e-14)


# ---------------------------------------------------------------------------
# 9. the pins catch plausible mistakes: compile wrong variants of oracle.c
#    (mutations applied here, on the CPU, to a temporary copy) and require
#    every variant to fail at least one pin.
# ---------------------------------------------------------------------------

MUTANTS = {
    "dropped_u_in_input_term": ("h[n] = a_bar * h[n] + b_bar * x;", "h[n] = a_bar * h[n] + b_bar;"),
    "decay_sign_flipped": ("double a_bar = exp(dt * Ad[n]);", "double a_bar = exp(-dt * Ad[n]);"),
    "decay_without_dt": ("double a_bar = exp(dt * Ad[n]);", "double a_bar = exp(Ad[n]);"),
    "B_and_C_swapped": ("double b_bar = dt * Bb[n * L + t];", "double b_bar = dt * Cb[n * L + t];"),
    "B_bar_without_dt": ("double b_bar = dt * Bb[n * L + t];", "double b_bar = Bb[n * L + t];"),
    "B_time_index_off_by_one": ("double b_bar = dt * Bb[n * L + t];",
                                "double b_bar = dt * Bb[n * L + (t > 0 ? t - 1 : 0)];"),
    "readout_before_update": ("                h[n] = a_bar * h[n] + b_bar * x;\n"
                              "                y += Cb[n * L + t] * h[n];",
                              "                y += Cb[n * L + t] * h[n];\n"
                              "                h[n] = a_bar * h[n] + b_bar * x;"),
    "skip_uses_dt": ("y += Dskip[d] * x;", "y += Dskip[d] * dt;"),
    "gate_is_sigmoid": ("y *= silu(zr[t]);", "y *= 1.0 / (1.0 + exp(-zr[t]));"),
    "bias_dropped": ("double dt = dr[t] + (bias ? bias[d] : 0.0);", "double dt = dr[t];"),
    "softplus_is_exp": ("dt = sp_exact(dt);\n            double x = ur[t];",
                        "dt = exp(dt);\n            double x = ur[t];"),
    "A_channel_ignored": ("const double *Ad = A + d * N;", "const double *Ad = A;"),
    "decode_dropped_dt_on_input": ("zoh_gain(dt, A[d * N + n]) : dt;", "zoh_gain(dt, A[d * N + n]) : 1.0;"),
    "zoh_gain_sign_flipped": ("return expm1(dt * a) / a;", "return expm1(-dt * a) / a;"),
    "zoh_gain_not_divided": ("return expm1(dt * a) / a;", "return expm1(dt * a);"),
    "zoh_gain_is_exp": ("return expm1(dt * a) / a;", "return exp(dt * a) / a;"),
    "scan_zoh_ignored": ("b_bar = zoh_gain(dt, Ad[n]) * Bb[n * L + t];", "b_bar = dt * Bb[n * L + t];"),
    "decode_zoh_ignored": ("double gain = zoh_flag ? zoh_gain(dt, A[d * N + n]) : dt;", "double gain = dt;"),
    "bwd_no_decay_propagation": ("                g[n] *= a;\n", "\n"),
    "bwd_dA_without_dt": ("dA[d * N + n] += g[n] * dt * a * hp;", "dA[d * N + n] += g[n] * a * hp;"),
    "bwd_dB_uses_C": ("dB[b * N * L + n * L + t] += g[n] * dt * ur[t];",
                      "dB[b * N * L + n * L + t] += g[n] * dt * Cb[n * L + t];"),
    "bwd_dC_uses_previous_state": ("dC[b * N * L + n * L + t] += gy * hs[(t + 1) * N + n];",
                                   "dC[b * N * L + n * L + t] += gy * hs[t * N + n];"),
    "bwd_softplus_derivative_dropped": ("double draw = softplus_flag ? ddt * sigm(dr[t] + (bias ? bias[d] : 0.0)) : ddt;",
                                        "double draw = ddt;"),
    "bwd_gate_derivative_sign": ("s * (1.0 + zr[t] * (1.0 - s));", "s * (1.0 - zr[t] * (1.0 - s));"),
    "conv_filter_reversed": ("acc += wd[j] * xr[src];", "acc += wd[K - 1 - j] * xr[src];"),
    "conv_window_off_by_one": ("int64_t src = t + j - (K - 1);", "int64_t src = t + j - K;"),
    "conv_bias_dropped": ("double acc = bias ? bias[d] : 0.0;", "double acc = 0.0;"),
    "conv_silu_dropped": ("silu_flag ? silu(acc) : acc;", "acc;"),
    "decode_bias_only_with_softplus": ("double dt = dt_in[r] + (bias ? bias[d] : 0.0);\n        if (softplus_flag)\n            dt = sp_exact(dt);",
                                       "double dt = dt_in[r];\n        if (softplus_flag)\n            dt = sp_exact(dt + (bias ? bias[d] : 0.0));"),
    "scan_bias_only_with_softplus": ("double dt = dr[t] + (bias ? bias[d] : 0.0);",
                                     "double dt = dr[t] + (bias && softplus_flag ? bias[d] : 0.0);"),
    "decode_bias_dropped": ("double dt = dt_in[r] + (bias ? bias[d] : 0.0);", "double dt = dt_in[r];"),
    "decode_gate_dropped": ("            y *= silu(z[r]);\n        out[r] = y;", "        out[r] = y;"),
}

PIN_CALLS = [
    test_A_zero_is_prefix_sum,
    lambda: test_lti_equals_convolution(True, False),
    lambda: test_lti_equals_convolution(False, False),
    lambda: test_lti_equals_convolution(False, True),
    test_lti_step_input_closed_form,
    lambda: test_tiny_unrolled_sum(4, 5, 2),
    test_delta_to_zero_preserves_state,
    test_large_delta_resets_state,
    lambda: test_decode_steps_reproduce_scan(True),
    lambda: test_decode_steps_reproduce_scan(False),
    lambda: test_split_scan_equals_scan(7),
    test_affine_composition_is_associative,
    test_linear_in_u,
    test_softplus_and_silu_spot_values,
    test_golden_halving_decay,
    test_zoh_constant_input_is_exact,
    test_zoh_small_A_is_euler,
    test_zoh_decode_steps_reproduce_scan,
    lambda: test_conv1d_matches_numpy_convolve(True),
    test_backward_matches_finite_differences,
    test_backward_without_softplus_gate_or_skip,
    test_conv1d_matches_torch_conv1d,
    test_conv1d_impulse_response,
]


def _compile_variant(src_text, out_dir, tag):
    import subprocess
    c = os.path.join(out_dir, f"m_{tag}.c")
    so = os.path.join(out_dir, f"m_{tag}.so")
    with open(c, "w") as f:
        f.write(src_text)
    subprocess.check_call(["gcc", "-O1", "-fopenmp", "-shared", "-fPIC", "-std=c11", c, "-o", so, "-lm"])
    return so


def _count_failures(lib_path):
    import ctypes
    lib = ctypes.CDLL(lib_path)
    P, I64 = ctypes.c_void_p, ctypes.c_int64
    lib.oracle_scan_f64.argtypes = [I64, I64, I64, I64, P, P, P, P, P, P, P, P, ctypes.c_int, ctypes.c_int,
                                    P, P, P]
    lib.oracle_state_update_f64.argtypes = [I64, I64, I64, P, P, P, P, P, P, P, P, P, ctypes.c_int,
                                            ctypes.c_int, P]
    lib.oracle_causal_conv1d_f64.argtypes = [I64, I64, I64, I64, P, P, P, ctypes.c_int, P]
    lib.oracle_scan_bwd_f64.argtypes = [I64, I64, I64, I64, P, P, P, P, P, P, P, P, ctypes.c_int,
                                        P, P, P, P, P, P, P, P, P]
    lib.oracle_num_threads.restype = ctypes.c_int
    saved = oracle._lib
    oracle._lib = lib
    fails = 0
    try:
        with np.errstate(all="ignore"):
            for call in PIN_CALLS:
                try:
                    call()
                except AssertionError:
                    fails += 1
    finally:
        oracle._lib = saved
    return fails


def test_mutants_are_caught(tmp_path):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "oracle.c")).read()
    # the unmutated copy passes every pin
    assert _count_failures(_compile_variant(src, str(tmp_path), "orig")) == 0
    for tag, (old, new) in MUTANTS.items():
        assert src.count(old) == 1, f"mutation site for {tag} not unique"
        so = _compile_variant(src.replace(old, new), str(tmp_path), tag)
        assert _count_failures(so) > 0, f"mutant {tag} passed every pin"
