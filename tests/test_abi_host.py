"""Host-side checks of the C ABI, no GPU needed.

* libmssm.so loads and exports every function include/mssm.h declares;
* argument validation returns the documented status before anything touches
  the device (descriptors carry fake, never-dereferenced device pointers).
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include")) if f.endswith(".h")]


@pytest.fixture(scope="module")
def lib():
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "_mssm_build", os.path.join(ROOT, "selective_state_space_46_b200", "build.py"))
    build = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(build)
    return ctypes.CDLL(build.build())


def declared_functions():
    names = set()
    for h in HEADERS:
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"\b(mssm_[a-z0-9_]+)\s*\(", text):
            names.add(m.group(1))
    return sorted(names)


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert {"mssm_selective_scan_fwd", "mssm_state_update"} <= set(names)
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"


# ---------------------------------------------------------------------------
# validation (fake pointers; every case below fails before any CUDA call)
# ---------------------------------------------------------------------------

class T(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int32), ("ndim", ctypes.c_int32),
                ("shape", ctypes.c_int64 * 4), ("stride", ctypes.c_int64 * 4)]


_fake = [0x10000]


def mk(shape, dtype=1, stride=None):
    t = T()
    _fake[0] += 1 << 30
    t.data = _fake[0]
    t.dtype = dtype
    t.ndim = len(shape)
    if stride is None:
        stride, acc = [], 1
        for s in reversed(shape):
            stride.insert(0, acc)
            acc *= s
    for i, (s, st) in enumerate(zip(shape, stride)):
        t.shape[i] = s
        t.stride[i] = st
    return t


def scan_args(Bt=2, D=8, L=32, N=16, dt=1, **over):
    a = dict(u=mk([Bt, D, L], dt), delta=mk([Bt, D, L], dt), A=mk([D, N], 0), B=mk([Bt, N, L], dt),
             C=mk([Bt, N, L], dt), D=mk([D], 0), z=mk([Bt, D, L], dt), delta_bias=mk([D], 0),
             out=mk([Bt, D, L], dt), last_state=mk([Bt, D, N], 0))
    a.update(over)
    return a


def call_scan(lib, a, softplus=1):
    P = lambda t: None if t is None else ctypes.byref(t)  # noqa: E731
    f = lib.mssm_selective_scan_fwd
    f.restype = ctypes.c_int
    return f(P(a["u"]), P(a["delta"]), P(a["A"]), P(a["B"]), P(a["C"]), P(a["D"]), P(a["z"]),
             P(a["delta_bias"]), softplus, P(a["out"]), P(a["last_state"]), None)


def last_error(lib):
    lib.mssm_last_error.restype = ctypes.c_char_p
    return lib.mssm_last_error().decode()


INVALID, UNSUPPORTED = 1, 2


@pytest.mark.parametrize("case,expect", [
    ("null_u", INVALID),
    ("null_out", INVALID),
    ("N8", UNSUPPORTED),
    ("delta_dtype", INVALID),
    ("A_bf16", INVALID),
    ("B_shape", INVALID),
    ("z_shape", INVALID),
    ("out_aliases_u", INVALID),
    ("inner_stride", UNSUPPORTED),
    ("last_state_dtype", INVALID),
    ("null_data", INVALID),
    ("bad_u_dtype", INVALID),
])
def test_scan_validation(lib, case, expect):
    a = scan_args()
    if case == "null_u":
        a["u"] = None
    elif case == "null_out":
        a["out"] = None
    elif case == "N8":
        a = scan_args(N=8)
    elif case == "delta_dtype":
        a["delta"] = mk([2, 8, 32], 0)
    elif case == "A_bf16":
        a["A"] = mk([8, 16], 1)
    elif case == "B_shape":
        a["B"] = mk([2, 16, 31], 1)
    elif case == "z_shape":
        a["z"] = mk([2, 7, 32], 1)
    elif case == "out_aliases_u":
        a["out"].data = a["u"].data
    elif case == "inner_stride":
        a["u"] = mk([2, 8, 32], 1, stride=[512, 64, 2])
    elif case == "last_state_dtype":
        a["last_state"] = mk([2, 8, 16], 1)
    elif case == "null_data":
        a["C"].data = None
    elif case == "bad_u_dtype":
        a["u"].dtype = 7
    assert call_scan(lib, a) == expect
    assert last_error(lib)


class Ext(ctypes.Structure):
    _fields_ = [("struct_size", ctypes.c_int32), ("discretization", ctypes.c_int32),
                ("h0", ctypes.POINTER(T)), ("cu_seqlens", ctypes.POINTER(T)), ("max_seqlen", ctypes.c_int64)]


def test_scan_rejects_rows_beyond_31_bits(lib):
    """2^31 rows (Bt * D) at L = 1 would fit in device memory, but the kernels index rows
    with 32-bit integers: the call is refused on the host, before any CUDA call (so this
    runs without a GPU; the descriptors' pointers are never dereferenced)."""
    a = scan_args(Bt=1 << 16, D=1 << 15, L=1)
    assert call_scan(lib, a) == UNSUPPORTED
    assert "31 bits" in last_error(lib)


@pytest.mark.parametrize("case", ["short_struct", "bad_disc", "h0_shape", "h0_dtype", "h0_inner_stride",
                                  "h0_aliases_last_state"])
def test_scan_ext_validation(lib, case):
    a = scan_args()
    h0 = mk([2, 8, 16], 0)
    ext = Ext(ctypes.sizeof(Ext), 0, ctypes.pointer(h0))
    expect = INVALID
    if case == "short_struct":
        ext.struct_size = 4
    elif case == "bad_disc":
        ext.discretization = 2
    elif case == "h0_shape":
        ext.h0 = ctypes.pointer(mk([2, 8, 8], 0))
        expect = INVALID
    elif case == "h0_dtype":
        ext.h0 = ctypes.pointer(mk([2, 8, 16], 1))
    elif case == "h0_inner_stride":
        ext.h0 = ctypes.pointer(mk([2, 8, 16], 0, stride=[256, 32, 2]))
        expect = UNSUPPORTED
    elif case == "h0_aliases_last_state":
        h0.data = a["last_state"].data
    P = lambda t: None if t is None else ctypes.byref(t)  # noqa: E731
    f = lib.mssm_selective_scan_fwd_ex
    f.restype = ctypes.c_int
    st = f(P(a["u"]), P(a["delta"]), P(a["A"]), P(a["B"]), P(a["C"]), P(a["D"]), P(a["z"]), P(a["delta_bias"]),
           1, ctypes.byref(ext), P(a["out"]), P(a["last_state"]), None)
    assert st == expect, last_error(lib)
    assert last_error(lib)


@pytest.mark.parametrize("case", ["cu_dtype", "cu_2d", "batch_not_1", "last_state_batches", "max_seqlen_big",
                                  "h0_batches"])
def test_scan_varlen_validation(lib, case):
    S, D, Tn = 3, 8, 40
    a = scan_args(Bt=1, D=D, L=Tn)
    a["last_state"] = mk([S, D, 16], 0)
    cu = mk([S + 1], 2)
    ext = Ext(ctypes.sizeof(Ext), 0, None, ctypes.pointer(cu), 20)
    if case == "cu_dtype":
        ext.cu_seqlens = ctypes.pointer(mk([S + 1], 0))
    elif case == "cu_2d":
        ext.cu_seqlens = ctypes.pointer(mk([1, S + 1], 2))
    elif case == "batch_not_1":
        a = scan_args(Bt=2, D=D, L=Tn)
        a["last_state"] = mk([S, D, 16], 0)
    elif case == "last_state_batches":
        a["last_state"] = mk([1, D, 16], 0)
    elif case == "max_seqlen_big":
        ext.max_seqlen = Tn + 1
    elif case == "h0_batches":
        ext.h0 = ctypes.pointer(mk([1, D, 16], 0))
    P = lambda t: None if t is None else ctypes.byref(t)  # noqa: E731
    f = lib.mssm_selective_scan_fwd_ex
    f.restype = ctypes.c_int
    st = f(P(a["u"]), P(a["delta"]), P(a["A"]), P(a["B"]), P(a["C"]), P(a["D"]), P(a["z"]), P(a["delta_bias"]),
           1, ctypes.byref(ext), P(a["out"]), P(a["last_state"]), None)
    assert st == INVALID, (st, last_error(lib))
    assert last_error(lib)


def test_conv_validation(lib):
    P = lambda t: None if t is None else ctypes.byref(t)  # noqa: E731
    f = lib.mssm_causal_conv1d_fwd
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_int64, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p]
    x, out = mk([2, 8, 32], 1), mk([2, 8, 32], 1)
    assert f(P(x), P(mk([8, 5], 0)), None, None, 0, 1, P(out), None) == UNSUPPORTED  # K = 5
    assert f(P(x), P(mk([8, 4], 1)), None, None, 0, 1, P(out), None) == INVALID      # bf16 weight
    out.data = x.data
    assert f(P(x), P(mk([8, 4], 0)), None, None, 0, 1, P(out), None) == INVALID      # alias
    out = mk([2, 8, 32], 1)
    assert f(P(x), P(mk([8, 4], 0)), None, P(mk([3], 2)), 10, 1, P(out), None) == INVALID  # Bt != 1
    g = lib.mssm_causal_conv1d_update
    g.restype = ctypes.c_int
    g.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p]
    xs, os_ = mk([2, 8], 1), mk([2, 8], 1)
    assert g(P(mk([2, 8, 0], 1)), P(xs), P(mk([8, 1], 0)), None, 1, P(os_), None) == UNSUPPORTED  # K = 1
    assert g(P(mk([2, 8, 2], 1)), P(xs), P(mk([8, 4], 0)), None, 1, P(os_), None) == INVALID      # state K-1


def test_decode_ex_rejects_unknown_discretization(lib):
    P = ctypes.byref
    f = lib.mssm_state_update_ex
    f.restype = ctypes.c_int
    st, x, dt = mk([4, 8, 16], 0), mk([4, 8], 1), mk([4, 8], 1)
    A, B, C, D, z, out = mk([8, 16], 0), mk([4, 16], 1), mk([4, 16], 1), mk([8], 0), mk([4, 8], 1), mk([4, 8], 1)
    assert f(P(st), P(x), P(dt), P(A), P(B), P(C), P(D), P(z), None, 1, 5, P(out), None) == INVALID
    assert "discretization" in last_error(lib)


def test_empty_problem_is_noop(lib):
    # Bt == 0 returns OK without touching the device
    a = scan_args(Bt=0)
    assert call_scan(lib, a) == 0


def test_bwd_refuses_too_many_chunks_before_launching(lib):
    """More than 65 535 chunks of 64 steps cannot be gridded: refused with UNSUPPORTED before the
    gradients are zeroed or anything else reaches the device (without a GPU a CUDA call would
    fail with MSSM_ERR_CUDA instead; the descriptors' pointers are never dereferenced)."""
    Bt, D, L, N = 1, 8, 65535 * 64 + 1, 16
    t = lambda shape, dt=1: ctypes.byref(mk(shape, dt))  # noqa: E731
    f = lib.mssm_selective_scan_bwd
    f.restype = ctypes.c_int
    st = f(t([Bt, D, L]), t([Bt, D, L]), t([D, N], 0), t([Bt, N, L]), t([Bt, N, L]), t([D], 0), t([Bt, D, L]),
           t([D], 0), 1, t([Bt, D, L]), t([Bt, D, L]), t([Bt, D, L]), t([D, N], 0), t([Bt, N, L], 0),
           t([Bt, N, L], 0), t([D], 0), t([Bt, D, L]), t([D], 0), None)
    assert st == UNSUPPORTED, (st, last_error(lib))
    assert "too large" in last_error(lib)


def test_decode_validation(lib):
    P = ctypes.byref
    f = lib.mssm_state_update
    f.restype = ctypes.c_int
    st, x, dt = mk([4, 8, 16], 0), mk([4, 8], 1), mk([4, 8], 1)
    A, B, C, D, z, out = mk([8, 16], 0), mk([4, 16], 1), mk([4, 16], 1), mk([8], 0), mk([4, 8], 1), mk([4, 8], 1)
    bad_state = mk([4, 8, 16], 1)
    assert f(P(bad_state), P(x), P(dt), P(A), P(B), P(C), P(D), P(z), P(out), None) == INVALID
    bad_A = mk([8, 32], 0)
    assert f(P(st), P(x), P(dt), P(bad_A), P(B), P(C), P(D), P(z), P(out), None) == UNSUPPORTED
    out.data = x.data
    assert f(P(st), P(x), P(dt), P(A), P(B), P(C), P(D), P(z), P(out), None) == INVALID
    assert f(None, P(x), P(dt), P(A), P(B), P(C), P(D), P(z), P(out), None) == INVALID


def test_options_and_strings(lib):
    lib.mssm_set_option.argtypes = [ctypes.c_int, ctypes.c_int64]
    assert lib.mssm_set_option(1, 2) == INVALID
    assert lib.mssm_set_option(2, 100) == INVALID      # not a multiple of 64
    assert lib.mssm_set_option(99, 0) == INVALID
    assert lib.mssm_set_option(4, 6) == INVALID
    for v in (5, 4, 3, 0):
        assert lib.mssm_set_option(4, v) == 0
    assert lib.mssm_set_option(5, 4) == INVALID and lib.mssm_set_option(5, -1) == INVALID
    for v in (1, 2, 3, 0):
        assert lib.mssm_set_option(5, v) == 0
    assert lib.mssm_set_option(6, 2) == INVALID
    assert lib.mssm_set_option(6, 1) == 0 and lib.mssm_set_option(6, 0) == 0
    assert lib.mssm_set_option(2, 128) == 0
    assert lib.mssm_set_option(2, 0) == 0
    for v in (16, 48, -32, 256):
        assert lib.mssm_set_option(7, v) == INVALID
    for v in (128, 64, 32, 0):
        assert lib.mssm_set_option(7, v) == 0
    for v in (-1, 3, 4):
        assert lib.mssm_set_option(8, v) == INVALID
    for v in (2, 1, 0):
        assert lib.mssm_set_option(8, v) == 0
    lib.mssm_status_string.restype = ctypes.c_char_p
    assert lib.mssm_status_string(2) == b"MSSM_ERR_UNSUPPORTED"
    lib.mssm_version.restype = ctypes.c_char_p
    assert re.match(rb"^\d+\.\d+\.\d+$", lib.mssm_version())


def test_scan_plan_measured_best():
    """The automatic plans of the benchmark workloads are the ones measured fastest on B200
    (sweeps of chunk length, rows per tile, rows per thread and schedule): a change to the cost
    model that moves one of them must be measured again."""
    import selective_state_space_46_b200 as m
    for opt in (m.MSSM_OPT_CHUNK_LEN, m.MSSM_OPT_SCHEDULE, m.MSSM_OPT_ROWS_PER_CTA, m.MSSM_OPT_ROWS_PER_THREAD):
        m.mssm_set_option(opt, 0)
    expect = {
        # 63.1 us; 32 rows chunk 128: 63.8, 64 rows chunk 128: 65.3, chunk 192: 66.2, split: 73.5
        (2, 1536, 2048, -1): ("summaries+forward", 32, 1, 192),
        # 746 us; chunk 256: 761, 1024: 752; two rows per thread: 1096-1107; forward only: 1139
        (8, 5120, 4096, -1): ("chained", 32, 1, 512),
        # 1662-1674 us; chunk 2560: 1759, 4608: 2031; 32 rows: 1737; split: 1780-1818;
        # two rows per thread: 1680-1769; fused: 1815
        (1, 2048, 131072, -1): ("summaries+forward", 64, 1, 3584),
        # many rows, short sequences, chained: chunk 256 211.0 us, 128: 223.6, 64: 247.9
        (8, 5120, 1024, -1): ("chained", 32, 1, 256),
        # 251.2 us; chunk 128: 258.4, 64: 289.2
        (64, 1536, 512, -1): ("chained", 32, 1, 256),
        # packed sequences (32 of up to 4096 steps): 64 rows chunk 256: 320.4 us, 384: 323.2,
        # 512: 332.7, 192: 327.8, 128: 343.2; 32 rows chunk 256: 343.4, 384: 351.7
        (32, 1536, 4096, 27048): ("summaries+forward", 64, 1, 320),
    }
    for (S, D, L, total), want in expect.items():
        plan = m.mssm_scan_plan(S, D, L, sm_count=148, total_len=total)
        got = (plan["schedule"], plan["rows_per_cta"], plan["rows_per_thread"], plan["chunk_len"])
        assert got == want, (S, D, L, plan)


def test_scan_plan_host_only(lib):
    """The launch plan is host logic: check its invariants without a GPU."""
    f = lib.mssm_scan_plan
    f.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int, ctypes.POINTER(ctypes.c_int),
                  ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_int)]
    rows, seg, nseg, sched = ctypes.c_int(), ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int()
    for Bt, D, L in [(1, 64, 256), (2, 1536, 2048), (8, 5120, 4096), (1, 2048, 131072), (3, 7, 1), (1, 1, 0),
                     (64, 8192, 100), (1, 16, 1 << 24)]:
        assert f(Bt, D, L, 148, ctypes.byref(rows), ctypes.byref(seg), ctypes.byref(nseg), ctypes.byref(sched)) == 0
        assert rows.value in (32, 64)
        assert seg.value % 64 == 0 and seg.value >= 64
        assert nseg.value >= 1 and nseg.value <= 65535
        assert sched.value in (0, 1, 2) and (sched.value == 0) == (nseg.value == 1)
        if L > 0:
            # the chunks cover the sequence exactly: every chunk but the last is full
            assert (nseg.value - 1) * seg.value < L <= nseg.value * seg.value
    # a shape with many row tiles runs its chunks chained, without summaries
    assert f(8, 5120, 4096, 148, ctypes.byref(rows), ctypes.byref(seg), ctypes.byref(nseg), ctypes.byref(sched)) == 0
    assert sched.value == 2 and rows.value == 32
    # few rows and a long sequence are split
    assert f(1, 2048, 131072, 148, ctypes.byref(rows), ctypes.byref(seg), ctypes.byref(nseg), ctypes.byref(sched)) == 0
    assert nseg.value > 1 and sched.value == 1
    # an explicit chunk length is honoured
    lib.mssm_set_option.argtypes = [ctypes.c_int, ctypes.c_int64]
    assert lib.mssm_set_option(2, 128) == 0
    assert f(1, 64, 1000, 148, ctypes.byref(rows), ctypes.byref(seg), ctypes.byref(nseg), ctypes.byref(sched)) == 0
    assert (seg.value, nseg.value) == (128, 8)
    assert lib.mssm_set_option(2, 0) == 0
    assert f(-1, 64, 1000, 148, None, None, None, None) == INVALID
    # every schedule can be forced (forward-only never splits)
    for value, mode in ((1, 0), (2, 1), (3, 2), (4, 3)):
        assert lib.mssm_set_option(4, value) == 0
        assert f(2, 1536, 2048, 148, ctypes.byref(rows), ctypes.byref(seg), ctypes.byref(nseg), ctypes.byref(sched)) == 0
        assert sched.value == mode and (nseg.value == 1) == (mode == 0)
    assert lib.mssm_set_option(4, 0) == 0
