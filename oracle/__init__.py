"""fp64 CPU oracle for the selective scan and the decode state update.

TEST INFRASTRUCTURE ONLY: the tests, the package smoke check and the
benchmark's CPU-baseline leg are the only callers.  The CUDA library never
imports, links or runs anything here, and this package imports nothing from
it.  The arithmetic lives in ``oracle.c`` (plain C, fp64, OpenMP over rows);
this module only builds that file with gcc and marshals numpy arrays.

Every function here is pinned by ``tests/test_oracle_pins.py``; no function is
"parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile ``oracle.c`` into ``liboracle.so`` (gcc, -O2, IEEE semantics, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fno-fast-math", "-fopenmp", "-shared", "-fPIC",
                               "-std=c11", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        lib.oracle_scan_f64.argtypes = [I64, I64, I64, I64, P, P, P, P, P, P, P, P,
                                        ctypes.c_int, ctypes.c_int, P, P, P]
        lib.oracle_scan_f64.restype = None
        lib.oracle_state_update_f64.argtypes = [I64, I64, I64, P, P, P, P, P, P, P, P, P,
                                                ctypes.c_int, ctypes.c_int, P]
        lib.oracle_state_update_f64.restype = None
        lib.oracle_causal_conv1d_f64.argtypes = [I64, I64, I64, I64, P, P, P, ctypes.c_int, P]
        lib.oracle_scan_bwd_f64.argtypes = [I64, I64, I64, I64, P, P, P, P, P, P, P, P, ctypes.c_int,
                                            P, P, P, P, P, P, P, P, P]
        lib.oracle_scan_bwd_f64.restype = None
        lib.oracle_causal_conv1d_f64.restype = None
        lib.oracle_num_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def num_threads() -> int:
    return _load().oracle_num_threads()


def _f64(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def scan(u, delta, A, B, C, D=None, z=None, delta_bias=None, softplus=True,
         h0=None, zoh=False) -> Tuple[np.ndarray, np.ndarray]:
    """Selective scan in fp64.

    Shapes: ``u, delta, z`` [Bt, D, L]; ``B, C`` [Bt, N, L]; ``A`` [D, N];
    ``D, delta_bias`` [D]; ``h0`` [Bt, D, N] (zero when omitted).  ``zoh``:
    zero-order-hold input gain (exp(delta A) - 1) / A instead of delta.
    Returns ``(y [Bt, D, L], last_state [Bt, D, N])`` as float64.
    """
    u, delta, A, B, C = map(_f64, (u, delta, A, B, C))
    D, z, delta_bias, h0 = map(_f64, (D, z, delta_bias, h0))
    Bt, Dd, L = u.shape
    N = A.shape[1]
    if N > 64:
        raise ValueError("oracle supports N <= 64")
    assert delta.shape == u.shape and B.shape == (Bt, N, L) and C.shape == (Bt, N, L)
    assert A.shape == (Dd, N)
    for v, shp in ((D, (Dd,)), (delta_bias, (Dd,)), (z, u.shape), (h0, (Bt, Dd, N))):
        assert v is None or v.shape == shp
    out = np.empty((Bt, Dd, L), np.float64)
    last = np.empty((Bt, Dd, N), np.float64)
    _load().oracle_scan_f64(Bt, Dd, L, N, _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C),
                            _ptr(D), _ptr(z), _ptr(delta_bias), int(bool(softplus)),
                            int(bool(zoh)), _ptr(h0), _ptr(out), _ptr(last))
    return out, last


def state_update(state, x, dt, A, B, C, D=None, z=None, dt_bias=None,
                 softplus=True, zoh=False) -> Tuple[np.ndarray, np.ndarray]:
    """One decode step in fp64 on a copy of ``state``.

    Shapes: ``state`` [Bt, D, N]; ``x, dt, z`` [Bt, D]; ``B, C`` [Bt, N]; ``A`` [D, N].
    Returns ``(new_state [Bt, D, N], y [Bt, D])``.
    """
    st = np.array(state, dtype=np.float64, copy=True, order="C")
    x, dt, A, B, C = map(_f64, (x, dt, A, B, C))
    D, z, dt_bias = map(_f64, (D, z, dt_bias))
    Bt, Dd, N = st.shape
    if N > 64:
        raise ValueError("oracle supports N <= 64")
    assert x.shape == (Bt, Dd) and dt.shape == (Bt, Dd) and A.shape == (Dd, N)
    assert B.shape == (Bt, N) and C.shape == (Bt, N)
    out = np.empty((Bt, Dd), np.float64)
    _load().oracle_state_update_f64(Bt, Dd, N, _ptr(st), _ptr(x), _ptr(dt), _ptr(A), _ptr(B),
                                    _ptr(C), _ptr(D), _ptr(z), _ptr(dt_bias),
                                    int(bool(softplus)), int(bool(zoh)), _ptr(out))
    return st, out


def scan_bwd(u, delta, A, B, C, D=None, z=None, delta_bias=None, softplus=True, dout=None) -> dict:
    """Gradients of ``scan`` (Euler, zero initial state) with respect to every input, for
    dLoss/dout = ``dout`` [Bt, D, L].  Returns a dict with du, ddelta, dA, dB, dC and, when
    the inputs are given, dD, dz, ddelta_bias (float64)."""
    u, delta, A, B, C, dout = map(_f64, (u, delta, A, B, C, dout))
    D, z, delta_bias = map(_f64, (D, z, delta_bias))
    Bt, Dd, L = u.shape
    N = A.shape[1]
    if N > 64:
        raise ValueError("oracle supports N <= 64")
    assert dout.shape == u.shape
    out = dict(du=np.empty_like(u), ddelta=np.empty_like(u), dA=np.empty_like(A), dB=np.empty_like(B),
               dC=np.empty_like(C), dD=None if D is None else np.empty_like(D),
               dz=None if z is None else np.empty_like(z),
               ddelta_bias=None if delta_bias is None else np.empty_like(delta_bias))
    _load().oracle_scan_bwd_f64(Bt, Dd, L, N, _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                                _ptr(z), _ptr(delta_bias), int(bool(softplus)), _ptr(dout),
                                _ptr(out["du"]), _ptr(out["ddelta"]), _ptr(out["dA"]), _ptr(out["dB"]),
                                _ptr(out["dC"]), _ptr(out["dD"]), _ptr(out["dz"]), _ptr(out["ddelta_bias"]))
    return out


def causal_conv1d(x, w, bias=None, silu=True) -> np.ndarray:
    """Causal depthwise conv1d along L (then SiLU) in fp64: ``x`` [Bt, D, L], ``w`` [D, K],
    ``bias`` [D].  Returns [Bt, D, L]."""
    x, w, bias = map(_f64, (x, w, bias))
    Bt, Dd, L = x.shape
    K = w.shape[1]
    assert w.shape == (Dd, K) and (bias is None or bias.shape == (Dd,))
    out = np.empty((Bt, Dd, L), np.float64)
    _load().oracle_causal_conv1d_f64(Bt, Dd, L, K, _ptr(x), _ptr(w), _ptr(bias), int(bool(silu)), _ptr(out))
    return out


def causal_conv1d_varlen(x, w, cu_seqlens, bias=None, silu=True) -> np.ndarray:
    """Causal conv1d (then SiLU) of packed sequences: ``x`` [1, D, T] with ``cu_seqlens``
    offsets; every sequence sees zeros before its own first step.  Built only from
    ``causal_conv1d`` on each slice."""
    cu = np.asarray(cu_seqlens, np.int64)
    x = np.asarray(x, np.float64)
    out = np.zeros(x.shape, np.float64)
    for s in range(len(cu) - 1):
        a, b = int(cu[s]), int(cu[s + 1])
        if b > a:
            out[..., a:b] = causal_conv1d(x[..., a:b], w, bias, silu)
    return out


def causal_conv1d_update(conv_state, x, w, bias=None, silu=True):
    """One decode step of the causal conv1d: ``conv_state`` [Bt, D, K-1] holds the previous
    K-1 inputs (oldest first), ``x`` [Bt, D] the new one.  Returns ``(new_state, out [Bt, D])``:
    the conv (then SiLU) at the newest position of the window [state, x], and the window
    without its oldest input.  Built only from ``causal_conv1d`` on the window."""
    st = np.asarray(conv_state, np.float64)
    win = np.concatenate([st, np.asarray(x, np.float64)[..., None]], axis=-1)  # [Bt, D, K]
    out = causal_conv1d(win, w, bias, silu)[..., -1]
    return win[..., 1:].copy(), out


def scan_varlen(u, delta, A, B, C, cu_seqlens, D=None, z=None, delta_bias=None, softplus=True,
                h0=None, zoh=False) -> Tuple[np.ndarray, np.ndarray]:
    """Selective scan of several sequences packed along L (the varlen layout): ``u, delta,
    z`` [1, D, T], ``B, C`` [1, N, T], ``cu_seqlens`` [S + 1] offsets (0 = c_0 <= ... <=
    c_S = T).  Sequence s covers steps c_s .. c_(s+1) - 1 and starts from ``h0[s]`` (zero
    when omitted): the state does not carry across a boundary.  Returns ``(y [1, D, T],
    last_state [S, D, N])``.  Built only from ``scan`` on each slice."""
    cu = np.asarray(cu_seqlens, np.int64)
    Dd, N = np.shape(A)
    T = np.shape(u)[-1]
    assert cu[0] == 0 and cu[-1] == T and (np.diff(cu) >= 0).all()
    S = len(cu) - 1
    y = np.zeros((1, Dd, T), np.float64)
    last = np.zeros((S, Dd, N), np.float64)
    for s in range(S):
        a, b = int(cu[s]), int(cu[s + 1])
        h_init = None if h0 is None else np.asarray(h0, np.float64)[s:s + 1]
        if b == a:
            last[s] = 0.0 if h_init is None else h_init[0]
            continue
        sl = (lambda v: None if v is None else np.asarray(v)[..., a:b])
        ys, hs = scan(sl(u), sl(delta), A, sl(B), sl(C), D, sl(z), delta_bias, softplus,
                      h0=h_init, zoh=zoh)
        y[..., a:b] = ys
        last[s] = hs[0]
    return y, last


# --------------------------------------------------------------------------
# convenience over synth.ScanInputs / synth.DecodeInputs
# --------------------------------------------------------------------------


def scan_inputs(inp, h0=None, zoh=False):
    """Oracle scan of a whole ``synth.ScanInputs`` problem."""
    return scan(inp.f64("u"), inp.f64("delta"), inp.f64("A"), inp.f64("B"), inp.f64("C"),
                inp.f64("D"), inp.f64("z"), inp.f64("delta_bias"), inp.softplus, h0=h0, zoh=zoh)


def scan_rows(inp, rows: Sequence[Tuple[int, int]]):
    """Oracle scan of selected rows ``(b, d)`` of a ``synth.ScanInputs`` problem.

    Returns ``(y [len(rows), L], last_state [len(rows), N])``.  Used to check
    full-size outputs at sampled rows without running the whole problem.
    """
    ys, hs = [], []
    for b, d in rows:
        u = _widen_slice(inp, "u", b, d)
        dl = _widen_slice(inp, "delta", b, d)
        z = _widen_slice(inp, "z", b, d)
        Bm = _widen_batch(inp, "B", b)
        Cm = _widen_batch(inp, "C", b)
        A = np.asarray(inp.A[d:d + 1], np.float64)
        D = None if inp.D is None else np.asarray(inp.D[d:d + 1], np.float64)
        bias = None if inp.delta_bias is None else np.asarray(inp.delta_bias[d:d + 1], np.float64)
        y, h = scan(u, dl, A, Bm, Cm, D, z, bias, inp.softplus)
        ys.append(y[0, 0])
        hs.append(h[0, 0])
    return np.stack(ys), np.stack(hs)


def scan_block(inp, b: int, d0: int, d1: int, h0=None, zoh: bool = False):
    """Oracle scan of channels ``d0 .. d1 - 1`` of batch ``b`` of a ``synth.ScanInputs`` problem
    (``h0`` [1, d1 - d0, N] or None).  Returns ``(y [1, d1 - d0, L], last_state [1, d1 - d0, N])``.
    Lets full-size outputs be checked on every row with bounded host memory."""
    from synth import to_f64  # input widening only (bit manipulation)

    def sl(name):
        a = getattr(inp, name)
        return None if a is None else to_f64(a[b:b + 1, d0:d1], inp.io_dtype)

    def ch(name):
        a = getattr(inp, name)
        return None if a is None else np.asarray(a[d0:d1], np.float64)

    return scan(sl("u"), sl("delta"), ch("A"), _widen_batch(inp, "B", b), _widen_batch(inp, "C", b),
                ch("D"), sl("z"), ch("delta_bias"), inp.softplus, h0=h0, zoh=zoh)


def _widen_slice(inp, name, b, d):
    a = getattr(inp, name)
    if a is None:
        return None
    sl = a[b:b + 1, d:d + 1]
    from synth import to_f64  # input widening only (bit manipulation)
    return to_f64(sl, inp.io_dtype)


def _widen_batch(inp, name, b):
    a = getattr(inp, name)
    from synth import to_f64
    return to_f64(a[b:b + 1], inp.io_dtype)


def state_update_inputs(inp, state=None, zoh=False):
    """Oracle decode step of a ``synth.DecodeInputs`` batch (``state`` overrides ``inp.state``)."""
    st = inp.state if state is None else state
    return state_update(st, inp.f64("x"), inp.f64("dt"), inp.f64("A"), inp.f64("B"),
                        inp.f64("C"), inp.f64("D"), inp.f64("z"), inp.f64("dt_bias"),
                        inp.softplus, zoh=zoh)
