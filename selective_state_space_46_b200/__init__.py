"""B200-native (sm_100a) Mamba-1 selective scan: Python binding of libmssm.so.

This module only marshals arguments: it turns torch tensors into the C ABI's
``mssm_tensor`` descriptors (pointer, dtype, shape, strides) and calls the
entry points declared in ``include/mssm.h`` with the same names.  Every step of
the computation runs in the library's CUDA kernels; there is no CPU or PyTorch
fallback, and importing fails loudly when the library has not been built.

Build the library with ``python selective_state_space_46_b200/build.py``.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

__all__ = [
    "MssmError", "mssm_selective_scan_fwd", "mssm_selective_scan_fwd_noalloc", "mssm_state_update",
    "mssm_state_update_ex",
    "mssm_get_error", "mssm_set_option", "mssm_shutdown", "mssm_version", "mssm_status_string",
    "mssm_last_error", "selective_scan_fwd", "state_update", "lib_path",
    "MSSM_OPT_FORCE_GENERAL_A", "MSSM_OPT_CHUNK_LEN", "MSSM_OPT_KERNEL_TIMING", "MSSM_OPT_SCHEDULE", "SCHEDULES",
    "MSSM_OPT_DECODE_PATH", "DECODE_PATHS", "MSSM_OPT_TEST_HOOKS", "MSSM_OPT_ROWS_PER_CTA", "MSSM_OPT_ROWS_PER_THREAD", "MSSM_ERR_TIMEOUT", "mssm_kernel_stats", "mssm_scan_plan",
    "mssm_selective_scan_fwd_ex", "MSSM_DISC_EULER", "MSSM_DISC_ZOH",
    "mssm_causal_conv1d_fwd", "mssm_causal_conv1d_update", "causal_conv1d", "causal_conv1d_update",
    "mssm_selective_scan_bwd", "selective_scan_bwd",
    "KERNEL_KINDS",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
lib_path = os.path.join(_HERE, "libmssm.so")
if not os.path.exists(lib_path):
    raise ImportError(f"{lib_path} is missing: build it with `python selective_state_space_46_b200/build.py` "
                      "(nvcc, sm_100a); there is no fallback implementation")
_lib = ctypes.CDLL(lib_path)

MSSM_F32, MSSM_BF16 = 0, 1
MSSM_OK, MSSM_ERR_INVALID_ARG, MSSM_ERR_UNSUPPORTED, MSSM_ERR_CUDA, MSSM_ERR_TIMEOUT = 0, 1, 2, 3, 4
MSSM_OPT_FORCE_GENERAL_A, MSSM_OPT_CHUNK_LEN, MSSM_OPT_KERNEL_TIMING, MSSM_OPT_SCHEDULE = 1, 2, 3, 4
MSSM_OPT_DECODE_PATH = 5
MSSM_OPT_TEST_HOOKS = 6
MSSM_OPT_ROWS_PER_CTA = 7
MSSM_OPT_ROWS_PER_THREAD = 8
MSSM_DISC_EULER, MSSM_DISC_ZOH = 0, 1
SCHEDULES = {"forward": 1, "summaries+forward": 2, "chained": 3, "fused": 4, "split": 5}
DECODE_PATHS = {"stream": 1, "bulk_tile": 2, "per_row": 3}
KERNEL_KINDS = ("scan_chunk_state", "scan_out", "state_update", "conv", "scan_bwd")


class mssm_tensor(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int32), ("ndim", ctypes.c_int32),
                ("shape", ctypes.c_int64 * 4), ("stride", ctypes.c_int64 * 4)]


class mssm_scan_ext(ctypes.Structure):
    _fields_ = [("struct_size", ctypes.c_int32), ("discretization", ctypes.c_int32),
                ("h0", ctypes.POINTER(mssm_tensor)), ("cu_seqlens", ctypes.POINTER(mssm_tensor)),
                ("max_seqlen", ctypes.c_int64)]


_P = ctypes.POINTER(mssm_tensor)
_V = ctypes.c_void_p
_lib.mssm_selective_scan_fwd.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_int, _P, _P, _V]
_lib.mssm_selective_scan_fwd.restype = ctypes.c_int
_lib.mssm_selective_scan_fwd_ex.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_int,
                                            ctypes.POINTER(mssm_scan_ext), _P, _P, _V]
_lib.mssm_selective_scan_fwd_ex.restype = ctypes.c_int
_lib.mssm_selective_scan_fwd_noalloc.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_int, _P, _P, _V]
_lib.mssm_selective_scan_fwd_noalloc.restype = ctypes.c_int
_lib.mssm_state_update.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _P, _V]
_lib.mssm_state_update.restype = ctypes.c_int
_lib.mssm_state_update_ex.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_int, ctypes.c_int, _P, _V]
_lib.mssm_state_update_ex.restype = ctypes.c_int
_lib.mssm_selective_scan_bwd.argtypes = [_P] * 8 + [ctypes.c_int] + [_P] * 9 + [_V]
_lib.mssm_selective_scan_bwd.restype = ctypes.c_int
_lib.mssm_causal_conv1d_fwd.argtypes = [_P, _P, _P, _P, ctypes.c_int64, ctypes.c_int, _P, _V]
_lib.mssm_causal_conv1d_fwd.restype = ctypes.c_int
_lib.mssm_causal_conv1d_update.argtypes = [_P, _P, _P, _P, ctypes.c_int, _P, _V]
_lib.mssm_causal_conv1d_update.restype = ctypes.c_int
_lib.mssm_status_string.argtypes = [ctypes.c_int]
_lib.mssm_status_string.restype = ctypes.c_char_p
_lib.mssm_last_error.restype = ctypes.c_char_p
_lib.mssm_get_error.argtypes = [_V]
_lib.mssm_get_error.restype = ctypes.c_int
_lib.mssm_set_option.argtypes = [ctypes.c_int, ctypes.c_int64]
_lib.mssm_set_option.restype = ctypes.c_int
_lib.mssm_shutdown.restype = ctypes.c_int
_lib.mssm_version.restype = ctypes.c_char_p
_lib.mssm_kernel_stats.argtypes = [ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_int64),
                                   ctypes.POINTER(ctypes.c_double), ctypes.c_int]
_lib.mssm_kernel_stats.restype = ctypes.c_int
_lib.mssm_scan_plan.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int,
                                ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int64),
                                ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_int)]
_lib.mssm_scan_plan.restype = ctypes.c_int
_lib.mssm_scan_plan_packed.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int,
                                       ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int64),
                                       ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_int)]
_lib.mssm_scan_plan_packed.restype = ctypes.c_int


class mssm_scan_plan_info(ctypes.Structure):
    _fields_ = [("struct_size", ctypes.c_int32), ("schedule", ctypes.c_int32), ("rows_per_cta", ctypes.c_int32),
                ("rows_per_thread", ctypes.c_int32), ("chunk_len", ctypes.c_int64), ("n_chunks", ctypes.c_int64),
                ("grid", ctypes.c_int32), ("reserved", ctypes.c_int32)]


_lib.mssm_scan_plan_query.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int,
                                      ctypes.c_int, ctypes.POINTER(mssm_scan_plan_info)]
_lib.mssm_scan_plan_query.restype = ctypes.c_int


class MssmError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{mssm_status_string(status)}: {message}")
        self.status = status


MSSM_I32 = 2
_DT = {torch.float32: MSSM_F32, torch.bfloat16: MSSM_BF16, torch.int32: MSSM_I32}


def _desc(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if t.dim() > 4:
        raise ValueError("tensors have at most 4 dims")
    d = mssm_tensor()
    d.data = t.data_ptr() if t.numel() > 0 else None
    d.dtype = _DT.get(t.dtype, -1)
    d.ndim = t.dim()
    for i, (s, st) in enumerate(zip(t.shape, t.stride())):
        d.shape[i] = s
        d.stride[i] = st
    return ctypes.byref(d), d


def _ref(x):
    return None if x is None else x[0]


def _stream(stream, ref: torch.Tensor):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream(ref.device).cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _check(status: int):
    if status != MSSM_OK:
        raise MssmError(status, mssm_last_error())


def mssm_status_string(status: int) -> str:
    return _lib.mssm_status_string(status).decode()


def mssm_last_error() -> str:
    return _lib.mssm_last_error().decode()


def mssm_version() -> str:
    return _lib.mssm_version().decode()


def mssm_set_option(option: int, value: int) -> None:
    _check(_lib.mssm_set_option(option, value))


def mssm_shutdown() -> None:
    _check(_lib.mssm_shutdown())


def mssm_kernel_stats(reset: bool = False) -> dict:
    """Launch counts and (when MSSM_OPT_KERNEL_TIMING is on) timed launches and summed ms, per kernel kind."""
    n = len(KERNEL_KINDS)
    launches = (ctypes.c_int64 * n)()
    timed = (ctypes.c_int64 * n)()
    ms = (ctypes.c_double * n)()
    _check(_lib.mssm_kernel_stats(launches, timed, ms, int(reset)))
    return {k: {"launches": launches[i], "timed": timed[i], "ms": ms[i]} for i, k in enumerate(KERNEL_KINDS)}


def mssm_scan_plan(Bt: int, D: int, L: int, sm_count: int = 0, total_len: int = -1, io_dtype: str = "bf16") -> dict:
    """Launch plan of the scan for a [Bt, D, L] problem, or for Bt packed sequences of at most
    L steps summing to ``total_len``, with ``io_dtype`` ('bf16' or 'f32') I/O (mssm_scan_plan_query;
    host only, launches nothing)."""
    info = mssm_scan_plan_info()
    info.struct_size = ctypes.sizeof(mssm_scan_plan_info)
    dt = {"bf16": MSSM_BF16, "f32": MSSM_F32}[io_dtype]
    _check(_lib.mssm_scan_plan_query(Bt, D, L, total_len, dt, sm_count, ctypes.byref(info)))
    return {"rows_per_cta": info.rows_per_cta, "rows_per_thread": info.rows_per_thread,
            "chunk_len": info.chunk_len, "n_chunks": info.n_chunks, "grid": info.grid,
            "schedule": ("forward", "summaries+forward", "chained", "fused", "split")[info.schedule]}


def mssm_get_error(stream=None) -> None:
    s = ctypes.c_void_p(None) if stream is None else (
        ctypes.c_void_p(stream.cuda_stream) if isinstance(stream, torch.cuda.Stream) else ctypes.c_void_p(int(stream)))
    _check(_lib.mssm_get_error(s))


def mssm_selective_scan_fwd(u, delta, A, B, C, D, z, delta_bias, softplus_flag, out, last_state,
                            stream=None) -> None:
    """Marshal torch tensors into ``mssm_selective_scan_fwd`` (see include/mssm.h)."""
    ds = [_desc(t) for t in (u, delta, A, B, C, D, z, delta_bias, out, last_state)]
    _check(_lib.mssm_selective_scan_fwd(*[_ref(x) for x in ds[:8]], int(softplus_flag),
                                        _ref(ds[8]), _ref(ds[9]), _stream(stream, u)))


def mssm_selective_scan_fwd_ex(u, delta, A, B, C, D, z, delta_bias, softplus_flag, out, last_state,
                               h0=None, discretization=MSSM_DISC_EULER, cu_seqlens=None, max_seqlen=0,
                               stream=None) -> None:
    """Marshal torch tensors into ``mssm_selective_scan_fwd_ex``: the scan from an initial
    state ``h0`` (None: zero) with the given discretisation, over packed sequences when
    ``cu_seqlens`` (int32 device offsets) and ``max_seqlen`` are given (see include/mssm.h)."""
    ds = [_desc(t) for t in (u, delta, A, B, C, D, z, delta_bias, out, last_state)]
    dh = _desc(h0)
    dc = _desc(cu_seqlens)
    ext = mssm_scan_ext(ctypes.sizeof(mssm_scan_ext), int(discretization),
                        None if dh is None else ctypes.pointer(dh[1]),
                        None if dc is None else ctypes.pointer(dc[1]), int(max_seqlen))
    _check(_lib.mssm_selective_scan_fwd_ex(*[_ref(x) for x in ds[:8]], int(softplus_flag), ctypes.byref(ext),
                                           _ref(ds[8]), _ref(ds[9]), _stream(stream, u)))


def mssm_selective_scan_fwd_noalloc(u, delta, A, B, C, D, z, delta_bias, softplus_flag, out, last_state,
                                    stream=None) -> None:
    """Marshal torch tensors into ``mssm_selective_scan_fwd_noalloc``: the same scan for
    callers that cannot allocate device memory during the call (see include/mssm.h)."""
    ds = [_desc(t) for t in (u, delta, A, B, C, D, z, delta_bias, out, last_state)]
    _check(_lib.mssm_selective_scan_fwd_noalloc(*[_ref(x) for x in ds[:8]], int(softplus_flag),
                                                _ref(ds[8]), _ref(ds[9]), _stream(stream, u)))


def mssm_state_update(state, x, dt, A, B, C, D, z, out, stream=None) -> None:
    """Marshal torch tensors into ``mssm_state_update`` (state updated in place)."""
    ds = [_desc(t) for t in (state, x, dt, A, B, C, D, z, out)]
    _check(_lib.mssm_state_update(*[_ref(v) for v in ds], _stream(stream, x)))


def mssm_state_update_ex(state, x, dt, A, B, C, D, z, dt_bias, softplus_flag, out,
                         discretization=MSSM_DISC_EULER, stream=None) -> None:
    """Marshal torch tensors into ``mssm_state_update_ex`` (state updated in place)."""
    ds = [_desc(t) for t in (state, x, dt, A, B, C, D, z, dt_bias)]
    do = _desc(out)
    _check(_lib.mssm_state_update_ex(*[_ref(v) for v in ds], int(softplus_flag), int(discretization), _ref(do),
                                     _stream(stream, x)))


def mssm_selective_scan_bwd(u, delta, A, B, C, D, z, delta_bias, softplus_flag, dout, du, ddelta, dA, dB, dC,
                            dD, dz, ddelta_bias, stream=None) -> None:
    """Marshal torch tensors into ``mssm_selective_scan_bwd`` (see include/mssm.h)."""
    ds = [_desc(t) for t in (u, delta, A, B, C, D, z, delta_bias)]
    gs = [_desc(t) for t in (dout, du, ddelta, dA, dB, dC, dD, dz, ddelta_bias)]
    _check(_lib.mssm_selective_scan_bwd(*[_ref(x) for x in ds], int(softplus_flag), *[_ref(x) for x in gs],
                                        _stream(stream, u)))


def selective_scan_bwd(u, delta, A, B, C, D=None, z=None, delta_bias=None, softplus=True, dout=None,
                       stream=None) -> dict:
    """Allocate the gradients with torch and run the backward scan on the GPU."""
    f32 = dict(device=u.device, dtype=torch.float32)
    g = dict(du=torch.empty_like(u), ddelta=torch.empty_like(u), dA=torch.empty(A.shape, **f32),
             dB=torch.empty(B.shape, **f32), dC=torch.empty(C.shape, **f32),
             dD=None if D is None else torch.empty(D.shape, **f32),
             dz=None if z is None else torch.empty_like(z),
             ddelta_bias=None if delta_bias is None else torch.empty(delta_bias.shape, **f32))
    mssm_selective_scan_bwd(u, delta, A, B, C, D, z, delta_bias, softplus, dout, g["du"], g["ddelta"], g["dA"],
                            g["dB"], g["dC"], g["dD"], g["dz"], g["ddelta_bias"], stream)
    return g


def mssm_causal_conv1d_fwd(x, weight, bias, out, cu_seqlens=None, max_seqlen=0, silu_flag=True,
                           stream=None) -> None:
    """Marshal torch tensors into ``mssm_causal_conv1d_fwd`` (see include/mssm.h)."""
    ds = [_desc(t) for t in (x, weight, bias, cu_seqlens)]
    _check(_lib.mssm_causal_conv1d_fwd(*[_ref(v) for v in ds], int(max_seqlen), int(silu_flag), _ref(_desc(out)),
                                       _stream(stream, x)))


def mssm_causal_conv1d_update(conv_state, x, weight, bias, out, silu_flag=True, stream=None) -> None:
    """Marshal torch tensors into ``mssm_causal_conv1d_update`` (conv_state updated in place)."""
    ds = [_desc(t) for t in (conv_state, x, weight, bias)]
    _check(_lib.mssm_causal_conv1d_update(*[_ref(v) for v in ds], int(silu_flag), _ref(_desc(out)),
                                          _stream(stream, x)))


# --------------------------------------------------------------------------
# allocation conveniences (torch allocates; the library computes)
# --------------------------------------------------------------------------

def causal_conv1d(x, weight, bias=None, silu=True, cu_seqlens=None, max_seqlen=None, out=None,
                  stream=None) -> torch.Tensor:
    """Causal depthwise conv1d (+ SiLU) of ``x`` [Bt, D, L] on the GPU; returns ``out``."""
    if not x.is_cuda:
        raise ValueError("causal_conv1d runs on CUDA tensors only")
    if out is None:
        out = torch.empty_like(x, memory_format=torch.contiguous_format)
    if cu_seqlens is not None and max_seqlen is None:
        max_seqlen = int((cu_seqlens[1:] - cu_seqlens[:-1]).max().item()) if cu_seqlens.numel() > 1 else 0
    mssm_causal_conv1d_fwd(x, weight, bias, out, cu_seqlens, max_seqlen or 0, silu, stream)
    return out


def causal_conv1d_update(conv_state, x, weight, bias=None, silu=True, out=None, stream=None) -> torch.Tensor:
    """One decode step of the conv on the GPU (``conv_state`` updated in place); returns ``out``."""
    if out is None:
        out = torch.empty_like(x, memory_format=torch.contiguous_format)
    mssm_causal_conv1d_update(conv_state, x, weight, bias, out, silu, stream)
    return out

def selective_scan_fwd(u, delta, A, B, C, D=None, z=None, delta_bias=None, softplus=True,
                       out=None, last_state=None, return_last_state=True, h0=None, zoh=False,
                       cu_seqlens=None, max_seqlen=None,
                       stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Allocate ``out`` (and ``last_state``) with torch and run the scan on the GPU
    (from ``h0`` when given; zero-order-hold input term when ``zoh``; packed sequences
    when ``cu_seqlens`` is given, with ``max_seqlen`` read back from it if omitted)."""
    if not u.is_cuda:
        raise ValueError("selective_scan_fwd runs on CUDA tensors only")
    if out is None:
        out = torch.empty_like(u, memory_format=torch.contiguous_format)
    nstate = u.shape[0] if cu_seqlens is None else cu_seqlens.shape[0] - 1
    if last_state is None and return_last_state:
        last_state = torch.empty(nstate, u.shape[1], A.shape[1], device=u.device, dtype=torch.float32)
    if cu_seqlens is not None and max_seqlen is None:
        max_seqlen = int((cu_seqlens[1:] - cu_seqlens[:-1]).max().item()) if nstate > 0 else 0
    if h0 is None and not zoh and cu_seqlens is None:
        mssm_selective_scan_fwd(u, delta, A, B, C, D, z, delta_bias, softplus, out, last_state, stream)
    else:
        mssm_selective_scan_fwd_ex(u, delta, A, B, C, D, z, delta_bias, softplus, out, last_state, h0=h0,
                                   discretization=MSSM_DISC_ZOH if zoh else MSSM_DISC_EULER,
                                   cu_seqlens=cu_seqlens, max_seqlen=max_seqlen or 0, stream=stream)
    return out, last_state


def state_update(state, x, dt, A, B, C, D=None, z=None, dt_bias=None, softplus=True, out=None,
                 zoh=False, stream=None) -> torch.Tensor:
    """Run one decode step on the GPU (``state`` updated in place); returns ``out``."""
    if not x.is_cuda:
        raise ValueError("state_update runs on CUDA tensors only")
    if out is None:
        out = torch.empty_like(x, memory_format=torch.contiguous_format)
    mssm_state_update_ex(state, x, dt, A, B, C, D, z, dt_bias, softplus, out,
                         discretization=MSSM_DISC_ZOH if zoh else MSSM_DISC_EULER, stream=stream)
    return out
