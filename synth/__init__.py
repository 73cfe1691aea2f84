"""Seeded synthetic inputs for the selective scan and the decode state update.

This module is shared by the CPU oracle tests and the CUDA path's tests and
benchmark. It only draws random numbers and rounds them to the storage
precision; it holds none of the method's arithmetic (no softplus, no
discretisation, no recurrence).

Input recipe (one generator stream per tensor, so a tensor's values do not
depend on which other tensors were drawn):

* ``A[d, n] = -(n + 1)``: the S4D-real initialisation that the page
  "Linear Attention vs Softmax Attention" builds in its Implementation section
  (``A_log = log(arange(1..N))`` repeated over channels, ``A = -exp(A_log)``).
* ``D[d] = 1``: the same listing initialises the skip parameter to ones.
* ``delta_raw ~ N(0, 1)``; a per-channel bias ``b_d = log(expm1(s_d))`` with
  ``log s_d ~ U(log lo, log hi)`` so that ``softplus(b_d)`` (the step at
  ``delta_raw = 0``) is log-uniform in ``[lo, hi]``.  ``[lo, hi]`` is
  ``[1e-3, 1e-1]`` for the prefill shapes and ``[1e-4, 1e-2]`` for the
  long-context shape.
* ``u, z ~ N(0, 1)`` with layout ``[batch, channels, length]``;
  ``B, C ~ N(0, 1)`` with layout ``[batch, N, length]``.
* decode: ``state ~ N(0, 0.1**2)`` ``[batch, channels, N]`` fp32; ``x, dt, z``
  ``[batch, channels]`` and ``B, C`` ``[batch, N]``, all ``N(0, 1)``.

Values stored as bf16 are rounded to nearest-even from the fp32 draw; both
the CUDA path and the oracle consume the same rounded values (the oracle
widens them to fp64 exactly).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np

N_STATE = 16

# --------------------------------------------------------------------------
# bf16 storage helpers (bit manipulation only)
# --------------------------------------------------------------------------


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (round to nearest, ties to even); returns uint16 bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    bits = x.view(np.uint32)
    # NaN stays NaN (quiet); everything else rounds to nearest even.
    lsb = (bits >> 16) & np.uint32(1)
    rounded = (bits + np.uint32(0x7FFF) + lsb) >> 16
    nan = np.isnan(x)
    if nan.any():
        rounded = np.where(nan, (bits >> 16) | np.uint32(0x40), rounded)
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns (uint16) to fp32 exactly."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def to_f64(a: Optional[np.ndarray], dtype: str) -> Optional[np.ndarray]:
    """Widen a stored tensor (``dtype`` 'bf16' = uint16 bits, or 'f32') to fp64."""
    if a is None:
        return None
    if dtype == "bf16" and a.dtype == np.uint16:
        return bf16_bits_to_f32(a).astype(np.float64)
    return np.asarray(a, dtype=np.float64)


# --------------------------------------------------------------------------
# generators
# --------------------------------------------------------------------------


def _rng(seed: int, stream: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, stream])))


def _normal(seed: int, stream: int, shape, std: float = 1.0) -> np.ndarray:
    out = _rng(seed, stream).standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        out *= np.float32(std)
    return out


def _store(x: np.ndarray, dtype: str) -> np.ndarray:
    return f32_to_bf16_bits(x) if dtype == "bf16" else np.ascontiguousarray(x, np.float32)


@dataclasses.dataclass
class ScanInputs:
    """One selective-scan problem. Tensors in ``io_dtype`` are uint16 bf16 bits
    (``io_dtype == 'bf16'``) or float32; ``A``, ``D``, ``delta_bias`` are float32."""

    batch: int
    dim: int
    length: int
    io_dtype: str
    u: np.ndarray            # [batch, dim, length]
    delta: np.ndarray        # [batch, dim, length] (pre-softplus step)
    A: np.ndarray            # [dim, N] f32
    B: np.ndarray            # [batch, N, length]
    C: np.ndarray            # [batch, N, length]
    D: Optional[np.ndarray]  # [dim] f32
    z: Optional[np.ndarray]  # [batch, dim, length]
    delta_bias: Optional[np.ndarray]  # [dim] f32
    softplus: bool
    cu_seqlens: Optional[np.ndarray] = None  # [S + 1] int32 offsets when the batch row packs S sequences

    def f64(self, name: str) -> Optional[np.ndarray]:
        a = getattr(self, name)
        if name in ("A", "D", "delta_bias"):
            return None if a is None else np.asarray(a, np.float64)
        return to_f64(a, self.io_dtype)


@dataclasses.dataclass
class DecodeInputs:
    """One decode step batch: ``state`` f32 [batch, dim, N]; the rest in ``io_dtype``."""

    batch: int
    dim: int
    io_dtype: str
    state: np.ndarray        # [batch, dim, N] f32
    x: np.ndarray            # [batch, dim]
    dt: np.ndarray           # [batch, dim]
    A: np.ndarray            # [dim, N] f32
    B: np.ndarray            # [batch, N]
    C: np.ndarray            # [batch, N]
    D: Optional[np.ndarray]  # [dim] f32
    z: Optional[np.ndarray]  # [batch, dim]
    dt_bias: Optional[np.ndarray]  # [dim] f32
    softplus: bool

    def f64(self, name: str) -> Optional[np.ndarray]:
        a = getattr(self, name)
        if name in ("A", "D", "dt_bias", "state"):
            return None if a is None else np.asarray(a, np.float64)
        return to_f64(a, self.io_dtype)


def s4d_real_A(dim: int, n_state: int = N_STATE) -> np.ndarray:
    """``A[d, n] = -(n + 1)`` as float32."""
    return -np.tile(np.arange(1, n_state + 1, dtype=np.float32), (dim, 1))


def log_uniform_bias(seed: int, dim: int, lo: float, hi: float) -> np.ndarray:
    """Per-channel bias whose softplus is log-uniform in ``[lo, hi]``."""
    s = np.exp(_rng(seed, 7).uniform(math.log(lo), math.log(hi), size=dim))
    return np.log(np.expm1(s)).astype(np.float32)


def make_scan_inputs(batch: int, dim: int, length: int, *, io_dtype: str = "bf16",
                     seed: int = 0, delta_range=(1e-3, 1e-1), with_z: bool = True,
                     with_D: bool = True, with_bias: bool = True, softplus: bool = True,
                     n_state: int = N_STATE) -> ScanInputs:
    shp = (batch, dim, length)
    u = _store(_normal(seed, 1, shp), io_dtype)
    delta = _store(_normal(seed, 2, shp), io_dtype)
    B = _store(_normal(seed, 3, (batch, n_state, length)), io_dtype)
    C = _store(_normal(seed, 4, (batch, n_state, length)), io_dtype)
    z = _store(_normal(seed, 5, shp), io_dtype) if with_z else None
    A = s4d_real_A(dim, n_state)
    D = np.ones(dim, np.float32) if with_D else None
    bias = log_uniform_bias(seed, dim, *delta_range) if with_bias else None
    return ScanInputs(batch, dim, length, io_dtype, u, delta, A, B, C, D, z, bias, softplus)


def make_decode_inputs(batch: int, dim: int, *, io_dtype: str = "bf16", seed: int = 0,
                       with_z: bool = True, with_D: bool = True, n_state: int = N_STATE,
                       dt_bias: bool = False, delta_range=(1e-3, 1e-1),
                       softplus: bool = True, state_std: float = 0.1,
                       step_stream: int = 0) -> DecodeInputs:
    """``step_stream`` selects an independent draw of the per-token tensors
    (x, dt, z, B, C) while the state and the parameters stay the same."""
    k = 100 + 10 * step_stream
    state = _normal(seed, 50, (batch, dim, n_state), std=state_std)
    x = _store(_normal(seed, k + 1, (batch, dim)), io_dtype)
    dt = _store(_normal(seed, k + 2, (batch, dim)), io_dtype)
    B = _store(_normal(seed, k + 3, (batch, n_state)), io_dtype)
    C = _store(_normal(seed, k + 4, (batch, n_state)), io_dtype)
    z = _store(_normal(seed, k + 5, (batch, dim)), io_dtype) if with_z else None
    A = s4d_real_A(dim, n_state)
    D = np.ones(dim, np.float32) if with_D else None
    bias = log_uniform_bias(seed, dim, *delta_range) if dt_bias else None
    return DecodeInputs(batch, dim, io_dtype, state, x, dt, A, B, C, D, z, bias, softplus)


# --------------------------------------------------------------------------
# the five workloads
# --------------------------------------------------------------------------

WORKLOADS = {
    # small oracle-scale problem, fp32 I/O, D = 1, no gate
    "scan_f32_1x64x256": dict(kind="scan", batch=1, dim=64, length=256, io_dtype="f32",
                              delta_range=(1e-3, 1e-1), with_z=False),
    # Mamba-130M-shaped prefill
    "scan_bf16_2x1536x2048": dict(kind="scan", batch=2, dim=1536, length=2048, io_dtype="bf16",
                                  delta_range=(1e-3, 1e-1), with_z=True),
    # Mamba-2.8B-shaped prefill
    "scan_bf16_8x5120x4096": dict(kind="scan", batch=8, dim=5120, length=4096, io_dtype="bf16",
                                  delta_range=(1e-3, 1e-1), with_z=True),
    # long context, slow decay spanning many chunks
    "scan_bf16_1x2048x131072": dict(kind="scan", batch=1, dim=2048, length=131072,
                                    io_dtype="bf16", delta_range=(1e-4, 1e-2), with_z=True),
    # the long-context shape cut to 16384 steps (inputs still larger than the L2): the case
    # the full ncu captures of the scan kernels run on
    "scan_bf16_1x2048x16384": dict(kind="scan", batch=1, dim=2048, length=16384,
                                   io_dtype="bf16", delta_range=(1e-4, 1e-2), with_z=True),
    # the causal conv1d (K = 4) + SiLU that produces u, at the Mamba-130M prefill shape
    "conv_bf16_2x1536x2048": dict(kind="conv", batch=2, dim=1536, length=2048, io_dtype="bf16", K=4),
    # the same conv at the Mamba-2.8B prefill shape (671 MB of traffic per call)
    "conv_bf16_8x5120x4096": dict(kind="conv", batch=8, dim=5120, length=4096, io_dtype="bf16", K=4),
    # packed variable-length prefill: 32 sequences of 64..4096 steps (log-uniform) over
    # Mamba-130M's 1536 channels, concatenated along L without padding
    "scan_varlen_bf16_1536x32seq": dict(kind="scan", batch=1, dim=1536, nseq=32, len_range=(64, 4096),
                                        io_dtype="bf16", delta_range=(1e-3, 1e-1), with_z=True),
    # one-token decode state update, timed over successive steps
    "decode_bf16_256x5120": dict(kind="decode", batch=256, dim=5120, io_dtype="bf16"),
}


@dataclasses.dataclass
class ConvInputs:
    """One causal conv1d problem: ``x`` [batch, dim, length] in ``io_dtype`` storage,
    ``weight`` [dim, K] and ``bias`` [dim] float32."""
    batch: int
    dim: int
    length: int
    io_dtype: str
    x: np.ndarray
    weight: np.ndarray
    bias: np.ndarray


def make_conv_inputs(batch: int, dim: int, length: int, K: int = 4, *, io_dtype: str = "bf16",
                     seed: int = 0) -> ConvInputs:
    """x ~ N(0, 1); weight ~ N(0, 1/K) (unit-variance output before SiLU); bias ~ N(0, 0.25)."""
    x = _store(_normal(seed, 20, (batch, dim, length)), io_dtype)
    w = _normal(seed, 21, (dim, K), std=1.0 / np.sqrt(K)).astype(np.float32)
    b = _normal(seed, 22, (dim,), std=0.5).astype(np.float32)
    return ConvInputs(batch, dim, length, io_dtype, x, w, b)


def varlen_lengths(nseq: int, lo: int, hi: int, seed: int = 0) -> np.ndarray:
    """Sequence lengths, log-uniform in [lo, hi], from their own stream."""
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, 99])))
    return np.exp(rng.uniform(np.log(lo), np.log(hi), size=nseq)).astype(np.int64)


def workload_inputs(name: str, seed: int = 0, batch: Optional[int] = None,
                    step_stream: int = 0):
    """Inputs of a named workload; ``batch`` overrides the batch size (shards, downscaled checks)."""
    w = dict(WORKLOADS[name])
    kind = w.pop("kind")
    if batch is not None:
        w["batch"] = batch
    if kind == "scan" and "nseq" in w:
        lengths = varlen_lengths(w["nseq"], *w["len_range"], seed=seed)
        inp = make_scan_inputs(1, w["dim"], int(lengths.sum()), io_dtype=w["io_dtype"], seed=seed,
                               delta_range=w["delta_range"], with_z=w["with_z"])
        inp.cu_seqlens = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
        return inp
    if kind == "scan":
        return make_scan_inputs(w["batch"], w["dim"], w["length"], io_dtype=w["io_dtype"],
                                seed=seed, delta_range=w["delta_range"], with_z=w["with_z"])
    if kind == "conv":
        return make_conv_inputs(w["batch"], w["dim"], w["length"], w["K"], io_dtype=w["io_dtype"], seed=seed)
    return make_decode_inputs(w["batch"], w["dim"], io_dtype=w["io_dtype"], seed=seed,
                              step_stream=step_stream)
