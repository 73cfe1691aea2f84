"""Benchmark of the B200 selective scan (and its decode step) through the C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl mssm|reference]

One step is one pass of the hot path over one batch of synthetic input:
for the scan workloads, one mssm_selective_scan_fwd call (softplus,
discretisation, recurrence, readout, D skip, gate, store, final state); for the
decode workload, one mssm_state_update call.  Inputs are resident in HBM when
the timed region starts.  The timed steps rotate through enough copies of the
workload's buffers to cover 4x the L2 (one copy when a single set is that
large), so no step finds its inputs in L2 and the write-back of one step's
dirty lines is paid inside the steps that follow; only a workload too small for
that (over 32 copies) flushes the L2 (a 256 MiB write) before each step
instead, outside the step's event bracket.  The K timed steps are captured into
one CUDA graph so host launch overhead cannot leak into device time: one event
pair brackets the K back-to-back steps (an event between steps drains the GPU
and costs several microseconds, a third of a 10 us step), or, with the L2
flushed between steps, one pair per step.  For the roofline the dominant kernel
is timed on its own, with events around each launch; a step that is a single
launch of it takes the step time instead, which those events would inflate.

Multi-GPU (``torchrun --nproc-per-node N bench.py --gpus N``): rows of the scan
are independent, so every rank runs its own batch of the same shape (weak
scaling, no collective on the data path); the step time is the max over ranks.

``--impl reference`` times the fp64 CPU oracle on the host cores instead, on a
bounded sample of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "selective-scan B·D·L elems/s and achieved HBM GB/s vs ~8 TB/s B200 peak"
DECODE_METRIC = "selective state update rows/s and achieved HBM GB/s vs ~8 TB/s B200 peak"
CONV_METRIC = "causal conv1d + SiLU B·D·L elems/s and achieved HBM GB/s vs ~8 TB/s B200 peak"
BWD_METRIC = "selective-scan backward B·D·L elems/s and achieved HBM GB/s vs ~8 TB/s B200 peak"
BWD_FLOP_PER_STATE = 22  # the forward recomputed (6) and the reverse step (16) per (element, state)
DEFAULT_WORKLOAD = "scan_bf16_1x2048x131072"
L2_FLUSH_BYTES = 256 << 20
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
N_STATE = 16


# --------------------------------------------------------------------------
# host-side helpers (also exercised by the multi-rank CPU tests)
# --------------------------------------------------------------------------

def rank_seed(rank: int, base: int = 0) -> int:
    """Each rank draws its own batch: seed = base + rank."""
    return base + rank


def reduce_max(value: float, dist=None) -> float:
    """Max of a float over all ranks (identity without a process group)."""
    if dist is None or not dist.is_available() or not dist.is_initialized():
        return value
    import torch
    backend = dist.get_backend()
    dev = torch.device("cuda", torch.cuda.current_device()) if backend == "nccl" else torch.device("cpu")
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def scan_algorithmic_bytes(batch, dim, length, io_bytes, has_z=True, has_D=True, has_bias=True,
                           last_state=True) -> int:
    """Bytes the scan must move once: u, delta, z, y per element; B, C per (batch, step);
    A, D, bias per channel; the final fp32 state per row."""
    elems = batch * dim * length
    b = elems * io_bytes * (3 + (1 if has_z else 0))            # u, delta, out (+ z)
    b += 2 * batch * N_STATE * length * io_bytes                 # B, C
    b += dim * (N_STATE * 4 + (4 if has_D else 0) + (4 if has_bias else 0))
    if last_state:
        b += batch * dim * N_STATE * 4
    return b


FP32_LANES_PER_SM = 128      # FP32 FMA lanes per SM (4 sub-partitions x 32)
FLOP_PER_STATE = 6           # per (element, state): decay multiply, (delta u) B_n multiply,
                             # FMA of the state update, FMA of the readout (an FMA = 2 flop)


def algorithmic_flops(units: int) -> int:
    """FP32 flops the method needs per scan element or decode row: 16 states x 6
    (transcendentals, which run on the SFU, are not counted)."""
    return units * N_STATE * FLOP_PER_STATE


def fp32_peak_tflops(sm_count: int, sm_mhz: float) -> float:
    """FP32 FMA-pipe peak from unit counts and clock: SMs x 128 lanes x 2 flop x clock."""
    return sm_count * FP32_LANES_PER_SM * 2 * sm_mhz * 1e6 / 1e12


def binding_roofline(alg_bytes: float, alg_flops: float, ms: float, hbm_gbs: float, alu_tflops: float) -> dict:
    """Roofline of one launch: the bound is whichever of HBM bytes / peak bandwidth and
    FP32 flops / peak FLOP rate takes longer; achieved and frac are against that bound,
    the other bound's fraction is kept beside it."""
    t_hbm = alg_bytes / (hbm_gbs * 1e9)
    t_alu = alg_flops / (alu_tflops * 1e12)
    gbs = alg_bytes / (ms / 1e3) / 1e9
    tfl = alg_flops / (ms / 1e3) / 1e12
    hbm = {"achieved": gbs, "peak": hbm_gbs, "unit": "GB/s", "frac": gbs / hbm_gbs}
    alu = {"achieved": tfl, "peak": alu_tflops, "unit": "TFLOP/s", "frac": tfl / alu_tflops}
    if t_alu > t_hbm:
        return {"bound": "alu", **alu, "other": {"bound": "hbm", **hbm}}
    return {"bound": "hbm", **hbm, "other": {"bound": "alu", **alu}}


def ring_size(set_bytes: int, l2_bytes: int, max_sets: int = 32) -> int:
    """Number of input/output buffer sets the timed steps rotate through so that no
    step finds its data in L2: one set when a set alone is 4x the L2, else enough sets
    to cover 4x the L2; 0 (flush the L2 between steps instead) if that needs more than
    max_sets."""
    if set_bytes >= 4 * l2_bytes:
        return 1
    r = -(-4 * l2_bytes // max(set_bytes, 1))
    return r if r <= max_sets else 0


def decode_algorithmic_bytes(batch, dim, io_bytes, has_z=True, has_D=True) -> int:
    """Per decode step: state read + write (fp32), x, dt, (z), y per row; B, C per batch; A, D per channel."""
    rows = batch * dim
    b = rows * N_STATE * 4 * 2
    b += rows * io_bytes * (3 + (1 if has_z else 0))
    b += 2 * batch * N_STATE * io_bytes
    b += dim * (N_STATE * 4 + (4 if has_D else 0))
    return b


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def max_sm_mhz(default: float = 1965.0) -> float:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["sm_max_mhz"])
    except Exception:
        return default


KERNEL_SOURCES = {
    "scan_out": ("device_common.cuh", "scan.cuh", "scan.cu", "scan_zoh.cu", "scan_dispatch.cuh"),
    "scan_chunk_state": ("device_common.cuh", "scan.cuh", "scan.cu", "scan_zoh.cu", "scan_dispatch.cuh"),
    "state_update": ("device_common.cuh", "decode.cuh", "decode.cu"),
    "conv": ("device_common.cuh", "conv.cuh", "conv.cu"),
    "scan_bwd": ("device_common.cuh", "bwd.cuh", "bwd.cu"),
}


def kernel_source_hash(kernel: str | None = None) -> str:
    """Hash of the device sources a kernel is built from (all of csrc/ when kernel is None)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "selective_state_space_46_b200", "csrc")
    names = KERNEL_SOURCES.get(kernel) if kernel else None
    for name in sorted(names or os.listdir(csrc)):
        if name.endswith((".cu", ".cuh", ".h")):
            with open(os.path.join(csrc, name), "rb") as f:
                h.update(name.encode() + b"\0" + f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str, plan: str | None = None):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on the
    kernel's current sources (and, for a scan, the same launch plan)."""
    p = os.path.join(ROOT, "profiles", f"traffic_{kernel}_{workload}.txt")
    if not os.path.exists(p):
        return None, None
    text = open(p).read()
    m_b = re.search(r"dram_bytes_per_launch\s*=\s*([0-9.eE+]+)", text)
    m_h = re.search(r"source_hash\s*=\s*([0-9a-f]+)", text)
    if not m_b or not m_h:
        return None, None
    if m_h.group(1) != kernel_source_hash(kernel):
        return None, "stale: kernel sources changed since the capture"
    m_p = re.search(r"plan\s*=\s*(.+)", text)
    if plan is not None and (not m_p or m_p.group(1).strip() != plan):
        return None, "stale: launch plan changed since the capture"
    scale = re.search(r"scale_to_full\s*=\s*([0-9.eE+]+)", text)
    val = float(m_b.group(1)) * (float(scale.group(1)) if scale else 1.0)
    return val, os.path.relpath(p, ROOT)


def recorded_step_traffic(kernel: str, workload: str, plan: str | None = None):
    """DRAM bytes of a whole step (every kernel of it), when the same summary recorded them."""
    val, src = recorded_traffic(kernel, workload, plan)
    if val is None:
        return None
    m_s = re.search(r"step_dram_bytes\s*=\s*([0-9.eE+]+)", open(os.path.join(ROOT, src)).read())
    return float(m_s.group(1)) if m_s else None


def plan_string(plan: dict | None) -> str | None:
    if not plan:
        return None
    return (f"{plan['schedule']} rows_per_cta={plan['rows_per_cta']} rows_per_thread={plan.get('rows_per_thread', 1)} "
            f"chunk_len={plan['chunk_len']} n_chunks={plan['n_chunks']}")


class ClockSampler:
    """Samples SM clocks and throttle reasons with nvidia-smi while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self._t = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return self
        self._t = threading.Thread(target=self._read, daemon=True)
        self._t.start()
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self._t:
            self._t.join(timeout=2)
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# --------------------------------------------------------------------------
# reference arm: the fp64 CPU oracle on the host cores
# --------------------------------------------------------------------------

def oracle_sample(workload: str, rows: int, zoh: bool = False, backward: bool = False):
    """A bounded sample of the workload for the CPU oracle: the first ``rows`` channels of batch 0
    (of every packed sequence, for a packed workload)."""
    import oracle
    inp = synth.workload_inputs(workload)
    if isinstance(inp, synth.ScanInputs):
        d = min(rows, inp.dim)
        args = dict(u=inp.f64("u")[:1, :d], delta=inp.f64("delta")[:1, :d], A=inp.f64("A")[:d],
                    B=inp.f64("B")[:1], C=inp.f64("C")[:1], D=None if inp.D is None else inp.f64("D")[:d],
                    z=None if inp.z is None else inp.f64("z")[:1, :d],
                    delta_bias=None if inp.delta_bias is None else inp.f64("delta_bias")[:d],
                    softplus=inp.softplus, zoh=zoh)
        units = d * inp.length
        disc = ", zero-order hold" if zoh else ""
        if backward:
            dout = np.random.default_rng(7).standard_normal(args["u"].shape)
            bargs = {k: v for k, v in args.items() if k != "zoh"}
            desc = f"backward, batch 0, channels 0..{d - 1}, all {inp.length} steps ({units} elements, serial)"
            return (lambda: oracle.scan_bwd(dout=dout, **bargs)), units, desc
        if inp.cu_seqlens is not None:
            cu = inp.cu_seqlens
            desc = (f"channels 0..{d - 1} of all {len(cu) - 1} packed sequences ({units} elements{disc})")
            return (lambda: oracle.scan_varlen(cu_seqlens=cu, **args)), units, desc
        desc = f"batch 0, channels 0..{d - 1}, all {inp.length} steps ({units} elements{disc})"
        return (lambda: oracle.scan(**args)), units, desc
    if isinstance(inp, synth.ConvInputs):
        d = min(rows, inp.dim)
        x = synth.to_f64(inp.x[:1, :d], inp.io_dtype)
        w, bias = inp.weight[:d].astype(np.float64), inp.bias[:d].astype(np.float64)
        units = d * inp.length
        return ((lambda: oracle.causal_conv1d(x, w, bias, True)), units,
                f"batch 0, channels 0..{d - 1}, all {inp.length} steps ({units} elements)")
    b = max(1, min(inp.batch, rows // inp.dim if rows >= inp.dim else 1))
    args = dict(state=inp.state[:b], x=inp.f64("x")[:b], dt=inp.f64("dt")[:b], A=inp.f64("A"),
                B=inp.f64("B")[:b], C=inp.f64("C")[:b], D=inp.f64("D"), z=inp.f64("z")[:b],
                dt_bias=None, softplus=inp.softplus)
    units = b * inp.dim
    return (lambda: oracle.state_update(**args)), units, f"batches 0..{b - 1} ({units} rows)"


def cpu_baseline(workload: str, budget_s: float = 10.0, zoh: bool = False, backward: bool = False):
    import oracle
    is_scan = WORKLOADS_KIND[workload] in ("scan", "conv")
    rows = (64 if backward else 512) if is_scan else 256 * 5120
    fn, units, desc = oracle_sample(workload, rows, zoh, backward)
    fn()  # build + warm
    t0 = time.perf_counter()
    n = 0
    while True:
        fn()
        n += 1
        el = time.perf_counter() - t0
        if el >= budget_s or n >= 10000:
            break
    return {"value": units * n / el, "unit": "elems/s" if is_scan else "rows/s",
            "cores": 1 if backward else oracle.num_threads(),
            "kind": "oracle", "sample": f"{desc}, repeated {n}x over {el:.1f} s (fp64, OpenMP over rows)"}


WORKLOADS_KIND = {k: v["kind"] for k, v in synth.WORKLOADS.items()}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    kind = WORKLOADS_KIND[args.workload]
    is_scan = kind in ("scan", "conv")
    fn, units, desc = oracle_sample(args.workload, (32 if args.backward else 256) if is_scan else 256 * 5120,
                                    args.zoh, args.backward)
    for _ in range(max(args.warmup, 0)):
        fn()
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        fn()
        times.append(time.perf_counter() - t0)
    ms = 1e3 * statistics.mean(times)
    value = units / (ms / 1e3)
    unit = "elems/s" if is_scan else "rows/s"
    line = {
        "impl": "reference",
        "metric": BWD_METRIC if args.backward else {"scan": METRIC, "conv": CONV_METRIC}.get(kind, DECODE_METRIC),
        "value": value, "unit": unit,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded)", "config": {"workload": args.workload, "sample": desc},
        "cpu_baseline": {"value": value, "unit": unit, "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------
# the GPU arm
# --------------------------------------------------------------------------

def run_mssm(args):
    import torch
    import torch.distributed as dist
    import selective_state_space_46_b200 as m

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    kind = WORKLOADS_KIND[args.workload]
    spec = synth.WORKLOADS[args.workload]
    io_bytes = 2 if spec["io_dtype"] == "bf16" else 4

    def to_dev(a):
        if a is None:
            return None
        if a.dtype == np.uint16:
            return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
        return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(dev)

    def pinned(a):
        if a is None:
            return None
        if a.dtype == np.uint16:
            t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
        else:
            t = torch.from_numpy(np.ascontiguousarray(a, np.float32))
        return t.pin_memory()

    seed = rank_seed(rank)
    m.mssm_set_option(m.MSSM_OPT_CHUNK_LEN, args.chunk_len)
    m.mssm_set_option(m.MSSM_OPT_ROWS_PER_CTA, args.rows_per_cta)
    m.mssm_set_option(m.MSSM_OPT_ROWS_PER_THREAD, args.rows_per_thread)
    m.mssm_set_option(m.MSSM_OPT_FORCE_GENERAL_A, 1 if args.general_a else 0)
    m.mssm_set_option(m.MSSM_OPT_DECODE_PATH, m.DECODE_PATHS.get(args.decode_path, 0))
    m.mssm_set_option(m.MSSM_OPT_SCHEDULE, m.SCHEDULES.get(args.schedule, 0))
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    props = torch.cuda.get_device_properties(dev)
    l2_bytes = int(getattr(props, "L2_cache_size", 0) or (126 << 20))
    if kind == "scan":
        inp = synth.workload_inputs(args.workload, seed=seed)
        host = {k: getattr(inp, k) for k in ("u", "delta", "A", "B", "C", "D", "z", "delta_bias")}
        units = inp.batch * inp.dim * inp.length
        varlen = inp.cu_seqlens is not None
        nstate = len(inp.cu_seqlens) - 1 if varlen else inp.batch
        max_seqlen = int(np.diff(inp.cu_seqlens).max()) if varlen else inp.length
        alg_bytes = scan_algorithmic_bytes(inp.batch, inp.dim, inp.length, io_bytes, inp.z is not None,
                                           inp.D is not None, inp.delta_bias is not None, last_state=False)
        alg_bytes += nstate * inp.dim * N_STATE * 4 + (4 * (nstate + 1) if varlen else 0)
        nsets = ring_size(alg_bytes, l2_bytes)
        d = {k: to_dev(v) for k, v in host.items()}
        cu_d = torch.from_numpy(inp.cu_seqlens).to(dev) if varlen else None
        sets = []
        for k in range(max(nsets, 1)):
            dk = d if k == 0 else {**d, **{n: d[n].clone() for n in ("u", "delta", "B", "C", "z") if d[n] is not None}}
            sets.append((dk, torch.empty_like(d["u"]), torch.empty(nstate, inp.dim, N_STATE, device=dev)))
        disc = m.MSSM_DISC_ZOH if args.zoh else m.MSSM_DISC_EULER

        def step(k=0):
            dk, out_k, last_k = sets[k % len(sets)]
            if varlen or args.zoh:
                m.mssm_selective_scan_fwd_ex(dk["u"], dk["delta"], dk["A"], dk["B"], dk["C"], dk["D"], dk["z"],
                                             dk["delta_bias"], inp.softplus, out_k, last_k, discretization=disc,
                                             cu_seqlens=cu_d, max_seqlen=max_seqlen if varlen else 0)
            else:
                m.mssm_selective_scan_fwd(dk["u"], dk["delta"], dk["A"], dk["B"], dk["C"], dk["D"], dk["z"],
                                          dk["delta_bias"], inp.softplus, out_k, last_k)
        config = {"workload": args.workload, "batch": inp.batch, "channels": inp.dim, "length": inp.length,
                  "state": N_STATE, "io_dtype": inp.io_dtype, "gate": inp.z is not None,
                  "softplus_bias": inp.delta_bias is not None, "D_skip": inp.D is not None,
                  "exp_path": "general (one exponential per state)" if args.general_a
                  else "structured A (powers of one exponential)",
                  "discretization": "zero-order hold" if args.zoh else "euler",
                  "chunk_len": args.chunk_len or "auto",
                  "plan": m.mssm_scan_plan(nstate, inp.dim, max_seqlen,
                                           total_len=inp.length if varlen else -1, io_dtype=inp.io_dtype)}
        if varlen:
            config.update({"sequences": nstate, "max_seqlen": max_seqlen, "packed_length": inp.length})
        metric, unit = METRIC, "elems/s"
        dom_kernel = "scan_out"
        set_bytes = alg_bytes
        if args.backward:
            if varlen or args.zoh:
                raise SystemExit("--backward covers the Euler scan of plain batches")
            # reads u, delta, z, dout, B, C; writes du, ddelta, dz (io dtype) and dB, dC (fp32)
            n_io = 7 if inp.z is not None else 5
            alg_bytes = (units * io_bytes * n_io + 2 * inp.batch * N_STATE * inp.length * (io_bytes + 4)
                         + inp.dim * N_STATE * 8 + inp.dim * 16)
            rng = np.random.default_rng(seed + 7)
            dout_h = rng.standard_normal(inp.u.shape).astype(np.float32)
            if inp.io_dtype == "bf16":
                dout_h = synth.f32_to_bf16_bits(dout_h)
            dout_d = to_dev(dout_h)
            grads = [m.selective_scan_bwd(d["u"], d["delta"], d["A"], d["B"], d["C"], d["D"], d["z"],
                                          d["delta_bias"], inp.softplus, dout_d) for _ in range(2)]

            def step(k=0):
                dk = sets[k % len(sets)][0]
                gk = grads[k % 2]
                m.mssm_selective_scan_bwd(dk["u"], dk["delta"], dk["A"], dk["B"], dk["C"], dk["D"], dk["z"],
                                          dk["delta_bias"], inp.softplus, dout_d, gk["du"], gk["ddelta"],
                                          gk["dA"], gk["dB"], gk["dC"], gk["dD"], gk["dz"], gk["ddelta_bias"])
            metric = BWD_METRIC
            dom_kernel = "scan_bwd"
            config["pass"] = "backward (chunk summaries both ways, then the per-chunk recompute and sweep)"
    elif kind == "conv":
        inp = synth.workload_inputs(args.workload, seed=seed)
        units = inp.batch * inp.dim * inp.length
        K = inp.weight.shape[1]
        alg_bytes = 2 * units * io_bytes + inp.dim * (K + 1) * 4
        set_bytes = alg_bytes
        nsets = ring_size(alg_bytes, l2_bytes)
        x0 = to_dev(inp.x)
        xs = [x0] + [x0.clone() for _ in range(max(nsets, 1) - 1)]
        outs_c = [torch.empty_like(x0) for _ in xs]
        w_d, b_d = to_dev(inp.weight), to_dev(inp.bias)
        d = {"x": x0}

        def step(k=0):
            j = k % len(xs)
            m.mssm_causal_conv1d_fwd(xs[j], w_d, b_d, outs_c[j], None, 0, True)
        config = {"workload": args.workload, "batch": inp.batch, "channels": inp.dim, "length": inp.length,
                  "kernel_size": K, "io_dtype": inp.io_dtype, "activation": "silu"}
        metric, unit = CONV_METRIC, "elems/s"
        dom_kernel = "conv"
    else:
        ring = [synth.workload_inputs(args.workload, seed=seed, step_stream=k) for k in range(8)]
        inp = ring[0]
        units = inp.batch * inp.dim
        alg_bytes = decode_algorithmic_bytes(inp.batch, inp.dim, io_bytes, inp.z is not None, inp.D is not None)
        # footprint of one step: the state once (read and written in place), the per-row inputs and y
        set_bytes = units * N_STATE * 4 + units * io_bytes * (4 if inp.z is not None else 3)
        nsets = ring_size(set_bytes, l2_bytes)
        state0 = to_dev(inp.state)
        states = [state0] + [state0.clone() for _ in range(max(nsets, 1) - 1)]
        A_d, D_d = to_dev(inp.A), to_dev(inp.D)
        dring = [{k: to_dev(getattr(r, k)) for k in ("x", "dt", "B", "C", "z")} for r in ring]
        outs = [torch.empty_like(dring[0]["x"]) for _ in states]

        def step(k=0):
            r = dring[k % len(dring)]
            j = k % len(states)
            m.mssm_state_update(states[j], r["x"], r["dt"], A_d, r["B"], r["C"], D_d, r["z"], outs[j])
        config = {"workload": args.workload, "batch": inp.batch, "channels": inp.dim, "state": N_STATE,
                  "io_dtype": inp.io_dtype, "input_ring": len(dring), "state_in_place": True,
                  "decode_path": args.decode_path}
        metric, unit = DECODE_METRIC, "rows/s"
        dom_kernel = "state_update"
    flush_between = nsets == 0
    if flush_between:
        l2_note = "flushed before every timed step (256 MiB write, outside the step's events)"
    else:
        l2_note = (f"not flushed: the steps rotate through {max(nsets, 1)} buffer set(s) of "
                   f"{set_bytes / 1e6:.1f} MB ({max(nsets, 1) * set_bytes / 1e6:.0f} MB >= 4x the "
                   f"{l2_bytes / 2**20:.0f} MiB L2), so no step finds its data in L2, and the write-back "
                   "of a step's dirty lines falls inside the following steps' timed regions")

    # ---- warm-up (also allocates the library's carry workspace before capture)
    for k in range(max(args.warmup, 3)):
        if flush_between:
            flush.zero_()
        step(k)
    torch.cuda.synchronize(dev)
    m.mssm_get_error()

    # ---- capture the K timed steps into one graph
    # external=True: the records become event nodes of the graph, so every replay re-records them
    # one event pair per step only when the L2 flush must stay outside the bracket
    npairs = args.steps if flush_between else 1
    starts = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(npairs)]
    ends = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(npairs)]
    before = m.mssm_kernel_stats()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        if not flush_between:
            starts[0].record()
        for k in range(args.steps):
            if flush_between:
                flush.zero_()
                starts[k].record()
            step(k)
            if flush_between:
                ends[k].record()
        if not flush_between:
            ends[0].record()
    after = m.mssm_kernel_stats()
    launches = sum(after[k]["launches"] - before[k]["launches"] for k in after)

    sampler = ClockSampler(local).start()
    # soak: keep the GPU at its loaded clocks for a while before the timed replay
    t_soak = time.perf_counter()
    while time.perf_counter() - t_soak < args.soak:
        g.replay()
        torch.cuda.synchronize(dev)

    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    g.replay()
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    m.mssm_get_error()
    per_step = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total_ms = reduce_max(sum(per_step), dist if world > 1 else None)
    ms_per_step = total_ms / args.steps
    value = units * world / (ms_per_step / 1e3)

    # ---- per-kernel durations (same launches, events bracketing each kernel)
    m.mssm_set_option(m.MSSM_OPT_KERNEL_TIMING, 1)
    m.mssm_kernel_stats(reset=True)
    for k in range(args.steps):
        if flush_between:
            flush.zero_()
        step(k)
    torch.cuda.synchronize(dev)
    ks = m.mssm_kernel_stats(reset=True)
    m.mssm_set_option(m.MSSM_OPT_KERNEL_TIMING, 0)
    kern = {k: {"launches_per_step": v["timed"] / args.steps,
                "ms_per_launch": (v["ms"] / v["timed"]) if v["timed"] else None}
            for k, v in ks.items() if v["timed"]}
    dom = kern.get(dom_kernel)
    peak, peak_kind = measured_peaks()
    dom_ms = dom["ms_per_launch"] if dom else None
    # a step that is exactly one launch of the dominant kernel: its back-to-back step time
    single = (dom is not None and launches == args.steps and
              all(v["launches_per_step"] == (1.0 if k == dom_kernel else 0.0) for k, v in kern.items()))
    dom_timing = "events around each launch"
    if single and not flush_between:
        dom_ms = ms_per_step
        dom_timing = "step time of back-to-back single-launch steps"
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    alu_peak = fp32_peak_tflops(sms, max_sm_mhz())
    # the conv: K FMAs per element (its SiLU runs on the SFU); the backward: BWD_FLOP_PER_STATE
    if kind == "conv":
        alg_flops = units * 2 * inp.weight.shape[1]
    elif kind == "scan" and args.backward:
        alg_flops = units * N_STATE * BWD_FLOP_PER_STATE
    else:
        alg_flops = algorithmic_flops(units)
    plan_key = (plan_string(config.get("plan")) if kind == "scan" and not args.backward else
                f"decode_path={args.decode_path}" if kind == "decode" else None)
    traffic, traffic_src = recorded_traffic(dom_kernel, args.workload, plan_key)
    roofline = binding_roofline(alg_bytes, alg_flops, dom_ms, peak, alu_peak) if dom_ms else {"bound": None}
    roofline.update({"kernel": dom_kernel, "ms_per_launch": dom_ms, "timing": dom_timing,
                     "peak_source": f"HBM: {peak_kind} copy rate; FP32: {sms} SMs x 128 lanes x 2 x "
                                    f"{max_sm_mhz():.0f} MHz",
                     "algorithmic_bytes_per_launch": alg_bytes, "algorithmic_flops_per_launch": alg_flops,
                     "traffic": traffic, "traffic_source": traffic_src,
                     "traffic_step": recorded_step_traffic(dom_kernel, args.workload, plan_key)})

    # ---- end to end: host buffers in pinned memory, copies inside the timed region
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, kind, inp, d if kind in ("scan", "conv") else None, dev, m, units, world)

    step_gbs = alg_bytes / (ms_per_step / 1e3) / 1e9
    line = {
        "metric": metric, "value": value, "unit": unit, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic (seeded; no datasets or weights)",
        "config": {**config, "l2": l2_note,
                   "parallelism": f"replicas x{world} (independent rows, no collective)",
                   "timing": ("CUDA events per step inside one captured graph" if flush_between else
                              "one CUDA event pair around the K back-to-back steps of one captured graph")},
        "hbm_gbs": step_gbs * world, "hbm_gbs_per_gpu": step_gbs,
        "hbm_frac_of_8tbs": step_gbs / NOMINAL_HBM_GBS, "hbm_frac_of_measured": step_gbs / peak,
        "kernels": kern, "roofline": roofline, "e2e": e2e, "gpu_launches": launches, "clocks": clocks,
        "source_hash": kernel_source_hash(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.workload, args.cpu_seconds, args.zoh, args.backward)
    if world > 1:
        dist.barrier()
        del g
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def run_e2e(args, kind, inp, d, dev, m, units, world):
    """The same metric end to end through the public API: every step copies its inputs from
    pinned host memory to the device, makes the C-ABI call and copies its results back.  Two
    device buffer sets and three streams pipeline the steps: the uploads of step k + 1 overlap
    the call and the downloads of step k (PCIe is full duplex, with a copy engine each way)."""
    import torch
    import torch.distributed as dist
    steps = max(2, min(args.steps, 20))

    def pin(a):
        if a is None:
            return None
        if a.dtype == np.uint16:
            t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
        else:
            t = torch.from_numpy(np.ascontiguousarray(a, np.float32))
        return t.pin_memory()

    def dev_like(v):
        return None if v is None else torch.empty(v.shape, dtype=v.dtype, device=dev)

    def host_like(v):
        return None if v is None else torch.empty(v.shape, dtype=v.dtype).pin_memory()

    def upload(h, dd):
        for k, v in h.items():
            if v is not None:
                dd[k].copy_(v, non_blocking=True)

    def download(dd, hh):
        for k, v in dd.items():
            if v is not None:
                hh[k].copy_(v, non_blocking=True)

    # per kind: host inputs h, and make_set() -> (device inputs, device results, host results, call)
    if kind == "conv":
        h = {"x": pin(inp.x)}
        w_d, b_d = pin(inp.weight).to(dev), pin(inp.bias).to(dev)

        def make_set():
            di = {"x": dev_like(h["x"])}
            do = {"y": torch.empty_like(di["x"])}
            return di, do, {"y": host_like(do["y"])}, (
                lambda: m.mssm_causal_conv1d_fwd(di["x"], w_d, b_d, do["y"], None, 0, True))
        path_out = "y"
    elif kind == "scan" and args.backward:
        names = ("u", "delta", "A", "B", "C", "D", "z", "delta_bias")
        h = {k: pin(getattr(inp, k)) for k in names}
        rng = np.random.default_rng(7)
        dout_h = rng.standard_normal(inp.u.shape).astype(np.float32)
        h["dout"] = pin(synth.f32_to_bf16_bits(dout_h) if inp.io_dtype == "bf16" else dout_h)

        def make_set():
            di = {k: dev_like(v) for k, v in h.items()}
            upload(h, di)
            torch.cuda.synchronize(dev)
            g = m.selective_scan_bwd(di["u"], di["delta"], di["A"], di["B"], di["C"], di["D"], di["z"],
                                     di["delta_bias"], inp.softplus, di["dout"])
            do = {k: v for k, v in g.items() if v is not None}
            return di, do, {k: host_like(v) for k, v in do.items()}, (
                lambda: m.mssm_selective_scan_bwd(di["u"], di["delta"], di["A"], di["B"], di["C"], di["D"], di["z"],
                                                  di["delta_bias"], inp.softplus, di["dout"], g["du"], g["ddelta"],
                                                  g["dA"], g["dB"], g["dC"], g["dD"], g["dz"], g["ddelta_bias"]))
        path_out = "every gradient"
    elif kind == "scan":
        names = ("u", "delta", "A", "B", "C", "D", "z", "delta_bias")
        h = {k: pin(getattr(inp, k)) for k in names}
        varlen = inp.cu_seqlens is not None
        if varlen:
            h["cu_seqlens"] = torch.from_numpy(inp.cu_seqlens).pin_memory()
        nstate = len(inp.cu_seqlens) - 1 if varlen else inp.batch
        max_seqlen = int(np.diff(inp.cu_seqlens).max()) if varlen else 0
        disc = m.MSSM_DISC_ZOH if args.zoh else m.MSSM_DISC_EULER

        def make_set():
            di = {k: dev_like(v) for k, v in h.items()}
            do = {"y": torch.empty_like(di["u"]), "last": torch.empty(nstate, inp.dim, N_STATE, device=dev)}
            return di, do, {k: host_like(v) for k, v in do.items()}, (
                lambda: m.mssm_selective_scan_fwd_ex(di["u"], di["delta"], di["A"], di["B"], di["C"], di["D"],
                                                     di["z"], di["delta_bias"], inp.softplus, do["y"], do["last"],
                                                     discretization=disc, cu_seqlens=di.get("cu_seqlens"),
                                                     max_seqlen=max_seqlen))
        path_out = "y and the final state"
    else:
        names = ("state", "x", "dt", "A", "B", "C", "D", "z")
        h = {k: pin(getattr(inp, k)) for k in names}

        def make_set():
            di = {k: dev_like(v) for k, v in h.items()}
            do = {"y": torch.empty_like(di["x"]), "state": di["state"]}
            return di, do, {k: host_like(v) for k, v in do.items()}, (
                lambda: m.mssm_state_update(di["state"], di["x"], di["dt"], di["A"], di["B"], di["C"], di["D"],
                                            di["z"], do["y"]))
        path_out = "y and the updated state"

    sets = [make_set() for _ in range(2)]
    h2d = sum(v.numel() * v.element_size() for v in h.values() if v is not None)
    d2h = sum(v.numel() * v.element_size() for v in sets[0][2].values() if v is not None)
    s_in, s_call, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    ev = {name: [torch.cuda.Event() for _ in sets] for name in ("in", "call", "out")}

    def run(n):
        for k in range(n):
            j = k % len(sets)
            di, do, ho, call = sets[j]
            with torch.cuda.stream(s_in):
                if k >= len(sets):
                    # the step before that has read this set's inputs and copied out its results
                    # (the decode state is both)
                    s_in.wait_event(ev["out"][j])
                upload(h, di)
                ev["in"][j].record(s_in)
            with torch.cuda.stream(s_call):
                s_call.wait_event(ev["in"][j])
                if k >= len(sets):
                    s_call.wait_event(ev["out"][j])  # this set's results were copied out
                call()
                ev["call"][j].record(s_call)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev["call"][j])
                download(do, ho)
                ev["out"][j].record(s_out)

    main = torch.cuda.current_stream(dev)
    run(len(sets))
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(main)
    for s in (s_in, s_call, s_out):
        s.wait_stream(main)
    run(steps)
    for s in (s_in, s_call, s_out):
        main.wait_stream(s)
    t1.record(main)
    torch.cuda.synchronize(dev)
    ms = reduce_max(t0.elapsed_time(t1), dist if world > 1 else None) / steps
    return {"value": units * world / (ms / 1e3), "unit": "elems/s" if kind in ("scan", "conv") else "rows/s",
            "ms_per_step": ms, "steps": steps, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "path": (f"pinned host buffers -> H2D copies -> C-ABI call -> D2H of {path_out}, every step; "
                     "two buffer sets on three streams, the uploads of one step overlapping the call and "
                     "downloads of the one before")}


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default 50; 1000 successive steps for the decode workload)")
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["mssm", "reference"], default="mssm")
    ap.add_argument("--workload", choices=sorted(synth.WORKLOADS), default=DEFAULT_WORKLOAD)
    ap.add_argument("--soak", type=float, default=1.5, help="seconds of untimed graph replays before timing")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--chunk-len", type=int, default=0, help="length split (0: automatic; multiple of 64)")
    ap.add_argument("--rows-per-cta", type=int, default=0, choices=[0, 32, 64, 128],
                    help="channels per row tile of the scan (0: automatic)")
    ap.add_argument("--rows-per-thread", type=int, default=0, choices=[0, 1, 2],
                    help="channels per thread of the scan kernels (0: automatic; 2: bf16 I/O only)")
    ap.add_argument("--decode-path", choices=["auto", "stream", "bulk_tile", "per_row"], default="auto",
                    help="decode kernel (MSSM_OPT_DECODE_PATH)")
    ap.add_argument("--zoh", action="store_true", help="zero-order-hold discretisation (scan workloads)")
    ap.add_argument("--schedule", choices=["auto", "forward", "summaries+forward", "chained", "fused", "split"],
                    default="auto", help="force a scan schedule (MSSM_OPT_SCHEDULE)")
    ap.add_argument("--backward", action="store_true", help="time the backward scan instead (scan workloads)")
    ap.add_argument("--general-a", action="store_true",
                    help="disable the structured-A path (one exponential per state)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3
    if args.steps is None:
        decode = synth.WORKLOADS[args.workload]["kind"] == "decode"
        args.steps = 1000 if decode and args.impl == "mssm" else 50
    if args.impl == "reference":
        return run_reference(args)
    return run_mssm(args)


if __name__ == "__main__":
    sys.exit(main())
