"""World-size-2 gloo tests (CPU) of the benchmark's multi-rank host logic.

The scan shards as independent replicas: each rank draws its own batch
(seed = rank), runs it with no collective on the data path, and the step time
is the max over ranks.  These tests run that logic on two CPU processes.
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        import synth
        seed = bench.rank_seed(rank)
        inp = synth.workload_inputs("scan_f32_1x64x256", seed=seed)
        # a fake per-rank duration: the reduction must return the largest one
        mx = bench.reduce_max(10.0 + rank * 2.5, dist)
        q.put((rank, seed, float(inp.u[0, 0, :4].sum()), mx))
    finally:
        dist.destroy_process_group()


def test_two_ranks_distinct_shards_and_max_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    (r0, s0, u0, m0), (r1, s1, u1, m1) = res
    assert (s0, s1) == (0, 1)
    assert u0 != u1                  # each rank works on its own batch
    assert m0 == m1 == 12.5          # both ranks see the max over ranks


def test_reduce_max_without_group_is_identity():
    import bench
    assert bench.reduce_max(3.25, None) == 3.25


def test_algorithmic_bytes_match_the_stated_figures():
    import bench
    # Mamba-130M-shaped prefill: 50.9 MB; decode step 256 x 5120: 178.6 MB
    b1 = bench.scan_algorithmic_bytes(2, 1536, 2048, 2)
    assert abs(b1 / 1e6 - 50.9) < 0.1
    bd = bench.decode_algorithmic_bytes(256, 5120, 2)
    assert abs(bd / 1e6 - 178.6) < 0.3


def test_binding_roofline_picks_the_slower_bound():
    import bench
    peak_fp32 = bench.fp32_peak_tflops(148, 1965.0)
    assert abs(peak_fp32 - 74.45) < 0.01                 # 148 x 128 x 2 x 1.965 GHz
    # prefill at 2 x 1536 x 2048: 96 flop against 8.09 B per element; the FP32 time
    # (8.1 us) exceeds the copy-rate time (7.8 us), so the FP32 pipe is the bound
    units = 2 * 1536 * 2048
    r = bench.binding_roofline(bench.scan_algorithmic_bytes(2, 1536, 2048, 2), bench.algorithmic_flops(units),
                               0.0405, 6539.5, peak_fp32)
    assert r["bound"] == "alu" and r["unit"] == "TFLOP/s" and r["other"]["bound"] == "hbm"
    assert abs(r["frac"] - r["achieved"] / peak_fp32) < 1e-12
    # decode: 96 flop against 136 B per row -> HBM
    rows = 256 * 5120
    r = bench.binding_roofline(bench.decode_algorithmic_bytes(256, 5120, 2), bench.algorithmic_flops(rows),
                               0.030, 6539.5, peak_fp32)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert abs(r["achieved"] - 178.6e6 / 30e-6 / 1e9) < 15


def test_ring_size_covers_four_l2():
    import bench
    l2 = 126 << 20
    assert bench.ring_size(1347 << 20, l2) == 1                   # one set is already > 4x L2
    r = bench.ring_size(50_900_000, l2)
    assert r == 11 and r * 50_900_000 >= 4 * l2 and (r - 1) * 50_900_000 < 4 * l2
    assert 0 < bench.ring_size(25_190_400, l2) <= 32               # the conv workload still rotates
    assert bench.ring_size(240_000, l2) == 0                      # tiny: flush instead
