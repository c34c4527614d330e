"""Host-side pieces of bench.py: algorithmic byte counts, the max-over-ranks timing reduction
with two gloo ranks on the CPU (the N-GPU replica path), the CPU-oracle baselines and their
diagnostics, and the reference arm launched under torchrun."""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def test_linear_bytes_q_proj_decode():
    # codes + w scales + int8 activations + act scale + fp16 output for 4096x4096, one token
    assert bench.linear_bytes(1, 4096, 4096, 2) == 4096 * 4096 // 4 + 4 * 4096 + 4096 + 4 + 2 * 4096
    assert bench.acts_bytes(1, 4096) == 3 * 4096 + 4
    # 4-bit weights: half a byte of codes per weight
    assert bench.linear_bytes(1, 4096, 4096, 2, "int4") == 4096 * 4096 // 2 + 4 * 4096 + 4096 + 4 + 2 * 4096


def test_traffic_records_match_the_current_kernels():
    # Each DRAM-traffic record is keyed by a hash of its kernel's sources and reported as null once
    # they change; every record on file must have been captured on the sources as they stand,
    # next to its ncu summary.
    for name, rec in bench.PROFILED_TRAFFIC.items():
        assert bench.profiled_traffic(name) == rec["bytes"] * rec.get("scale", 1.0), name
        assert os.path.exists(os.path.join(bench.ROOT, rec["profile"])), name
    assert bench.profiled_traffic("single") is None  # no record: null, not a guess


def test_every_workload_has_a_bench_choice():
    from w2a4_gemm_b200 import synth
    names = {bench.workload_def(w).name for w in ("decode", "decode16", "prefill", "single", "decode_w4",
                                                     "decode16_w4", "prefill_w4")}
    assert names == set(synth.WORKLOADS)


def test_peaks_reads_measured_file_or_fallback():
    p = bench.peaks()
    assert p["hbm_gbs"] > 1000 and p["int8_tops"] > 1000
    assert p["source"] in ("measured", "fallback")


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        out[rank] = bench.max_over_ranks(1.5 + rank, world)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_two_ranks():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert out[0] == out[1] == 2.5


def test_max_over_ranks_single_process_is_identity():
    assert bench.max_over_ranks(3.25, 1) == 3.25


def test_cpu_baseline_reports_all_cores_and_one_core():
    import oracle
    before = oracle.threads()
    obj = bench.cpu_baseline_obj(bench.workload_def("single"), budget_s=0.2)
    assert obj["kind"] == "oracle" and obj["cores"] == before and obj["value"] > 0
    assert obj["single_core"]["cores"] == 1 and obj["single_core"]["value"] > 0
    assert oracle.threads() == before  # the thread count is put back


def test_excess_kurtosis_known_values():
    import numpy as np
    import torch
    assert bench.excess_kurtosis(torch.tensor([-1.0, 1.0, -1.0, 1.0])) == -2.0   # two-point law
    g = torch.from_numpy(np.random.default_rng(0).normal(size=400_000))
    assert abs(bench.excess_kurtosis(g)) < 0.05                                   # Gaussian: 0
    t = torch.from_numpy(np.random.default_rng(1).standard_t(6, size=400_000))
    assert 2.0 < bench.excess_kurtosis(t) < 4.5                                   # t(6): 6/(6-4) = 3


def test_per_projection_mse_weights_modules_by_size():
    mods = [(0, "q", 2, 4, 0), (0, "down", 1, 8, 1), (1, "q", 1, 4, 2)]
    rows = {"qift": [[1.0, 3.0], [5.0], [8.0]]}
    got = bench.per_projection_mse(mods, rows)["qift"]
    # q: (1 + 3) * 4 + 8 * 4 over 3 rows of 4 -> 48 / 12; down: 5 * 8 / 8
    assert got == {"q": 4.0, "down": 5.0}


def test_reference_arm_under_torchrun_prints_one_line_from_rank_0():
    # Launched the way the multi-GPU runs are (one process per rank): rank 0 alone times the
    # oracle and prints; the other rank exits 0 without work.
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py", "--impl", "reference",
           "--workload", "single", "--steps", "2", "--warmup", "1"]
    r = subprocess.run(cmd, cwd=root, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0
