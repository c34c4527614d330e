"""Benchmark of the Qift W2A4 linear path on B200 (one JSON line on stdout).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload decode|decode16|prefill|single|offline|decode_w4|decode16_w4|prefill_w4]

Workloads (synthetic, seeded; shapes of LLaMA linear modules):
  decode   (default) LLaMA-7B q_proj 4096x4096, 1 token, 4096-point Hadamard, Qift {+-1,+-3}
  decode16 LLaMA-3.1-8B MLP (gate/up 14336x4096, down 4096x14336), 16 tokens, 128-block, PoT
  prefill  LLaMA-7B MLP (gate/up 11008x4096, down 4096x11008), 2048 tokens, 128-block, Qift
  single   one 256x512 linear, 8 tokens (parity case; timed for completeness)
  decode_w4, decode16_w4, prefill_w4
           the decode, decode16 and prefill shapes with 4-bit weights ({-7..7} * s per channel),
           the W4 layers of a mixed W2/W4 model: W4A4 linear (CUDA-core GEMV at one token, the
           tensor-core skinny GEMM at 16, the tcgen05 pair GEMM at 2048)
  offline  offline quantization of a full 8B-shaped model (224 modules, 6.98 G weights):
           128-block rotation + per-row scale search + encode + pack for the Qift, PoT and
           standard level sets; reports weights/s and the reconstruction MSE of each set

A step is one online forward pass over one batch: qift_quantize_acts (rotation + INT4) of
every distinct input (an MLP's gate and up read the same one) and qift_linear for every linear
of the workload.  The weights are quantized once, offline
(qift_rotate + qift_quantize_weights), and are resident in HBM; those two offline stages are
timed in the same run and reported under "stages".  Decode workloads cycle through enough
distinct weight copies that every step streams its codes from HBM, not L2.

Timing: the `--steps` steps are one CUDA graph, replayed once between CUDA events on the
replaying stream, after a device-side sleep that lets the host submit the graph before the
start event (so the region holds the kernels only).  Each per-kernel stage is a chain of a fixed
number of back-to-back launches (200 at decode sizes), timed the same way: the median of ten
replays, with the min and max beside it.  The default run (decode) also records the prefill
GEMM (2048 tokens, TOPS against the int8 peak, with the vendor int8 GEMM measured beside it)
and the 16-token PoT MLP decode under "stages", so one run covers both halves of the metric.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "W2A4 Qift linear: decode GB/s & prefill TOPS, % of B200 roofline"
L2_BYTES = 126 * 1024 * 1024


def peaks():
    """HBM GB/s and int8 dense TOPS (burst, sustained) from the measured peak file."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    src = "measured"
    try:
        with open(path) as f:
            p = json.load(f)
        hbm, bf16, bf16s = p["hbm_gbs"], p["bf16_tflops"], p.get("bf16_tflops_sustained", p["bf16_tflops"])
    except (OSError, KeyError, ValueError):
        hbm, bf16, bf16s, src = 6650.0, 1590.0, 1400.0, "fallback"
    # int8 dense = bf16 dense x 2 (nominal 4.5 vs 2.25 PFLOP/s per GPU).
    return dict(hbm_gbs=hbm, int8_tops=2.0 * bf16, int8_tops_sustained=2.0 * bf16s, source=src)


# DRAM traffic per launch (dram__bytes_read.sum + dram__bytes_write.sum) of the dominant kernel,
# from one ncu capture of the same workload (summaries in profiles/).  Each entry is keyed by a
# hash of the kernel's sources; if they have changed since the capture the traffic is reported
# as null.  `scale` converts the captured launch to the benchmarked one when the shapes differ
# (traffic grows in proportion to the weights processed).
PROFILED_TRAFFIC = {
    "decode": dict(files=("linear_gemv.cu", "common.cuh"), sha="b4c3a19ee0236ba1", bytes=4226048 + 0,
                   profile="profiles/gemv1_kernel_q_proj_decode_T1.md"),
    "prefill": dict(files=("linear_gemm_tc.cu", "tc.cuh", "common.cuh"), sha="6f280e4dafa17a5e",
                    bytes=19754752 + 2899456, profile="profiles/w2a4_gemm_pair_kernel_mlp_prefill_T2048.md"),
    "decode16": dict(files=("linear_skinny.cu", "common.cuh"), sha="4ec14ac10ad3f139", bytes=14840320 + 0,
                     profile="profiles/skinny_kernel_mlp_decode_T16_pot.md"),
    "decode_w4": dict(files=("linear_w4.cu", "common.cuh"), sha="bec1d0cc3845435a", bytes=8418560 + 0,
                      profile="profiles/w4_gemv1_kernel_q_proj_decode_T1_w4.md"),
    "decode16_w4": dict(files=("linear_skinny.cu", "common.cuh"), sha="4ec14ac10ad3f139", bytes=29514240 + 256,
                        profile="profiles/skinny_kernel_mlp_decode_T16_w4.md"),
    "offline": dict(files=("quantize_weights.cu", "common.cuh"), sha="00f7bc2d84fdc9a9",
                    bytes=67153920 + 1506816, scale=14336 * 4096 / (4096 * 4096),
                    profile="profiles/quant_weights_kernel_q_proj_4096x4096.md"),
}


def profiled_traffic(workload):
    import hashlib
    e = PROFILED_TRAFFIC.get(workload)
    if not e:
        return None
    h = hashlib.sha1()
    for f in e["files"]:
        with open(os.path.join(ROOT, "w2a4_gemm_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    if h.hexdigest()[:16] != e["sha"]:
        return None
    return e["bytes"] * e.get("scale", 1.0)


# ----------------------------------------------------------------------------- workloads
def workload_def(name):
    from w2a4_gemm_b200 import synth
    return {"decode": synth.LLAMA7B_QPROJ_DECODE, "decode16": synth.LLAMA31_8B_MLP_DECODE16,
            "prefill": synth.LLAMA7B_MLP_PREFILL, "single": synth.SINGLE_256x512,
            "decode_w4": synth.LLAMA7B_QPROJ_DECODE_W4, "decode16_w4": synth.LLAMA31_8B_MLP_DECODE16_W4,
            "prefill_w4": synth.LLAMA7B_MLP_PREFILL_W4}[name]


def code_bytes(N, K, levelset):
    """Bytes of packed weight codes: 2 bits per weight, 4 for the 4-bit set."""
    return N * K // 2 if levelset == "int4" else N * K // 4


def linear_bytes(T, N, K, out_bytes, levelset="qift"):
    """Algorithmic HBM bytes of one qift_linear: codes + w scales + int8 acts + act scales + y."""
    return code_bytes(N, K, levelset) + 4 * N + T * K + 4 * T + T * N * out_bytes


def acts_bytes(T, K):
    """Algorithmic HBM bytes of one qift_quantize_acts: fp16 in, int8 + scale out."""
    return 2 * T * K + T * K + 4 * T


# ------------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not self.path:
            return None
        rows = []
        with open(self.path) as f:
            for ln in f:
                p = [x.strip() for x in ln.split(",")]
                if len(p) >= 9 and p[1].replace(".", "").isdigit():
                    rows.append(p)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for i, n in enumerate(names):
                if r[5 + i].lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": float(rows[0][2]), "samples": len(rows),
                "power_w_max": max(float(r[3]) for r in rows if r[3].replace(".", "").isdigit()) if rows else None,
                "reasons": sorted(reasons)}


# ----------------------------------------------------------------------------- our path
class OursState:
    """Device-resident inputs of one workload: quantized weight copies and activation slots."""

    def __init__(self, wl, torch, qg, copies):
        self.wl, self.torch, self.qg = wl, torch, qg
        dev = torch.device("cuda")
        self.out_dt = torch.float16 if wl.out_dtype == "f16" else torch.float32
        self.layers = []
        self.offline = []
        first = {}  # linears that read the same input (an MLP's gate and up) share one quantization
        for lin in wl.linears:
            W = torch.from_numpy(wl.w(lin)).to(dev)
            w_rot = qg.qift_rotate(W, wl.w_block)
            codes, s_w, _ = qg.qift_quantize_weights(w_rot, wl.levelset, with_mse=False)
            self.offline.append((W, lin))
            cc = [codes] + [codes.clone() for _ in range(copies - 1)]
            sc = [s_w] + [s_w.clone() for _ in range(copies - 1)]
            T, K, N = wl.tokens, lin.n_in, lin.n_out
            key = (lin.x_seed, lin.n_in)
            if key in first:
                src = first[key]
                xs, q, sa, quant = src["x"], src["q"], src["sa"], False
            else:
                xs = [torch.from_numpy(wl.x(lin)).to(dev) for _ in range(1)]
                xs = xs + [xs[0].clone() for _ in range(copies - 1)]
                q = [torch.empty((T, K), dtype=torch.int8, device=dev) for _ in range(copies)]
                sa = [torch.empty(T, dtype=torch.float32, device=dev) for _ in range(copies)]
                quant = True
            y = [torch.empty((T, N), dtype=self.out_dt, device=dev) for _ in range(copies)]
            L = dict(lin=lin, codes=cc, s_w=sc, x=xs, q=q, sa=sa, y=y, quant=quant)
            if quant:
                first[key] = L
            self.layers.append(L)
        self.copies = copies

    def step(self, i):
        qg, wl = self.qg, self.wl
        c = i % self.copies
        for L in self.layers:
            if L["quant"]:
                qg.qift_quantize_acts(L["x"][c], wl.a_block, out_q=L["q"][c], out_scales=L["sa"][c])
            qg.qift_linear(L["q"][c], L["sa"][c], L["codes"][c], L["s_w"][c], wl.levelset, self.out_dt,
                           out=L["y"][c])

    def launches_per_step(self):
        return sum(1 + int(L["quant"]) for L in self.layers)


def library_int8_tops(torch, n=8192, reps=10):
    """Dense int8 TOPS of the vendor library GEMM (torch._int_mm, int8 x int8 -> int32) on an
    n x n x n problem: the best of `reps` launches, each timed with CUDA events."""
    a = torch.randint(-7, 8, (n, n), dtype=torch.int8, device="cuda")
    b = torch.randint(-7, 8, (n, n), dtype=torch.int8, device="cuda")
    for _ in range(3):
        torch._int_mm(a, b)
    best = float("inf")
    for _ in range(reps):
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        torch._int_mm(a, b)
        e.record()
        torch.cuda.synchronize()
        best = min(best, s.elapsed_time(e) / 1e3)
    return 2.0 * n ** 3 / best / 1e12


def max_over_ranks(value: float, world: int) -> float:
    """The largest of every rank's value (one all-reduce); the value itself on one rank."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def capture(torch, fn, iters, offset=0):
    """A CUDA graph of fn(offset) .. fn(offset + iters - 1): the launches go through the C ABI
    onto the capturing stream, so replaying the graph replays exactly those kernels."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        for i in range(iters):
            fn(offset + i)
    torch.cuda.synchronize()
    return g


# GPU cycles the stream sleeps before the start event of every timed region (about 1 ms): the
# host submits the graph meanwhile, so the region holds only the graph's kernels and not the
# time the host takes to launch it.  Without it a short region (a few dozen launches) also
# counts the gap between the start event and the graph's first kernel, and the per-launch
# figure depends on how many launches the graph holds.
PREROLL_CYCLES = 2_000_000


def time_graph(torch, g):
    """Seconds of one replay: CUDA events on the replaying stream around the graph, after a
    device-side pre-roll, synchronised on both sides."""
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    torch.cuda._sleep(PREROLL_CYCLES)
    s.record()
    g.replay()
    e.record()
    torch.cuda.synchronize()
    return s.elapsed_time(e) / 1e3


def time_region(torch, fn, iters):
    """Seconds for fn(0..iters-1) replayed as one CUDA graph (captured, uploaded, then timed)."""
    g = capture(torch, fn, iters)
    g.replay()
    torch.cuda.synchronize()
    return time_graph(torch, g)


def chain_stats(torch, fn, launches, replays=10):
    """Per-launch seconds of fn(0..launches-1) captured as one CUDA graph of back-to-back
    launches: the median, min and max over `replays` timed replays (one untimed replay first)."""
    g = capture(torch, fn, launches)
    g.replay()
    torch.cuda.synchronize()
    ts = sorted(time_graph(torch, g) / launches for _ in range(replays))
    del g
    return {"s": statistics.median(ts), "s_min": ts[0], "s_max": ts[-1], "launches": launches, "replays": replays}


def stage_record(st, bytes_=None, ops=None, pk=None, bound="hbm", **extra):
    """A stage's JSON record from chain_stats: microseconds (median, min, max) and the rate."""
    r = {"us": st["s"] * 1e6, "us_min": st["s_min"] * 1e6, "us_max": st["s_max"] * 1e6,
         "launches": st["launches"], "replays": st["replays"], "bound": bound}
    if bytes_ is not None:
        r["bytes"] = bytes_
        r["GB/s"] = bytes_ / st["s"] / 1e9
        if pk is not None:
            r["frac_hbm"] = r["GB/s"] / pk["hbm_gbs"]
    if ops is not None:
        r["TOPS"] = ops / st["s"] / 1e12
        if pk is not None and bound == "tensor":
            r["frac_int8"] = r["TOPS"] / pk["int8_tops"]
    r.update(extra)
    return r


STAGE_LAUNCHES = 200  # launches per timed chain of a per-kernel stage (decode sizes)
STAGE_REPLAYS = 10


def decode_copies(wl):
    """Weight copies cycled step to step so that every decode step streams its codes from HBM:
    about three times the L2 in total."""
    wbytes = sum(code_bytes(l.n_out, l.n_in, wl.levelset) for l in wl.linears)
    return max(1, min(64, int(np.ceil(3 * L2_BYTES / max(wbytes, 1))))), wbytes


def linear_stage(torch, qg, st, L, pk, launches, replays, T, out_b):
    """Chain of qift_linear launches over the cycled copies of one layer."""
    wl, copies, lin = st.wl, st.copies, L["lin"]
    fn = lambda i: qg.qift_linear(L["q"][i % copies], L["sa"][i % copies], L["codes"][i % copies],
                                  L["s_w"][i % copies], wl.levelset, st.out_dt, out=L["y"][i % copies])
    N, K = lin.n_out, lin.n_in
    bound = "tensor" if T > 16 else "hbm"
    return stage_record(chain_stats(torch, fn, launches, replays),
                        bytes_=linear_bytes(T, N, K, out_b, wl.levelset), ops=2 * T * N * K, pk=pk,
                        bound=bound, shape=[T, N, K])


def prefill_stage(torch, qg, pk, replays=STAGE_REPLAYS):
    """The LLaMA-7B MLP prefill (2048 tokens): the tensor-core GEMM of each distinct shape and a
    whole MLP step, TOPS against the int8 peak, and the vendor int8 GEMM measured beside it."""
    from w2a4_gemm_b200 import synth
    wl = synth.LLAMA7B_MLP_PREFILL
    st = OursState(wl, torch, qg, 3)  # three input sets cycled: 3 x 65 MB per GEMM > L2
    T = wl.tokens
    ops = sum(2 * T * l.n_out * l.n_in for l in wl.linears)
    step = chain_stats(torch, st.step, 6, replays)
    out = {"workload": wl.name, "step": stage_record(step, ops=ops, pk=pk, bound="tensor",
                                                     what="qift_quantize_acts x2 + qift_linear x3")}
    seen = set()
    for L in st.layers:
        key = (L["lin"].n_out, L["lin"].n_in)
        if key in seen:
            continue
        seen.add(key)
        out[L["lin"].name] = linear_stage(torch, qg, st, L, pk, 30, replays, T, 2)
    g = out["gate_proj"]
    out["roofline"] = {"bound": "tensor", "achieved": g["TOPS"], "peak": pk["int8_tops"], "unit": "TOPS",
                       "frac": g["TOPS"] / pk["int8_tops"], "traffic": profiled_traffic("prefill"),
                       "kernel": "w2a4_gemm_pair_kernel (qift_linear, gate_proj 11008x4096, 2048 tokens)",
                       "peak_source": pk["source"] + " bf16 burst x 2 (int8 nominal ratio)",
                       "datasheet_int8_tops": 4500.0, "frac_datasheet": g["TOPS"] / 4500.0}
    try:
        lib_tops = library_int8_tops(torch)
        out["roofline"]["library_int8"] = {
            "tops": lib_tops, "frac": g["TOPS"] / lib_tops,
            "what": "torch._int_mm (the vendor int8 GEMM) at 8192^3, best of 10, same run"}
    except RuntimeError as e:  # an int8 GEMM the installed library does not offer on this GPU
        out["roofline"]["library_int8"] = {"tops": None, "error": str(e).splitlines()[0][:200]}
    del st
    torch.cuda.empty_cache()
    return out


def decode16_stage(torch, qg, pk, replays=STAGE_REPLAYS):
    """The LLaMA-3.1-8B MLP decode at 16 tokens (PoT): a whole step and each distinct linear."""
    from w2a4_gemm_b200 import synth
    wl = synth.LLAMA31_8B_MLP_DECODE16
    copies, _ = decode_copies(wl)
    st = OursState(wl, torch, qg, copies)
    T = wl.tokens
    by = sum(linear_bytes(T, l.n_out, l.n_in, 2, wl.levelset) for l in wl.linears)
    out = {"workload": wl.name,
           "step": stage_record(chain_stats(torch, st.step, 50, replays), bytes_=by, pk=pk,
                                what="qift_quantize_acts x2 + qift_linear x3")}
    seen = set()
    for L in st.layers:
        key = (L["lin"].n_out, L["lin"].n_in)
        if key in seen:
            continue
        seen.add(key)
        out[L["lin"].name] = linear_stage(torch, qg, st, L, pk, STAGE_LAUNCHES, replays, T, 2)
    g = out["gate_proj"]
    out["roofline"] = {"bound": "hbm", "achieved": g["GB/s"], "peak": pk["hbm_gbs"], "unit": "GB/s",
                       "frac": g["frac_hbm"], "traffic": profiled_traffic("decode16"),
                       "kernel": "skinny_kernel (qift_linear, gate_proj 14336x4096, 16 tokens, PoT)",
                       "peak_source": pk["source"] + " copy bandwidth, burst"}
    del st
    torch.cuda.empty_cache()
    return out


def run_ours(args, rank, world):
    import torch
    import w2a4_gemm_b200 as qg
    from w2a4_gemm_b200 import build
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    build.build()
    qg.lib()
    torch.cuda.set_device(rank % torch.cuda.device_count())
    wl = workload_def(args.workload)
    pk = peaks()
    T = wl.tokens
    decode = T <= 16
    copies, wbytes = decode_copies(wl) if decode else (3, 0)
    st = OursState(wl, torch, qg, copies)
    out_b = 2 if wl.out_dtype == "f16" else 4
    step_bytes = sum(linear_bytes(T, l.n_out, l.n_in, out_b, wl.levelset) for l in wl.linears)
    step_ops = sum(2 * T * l.n_out * l.n_in for l in wl.linears)

    for i in range(args.warmup):
        st.step(i)
    torch.cuda.synchronize()

    # The timed region: exactly `steps` steps, captured as one CUDA graph and replayed once
    # (after one untimed replay that uploads it), CUDA events on the replaying stream.
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    g_steps = capture(torch, st.step, args.steps, offset=args.warmup)
    g_steps.replay()  # upload and warm the graph itself (not timed)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    with ClockSampler(torch.cuda.current_device()) as clk:
        secs = max_over_ranks(time_graph(torch, g_steps), world)
    clocks = clk.summary()
    del g_steps

    # Per-kernel live timing: chains of one kernel over the same cycled inputs, a fixed number
    # of launches whatever --steps is, the median of STAGE_REPLAYS replays with its spread.
    L0 = st.layers[0]
    lin0 = L0["lin"]
    N0, K0 = lin0.n_out, lin0.n_in
    reps = STAGE_LAUNCHES if decode else 30
    a_fn = lambda i: qg.qift_quantize_acts(L0["x"][i % copies], wl.a_block, out_q=L0["q"][i % copies],
                                           out_scales=L0["sa"][i % copies])
    stages = {
        "a3a4_quantize_acts": stage_record(chain_stats(torch, a_fn, reps, STAGE_REPLAYS),
                                           bytes_=acts_bytes(T, K0), pk=pk),
        "a5_linear": linear_stage(torch, qg, st, L0, pk, reps, STAGE_REPLAYS, T, out_b),
    }
    lin_b = stages["a5_linear"]["bytes"]
    if T <= 4 and K0 % 64 == 0 and K0 <= 16384 and wl.levelset in ("qift", "pot", "int4"):
        f_fn = lambda i: qg.qift_decode_linear(L0["x"][i % copies], wl.a_block, L0["codes"][i % copies],
                                               L0["s_w"][i % copies], wl.levelset, st.out_dt,
                                               out=L0["y"][i % copies])
        fb = 2 * T * K0 + code_bytes(N0, K0, wl.levelset) + 4 * N0 + T * N0 * out_b  # x in, codes, scales, y out
        stages["a3a4a5_fused_decode"] = stage_record(chain_stats(torch, f_fn, reps, STAGE_REPLAYS), bytes_=fb,
                                                     pk=pk, entry="qift_decode_linear (one launch)")
    W, _ = st.offline[0]
    w_rot = torch.empty_like(W)
    rot_b = 8 * N0 * K0
    stages["a1_rotate_weights"] = stage_record(
        chain_stats(torch, lambda i: qg.qift_rotate(W, wl.w_block, out=w_rot), 5, 5), bytes_=rot_b, pk=pk)
    qw = chain_stats(torch, lambda i: qg.qift_quantize_weights(w_rot, wl.levelset, with_mse=False), 2, 3)
    stages["a2_quantize_weights"] = stage_record(qw, bound="alu", weights_per_s=N0 * K0 / qw["s"],
                                                 candidate_evals_per_s=N0 * K0 * 100 / qw["s"])

    a5 = stages["a5_linear"]
    if decode:
        value = world * step_bytes * args.steps / secs / 1e9
        unit = "GB/s"
        roof = {"bound": "hbm", "achieved": a5["GB/s"], "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": a5["frac_hbm"], "traffic": profiled_traffic(args.workload),
                "kernel": ("qift_linear, 4-bit weights (" + ("CUDA-core GEMV" if T == 1 else "tensor-core skinny GEMM")
                           + ")") if wl.levelset == "int4" else "qift_linear (GEMV)",
                "launch_us": a5["us"], "launch_us_spread": [a5["us_min"], a5["us_max"]],
                "timing": f"median of {STAGE_REPLAYS} replays of a CUDA graph of {reps} back-to-back launches",
                "peak_source": pk["source"] + " copy bandwidth, burst"}
    else:
        value = world * step_ops * args.steps / secs / 1e12
        unit = "TOPS"
        roof = {"bound": "tensor", "achieved": a5["TOPS"], "peak": pk["int8_tops"], "unit": "TOPS",
                "frac": a5["frac_int8"], "traffic": profiled_traffic(args.workload),
                "kernel": "qift_linear (GEMM)", "launch_us": a5["us"],
                "launch_us_spread": [a5["us_min"], a5["us_max"]],
                "timing": f"median of {STAGE_REPLAYS} replays of a CUDA graph of {reps} back-to-back launches",
                "peak_source": pk["source"] + " bf16 burst x 2 (int8 nominal ratio)"}
        try:
            lib_tops = library_int8_tops(torch)
            roof["library_int8"] = {"tops": lib_tops, "frac": a5["TOPS"] / lib_tops,
                                    "what": "torch._int_mm (the vendor int8 GEMM) at 8192^3, best of 10, same run"}
        except RuntimeError as e:  # an int8 GEMM the installed library does not offer on this GPU
            roof["library_int8"] = {"tops": None, "error": str(e).splitlines()[0][:200]}

    # End to end through the public API: every step copies its x from pinned host memory to the
    # device, runs the calls and copies y back to pinned host memory.  As in a serving loop the
    # copies run on their own streams and overlap the neighbouring steps' kernels: the inputs of
    # step i go in while earlier steps compute, at most `depth` steps ahead and never into a
    # device slot an unfinished step still reads; y of step i comes back while later steps
    # compute, and a step whose output slot is still being copied out waits for that copy.  The
    # whole pipeline is one CUDA graph timed between events on the capture stream.
    hx = [torch.from_numpy(wl.x(L["lin"])).pin_memory() if L["quant"] else None for L in st.layers]
    hy = [torch.empty((T, L["lin"].n_out), dtype=st.out_dt).pin_memory() for L in st.layers]
    h2d_s, d2h_s = torch.cuda.Stream(), torch.cuda.Stream()

    depth = min(4, copies)

    def e2e_pipeline(n, offset):
        cur = torch.cuda.current_stream()
        h2d_s.wait_stream(cur)
        d2h_s.wait_stream(cur)
        done, out_done = [], []
        for i in range(n):
            c = (offset + i) % copies
            if i >= depth:
                h2d_s.wait_event(done[i - depth])
            ein = torch.cuda.Event()
            with torch.cuda.stream(h2d_s):
                for j, L in enumerate(st.layers):
                    if L["quant"]:
                        L["x"][c].copy_(hx[j], non_blocking=True)
                ein.record(h2d_s)
            cur.wait_event(ein)
            if i >= copies:
                cur.wait_event(out_done[i - copies])  # y slot c is free again
            for j, L in enumerate(st.layers):
                if L["quant"]:
                    qg.qift_quantize_acts(L["x"][c], wl.a_block, out_q=L["q"][c], out_scales=L["sa"][c])
                qg.qift_linear(L["q"][c], L["sa"][c], L["codes"][c], L["s_w"][c], wl.levelset, st.out_dt,
                               out=L["y"][c])
            eout = torch.cuda.Event()
            eout.record(cur)
            done.append(eout)
            d2h_s.wait_event(eout)
            eod = torch.cuda.Event()
            with torch.cuda.stream(d2h_s):
                for j, L in enumerate(st.layers):
                    hy[j].copy_(L["y"][c], non_blocking=True)
                eod.record(d2h_s)
            out_done.append(eod)
        cur.wait_stream(h2d_s)
        cur.wait_stream(d2h_s)

    e2e_pipeline(args.warmup, 0)
    torch.cuda.synchronize()
    g_e2e = capture(torch, lambda off: e2e_pipeline(args.steps, off), 1, offset=args.warmup)
    g_e2e.replay()  # upload and warm the graph itself (not timed)
    torch.cuda.synchronize()
    e2e_secs = max_over_ranks(time_graph(torch, g_e2e), world)
    del g_e2e
    h2d = sum(x.numel() * x.element_size() for x in hx if x is not None)
    d2h = sum(y.numel() * y.element_size() for y in hy)
    e2e_val = world * (step_bytes if decode else step_ops) * args.steps / e2e_secs / (1e9 if decode else 1e12)

    # The default (decode) run also records the other two online configurations, so that one
    # run measures both halves of the metric: the 2048-token prefill GEMM (TOPS against the
    # int8 peak) and the 16-token PoT MLP decode (GB/s against HBM).
    launches = st.launches_per_step() * args.steps
    if args.workload == "decode" and not args.no_extra_stages:
        del st
        torch.cuda.empty_cache()
        stages["prefill"] = prefill_stage(torch, qg, pk)
        stages["decode16"] = decode16_stage(torch, qg, pk)

    line = {
        "metric": METRIC, "value": value, "unit": unit, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "int8", "data": "synthetic",
        "config": {"workload": wl.name, "description": wl.description, "tokens": T,
                   "linears": [[l.name, l.n_out, l.n_in] for l in wl.linears], "levelset": wl.levelset,
                   "hadamard_block": wl.a_block, "out_dtype": wl.out_dtype,
                   "parallelism": f"replicas{world}" if world > 1 else "single",
                   "l2": (f"inputs larger than L2: {copies} weight copies ({copies * wbytes / 1e6:.0f} MB codes) "
                          "cycled step to step") if decode else "inputs larger than L2 (activations + outputs)",
                   "step": "qift_quantize_acts once per distinct input (gate and up share theirs) + "
                           "qift_linear per linear; weights quantized offline"},
        "roofline": roof, "e2e": {"value": e2e_val, "unit": unit, "h2d_bytes_per_step": h2d,
                                  "d2h_bytes_per_step": d2h,
                                  "copies": "pinned host <-> device every step, on their own streams, "
                                            f"overlapping the neighbouring steps' kernels ({depth} steps deep)"},
        "gpu_launches": launches, "clocks": clocks, "stages": stages,
    }
    return line


# ------------------------------------------------------------------------- CPU oracle arm
def oracle_step_fn(wl, sample_tokens):
    """Returns (step callable, bytes or ops per step, description) for the CPU oracle."""
    import oracle
    prepared = []
    seen = set()
    for lin in wl.linears:
        W = wl.w(lin)
        if wl.levelset == "int4":
            codes, s_w, _, _ = oracle.quantize_weights_w4(oracle.rotate_f32(W, wl.w_block))
        else:
            codes, s_w, _, _ = oracle.quantize_weights(oracle.rotate_f32(W, wl.w_block), wl.levelset)
        x = wl.x(lin)[:sample_tokens]
        key = (lin.x_seed, lin.n_in)  # linears reading the same input share one quantization
        prepared.append((lin, codes, s_w, x, key not in seen))
        seen.add(key)

    def step():
        q = sa = None
        for lin, codes, s_w, x, quant in prepared:
            if quant:
                q, sa, _ = oracle.quantize_acts(x, wl.a_block)
            if wl.levelset == "int4":
                oracle.linear_w4(q, sa, codes, s_w, np.float16)
            else:
                oracle.linear(q, sa, codes, s_w, wl.levelset, np.float16)

    return step, prepared


def time_cpu_steps(step, budget_s):
    """Seconds per oracle step (one untimed step first) over about budget_s; and the count."""
    step()
    n, t0 = 0, time.perf_counter()
    while True:
        step()
        n += 1
        if time.perf_counter() - t0 > budget_s:
            break
    return (time.perf_counter() - t0) / n, n


def cpu_baseline_obj(wl, budget_s=10.0):
    """The oracle on every host core, then (a quarter of the budget) on one core."""
    import oracle
    T = 1
    decode = wl.tokens <= 16
    step, prepared = oracle_step_fn(wl, T)
    by = sum(linear_bytes(T, p[0].n_out, p[0].n_in, 2, wl.levelset) for p in prepared)
    ops = sum(2 * T * p[0].n_out * p[0].n_in for p in prepared)
    secs, n = time_cpu_steps(step, budget_s)
    all_cores = oracle.threads()
    oracle.set_threads(1)
    try:
        secs1, n1 = time_cpu_steps(step, budget_s / 4)
    finally:
        oracle.set_threads(all_cores)
    rate = (lambda sec: by / sec / 1e9) if decode else (lambda sec: ops / sec / 1e12)
    return {"value": rate(secs), "unit": "GB/s" if decode else "TOPS", "cores": all_cores, "kind": "oracle",
            "sample": f"{n} oracle steps of {T} token(s) over all linears of the workload "
                      f"(quantize_acts + linear in plain C); {secs * 1e3:.1f} ms per step",
            "single_core": {"value": rate(secs1), "cores": 1, "sample": f"{n1} steps, {secs1 * 1e3:.1f} ms per step"}}


def run_reference(args):
    # The oracle as it stands, one token per step (a bounded sample of the workload).
    wl = workload_def(args.workload)
    T = 1
    decode = wl.tokens <= 16
    step, prepared = oracle_step_fn(wl, T)
    for _ in range(min(args.warmup, 3)):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    secs = (time.perf_counter() - t0)
    by = sum(linear_bytes(T, l.n_out, l.n_in, 2, wl.levelset) for l, *_ in prepared)
    ops = sum(2 * T * l.n_out * l.n_in for l, *_ in prepared)
    val = (by if decode else ops) * args.steps / secs / (1e9 if decode else 1e12)
    unit = "GB/s" if decode else "TOPS"
    import oracle
    return {"impl": "reference", "metric": METRIC, "value": val, "unit": unit, "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "int64", "data": "synthetic",
            "config": {"workload": wl.name, "tokens_per_step": T},
            "cpu_baseline": {"value": val, "unit": unit, "cores": oracle.threads(), "kind": "oracle",
                             "sample": f"{args.steps} oracle steps of {T} token(s)"},
            "e2e": {"value": val, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ------------------------------------------------------------------ offline (8B-shaped model)
ALU_EVAL_INSTR = 6  # compare, select, subtract, square, widen to fp64, fp64 add per candidate


def alu_peak_evals(sm_mhz=1965.0, sms=148):
    """Issue-bound peak of candidate evaluations per second: 4 schedulers x 32 lanes per SM."""
    return sms * 4 * 32 * sm_mhz * 1e6 / ALU_EVAL_INSTR


def excess_kurtosis(x) -> float:
    """Excess kurtosis E[(x - mean)^4] / var^2 - 3 of all entries of a tensor, in float64 (0 for a
    Gaussian; the Hadamard rotation should bring heavy-tailed rows towards it)."""
    d = x.double().flatten()
    d = d - d.mean()
    v = (d * d).mean()
    return float((d ** 4).mean() / (v * v) - 3.0)


def per_projection_mse(mods, row_mse_by_set):
    """Reconstruction MSE per projection name over all layers: {set: {proj: mse}}.  row_mse_by_set
    maps a set to one array of per-row MSEs per module, aligned with `mods` (layer, proj, n_out,
    n_in, seed)."""
    out = {}
    for ls, per_mod in row_mse_by_set.items():
        num, den = {}, {}
        for (_, proj, n_out, n_in, _), m in zip(mods, per_mod):
            num[proj] = num.get(proj, 0.0) + float(np.asarray(m, dtype=np.float64).sum()) * n_in
            den[proj] = den.get(proj, 0) + n_out * n_in
        out[ls] = {p: num[p] / den[p] for p in num}
    return out


def run_offline(args, rank, world):
    import torch
    import w2a4_gemm_b200 as qg
    from w2a4_gemm_b200 import build, synth
    build.build()
    qg.lib()
    torch.cuda.set_device(rank % torch.cuda.device_count())
    dev = torch.device("cuda")
    mods = synth.model_8b_modules()
    # Weights resident in HBM before timing (27.9 GB fp32), drawn on the device, seeded.
    W = [synth.weights_t4_device(n_out, n_in, seed, dev) for (_, _, n_out, n_in, seed) in mods]
    torch.cuda.synchronize()
    biggest = max(w.numel() for w in W)
    rot = torch.empty(biggest, dtype=torch.float32, device=dev)
    codes = torch.empty(biggest // 16, dtype=torch.int32, device=dev)
    scales = torch.empty(max(w.shape[0] for w in W), dtype=torch.float32, device=dev)
    mse = {ls: [torch.empty(w.shape[0], dtype=torch.float64, device=dev) for w in W] for ls in ("qift", "pot", "std")}
    L = qg.lib()

    def step(_i):
        for j, w in enumerate(W):
            n_out, n_in = w.shape
            r = rot[: w.numel()].view(n_out, n_in)
            qg.qift_rotate(w, synth.MODEL_8B_BLOCK, out=r)
            for ls in ("qift", "pot", "std"):
                st = L.qift_quantize_weights(qg._ptr(r), n_out, n_in, qg.LEVELSETS[ls], 100, 0.2, 1.0,
                                             qg._ptr(codes), qg._ptr(scales), qg._ptr(mse[ls][j]),
                                             qg._stream(None))
                qg._check(st, "qift_quantize_weights")

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    s0, e0 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clk:
        torch.cuda.synchronize()
        s0.record()
        for i in range(args.steps):
            step(i)
        e0.record()
        torch.cuda.synchronize()
        secs = max_over_ranks(s0.elapsed_time(e0) / 1e3, world)
    clocks = clk.summary()
    n_w = sum(w.numel() for w in W)
    value = world * 3 * n_w * args.steps / secs
    set_mse = {ls: float(sum((m * w.shape[1]).sum().item() for m, w in zip(mse[ls], W)) / n_w) for ls in mse}
    # The comparison baseline the page names (conventional asymmetric W2), outside the timed
    # region: the same rotation and candidate grid, with a per-row zero point.
    zeros = torch.empty(max(w.shape[0] for w in W), dtype=torch.int32, device=dev)
    asym_rows = []
    for w in W:
        n_out, n_in = w.shape
        r = rot[: w.numel()].view(n_out, n_in)
        qg.qift_rotate(w, synth.MODEL_8B_BLOCK, out=r)
        m_asym = torch.empty(n_out, dtype=torch.float64, device=dev)
        qg._check(L.qift_quantize_weights_asym(qg._ptr(r), n_out, n_in, 100, 0.2, 1.0, qg._ptr(codes),
                                               qg._ptr(scales), qg._ptr(zeros), qg._ptr(m_asym),
                                               qg._stream(None)), "qift_quantize_weights_asym")
        asym_rows.append(m_asym.cpu().numpy())
    set_mse["asym"] = float(sum(float(m.sum()) * w.shape[1] for m, w in zip(asym_rows, W)) / n_w)
    rows_by_set = {ls: [m.cpu().numpy() for m in mse[ls]] for ls in mse}
    rows_by_set["asym"] = asym_rows
    proj_mse = per_projection_mse(mods, rows_by_set)
    # Kurtosis of layer 0's projections before and after the rotation (a diagnostic of the
    # Gaussianisation the rotation is there for), outside the timed region.
    kurt = {}
    for j, (layer, proj, n_out, n_in, _) in enumerate(mods):
        if layer != 0:
            break
        r = rot[: W[j].numel()].view(n_out, n_in)
        qg.qift_rotate(W[j], synth.MODEL_8B_BLOCK, out=r)
        kurt[proj] = {"before": excess_kurtosis(W[j]), "after": excess_kurtosis(r)}

    # Live per-kernel timing of the two offline kernels on the largest module.
    wbig = max(W, key=lambda w: w.numel())
    n_out, n_in = wbig.shape
    rb = rot[: wbig.numel()].view(n_out, n_in)
    t_rot = time_region(torch, lambda i: qg.qift_rotate(wbig, synth.MODEL_8B_BLOCK, out=rb), 5) / 5
    t_qw = time_region(torch, lambda i: L.qift_quantize_weights(qg._ptr(rb), n_out, n_in, 0, 100, 0.2, 1.0,
                                                                qg._ptr(codes), qg._ptr(scales), None,
                                                                qg._stream(None)), 3) / 3
    t_fused = time_region(torch, lambda i: qg._check(L.qift_rotate_quantize_weights(
        qg._ptr(wbig), n_out, n_in, synth.MODEL_8B_BLOCK, 0, 100, 0.2, 1.0, qg._ptr(codes), qg._ptr(scales), None,
        qg._stream(None)), "qift_rotate_quantize_weights"), 3) / 3
    evals = n_out * n_in * 100 / t_qw
    sm_mhz = (clocks or {}).get("sm_mhz") or 1965.0
    peak = alu_peak_evals(sm_mhz)
    rot_b = 8 * wbig.numel()
    return {
        "metric": METRIC, "value": value, "unit": "weights/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32+f64", "data": "synthetic",
        "config": {"workload": "offline_8b_model_224_modules",
                   "description": "rotate (128-block) + 100-point scale search + encode + pack of all 224 "
                                  "linear modules of an 8B-shaped model, for each of the Qift, PoT and standard "
                                  "level sets; Student-t(4)*0.02 weights drawn on the device",
                   "weights": n_w, "level_sets": ["qift", "pot", "std"], "grid_points": 100,
                   "mse_baseline": "asym: conventional asymmetric W2 (scale + zero point), not timed",
                   "l2": "inputs larger than L2 (27.9 GB of fp32 weights)",
                   "reconstruction_mse": set_mse, "reconstruction_mse_per_projection": proj_mse,
                   "excess_kurtosis_layer0": kurt,
                   "parallelism": f"replicas{world}" if world > 1 else "single"},
        "roofline": {"bound": "alu", "achieved": evals / 1e12, "peak": peak / 1e12, "unit": "T candidate-evals/s",
                     "frac": evals / peak, "traffic": profiled_traffic("offline"),
                     "kernel": "quant_weights_kernel (qift_quantize_weights)",
                     "peak_source": f"issue-bound: 148 SMs x 128 lanes x {sm_mhz:.0f} MHz / {ALU_EVAL_INSTR} "
                                    "instructions per candidate evaluation"},
        "e2e": None, "gpu_launches": len(W) * 4 * args.steps, "clocks": clocks,
        "stages": {"a1_rotate_weights": {"ms": t_rot * 1e3, "GB/s": rot_b / t_rot / 1e9,
                                         "frac_hbm": rot_b / t_rot / 1e9 / peaks()["hbm_gbs"], "bound": "hbm"},
                   "a2_quantize_weights": {"ms": t_qw * 1e3, "candidate_evals_per_s": evals, "bound": "alu",
                                           "frac_alu": evals / peak},
                   "a1a2_fused_rotate_quantize": {"ms": t_fused * 1e3, "two_calls_ms": (t_rot + t_qw) * 1e3,
                                                  "entry": "qift_rotate_quantize_weights (one level set)"}},
    }


def offline_cpu_baseline(budget_s=10.0):
    """The oracle's rotate + quantize (three level sets) on a bounded sample of module rows, on
    every host core and then (a quarter of the budget) on one core."""
    import oracle
    from w2a4_gemm_b200 import synth
    rows = 16
    sample = [synth.weights(rows, n_in, (seed,)) for (_, _, _, n_in, seed) in synth.model_8b_modules()[:7]]

    def rate(budget):
        n, t0 = 0, time.perf_counter()
        while True:
            for w in sample:
                wr = oracle.rotate_f32(w, synth.MODEL_8B_BLOCK)
                for ls in ("qift", "pot", "std"):
                    oracle.quantize_weights(wr, ls)
                n += 3 * w.size
            if time.perf_counter() - t0 > budget:
                break
        secs = time.perf_counter() - t0
        return n / secs, secs

    all_cores = oracle.threads()
    val, secs = rate(budget_s)
    oracle.set_threads(1)
    try:
        val1, secs1 = rate(budget_s / 4)
    finally:
        oracle.set_threads(all_cores)
    return {"value": val, "unit": "weights/s", "cores": all_cores, "kind": "oracle",
            "sample": f"{rows} rows of each of the 7 projections of one layer, 3 level sets, repeated for "
                      f"{secs:.1f} s",
            "single_core": {"value": val1, "cores": 1, "sample": f"the same, repeated for {secs1:.1f} s"}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["decode", "decode16", "prefill", "single", "offline", "decode_w4",
                                           "decode16_w4", "prefill_w4"], default="decode")
    ap.add_argument("--cpu-budget", type=float, default=10.0)
    ap.add_argument("--no-extra-stages", action="store_true",
                    help="decode workload only: skip the prefill and 16-token decode stages")
    args = ap.parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)))
        return

    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", rank)))
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    if args.workload == "offline":
        line = run_offline(args, rank, world)
    else:
        line = run_ours(args, rank, world)
    if rank == 0:
        if world == 1:
            line["cpu_baseline"] = (offline_cpu_baseline(args.cpu_budget) if args.workload == "offline"
                                    else cpu_baseline_obj(workload_def(args.workload), args.cpu_budget))
        else:
            line["cpu_baseline"] = None
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
