#!/usr/bin/env python
"""Throughput of the block-scaled FP4 hot path on B200.

Headline workload (one step): NVFP4 two-level quantisation of an 8192 x 8192 bf16 activation
(N(0,1) with 0.1% of the columns x U(50,100), seed 5), once plain and once with adaptive 4/6 —
each a two-pass call (tensor amax, then per-block E4M3 scale + E2M1 encode + pack).  The value is
algorithmic GB/s: 4.5625 bytes per element per call (2 amax read + 2 read + 0.5 nibbles + 1/16
scale) over the device time of the step.  Secondary lines measure the other workloads (MXFP4
quantise + dequantise, fused Walsh-Hadamard + NVFP4 with stochastic rounding, the NVFP4 and MXFP4
block-scaled GEMMs and the down_proj quantise + GEMM pipeline).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--no-secondary]

With --gpus N > 1 the bench runs one process per GPU: under torchrun it reads RANK, LOCAL_RANK and
WORLD_SIZE (which must equal N); started alone it spawns the N ranks itself (127.0.0.1 rendezvous).
Every rank quantises its own copy of the workload (independent problems, weak scaling, no
collective on the data path); the step time is the max over ranks.
Timing: CUDA events on the launching stream per step, L2 flushed (a 256 MiB write) before every
timed step, outside the events; clocks sampled with nvidia-smi during the timed loop.
"""
from __future__ import annotations

import argparse
import ctypes
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import block_scaled_fp4_amax_b200 as fp4  # noqa: E402
from block_scaled_fp4_amax_b200 import synth  # noqa: E402

METRIC = "FP4 quantize GB/s vs HBM peak; block-scaled FP4 GEMM TFLOPS vs FP4 peak"
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
NV_BYTES_2PASS = 4.5625     # bytes per element, two-pass NVFP4 (bf16 in)
NV_BYTES_1PASS = 2.5625     # bytes per element, one quantise launch (bf16 in)
PROFILE_DIR = os.path.join(ROOT, "profiles")


# ---------------------------------------------------------------------------------------------
def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        d["source"] = "measured"
        return d
    d = dict(FALLBACK)
    d["source"] = "fallback"
    return d


def profile_value(name, key):
    """A `key: value` figure recorded in profiles/<name>.md (from that kernel's ncu capture), if any."""
    path = os.path.join(PROFILE_DIR, name + ".md")
    if not os.path.exists(path):
        return None
    for ln in open(path):
        if ln.startswith(key + ":"):
            v = ln.split(":", 1)[1].strip()
            return None if v in ("", "null") else float(v)
    return None


def profile_traffic(name):
    """Per-launch DRAM bytes (read + write) recorded in profiles/<name>.md, if any."""
    return profile_value(name, "traffic_bytes_per_launch")


class Clocks:
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.p = None

    def start(self):
        try:
            self.p = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                                       "--format=csv,noheader,nounits", "-lms", "50"],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None
        time.sleep(0.3)

    def stop(self, t0, t1):
        if self.p is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.1)
        self.p.terminate()
        self.p.wait()
        self.f.flush()
        rows = []
        for ln in open(self.f.name):
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 10:
                continue
            try:
                ts = time.mktime(time.strptime(parts[0].split(".")[0], "%Y/%m/%d %H:%M:%S"))
            except ValueError:
                continue
            rows.append((ts, parts))
        load = [p for ts, p in rows if t0 - 1 <= ts <= t1 + 1] or [p for _, p in rows]
        if not load:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(p[2]) for p in load if p[2].replace(".", "").isdigit()]
        mx = [float(p[3]) for p in load if p[3].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for p in load for i in range(4) if p[6 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(load)}


def _free_port():
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def _rank_main(local, world, port, argv):
    os.environ.update(RANK=str(local), LOCAL_RANK=str(local), WORLD_SIZE=str(world),
                      LOCAL_WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    main(argv)


def spawn_ranks(n, argv):
    """One process per GPU without an external launcher: N spawned ranks (no CUDA call in this
    parent before they start), each running main() with the torchrun environment set."""
    import torch.multiprocessing as tmp
    tmp.start_processes(_rank_main, args=(n, _free_port(), argv), nprocs=n, join=True, start_method="spawn")


def dist():
    """One process per GPU (torchrun env); NCCL on GPUs, gloo where there is no GPU (host tests)."""
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    if ws > 1:
        import datetime
        import torch.distributed as td
        local = int(os.environ.get("LOCAL_RANK", "0"))
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        td.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
        return td, td.get_rank(), ws, local
    return None, 0, 1, 0


def barrier(td):
    if td is not None:
        td.barrier()


def max_over_ranks(td, v):
    if td is None:
        return v
    dev = "cuda" if td.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    td.all_reduce(t, op=td.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world, bytes_per_rank_step, ms_step_max):
    """Whole-job GB/s: the bytes all ranks processed in a step over the slowest rank's step time."""
    return world * bytes_per_rank_step / (ms_step_max * 1e-3) / 1e9


def timed(fn, K, W, flush, td, events_per_step=True):
    """W warm-up calls, then K timed calls, each preceded by an L2 flush outside its events.
    Returns per-step device milliseconds."""
    s = torch.cuda.current_stream()
    for _ in range(W):
        flush()
        fn()
    barrier(td)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    for a, b in ev:
        flush()
        a.record(s)
        fn()
        b.record(s)
    torch.cuda.synchronize()
    barrier(td)
    return [a.elapsed_time(b) for a, b in ev]


# ---------------------------------------------------------------------------------------------
# Workloads (C-ABI calls on preallocated device buffers)

class NvStep:
    """One headline step: nvfp4_quantize(x) plain, then with four-over-six (two passes each)."""

    def __init__(self, x, dev):
        L = fp4.lib()
        self.L = L
        self.x = x
        rows, cols = x.shape
        self.rows, self.cols = rows, cols
        self.q = [torch.empty((rows, cols // 2), dtype=torch.uint8, device=dev) for _ in range(2)]
        self.s = [torch.empty(rows * cols // 16, dtype=torch.uint8, device=dev) for _ in range(2)]
        self.g = [torch.empty(1, dtype=torch.float32, device=dev) for _ in range(2)]
        self.c = [torch.empty(4, dtype=torch.int64, device=dev) for _ in range(2)]
        self.ws = torch.empty(fp4.workspace_size(fp4.OP_NVFP4_QUANTIZE), dtype=torch.uint8, device=dev)

    def call(self, i, four_six, global_in=None, counts=True):
        st = self.L.nvfp4_quantize(ctypes.c_void_p(self.x.data_ptr()), fp4.BF16, self.rows, self.cols, 16, fp4.RNE,
                                   int(four_six), 0, fp4.ROWMAJOR,
                                   None if global_in is None else ctypes.c_void_p(global_in.data_ptr()),
                                   ctypes.c_void_p(self.g[i].data_ptr()), ctypes.c_void_p(self.q[i].data_ptr()),
                                   ctypes.c_void_p(self.s[i].data_ptr()),
                                   ctypes.c_void_p(self.c[i].data_ptr()) if counts else None,
                                   ctypes.c_void_p(self.ws.data_ptr()), self.ws.numel(),
                                   ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        if st != 0:
            raise RuntimeError(self.L.fp4_last_error().decode())

    def __call__(self):
        self.call(0, False)
        self.call(1, True)

    launches_per_step = 4  # amax + quantise, twice


def run_ours(args, td, rank, world, local):
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    pk = peaks()
    flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def flush():
        flush_buf.zero_()

    x_cpu = synth.nv_outliers()
    x = x_cpu.to(dev)
    n = x.numel()
    step = NvStep(x, dev)

    clocks = Clocks(torch.cuda.current_device() if "CUDA_VISIBLE_DEVICES" not in os.environ else
                    os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local])
    clocks.start()
    t0 = time.time()
    ms = timed(step, args.steps, args.warmup, flush, td)
    t1 = time.time()
    clk = clocks.stop(t0, t1)
    ms_step = max_over_ranks(td, sum(ms) / len(ms))
    bytes_step = 2 * NV_BYTES_2PASS * n
    value = job_throughput(world, bytes_step, ms_step)

    traffic = profile_traffic("nvfp4_quantize_8192x8192")  # read before any timing
    ipe = profile_value("nvfp4_quantize_8192x8192", "thread_instructions_per_element")
    # dominant kernel: the quantise launch (4/6 variant), timed alone with a caller-fixed s_g (the
    # one derived in the step).  Without a counter buffer the call enqueues that launch and nothing
    # else (with one it first zeroes the counters on the stream); the instantiation is the same.
    g = step.g[1].clone()
    kms = timed(lambda: step.call(1, True, global_in=g, counts=False), args.steps, args.warmup, flush, td)
    k_ms = max_over_ranks(td, sum(kms) / len(kms))
    k_bytes = NV_BYTES_1PASS * n
    achieved = k_bytes / (k_ms * 1e-3) / 1e9
    roof = {"kernel": "quantize_kernel<bf16, NVFP4, RNE, 4/6> (one launch, 8192x8192)", "bound": "hbm",
            "timed": "CUDA events around the launch alone (no counter buffer, so no counter memset)",
            "achieved": round(achieved, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
            "frac": round(achieved / pk["hbm_gbs"], 4), "peak_source": pk["source"],
            "frac_of_nominal_8tbs": round(achieved / 8000.0, 4),
            "traffic": traffic, "traffic_source": "ncu dram__bytes_read.sum + dram__bytes_write.sum of one launch of "
                                                  "this kernel on this workload, profiles/nvfp4_quantize_8192x8192.md",
            "algorithmic_bytes_per_launch": k_bytes}
    if ipe:
        # the kernel is issue-bound: its ceiling at one warp instruction per scheduler per clock
        # (SMs x 4 schedulers x 32 lanes x the SM clock sampled under load), at the thread
        # instructions per element of its ncu capture
        mhz = clk.get("sm_mhz") or clk.get("sm_max_mhz") or 1965.0
        tips = torch.cuda.get_device_properties(dev).multi_processor_count * 4 * 32 * mhz * 1e6
        ceil_gbs = tips / ipe * NV_BYTES_1PASS / 1e9
        roof["issue_ceiling"] = {"thread_instructions_per_element": ipe,
                                 "source": "ncu smsp__thread_inst_executed.sum of one launch / elements, "
                                           "profiles/nvfp4_quantize_8192x8192.md",
                                 "thread_instructions_per_s": round(tips / 1e12, 2), "unit": "T/s",
                                 "ceiling_GB/s": round(ceil_gbs, 1), "frac_of_ceiling": round(achieved / ceil_gbs, 4)}

    # end to end through the public binding: pinned host input -> device -> both calls -> host
    host_in = x_cpu.pin_memory()
    host_q = [torch.empty((8192, 4096), dtype=torch.uint8).pin_memory() for _ in range(2)]
    host_s = [torch.empty(8192 * 512, dtype=torch.uint8).pin_memory() for _ in range(2)]
    host_g = [torch.empty(1, dtype=torch.float32).pin_memory() for _ in range(2)]
    xd = torch.empty_like(x)

    def e2e_step():
        xd.copy_(host_in, non_blocking=True)
        for i, fs in enumerate((False, True)):
            q, s, gg, c = fp4.nvfp4_quantize(xd, four_six=fs, workspace=step.ws)
            host_q[i].copy_(q, non_blocking=True)
            host_s[i].copy_(s, non_blocking=True)
            host_g[i].copy_(gg, non_blocking=True)

    ems = timed(e2e_step, max(3, args.steps // 10), args.warmup, flush, td)
    e_ms = max_over_ranks(td, sum(ems) / len(ems))
    e2e = {"value": round(job_throughput(world, bytes_step, e_ms), 1), "unit": "GB/s",
           "h2d_bytes_per_step": int(host_in.numel() * 2),
           "d2h_bytes_per_step": int(sum(t.numel() * t.element_size() for t in host_q + host_s + host_g)),
           "ms_per_step": round(e_ms, 4)}

    line = {"metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_step, 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16->e2m1 (fp32 arithmetic)",
            "data": "synthetic (seeded numpy; no dataset)",
            "config": {"workload": "NVFP4 two-level quantisation 8192x8192 bf16, N(0,1) + 0.1% outlier "
                                   "columns x U(50,100), seed 5; plain + adaptive 4/6, two passes each",
                       "rows": 8192, "cols": 8192, "block": 16, "global_scale": "amax/(6*448); 4/6: amax/(6*256)",
                       "l2": "flushed before every timed step (256 MiB write, outside the events)",
                       "parallelism": f"replicas x{world}"},
            "roofline": roof, "e2e": e2e, "gpu_launches": NvStep.launches_per_step * args.steps,
            "clocks": clk}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:  # the oracle baseline is a 1-GPU figure
        line["cpu_baseline"] = cpu_baseline(x_cpu)
    if not args.no_secondary:
        line["secondary"] = secondary(args, dev, flush, td, pk)
    return line


def _oracle_chunk(xs, g_plain, g46):
    """One thread's share of the all-cores oracle timing: plain then 4/6 on its rows, under the
    global scales of the whole sample (the single-threaded leg's), so the codes are the same."""
    import oracle as O
    O.nvfp4_quantize(xs, four_six=False, global_in=g_plain)
    O.nvfp4_quantize(xs, four_six=True, global_in=g46)
    return xs.shape[0]


def cpu_baseline(x_cpu, rows=4096, max_workers=64):
    """The oracle as it stands on the first `rows` rows of the workload: single-threaded (both
    passes of each call), then the quantise passes of the same rows split over one thread per host
    core, each thread given the sample's global scales from the single-threaded run.  The oracle is
    C called through ctypes, which releases the GIL for the call and keeps no global state, so the
    threads run in parallel."""
    import concurrent.futures as cf
    import oracle as O
    xs = synth.as_f32_numpy(x_cpu[:rows])
    t = time.perf_counter()
    g_plain = O.nvfp4_quantize(xs, four_six=False)[2]
    g46 = O.nvfp4_quantize(xs, four_six=True)[2]
    dt = time.perf_counter() - t
    b = 2 * NV_BYTES_2PASS * xs.size
    out = {"value": round(b / dt / 1e9, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
           "sample": f"first {rows} of 8192 rows (plain + 4/6, two passes each), {dt:.1f} s single-threaded C oracle"}
    n = max(1, min(os.cpu_count() or 1, max_workers, rows))
    chunks = np.array_split(xs, n)
    with cf.ThreadPoolExecutor(max_workers=n) as ex:
        t = time.perf_counter()
        done = sum(ex.map(lambda c: _oracle_chunk(c, g_plain, g46), chunks))
        dt_all = time.perf_counter() - t
    assert done == rows
    b1 = 2 * NV_BYTES_1PASS * xs.size
    out["all_cores"] = {"value": round(b1 / dt_all / 1e9, 4), "unit": "GB/s", "cores": n,
                        "sample": f"the same rows' quantise passes (plain + 4/6) over {n} threads under the "
                                  f"single-threaded run's global scales, {dt_all:.2f} s; bytes counted for one "
                                  f"pass per call"}
    return out


# ---------------------------------------------------------------------------------------------
def secondary(args, dev, flush, td, pk):
    out = []
    K = max(20, args.steps // 4)
    W = args.warmup
    # config 1: MXFP4 quantise + dequantise, 256 x 512 fp32
    x1 = synth.mx_small().to(dev)

    def c1():
        q, s, c = fp4.mx_quantize(x1)
        fp4.fp4_dequantize(q, s, fp4.MXFP4)

    ms = timed(c1, K, W, flush, td)
    t = statistics.median(ms)
    b = x1.numel() * (4 + 0.5 + 1 / 32) * 2
    out.append({"workload": "MXFP4 quantise + dequantise 256x512 fp32 (launch-bound, L2-resident)",
                "ms": round(t, 5), "GB/s": round(b / (t * 1e-3) / 1e9, 1)})
    # config 3: fused FWHT + NVFP4 + SR, 16384 x 8192 bf16
    x3 = synth.fwht_laplace().to(dev)
    ws = torch.empty(fp4.workspace_size(fp4.OP_FWHT_QUANTIZE), dtype=torch.uint8, device=dev)
    # the workspace that lets the two-pass call keep its fp32 rotation (rotate once)
    wsr = torch.empty(fp4.workspace_size(fp4.OP_FWHT_QUANTIZE_STORED, 16384, 8192), dtype=torch.uint8, device=dev)

    def c3():
        fp4.fwht_quantize(x3, fmt=fp4.NVFP4, round=fp4.STOCHASTIC, seed=7, workspace=wsr)

    ms = timed(c3, K, W, flush, td)
    t = statistics.median(ms)
    b = NV_BYTES_2PASS * x3.numel()
    out.append({"workload": "FWHT d=8192 + NVFP4 + stochastic rounding, 16384x8192 bf16, two passes",
                "route": "rotate once, fp32 rotation kept in the workspace (4 B/element each way beyond "
                         "the algorithmic bytes)",
                "ms": round(t, 4), "GB/s": round(b / (t * 1e-3) / 1e9, 1),
                "frac_hbm": round(b / (t * 1e-3) / 1e9 / pk["hbm_gbs"], 4)})
    ms = timed(lambda: fp4.fwht_quantize(x3, fmt=fp4.NVFP4, round=fp4.STOCHASTIC, seed=7, workspace=ws), K, W,
               flush, td)
    t = statistics.median(ms)
    out.append({"workload": "FWHT d=8192 + NVFP4 + stochastic rounding, 16384x8192 bf16, two passes",
                "route": "minimal workspace: each pass rotates", "ms": round(t, 4),
                "GB/s": round(b / (t * 1e-3) / 1e9, 1), "frac_hbm": round(b / (t * 1e-3) / 1e9 / pk["hbm_gbs"], 4)})
    # the same with the randomised rotation c*H*D (seeded sign bits, one 32-bit word per 32 channels)
    sg = torch.from_numpy(synth.rht_signs(8192, 33).view(np.int32)).to(dev)

    def c3r():
        fp4.fwht_quantize(x3, fmt=fp4.NVFP4, round=fp4.STOCHASTIC, seed=7, workspace=wsr, signs=sg)

    ms = timed(c3r, K, W, flush, td)
    t = statistics.median(ms)
    out.append({"workload": "randomised FWHT (c*H*D) d=8192 + NVFP4 + stochastic rounding, 16384x8192 bf16",
                "ms": round(t, 4), "GB/s": round(b / (t * 1e-3) / 1e9, 1),
                "frac_hbm": round(b / (t * 1e-3) / 1e9 / pk["hbm_gbs"], 4)})
    # the same randomised rotation into IF4 blocks (round to nearest)

    def c3i():
        fp4.fwht_quantize(x3, fmt=fp4.NVFP4, if4=True, workspace=wsr, signs=sg)

    ms = timed(c3i, K, W, flush, td)
    t = statistics.median(ms)
    out.append({"workload": "randomised FWHT (c*H*D) d=8192 + IF4 (E2M1 or INT4 per 16-block), 16384x8192 bf16",
                "ms": round(t, 4), "GB/s": round(b / (t * 1e-3) / 1e9, 1),
                "frac_hbm": round(b / (t * 1e-3) / 1e9 / pk["hbm_gbs"], 4)})
    del x3
    # SwiGLU fused ahead of the rotation: g, u bf16 [16384, 8192] read in both passes
    gg, uu = (t_.to(dev) for t_ in synth.swiglu_inputs(16384, 8192, seed=3))

    def c3s():
        fp4.swiglu_fwht_quantize(gg, uu, fmt=fp4.NVFP4, round=fp4.STOCHASTIC, seed=7, workspace=wsr)

    ms = timed(c3s, K, W, flush, td)
    t = statistics.median(ms)
    bs = (2 * 2 * 2 + 0.5 + 1 / 16) * gg.numel()
    out.append({"workload": "SiLU(g)*u -> FWHT d=8192 -> NVFP4 + stochastic rounding, 16384x8192 bf16 g and u",
                "ms": round(t, 4), "GB/s": round(bs / (t * 1e-3) / 1e9, 1),
                "frac_hbm": round(bs / (t * 1e-3) / 1e9 / pk["hbm_gbs"], 4)})
    del gg, uu, wsr
    # IF4 (E2M1 or INT4 per block) on the headline tensor: two passes, and the quantise pass alone
    xi = synth.nv_outliers().to(dev)
    gi = torch.empty(1, dtype=torch.float32, device=dev)
    wsq = torch.empty(fp4.workspace_size(fp4.OP_NVFP4_QUANTIZE), dtype=torch.uint8, device=dev)
    fp4.nvfp4_quantize(xi, if4=True, workspace=wsq)

    def cif4():
        fp4.nvfp4_quantize(xi, if4=True, workspace=wsq)

    ms = timed(cif4, K, W, flush, td)
    t = statistics.median(ms)
    gi.copy_(fp4.nvfp4_quantize(xi, workspace=wsq)[2])
    ms1 = timed(lambda: fp4.nvfp4_quantize(xi, if4=True, global_in=gi), K, W, flush, td)
    t1 = statistics.median(ms1)
    # the same quantise pass on N(0,1) without outliers (the rotated-data case IF4 is aimed at)
    xn = synth.normal_bf16(8192, 8192, 8)
    xn = xn.to(dev)
    gn = fp4.nvfp4_quantize(xn, workspace=wsq)[2].clone()
    msn = timed(lambda: fp4.nvfp4_quantize(xn, if4=True, global_in=gn), K, W, flush, td)
    tn = statistics.median(msn)
    out.append({"workload": "IF4 quantisation (E2M1 or INT4 per 16-block) 8192x8192 bf16 outliers, two passes",
                "ms": round(t, 4), "GB/s": round(NV_BYTES_2PASS * xi.numel() / (t * 1e-3) / 1e9, 1),
                "quantise_pass_ms": round(t1, 4),
                "quantise_pass_GB/s": round(NV_BYTES_1PASS * xi.numel() / (t1 * 1e-3) / 1e9, 1),
                "quantise_pass_frac_hbm": round(NV_BYTES_1PASS * xi.numel() / (t1 * 1e-3) / 1e9 / pk["hbm_gbs"], 4),
                "quantise_pass_gaussian_ms": round(tn, 4),
                "quantise_pass_gaussian_frac_hbm":
                    round(NV_BYTES_1PASS * xn.numel() / (tn * 1e-3) / 1e9 / pk["hbm_gbs"], 4)})
    # dequantisation of the headline tensor's NVFP4 encoding (4/6 codes), to bf16 and to fp32
    xd = synth.nv_outliers().to(dev)
    qd, sd, gd, _ = fp4.nvfp4_quantize(xd, four_six=True, workspace=wsq)
    del xd
    od = {torch.bfloat16: torch.empty((8192, 8192), dtype=torch.bfloat16, device=dev),
          torch.float32: torch.empty((8192, 8192), dtype=torch.float32, device=dev)}
    for dt_, nbytes in ((torch.bfloat16, 2), (torch.float32, 4)):
        ms = timed(lambda: fp4.fp4_dequantize(qd, sd, fp4.NVFP4, gd, out=od[dt_]), K, W, flush, td)
        t = statistics.median(ms)
        bd = qd.numel() * 2 * (0.5 + 1 / 16 + nbytes)
        out.append({"workload": f"NVFP4 dequantisation 8192x8192 to {'bf16' if nbytes == 2 else 'fp32'}",
                    "ms": round(t, 4), "GB/s": round(bd / (t * 1e-3) / 1e9, 1),
                    "frac_hbm": round(bd / (t * 1e-3) / 1e9 / pk["hbm_gbs"], 4)})
    del qd, sd, od

    # The FP4 dense peak is derived, not measured: the measured bf16 cuBLAS peak times the nominal
    # dense FP4 / BF16 ratio (9 / 2.25 PFLOP/s).  The datasheet's dense FP4 figure is given beside it.
    fp4_peak = 4.0 * pk["bf16_tflops"]
    fp4_datasheet = 9000.0
    # config 4: NVFP4 GEMM 8192^3
    A = fp4.nvfp4_quantize(synth.gemm_operand(8192, 8192, 1).to(dev), layout=fp4.MMA_TILED)
    B = fp4.nvfp4_quantize(synth.gemm_operand(8192, 8192, 2).to(dev), layout=fp4.MMA_TILED)
    C = torch.empty((8192, 8192), dtype=torch.bfloat16, device=dev)
    gws = torch.empty(256, dtype=torch.uint8, device=dev)
    ms = timed(lambda: fp4.fp4_block_gemm(fp4.NVFP4, A[0], A[1], B[0], B[1], A[2], B[2], out=C, workspace=gws),
               K, W, flush, td)
    t = statistics.median(ms)
    tf = 2 * 8192 ** 3 / (t * 1e-3) / 1e12
    out.append({"workload": "NVFP4 block-scaled GEMM M=N=K=8192 (E4M3 per 16, fp32 accumulate, bf16 out)",
                "ms": round(t, 4), "TFLOP/s": round(tf, 1), "frac_fp4_peak": round(tf / fp4_peak, 4),
                "fp4_peak": fp4_peak,
                "peak_source": f"derived: {pk['source']} bf16 burst x 4 (nominal dense FP4/BF16 ratio)",
                "frac_fp4_datasheet": round(tf / fp4_datasheet, 4),
                "fp4_datasheet": fp4_datasheet, "datasheet_source": "B200 dense FP4 9 PFLOP/s (NVIDIA, without sparsity)"})
    # the IF4 GEMM on the same operands quantised to IF4 blocks: fp16 expansion of both operands,
    # then the kind::f16 tensor-core GEMM (against the fp16/bf16 dense peak, the measured bf16 burst)
    del A, B
    A = fp4.nvfp4_quantize(synth.gemm_operand(8192, 8192, 1).to(dev), if4=True, layout=fp4.MMA_TILED)
    B = fp4.nvfp4_quantize(synth.gemm_operand(8192, 8192, 2).to(dev), if4=True, layout=fp4.MMA_TILED)
    iws = torch.empty(fp4.workspace_size(fp4.OP_BLOCK_GEMM_IF4, 16384, 8192), dtype=torch.uint8, device=dev)
    ms = timed(lambda: fp4.fp4_block_gemm(fp4.IF4, A[0], A[1], B[0], B[1], A[2], B[2], out=C, workspace=iws),
               K, W, flush, td)
    t = statistics.median(ms)
    tf = 2 * 8192 ** 3 / (t * 1e-3) / 1e12
    out.append({"workload": "IF4 GEMM M=N=K=8192 (IF4-quantised N(0,1) operands; fp16 expansion + kind::f16 GEMM)",
                "ms": round(t, 4), "TFLOP/s": round(tf, 1), "frac_f16_peak": round(tf / pk["bf16_tflops"], 4),
                "f16_peak": pk["bf16_tflops"],
                "peak_source": f"{pk['source']} bf16 burst (the fp16 dense rate is the same)"})
    del A, B, C, iws
    # config 5: MXFP4 down_proj, activations and weights quantised then GEMM, timed end to end
    a = synth.swiglu_act().to(dev)
    w = synth.weight().to(dev)
    C = torch.empty((4096, 8192), dtype=torch.bfloat16, device=dev)
    st = {}

    def c5():
        Aq = fp4.mx_quantize(a, layout=fp4.MMA_TILED)
        Bq = fp4.mx_quantize(w, layout=fp4.MMA_TILED)
        st["ab"] = (Aq, Bq)
        fp4.fp4_block_gemm(fp4.MXFP4, Aq[0], Aq[1], Bq[0], Bq[1], out=C, workspace=gws)

    # the weight quantise launch alone, into preallocated outputs (no allocation in the timed
    # region), timed before the GEMM loops so that their power state does not carry into it
    Bw = fp4.mx_quantize(w, layout=fp4.MMA_TILED)
    wout = (torch.empty_like(Bw[0]), torch.empty_like(Bw[1]), None, torch.empty_like(Bw[2]))
    ms = timed(lambda: fp4.mx_quantize(w, layout=fp4.MMA_TILED, out=wout), K, W, flush, td)
    t_w = statistics.median(ms)
    del Bw, wout
    ms = timed(c5, K, W, flush, td)
    t_all = statistics.median(ms)
    Aq, Bq = st["ab"]
    ms = timed(lambda: fp4.fp4_block_gemm(fp4.MXFP4, Aq[0], Aq[1], Bq[0], Bq[1], out=C, workspace=gws), K, W, flush, td)
    t_g = statistics.median(ms)
    flop = 2 * 4096 * 8192 * 28672
    qbytes = w.numel() * (2 + 0.5 + 1 / 32)
    out.append({"workload": "MXFP4 down_proj 4096x8192x28672: quantise activations + weights, then GEMM",
                "ms_end_to_end": round(t_all, 4), "gemm_ms": round(t_g, 4),
                "gemm_TFLOP/s": round(flop / (t_g * 1e-3) / 1e12, 1),
                "gemm_frac_fp4_peak": round(flop / (t_g * 1e-3) / 1e12 / fp4_peak, 4),
                "gemm_frac_fp4_datasheet": round(flop / (t_g * 1e-3) / 1e12 / fp4_datasheet, 4),
                "weight_quantise_GB/s": round(qbytes / (t_w * 1e-3) / 1e9, 1),
                "weight_quantise_frac_hbm": round(qbytes / (t_w * 1e-3) / 1e9 / pk["hbm_gbs"], 4),
                "end_to_end_TFLOP/s": round(flop / (t_all * 1e-3) / 1e12, 1)})
    # the same GEMM on the FP8 tensor-core route: E4M3 expansions of the MXFP4 operands, then
    # kind::mxf8f6f4 (the 1-SM kernel); against the dense FP8 peak, the measured bf16 peak x 2
    A8 = fp4.fp4_to_e4m3(Aq[0])
    B8 = fp4.fp4_to_e4m3(Bq[0])
    ms = timed(lambda: (fp4.fp4_to_e4m3(Aq[0], out=A8), fp4.fp4_to_e4m3(Bq[0], out=B8)), K, W, flush, td)
    t_x = statistics.median(ms)
    ms = timed(lambda: fp4.fp4_block_gemm_e4m3(A8, Aq[1], B8, Bq[1], out=C, workspace=gws), K, W, flush, td)
    t_8 = statistics.median(ms)
    fp8_peak = 2.0 * pk["bf16_tflops"]
    xbytes = (Aq[0].numel() + Bq[0].numel()) * 3  # read the nibbles, write twice as many bytes
    out.append({"workload": "MXFP4 down_proj 4096x8192x28672 on the FP8 route: E4M3 expansion, kind::mxf8f6f4 GEMM",
                "expand_ms": round(t_x, 4), "expand_GB/s": round(xbytes / (t_x * 1e-3) / 1e9, 1),
                "expand_frac_hbm": round(xbytes / (t_x * 1e-3) / 1e9 / pk["hbm_gbs"], 4),
                "gemm_ms": round(t_8, 4), "gemm_TFLOP/s": round(flop / (t_8 * 1e-3) / 1e12, 1),
                "gemm_frac_fp8_peak": round(flop / (t_8 * 1e-3) / 1e12 / fp8_peak, 4), "fp8_peak": fp8_peak,
                "peak_source": f"derived: {pk['source']} bf16 burst x 2 (nominal dense FP8/BF16 ratio)",
                "gemm_frac_fp8_datasheet": round(flop / (t_8 * 1e-3) / 1e12 / 4500.0, 4)})
    return out


# ---------------------------------------------------------------------------------------------
def run_reference(args, rank):
    """The oracle (plain C, single thread) on a bounded sample of the headline workload."""
    import oracle as O
    # about 2 s of single-threaded oracle work per 512 rows (plain + 4/6): size the per-step sample
    # so that the whole run stays near two minutes whatever --steps is
    rows = max(16, min(512, 30720 // max(1, args.steps)))
    x = synth.as_f32_numpy(synth.nv_outliers()[:rows])
    for _ in range(args.warmup):
        O.nvfp4_quantize(x[:64], four_six=False)
    ts = []
    for _ in range(args.steps):
        t = time.perf_counter()
        O.nvfp4_quantize(x, four_six=False)
        O.nvfp4_quantize(x, four_six=True)
        ts.append(time.perf_counter() - t)
    dt = statistics.mean(ts)
    b = 2 * NV_BYTES_2PASS * x.size
    v = round(b / dt / 1e9, 4)
    sample = f"first {rows} of 8192 rows per step (plain + 4/6), single-threaded C oracle"
    return {"impl": "reference", "metric": METRIC, "value": v, "unit": "GB/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(dt * 1e3, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "fp32 arithmetic (CPU)", "data": "synthetic (seeded numpy; no dataset)",
            "config": {"workload": "NVFP4 two-level quantisation 8192x8192 bf16, N(0,1) + 0.1% outlier columns "
                                   "x U(50,100), seed 5; plain + adaptive 4/6, two passes each", "rows_sampled": rows},
            "cpu_baseline": {"kind": "oracle", "cores": 1, "sample": sample, "value": v, "unit": "GB/s"},
            "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


CASES = ("nv", "nv46", "nv_amax", "if4", "mx", "fwht", "fwht_rht_if4", "swiglu_fwht", "gemm_nv", "gemm_mx",
         "gemm_e4m3", "gemm_if4", "dequant")


def run_case(name, reps):
    """Run one kernel on its full-size workload `reps` times (for profiler captures)."""
    dev = torch.device("cuda", 0)
    if name in ("nv", "nv46", "nv_amax", "if4"):
        x = synth.nv_outliers().to(dev)
        # the global scale the two-pass call derives for this mode, fixed, so that each rep is one
        # quantise launch on exactly the data the headline step quantises
        g = fp4.nvfp4_quantize(x, four_six=(name == "nv46"), if4=(name == "if4"))[2].clone()
        for _ in range(reps):
            if name == "nv_amax":
                fp4.nvfp4_quantize(x)
            else:
                fp4.nvfp4_quantize(x, four_six=(name == "nv46"), if4=(name == "if4"), global_in=g)
    elif name == "mx":
        a = synth.swiglu_act().to(dev)
        for _ in range(reps):
            fp4.mx_quantize(a, layout=fp4.MMA_TILED)
    elif name == "fwht":
        x = synth.fwht_laplace().to(dev)
        for _ in range(reps):
            fp4.fwht_quantize(x, fmt=fp4.NVFP4, round=fp4.STOCHASTIC, seed=7)
    elif name == "fwht_rht_if4":
        x = synth.fwht_laplace().to(dev)
        sg = torch.from_numpy(synth.rht_signs(8192, 33).view(np.int32)).to(dev)
        for _ in range(reps):
            fp4.fwht_quantize(x, fmt=fp4.NVFP4, if4=True, signs=sg)
    elif name == "swiglu_fwht":
        g, u = (t_.to(dev) for t_ in synth.swiglu_inputs(16384, 8192, seed=3))
        for _ in range(reps):
            fp4.swiglu_fwht_quantize(g, u, fmt=fp4.NVFP4, round=fp4.STOCHASTIC, seed=7)
    elif name == "gemm_if4":
        A = fp4.nvfp4_quantize(synth.gemm_operand(8192, 8192, 1).to(dev), if4=True, layout=fp4.MMA_TILED)
        B = fp4.nvfp4_quantize(synth.gemm_operand(8192, 8192, 2).to(dev), if4=True, layout=fp4.MMA_TILED)
        for _ in range(reps):
            fp4.fp4_block_gemm(fp4.IF4, A[0], A[1], B[0], B[1], A[2], B[2])
    elif name == "dequant":
        x = synth.nv_outliers().to(dev)
        q, s, g, _ = fp4.nvfp4_quantize(x)
        for _ in range(reps):
            fp4.fp4_dequantize(q, s, fp4.NVFP4, g, out_dtype=torch.bfloat16)
    elif name == "gemm_e4m3":
        A = fp4.mx_quantize(synth.swiglu_act().to(dev), layout=fp4.MMA_TILED)
        B = fp4.mx_quantize(synth.weight().to(dev), layout=fp4.MMA_TILED)
        A8, B8 = fp4.fp4_to_e4m3(A[0]), fp4.fp4_to_e4m3(B[0])
        for _ in range(reps):
            fp4.fp4_block_gemm_e4m3(A8, A[1], B8, B[1])
    elif name in ("gemm_nv", "gemm_mx"):
        if name == "gemm_nv":
            A = fp4.nvfp4_quantize(synth.gemm_operand(8192, 8192, 1).to(dev), layout=fp4.MMA_TILED)
            B = fp4.nvfp4_quantize(synth.gemm_operand(8192, 8192, 2).to(dev), layout=fp4.MMA_TILED)
            args = (fp4.NVFP4, A[0], A[1], B[0], B[1], A[2], B[2])
        else:
            A = fp4.mx_quantize(synth.swiglu_act().to(dev), layout=fp4.MMA_TILED)
            B = fp4.mx_quantize(synth.weight().to(dev), layout=fp4.MMA_TILED)
            args = (fp4.MXFP4, A[0], A[1], B[0], B[1])
        for _ in range(reps):
            fp4.fp4_block_gemm(*args)
    torch.cuda.synchronize()
    print(json.dumps({"case": name, "reps": reps, "ok": True}))


def dist_check(args):
    """The multi-rank plumbing alone (no GPU work): every rank reports a step time of 1 + rank/2 ms;
    rank 0 prints the world size, the max over ranks and the whole-job throughput of 1 GB per rank."""
    td, rank, world, _ = dist()
    try:
        barrier(td)
        m = max_over_ranks(td, 1.0 + 0.5 * rank)
        if rank == 0:
            print(json.dumps({"world": world, "max_ms": m, "GB/s": job_throughput(world, 1e9, m)}))
    finally:
        if td is not None:
            td.destroy_process_group()


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--case", choices=CASES, help="run one kernel on its workload (profiling)")
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-secondary", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--dist-check", action="store_true", help="run only the multi-rank helpers (no GPU work)")
    args = ap.parse_args(argv)
    env_world = os.environ.get("WORLD_SIZE")
    if env_world is None and args.gpus > 1:
        spawn_ranks(args.gpus, sys.argv[1:] if argv is None else argv)
        return
    if env_world is not None and int(env_world) != args.gpus:
        raise SystemExit(f"bench.py: WORLD_SIZE={env_world} but --gpus {args.gpus}")
    if args.dist_check:
        dist_check(args)
        return
    if args.case:
        run_case(args.case, args.reps)
        return
    args.warmup = max(args.warmup, 3)
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        if rank != 0:
            return
        print(json.dumps(run_reference(args, rank)))
        return
    td, rank, world, local = dist()
    try:
        line = run_ours(args, td, rank, world, local)
        if rank == 0:
            print(json.dumps(line))
    finally:
        if td is not None:
            td.destroy_process_group()


if __name__ == "__main__":
    main()
