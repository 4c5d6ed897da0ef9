#!/usr/bin/env python3
"""Benchmark of the fine-grained-scaled FP8 GEMM on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one GEMM call over the headline workload (the decode-shaped dense
problem M=128, N=2112, K=7168, the shape the DeepGEMM pages quote their
largest speed-up on) with inputs resident in HBM.  L2 is flushed (a 512 MiB
write) before every timed launch and each launch is timed alone with CUDA
events on its stream.  Rank 0 prints one JSON line with the headline value,
a roofline object for the GEMM kernel, the end-to-end number through the
public API with host buffers, the CPU oracle as a baseline, the SM clocks seen
under load and the per-shape numbers of all five workloads.

With N>1 (torchrun, one process per GPU) each rank runs its own replica of
the workload (the dense GEMM has no exchange step: replicas only), the time is
the max over ranks and the value counts the work of all ranks.

--impl reference times the CPU oracle (the only reference that exists for
this method) on the same workload and metric, rank 0 only.

--scales ue8m0 times the separately declared UE8M0 block-scaled mode instead
(inputs quantised with power-of-two scales, packed four to an int32; the
tensor core applies them).  The default run also reports that mode's
per-shape numbers under "ue8m0_shapes"; the headline stays the fp32-scale
mode.  It also times the NN, TN and TT operand layouts of the dense GEMM on
the decode and prefill shapes ("layout_shapes").
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import dg_inputs as gi  # noqa: E402

METRIC = "FP8 TFLOPS per shape and % of 1-GPU roofline (dense, contiguous, masked MoE)"
HEADLINE = "dense_decode"
L2_FLUSH_BYTES = 512 << 20


# ------------------------------------------------------------------ helpers

def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            mp = json.load(f)
        return dict(hbm_gbs=float(mp["hbm_gbs"]), bf16_tflops=float(mp["bf16_tflops"]),
                    bf16_sustained=float(mp.get("bf16_tflops_sustained", mp["bf16_tflops"])),
                    source="measured")
    except (OSError, KeyError, ValueError):
        return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_sustained=1400.0, source="fallback")


def workload_cost(p):
    """Algorithmic FLOPs and bytes (each tensor moved once; valid rows only)."""
    kind = p["kind"]
    K, N = p["K"], p["N"]
    nkb = K // 128
    nbn = (N + 127) // 128
    if kind == "dense":
        M = p["M"]
        flop = 2.0 * M * N * K
        byts = M * K + N * K + 4 * M * nkb + 4 * nbn * nkb + 2 * M * N
        rows = M
    elif kind == "contiguous":
        rows = int((p["m_indices"] >= 0).sum())
        G = p["G"]
        flop = 2.0 * rows * N * K
        byts = rows * K + G * N * K + 4 * rows * nkb + 4 * G * nbn * nkb + 2 * rows * N + 4 * p["M"]
    else:
        G = p["G"]
        rows = int(np.minimum(p["masked_m"], p["max_m"]).sum())
        flop = 2.0 * rows * N * K
        byts = rows * K + G * N * K + 4 * rows * nkb + 4 * G * nbn * nkb + 2 * rows * N + 4 * G
    return flop, float(byts), rows


def roofline(flop, byts, pk):
    fp8_peak = 2.0 * pk["bf16_tflops"]  # nominal fp8/bf16 dense ratio 4.5/2.25
    t_tensor = flop / (fp8_peak * 1e12)
    t_hbm = byts / (pk["hbm_gbs"] * 1e9)
    bound = "tensor" if t_tensor >= t_hbm else "hbm"
    return bound, max(t_tensor, t_hbm), fp8_peak


def kernel_hash():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "moe_grouped_gemm_wt_b200", "csrc")
    for fn in sorted(os.listdir(csrc)):
        if fn.endswith((".cu", ".cuh")):
            with open(os.path.join(csrc, fn), "rb") as f:
                h.update(fn.encode() + f.read())
    return h.hexdigest()[:16]


def ncu_traffic(workload, ue8m0=False):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel sources (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            t = json.load(f)
        e = t.get(workload + (":ue8m0" if ue8m0 else ""))
        if e and e.get("kernel_hash") == kernel_hash():
            return float(e["dram_bytes_per_launch"])
    except (OSError, ValueError):
        pass
    return None


class ClockSampler:
    """nvidia-smi clocks/throttle sampling while the GPU is busy."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,utilization.gpu,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.dev), "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=2)
        samples = []
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                samples.append(dict(sm=float(parts[0]), smmax=float(parts[1]),
                                    power=float(parts[2]), util=float(parts[3]),
                                    hw=parts[5], hwt=parts[6], swt=parts[7], pcap=parts[8]))
            except ValueError:
                continue
        if not samples:
            return dict(sm_mhz=None, sm_max_mhz=None, reasons=[], samples=0)
        busy = [s for s in samples if s["util"] >= 30] or samples
        reasons = set()
        for s in busy:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("pcap", "sw_power_cap")):
                if s[key].lower() == "active":
                    reasons.add(name)
        return dict(sm_mhz=statistics.median(s["sm"] for s in busy),
                    sm_max_mhz=max(s["smmax"] for s in busy),
                    reasons=sorted(reasons), samples=len(busy))


# ------------------------------------------------------------ our library

def pack_ue8m0(dg, p, d):
    """The UE8M0 mode's packed scale words, built on the device from the
    fp32 power-of-two scales (dg_transform_sf_ue8m0)."""
    rows = p["M"] if p["kind"] != "masked" else p["max_m"]
    d["sfa"] = dg.dg_transform_sf_ue8m0(d["sA"], rows, mn_major=True)
    d["sfb"] = dg.dg_transform_sf_ue8m0(d["sB"], d["sB"].shape[-2], mn_major=False)


def to_device(p, torch, dev, dg=None):
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    a_mn, b_mn = OPERAND_LAYOUTS.get(p.get("layout"), (False, False))
    out = dict(A=t(p["A"].T if a_mn else p["A"]), B=t(p["B"].T if b_mn else p["B"]),
               sA=t(gi.sa_to_kernel_layout(p["sA"])), sB=t(p["sB"]))
    if p["kind"] == "dense":
        out["D"] = torch.empty((p["M"], p["N"]), dtype=torch.bfloat16, device=dev)
    elif p["kind"] == "contiguous":
        out["m_indices"] = t(p["m_indices"])
        out["D"] = torch.empty((p["M"], p["N"]), dtype=torch.bfloat16, device=dev)
    else:
        out["masked_m"] = t(p["masked_m"])
        out["D"] = torch.empty((p["G"], p["max_m"], p["N"]), dtype=torch.bfloat16, device=dev)
    if p.get("ue8m0"):
        pack_ue8m0(dg, p, out)
    return out


def call(dg, p, d, stream=None):
    if p.get("ue8m0"):
        if p["kind"] == "dense":
            dg.dg_fp8_gemm_nt_ue8m0(d["A"], d["sfa"], d["B"], d["sfb"], d["D"], stream=stream)
        elif p["kind"] == "contiguous":
            dg.dg_fp8_grouped_gemm_contiguous_ue8m0(d["A"], d["sfa"], d["B"], d["sfb"], d["D"],
                                                    d["m_indices"], stream=stream)
        else:
            dg.dg_fp8_grouped_gemm_masked_ue8m0(d["A"], d["sfa"], d["B"], d["sfb"], d["D"], d["masked_m"],
                                                expected_m=int(np.mean(p["masked_m"])), stream=stream)
        return
    if p.get("layout"):
        getattr(dg, "dg_fp8_gemm_" + p["layout"])(d["A"], d["sA"], d["B"], d["sB"], d["D"], stream=stream)
    elif p["kind"] == "dense":
        dg.dg_fp8_gemm_nt(d["A"], d["sA"], d["B"], d["sB"], d["D"], stream=stream)
    elif p["kind"] == "contiguous":
        dg.dg_fp8_grouped_gemm_contiguous(d["A"], d["sA"], d["B"], d["sB"], d["D"], d["m_indices"],
                                          stream=stream)
    else:
        dg.dg_fp8_grouped_gemm_masked(d["A"], d["sA"], d["B"], d["sB"], d["D"], d["masked_m"],
                                      expected_m=int(np.mean(p["masked_m"])), stream=stream)


def reduce_max_ms(ms, dist, device, world):
    """Max over ranks of a per-rank time (ms); every rank gets the result."""
    if world <= 1:
        return ms
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_value(flop_per_rank, world, ms):
    """Whole-job throughput (TFLOPS): every rank's work over the slowest rank's time."""
    return flop_per_rank * world / (ms * 1e-3) / 1e12


def shard_experts(p, rank, world):
    """Expert parallelism for the grouped workloads: rank r keeps experts
    [r*G/world, (r+1)*G/world) -- their rows of A and sA (contiguous: the
    groups' segments, each with the padding rows that follow it; masked:
    whole groups), their B, sB and metadata, with group indices renumbered
    from 0.  No exchange is needed: every expert's output rows live on the
    rank that computes them."""
    G = p["G"]
    g0, g1 = rank * G // world, (rank + 1) * G // world
    q = dict(p)
    q["G"] = g1 - g0
    q["group0"] = g0  # the shard's first expert in the whole problem
    q["B"], q["sB"] = p["B"][g0:g1], p["sB"][g0:g1]
    if p["kind"] == "masked":
        for k in ("A", "sA", "masked_m"):
            q[k] = p[k][g0:g1]
        return q
    mi = np.asarray(p["m_indices"])
    # owner of each row: its group, or for a padding row the group before it
    owner = np.maximum.accumulate(np.where(mi >= 0, mi, -1))
    owner[owner < 0] = 0
    rows = np.flatnonzero((owner >= g0) & (owner < g1))
    lo, hi = (int(rows[0]), int(rows[-1]) + 1) if rows.size else (0, 0)
    q["A"], q["sA"] = p["A"][lo:hi], p["sA"][lo:hi]
    q["m_indices"] = np.where(mi[lo:hi] >= 0, mi[lo:hi] - g0, -1).astype(np.int32)
    q["M"] = hi - lo
    q["row0"] = lo  # the shard's first row in the whole problem
    return q


def workload_label(p, name):
    if p["kind"] == "dense":
        return f"{name} M={p['M']} N={p['N']} K={p['K']}"
    if p["kind"] == "contiguous":
        return f"{name} G={p['G']} M_total={p['M']} N={p['N']} K={p['K']}"
    return f"{name} G={p['G']} max_m={p['max_m']} N={p['N']} K={p['K']} sum_masked_m={int(p['masked_m'].sum())}"


# Operand layouts of the dense GEMM besides NT: (A stored M-major, B stored
# N-major) for the layout entry points dg_fp8_gemm_nn / _tn / _tt.
OPERAND_LAYOUTS = {"nn": (False, True), "tn": (True, True), "tt": (True, False)}


def tile_label(dg, p):
    base = 3 if p.get("ue8m0") else 0  # describe_config layouts 3-5: the UE8M0 mode
    if p.get("layout"):
        return f"operand layout {p['layout']} (one-CTA tiles, MN-major boxes)"
    if p["kind"] == "dense":
        return dg.dg_describe_config(base, p["M"], p["N"], p["K"], 1)
    if p["kind"] == "contiguous":
        return dg.dg_describe_config(base + 1, p["M"], p["N"], p["K"], p["G"])
    return dg.dg_describe_config(base + 2, int(np.mean(p["masked_m"])), p["N"], p["K"], p["G"])


def make_problem(name, ue8m0):
    p = gi.make_workload(name, ue8m0=ue8m0)
    p["ue8m0"] = ue8m0
    return p


def time_kernel(torch, dg, p, d, steps, warmup, flush, kernel_times=None):
    """Per-launch CUDA-event times (ms) with an L2 flush before each launch.
    With kernel_times (a list), each launch's device time from its first CTA's
    start to its last CTA's end (the library's %globaltimer stamps, ms) is
    appended to it: the launch without the launch latency the events see."""
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        flush.zero_()
        call(dg, p, d)
    torch.cuda.synchronize()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    stamps = torch.zeros((steps, 2), dtype=torch.int64, device=d["A"].device)
    stamps[:, 0] = 2 ** 63 - 1
    try:
        for i in range(steps):
            flush.zero_()
            if kernel_times is not None:
                dg.dg_set_timing_stamps(stamps[i])
            starts[i].record(stream)
            call(dg, p, d)
            ends[i].record(stream)
    finally:
        dg.dg_set_timing_stamps(None)
    torch.cuda.synchronize()
    st = dg.dg_get_device_status()
    if st != 0:
        raise RuntimeError(f"device status {dg.dg_status_string(st)} during the benchmark")
    if kernel_times is not None:
        v = stamps.cpu().numpy()
        kernel_times.extend(((v[:, 1] - v[:, 0]) * 1e-6).tolist())
    return [s.elapsed_time(e) for s, e in zip(starts, ends)]


def launch_floor_ms(torch, steps, flush):
    """An empty kernel timed like the GEMM (flush, then events around one
    launch): the launch latency inside every event-timed figure."""
    stream = torch.cuda.current_stream()
    out = []
    for i in range(steps + 3):
        flush.zero_()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record(stream)
        torch.cuda._sleep(0)
        e.record(stream)
        torch.cuda.synchronize()
        if i >= 3:
            out.append(s.elapsed_time(e))
    return statistics.median(out)


def host_us_per_call(torch, dg, p, d, calls=1000):
    """Host time of one call of the C ABI function (through ctypes, no
    binding checks) over back-to-back enqueues: validation, planning, the
    tensor-map cache lookup and the launch."""
    lib = dg.load_library()
    torch.cuda.synchronize()
    if p["kind"] != "dense" or p.get("ue8m0"):
        return None
    args = [d["A"].data_ptr(), d["sA"].data_ptr(), d["B"].data_ptr(), d["sB"].data_ptr(), d["D"].data_ptr(),
            p["M"], p["N"], p["K"], None]
    lib.dg_fp8_gemm_nt(*args)
    t0 = time.perf_counter()
    for _ in range(calls):
        lib.dg_fp8_gemm_nt(*args)
    t1 = time.perf_counter()
    torch.cuda.synchronize()
    return (t1 - t0) / calls * 1e6


def time_e2e(torch, dg, p, steps, warmup, dev):
    """Through the public API with host buffers: pinned host inputs copied in,
    the GEMM, the output copied back -- all inside the timed region."""
    host = {k: torch.from_numpy(np.ascontiguousarray(v)).pin_memory()
            for k, v in (("A", p["A"]), ("B", p["B"]), ("sA", gi.sa_to_kernel_layout(p["sA"])),
                         ("sB", p["sB"]))}
    d = to_device(p, torch, dev, dg)
    out_host = torch.empty(d["D"].shape, dtype=torch.bfloat16).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = out_host.numel() * out_host.element_size()
    stream = torch.cuda.current_stream()

    def one():
        for k in host:
            d[k].copy_(host[k], non_blocking=True)
        if p.get("ue8m0"):
            pack_ue8m0(dg, p, d)  # the scale packing is part of the user's call path
        call(dg, p, d)
        out_host.copy_(d["D"], non_blocking=True)

    for _ in range(warmup):
        one()
    torch.cuda.synchronize()
    s = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)
    s.record(stream)
    for _ in range(steps):
        one()
    e.record(stream)
    torch.cuda.synchronize()
    return s.elapsed_time(e) / steps, h2d, d2h


def cpu_oracle_rate(p, budget_s=10.0):
    """The oracle as it stands on this host: FLOP/s over repeated whole-problem
    passes (at least one) within about budget_s seconds."""
    import oracle
    oracle.build()
    flop, _, _ = workload_cost(p)
    t0 = time.perf_counter()
    n = 0
    while True:
        oracle.gemm_nt(p["A"], p["sA"], p["B"], p["sB"], want_f64=False)
        n += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    return flop * n / dt / 1e12, oracle.num_threads(), n, dt


# ------------------------------------------------------------------- arms

def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    oracle.build()
    p = gi.make_workload(HEADLINE)
    rows = 16  # bounded sample of the workload per step: 16 of its 128 rows
    sub = dict(p, A=p["A"][:rows], sA=p["sA"][:rows], M=rows)
    flop, _, _ = workload_cost(sub)
    for _ in range(args.warmup):
        oracle.gemm_nt(sub["A"], sub["sA"], sub["B"], sub["sB"], want_f64=False)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle.gemm_nt(sub["A"], sub["sA"], sub["B"], sub["sB"], want_f64=False)
        times.append(time.perf_counter() - t0)
    ms = 1e3 * sum(times) / len(times)
    value = flop / (ms * 1e-3) / 1e12
    cores = oracle.num_threads()
    sample = f"rows 0..{rows - 1} of the {p['M']}x{p['N']}x{p['K']} problem per step"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOPS",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1) quantised to e4m3 with 1x128 / 128x128 fp32 scales)",
        "config": {"workload": "dense_decode M=128 N=2112 K=7168", "sample": sample},
        "cpu_baseline": {"value": value, "unit": "TFLOPS", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_ours(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)

    from moe_grouped_gemm_wt_b200 import build as b
    if not os.path.exists(b.LIB):
        b.build()
    import moe_grouped_gemm_wt_b200 as dg
    dg.load_library()

    pk = peaks()
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    ue8m0 = args.scales == "ue8m0"
    p = make_problem(args.workload, ue8m0)
    # Grouped workloads on several ranks: expert parallel, the fixed problem
    # split by expert (strong scaling); dense workloads: one replica per rank
    # (weak scaling).
    expert_parallel = world > 1 and p["kind"] != "dense"
    flop_job = workload_cost(p)[0] if expert_parallel else None
    if expert_parallel:
        if world > p["G"]:
            raise SystemExit(f"expert parallel: {world} ranks for {p['G']} experts")
        p = shard_experts(p, rank, world)
    d = to_device(p, torch, dev, dg)
    flop, byts, _ = workload_cost(p)

    sampler = ClockSampler(local)
    sampler.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    ktimes = []
    times = time_kernel(torch, dg, p, d, args.steps, max(args.warmup, 3), flush, ktimes)
    torch.cuda.synchronize()
    ms = reduce_max_ms(sum(times) / len(times), dist, dev, world)
    kernel_ms = reduce_max_ms(sum(ktimes) / len(ktimes), dist, dev, world)
    floor_ms = launch_floor_ms(torch, 10, flush)
    if world > 1:
        dist.barrier()

    # per-shape sweeps (every rank runs them; rank 0 reports): the mode
    # timed above, and, after a default fp32-scale run, the UE8M0 mode too
    def sweep(sweep_ue8m0):
        out = {}
        for name in gi.WORKLOADS:
            # a shard is not the shape
            same = name == args.workload and not expert_parallel and sweep_ue8m0 == ue8m0
            q = p if same else make_problem(name, sweep_ue8m0)
            dq = d if same else to_device(q, torch, dev, dg)
            kq = []
            tq = time_kernel(torch, dg, q, dq, max(10, min(args.steps, 30)), 3, flush, kq)
            mq = statistics.median(tq)
            kmq = statistics.median(kq)
            fq, bq, rows = workload_cost(q)
            bound, t_roof, _ = roofline(fq, bq, pk)
            out[name] = {
                "us": mq * 1e3, "tflops": fq / (mq * 1e-3) / 1e12,
                "bound": bound, "roofline_us": t_roof * 1e6,
                "frac_of_roofline": t_roof / (mq * 1e-3),
                "kernel_us": kmq * 1e3, "kernel_frac_of_roofline": t_roof / (kmq * 1e-3),
                "valid_rows": rows, "tile": tile_label(dg, q),
            }
            if not same:
                del dq
                torch.cuda.empty_cache()
        return out

    # the NN / TN / TT operand layouts on the two dense shapes (fp32 scales)
    def sweep_layouts():
        out = {}
        for name in ("dense_decode", "dense_prefill"):
            for lay in sorted(OPERAND_LAYOUTS):
                q = make_problem(name, False)
                q["layout"] = lay
                dq = to_device(q, torch, dev, dg)
                kq = []
                tq = time_kernel(torch, dg, q, dq, max(10, min(args.steps, 30)), 3, flush, kq)
                mq, kmq = statistics.median(tq), statistics.median(kq)
                fq, bq, _ = workload_cost(q)
                bound, t_roof, _ = roofline(fq, bq, pk)
                out[f"{name}:{lay}"] = {
                    "us": mq * 1e3, "tflops": fq / (mq * 1e-3) / 1e12, "bound": bound,
                    "frac_of_roofline": t_roof / (mq * 1e-3), "kernel_us": kmq * 1e3,
                    "kernel_frac_of_roofline": t_roof / (kmq * 1e-3), "tile": tile_label(dg, q),
                }
                del dq
                torch.cuda.empty_cache()
        return out

    shapes, ue8m0_shapes, layout_shapes = {}, None, None
    if not args.no_shapes:
        shapes = sweep(ue8m0)
        if not ue8m0 and not args.no_ue8m0_shapes:
            ue8m0_shapes = sweep(True)
        if not ue8m0 and not args.no_layout_shapes:
            layout_shapes = sweep_layouts()
    clocks = sampler.stop()

    e2e_ms, h2d, d2h = time_e2e(torch, dg, p, max(10, min(args.steps, 50)), 3, dev)
    host_us = host_us_per_call(torch, dg, p, d)

    value = flop_job / (ms * 1e-3) / 1e12 if expert_parallel else whole_job_value(flop, world, ms)
    bound, t_roof, fp8_peak = roofline(flop, byts, pk)
    if bound == "hbm":
        achieved = byts / (ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / pk["hbm_gbs"]}
    else:
        achieved = flop / (ms * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": fp8_peak, "unit": "TFLOP/s",
                "frac": achieved / fp8_peak}
    roof["traffic"] = ncu_traffic(args.workload, ue8m0)
    roof["peak_source"] = pk["source"] + (" (fp8 = 2 x measured bf16)" if bound == "tensor" else "")

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and p["kind"] == "dense":
        rate, cores, npass, dt = cpu_oracle_rate(p, args.cpu_budget)
        cpu = {"value": rate, "unit": "TFLOPS", "cores": cores, "kind": "oracle",
               "sample": f"{npass} whole passes of the {p['M']}x{p['N']}x{p['K']} problem in {dt:.1f} s"}

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": world,
        "steps": args.steps, "warmup": max(args.warmup, 3), "ms_per_step": ms,
        "higher_is_better": True, "scaling": "strong" if expert_parallel else "weak",
        "vs_baseline": None,
        "dtype": ("fp8_e4m3 (UE8M0 block-scaled MMA, fp32 accumulate, bf16 out)" if ue8m0
                  else "fp8_e4m3 (fp32 promotion, bf16 out)"),
        "data": ("synthetic (seeded N(0,1) quantised to e4m3 with 1x128 / 128x128 power-of-two scales, "
                 "packed UE8M0)" if ue8m0 else
                 "synthetic (seeded N(0,1) quantised to e4m3 with 1x128 / 128x128 fp32 scales)"),
        "config": {"workload": workload_label(p, args.workload),
                   "l2": "flushed before every timed launch (512 MiB write)",
                   "parallelism": (f"expert parallel x{world} (this rank: {p['G']} experts)"
                                   if expert_parallel else f"replicas x{world}"),
                   "tile": tile_label(dg, p),
                   "scales": "ue8m0 (separately declared block-scaled mode)" if ue8m0 else "fp32"},
        "roofline": roof,
        "frac_of_roofline": t_roof / (ms * 1e-3),
        # the same launches timed on the device from the first CTA's start to
        # the last CTA's end (%globaltimer stamps), and an empty kernel timed
        # like the GEMM: the event-timed figure is roughly their sum
        "kernel_us": kernel_ms * 1e3,
        "kernel_frac_of_roofline": t_roof / (kernel_ms * 1e-3),
        "launch_floor_us": floor_ms * 1e3,
        "host_us_per_call": host_us,
        "cpu_baseline": cpu,
        "e2e": {"value": flop / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOPS",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": args.steps,
        "clocks": clocks,
        "shapes": shapes,
    }
    if ue8m0_shapes is not None:
        line["ue8m0_shapes"] = ue8m0_shapes
    if layout_shapes is not None:
        line["layout_shapes"] = layout_shapes
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-shapes", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=10.0)
    ap.add_argument("--scales", choices=("fp32", "ue8m0"), default="fp32",
                    help="fp32 scales (the headline mode) or the UE8M0 block-scaled mode")
    ap.add_argument("--no-layout-shapes", action="store_true",
                    help="skip the NN / TN / TT operand-layout timings of the dense shapes")
    ap.add_argument("--no-ue8m0-shapes", action="store_true",
                    help="skip the UE8M0 mode's per-shape sweep of a default run")
    ap.add_argument("--workload", choices=sorted(gi.WORKLOADS), default=HEADLINE,
                    help="workload timed as the step (default: the decode-shaped dense GEMM)")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
