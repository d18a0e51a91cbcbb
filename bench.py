#!/usr/bin/env python
"""Benchmark the SageSLA hot path (prepare -> select -> forward) on B200.

One step = one pass of the whole path over one batch of synthetic input: sagesla_prepare,
sagesla_select and sagesla_forward through the C ABI. Default workload: the Wan-1.3B
480p-shaped layer (B=1, H=12, N=32760, d=128, rho=0.1, nu=0.45).

Prints one JSON line on rank 0. Multi-GPU (torchrun): rank r runs batch element r of an
N-element job, the workload's shape with its own seeded input (the path has no exchange
step); the step time is the max over ranks and `value` counts the work of all ranks.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME|sweep]
  python bench.py --impl reference ...   # the CPU oracle on a bounded sample (rank 0)
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from quantized_block_sparse_b200.inputs import SWEEP_RHOS, WORKLOADS, make_workload_qkv  # noqa: E402

METRIC = "SageSLA fwd ms/call & dense-equiv TOPS at Wan-1.3B 480p shape; % tensor roofline"
UNIT = "dense-equiv TOPS"
INT8_TO_BF16_RATE = 2.0  # dense INT8 : BF16 tensor rate on B200: nominal 4.5 : 2.25 POPS;
                         # a tcgen05 M128 N128 issue-rate probe gave 8124 : 4064 MAC/clk/SM
PROBE_BF16_MAC_PER_CLK_SM = 4064  # that probe's bf16 rate: back-to-back kind::f16 MMAs
N_SM = 148
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def dense_equiv_ops(wl) -> float:
    return 4.0 * wl.B * wl.H * float(wl.N) ** 2 * wl.d


def forward_work(wl, nB, k_c, m):
    """Algorithmic tensor work of one sagesla_forward over the executed blocks: INT8 QK^T
    ops and BF16 flops (P.V over the critical pairs, the marginal gather-sum and the
    phi(Q~).H product per query block)."""
    heads = wl.B * wl.H
    pair = 2.0 * 64 * 64 * 128
    int8 = heads * nB * k_c * pair
    bf16 = heads * nB * (k_c * pair + (2.0 * m * 128 * 129 + 2.0 * 64 * 128 * 129 if m > 0 else 0.0))
    return {"int8_ops": int8, "bf16_flops": bf16}


def profiled_traffic(workload: str):
    """DRAM bytes per attn_kernel launch from the committed ncu summary, or None.

    The summary records the sha256 prefix of the kernel source it was taken on (comments
    and whitespace removed, so only code counts); once the code has changed the counters
    no longer describe the kernel and None is returned.
    """
    import hashlib
    import re
    summary = os.path.join(ROOT, "profiles", f"attn_kernel_{workload}.md")
    src = os.path.join(ROOT, "quantized_block_sparse_b200", "csrc", "attention.cu")
    if not (os.path.exists(summary) and os.path.exists(src)):
        return None
    fields = {}
    with open(summary) as f:
        for line in f:
            if ":" in line and not line.startswith(("|", "#", " ")):
                key, _, val = line.partition(":")
                fields[key.strip()] = val.strip()
    with open(src) as f:
        code = f.read()
    code = re.sub(r"/\*.*?\*/", " ", code, flags=re.S)
    code = re.sub(r"//[^\n]*", " ", code)
    code = re.sub(r"\s+", " ", code).strip()
    sha = hashlib.sha256(code.encode()).hexdigest()
    prefix = fields.get("source_sha256_prefix")
    if not prefix or not sha.startswith(prefix) or "dram_bytes_per_launch" not in fields:
        return None
    return int(fields["dram_bytes_per_launch"])


def probe_ex2_rates(dev, iters=2048):
    """The SFU exponential rate of this GPU, measured by the library's probe kernel (one CTA
    per SM, 8 independent chains of dependent exponentials per thread, SM cycles read on the
    device): per form, the median over the CTAs of exponentials per SM clock, and the number
    of distinct SMs the CTAs ran on. Form 0 is ex2.approx.ftz.f32 (the kernels' form), forms 1
    and 2 ex2.approx.f16x2 and ex2.approx.ftz.bf16x2 (two exponentials per instruction)."""
    import torch

    from quantized_block_sparse_b200 import sagesla as S
    n = torch.cuda.get_device_properties(dev).multi_processor_count
    out = torch.zeros(3 * n, dtype=torch.int64, device=dev)
    res = {}
    for form in (0, 1, 2):
        S.sagesla_probe_ex2(form, 64, out)  # warm-up (module load, clocks)
        S.sagesla_probe_ex2(form, iters, out)
        torch.cuda.synchronize(dev)
        a = out.view(n, 3).cpu().numpy()
        res[form] = (float(np.median(a[:, 0] / a[:, 1])), int(len(set(a[:, 2].tolist()))))
    return res


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


# ------------------------------------------------------------------ CPU oracle timing
def _oracle_rows(args):
    """Worker: the oracle's forward (steps 5-7) for some query blocks of one head."""
    prep, v, sel, qblocks = args
    from threadpoolctl import threadpool_limits

    import oracle as O
    with threadpool_limits(1):
        O.forward(prep, v, sel, heads=[(0, 0)], qblocks=qblocks)
    return len(qblocks)


def _warm(_):
    """Worker start-up task: keeps the worker busy briefly so every worker gets spawned."""
    time.sleep(0.5)
    return os.getpid()


def oracle_pool(wl, procs=None):
    """A spawn-started process pool for the oracle's forward, its workers already running."""
    import concurrent.futures as cf
    import multiprocessing as mp
    nB = -(-wl.N // 64)
    procs = procs or max(1, min(len(os.sched_getaffinity(0)), nB, 32))
    ex = cf.ProcessPoolExecutor(procs, mp_context=mp.get_context("spawn"))
    list(ex.map(_warm, range(procs)))
    return ex, procs


def oracle_head_time(q, k, v, wl, pool):
    """Time the CPU oracle on one whole head of the workload, as it stands.

    prepare and select run in this process; the forward's query blocks are split into one
    contiguous chunk per worker of `pool` (from oracle_pool: spawn-started, one BLAS thread
    each). Every worker recomputes the head's linear states, as the oracle does per call.
    Returns (seconds, processes used, sample text).
    """
    import oracle as O
    ex, procs = pool
    nB = -(-wl.N // 64)
    qf, kf, vf = (t[:1, :1].float().numpy() for t in (q, k, v))
    chunks = [c.tolist() for c in np.array_split(np.arange(nB), procs) if len(c)]
    t0 = time.perf_counter()
    prep = O.prepare(qf, kf)
    sel = O.select(prep.q_bar, prep.k_bar, wl.rho, wl.nu)
    done = sum(ex.map(_oracle_rows, [(prep, vf, sel, c) for c in chunks]))
    secs = time.perf_counter() - t0
    assert done == nB
    sample = (f"1 of {wl.B * wl.H} heads, whole and measured: prepare+select in one process, "
              f"forward over all {nB} query blocks split across {len(chunks)} spawned processes "
              f"(each recomputes the head's linear states); {secs:.1f} s wall")
    return secs, len(chunks), sample


def run_reference(args, wl):
    """`--impl reference`: the CPU oracle, as it stands, on one whole head per step."""
    rank, _, _ = rank_env()
    if rank != 0:
        return 0
    q, k, v = make_workload_qkv(wl)
    times = []
    cores, sample = 0, ""
    pool = oracle_pool(wl)
    try:
        for step in range(args.warmup + args.steps):
            secs, cores, sample = oracle_head_time(q, k, v, wl, pool)
            if step >= args.warmup:
                times.append(secs)
    finally:
        pool[0].shutdown()
    per_head = statistics.mean(times)
    value = dense_equiv_ops(wl) / (wl.B * wl.H) / per_head / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": per_head * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64/f32 (CPU oracle)", "data": "synthetic",
        "config": workload_config(wl),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample + "; one step = one head (value = one head's "
                                            "dense-equivalent ops / its measured time)"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


WORKLOAD_TITLES = {
    "480p": "Wan-1.3B 480p-shaped SageSLA layer",
    "720p": "Wan-14B 720p-shaped SageSLA layer",
    "480p_14b": "Wan2.1-14B 480p-shaped SageSLA layer",
    "480p_topk015": "Wan-1.3B 480p-shaped SageSLA layer, sla_topk 0.15",
    "720p_i2v": "Wan2.2-I2V-A14B 720p-shaped SageSLA layer",
    "dense": "dense SageAttention layer (rho = 1, no linear branch)",
    "tiny": "tiny SageSLA test layer",
}
WORKLOAD_TITLES.update({f"sweep_rho{r:g}": f"480p sparsity sweep, B=2, rho={r:g}, nu=(1-rho)/2"
                        for r in SWEEP_RHOS})


def workload_config(wl):
    return {"workload": WORKLOAD_TITLES.get(wl.name, f"{wl.name} SageSLA layer"),
            "B": wl.B, "H": wl.H, "N": wl.N, "d": wl.d, "grid_thw": list(wl.grid),
            "rho": wl.rho, "nu": wl.nu, "block": 64, "seed": wl.seeds[0],
            "l2": "no flush; per-step working set ~1.2 GB (inputs 300 MB + states) exceeds the 126 MB L2",
            "parallelism": "batch sharded over ranks: rank r runs element r (seed + r); no data-path collective"}


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.dev)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons, power = [], None, set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
                power.append(float(parts[3]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        loaded = [s for s, p in zip(sm, power) if p > 200] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ ranks
# One process per GPU (torchrun). The path has no exchange step: rank r runs batch element
# r of the job on its own; ranks meet only for barriers around the timed region and for
# the max of the per-rank times.
def rank_env():
    """(rank, world, local_rank) from the torchrun environment (1 process without it)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init_ranks(world: int, backend: str, device=None, timeout_s: float = 120.0):
    """Process group for world > 1 (short timeout so a missing rank ends with an error)."""
    if world <= 1:
        return
    import datetime

    import torch.distributed as dist
    kw = {"device_id": device} if backend == "nccl" else {}
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)


def max_over_ranks_of(x: float, world: int, device=None) -> float:
    """The largest per-rank value (the job's step time is its slowest rank's)."""
    if world <= 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tops(ops_per_rank: float, world: int, step_ms: float) -> float:
    """Throughput of the whole job: the work of all ranks over the slowest rank's time."""
    return ops_per_rank * world / (step_ms * 1e-3) / 1e12


def gpu_local_cpus(device_index: int):
    """The CPUs NVML reports as local to the GPU (its NUMA node), or None."""
    try:
        import pynvml
        import torch
        pr = torch.cuda.get_device_properties(device_index)
        bus = f"{pr.pci_domain_id:08x}:{pr.pci_bus_id:02x}:{pr.pci_device_id:02x}.0"
        pynvml.nvmlInit()
        try:
            handle = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            words = pynvml.nvmlDeviceGetCpuAffinity(handle, (os.cpu_count() + 63) // 64)
        finally:
            pynvml.nvmlShutdown()
        cpus = {64 * i + b for i, w in enumerate(words) for b in range(64) if (w >> b) & 1}
        cpus &= os.sched_getaffinity(0)
        return cpus or None
    except Exception:
        return None


# ------------------------------------------------------------------ GPU arm
def run_ours(args, wl):
    import torch
    import torch.distributed as dist

    from quantized_block_sparse_b200 import sagesla as S

    rank, world, local = rank_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    init_ranks(world, "nccl", dev)

    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(x: float) -> float:
        return max_over_ranks_of(x, world, dev)

    S.lib()
    # rank r takes batch element r of an N-element job: its own seeded input, same shape
    q, k, v = make_workload_qkv(wl, seed=wl.seeds[0] + rank)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    eng = S.SageSLA(wl.B, wl.H, wl.N, wl.rho, wl.nu, device=dev)
    stream = torch.cuda.current_stream(dev)

    for _ in range(args.warmup):
        eng(qd, kd, vd)
    torch.cuda.synchronize(dev)
    eng.check()

    # ---- device-timed region (inputs resident in HBM)
    clocks = ClockSampler(torch.cuda.get_device_properties(dev).index if hasattr(
        torch.cuda.get_device_properties(dev), "index") else local)
    clocks.start()
    time.sleep(0.3)
    barrier()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        eng(qd, kd, vd)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    clk = clocks.stop()
    step_ms = max_over_ranks(e0.elapsed_time(e1) / args.steps)
    eng.check()

    # ---- per-kernel device time (launch tracing: CUDA events around each launch)
    L = S.lib()
    L.sagesla_trace_enable(1)
    for _ in range(args.steps):
        eng(qd, kd, vd)
    torch.cuda.synchronize(dev)
    L.sagesla_trace_enable(0)
    import ctypes
    buf = ctypes.create_string_buffer(1 << 16)
    L.sagesla_trace_read(buf, len(buf))
    kern = {}
    launches = 0
    for line in buf.value.decode().strip().splitlines():
        name, cnt, tot = line.split()
        kern[name] = {"launches": int(cnt), "avg_ms": float(tot) / int(cnt)}
        launches += int(cnt)
    launches_per_step = launches / args.steps
    # the launches of sagesla_forward (S5-S8)
    fwd_kernels = ("zb_kernel", "hgemm_kernel", "pair_kernel", "attn_kernel")
    fwd_ms = sum(kern[n]["avg_ms"] * kern[n]["launches"] / args.steps for n in fwd_kernels if n in kern)

    # ---- end to end through the public API: pinned host inputs in, output back to host.
    # A user's pipeline: step s copies its inputs in on one copy stream while step s-1
    # computes, and its output goes back on another while step s+1 computes (two device
    # input sets and two output buffers; host->device and device->host overlap). Every
    # step's copies are inside the timed region, which ends when the last output has
    # reached the host.
    # Pinned host buffers on the GPU's NUMA node (allocated while the process runs on the
    # GPU-local CPUs; the previous CPU set is restored afterwards).
    local_cpus = gpu_local_cpus(local)
    saved_cpus = os.sched_getaffinity(0)
    if local_cpus:
        os.sched_setaffinity(0, local_cpus)
    try:
        qh, kh, vh = (t.pin_memory() for t in (q, k, v))
        ohs = [torch.empty_like(q).pin_memory() for _ in range(2)]
        for t in ohs:
            t.zero_()
    finally:
        os.sched_setaffinity(0, saved_cpus)
    h2d = sum(t.numel() * t.element_size() for t in (qh, kh, vh))
    d2h = ohs[0].numel() * ohs[0].element_size()
    ins = [(qd, kd, vd), tuple(torch.empty_like(t) for t in (qd, kd, vd))]
    outs = [torch.empty_like(qd) for _ in range(2)]
    cs_in, cs_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()  # noqa: E731
    in_ready, in_free, out_ready, out_done = ([ev(), ev()] for _ in range(4))

    def pipelined(n_steps):
        for st in range(n_steps):
            b = st & 1
            with torch.cuda.stream(cs_in):
                if st >= 2:
                    cs_in.wait_event(in_free[b])     # step st-2 has finished reading ins[b]
                for dst, src in zip(ins[b], (qh, kh, vh)):
                    dst.copy_(src, non_blocking=True)
                in_ready[b].record(cs_in)
            stream.wait_event(in_ready[b])
            if st >= 2:
                stream.wait_event(out_done[b])       # outs[b] of step st-2 is on the host
            eng(*ins[b], out=outs[b])
            in_free[b].record(stream)
            out_ready[b].record(stream)
            with torch.cuda.stream(cs_out):
                cs_out.wait_event(out_ready[b])
                ohs[b].copy_(outs[b], non_blocking=True)
                out_done[b].record(cs_out)
        for b in range(min(2, n_steps)):
            stream.wait_event(out_done[b])

    pipelined(2)
    torch.cuda.synchronize(dev)
    barrier()
    e0.record(stream)
    pipelined(args.steps)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.steps)
    eng.check()
    assert torch.equal(ohs[(args.steps - 1) & 1], outs[(args.steps - 1) & 1].cpu())

    # ---- roofline of the dominant kernel (the block-sparse attention)
    peaks, peak_src = load_peaks()
    nB, k_c, n_neg, m = S.sagesla_counts(wl.B, wl.H, wl.N, wl.rho, wl.nu)
    pairs = wl.B * wl.H * nB * k_c
    tile_ops = 2.0 * 64 * 64 * 128
    # INT8 QK^T + BF16 PV, plus the linear term phi(Q~) H_i (64 x 128 x 128 per query block)
    # that the kernel forms after its last step when there are marginal blocks
    lin_flops = wl.B * wl.H * nB * 2.0 * 64 * 128 * 128 if m > 0 else 0.0
    bf16_equiv = pairs * tile_ops / INT8_TO_BF16_RATE + pairs * tile_ops + lin_flops
    att_ms = kern.get("attn_kernel", {}).get("avg_ms", float("nan"))
    achieved = bf16_equiv / (att_ms * 1e-3) / 1e12
    peak = float(peaks["bf16_tflops"])
    # second denominator: the tcgen05 probe rate at the SM clock sampled during the run
    sm_mhz = clk.get("sm_mhz") or 1965.0
    peak_probe = PROBE_BF16_MAC_PER_CLK_SM * 2 * N_SM * sm_mhz * 1e6 / 1e12
    # SFU floor of the attention kernel: one exponential per (query row, key) of every
    # executed critical pair, plus phi(Q~) of the linear term (one per element of Q, an upper
    # bound: phi takes the exponential only for x <= 0), over the probed ex2 rate
    rates = probe_ex2_rates(dev)
    exps = pairs * 64.0 * 64.0 + (wl.B * wl.H * float(wl.N) * wl.d if m > 0 else 0.0)
    sfu_peak = rates[0][0] * N_SM * sm_mhz * 1e6 / 1e9  # Gexp/s
    sfu_achieved = exps / (att_ms * 1e-3) / 1e9
    # forward-level roofline: every executed block of sagesla_forward on the tensor pipe
    fwd = forward_work(wl, nB, k_c, m)
    t_roof_s = fwd["int8_ops"] / (INT8_TO_BF16_RATE * peak * 1e12) + fwd["bf16_flops"] / (peak * 1e12)

    line = {
        "metric": METRIC,
        "value": whole_job_tops(dense_equiv_ops(wl), world, step_ms),
        "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": step_ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int8 QK^T + bf16 PV (fp32 accumulate)", "data": "synthetic",
        "config": workload_config(wl),
        "fwd_ms": fwd_ms,
        "fwd_dense_equiv_tops": dense_equiv_ops(wl) / (fwd_ms * 1e-3) / 1e12 if fwd_ms else None,
        "kernels_ms": {n: round(x["avg_ms"], 5) for n, x in kern.items()},
        "roofline": {"kernel": "attn_kernel", "bound": "tensor", "achieved": achieved,
                     "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak,
                     "traffic": profiled_traffic(wl.name),
                     "peak_tcgen05_probe": peak_probe, "frac_tcgen05_probe": achieved / peak_probe,
                     "note": (f"bf16-equivalent: INT8 QK^T ops / {INT8_TO_BF16_RATE:g} + BF16 PV flops over "
                              f"{pairs} executed 64x64 block pairs + phi(Q~)H_i 2*64*128*128 per query "
                              f"block ({lin_flops / 1e9:.1f} GF); peak = {peak_src} cuBLAS bf16 burst "
                              f"(of {peak_src}); peak_tcgen05_probe = {PROBE_BF16_MAC_PER_CLK_SM} bf16 "
                              f"MAC/clk/SM x 2 x {N_SM} SMs x the sampled SM clock; traffic = DRAM bytes "
                              f"per launch from the committed ncu summary (null once the kernel source "
                              f"differs from the profiled one)")},
        "roofline_sfu": {"kernel": "attn_kernel", "bound": "sfu", "exps": exps,
                         "achieved": sfu_achieved, "peak": sfu_peak, "unit": "Gexp/s",
                         "frac": sfu_achieved / sfu_peak, "t_sfu_ms": exps / (sfu_peak * 1e9) * 1e3,
                         "ex2_f32_per_clk_sm": rates[0][0], "ex2_f16x2_per_clk_sm": rates[1][0],
                         "ex2_bf16x2_per_clk_sm": rates[2][0],
                         "probe_sms": rates[0][1],
                         "note": (f"exponentials: 4096 per executed 64x64 critical pair ({pairs}) + one "
                                  f"per element of Q for phi(Q~) when m > 0 (upper bound); peak = the "
                                  f"probed ex2.approx.ftz.f32 rate per SM clock (median over one CTA "
                                  f"per SM) x {N_SM} SMs x the sampled SM clock")},
        "roofline_forward": {"bound": "tensor", "int8_ops": fwd["int8_ops"],
                             "bf16_flops": fwd["bf16_flops"], "t_roof_ms": t_roof_s * 1e3,
                             "fwd_ms": fwd_ms, "frac": t_roof_s * 1e3 / fwd_ms if fwd_ms else None,
                             "frac_tcgen05_probe": (t_roof_s * 1e3 * peak / peak_probe / fwd_ms
                                                    if fwd_ms else None),
                             "note": "sagesla_forward over the executed blocks: INT8 QK^T (critical "
                                     "pairs) at 2x the bf16 peak; BF16 P.V, the marginal gather "
                                     "2*m*128*129 and phi(Q)H 2*64*128*129 per query block (if m > 0) "
                                     "at the bf16 peak; frac = t_roof / measured forward time"},
        "e2e": {"value": whole_job_tops(dense_equiv_ops(wl), world, e2e_ms), "unit": UNIT, "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "pinned_host_memory": "GPU-local NUMA node" if local_cpus else "default placement"},
        "gpu_launches": int(round(launches_per_step * args.steps)),
        "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        pool = oracle_pool(wl)
        try:
            secs, cores, sample = oracle_head_time(q, k, v, wl, pool)
        finally:
            pool[0].shutdown()
        line["cpu_baseline"] = {"value": dense_equiv_ops(wl) / (wl.B * wl.H) / secs / 1e12,
                                "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample,
                                "ms_per_head": secs * 1e3}
    if rank == 0:
        print(json.dumps(line), flush=True)
    del eng
    if world > 1:
        dist.destroy_process_group()
    return 0


def run_heads(args, wl):
    """`--parallel heads`: one layer's B*H heads split over the ranks (strong scaling).

    Rank r runs prepare -> select -> forward on its contiguous range of heads; with
    --gather (the default) every step ends with an all-gather of the outputs, so each rank
    holds the whole layer's output. value = the whole layer's dense-equivalent ops over the
    slowest rank's step time.
    """
    import torch
    import torch.distributed as dist

    from quantized_block_sparse_b200 import sagesla as S
    from quantized_block_sparse_b200.heads_parallel import HeadParallelSageSLA, local_heads

    rank, world, local = rank_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    init_ranks(world, "nccl", dev)

    def barrier():
        if world > 1:
            dist.barrier()

    S.lib()
    q, k, v = make_workload_qkv(wl)  # the same layer on every rank; each keeps its heads
    ql, kl, vl = (local_heads(t, rank, world).contiguous() for t in (q, k, v))
    qd, kd, vd = ql.to(dev), kl.to(dev), vl.to(dev)
    layer = HeadParallelSageSLA(wl.B, wl.H, wl.N, wl.rho, wl.nu, rank, world, device=dev)
    gather = not args.no_gather
    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        layer(qd, kd, vd, gather=gather)
    torch.cuda.synchronize(dev)
    layer.check()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    barrier()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        out = layer(qd, kd, vd, gather=gather)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    clk = clocks.stop()
    step_ms = max_over_ranks_of(e0.elapsed_time(e1) / args.steps, world, dev)
    layer.check()
    # end to end: the rank's inputs from pinned host memory, the gathered output back
    qh, kh, vh = (t.pin_memory() for t in (ql, kl, vl))
    oh = torch.empty(tuple(out.shape), dtype=out.dtype).pin_memory()
    barrier()
    torch.cuda.synchronize(dev)
    e0.record(stream)
    for _ in range(args.steps):
        for dst, src in zip((qd, kd, vd), (qh, kh, vh)):
            dst.copy_(src, non_blocking=True)
        o = layer(qd, kd, vd, gather=gather)
        oh.copy_(o, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    e2e_ms = max_over_ranks_of(e0.elapsed_time(e1) / args.steps, world, dev)
    ops = dense_equiv_ops(wl)
    line = {
        "metric": METRIC, "value": ops / (step_ms * 1e-3) / 1e12, "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms,
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
        "dtype": "int8 QK^T + bf16 PV (fp32 accumulate)", "data": "synthetic",
        "config": dict(workload_config(wl), parallelism=(
            f"heads split over {world} ranks (rank r: heads {layer.lo}..{layer.hi - 1} on rank "
            f"{rank}); " + ("NCCL all-gather of the outputs each step" if gather else "no gather"))),
        "e2e": {"value": ops / (e2e_ms * 1e-3) / 1e12, "unit": UNIT, "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in (qh, kh, vh)),
                "d2h_bytes_per_step": oh.numel() * oh.element_size()},
        "gpu_launches": None, "clocks": clk,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    del layer
    if world > 1:
        dist.destroy_process_group()
    return 0


def _timed(fn, steps, warmup, stream):
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps


def _kernel_times(fn, S):
    """Per-kernel average device time (ms) of one call of fn, from the library's launch trace."""
    import ctypes

    import torch
    L = S.lib()
    L.sagesla_trace_enable(1)
    fn()
    torch.cuda.synchronize()
    L.sagesla_trace_enable(0)
    buf = ctypes.create_string_buffer(1 << 16)
    L.sagesla_trace_read(buf, len(buf))
    out, launches = {}, 0
    for line in buf.value.decode().strip().splitlines():
        name, cnt, tot = line.split()
        out[name] = round(float(tot) / int(cnt), 5)
        launches += int(cnt)
    return out, launches


def run_backward(args, wl):
    """`--op backward`: sagesla_backward (dQ, dK, dV for an upstream gradient) on the workload."""
    import torch

    from quantized_block_sparse_b200 import sagesla as S
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    S.lib()
    q, k, v = make_workload_qkv(wl)
    do = torch.randn(*q.shape, generator=torch.Generator().manual_seed(9)).to(torch.bfloat16)
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    eng = S.SageSLA(wl.B, wl.H, wl.N, wl.rho, wl.nu, device=dev)
    eng(qd, kd, vd)
    ws = S.sagesla_backward(qd, kd, vd, dod, eng.prep, eng.sel)[3]
    fn = lambda: S.sagesla_backward(qd, kd, vd, dod, eng.prep, eng.sel, workspace=ws)  # noqa: E731
    clocks = ClockSampler(0)
    clocks.start()
    time.sleep(0.3)
    ms = _timed(fn, args.steps, args.warmup, torch.cuda.current_stream(dev))
    clk = clocks.stop()
    S.sagesla_check_status(ws)
    kern, launches = _kernel_times(fn, S)
    nB, k_c, n_neg, m = S.sagesla_counts(wl.B, wl.H, wl.N, wl.rho, wl.nu)
    heads = wl.B * wl.H
    gemm = 2.0 * 64 * 64 * 128
    # algorithmic work: 5 GEMMs per critical pair (S, dP, dV, dK, dQ), the linear branch's
    # phi(Q)H, dn H^T, phi(Q)^T dn per query block and phi(K)G, V G^T per key block, and the
    # two masked sums H = M h and G = M^T dH over the marginal blocks
    flops = heads * nB * k_c * 5 * gemm
    if m > 0:
        flops += heads * nB * (3 + 2) * 2.0 * 64 * 128 * 128 + 2 * heads * nB * m * 2.0 * 128 * 128
    peaks, src = load_peaks()
    peak = float(peaks["bf16_tflops"])
    achieved = flops / (ms * 1e-3) / 1e12
    line = {"op": "backward", "metric": "SageSLA backward ms/call (dQ, dK, dV)", "value": ms,
            "unit": "ms", "higher_is_better": False, "steps": args.steps, "warmup": args.warmup,
            "dtype": "bf16 operands, fp32 accumulate (mma.sync tensor-core path)",
            "data": "synthetic", "config": workload_config(wl), "kernels_ms": kern,
            "gpu_launches": launches,
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak, "traffic": None,
                         "note": f"algorithmic {flops / 1e12:.3f} TFLOP per call over the executed "
                                 f"blocks; peak = {src} cuBLAS bf16 burst"},
            "clocks": clk}
    print(json.dumps(line), flush=True)
    return 0


W8A8_SHAPES = {  # Wan-1.3B linear layers at 480p: tokens x hidden 1536, FFN 8960
    "qkv": (32760, 4608, 1536), "out": (32760, 1536, 1536), "ffn_up": (32760, 8960, 1536),
    "ffn_down": (32760, 1536, 8960)}


def run_w8a8(args):
    """`--op w8a8`: the W8A8 block-wise INT8 linear layer on the Wan-1.3B 480p shapes."""
    import torch

    from quantized_block_sparse_b200 import sagesla as S
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    S.lib()
    peaks, src = load_peaks()
    peak_i8 = INT8_TO_BF16_RATE * float(peaks["bf16_tflops"])
    g = torch.Generator(device=dev).manual_seed(0)
    rc = 0
    for name, (M, N, K) in W8A8_SHAPES.items():
        x = torch.randn(M, K, device=dev, generator=g).to(torch.bfloat16)
        w = (torch.randn(N, K, device=dev, generator=g) * 0.05).to(torch.bfloat16)
        x8, sx = S.sagesla_w8a8_quantize(x)
        w8, sw = S.sagesla_w8a8_quantize(w)
        y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        ws = torch.zeros(256, dtype=torch.uint8, device=dev)
        stream = torch.cuda.current_stream(dev)
        t_gemm = _timed(lambda: S.sagesla_w8a8_linear(x8, sx, w8, sw, None, workspace=ws, out=y),  # noqa: E731
                        args.steps, args.warmup, stream)
        t_q = _timed(lambda: S.sagesla_w8a8_quantize(x), args.steps, args.warmup, stream)  # noqa: E731
        S.sagesla_check_status(ws)
        tops = 2.0 * M * N * K / (t_gemm * 1e-3) / 1e12
        qgbs = (M * K * 3 + (M // 128 + 1) * (K // 128) * 4) / (t_q * 1e-3) / 1e9
        line = {"op": "w8a8", "metric": "W8A8 block-wise INT8 linear (128x128 tiles) TOPS",
                "value": tops, "unit": "TOPS", "higher_is_better": True, "steps": args.steps,
                "warmup": args.warmup, "dtype": "int8 x int8 -> s32, fp32 scaling, bf16 out",
                "data": "synthetic", "config": {"layer": name, "M": M, "N": N, "K": K},
                "gemm_ms": t_gemm, "quantize_ms": t_q,
                "roofline": {"bound": "tensor", "achieved": tops, "peak": peak_i8, "unit": "TOPS",
                             "frac": tops / peak_i8, "traffic": None,
                             "note": f"INT8 peak = {INT8_TO_BF16_RATE:g} x the {src} cuBLAS bf16 burst"},
                "quantize_roofline": {"bound": "hbm", "achieved": qgbs,
                                      "peak": float(peaks["hbm_gbs"]), "unit": "GB/s",
                                      "frac": qgbs / float(peaks["hbm_gbs"])}}
        print(json.dumps(line), flush=True)
    return rc


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="480p", choices=sorted(WORKLOADS) + ["sweep"],
                    help="'sweep' runs the five sparsity-sweep points, one JSON line each")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--parallel", default="batch", choices=["batch", "heads"],
                    help="batch: rank r runs batch element r (default, weak scaling); heads: one "
                         "layer's heads split over the ranks (strong scaling)")
    ap.add_argument("--no-gather", action="store_true",
                    help="with --parallel heads: skip the all-gather of the outputs")
    ap.add_argument("--op", default="attention", choices=["attention", "backward", "w8a8"],
                    help="attention: the SageSLA forward path (default); backward: sagesla_backward; "
                         "w8a8: the W8A8 linear layer on the Wan-1.3B shapes")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3) if args.impl == "ours" else args.warmup
    if args.op == "w8a8":
        return run_w8a8(args)
    names = [f"sweep_rho{r:g}" for r in SWEEP_RHOS] if args.workload == "sweep" else [args.workload]
    if args.op == "backward":
        return max(run_backward(args, WORKLOADS[n]) for n in names)
    rc = 0
    for name in names:
        wl = WORKLOADS[name]
        if args.impl == "reference":
            rc |= run_reference(args, wl)
        else:
            rc |= (run_heads if args.parallel == "heads" else run_ours)(args, wl)
    return rc


if __name__ == "__main__":
    sys.exit(main())
