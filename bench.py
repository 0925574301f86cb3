#!/usr/bin/env python3
"""Benchmark of the H-BitLinear forward pass (BitNet v2) on B200.

One step = the hot path over one batch: RMSNorm -> Hadamard -> a4 quantisation -> ternary
product -> dequant, for both H-BitLinear layers of a 7B-like block (attention output Wo 4096->4096
and FFN down Wdown 16384->4096) at 8192 tokens. Weights are packed once before timing (offline).
Activations are synthetic (seeded Laplace body + 1% outlier channels x50, bf16).

Prints one JSON line (rank 0). `--impl reference` times the CPU oracle instead, on a bounded
sample of the same workload.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
  (N > 1: launched by torch.distributed.run; every rank runs an independent replica)
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from hadamard_bit_quant_hbl_b200 import inputs  # noqa: E402

METRIC = "H-BitLinear tokens/s and effective TOPS at 7B-like shapes; % of HBM/int8 roofline"
UNIT = "tokens/s"
M_TOKENS = 8192
LAYERS = ("wo_7b_a4", "wdown_7b_a4")
SWEEP_TOKENS = (1, 16, 64, 512)
WORKLOAD = ("7B-like H-BitLinear layer pair: Wo 4096->4096 + Wdown 16384->4096, a4 absmean, "
            "8192 tokens, bf16 in / bf16 out")
# DRAM bytes per launch of the dominant kernel (dram__bytes_read.sum + dram__bytes_write.sum from
# one ncu capture of the Wdown product at 8192 tokens), with the hash of the kernel source it was
# taken on (reported as null once the source has changed).
NCU_TRAFFIC = {
    "gemm_tc2[wdown_7b_a4]": {"bytes": 609.441280e6 + 73.982208e6, "src": "gemm_tc2.cuh", "sha": "84b987541e8b8b62"},
}


def product_kernel(M):
    """Name and source file of the product kernel hbl_ternary_gemm runs for M tokens."""
    if M <= 4:
        return "gemm_decode", "gemm_decode.cuh"
    return ("gemm_swap", "gemm_swap.cuh") if M <= 256 else ("gemm_tc2", "gemm_tc2.cuh")


def nfq_kernel(K, had_block, M):
    """Name of the fused activation kernel hbl_norm_fht_quant runs on M rows (no gain): the
    tensor-core kernels from 17 rows of 16384 features, 65 rows of 8192 and 257 rows otherwise."""
    if had_block == 1:
        return "norm_quant"
    if had_block == 0 and K == 16384:
        return "norm_fht_quant_tc" if M >= 17 else "norm_fht_quant"
    if had_block == 0 and K in (4096, 8192):
        return "norm_fht_quant_tc2" if M >= (65 if K == 8192 else 257) else "norm_fht_quant"
    if had_block == 256 and K <= 16384 and K & (K - 1):
        return "norm_fht_quant_tc" if M >= 257 else "norm_fht_quant"
    return "norm_fht_quant"


def act_bytes(M, K, abits):
    """Algorithmic HBM bytes of the fused activation step: the bf16 input, the codes at their
    bit width (a4: half a byte per feature), one fp32 scale per row."""
    return 2 * M * K + (M * K * abits) // 8 + 4 * M


def act_container_bytes(M, K):
    """Bytes the activation kernel moves when it writes one int8 container per code (the format
    the tensor-core products read)."""
    return 2 * M * K + M * K + 4 * M


def weight_bytes(M, K, N):
    """Weight bytes the product kernel reads for M tokens: the 2-bit section up to 256 tokens,
    the int8 section above."""
    return (K * N) // 4 if M <= 256 else K * N


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p["hbm_gbs"], p["bf16_tflops"], p["bf16_tflops_sustained"], "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


def src_hash(name):
    with open(os.path.join(ROOT, "hadamard_bit_quant_hbl_b200", "csrc", name), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


class ClockSampler:
    """Polls SM clock and clock-event reasons through NVML (read-only) while running."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, device_index):
        self.samples, self.reasons, self.max_mhz = [], 0, None
        self._stop = threading.Event()
        self._ok = False
        try:
            import pynvml

            pynvml.nvmlInit()
            self._nv = pynvml
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            phys = int(vis.split(",")[device_index]) if vis and vis.split(",")[0].isdigit() else device_index
            self._h = pynvml.nvmlDeviceGetHandleByIndex(phys)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._ok = True
        except Exception:
            pass

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                get = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                    nv.nvmlDeviceGetCurrentClocksThrottleReasons
                self.reasons |= get(self._h)
            except Exception:
                pass
            time.sleep(0.005)

    def __enter__(self):
        if self._ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        if self._ok:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        names = [n for b, n in self.REASONS.items() if self.reasons & b and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz, "reasons": names,
                "samples": len(self.samples)}


def dist_setup(n_gpus, backend="nccl"):
    """Rank, world size and local rank from the launcher's environment; with more than one rank a
    process group (NCCL on the GPUs; gloo for the host-side tests) with a short timeout, so that
    ranks waiting for a lost peer end with an error instead of hanging."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist

        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def max_over_ranks(value, world, device=None):
    """The largest `value` over all ranks (a job takes as long as its slowest replica); the value
    itself with one rank. Every rank must call it, in the same order."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank, world, ms_per_step):
    """Whole-job tokens/s: every rank's tokens over the slowest rank's step time."""
    return tokens_per_rank * world / (ms_per_step / 1e3)


# ---------------------------------------------------------------- CPU oracle (reference arm)

def oracle_prepare(rows_per_layer):
    """Inputs of the oracle sample: the first `rows_per_layer` token rows of each layer, with the
    weights ternarised beforehand (offline, like the GPU path)."""
    import oracle

    prepared = []
    for name in LAYERS:
        spec = inputs.WORKLOADS[name].with_m(rows_per_layer)
        t, alpha = oracle.absmean_ternarize(inputs.weights(spec))
        prepared.append((spec, inputs.activations(spec), t, alpha))
    return prepared


def oracle_step(prepared):
    """One oracle pass of S1-S5 over the prepared rows of both layers; returns seconds."""
    import oracle

    t0 = time.perf_counter()
    for spec, x, t, alpha in prepared:
        q, s = oracle.norm_fht_quant(x, None, spec.had_block, 4, "absmean")
        oracle.dequant(oracle.ternary_matmul(q, t), s, alpha)
    return time.perf_counter() - t0


# The oracle on all host cores: a spawned process pool (never forked from a process that has
# used the GPU), each worker mapping the ternarised weights and the sample rows from files, and
# running S1-S3 then S4-S5 on a slice of rows.
_CPU_DATA = {}


def _cpu_init(files):
    global _CPU_DATA
    import oracle  # noqa: F401  (imported before timing)

    _CPU_DATA = {name: (np.load(tp, mmap_mode="r"), alpha, np.load(xp, mmap_mode="r"), had)
                 for name, (tp, alpha, xp, had) in files.items()}


def _cpu_task(task):
    import oracle

    name, r0, r1 = task
    t, alpha, x, had = _CPU_DATA[name]
    t0 = time.perf_counter()
    q, s = oracle.norm_fht_quant(np.array(x[r0:r1]), None, had, 4, "absmean")
    t1 = time.perf_counter()
    oracle.dequant(oracle.ternary_matmul(q, t), s, alpha)
    return t1 - t0, time.perf_counter() - t1


def cpu_baseline(rows_one_core):
    """Times the oracle, as it stands, on the host: on one core over the first `rows_one_core`
    token rows of each layer, and on all available cores (one worker process per core, capped by
    free memory: each worker widens the ternary weights to int64) over `rows_one_core` rows per
    worker and layer. S1-S3 (norm, transform, quantise) and S4-S5 (integer product, dequant) are
    timed separately. Returns the cpu_baseline object of the bench line (its value: all cores)."""
    import multiprocessing as mp
    import shutil
    import tempfile

    import oracle

    try:
        cores = len(os.sched_getaffinity(0))
    except AttributeError:
        cores = os.cpu_count() or 1
    try:
        import psutil

        cores = max(1, min(cores, int(psutil.virtual_memory().available / 1.5e9)))
    except Exception:
        pass
    rows_all = rows_one_core * cores
    tmp = tempfile.mkdtemp(prefix="hbl_oracle_")
    try:
        files, prepared = {}, []
        for name in LAYERS:
            spec = inputs.WORKLOADS[name].with_m(rows_all)
            t, alpha = oracle.absmean_ternarize(inputs.weights(spec))
            x = inputs.activations(spec)
            tp, xp = os.path.join(tmp, f"{name}_t.npy"), os.path.join(tmp, f"{name}_x.npy")
            np.save(tp, t)
            np.save(xp, x)
            files[name] = (tp, alpha, xp, spec.had_block)
            prepared.append((name, t, alpha, x[:rows_one_core], spec.had_block))
        # one core, in this process
        t13 = t45 = 0.0
        for name, t, alpha, x, had in prepared:
            t0 = time.perf_counter()
            q, s_ = oracle.norm_fht_quant(x, None, had, 4, "absmean")
            t1 = time.perf_counter()
            oracle.dequant(oracle.ternary_matmul(q, t), s_, alpha)
            t13 += t1 - t0
            t45 += time.perf_counter() - t1
        del prepared
        one = {"value": rows_one_core / (t13 + t45), "unit": UNIT, "cores": 1,
               "s1_s3_s": t13, "s4_s5_s": t45,
               "sample": f"first {rows_one_core} token rows of each layer"}
        # all cores: slices of rows_one_core rows, one per worker and layer
        tasks = [(name, r0, r0 + rows_one_core) for name in LAYERS for r0 in range(0, rows_all, rows_one_core)]
        with mp.get_context("spawn").Pool(cores, initializer=_cpu_init, initargs=(files,)) as pool:
            pool.map(_cpu_task, [(LAYERS[0], 0, 1)] * cores)  # workers up (imports, file maps)
            w0 = time.perf_counter()
            parts = pool.map(_cpu_task, tasks, chunksize=1)
            wall = time.perf_counter() - w0
        busy13 = sum(p[0] for p in parts)
        busy45 = sum(p[1] for p in parts)
        return {"value": rows_all / wall, "unit": UNIT, "cores": cores, "kind": "oracle",
                "sample": f"first {rows_all} token rows of each layer ({rows_one_core} per worker and layer), "
                          f"S1-S5 with weights ternarised before timing, {wall:.1f} s on {cores} worker processes",
                "s1_s3_share": busy13 / (busy13 + busy45), "s4_s5_share": busy45 / (busy13 + busy45),
                "one_core": one}
    finally:
        shutil.rmtree(tmp, ignore_errors=True)


def run_reference(args, world, rank):
    if rank != 0:
        return
    rows = max(1, args.ref_step_rows)
    prepared = oracle_prepare(rows)
    for _ in range(args.warmup):
        oracle_step(prepared)
    times = [oracle_step(prepared) for _ in range(args.steps)]
    t = sum(times) / len(times)
    value = rows / t
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64/int64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "global_batch": M_TOKENS, "sample_rows_per_layer": rows},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": f"first {rows} token rows of each layer per step, S1-S5 "
                                   "(weights ternarised before timing)"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- GPU arm

def run_ours(args, world, rank, local):
    import torch

    import hadamard_bit_quant_hbl_b200 as hbl

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    layers = []
    for name in LAYERS:
        spec = inputs.WORKLOADS[name].with_m(M_TOKENS)
        x = inputs.activations(spec)
        W = torch.from_numpy(inputs.weights(spec)).to(dev)
        packed, alpha = hbl.hbl_pack_weights(W)
        del W
        X = torch.from_numpy(x.view(np.int16)).to(dev).view(torch.bfloat16)
        Xh = torch.from_numpy(x.view(np.int16)).pin_memory()
        fmt = hbl.HBL_CODES_I8
        codes = torch.empty((spec.M, spec.K), dtype=torch.uint8, device=dev)
        s_x = torch.empty(spec.M, dtype=torch.float32, device=dev)
        Y = torch.empty((spec.M, spec.N), dtype=torch.bfloat16, device=dev)
        Yh = torch.empty((spec.M, spec.N), dtype=torch.bfloat16).pin_memory()
        ws = torch.empty(hbl.hbl_forward_workspace(spec.M, spec.K, hbl.HBL_Q_A4_ABSMEAN), dtype=torch.uint8, device=dev)
        layers.append(dict(spec=spec, X=X, Xh=Xh, packed=packed, alpha=alpha, codes=codes, s_x=s_x, Y=Y, Yh=Yh,
                           ws=ws, fmt=fmt))
    stream = torch.cuda.current_stream(dev)
    sh = stream.cuda_stream

    def step(ev=None):
        for i, L in enumerate(layers):
            sp = L["spec"]
            hbl.hbl_norm_fht_quant(L["X"], None, sp.had_block, hbl.HBL_Q_A4_ABSMEAN, 1e-6, 0.0, L["fmt"], L["codes"],
                                   L["s_x"], stream=sh)
            if ev is not None:
                ev[2 * i].record(stream)
            hbl.hbl_ternary_gemm(L["codes"], L["fmt"], 4, L["s_x"], L["packed"], L["alpha"], sp.N, sp.K, L["Y"],
                                 hbl.HBL_OUT_BF16, None, stream=sh)
            if ev is not None:
                ev[2 * i + 1].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st = hbl.hbl_device_status()
    if st != hbl.HBL_OK:
        raise RuntimeError(hbl.hbl_status_string(st))

    # ---- timed region: exactly K steps, events between every kernel pair
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    start = torch.cuda.Event(enable_timing=True)
    if world > 1:
        import torch.distributed as dist

        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        start.record(stream)
        for k in range(args.steps):
            step(evs[k])
        while not evs[-1][-1].query():  # poll (releases the GIL) so that the clock sampler runs
            time.sleep(0.0005)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    total_ms = start.elapsed_time(evs[-1][-1])
    # per-kernel averages: [nfq Wo, gemm Wo, nfq Wdown, gemm Wdown]
    per = np.zeros(4)
    for k in range(args.steps):
        prev = start if k == 0 else evs[k - 1][3]
        marks = [prev] + evs[k]
        for j in range(4):
            per[j] += marks[j].elapsed_time(marks[j + 1])
    per /= args.steps
    # per-kernel split of the first pair includes the launch of the nfq kernel of layer 0 only
    total_ms = max_over_ranks(total_ms, world, dev)
    ms_step = total_ms / args.steps
    tokens = M_TOKENS * world
    value = job_throughput(M_TOKENS, world, ms_step)

    # ---- end to end through the public API with host buffers (pinned), copies inside the timed
    # region. Steps are pipelined as a serving loop would: the host->device copy of step k+1 and
    # the device->host copy of step k-1 run on their own streams while step k computes (PCIe is
    # full duplex); inputs and outputs are double-buffered on the device.
    e2e_steps = 0 if args.no_e2e else max(3, min(args.steps, 20))
    e2e_ms = float("nan")
    if e2e_steps:
        s_in, s_comp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
        Xd = [[L["X"], torch.empty_like(L["X"])] for L in layers]
        Yd = [[L["Y"], torch.empty_like(L["Y"])] for L in layers]

        def e2e_run(nsteps):
            ev_in, ev_comp, ev_out = [], [], []
            for k in range(nsteps):
                b = k % 2
                with torch.cuda.stream(s_in):
                    if k >= 2:
                        s_in.wait_event(ev_comp[k - 2])  # buffer b's inputs are consumed
                    for i, L in enumerate(layers):
                        Xd[i][b].copy_(L["Xh"].view(torch.bfloat16), non_blocking=True)
                    ev_in.append(torch.cuda.Event())
                    ev_in[k].record(s_in)
                s_comp.wait_event(ev_in[k])
                if k >= 2:
                    s_comp.wait_event(ev_out[k - 2])  # buffer b's outputs have left
                for i, L in enumerate(layers):
                    hbl.hbl_forward(Xd[i][b], L["packed"], L["alpha"], L["spec"].N, None, L["spec"].had_block,
                                    hbl.HBL_Q_A4_ABSMEAN, workspace=L["ws"], Y=Yd[i][b], out_dtype=hbl.HBL_OUT_BF16,
                                    stream=s_comp.cuda_stream)
                ev_comp.append(torch.cuda.Event())
                ev_comp[k].record(s_comp)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(ev_comp[k])
                    for i, L in enumerate(layers):
                        L["Yh"].copy_(Yd[i][b], non_blocking=True)
                    ev_out.append(torch.cuda.Event())
                    ev_out[k].record(s_out)

        e2e_run(2)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s_in)
        e2e_run(e2e_steps)
        e1.record(s_out)  # the last step's output copy follows every earlier operation
        torch.cuda.synchronize()
        e2e_ms = e0.elapsed_time(e1) / e2e_steps
        del Xd, Yd
    e2e_ms = max_over_ranks(e2e_ms, world, dev)
    h2d = sum(L["X"].numel() * 2 for L in layers)
    d2h = sum(L["Y"].numel() * 2 for L in layers)

    # ---- token-count sweep of the same layer pair (CUDA-graph replay over rotating weight copies)
    sweep = [] if args.no_sweep else run_sweep(layers, dev, args)
    hbm, bf16, bf16_sus, peak_src = peaks()
    int8_peak_tops = 2.0 * bf16  # burst bf16 x nominal dense int8:bf16 ratio (4.5 : 2.25 PFLOP/s)
    configs = [] if args.no_configs else time_configs(dev, hbm, int8_peak_tops)

    st = hbl.hbl_device_status()
    if st != hbl.HBL_OK:
        raise RuntimeError(hbl.hbl_status_string(st))
    if rank != 0:
        return

    kern = []
    for i, L in enumerate(layers):
        sp = L["spec"]
        nfq_bytes = act_bytes(sp.M, sp.K, 4)
        gemm_ops = 2.0 * sp.M * sp.N * sp.K
        kern.append({"kernel": f"{nfq_kernel(sp.K, sp.had_block, sp.M)}[{sp.name}]", "ms": per[2 * i], "bound": "hbm",
                     "achieved": nfq_bytes / (per[2 * i] / 1e3) / 1e9, "unit": "GB/s",
                     "frac": nfq_bytes / (per[2 * i] / 1e3) / 1e9 / hbm, "algorithmic_bytes": nfq_bytes,
                     "moved_bytes": act_container_bytes(sp.M, sp.K),
                     "note": "frac on a4 algorithmic bytes (packed int4 codes); the kernel writes one int8 "
                             "container per code, moved_bytes - algorithmic_bytes is that overhead"})
        kern.append({"kernel": f"{product_kernel(sp.M)[0]}[{sp.name}]", "ms": per[2 * i + 1], "bound": "tensor",
                     "achieved": gemm_ops / (per[2 * i + 1] / 1e3) / 1e12, "unit": "TOP/s",
                     "frac": gemm_ops / (per[2 * i + 1] / 1e3) / 1e12 / int8_peak_tops})
    dom = max(kern, key=lambda k: k["ms"])
    # algorithmic bytes of the dominant (Wdown) product: a4 codes, 2-bit weights, bf16 output
    dom_layer = layers[-1]["spec"]
    dom_bytes = dom_layer.M * dom_layer.K // 2 + dom_layer.K * dom_layer.N // 4 + 2 * dom_layer.M * dom_layer.N
    traffic = None
    rec = NCU_TRAFFIC.get(dom["kernel"])
    if rec and src_hash(rec["src"]) == rec["sha"]:  # null once the kernel source has changed
        traffic = rec["bytes"]
    eff_tops = sum(2.0 * L["spec"].M * L["spec"].N * L["spec"].K for L in layers) / (ms_step / 1e3) / 1e12

    # CPU baseline: the oracle on a bounded sample (rank 0, N = 1 only)
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(args.ref_rows)

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int8 codes x ternary, int32 accumulate; fp32 transform",
        "data": "synthetic (seeded Laplace + outlier channels, bf16)",
        "config": {"workload": WORKLOAD, "global_batch": M_TOKENS * world, "tokens_per_gpu": M_TOKENS,
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": "inputs larger than L2 (335 MB of bf16 activations per step)"},
        "effective_tops": eff_tops,
        "roofline": {"bound": dom["bound"], "achieved": dom["achieved"],
                     "peak": int8_peak_tops if dom["bound"] == "tensor" else hbm,
                     "unit": "TOP/s" if dom["bound"] == "tensor" else "GB/s", "frac": dom["frac"],
                     "traffic": traffic, "kernel": dom["kernel"],
                     "peak_source": (f"{peak_src} bf16 burst x2 (int8:bf16 nominal ratio; the timed region is "
                                     f"short, so the burst figure applies)"
                                     if dom["bound"] == "tensor" else f"{peak_src} HBM copy"),
                     "frac_of_sustained_peak": (dom["achieved"] / (2.0 * bf16_sus) if dom["bound"] == "tensor"
                                                else None),
                     "algorithmic_bytes": dom_bytes,
                     "traffic_note": "DRAM bytes above the algorithmic ones: A tiles re-read per 256-column tile "
                                     "and weights read as int8 (the kernel is bound by the tensor pipe)"},
        "kernels": kern,
        "e2e": ({"value": tokens / (e2e_ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                 "d2h_bytes_per_step": d2h} if e2e_steps else None),
        "gpu_launches": 4 * args.steps,
        "sweep": sweep,
        "configs": configs,
        "clocks": clk.summary(),
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)


def run_sweep(layers, dev, args):
    """Per token count M: one step = hbl_forward of Wo then Wdown on the first M rows. A CUDA
    graph holds R consecutive steps, each on its own copy of the packed weights, so that the
    weight bytes of a step come from HBM (R copies of the bytes the product reads exceed L2)
    without a flush kernel in the timed region. Reports tokens/s, effective TOPS and the
    bandwidth on the weight bytes the product reads (2-bit up to 256 tokens, int8 above)."""
    import torch

    import hadamard_bit_quant_hbl_b200 as hbl

    R = 8
    copies = [[L["packed"]] + [L["packed"].clone() for _ in range(R - 1)] for L in layers]
    out = []
    for M in SWEEP_TOKENS:
        bufs = []
        for L in layers:
            sp = L["spec"]
            Y = torch.empty((M, sp.N), dtype=torch.bfloat16, device=dev)
            ws = torch.empty(hbl.hbl_forward_workspace(M, sp.K, hbl.HBL_Q_A4_ABSMEAN), dtype=torch.uint8, device=dev)
            bufs.append((L, L["X"][:M], Y, ws))

        def steps(s):
            for r in range(R):
                for i, (L, X, Y, ws) in enumerate(bufs):
                    hbl.hbl_forward(X, copies[i][r], L["alpha"], L["spec"].N, None, L["spec"].had_block,
                                    hbl.HBL_Q_A4_ABSMEAN, workspace=ws, Y=Y, out_dtype=hbl.HBL_OUT_BF16, stream=s)

        cap = torch.cuda.Stream(dev)
        with torch.cuda.stream(cap):
            steps(cap.cuda_stream)  # warm-up outside capture (one-time host setup)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap):
            steps(cap.cuda_stream)
        torch.cuda.synchronize()
        reps = max(5, min(args.sweep_steps // R, 50))
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        cur = torch.cuda.current_stream(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(cur)
        for _ in range(reps):
            g.replay()
        e1.record(cur)
        e1.synchronize()
        ms = e0.elapsed_time(e1) / (reps * R)
        wbytes = sum(weight_bytes(M, L["spec"].K, L["spec"].N) for L in layers)
        ops = sum(2.0 * M * L["spec"].N * L["spec"].K for L in layers)
        out.append({"M": M, "ms_per_step": ms, "tokens_per_s": M / (ms / 1e3), "effective_tops": ops / (ms / 1e3) / 1e12,
                    "weight_bytes": wbytes, "weight_GBps": wbytes / (ms / 1e3) / 1e9,
                    "product": product_kernel(M)[0],
                    "l2": f"{R} weight copies rotated per graph replay"})
        del g
    del copies
    return out


CONFIG_CASES = [("wo_1p3b_a4", "1.3B-like Wo a4, 2048 x 2048 -> 2048"),
                ("wdown_3b_a4", "3B-like Wdown a4, 4096 x 8192 -> 2560"),
                ("wdown_nonpow2_a4", "Wdown a4 with block-diagonal transform (43 x 256), 8192 x 11008 -> 4096")]


def time_configs(dev, hbm, int8_peak, reps=20):
    """CUDA-event times of the activation kernel and of the product kernel, each launched alone
    on its own stream, for the other full-size workloads. Every launch works on the next of
    several copies of its inputs and outputs whose total exceeds L2."""
    import torch

    import hadamard_bit_quant_hbl_b200 as hbl

    out = []
    s = torch.cuda.Stream(dev)
    for name, label in CONFIG_CASES:
        spec = inputs.WORKLOADS[name]
        M, K, N = spec.M, spec.K, spec.N
        quant = hbl.HBL_Q_A8_ABSMAX if spec.abits == 8 else hbl.HBL_Q_A4_ABSMEAN
        X0 = torch.from_numpy(inputs.activations(spec).view(np.int16)).to(dev).view(torch.bfloat16)
        p0, alpha = hbl.hbl_pack_weights(torch.from_numpy(inputs.weights(spec)).to(dev))
        nb_act = 3 * M * K + 4 * M
        nb_prod = M * K + p0.numel() + 2 * M * N
        na = max(2, -(-400_000_000 // nb_act))
        npd = max(2, -(-400_000_000 // nb_prod))
        acts = [(X0 if i == 0 else X0.clone(), torch.empty((M, K), dtype=torch.uint8, device=dev),
                 torch.empty(M, dtype=torch.float32, device=dev)) for i in range(na)]
        prods = [(acts[i % na][1], acts[i % na][2], p0 if i == 0 else p0.clone(),
                  torch.empty((M, N), dtype=torch.bfloat16, device=dev)) for i in range(npd)]

        def act(j):
            X, codes, sx = acts[j % na]
            hbl.hbl_norm_fht_quant(X, None, spec.had_block, quant, 1e-6, 0.0, hbl.HBL_CODES_I8, codes, sx,
                                   stream=s.cuda_stream)

        def prod(j):
            codes, sx, packed, Y = prods[j % npd]
            hbl.hbl_ternary_gemm(codes, hbl.HBL_CODES_I8, spec.abits, sx, packed, alpha, N, K, Y, hbl.HBL_OUT_BF16,
                                 None, stream=s.cuda_stream)

        res = {}
        with torch.cuda.stream(s):
            for j in range(na):
                act(j)  # every codes buffer written before the products read them
            for fn, key in ((act, "act"), (prod, "prod")):
                for j in range(3):
                    fn(j)
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(s)
                for j in range(reps):
                    fn(j)
                e1.record(s)
                e1.synchronize()
                res[key] = e0.elapsed_time(e1) / reps * 1e3  # us
        st = hbl.hbl_device_status()
        if st != hbl.HBL_OK:
            raise RuntimeError(hbl.hbl_status_string(st))
        ab = act_bytes(M, K, spec.abits)
        ops = 2.0 * M * N * K
        out.append({
            "config": label, "M": M, "K": K, "N": N, "had_block": spec.had_block,
            "activation": {"kernel": nfq_kernel(K, spec.had_block, M), "us": res["act"], "bound": "hbm",
                           "algorithmic_bytes": ab, "moved_bytes": act_container_bytes(M, K),
                           "GBps": ab / res["act"] / 1e3, "frac": ab / res["act"] / 1e3 / hbm},
            "product": {"kernel": product_kernel(M)[0], "us": res["prod"], "bound": "tensor",
                        "TOPs": ops / res["prod"] / 1e6, "frac": ops / res["prod"] / 1e6 / int8_peak},
            "forward_us": res["act"] + res["prod"], "tokens_per_s": M / ((res["act"] + res["prod"]) / 1e6),
            "l2": f"{na} activation and {npd} product input copies rotated"})
        del acts, prods, X0, p0
    return out


def run_profile_product(M):
    """Runs the activation kernel once and the product three times on the Wdown shape with M
    tokens (a small, self-contained target for an ncu capture of one product kernel)."""
    import torch

    import hadamard_bit_quant_hbl_b200 as hbl

    torch.cuda.set_device(0)
    spec = inputs.WORKLOADS["wdown_7b_a4"].with_m(M)
    X = torch.from_numpy(inputs.activations(spec).view(np.int16)).cuda().view(torch.bfloat16)
    packed, alpha = hbl.hbl_pack_weights(torch.from_numpy(inputs.weights(spec)).cuda())
    codes, s_x = hbl.hbl_norm_fht_quant(X, None, 0, hbl.HBL_Q_A4_ABSMEAN, 1e-6, 0.0, hbl.HBL_CODES_I8)
    for _ in range(3):
        hbl.hbl_ternary_gemm(codes, hbl.HBL_CODES_I8, 4, s_x, packed, alpha, spec.N, spec.K, out_dtype=hbl.HBL_OUT_BF16)
    torch.cuda.synchronize()
    st = hbl.hbl_device_status()
    if st != hbl.HBL_OK:
        raise RuntimeError(hbl.hbl_status_string(st))
    print(f"product {product_kernel(M)[0]}: M={M} K={spec.K} N={spec.N}, 3 launches", flush=True)


def run_profile_activation(name, M):
    """Runs the fused activation kernel (a4 absmean, int8 codes) three times on one workload with
    M tokens: a small, self-contained target for an ncu capture; no bench line."""
    import torch

    import hadamard_bit_quant_hbl_b200 as hbl

    torch.cuda.set_device(0)
    spec = inputs.WORKLOADS[name].with_m(M)
    quant = hbl.HBL_Q_A8_ABSMAX if spec.abits == 8 else hbl.HBL_Q_A4_ABSMEAN
    X = torch.from_numpy(inputs.activations(spec).view(np.int16)).cuda().view(torch.bfloat16)
    codes = torch.empty((M, spec.K), dtype=torch.uint8, device="cuda")
    s_x = torch.empty(M, dtype=torch.float32, device="cuda")
    for _ in range(3):
        hbl.hbl_norm_fht_quant(X, None, spec.had_block, quant, 1e-6, 0.0, hbl.HBL_CODES_I8, codes, s_x)
    torch.cuda.synchronize()
    st = hbl.hbl_device_status()
    if st != hbl.HBL_OK:
        raise RuntimeError(hbl.hbl_status_string(st))
    print(f"activation {nfq_kernel(spec.K, spec.had_block, M)}: {name} M={M} K={spec.K}, 3 launches", flush=True)


def run_profile_forward(M, name="wdown_7b_a4", decode=False):
    """Runs hbl_forward three times on one workload with M tokens (with `decode`, one token through
    hbl_forward_decode: the fused decode kernel, one launch per layer); an ncu target, no bench
    line."""
    import torch

    import hadamard_bit_quant_hbl_b200 as hbl

    torch.cuda.set_device(0)
    spec = inputs.WORKLOADS[name].with_m(M)
    X = torch.from_numpy(inputs.activations(spec).view(np.int16)).cuda().view(torch.bfloat16)
    packed, alpha = hbl.hbl_pack_weights(torch.from_numpy(inputs.weights(spec)).cuda())
    for _ in range(3):
        if decode:
            hbl.hbl_forward_decode(X, packed, alpha, spec.N, None, 0, hbl.HBL_Q_A4_ABSMEAN, out_dtype=hbl.HBL_OUT_BF16)
        else:
            hbl.hbl_forward(X, packed, alpha, spec.N, None, 0, hbl.HBL_Q_A4_ABSMEAN, out_dtype=hbl.HBL_OUT_BF16)
    torch.cuda.synchronize()
    st = hbl.hbl_device_status()
    if st != hbl.HBL_OK:
        raise RuntimeError(hbl.hbl_status_string(st))
    print(f"forward: {name} M={M}, 3 calls", flush=True)


def run_profile_qkv(M, H=32, D=128, bits=3):
    """Runs the post-RoPE QKV quantiser three times on M tokens x H heads x D (positions 0..M-1):
    an ncu target; no bench line."""
    import torch

    import hadamard_bit_quant_hbl_b200 as hbl

    torch.cuda.set_device(0)
    X = torch.from_numpy(inputs.qkv_states(M, H, D).view(np.int16)).cuda().view(torch.bfloat16)
    pos = torch.arange(M, dtype=torch.int32, device="cuda")
    for _ in range(3):
        hbl.hbl_qkv_quant(X, H, D, bits, pos=pos)
    torch.cuda.synchronize()
    st = hbl.hbl_device_status()
    if st != hbl.HBL_OK:
        raise RuntimeError(hbl.hbl_status_string(st))
    print(f"qkv_quant: M={M} H={H} D={D} bits={bits}, 3 launches", flush=True)


ACTIVATION_CASES = [("wo_7b_a4", 8192), ("wdown_7b_a4", 8192), ("wdown_3b_a4", 4096),
                    ("wdown_nonpow2_a4", 8192), ("wo_1p3b_a4", 2048), ("qkv_7b_plain_a4", 8192)]


def run_activation_only(reps=50):
    """Times the fused activation kernel (hbl_norm_fht_quant, a4 absmean, int8 codes) alone on
    each workload width, with CUDA events on its stream. Each launch works on the next of several
    input/output copies whose total exceeds L2, so that no launch finds its data in L2. Prints one
    line per workload with the rate on the algorithmic bytes (the bf16 input, half a byte per a4
    code, one scale per row) and on the bytes moved (one int8 container per code); no bench line."""
    import torch

    import hadamard_bit_quant_hbl_b200 as hbl

    torch.cuda.set_device(0)
    peak, _, _, peak_src = peaks()
    for name, M in ACTIVATION_CASES:
        spec = inputs.WORKLOADS[name].with_m(M)
        K = spec.K
        nbytes = M * K * 3 + M * 4
        ncopy = max(2, -(-400_000_000 // nbytes))
        X0 = torch.from_numpy(inputs.activations(spec).view(np.int16)).cuda().view(torch.bfloat16)
        bufs = [(X0.clone(), torch.empty((M, K), dtype=torch.uint8, device="cuda"),
                 torch.empty(M, dtype=torch.float32, device="cuda")) for _ in range(ncopy)]
        del X0
        s = torch.cuda.Stream()

        def launch(j):
            X, codes, sx = bufs[j % ncopy]
            hbl.hbl_norm_fht_quant(X, None, spec.had_block, hbl.HBL_Q_A4_ABSMEAN, 1e-6, 0.0, hbl.HBL_CODES_I8,
                                   codes, sx, stream=s.cuda_stream)

        with torch.cuda.stream(s):
            for j in range(max(5, ncopy)):
                launch(j)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(s)
            for j in range(reps):
                launch(j)
            e1.record(s)
        e1.synchronize()
        st = hbl.hbl_device_status()
        if st != hbl.HBL_OK:
            raise RuntimeError(hbl.hbl_status_string(st))
        us = e0.elapsed_time(e1) / reps * 1000
        kern = nfq_kernel(K, spec.had_block, M)
        ab = act_bytes(M, K, spec.abits)
        print(f"{kern:18s} {name:18s} M={M:5d} K={K:6d} had_block={spec.had_block:4d} {us:8.1f} us "
              f"{ab / us / 1e3:7.1f} GB/s {ab / us / 1e3 / peak:6.3f} of {peak_src} HBM on a4 algorithmic bytes "
              f"({nbytes / us / 1e3 / peak:6.3f} on the int8-container bytes moved; {ncopy} copies rotated)",
              flush=True)
        del bufs
    # the low-bit QKV states: 8192 tokens x 32 heads x 128, RoPE at positions 0..8191, 3 bits;
    # algorithmic bytes: the bf16 states, the packed codes, one fp32 scale per head
    M, H, D, bits = 8192, 32, 128, 3
    nbytes = 2 * M * H * D + M * H * D * bits // 8 + 4 * M * H
    ncopy = max(2, -(-400_000_000 // nbytes))
    X0 = torch.from_numpy(inputs.qkv_states(M, H, D).view(np.int16)).cuda().view(torch.bfloat16)
    pos = torch.arange(M, dtype=torch.int32, device="cuda")
    bufs = [(X0.clone(), torch.empty((M, H, D * bits // 8), dtype=torch.uint8, device="cuda"),
             torch.empty((M, H), dtype=torch.float32, device="cuda")) for _ in range(ncopy)]
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        for j in range(max(5, ncopy)):
            X, c, g = bufs[j % ncopy]
            hbl.hbl_qkv_quant(X, H, D, bits, pos=pos, codes=c, gamma=g, stream=s.cuda_stream)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s)
        for j in range(reps):
            X, c, g = bufs[j % ncopy]
            hbl.hbl_qkv_quant(X, H, D, bits, pos=pos, codes=c, gamma=g, stream=s.cuda_stream)
        e1.record(s)
    e1.synchronize()
    st = hbl.hbl_device_status()
    if st != hbl.HBL_OK:
        raise RuntimeError(hbl.hbl_status_string(st))
    us = e0.elapsed_time(e1) / reps * 1000
    print(f"{'qkv_quant':18s} {'qkv_7b_states':18s} M={M:5d} H={H} D={D} bits={bits} RoPE {us:8.1f} us "
          f"{nbytes / us / 1e3:7.1f} GB/s {nbytes / us / 1e3 / peak:6.3f} of {peak_src} HBM on its algorithmic bytes "
          f"({ncopy} copies rotated)", flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--ref-rows", type=int, default=32,
                    help="token rows per layer in the one-core CPU-baseline sample (and per worker on all cores)")
    ap.add_argument("--ref-step-rows", type=int, default=1, help="token rows per layer in one reference step")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end measurement")
    ap.add_argument("--no-sweep", action="store_true", help="skip the token-count sweep")
    ap.add_argument("--sweep-steps", type=int, default=100)
    ap.add_argument("--no-configs", action="store_true", help="skip the per-kernel times of the other workloads")
    ap.add_argument("--profile-product", type=int, default=0, metavar="M",
                    help="only run the Wdown product three times with M tokens (an ncu target); no bench line")
    ap.add_argument("--activation-only", action="store_true",
                    help="only time the fused activation kernel alone on each workload width; no bench line")
    ap.add_argument("--profile-activation", nargs=2, metavar=("WORKLOAD", "M"),
                    help="only run the activation kernel of one workload three times (an ncu target)")
    ap.add_argument("--profile-forward", nargs="+", metavar=("M", "WORKLOAD"),
                    help="only run hbl_forward three times with M tokens on a workload (default the 7B Wdown; "
                         "an ncu target)")
    ap.add_argument("--profile-decode", default=None, metavar="WORKLOAD",
                    help="only run hbl_forward_decode (one token, one launch) three times on a workload "
                         "(an ncu target)")
    ap.add_argument("--profile-qkv", type=int, default=0, metavar="M",
                    help="only run the QKV quantiser three times on M tokens x 32 heads x 128 (an ncu target)")
    args = ap.parse_args()
    if args.activation_only:
        run_activation_only()
        return
    if args.profile_activation:
        run_profile_activation(args.profile_activation[0], int(args.profile_activation[1]))
        return
    if args.profile_qkv:
        run_profile_qkv(args.profile_qkv)
        return
    if args.profile_forward:
        run_profile_forward(int(args.profile_forward[0]), *args.profile_forward[1:2])
        return
    if args.profile_decode:
        run_profile_forward(1, args.profile_decode, decode=True)
        return
    if args.profile_product:
        run_profile_product(args.profile_product)
        return
    world, rank, local = dist_setup(args.gpus) if args.impl == "ours" else (
        int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")), 0)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_ours(args, world, rank, local)
    finally:
        if args.impl == "ours" and world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
