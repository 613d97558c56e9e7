"""Benchmark of certified Top-k attention (libcta) on B200.

Headline workload: 128K GQA decode - batch 1, 32 query heads, 8 KV heads,
d = 128, n = 131072 bf16 KV cache with sink / recent-window / needle
structure, eps = 0.01, a fresh query set every step (64-step cycle).  One
step = one call of cta_certified_topk_attn over all 32 query heads: four
kernels (logits with level histograms, row brackets, the bracketed value
pass, the exact cut with indices and outputs), err and KL on.  The metric is
query heads per second; the roofline is HBM bandwidth.  Also reported: the
same workload at eps = 0.1, the 32K decode (batch 4), end-to-end rates
through the C ABI with host buffers (with and without the indices), the tiny
config's microseconds per call, the Gaussian sweep and the BERT-shaped
all-query workload.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl libcta|reference]

N > 1 runs under torchrun, one process per GPU, each rank an independent
replica of the workload (rows shard with no exchange step: weak scaling); the
time is the maximum over ranks.  ``--impl reference`` times the fp64 CPU
oracle on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "certified top-k attn query-heads/s & HBM GB/s (% of peak) at n=32K/128K"
UNIT = "query-heads/s"
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "traffic.json")
# the source files of each decode kernel (a profiled traffic figure counts only
# while these are unchanged since its capture)
KERNEL_FILES = {"score_kv_tc_kernel": ("score_kv_tc.cu", "common.cuh", "umma.cuh"),
                "bracket_tc_kernel": ("gather_tc.cu", "common.cuh"),
                "gather_tc_kernel": ("gather_tc.cu", "common.cuh", "umma.cuh"),
                "settle_tc_kernel": ("settle_tc.cu", "common.cuh")}
NOMINAL_HBM_GBS = 8000.0  # B200 HBM3e, nominal (the measured copy peak is the roofline's denominator)
# the four kernels of one decode call (bf16 K, V with d = 128), in launch order
DECODE_PHASES = ("logits", "brackets", "values", "settle")
DECODE_KERNELS = {"logits": "score_kv_tc_kernel", "brackets": "bracket_tc_kernel",
                  "values": "gather_tc_kernel", "settle": "settle_tc_kernel"}


# --------------------------------------------------------------------------
# distributed plumbing (tested on CPU with gloo)


def dist_env():
    """(rank, world, local_rank) from torchrun's environment, or (0, 1, 0)."""
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def init_dist(world: int, backend: str):
    import datetime
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return dist if world > 1 else None


def barrier(dist, device=None):
    if dist is not None:
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def max_over_ranks(x: float, dist, device) -> float:
    """Largest value of x over all ranks (the job's time is its slowest rank)."""
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(rows_per_step: int, steps: int, world: int, seconds: float) -> float:
    """Whole-job throughput: the units every rank processed / the slowest time."""
    return rows_per_step * steps * world / seconds


# --------------------------------------------------------------------------
# measurement helpers


def measured_peaks() -> tuple[float, str]:
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def kernel_source_hash(kernel: str) -> str:
    h = hashlib.sha256()
    for name in KERNEL_FILES[kernel]:
        with open(os.path.join(ROOT, "certified_top_sparse_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, or
    None when it is missing or the kernel's sources changed since the capture."""
    try:
        with open(PROFILE_TRAFFIC) as f:
            rec = json.load(f)
    except Exception:
        return None
    k = rec.get("kernels", {}).get(kernel)
    if k is None or kernel not in KERNEL_FILES or k.get("source_hash") != kernel_source_hash(kernel):
        return None
    return k.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi SM clocks and throttle reasons sampled during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu = gpu_id
        self.proc = None
        self.path = f"/tmp/cta_clocks_{os.getpid()}.csv"

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            self.proc.wait(timeout=10)

    def summary(self) -> dict:
        try:
            lines = [l.split(",") for l in open(self.path).read().strip().splitlines()]
        except Exception:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        rows = [[c.strip() for c in l] for l in lines if len(l) >= 9]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        loaded = [s for s in sm if mx and s >= 0.5 * max(mx)] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}


# --------------------------------------------------------------------------
# the libcta arm


def algorithmic_bytes(prob, k_rows=None) -> dict:
    """Bytes one step must move at minimum: K once per KV head for the logits,
    every V row once per KV head for the output (the exact head-tail error
    needs the dropped rows too; at k/n ~ 0.9 with four query heads per KV head
    the union of the kept rows is every row as well), q and outputs
    (negligible), and the kept indices written (reported separately).  Per
    kernel: the logits pass reads K, the value pass reads V, the last kernel
    writes the indices (and reads one bit per key of the kept-for-certain mask)."""
    kv = prob.batch * prob.n_kv_heads * prob.n * prob.d * prob.K.element_size()
    idx = 0 if k_rows is None else int(k_rows.sum()) * 4
    mask = prob.rows * prob.n // 8
    return {"logits": kv, "brackets": 0, "values": kv, "settle": idx + mask, "step": 2 * kv,
            "idx_write": idx}


def decode_config(workload: str, prob, eps: float, world: int) -> dict:
    """The bench line's `config` for a decode workload (the same in both arms)."""
    nq = len(prob.meta["q_steps"]) if "q_steps" in prob.meta else 1
    kv = 2 * prob.batch * prob.n_kv_heads * prob.n * prob.d * prob.K.element_size()
    return {
        "workload": (f"{workload}: batch {prob.batch}, {prob.n_heads} query heads, "
                     f"{prob.n_kv_heads} KV heads, d={prob.d}, n={prob.n}, bf16 KV cache "
                     f"(sink/window/needle structure), eps={eps}, "
                     + ("fresh queries each step (64-step cycle)" if nq > 1 else "fixed queries")),
        "input_dtype": "bf16", "query_heads_per_step": prob.rows, "err_and_kl": True,
        "l2": "inputs larger than L2 (K+V %.0f MB per step); no flush" % (kv / 1e6),
        "parallelism": f"replicas x{world}",
    }


def run_libcta(args, rank, world, local_rank) -> dict | None:
    import torch
    import certified_top_sparse_b200 as cta
    from certified_top_sparse_b200 import workloads as W

    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    dist = init_dist(world, "nccl")
    prob = W.decode128k() if args.workload == "decode128k" else W.decode32k()
    eps = args.eps if args.eps is not None else prob.eps
    if args.workload == "decode128k":
        q_steps = prob.meta["q_steps"].to(device)                   # [64, B, H, 1, d]
    else:
        q_steps = prob.q.unsqueeze(0).to(device)
    K, V = prob.K.to(device), prob.V.to(device)
    rows = prob.rows
    rshape = (prob.batch, prob.n_heads, prob.m)
    out = torch.empty_like(q_steps[0])
    k_out = torch.empty(rshape, dtype=torch.int32, device=device)
    idx = torch.empty((*rshape, prob.n), dtype=torch.int32, device=device)
    tv = torch.empty(rshape, dtype=torch.float32, device=device)
    err = torch.empty(rshape, dtype=torch.float32, device=device)
    kl = torch.empty(rshape, dtype=torch.float32, device=device)
    status = torch.zeros(1, dtype=torch.int32, device=device)
    ws = torch.empty(cta.cta_workspace_size(prob.n, prob.d, prob.n_heads, prob.n_kv_heads,
                                            batch=prob.batch), dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)
    nq = q_steps.shape[0]

    def step(t, events=None, with_err=True):
        cta.cta_certified_topk_attn(q_steps[t % nq], K, V, eps, out=out, k_out=k_out, idx_out=idx,
                                    tv_out=tv, err_out=err, kl_out=kl, want_err=with_err,
                                    want_kl=with_err, workspace=ws, status_dev=status,
                                    stream=stream, phase_events=events)

    for t in range(args.warmup):
        step(t)
    torch.cuda.synchronize(device)
    assert int(status.item()) == 0, f"device status {int(status.item()):#x}"

    # per-phase events, one set per step, recorded inside the timed region
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    for s in ev:
        for e in s:
            e.record(stream)
    handles = [(ctypes.c_void_p * 5)(*[e.cuda_event for e in s]) for s in ev]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(device)

    visible = os.environ.get("CUDA_VISIBLE_DEVICES")
    gpu_id = visible.split(",")[local_rank].strip() if visible else str(local_rank)
    # Headline: K back-to-back steps with events only around the region (an
    # event between two kernels would stop the value pass from launching while
    # selection runs and adds a gap per phase).  Then the same K steps again
    # with the per-phase events, for the phase times and the roofline.
    with ClockSampler(gpu_id) as clocks:
        barrier(dist, device)
        torch.cuda.synchronize(device)
        start.record(stream)
        for t in range(args.steps):
            step(t)
        stop.record(stream)
        torch.cuda.synchronize(device)
        barrier(dist, device)
    ms = start.elapsed_time(stop)
    seconds = max_over_ranks(ms / 1e3, dist, device)
    value = aggregate(rows, args.steps, world, seconds)
    p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(dist, device)
    torch.cuda.synchronize(device)
    p0.record(stream)
    for t in range(args.steps):
        step(t, ctypes.cast(handles[t], ctypes.c_void_p))
    p1.record(stream)
    torch.cuda.synchronize(device)
    phased_seconds = max_over_ranks(p0.elapsed_time(p1) / 1e3, dist, device)
    phase = [0.0] * 4
    for s in ev:
        for j in range(4):
            phase[j] += s[j].elapsed_time(s[j + 1])
    phase = [p / args.steps for p in phase]

    # the same step without the error term and KL (out, k, idx, tv only): the
    # dropped rows' value sums are skipped, so the output pass does half the FMAs
    ne_steps = max(1, min(args.steps, 2000))
    for t in range(3):
        step(t, with_err=False)
    torch.cuda.synchronize(device)
    barrier(dist, device)
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s0.record(stream)
    for t in range(ne_steps):
        step(t, with_err=False)
    s1.record(stream)
    torch.cuda.synchronize(device)
    ne_seconds = max_over_ranks(s0.elapsed_time(s1) / 1e3, dist, device)
    for t in range(ne_steps):  # phase times, in a region of their own
        step(t, ctypes.cast(handles[t], ctypes.c_void_p), with_err=False)
    torch.cuda.synchronize(device)
    ne_phase = [0.0] * 4
    for s in ev[:ne_steps]:
        for j in range(4):
            ne_phase[j] += s[j].elapsed_time(s[j + 1])
    ne_phase = [p / ne_steps for p in ne_phase]

    # End to end through the public call with host buffers: every step's q comes
    # in from pinned host memory and its results (out, and k/TV/err/KL packed in
    # one buffer) go back to pinned host memory, on a copy stream that overlaps
    # the neighbouring steps' kernels; device and host buffers are double
    # buffered and ordered by events.  idx stays on the device.
    host_q = q_steps.cpu().pin_memory()
    host_out = [torch.empty_like(out, device="cpu").pin_memory() for _ in range(2)]
    host_small = [torch.empty((4, *rshape), dtype=torch.float32).pin_memory() for _ in range(2)]
    dev_q = [torch.empty_like(q_steps[0]) for _ in range(2)]
    dev_out = [out, torch.empty_like(out)]
    dev_small = [torch.empty((4, *rshape), dtype=torch.float32, device=device) for _ in range(2)]
    copy = torch.cuda.Stream(device)
    ev_done = [torch.cuda.Event() for _ in range(2)]   # step t's kernels have finished
    ev_ready = [torch.cuda.Event() for _ in range(2)]  # step t's q is in; its buffers are free
    e2e_steps = max(1, min(args.steps, 2000))

    def e2e_prime(t):  # q of steps t, t + 1 before the first of them
        for j in (t, t + 1):
            with torch.cuda.stream(copy):
                dev_q[j % 2].copy_(host_q[j % nq], non_blocking=True)
                ev_ready[j % 2].record(copy)

    def e2e_step(t):
        b = t % 2
        stream.wait_event(ev_ready[b])  # the one cross-stream wait of the compute stream
        sm = dev_small[b]
        cta.cta_certified_topk_attn(dev_q[b], K, V, eps, out=dev_out[b],
                                    k_out=sm[0].view(torch.int32), idx_out=idx, tv_out=sm[1],
                                    err_out=sm[2], kl_out=sm[3], workspace=ws, status_dev=status,
                                    stream=stream)
        ev_done[b].record(stream)
        with torch.cuda.stream(copy):
            copy.wait_event(ev_done[b])
            host_out[b].copy_(dev_out[b], non_blocking=True)   # step t's results out
            host_small[b].copy_(sm, non_blocking=True)         # (k as raw int32 bits)
            dev_q[b].copy_(host_q[(t + 2) % nq], non_blocking=True)  # step t + 2's q in
            ev_ready[b].record(copy)

    e2e_prime(0)
    for t in range(3):
        e2e_step(t)
    torch.cuda.synchronize(device)
    barrier(dist, device)
    s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s2.record(stream)
    e2e_prime(0)
    for t in range(e2e_steps):
        e2e_step(t)
    stream.wait_event(ev_ready[(e2e_steps - 1) % 2])  # the last results are on the host
    e2.record(stream)
    torch.cuda.synchronize(device)
    e2e_seconds = max_over_ranks(s2.elapsed_time(e2) / 1e3, dist, device)
    # the last step's results, read on the host, match the device's
    last = (e2e_steps - 1) % 2
    assert torch.equal(host_out[last], dev_out[last].cpu()), "e2e results differ from the device's"
    h2d = q_steps[0].numel() * q_steps[0].element_size()
    d2h = out.numel() * out.element_size() + 4 * rows * 4

    # The same, with the kept indices copied back too (idx is the largest
    # result: rows x n int32 per step; the copy crosses PCIe and bounds the rate).
    ei_steps = max(1, min(args.steps, 200))
    host_idx = [torch.empty_like(idx, device="cpu").pin_memory() for _ in range(2)]
    dev_idx = [idx, torch.empty_like(idx)]

    def e2e_idx_step(t):
        b = t % 2
        stream.wait_event(ev_ready[b])
        sm = dev_small[b]
        cta.cta_certified_topk_attn(dev_q[b], K, V, eps, out=dev_out[b],
                                    k_out=sm[0].view(torch.int32), idx_out=dev_idx[b], tv_out=sm[1],
                                    err_out=sm[2], kl_out=sm[3], workspace=ws, status_dev=status,
                                    stream=stream)
        ev_done[b].record(stream)
        with torch.cuda.stream(copy):
            copy.wait_event(ev_done[b])
            host_out[b].copy_(dev_out[b], non_blocking=True)
            host_small[b].copy_(sm, non_blocking=True)
            host_idx[b].copy_(dev_idx[b], non_blocking=True)
            dev_q[b].copy_(host_q[(t + 2) % nq], non_blocking=True)
            ev_ready[b].record(copy)

    torch.cuda.synchronize(device)
    e2e_prime(0)
    for t in range(3):
        e2e_idx_step(t)
    torch.cuda.synchronize(device)
    barrier(dist, device)
    s3, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s3.record(stream)
    e2e_prime(0)
    for t in range(ei_steps):
        e2e_idx_step(t)
    stream.wait_event(ev_ready[(ei_steps - 1) % 2])
    e3.record(stream)
    torch.cuda.synchronize(device)
    ei_seconds = max_over_ranks(s3.elapsed_time(e3) / 1e3, dist, device)
    last = (ei_steps - 1) % 2
    assert torch.equal(host_idx[last], dev_idx[last].cpu()), "e2e indices differ from the device's"
    d2h_idx = d2h + idx.numel() * idx.element_size()

    assert int(status.item()) == 0, f"device status {int(status.item()):#x}"
    nbytes = algorithmic_bytes(prob, k_out.reshape(-1).cpu())
    peak, peak_kind = measured_peaks()
    names = DECODE_PHASES
    dom = max(range(4), key=lambda j: phase[j])
    dom_name = names[dom]
    dom_bytes = nbytes.get(dom_name, 0)
    achieved = dom_bytes / (phase[dom] / 1e3) / 1e9 if dom_bytes else None
    step_gbs = nbytes["step"] / (seconds / args.steps) / 1e9
    ne_dom = max(range(4), key=lambda j: ne_phase[j])
    ne_bytes = nbytes.get(names[ne_dom], 0)
    ne_achieved = ne_bytes / (ne_phase[ne_dom] / 1e3) / 1e9 if ne_bytes else None
    kernel_rates = {
        nm: {"kernel": DECODE_KERNELS[nm], "ms": round(phase[j], 5),
             "algorithmic_bytes": nbytes[nm],
             "gbs": (nbytes[nm] / (phase[j] / 1e3) / 1e9) if nbytes[nm] and phase[j] > 0 else None}
        for j, nm in enumerate(names)}
    res = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": seconds * 1e3 / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": decode_config(args.workload, prob, eps, world),
        "roofline": {
            "bound": "hbm", "kernel": DECODE_KERNELS[dom_name], "achieved": achieved, "peak": peak,
            "unit": "GB/s", "frac": achieved / peak if achieved else None,
            "traffic": profiled_traffic(DECODE_KERNELS[dom_name]),
            "algorithmic_bytes_per_launch": dom_bytes, "peak_source": peak_kind,
        },
        "step_roofline": {"achieved_gbs": step_gbs, "frac": step_gbs / peak,
                          "peak": peak, "peak_source": peak_kind,
                          "frac_of_nominal": step_gbs / NOMINAL_HBM_GBS,
                          "nominal_peak": NOMINAL_HBM_GBS,
                          "algorithmic_bytes_per_step": nbytes["step"],
                          "idx_write_bytes_per_step": nbytes["idx_write"],
                          "note": "the whole step (K and V once, ms_per_step) against the measured "
                                  "copy peak and the nominal 8 TB/s; 'roofline' is the dominant "
                                  "kernel alone"},
        "phase_ms": dict(zip(names, [round(p, 5) for p in phase])),
        "kernels": kernel_rates,
        "phase_region": {"ms_per_step": phased_seconds * 1e3 / args.steps,
                         "note": "phase_ms and the roofline come from a second run of the same "
                                 "steps with CUDA events between the kernels (which serialise "
                                 "them); value and ms_per_step from the run without"},
        "e2e": {"value": aggregate(rows, e2e_steps, world, e2e_seconds), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "note": "every step: q copied in from pinned host memory, out and k/tv/err/kl "
                        "copied back to pinned host memory, on a copy stream overlapping the "
                        "neighbouring steps' kernels (double-buffered, one event wait per step "
                        "on the compute stream); the KV cache is resident and idx stays on "
                        "the device"},
        "e2e_with_idx": {"value": aggregate(rows, ei_steps, world, ei_seconds), "unit": UNIT,
                         "steps": ei_steps, "h2d_bytes_per_step": h2d,
                         "d2h_bytes_per_step": d2h_idx,
                         "note": "as e2e, with idx_out ([rows, n] int32) also copied back to pinned "
                                 "host memory every step; 'e2e' (idx left on the device, as a "
                                 "decode loop keeps it) is the headline"},
        "no_err": {
            "value": aggregate(rows, ne_steps, world, ne_seconds), "unit": UNIT,
            "steps": ne_steps, "ms_per_step": ne_seconds * 1e3 / ne_steps,
            "phase_ms": dict(zip(names, [round(p, 5) for p in ne_phase])),
            "roofline": {"bound": "hbm", "kernel": DECODE_KERNELS[names[ne_dom]], "achieved": ne_achieved,
                         "peak": peak, "unit": "GB/s",
                         "frac": ne_achieved / peak if ne_achieved else None,
                         "algorithmic_bytes_per_launch": ne_bytes},
            "note": "err_out and kl_out not requested; timed after the main region",
        },
        # logits, row brackets, value pass, cut/indices/outputs: four per call
        "gpu_launches": 4 * args.steps,
        "k_over_n_mean": float(k_out.float().mean().item() / prob.n),
        "clocks": clocks.summary(),
    }
    if dist is not None:
        dist.destroy_process_group()
    return res if rank == 0 else None


def measured_bf16_tflops() -> tuple[float, str]:
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return 1590.0, "fallback"


def run_all_query(steps: int, warmup: int) -> dict:
    """The BERT-shaped all-query workload (self-attention, m = n = 512, d = 64,
    bf16, 8 x 12 heads): logits and value sums on tcgen05, warp-per-row
    selection.  Query rows per second, per-phase times, the tensor kernels'
    MMA rate and the selection kernel's HBM rate."""
    import torch
    import certified_top_sparse_b200 as cta
    from certified_top_sparse_b200 import workloads as W

    device = torch.device("cuda", torch.cuda.current_device())
    prob = W.bert()
    q, K, V = prob.q.to(device), prob.K.to(device), prob.V.to(device)
    rshape = (prob.batch, prob.n_heads, prob.m)
    out = torch.empty_like(q)
    k_out = torch.empty(rshape, dtype=torch.int32, device=device)
    idx = torch.empty((*rshape, prob.n), dtype=torch.int32, device=device)
    tv = torch.empty(rshape, dtype=torch.float32, device=device)
    err = torch.empty(rshape, dtype=torch.float32, device=device)
    kl = torch.empty(rshape, dtype=torch.float32, device=device)
    status = torch.zeros(1, dtype=torch.int32, device=device)
    ws = torch.empty(cta.cta_workspace_size(prob.n, prob.d, prob.n_heads, prob.n_kv_heads,
                                            batch=prob.batch, m=prob.m),
                     dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(steps)]
    for s in ev:
        for e in s:
            e.record(stream)
    handles = [(ctypes.c_void_p * 5)(*[e.cuda_event for e in s]) for s in ev]
    result = {}
    for with_err in (True, False):
        def step(events=None):
            cta.cta_certified_topk_attn(q, K, V, prob.eps, out=out, k_out=k_out, idx_out=idx,
                                        tv_out=tv, err_out=err, kl_out=kl, want_err=with_err,
                                        want_kl=with_err, workspace=ws, status_dev=status,
                                        stream=stream, phase_events=events)
        for _ in range(warmup):
            step()
        torch.cuda.synchronize(device)
        start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record(stream)
        for t in range(steps):  # timed without events between the kernels
            step()
        stop.record(stream)
        for t in range(steps):  # phase times, in a region of their own
            step(ctypes.cast(handles[t], ctypes.c_void_p))
        torch.cuda.synchronize(device)
        assert int(status.item()) == 0, f"device status {int(status.item()):#x}"
        sec = start.elapsed_time(stop) / 1e3
        ph = [sum(s[j].elapsed_time(s[j + 1]) for s in ev) / steps for j in range(4)]
        rows, n, d = prob.rows, prob.n, prob.d
        qk_flop = 2.0 * rows * n * d
        pv_flop = 2.0 * rows * n * d * (4 if with_err else 2)  # hi/lo parts; head (and tail)
        sel_bytes = 4.0 * rows * n + 4.0 * float(k_out.sum().item())
        peak_tf, peak_kind = measured_bf16_tflops()
        hbm, _ = measured_peaks()
        result["err_on" if with_err else "err_off"] = {
            "value": rows * steps / sec, "unit": "query-rows/s", "ms_per_step": sec * 1e3 / steps,
            "phase_ms": {"logits_tcgen05": round(ph[0], 5), "select": round(ph[1], 5),
                         "values_tcgen05_and_finalise": round(ph[2], 5)},
            "tensor": {"qk_tflops": qk_flop / (ph[0] / 1e3) / 1e12,
                       "pv_tflops": pv_flop / (ph[2] / 1e3) / 1e12,
                       "peak_bf16_tflops": peak_tf, "peak_source": peak_kind},
            "select_roofline": {"bound": "hbm", "achieved": sel_bytes / (ph[1] / 1e3) / 1e9,
                                "peak": hbm, "unit": "GB/s",
                                "frac": sel_bytes / (ph[1] / 1e3) / 1e9 / hbm,
                                "algorithmic_bytes": sel_bytes},
        }
    result["config"] = {"workload": "bert all-query: batch 8, 12 heads, m = n = 512, d = 64, bf16, "
                                    "heads 6-11 with planted keys, eps = 0.01",
                        "steps": steps, "warmup": warmup, "k_over_n_mean":
                            float(k_out.float().mean().item() / prob.n)}
    return result


def run_tiny(steps: int, warmup: int) -> dict:
    """The tiny Gaussian-score workload (batch 1, 8 heads, d = 64, n = 1024,
    fp32, eps = 0.01): microseconds per call, back to back on one stream
    (launch-bound: three kernels per call)."""
    import torch
    import certified_top_sparse_b200 as cta
    from certified_top_sparse_b200 import workloads as W

    device = torch.device("cuda", torch.cuda.current_device())
    prob = W.tiny()
    q, K, V = prob.q.to(device), prob.K.to(device), prob.V.to(device)
    rshape = (prob.batch, prob.n_heads, prob.m)
    out = torch.empty_like(q)
    k_out = torch.empty(rshape, dtype=torch.int32, device=device)
    idx = torch.empty((*rshape, prob.n), dtype=torch.int32, device=device)
    tv = torch.empty(rshape, dtype=torch.float32, device=device)
    err = torch.empty(rshape, dtype=torch.float32, device=device)
    status = torch.zeros(1, dtype=torch.int32, device=device)
    ws = torch.empty(cta.cta_workspace_size(prob.n, prob.d, prob.n_heads, prob.n_kv_heads,
                                            batch=prob.batch, dtype=cta.CTA_F32),
                     dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)

    def step():
        cta.cta_certified_topk_attn(q, K, V, prob.eps, out=out, k_out=k_out, idx_out=idx,
                                    tv_out=tv, err_out=err, workspace=ws, status_dev=status,
                                    stream=stream)
    for _ in range(warmup):
        step()
    torch.cuda.synchronize(device)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        step()
    b.record(stream)
    torch.cuda.synchronize(device)
    assert int(status.item()) == 0, f"device status {int(status.item()):#x}"
    us = a.elapsed_time(b) / steps * 1e3
    return {"us_per_call": us, "unit": "us/call", "steps": steps, "gpu_launches_per_call": 3,
            "config": {"workload": "tiny: batch 1, 8 heads, d=64, n=1024, fp32, Gaussian scores "
                                   "(sigma 1, 2, 3 over the heads), eps=0.01, err on"},
            "k_over_n_mean": float(k_out.float().mean().item() / prob.n)}


def run_sweep(reps: int) -> dict:
    """The Gaussian-score sweep (fp32, d = 64, 256 query rows sharing one K per
    cell): per (n, sigma, eps) cell the time per call (the mean of `reps`
    calls), the logits' FMA rate and the mean k/n beside the Gaussian rule
    Phi_c(sigma + Phi^-1(eps))."""
    import torch
    import certified_top_sparse_b200 as cta
    from certified_top_sparse_b200 import workloads as W
    from statistics import NormalDist

    device = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream(device)
    nd = NormalDist()
    cells = []
    for n in W.SWEEP_N:
        for sigma in W.SWEEP_SIGMA:
            prob = W.sweep_cell(n, sigma)
            q, K, V = prob.q.to(device), prob.K.to(device), prob.V.to(device)
            rshape = (prob.batch, prob.n_heads, prob.m)
            out = torch.empty_like(q)
            k_out = torch.empty(rshape, dtype=torch.int32, device=device)
            idx = torch.empty((*rshape, prob.n), dtype=torch.int32, device=device)
            tv = torch.empty(rshape, dtype=torch.float32, device=device)
            status = torch.zeros(1, dtype=torch.int32, device=device)
            ws = torch.empty(cta.cta_workspace_size(prob.n, prob.d, prob.n_heads, prob.n_kv_heads,
                                                    m=prob.m, dtype=cta.CTA_F32),
                             dtype=torch.uint8, device=device)
            for eps in W.SWEEP_EPS:
                def step():
                    cta.cta_certified_topk_attn(q, K, V, eps, out=out, k_out=k_out, idx_out=idx,
                                                tv_out=tv, workspace=ws, status_dev=status,
                                                stream=stream)
                for _ in range(2):
                    step()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                for _ in range(reps):
                    step()
                b.record(stream)
                torch.cuda.synchronize(device)
                assert int(status.item()) == 0, f"device status {int(status.item()):#x}"
                us = a.elapsed_time(b) / reps * 1e3
                rule = 1.0 - nd.cdf(sigma + nd.inv_cdf(eps))
                cells.append({"n": n, "sigma": sigma, "eps": eps, "us_per_call": round(us, 2),
                              "logit_tflops": 2.0 * prob.m * n * prob.d / (us * 1e-6) / 1e12,
                              "k_over_n": float(k_out.float().mean().item() / n),
                              "gaussian_rule": rule})
            del q, K, V, idx, ws
    return {"cells": cells, "unit": "us/call",
            "config": {"workload": "Gaussian-score sweep: fp32, d=64, 256 query rows per cell "
                                   "sharing K ~ N(0, I), |q| = sigma sqrt(d); n x sigma x eps = "
                                   "4 x 4 x 3 cells", "reps_per_cell": reps}}


# --------------------------------------------------------------------------
# the oracle (CPU) as the reference arm and the cpu_baseline leg


def oracle_sample(prob, q, n_keys: int, rows: int, threads: int):
    """Run the oracle on the first `rows` query heads of one step over the
    first `n_keys` keys; returns wall seconds."""
    import oracle
    from certified_top_sparse_b200 import workloads as W
    g = prob.n_heads // prob.n_kv_heads
    kv_groups = max(1, math.ceil(rows / g))
    qs = q[:, : kv_groups * g].contiguous()
    K = prob.K[:, :kv_groups, :n_keys].contiguous()
    V = prob.V[:, :kv_groups, :n_keys].contiguous()
    t0 = time.perf_counter()
    oracle.certified_topk_attn(W.raw_words(qs), W.raw_words(K), W.raw_words(V), prob.eps,
                               n_heads=kv_groups * g, n_kv_heads=kv_groups, dtype=oracle.BF16,
                               batch=prob.batch, threads=threads)
    return time.perf_counter() - t0, kv_groups * g * prob.batch


def cpu_baseline(prob, budget_rows: int | None = None) -> dict:
    """The oracle as it stands, all host cores, on whole decode steps."""
    threads = os.cpu_count() or 1
    # about 10-30 core-seconds: whole decode steps (all query heads) at full n
    steps = 2 if budget_rows is None else 1
    rows = budget_rows or prob.rows
    total, done = 0.0, 0
    for t in range(steps):
        qt = prob.meta["q_steps"][1 + t] if "q_steps" in prob.meta else prob.q
        secs, r = oracle_sample(prob, qt, prob.n, rows, threads)
        total += secs
        done += r
    return {"value": done / total, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{done} query heads ({steps} decode step(s), every head) at full "
                      f"n={prob.n}: {total:.2f} s wall on {threads} threads"}


def run_reference(args, rank, world) -> dict | None:
    """bench.py --impl reference: the fp64 oracle on host cores, rank 0 only."""
    if rank != 0:
        return None
    from certified_top_sparse_b200 import workloads as W
    prob = W.decode128k() if args.workload == "decode128k" else W.decode32k()
    threads = os.cpu_count() or 1
    g = prob.n_heads // prob.n_kv_heads
    rows = min(prob.rows, max(g, threads))
    # size the per-step sample so that warm-up + steps take about two minutes
    budget = 120.0 / max(1, args.steps + args.warmup)
    probe_keys = max(1024, prob.n // 64)
    t_probe, _ = oracle_sample(prob, prob.q, probe_keys, rows, threads)
    keys = int(min(prob.n, max(256, probe_keys * budget / max(t_probe, 1e-6))))
    q_steps = prob.meta.get("q_steps")
    for t in range(args.warmup):
        oracle_sample(prob, prob.q if q_steps is None else q_steps[t % len(q_steps)], keys, rows,
                      threads)
    total, done = 0.0, 0
    for t in range(args.steps):
        secs, r = oracle_sample(prob, prob.q if q_steps is None else q_steps[t % len(q_steps)],
                                keys, rows, threads)
        total += secs
        done += r
    value = done * (keys / prob.n) / total
    sample = (f"{rows} query heads per step over the first {keys} of n={prob.n} keys; value scaled "
              f"by {keys}/{prob.n} (work is ~linear in n, the per-row sort n log n, so the "
              f"scaling slightly favours the oracle)")
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total * 1e3 / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": decode_config(args.workload, prob,
                                args.eps if args.eps is not None else prob.eps, world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=4000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=("libcta", "reference"), default="libcta")
    ap.add_argument("--workload", choices=("decode128k", "decode32k"), default="decode128k")
    ap.add_argument("--eps", type=float, default=None)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--secondary", choices=("decode32k", "none"), default="decode32k",
                    help="also measure this workload (same method, fewer steps) and nest it")
    ap.add_argument("--all-query", choices=("bert", "none"), default="bert",
                    help="also measure the BERT-shaped all-query workload (tensor-core path)")
    ap.add_argument("--no-extras", dest="extras", action="store_false",
                    help="skip the eps = 0.1 line, the tiny-call timing and the Gaussian sweep")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank, world, local_rank = dist_env()
    if args.impl == "reference":
        res = run_reference(args, rank, world)
    else:
        res = run_libcta(args, rank, world, local_rank)
        if res is not None and args.secondary != "none" and args.secondary != args.workload \
                and world == 1:
            sub = argparse.Namespace(**{**vars(args), "workload": args.secondary,
                                        "steps": max(100, args.steps // 4)})
            r2 = run_libcta(sub, rank, world, local_rank)
            res["secondary"] = {k: r2[k] for k in ("value", "ms_per_step", "config", "roofline",
                                                   "step_roofline", "phase_ms", "k_over_n_mean",
                                                   "no_err")}
        if res is not None and world == 1 and args.extras and args.workload == "decode128k":
            # the same workload at eps = 0.1 (the other eps the 128K config names)
            sub = argparse.Namespace(**{**vars(args), "eps": 0.1, "steps": max(100, args.steps // 2)})
            r3 = run_libcta(sub, rank, world, local_rank)
            res["eps_0.1"] = {k: r3[k] for k in ("value", "ms_per_step", "config", "roofline",
                                                 "step_roofline", "phase_ms", "k_over_n_mean",
                                                 "e2e")}
        if res is not None and world == 1 and args.extras:
            res["tiny"] = run_tiny(steps=max(200, args.steps // 2), warmup=args.warmup)
            res["sweep"] = run_sweep(reps=5)
        if res is not None and args.all_query != "none" and world == 1:
            res["all_query"] = run_all_query(steps=max(20, args.steps // 40), warmup=args.warmup)
        if res is not None and world == 1 and not args.no_cpu_baseline:
            from certified_top_sparse_b200 import workloads as W
            prob = W.decode128k() if args.workload == "decode128k" else W.decode32k()
            res["cpu_baseline"] = cpu_baseline(prob)
    if res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
