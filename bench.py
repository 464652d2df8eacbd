#!/usr/bin/env python3
"""Benchmark of the block-sparse causal attention forward on B200.

One step = one pass of the hot path over one batch of the headline workload:
the layout is compiled once (it is data-independent, and its planning time is
reported on its own, as the BF1 page times topology separately), then every
step is one ``bsa_forward`` over all heads and query blocks.  ``value`` is the
effective throughput 4*d*(kept token pairs) / time over the timed steps with
inputs resident in HBM; ``e2e`` repeats the metric through the public API from
pinned host buffers (layout compile + H2D of q, k, v + forward + D2H of o and
lse inside every timed step).

``python bench.py [--gpus N --steps K --warmup W] [--impl reference]``; under
torchrun the global batch is one problem of the workload per rank and each
rank runs its own (the work items of this path share nothing, so there is no
data-path collective); rank 0 prints one JSON line with the max-over-ranks
device time and the whole-job throughput.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from block_sparse_long_bsa_b200 import inputs as synth                  # noqa: E402
from block_sparse_long_bsa_b200 import sharding                         # noqa: E402
from block_sparse_long_bsa_b200.workloads import WORKLOADS, ORDER, HEADLINE  # noqa: E402

METRIC = "block-sparse attn fwd effective TFLOPS (4·d·kept pairs/s), % of B200 bf16 peak"
UNIT = "TFLOP/s"
FALLBACK_PEAKS = {"bf16_tflops": 1590.0, "hbm_gbs": 6650.0, "bf16_tflops_sustained": 1400.0}
CSRC = os.path.join(ROOT, "block_sparse_long_bsa_b200", "csrc")
# every source the forward kernel is compiled or launched from: the kernel,
# the device helpers it includes and the tensor-map encoding of its boxes
KERNEL_SRCS = [os.path.join(CSRC, f) for f in
               ("bsa_fwd_sm100a.cu", "bsa_device.cuh", "bsa_tmap.cpp", "bsa_tmap.h")]
THROTTLE_BITS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
                 0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
                 0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
                 0x100: "display_clock_setting"}


# ------------------------------------------------------------------ helpers
def kept_pairs_of_layout(row_ptr, col_idx, n, B, L):
    """Token pairs allowed by a CSR layout (diagonal block counted causally)."""
    nb = -(-n // B)
    row_ptr = [int(x) for x in row_ptr]
    col_idx = [int(x) for x in col_idx]
    pairs = 0
    for h in range(L):
        for i in range(nb):
            rows_i = min(n, (i + 1) * B) - i * B
            for j in col_idx[row_ptr[h * nb + i]:row_ptr[h * nb + i + 1]]:
                if j < i:
                    pairs += rows_i * (min(n, (j + 1) * B) - j * B)
                elif j == i:
                    pairs += rows_i * (rows_i + 1) // 2
    return pairs


def workload_work(w, row_ptr, col_idx):
    pairs_per_layout_head = []
    nb = w.n_blocks
    for h in range(w.layout_heads):
        rp = row_ptr[h * nb:(h + 1) * nb + 1] - row_ptr[h * nb]
        ci = col_idx[row_ptr[h * nb]:row_ptr[(h + 1) * nb]]
        pairs_per_layout_head.append(kept_pairs_of_layout(rp, ci, w.n, w.B, 1))
    reps = w.heads // w.layout_heads
    pairs = sum(pairs_per_layout_head) * reps
    flops = 4 * w.d * pairs
    compulsory = 2 * (2 * w.heads * w.n * w.d + 2 * w.kv_heads * w.n * w.d) + 4 * w.heads * w.n
    return pairs, flops, compulsory


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            pk = json.load(fh)
        return pk, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_sha():
    """sha256 over the forward kernel's sources, in a fixed order."""
    h = hashlib.sha256()
    for path in KERNEL_SRCS:
        with open(path, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


E2E_GROUPS = 8   # key/value-head runs of the end-to-end call


def profiled_traffic(workload):
    """DRAM bytes per launch from the committed ncu summary, if it still
    matches the kernel source; else None."""
    path = os.path.join(ROOT, "profiles", f"bsa_fwd_sm100a_{workload}.md")
    try:
        text = open(path).read()
    except OSError:
        return None
    sha = re.search(r"kernel_sha256:\s*([0-9a-f]{64})", text)
    tr = re.search(r"traffic_bytes_per_launch:\s*([0-9]+)", text)
    if not sha or not tr or sha.group(1) != kernel_sha():
        return None
    return int(tr.group(1))


class ClockSampler:
    """SM clock, max clock, power and clock-event (throttle) reasons, sampled
    in a thread during the run: through NVML every ``period_ms`` (the timed
    region of a step is well under a millisecond, so the sampling is dense),
    else through ``nvidia-smi -lms``.  Read-only: no setting is changed."""

    def __init__(self, cuda_index: int, period_ms: float = 2.0):
        self.cuda_index = cuda_index
        self.period = period_ms / 1e3
        self.samples = []
        self.proc = None
        self.thread = None
        self.stop_flag = threading.Event()
        self.source = "none"

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        try:
            import torch
            pr = torch.cuda.get_device_properties(self.cuda_index)
            bus = f"{pr.pci_domain_id:08x}:{pr.pci_bus_id:02x}:{pr.pci_device_id:02x}.0"
            return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.cuda_index)

    def start(self):
        try:
            nv, h = self._nvml_handle()
            max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
        except Exception:
            return self._start_smi()
        self.source = "nvml"

        def poll():
            while not self.stop_flag.is_set():
                try:
                    mhz = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                    pw = nv.nvmlDeviceGetPowerUsage(h) / 1e3
                    rs = int(nv.nvmlDeviceGetCurrentClocksEventReasons(h))
                    self.samples.append((time.time(), mhz, max_mhz, pw, rs))
                except Exception:
                    pass
                time.sleep(self.period)
        self.thread = threading.Thread(target=poll, daemon=True)
        self.thread.start()

    def _start_smi(self):
        cmd = ["nvidia-smi", "-i", str(self.cuda_index),
               "--query-gpu=clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active",
               "--format=csv,noheader,nounits", "-lms", "100"]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
        except OSError:
            self.proc = None
            return
        self.source = "nvidia-smi"

        def reader():
            for line in self.proc.stdout:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 4:
                    try:
                        self.samples.append((time.time(), float(parts[0]), float(parts[1]),
                                             float(parts[2]) if parts[2] not in ("[N/A]", "N/A") else 0.0,
                                             int(parts[3], 16) if parts[3].startswith("0x") else 0))
                    except ValueError:
                        pass
        self.thread = threading.Thread(target=reader, daemon=True)
        self.thread.start()

    def stop(self):
        self.stop_flag.set()
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.thread:
            self.thread.join(timeout=5)

    def summary(self, t0, t1):
        win = [s for s in self.samples if t0 <= s[0] <= t1]
        note = "timed region"
        if len(win) < 3:
            win = [s for s in self.samples if s[0] <= t1]
            note = "warm-up and timed region"
        if not win:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "window": "none"}
        loaded = [s for s in win if not (s[4] & 0x1)] or win
        mhz = sorted(s[1] for s in loaded)
        reasons = 0
        for s in loaded:
            reasons |= s[4]
        names = [nm for bit, nm in THROTTLE_BITS.items() if reasons & bit]
        return {"sm_mhz": mhz[len(mhz) // 2], "sm_max_mhz": max(s[2] for s in win),
                "reasons": names, "power_w_max": max(s[3] for s in win),
                "samples": len(loaded), "window": note, "source": self.source}


def threads_in_use():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        if info:
            return max(int(i.get("num_threads", 1)) for i in info)
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


# ------------------------------------------------------------------ CPU oracle legs
def oracle_sample(w, sets, bits, budget_s, seed=7):
    """Time the fp64 oracle on randomly drawn (head, query block) items until
    about ``budget_s`` seconds of CPU work; returns (pairs, seconds, items)."""
    from oracle import attention as OA
    qf, kf, vf = (synth.bf16_bits_to_f64(x) for x in bits)   # upcast once, outside the clock
    rng = np.random.default_rng(seed)
    scale = 1.0 / math.sqrt(w.d)
    pairs = 0
    items = 0
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < budget_s:
        f = int(rng.integers(w.heads))
        i = int(rng.integers(w.n_blocks))
        row = sets[f % w.layout_heads][i]
        OA.forward_block_rows(qf, kf, vf, sets, w.B, scale, f, i)
        rows_i = min(w.n, (i + 1) * w.B) - i * w.B
        for j in row:
            if j < i:
                pairs += rows_i * (min(w.n, (j + 1) * w.B) - j * w.B)
            elif j == i:
                pairs += rows_i * (rows_i + 1) // 2
        items += 1
    return pairs, time.perf_counter() - t0, items


def sample_bits(w, heads_needed):
    """Seeded inputs of the workload restricted to the first heads (CPU legs)."""
    h = min(w.heads, heads_needed)
    g = w.heads // w.kv_heads
    kvh = max(1, -(-h // g))
    q = synth.normal_bf16_bits((w.heads, w.n, w.d), synth.Q_SEED)[:h]
    k = synth.normal_bf16_bits((w.kv_heads, w.n, w.d), synth.K_SEED)[:kvh]
    v = synth.normal_bf16_bits((w.kv_heads, w.n, w.d), synth.V_SEED)[:kvh]
    return q, k, v, h


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from oracle import layouts as OL
    sets = OL.kept_sets_for(w)
    q, k, v, h = sample_bits(w, 2)
    import dataclasses
    wh = dataclasses.replace(w, batch=1, q_heads=h, kv_heads_per_seq=max(1, h // (w.heads // w.kv_heads)))
    per_step = max(0.5, min(8.0, 150.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_sample(wh, sets, (q, k, v), per_step / 4)
    tot_pairs, tot_s, tot_items = 0, 0.0, 0
    for s in range(args.steps):
        p, t, it = oracle_sample(wh, sets, (q, k, v), per_step, seed=100 + s)
        tot_pairs, tot_s, tot_items = tot_pairs + p, tot_s + t, tot_items + it
    value = 4 * w.d * tot_pairs / tot_s / 1e12
    cores = threads_in_use()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot_s / max(1, args.steps),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic N(0,1) bf16 inputs upcast exactly to fp64, seeds 0/1/2; layout seed 17",
        "config": workload_config(w, args.gpus),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"{tot_items} random (head, query block) tiles of heads 0..{h - 1}, "
                                   f"~{per_step:.1f} s of fp64 oracle work per step"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(w, gpus):
    return {"workload": w.name, "batch": w.batch, "global_batch": w.batch * gpus, "q_heads": w.q_heads,
            "kv_heads": w.kv_heads_per_seq, "n": w.n, "d": w.d, "B": w.B,
            "layout_heads": w.layout_heads, "pattern": w.description,
            "parallelism": f"dp{gpus} (one problem per GPU, no data-path collective)",
            "l2": "inputs exceed the 126 MB L2 and a 256 MiB buffer is written between timed steps"}


# ------------------------------------------------------------------ GPU arm
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=HEADLINE, choices=ORDER)
    ap.add_argument("--no-per-config", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--only-device", action="store_true",
                    help="device-timed leg only (no e2e, CPU baseline or other workloads); "
                         "the form used for profiler captures")
    ap.add_argument("--leg", default=None, choices=["backward", "bsbr", "decode"],
                    help="time one secondary leg alone on --workload (backward), the BSBR "
                         "workload (bsbr) or the headline route's decode (decode) and print its "
                         "JSON; the form used for profiler captures")
    ap.add_argument("--n", type=int, default=None,
                    help="with --leg backward or decode: the workload's geometry at this sequence length "
                         "(a smaller case for full profiler captures)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    w = WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w)
    if args.leg is not None:
        return run_leg(args, w)

    import torch
    import torch.distributed as dist
    import block_sparse_long_bsa_b200 as bsa

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA GPU")
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.cuda.current_device()
    stream = torch.cuda.current_stream()
    bsa.load_library()

    def barrier():
        if world > 1:
            dist.barrier()

    # --- layout (planning timed on its own): the first build of the process,
    # then the median of warm builds with upload and of host-only compiles
    t0 = time.perf_counter()
    lay = bsa.Layout.for_workload(w, dev)
    layout_first_ms = 1e3 * (time.perf_counter() - t0)

    def median_ms(fn, reps=5):
        ts = []
        for _ in range(reps):
            t1 = time.perf_counter()
            fn().close()
            ts.append(1e3 * (time.perf_counter() - t1))
        return sorted(ts)[len(ts) // 2]

    layout_ms = median_ms(lambda: bsa.Layout.for_workload(w, dev))
    layout_host_ms = median_ms(lambda: bsa.Layout.for_workload(w, -1))
    row_ptr, col_idx = lay.csr()
    pairs, flops, compulsory = workload_work(w, row_ptr, col_idx)

    # --- inputs (seeded, synthetic; resident in HBM for the device-timed value).
    # The global batch is one problem of the workload per rank; rank r owns
    # problem r and draws its inputs from that problem's seeds.
    mine = sharding.shard(world, world, rank)
    seeds = sharding.element_seeds(mine.start)
    qb, kb, vb = synth.qkv_bits(w.heads, w.kv_heads, w.n, w.d, seeds)

    def to_dev(bits):
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(dev)

    q, k, v = to_dev(qb), to_dev(kb), to_dev(vb)
    o = torch.empty_like(q)
    lse = torch.empty((w.heads, w.n), dtype=torch.float32, device=dev)
    scale = 1.0 / math.sqrt(w.d)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)

    def fwd():
        bsa.bsa_forward(q, k, v, lay.handle, w.B, w.n, w.heads, w.kv_heads, w.d, scale, o, lse, stream)

    sampler = ClockSampler(dev)
    sampler.start()
    time.sleep(0.3)
    for _ in range(args.warmup):
        flush.fill_(1.0)
        fwd()
    torch.cuda.synchronize()
    bsa.bsa_get_status(lay.handle)

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    wall0 = time.time()
    for s in range(args.steps):
        flush.fill_(float(s))
        starts[s].record(stream)
        fwd()
        ends[s].record(stream)
    torch.cuda.synchronize()
    barrier()
    wall1 = time.time()
    bsa.bsa_get_status(lay.handle)
    step_ms = [a.elapsed_time(b) for a, b in zip(starts, ends)]
    local_total_ms = float(sum(step_ms))
    total_ms = sharding.max_over_ranks(local_total_ms, world, dev)
    ms_per_step = total_ms / args.steps
    value = sharding.aggregate_rate(flops * args.steps, world, total_ms * 1e-3) / 1e12
    clocks = sampler.summary(wall0 - 0.05, wall1 + 0.05)
    # distribution of the cold (flushed) steps above, and a warm figure taken
    # after the timed region: back-to-back launches with no flush between them
    cold = sorted(step_ms)
    warm_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(20)]
    for a_ev, b_ev in warm_ev:
        a_ev.record(stream)
        fwd()
        b_ev.record(stream)
    torch.cuda.synchronize()
    warm = sorted(a_ev.elapsed_time(b_ev) for a_ev, b_ev in warm_ev)
    step_stats = {"cold_median": cold[len(cold) // 2], "cold_p10": cold[len(cold) // 10],
                  "cold_p90": cold[min(len(cold) - 1, (9 * len(cold)) // 10)],
                  "warm_median": warm[len(warm) // 2],
                  "note": "per-launch ms on this rank; cold = 256 MiB written before each timed launch, "
                          "warm = 20 launches back to back after the timed region"}

    if args.only_device:
        if rank == 0:
            print(json.dumps({"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
                              "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
                              "config": workload_config(w, world), "partial": "device leg only"}),
                  flush=True)
        sampler.stop()
        lay.close()
        if world > 1:
            dist.destroy_process_group()
        return 0

    # --- e2e through the public API from pinned host buffers
    hq = torch.from_numpy(qb.view(np.int16)).view(torch.bfloat16).pin_memory()
    hk = torch.from_numpy(kb.view(np.int16)).view(torch.bfloat16).pin_memory()
    hv = torch.from_numpy(vb.view(np.int16)).view(torch.bfloat16).pin_memory()
    ho = torch.empty(hq.shape, dtype=torch.bfloat16).pin_memory()
    hl = torch.empty((w.heads, w.n), dtype=torch.float32).pin_memory()
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    p = w.pattern

    def e2e_step():
        # the public C entry for host buffers: copies in key/value-head runs
        # that overlap the other runs' compute
        lay2 = bsa.Layout(p.kind, w.n, w.B, w.layout_heads, dev, window=p.window,
                          global_first=p.global_first, dyadic_kmin=p.dyadic_kmin,
                          density=p.density, seed=p.seed)
        bsa.bsa_forward_host(hq, hk, hv, lay2.handle, w.B, w.n, w.heads, w.kv_heads, w.d, scale,
                             dq, dk, dv, o, lse, ho, hl, E2E_GROUPS, stream)
        return lay2

    for _ in range(2):
        e2e_step().close()
    torch.cuda.synchronize()
    barrier()
    e_start = torch.cuda.Event(enable_timing=True)
    e_end = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e_start.record(stream)
    keep = []
    for _ in range(args.e2e_steps):
        keep.append(e2e_step())
    e_end.record(stream)
    torch.cuda.synchronize()
    for l2 in keep:
        l2.close()
    e2e_ms = sharding.max_over_ranks(e_start.elapsed_time(e_end), world, dev)
    e2e_value = sharding.aggregate_rate(flops * args.e2e_steps, world, e2e_ms * 1e-3) / 1e12
    layout_bytes = 4 * (len(row_ptr) + len(col_idx) + len(row_ptr) - 1)
    pairs, flops = int(pairs), int(flops)
    h2d = q.numel() * 2 + k.numel() * 2 + v.numel() * 2 + layout_bytes
    d2h = o.numel() * 2 + lse.numel() * 4

    # --- other workloads (same kernel, same protocol, fewer steps) on rank 0
    per_config = {}
    if rank == 0 and not args.no_per_config:
        del hq, hk, hv, ho, hl, dq, dk, dv
        for name in ORDER:
            if name == w.name:
                continue
            per_config[name] = bench_other(WORKLOADS[name], dev, stream, flush, bsa, torch)
    decode = bench_decode(dev, stream, flush, bsa, torch) if rank == 0 and not args.no_per_config else None
    backward = ({name: bench_backward(WORKLOADS[name], dev, stream, flush, bsa, torch)
                 for name in (HEADLINE, "band_global_32k")}
                if rank == 0 and not args.no_per_config else None)
    bsbr = bench_bsbr(WORKLOADS["bsbr_block_diagonal"], dev, stream, flush, bsa, torch) \
        if rank == 0 and not args.no_per_config else None

    peaks, peak_src = load_peaks()
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    kernel_tflops = flops / (ms_per_step * 1e-3) / 1e12
    roofline = {"bound": "tensor", "achieved": kernel_tflops, "peak": peak, "unit": "TFLOP/s",
                "frac": kernel_tflops / peak, "traffic": profiled_traffic(w.name),
                "peak_source": f"bf16_tflops (burst) of {peak_src}",
                "algorithmic_flops_per_launch": flops,
                "hbm_gbs_compulsory": compulsory / (ms_per_step * 1e-3) / 1e9}

    # --- CPU oracle baseline (rank 0, one GPU only)
    cpu = None
    if rank == 0 and world == 1 and args.cpu_budget > 0:
        from oracle import layouts as OL
        sets = OL.kept_sets_for(w)
        sq, sk, sv, hh = sample_bits(w, 2)
        import dataclasses
        wh = dataclasses.replace(w, q_heads=hh, kv_heads_per_seq=max(1, hh // (w.heads // w.kv_heads)))
        ps, secs, its = oracle_sample(wh, sets, (sq, sk, sv), args.cpu_budget)
        cpu = {"value": 4 * w.d * ps / secs / 1e12, "unit": UNIT, "cores": threads_in_use(),
               "kind": "oracle",
               "sample": f"{its} random (head, query block) tiles of heads 0..{hh - 1} in {secs:.1f} s "
                         f"(fp64 NumPy, BLAS threads as reported)"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "step_ms": step_stats, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic N(0,1) bf16 from numpy default_rng, q/k/v seeds 3r/3r+1/3r+2 on rank r; "
                    "layout seed 17",
            "config": workload_config(w, world),
            "frac_of_peak": value / world / peak,
            "layout_build_ms": layout_ms,
            "layout_build": {"first_ms": layout_first_ms, "warm_median_ms": layout_ms,
                             "host_compile_median_ms": layout_host_ms,
                             "note": "bsa_build_layout with upload (first call of the process, then the "
                                     "median of 5), and host-only compiles; outside every timed region"},
            "kept_pairs": pairs,
            "gpu_launches": args.steps,
            "clocks": clocks,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": args.e2e_steps,
                    "includes": f"layout compile+upload, then bsa_forward_host: H2D q/k/v, forward and "
                                f"D2H o/lse in {E2E_GROUPS} key/value-head runs whose copies overlap"},
            "roofline": roofline,
            "cpu_baseline": cpu,
            "per_config": per_config,
            "decode": decode,
            "backward": backward,
            "bsbr": bsbr,
        }
        print(json.dumps(line), flush=True)
    sampler.stop()
    lay.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_leg(args, w):
    """One secondary leg alone (no headline, e2e or CPU legs), one JSON line."""
    import dataclasses
    import torch
    import block_sparse_long_bsa_b200 as bsa
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA GPU")
    bsa.load_library()
    dev = torch.cuda.current_device()
    stream = torch.cuda.current_stream()
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device=dev)
    if args.leg == "backward":
        if args.n is not None:
            w = dataclasses.replace(w, n=args.n)
        res = bench_backward(w, dev, stream, flush, bsa, torch, steps=args.steps, warmup=args.warmup)
    elif args.leg == "decode":
        if args.n is not None:
            w = dataclasses.replace(w, n=args.n)
        res = bench_decode(dev, stream, flush, bsa, torch, steps=args.steps, warmup=args.warmup, n=args.n)
    else:
        w = WORKLOADS["bsbr_block_diagonal"]
        res = bench_bsbr(w, dev, stream, flush, bsa, torch, steps=args.steps, warmup=args.warmup)
    print(json.dumps({"leg": args.leg, "workload": w.name, "n": w.n, "result": res}), flush=True)
    return 0


def bench_other(w, dev, stream, flush, bsa, torch, steps=10, warmup=3):
    lay = bsa.Layout.for_workload(w, dev)
    row_ptr, col_idx = lay.csr()
    pairs, flops, compulsory = workload_work(w, row_ptr, col_idx)
    gen = torch.Generator(device=dev)
    gen.manual_seed(1234)
    q = torch.randn((w.heads, w.n, w.d), device=dev, generator=gen).to(torch.bfloat16)
    k = torch.randn((w.kv_heads, w.n, w.d), device=dev, generator=gen).to(torch.bfloat16)
    v = torch.randn((w.kv_heads, w.n, w.d), device=dev, generator=gen).to(torch.bfloat16)
    o = torch.empty_like(q)
    lse = torch.empty((w.heads, w.n), dtype=torch.float32, device=dev)
    scale = 1.0 / math.sqrt(w.d)
    ms = []
    for s in range(warmup + steps):
        flush.fill_(float(s))
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        bsa.bsa_forward(q, k, v, lay.handle, w.B, w.n, w.heads, w.kv_heads, w.d, scale, o, lse, stream)
        b.record(stream)
        if s >= warmup:
            ms.append((a, b))
    torch.cuda.synchronize()
    bsa.bsa_get_status(lay.handle)
    t = sorted(a.elapsed_time(b) for a, b in ms)
    med = t[len(t) // 2]
    lay.close()
    del q, k, v, o, lse
    return {"ms_median": med, "tflops": flops / (med * 1e-3) / 1e12, "kept_pairs": pairs,
            "hbm_gbs_compulsory": compulsory / (med * 1e-3) / 1e9,
            "data": "torch.randn on device, seed 1234"}


def bench_backward(w, dev, stream, flush, bsa, torch, steps=10, warmup=3):
    """Gradients (dq, dk, dv) of the forward on a workload: one bsa_backward
    call per step (the D kernel, the dq kernel, the dk/dv kernel and two
    clears), timed with CUDA events on the launching stream.  Effective
    TFLOP/s counts 10 d flops per kept pair (the S, dP, dq, dk and dv
    products, 2 d each); the kernels compute S and dP twice, 14 d per pair."""
    lay = bsa.Layout.for_workload(w, dev)
    row_ptr, col_idx = lay.csr()
    pairs, flops_fwd, _ = workload_work(w, row_ptr, col_idx)
    flops = flops_fwd * 10 // 4
    gen = torch.Generator(device=dev)
    gen.manual_seed(4321)
    q = torch.randn((w.heads, w.n, w.d), device=dev, generator=gen).to(torch.bfloat16)
    k = torch.randn((w.kv_heads, w.n, w.d), device=dev, generator=gen).to(torch.bfloat16)
    v = torch.randn((w.kv_heads, w.n, w.d), device=dev, generator=gen).to(torch.bfloat16)
    do = torch.randn((w.heads, w.n, w.d), device=dev, generator=gen).to(torch.bfloat16)
    o = torch.empty_like(q)
    lse = torch.empty((w.heads, w.n), dtype=torch.float32, device=dev)
    dq = torch.empty(q.shape, dtype=torch.float32, device=dev)
    dk = torch.empty(k.shape, dtype=torch.float32, device=dev)
    dv = torch.empty(v.shape, dtype=torch.float32, device=dev)
    ws = torch.empty((w.heads, w.n), dtype=torch.float32, device=dev)
    scale = 1.0 / math.sqrt(w.d)
    bsa.bsa_forward(q, k, v, lay.handle, w.B, w.n, w.heads, w.kv_heads, w.d, scale, o, lse, stream)
    ev = []
    for st in range(warmup + steps):
        flush.fill_(float(st))
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        bsa.bsa_backward(q, k, v, o, lse, do, lay.handle, w.B, w.n, w.heads, w.kv_heads, w.d, scale,
                         dq, dk, dv, ws, stream)
        b.record(stream)
        if st >= warmup:
            ev.append((a, b))
    torch.cuda.synchronize()
    bsa.bsa_get_status(lay.handle)
    ts = sorted(a.elapsed_time(b) for a, b in ev)
    med = ts[len(ts) // 2]
    peak = float(load_peaks()[0].get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    lay.close()
    del q, k, v, do, o, lse, dq, dk, dv, ws
    tf = flops / (med * 1e-3) / 1e12
    return {"ms_median": med, "effective_tflops": tf, "frac_of_measured_peak": tf / peak,
            "algorithmic_flops": flops, "kept_pairs": pairs, "launches_per_call": 3,
            "data": "torch.randn on device, seed 4321; L2 flushed between steps"}


def bench_bsbr(w, dev, stream, flush, bsa, torch, steps=20, warmup=3):
    """BSBR attention on its workload: the within-chunk forward (bsa_forward on
    the block-diagonal layout) plus the between-chunk retrieval
    (bsa_bsbr_retrieval), and the retrieval alone.  The retrieval's
    algorithmic HBM bytes: k and v read, the chunk states and meta keys
    written and read once, q read, o read and written."""
    lay = bsa.Layout.for_workload(w, dev)
    gen = torch.Generator(device=dev)
    gen.manual_seed(777)
    q = torch.randn((w.heads, w.n, w.d), device=dev, generator=gen).to(torch.bfloat16)
    k = torch.randn((w.kv_heads, w.n, w.d), device=dev, generator=gen).to(torch.bfloat16)
    v = torch.randn((w.kv_heads, w.n, w.d), device=dev, generator=gen).to(torch.bfloat16)
    o = torch.empty_like(q)
    lse = torch.empty((w.heads, w.n), dtype=torch.float32, device=dev)
    need = bsa.bsa_bsbr_workspace_bytes(w.n, w.B, w.kv_heads, w.d)
    ws = torch.empty(((need + 15) // 16) * 4, dtype=torch.float32, device=dev)
    scale = 1.0 / math.sqrt(w.d)
    chunks = -(-w.n // w.B)
    res = {}
    for leg in ("forward_plus_retrieval", "retrieval_only"):
        ev = []
        for st in range(warmup + steps):
            flush.fill_(float(st))
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            if leg == "forward_plus_retrieval":
                bsa.bsa_forward(q, k, v, lay.handle, w.B, w.n, w.heads, w.kv_heads, w.d, scale, o, lse, stream)
            bsa.bsa_bsbr_retrieval(q, k, v, lay.handle, w.B, w.n, w.heads, w.kv_heads, w.d, scale, o, ws,
                                   ws.numel() * 4, stream)
            b.record(stream)
            if st >= warmup:
                ev.append((a, b))
        torch.cuda.synchronize()
        bsa.bsa_get_status(lay.handle)
        ts = sorted(a.elapsed_time(b) for a, b in ev)
        res[leg] = {"us_median": ts[len(ts) // 2] * 1e3}
    elem = w.n * w.d * 2
    bytes_ret = (2 * w.kv_heads * elem + 3 * w.heads * elem
                 + 2 * w.kv_heads * chunks * w.d * (w.d + 1) * 4)
    us = res["retrieval_only"]["us_median"]
    hbm = float(load_peaks()[0].get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    gbs = bytes_ret / (us * 1e-6) / 1e9
    res["retrieval_only"].update({"algorithmic_bytes": bytes_ret, "gbs": gbs, "frac_of_measured_hbm": gbs / hbm,
                                  "launches": 2})
    res["workload"] = (f"BSBR: batch {w.batch} x {w.q_heads} heads, n={w.n}, d={w.d}, chunks of B={w.B} "
                       f"({chunks} chunks)")
    res["data"] = "torch.randn on device, seed 777; L2 flushed between steps"
    lay.close()
    del q, k, v, o, lse, ws
    return res


def bench_decode(dev, stream, flush, bsa, torch, batches=(1, 32), steps=20, warmup=3, n=None):
    """Selected-page decode on the headline route: each sequence's new token at
    the last position of a 32K context, reading its block row's kept pages
    through a shuffled page table.  Reports time per step and the unique
    key/value bytes of the kept pages (what a step must read) per second."""
    import dataclasses
    w = WORKLOADS[HEADLINE]
    if n is not None:
        w = dataclasses.replace(w, n=n)
    lay = bsa.Layout.for_workload(w, dev)
    row_ptr, col_idx = lay.csr()
    H, hkv, B, d, n = w.q_heads, w.kv_heads_per_seq, w.B, w.d, w.n
    nb = -(-n // B)
    t = n - 1
    i = t // B
    kept = [int(j) for j in col_idx[row_ptr[i]:row_ptr[i + 1]]]
    toks = sum(min(B, t + 1 - j * B) for j in kept)
    hbm = float(load_peaks()[0].get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    out = {"workload": f"BF1 dyadic route, token at position {t} of a {n}-token context, "
                       f"{H}/{hkv} heads, d={d}, B={B} pages",
           "kept_blocks": len(kept), "l2": "256 MiB written between steps"}
    gen = torch.Generator(device=dev)
    gen.manual_seed(99)
    for batch in batches:
        pages = batch * nb
        kc = torch.randn((pages, hkv, B, d), device=dev, generator=gen).to(torch.bfloat16)
        vc = torch.randn((pages, hkv, B, d), device=dev, generator=gen).to(torch.bfloat16)
        table = torch.randperm(pages, device=dev, generator=gen).to(torch.int32).view(batch, nb).contiguous()
        q = torch.randn((batch * H, d), device=dev, generator=gen).to(torch.bfloat16)
        pos = torch.full((batch,), t, dtype=torch.int32, device=dev)
        o = torch.empty_like(q)
        lse = torch.empty((batch * H,), dtype=torch.float32, device=dev)
        ev = []
        for st in range(warmup + steps):
            flush.fill_(float(st))
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            bsa.bsa_decode(q, kc, vc, table, nb, pages, pos, lay.handle, batch, batch * H,
                           batch * hkv, d, 1.0 / math.sqrt(d), o, lse, stream)
            b.record(stream)
            if st >= warmup:
                ev.append((a, b))
        torch.cuda.synchronize()
        bsa.bsa_get_status(lay.handle)
        ts = sorted(a.elapsed_time(b) for a, b in ev)
        us = ts[len(ts) // 2] * 1e3
        kv_bytes = batch * hkv * toks * d * 2 * 2
        io_bytes = batch * H * d * 2 * 2 + batch * H * 4
        gbs = (kv_bytes + io_bytes) / (us * 1e-6) / 1e9
        out[f"batch_{batch}"] = {"us_per_step": us, "tokens_per_s": batch / (us * 1e-6),
                                 "bytes_per_step": kv_bytes + io_bytes, "gbs": gbs,
                                 "frac_of_measured_hbm": gbs / hbm}
        del kc, vc, table, q, pos, o, lse
    lay.close()
    return out


if __name__ == "__main__":
    sys.exit(main())
