#!/usr/bin/env python
"""Throughput of the fused attention forward on B200.

One step = the whole hot path over one batch: a non-causal and a causal
forward of the largest single-GPU workload (batch 1, 16 heads, sequence
32768, head dim 128, BF16, K drawn x3), inputs resident in HBM.  The metric
is attention-forward TFLOPS, counting 4*b*h*s_q*s_k*d FLOPs per forward,
halved for the causal one.  The same line carries a per-configuration block:
every workload, both masks, each launch timed alone with CUDA events after
an L2 flush.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload NAME] [--no-configs]

Prints one JSON line (rank 0).  Multi-GPU runs (torchrun) are replicas: each
rank runs its own batch (weak scaling), timed on the device, max over ranks.
"""
from __future__ import annotations

import argparse
import glob
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from scaled_dot_product_10_b200.workloads import WORKLOADS, sample_rows, workload_qkv  # noqa: E402

METRIC = "attn fwd TFLOPS (bf16, d=128, causal & non-causal) and % of B200 BF16 peak"
UNIT = "TFLOPS"
SPEC_PEAK_TFLOPS = 2250.0
FALLBACK_PEAKS = {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0}
MODES = (False, True)  # non-causal, causal


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="mha_b1_h16_s32768_k3", choices=sorted(WORKLOADS))
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the per-configuration timing block")
    ap.add_argument("--config-launches", type=int, default=20,
                    help="timed launches per (configuration, mask) in that block")
    ap.add_argument("--only", choices=["configs", "split", "bwd", "fp8"],
                    help="run only the per-configuration block or only the split-KV cases "
                         "(for profiling) and print them as one JSON line")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--reference-seconds", type=float, default=150.0,
                    help="--impl reference: total oracle time the run is sized for")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for f in sorted(glob.glob(os.path.join(ROOT, "scaled_dot_product_10_b200", "csrc", "*"))):
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


FWD_SOURCES = ("attn_fwd_kernel.cuh", "attn_common.cuh", "sm100_ptx.cuh", "attn_api.cu")


def fwd_kernel_hash() -> str:
    """Hash of the sources the forward kernel and its launch are built from."""
    h = hashlib.sha256()
    for name in FWD_SOURCES:
        with open(os.path.join(ROOT, "scaled_dot_product_10_b200", "csrc", name), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def committed_traffic(workload: str):
    """DRAM bytes per launch of the forward on this workload from the
    committed ncu capture (profiles/traffic.json), if it was taken on the
    current forward sources; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    entry = d.get("workloads", {}).get(workload)
    if not entry or entry.get("fwd_kernel_hash") != fwd_kernel_hash():
        return None
    return entry.get("dram_bytes_per_launch")


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML (read-only) while
    the timed region runs."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, index: int, period_s: float = 0.02):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._period = period_s
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            uuid = None
            try:
                uuid = torch.cuda.get_device_properties(index).uuid
            except Exception:
                pass
            self._h = None
            if uuid is not None:
                for i in range(pynvml.nvmlDeviceGetCount()):
                    h = pynvml.nvmlDeviceGetHandleByIndex(i)
                    u = pynvml.nvmlDeviceGetUUID(h)
                    u = u.decode() if isinstance(u, bytes) else u
                    if str(uuid) in u:
                        self._h = h
            if self._h is None:
                self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nv = None

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                get = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                    nv.nvmlDeviceGetCurrentClocksThrottleReasons
                r = get(self._h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self._period)

    def __enter__(self):
        if self._nv is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        if self._nv is not None:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """Max of a host float over all ranks (one small all-reduce, not on the
    data path).  Works on NCCL (CUDA tensor) and gloo (CPU tensor)."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(world: int, flops_per_step: float, steps: int, max_ms: float) -> float:
    """Whole-job throughput: every rank runs the same per-rank work (weak
    scaling), divided by the slowest rank's device time."""
    return world * flops_per_step * steps / (max_ms * 1e-3) / 1e12


def clocks_over_ranks(summary: dict, world: int) -> dict:
    """The clock record of the whole job from every rank's sampler summary
    (one small collective after the timed region, taken by every rank): the
    slowest rank's median SM clock, the reasons seen on any rank, the samples
    of all ranks and each rank's median."""
    if world == 1:
        return summary
    import torch.distributed as dist
    every = [None] * world
    dist.all_gather_object(every, summary)
    mhz = [s["sm_mhz"] for s in every]
    known = [m for m in mhz if m is not None]
    return {"sm_mhz": min(known) if known else None, "sm_max_mhz": every[0]["sm_max_mhz"],
            "reasons": sorted(set().union(*(s["reasons"] for s in every))),
            "samples": sum(s["samples"] for s in every), "per_rank_sm_mhz": mhz}


# ------------------------------------------------------------------ oracle arm
def _head_slices(w, q, k, v, i):
    """The i-th (batch, query head) of the workload, cycling through all of
    them: the slices of Q, K and V that head reads."""
    group = w.h_q // w.h_kv
    bi, hi = i % w.batch, (i // w.batch) % w.h_q
    gi = hi // group
    return (q[bi:bi + 1, :, hi:hi + 1].contiguous(), k[bi:bi + 1, :, gi:gi + 1].contiguous(),
            v[bi:bi + 1, :, gi:gi + 1].contiguous())


def _oracle_step(w, qs, ks, vs, n_rows, seed):
    """The FP64 oracle on n_rows seeded rows of one head, both masks.
    Returns (FLOPs in the metric's convention, seconds)."""
    import oracle
    d = 128
    rows = sample_rows(1, 1, w.seq, n_rows, seed=seed, include_edges=False)
    t0 = time.perf_counter()
    f = 0.0
    for causal in MODES:
        oracle.attn_fwd(qs, ks, vs, causal, w.scale, rows=rows)
        f += float(4 * d * ((rows.astype("int64") + 1).sum() if causal else w.seq * rows.size))
    return f, time.perf_counter() - t0


def oracle_sample_rate(w, target_s: float):
    """Time the FP64 oracle on a bounded sample of the workload: per step one
    (batch, query head) slice (so decoding inputs the sample never reads is
    not counted as oracle time) and a seeded row sample of it, both masks,
    steps repeated until about target_s seconds.  Returns (TFLOPS in the
    metric's convention, seconds, rows per step, steps, threads)."""
    import oracle
    q, k, v = workload_qkv(w)
    # Size the row sample so one step costs about target_s / 8.
    qs, ks, vs = _head_slices(w, q, k, v, 0)
    _, t1 = _oracle_step(w, qs, ks, vs, 8, w.seed + 1)
    n = max(1, min(w.seq, int(8 * (target_s / 8) / max(t1, 1e-6))))
    flops = secs = 0.0
    steps = 0
    while secs < target_s and steps < 64:
        qs, ks, vs = _head_slices(w, q, k, v, steps)
        f, t = _oracle_step(w, qs, ks, vs, n, w.seed + 2 + steps)
        flops += f
        secs += t
        steps += 1
    return flops / secs / 1e12, secs, n, steps, oracle.num_threads()


def run_reference(args, world, rank):
    if rank != 0:
        return 0
    w = WORKLOADS[args.workload]
    per_step = args.reference_seconds / max(1, args.steps + args.warmup)
    import oracle
    q, k, v = workload_qkv(w)
    times, flops_total = [], 0.0
    rows_n = 1
    for i in range(args.warmup + args.steps):
        # One (batch, query head) of the workload per step at its full
        # sequence length, on a seeded row sample sized in the warm-up.
        qs, ks, vs = _head_slices(w, q, k, v, i)
        f, dt = _oracle_step(w, qs, ks, vs, rows_n, w.seed + 100 + i)
        if i < args.warmup:
            # size the sample so one step costs about `per_step` seconds
            rows_n = max(1, min(w.seq, int(rows_n * per_step / max(dt, 1e-6))))
            continue
        times.append(dt)
        flops_total += f
    total_t = sum(times)
    value = flops_total / total_t / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total_t / len(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "h_q": w.h_q, "h_kv": w.h_kv,
                   "seq": w.seq, "head_dim": 128, "modes": ["noncausal", "causal"]},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.num_threads(),
                         "kind": "oracle",
                         "sample": f"{rows_n} seeded query rows of one (batch, head) per step "
                                   f"(cycling through the workload's heads), both masks"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ our arm
def run_ours(args, world, rank, local):
    from scaled_dot_product_10_b200 import attn

    w = WORKLOADS[args.workload]
    attn.load_library()
    q, k, v = workload_qkv(w)
    if rank:
        # replicas: each rank runs its own batch of the same shape
        g = torch.Generator().manual_seed(w.seed + rank)
        q = torch.randn(q.shape, generator=g).to(torch.bfloat16)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    od = torch.empty_like(qd)
    ld = torch.empty((w.batch, w.h_q, w.seq), dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()
    sh = stream.cuda_stream
    qp, kp, vp, op, lp = qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), od.data_ptr(), ld.data_ptr()

    def launch(causal):
        rc = attn.attn_fwd_raw(qp, kp, vp, op, lp, w.batch, w.h_q, w.h_kv, w.seq, w.seq, 128,
                               causal, w.scale, sh)
        if rc != attn.ATTN_OK:
            raise attn.AttnError(rc, "attn_fwd")

    for _ in range(args.warmup):
        for causal in MODES:
            launch(causal)
    torch.cuda.synchronize()

    K = args.steps
    ev = {m: [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(K)] for m in MODES}
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize()
    with sampler:
        t_start.record(stream)
        for i in range(K):
            for causal in MODES:
                a, b = ev[causal][i]
                a.record(stream)
                launch(causal)
                b.record(stream)
        t_end.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    rc = attn.attn_status()
    if rc != attn.ATTN_OK:
        raise attn.AttnError(rc, "kernel status after the timed region")

    total_ms = max_over_ranks(t_start.elapsed_time(t_end), world)
    launch_ms = {m: sum(a.elapsed_time(b) for a, b in ev[m]) / K for m in MODES}
    flops_step = sum(w.flops(m) for m in MODES)
    value = whole_job_tflops(world, flops_step, K, total_ms)

    peaks, peak_src = load_peaks()
    achieved = flops_step / (sum(launch_ms.values()) * 1e-3) / 1e12
    peak = float(peaks["bf16_tflops"])
    traffic = committed_traffic(w.name)
    roofline = {
        "bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
        "frac": achieved / peak,
        "traffic": (sum(traffic[m] for m in ("noncausal", "causal")) / 2 if traffic else None),
        "peak_source": f"{peak_src} bf16 burst (cuBLAS 8192^3)",
        "frac_of_sustained": achieved / float(peaks.get("bf16_tflops_sustained", peak)),
        "frac_of_spec_2250": achieved / SPEC_PEAK_TFLOPS,
        "kernel": "attn_fwd_sm100_kernel",
    }
    modes = {("causal" if m else "noncausal"): {
        "ms_per_launch": launch_ms[m], "tflops": w.flops(m) / (launch_ms[m] * 1e-3) / 1e12}
        for m in MODES}

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": total_ms / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": f"synthetic (seeded N(0,1) BF16; inputs {w.input_bytes() / 1e6:.0f} MB > 126 MB "
                "L2, no flush needed)",
        "config": {"workload": w.name, "batch": w.batch, "h_q": w.h_q, "h_kv": w.h_kv,
                   "seq": w.seq, "head_dim": 128, "modes": ["noncausal", "causal"],
                   "l2": "inputs larger than L2", "parallelism": f"replicas x{world}"},
        "modes": modes,
        "pct_of_spec_peak": 100.0 * value / world / SPEC_PEAK_TFLOPS,
        "roofline": roofline,
        "clocks": clocks_over_ranks(sampler.summary(), world),
        "gpu_launches": 2 * K,
        "kernel_hash": kernel_source_hash(),
        "fwd_kernel_hash": fwd_kernel_hash(),
    }

    if not args.no_e2e:
        line["e2e"] = run_e2e(args, w, q, k, v, world)
    if world == 1 and not args.no_configs:
        line["configs"] = run_configs(args, peaks, peak_src)
        line["configs"]["split_kv"] = run_split_cases(args, peaks)
        line["configs"]["backward"] = run_backward(args, peaks)
        line["configs"]["fp8"] = run_fp8(args, peaks)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tfl, secs, n, steps, cores = oracle_sample_rate(w, args.cpu_seconds)
        line["cpu_baseline"] = {
            "value": tfl, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{steps} (batch, head) slices of {w.name}, {n} seeded query rows each, "
                      f"both masks, {secs:.1f} s; FLOPs counted as 4*d*visible keys per row"}
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_configs(args, peaks, peak_src="measured"):
    """Every workload, both masks: each launch timed alone with CUDA events on
    the launching stream after a 256 MB L2 flush (so the small workloads are
    not measured from a warm L2).  Median over the timed launches."""
    from scaled_dot_product_10_b200 import attn
    peak = float(peaks["bf16_tflops"])
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    stream = torch.cuda.current_stream()
    sh = stream.cuda_stream
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    out = {}
    for name, w in WORKLOADS.items():
        q, k, v = (t.cuda() for t in workload_qkv(w))
        o = torch.empty_like(q)
        lse = torch.empty((w.batch, w.h_q, w.seq), dtype=torch.float32, device="cuda")
        ptrs = (q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr())
        entry = {}
        for causal in MODES:
            def launch():
                rc = attn.attn_fwd_raw(*ptrs, w.batch, w.h_q, w.h_kv, w.seq, w.seq, 128, causal,
                                       w.scale, sh)
                if rc != attn.ATTN_OK:
                    raise attn.AttnError(rc, "attn_fwd")
            for _ in range(3):
                launch()
            times = []
            for _ in range(args.config_launches):
                flush.zero_()
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                a.record(stream)
                launch()
                b.record(stream)
                times.append((a, b))
            torch.cuda.synchronize()
            elapsed = [a.elapsed_time(b) for a, b in times]
            ms = statistics.median(elapsed)
            tf = w.flops(causal) / (ms * 1e-3) / 1e12
            gbs = w.algorithmic_bytes() / (ms * 1e-3) / 1e9
            entry["causal" if causal else "noncausal"] = {
                "ms_per_launch": ms, "ms_min": min(elapsed), "tflops": tf, "frac": tf / peak,
                "frac_of_spec_2250": tf / SPEC_PEAK_TFLOPS, "alg_gbs": gbs,
                "hbm_frac": gbs / hbm}
        rc = attn.attn_status()
        if rc != attn.ATTN_OK:
            raise attn.AttnError(rc, f"kernel status after {name}")
        out[name] = entry
        del q, k, v, o, lse
    del flush
    torch.cuda.empty_cache()
    return {"timing": f"median (and min) of {args.config_launches} launches per mask, each "
                      "after a 256 MB L2 flush; CUDA events on the launching stream",
            "frac_of": f"{peak_src} bf16 burst peak", "workloads": out}


# Few query rows over long key sequences: where the pairs of one launch leave
# SMs idle and the split-KV forward pays off.
# (name, batch, h_q, h_kv, s_q, s_k, seed); non-causal, N(0,1) BF16.
SPLIT_CASES = [
    ("few_q_b1_h16_q256_k32768", 1, 16, 16, 256, 32768, 1101),
    ("few_q_b1_h16_q512_k32768", 1, 16, 16, 512, 32768, 1102),
    ("few_q_b2_h16_q128_k16384", 2, 16, 16, 128, 16384, 1103),
    ("few_q_gqa_b1_h32_kv4_q256_k65536", 1, 32, 4, 256, 65536, 1104),
]


def run_split_cases(args, peaks):
    """attn_fwd against attn_fwd_split (the library's range count; forward
    plus merge) on the few-query cases, each launch timed alone after an L2
    flush, median of the timed launches."""
    from scaled_dot_product_10_b200 import attn
    from scaled_dot_product_10_b200.workloads import make_qkv
    peak = float(peaks["bf16_tflops"])
    stream = torch.cuda.current_stream()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")

    def timed(f):
        for _ in range(3):
            f()
        ev = []
        for _ in range(args.config_launches):
            flush.zero_()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            f()
            b.record(stream)
            ev.append((a, b))
        torch.cuda.synchronize()
        return statistics.median(a.elapsed_time(b) for a, b in ev)

    out = {}
    for name, b, hq, hkv, sq, sk, seed in SPLIT_CASES:
        q, k, v = (t.cuda() for t in make_qkv(b, hq, hkv, sq, sk, seed=seed))
        scale = 1.0 / math.sqrt(128)
        o = torch.empty_like(q)
        lse = torch.empty((b, hq, sq), dtype=torch.float32, device="cuda")
        n = attn.num_splits(b, hq, hkv, sq, sk)
        ws = torch.empty(attn.split_workspace_bytes(b, hq, sq, n), dtype=torch.uint8,
                         device="cuda")
        t_plain = timed(lambda: attn.attn_fwd(q, k, v, scale=scale, o=o, lse=lse))
        t_split = timed(lambda: attn.attn_fwd_split(q, k, v, scale=scale, n_splits=n, o=o,
                                                    lse=lse, workspace=ws))
        rc = attn.attn_status()
        if rc != attn.ATTN_OK:
            raise attn.AttnError(rc, f"kernel status after {name}")
        flops = 4.0 * b * hq * sq * sk * 128
        byts = 2 * (b * sq * hq * 128 * 2) + 2 * (b * sk * hkv * 128 * 2) + b * hq * sq * 4
        out[name] = {"n_splits": n, "ms_attn_fwd": t_plain, "ms_split": t_split,
                     "tflops_attn_fwd": flops / (t_plain * 1e-3) / 1e12,
                     "tflops_split": flops / (t_split * 1e-3) / 1e12,
                     "frac_split": flops / (t_split * 1e-3) / 1e12 / peak,
                     "speedup": t_plain / t_split,
                     "alg_gbs_split": byts / (t_split * 1e-3) / 1e9}
    return out


BWD_WORKLOADS = ["mha_b8_h16_s4096", "mha_b4_h16_s8192", "gqa_b8_h16_kv2_s2048"]


def run_backward(args, peaks):
    """attn_bwd (prep + dK/dV + dQ launches) on a few workloads, both masks,
    each call timed alone after an L2 flush; TFLOPS count 2.5x the forward's
    FLOPs (the five GEMM-sized products of the standard backward, although
    this one recomputes Q K^T and dO V^T for dQ)."""
    from scaled_dot_product_10_b200 import attn
    peak = float(peaks["bf16_tflops"])
    stream = torch.cuda.current_stream()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    out = {}
    for name in BWD_WORKLOADS:
        w = WORKLOADS[name]
        q, k, v = (t.cuda() for t in workload_qkv(w))
        dout = torch.randn(q.shape, generator=torch.Generator("cuda").manual_seed(w.seed + 50),
                           device="cuda").to(torch.bfloat16)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        ws = torch.empty(attn.bwd_workspace_bytes(w.batch, w.h_q, w.seq), dtype=torch.uint8,
                         device="cuda")
        entry = {}
        for causal in MODES:
            o, lse = attn.attn_fwd(q, k, v, causal=causal, scale=w.scale)

            def call():
                attn.attn_bwd(q, k, v, o, lse, dout, causal=causal, scale=w.scale, dq=dq, dk=dk,
                              dv=dv, workspace=ws)
            for _ in range(3):
                call()
            ev = []
            for _ in range(max(5, args.config_launches // 2)):
                flush.zero_()
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                a.record(stream)
                call()
                b.record(stream)
                ev.append((a, b))
            torch.cuda.synchronize()
            ms = statistics.median(a.elapsed_time(b) for a, b in ev)
            tf = 2.5 * w.flops(causal) / (ms * 1e-3) / 1e12
            entry["causal" if causal else "noncausal"] = {"ms_per_call": ms, "tflops": tf,
                                                          "frac": tf / peak}
        rc = attn.attn_status()
        if rc != attn.ATTN_OK:
            raise attn.AttnError(rc, f"kernel status after backward {name}")
        out[name] = entry
        del q, k, v, dout, dq, dk, dv, ws
    del flush
    torch.cuda.empty_cache()
    return out


FP8_WORKLOADS = ["mha_b8_h16_s4096", "mha_b1_h16_s32768_k3", "gqa_b8_h16_kv2_s2048"]


def run_fp8(args, peaks):
    """attn_fwd_fp8 on E4M3 versions of a few workloads (per-tensor scales),
    both masks, each launch timed alone after an L2 flush.  The fraction is
    of the FP8 dense peak, taken as the measured BF16 peak x 2 (the nominal
    FP8 / BF16 tensor-core ratio)."""
    from scaled_dot_product_10_b200 import attn
    from scaled_dot_product_10_b200.workloads import make_qkv_fp8
    peak8 = 2.0 * float(peaks["bf16_tflops"])
    stream = torch.cuda.current_stream()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    out = {}
    for name in FP8_WORKLOADS:
        w = WORKLOADS[name]
        q8, k8, v8, qs, ks, vs = make_qkv_fp8(w.batch, w.h_q, w.h_kv, w.seq, w.seq, seed=w.seed,
                                              k_scale=w.k_scale)
        q8, k8, v8 = q8.cuda(), k8.cuda(), v8.cuda()
        o = torch.empty(q8.shape, dtype=torch.bfloat16, device="cuda")
        lse = torch.empty((w.batch, w.h_q, w.seq), dtype=torch.float32, device="cuda")
        entry = {}
        for causal in MODES:
            def call():
                attn.attn_fwd_fp8(q8, k8, v8, qs, ks, vs, causal=causal, scale=w.scale, o=o,
                                  lse=lse)
            for _ in range(3):
                call()
            ev = []
            for _ in range(args.config_launches):
                flush.zero_()
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                a.record(stream)
                call()
                b.record(stream)
                ev.append((a, b))
            torch.cuda.synchronize()
            ms = statistics.median(a.elapsed_time(b) for a, b in ev)
            tf = w.flops(causal) / (ms * 1e-3) / 1e12
            entry["causal" if causal else "noncausal"] = {"ms_per_launch": ms, "tflops": tf,
                                                          "frac_of_fp8_peak": tf / peak8}
        rc = attn.attn_status()
        if rc != attn.ATTN_OK:
            raise attn.AttnError(rc, f"kernel status after FP8 {name}")
        out[name] = entry
        del q8, k8, v8, o, lse
    del flush
    torch.cuda.empty_cache()
    return {"fp8_peak_tflops": peak8, "workloads": out}


def run_e2e(args, w, q, k, v, world):
    """Same metric through the host-buffer C entry point: pinned host inputs,
    H2D copies, the forward, and D2H of O and LSE inside the timed region."""
    from scaled_dot_product_10_b200 import attn
    qh, kh, vh = q.pin_memory(), k.pin_memory(), v.pin_memory()
    oh = torch.empty_like(qh).pin_memory()
    lh = torch.empty((w.batch, w.h_q, w.seq), dtype=torch.float32).pin_memory()
    ws = torch.empty(attn.host_workspace_bytes(w.batch, w.h_q, w.h_kv, w.seq, w.seq),
                     dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    def step():
        for causal in MODES:
            attn.attn_fwd_host(qh, kh, vh, oh, lh, ws, causal=causal, scale=w.scale,
                               stream=stream)

    for _ in range(max(1, args.warmup)):  # the same warm-up as the device-timed region
        step()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    barrier(world)
    a.record(stream)
    for _ in range(args.e2e_steps):
        step()
    b.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(a.elapsed_time(b), world)
    flops_step = sum(w.flops(m) for m in MODES)
    n_in = sum(t.numel() * t.element_size() for t in (qh, kh, vh))
    n_out = oh.numel() * oh.element_size() + lh.numel() * lh.element_size()
    return {"value": whole_job_tflops(world, flops_step, args.e2e_steps, ms), "unit": UNIT,
            "h2d_bytes_per_step": len(MODES) * n_in, "d2h_bytes_per_step": len(MODES) * n_out,
            "steps": args.e2e_steps, "ms_per_step": ms / args.e2e_steps}


def main():
    args = parse_args()
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        return run_reference(args, world, rank)
    world, rank, local = dist_setup(args)
    if args.gpus != world and rank == 0:
        # The line reports the ranks that actually ran (n_gpus = WORLD_SIZE).
        print(f"bench.py: --gpus {args.gpus} but {world} rank(s) running; launch N > 1 with "
              "torchrun --nproc-per-node N", file=sys.stderr, flush=True)
    if args.only:
        from scaled_dot_product_10_b200 import attn
        attn.load_library()
        peaks, peak_src = load_peaks()
        if args.only == "configs":
            part = run_configs(args, peaks, peak_src)
        else:
            part = {"split": run_split_cases, "bwd": run_backward,
                    "fp8": run_fp8}[args.only](args, peaks)
        print(json.dumps({"only": args.only, args.only: part}), flush=True)
        return 0
    try:
        run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
