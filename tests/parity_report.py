"""Per-config report: kernel time, TFLOPS and parity against the oracle.

Test infrastructure (needs a GPU; not collected by pytest).  For every
workload config and both masks it times the CUDA path with CUDA events on
the launching stream (3 warm-up launches, then 20 timed ones: median and
minimum), and compares O and LSE with the FP64 oracle on the same rows the
parity tests use (all rows of the tiny config; 256 sampled rows per head on
the 2K/4K configs; 512 on the 8K-32K ones), timing the oracle on those rows.

    python tests/parity_report.py [--split-only] [out.jsonl]

prints one markdown table row per (config, mask) and, if a path is given,
writes the same figures as JSON lines.  A second table times the split-KV
forward (attn_fwd_split with the library's range count, forward + merge)
against attn_fwd on few-query, long-key shapes that leave most SMs idle
unsplit, with parity of the split result on 64 sampled rows per head.
"""
from __future__ import annotations

import json
import os
import sys
import time

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
sys.path.insert(0, ROOT)
sys.path.insert(0, HERE)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import oracle  # noqa: E402
from parity import gather_rows, metrics  # noqa: E402
from scaled_dot_product_10_b200 import attn  # noqa: E402
from scaled_dot_product_10_b200.workloads import (  # noqa: E402
    WORKLOADS, make_qkv, sample_rows, workload_qkv)

SPEC_TFLOPS = 2250.0
# (name, batch, h_q, h_kv, s_q, s_k, seed): non-causal, N(0,1) BF16 inputs.
SPLIT_CASES = [
    ("few_q_b1_h16_q256_k32768", 1, 16, 16, 256, 32768, 1101),
    ("few_q_b1_h16_q512_k32768", 1, 16, 16, 512, 32768, 1102),
    ("few_q_b2_h16_q128_k16384", 2, 16, 16, 128, 16384, 1103),
    ("few_q_gqa_b1_h32_kv4_q256_k65536", 1, 32, 4, 256, 65536, 1104),
]


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        for key in ("bf16_tflops", "bf16_tflops_burst"):
            if key in d:
                return float(d[key]), "measured"
    return 1590.0, "fallback"


def time_launches(f, warmup=3, n=20):
    s = torch.cuda.current_stream()
    for _ in range(warmup):
        f()
    torch.cuda.synchronize()
    ts = []
    for _ in range(n):
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(s)
        f()
        b.record(s)
        b.synchronize()
        ts.append(a.elapsed_time(b))
    return float(np.median(ts)), float(np.min(ts))


def main():
    argv = [a for a in sys.argv[1:] if a != "--split-only"]
    split_only = len(argv) != len(sys.argv) - 1
    out = open(argv[0], "w") if argv else None
    peak, peak_src = measured_peak()
    threads = oracle.num_threads()
    if not split_only:
        print(f"| config | mode | TFLOPS (median) | % of 2250 | % of {peak_src} {peak} | "
              "ms median / min | alg. GB/s | max abs dO | rel-L2 O | max abs dLSE | "
              f"oracle s (rows) / {threads} threads |")
        print("|---|---|---|---|---|---|---|---|---|---|---|")
    for name, w in ([] if split_only else WORKLOADS.items()):
        q, k, v = workload_qkv(w)
        qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
        o = torch.empty_like(qd)
        lse = torch.empty((w.batch, w.h_q, w.seq), dtype=torch.float32, device="cuda")
        if w.batch * w.h_q * w.seq <= 4096:
            rows = None
        else:
            rows = sample_rows(w.batch, w.h_q, w.seq, 512 if w.sampled else 256,
                               seed=w.seed + 7919)
        for causal in (False, True):
            f = lambda: attn.attn_fwd(qd, kd, vd, causal=causal, scale=w.scale, o=o, lse=lse)
            med, mn = time_launches(f)
            rc = attn.attn_status()
            assert rc == attn.ATTN_OK, attn.attn_strerror(rc)
            t0 = time.perf_counter()
            o_ref, l_ref, _ = oracle.attn_fwd(q, k, v, causal, w.scale, rows=rows)
            t_oracle = time.perf_counter() - t0
            oo, ll = gather_rows(o, lse, rows)
            m = metrics(oo, ll, o_ref, l_ref)
            tflops = w.flops(causal) / (med * 1e-3) / 1e12
            gbs = w.algorithmic_bytes() / (med * 1e-3) / 1e9
            n_rows = w.batch * w.h_q * (w.seq if rows is None else rows.shape[-1])
            rec = {"config": name, "causal": causal, "tflops": tflops, "ms_median": med,
                   "ms_min": mn, "alg_gbs": gbs, "frac_spec": tflops / SPEC_TFLOPS,
                   "frac_measured": tflops / peak, **m, "oracle_s": t_oracle,
                   "oracle_rows": n_rows, "oracle_threads": threads}
            if out:
                out.write(json.dumps(rec) + "\n")
            print(f"| {name} | {'causal' if causal else 'non-causal'} | {tflops:.1f} | "
                  f"{100 * tflops / SPEC_TFLOPS:.1f} % | {100 * tflops / peak:.1f} % | "
                  f"{med:.3f} / {mn:.3f} | {gbs:.0f} | {m['max_abs_o']:.2e} | "
                  f"{m['rel_l2_o']:.2e} | {m['max_abs_lse']:.2e} | "
                  f"{t_oracle:.1f} ({n_rows} rows) |", flush=True)
    if not split_only:
        print()
    print("| split case | n ranges | attn_fwd TFLOPS (ms) | attn_fwd_split TFLOPS (ms) | speed-up | "
          "alg. GB/s split | max abs dO | rel-L2 O | max abs dLSE |")
    print("|---|---|---|---|---|---|---|---|---|")
    for name, b, hq, hkv, sq, sk, seed in SPLIT_CASES:
        q, k, v = make_qkv(b, hq, hkv, sq, sk, seed=seed)
        qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
        scale = 1.0 / np.sqrt(128.0)
        o = torch.empty_like(qd)
        lse = torch.empty((b, hq, sq), dtype=torch.float32, device="cuda")
        n = attn.num_splits(b, hq, hkv, sq, sk)
        ws = torch.empty(attn.split_workspace_bytes(b, hq, sq, n), dtype=torch.uint8, device="cuda")
        t_plain, _ = time_launches(lambda: attn.attn_fwd(qd, kd, vd, scale=scale, o=o, lse=lse))
        t_split, _ = time_launches(lambda: attn.attn_fwd_split(qd, kd, vd, scale=scale, n_splits=n,
                                                               o=o, lse=lse, workspace=ws))
        rc = attn.attn_status()
        assert rc == attn.ATTN_OK, attn.attn_strerror(rc)
        rows = sample_rows(b, hq, sq, 64, seed=seed + 7919)
        o_ref, l_ref, _ = oracle.attn_fwd(q, k, v, False, scale, rows=rows)
        oo, ll = gather_rows(o, lse, rows)
        m = metrics(oo, ll, o_ref, l_ref)
        flops = 4.0 * b * hq * sq * sk * 128
        byts = 2 * (b * sq * hq * 128 * 2) + 2 * (b * sk * hkv * 128 * 2) + b * hq * sq * 4
        tf_p, tf_s = flops / (t_plain * 1e-3) / 1e12, flops / (t_split * 1e-3) / 1e12
        rec = {"split_case": name, "n_splits": n, "tflops_attn_fwd": tf_p, "ms_attn_fwd": t_plain,
               "tflops_split": tf_s, "ms_split": t_split, "alg_gbs_split": byts / (t_split * 1e-3) / 1e9,
               **m}
        if out:
            out.write(json.dumps(rec) + "\n")
        print(f"| {name} | {n} | {tf_p:.1f} ({t_plain:.3f}) | {tf_s:.1f} ({t_split:.3f}) | "
              f"{t_plain / t_split:.2f}x | {rec['alg_gbs_split']:.0f} | {m['max_abs_o']:.2e} | "
              f"{m['rel_l2_o']:.2e} | {m['max_abs_lse']:.2e} |", flush=True)
    if out:
        out.close()


if __name__ == "__main__":
    main()
