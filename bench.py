#!/usr/bin/env python3
"""Benchmark of one GQA decode step (KV append + split-KV decode with its in-kernel merge) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

One step = gqa_kv_append then gqa_decode on one batch of the workload, through the C ABI.
`value` is the whole-job KV-read throughput: ideal KV bytes (2 * sum(n_b) * H_kv * d * 2 B) of
all steps on all ranks divided by the device-timed duration (CUDA events, max over ranks).
The KV cache is resident state; each rank runs an independent replica (the decode of one
sequence needs nothing from any other), so scaling is weak and there is no collective on the
data path.  Two copies of the cache (2 x 268 MB for the default workload, more than the 126 MB
L2) alternate between steps, so each step reads its cache from HBM.

--impl reference times the CPU oracle (test infrastructure) on the host cores on a bounded
sample of the same workload, as the reference arm.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

METRIC = "GQA decode: achieved KV-read HBM GB/s (% of B200 peak); µs per decode step"
DEFAULT_WORKLOAD = "llama2_70b_layer"
PROFILE_DIR = os.path.join(ROOT, "profiles")
SPLIT_KERNEL_SOURCES = ["decode_tc.cu", "device.cuh", "schedule.cuh"]
SPLIT8_KERNEL_SOURCES = ("decode_tc8.cu", "device.cuh", "schedule.cuh")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="budget of the CPU-oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--profile-run", action="store_true",
                    help="only run warmup + steps plain API steps (one cache copy, no timing "
                         "report): the command ncu captures")
    return ap.parse_args()


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def max_over_ranks(x: float, pg, device) -> float:
    """Max of a per-rank number over all ranks (the whole job is as slow as its slowest rank)."""
    if pg is None:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def split_kernel_hash(sources=None) -> str:
    h = hashlib.sha256()
    for name in sources or SPLIT_KERNEL_SOURCES:
        with open(os.path.join(ROOT, "grouped_query_attention_decode_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str, fp8: bool = False):
    """dram bytes per launch of the split kernel from a committed ncu summary, when it was taken
    on the current kernel source; else None."""
    stem = "split_tc8" if fp8 else "split_tc"
    p = os.path.join(PROFILE_DIR, f"{stem}_{workload}.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    sources = SPLIT8_KERNEL_SOURCES if fp8 else SPLIT_KERNEL_SOURCES
    if d.get("kernel_source_hash") != split_kernel_hash(sources):
        return None
    return d.get("dram_bytes_per_launch_full_size")


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 200 ms in the background."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, enabled: bool = True):
        self.proc = None
        self.path = None
        self.gpu = gpu_index
        if not enabled:
            return
        try:
            # the raw samples (GQA_CLOCKS_DIR, else the temp directory); the JSON line carries
            # their summary
            out_dir = os.environ.get("GQA_CLOCKS_DIR") or tempfile.gettempdir()
            os.makedirs(out_dir, exist_ok=True)
            self.path = os.path.join(out_dir, f"clocks_bench_rank{gpu_index}.csv")
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(gpu_index), f"--query-gpu=timestamp,{self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"], stdout=self.fh,
                stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                c = [x.strip() for x in line.split(",")]
                if len(c) >= 10:
                    rows.append(c)
        if not rows:
            return None
        sm = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        smax = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[6 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(rows)}


def bench_ours(args, rank, world, local):
    import numpy as np

    import grouped_query_attention_decode_b200 as gqa
    from grouped_query_attention_decode_b200 import inputs

    assert torch.cuda.is_available(), "the ours arm needs a CUDA device"
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
        pg = dist
    w = inputs.WORKLOADS[args.workload]
    x = inputs.make_inputs(w)
    lengths = x["lengths"].tolist()
    ideal = inputs.ideal_kv_bytes(w, lengths)
    K, W = args.steps, args.warmup
    assert W >= 3
    q = x["q"].to(dev)
    kn, vn = x["k_new"].to(dev), x["v_new"].to(dev)
    block_table = None
    if w.page_size > 0:
        paged = inputs.make_paged(x, w.page_size)
        block_table = paged["block_table"].to(dev)
        caches = [(paged["k_pool"].to(dev), paged["v_pool"].to(dev))]
    else:
        caches = [(x["k_cache"].to(dev), x["v_cache"].to(dev))]
    caches.append((caches[0][0].clone(), caches[0][1].clone()))
    lens0 = x["seq_lens_pre"].to(dev)
    out = torch.empty(tuple(q.shape), dtype=torch.float32, device=dev)
    if w.queries > 1:
        nws = gqa.load_library().gqa_decode_multi_workspace_size(w.B, w.queries, w.H_q, w.H_kv, w.d,
                                                                 gqa.DTYPE_BF16 if w.dtype == torch.bfloat16 else gqa.DTYPE_F32)
        ws = torch.zeros(nws, dtype=torch.uint8, device=dev)
    elif w.fp8:
        ws = gqa.alloc_workspace_fp8(w.B, w.H_q, w.H_kv, w.d, device=dev)
    else:
        ws = gqa.alloc_workspace(w.B, w.H_q, w.H_kv, w.d, w.dtype, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    ks = x["k_scale"].to(dev) if w.fp8 else None
    vs = x["v_scale"].to(dev) if w.fp8 else None

    def do_append(i, lens_row, kk=kn, vv=vn):
        kc, vc = caches[i & 1]
        if w.fp8:
            if block_table is not None:
                gqa.kv_append_paged_fp8(kk, vv, kc, vc, ks, vs, block_table, lens_row, status=status)
            else:
                gqa.kv_append_fp8(kk, vv, kc, vc, ks, vs, lens_row, status=status)
        elif block_table is not None:
            gqa.kv_append_paged(kk, vv, kc, vc, block_table, lens_row, status=status)
        elif w.queries > 1:
            gqa.kv_append_multi(kk, vv, kc, vc, lens_row, status=status)
        else:
            gqa.kv_append(kk, vv, kc, vc, lens_row, status=status)

    def do_decode(i, lens_row, qq=q):
        kc, vc = caches[i & 1]
        if w.fp8:
            if block_table is not None:
                gqa.decode_paged_fp8(qq, kc, vc, ks, vs, block_table, lens_row, x["scale"], out=out,
                                     workspace=ws, status=status)
            else:
                gqa.decode_fp8(qq, kc, vc, ks, vs, lens_row, x["scale"], window=w.window, out=out,
                               workspace=ws, status=status)
        elif block_table is not None:
            gqa.decode_paged(qq, kc, vc, block_table, lens_row, x["scale"], out=out, workspace=ws,
                             status=status)
        elif w.queries > 1:
            gqa.decode_multi(qq, kc, vc, lens_row, x["scale"], out=out, workspace=ws, status=status)
        elif w.window > 0:
            gqa.decode_window(qq, kc, vc, lens_row, w.window, x["scale"], out=out, workspace=ws,
                              status=status)
        else:
            gqa.decode(qq, kc, vc, lens_row, x["scale"], out=out, workspace=ws, status=status)

    def step(i, lens_row, qq=q, kk=kn, vv=vn):
        do_append(i, lens_row, kk, vv)
        do_decode(i, lens_row, qq)

    # correctness guard before timing
    lens_chk = lens0.clone()
    step(0, lens_chk)
    torch.cuda.synchronize()
    assert int(status.item()) == 0, f"device status {int(status.item())}"

    # Main timing: steps captured in a CUDA graph (launch overhead off the host); every step
    # appends into its own pre-set length row, and one copy at the top of the graph re-arms
    # the rows for the next replay.
    ng = max(g for g in range(1, 65) if K % g == 0)
    lens_rows = lens0.repeat(ng, 1).contiguous()
    lens_init = lens_rows.clone()
    graph = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(cap):
        with torch.cuda.graph(graph, stream=cap):
            lens_rows.copy_(lens_init)
            for i in range(ng):
                step(i, lens_rows[i])
    torch.cuda.current_stream().wait_stream(cap)
    stream = torch.cuda.current_stream()
    for _ in range(max(1, -(-W // ng))):
        graph.replay()
    torch.cuda.synchronize()
    if pg is not None:
        pg.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(local, enabled=not args.no_clocks)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(K // ng):
        graph.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    if pg is not None:
        pg.barrier()
    t_ms = e0.elapsed_time(e1)
    assert int(status.item()) == 0, f"device status {int(status.item())}"
    del graph

    # Per-kernel timing: the split-KV kernel alone (the decode is one kernel), kp launches back
    # to back on the two cache copies with CUDA events on the launching stream around the
    # batch.  The launches are queued behind a GPU-side sleep on a side stream, so the GPU
    # never waits for the host; consecutive launches overlap only as programmatic dependent
    # launch allows (a prologue with the previous kernel's last CTAs).
    kp = min(K, 500)
    lens_dec = x["lengths"].to(dev)
    for i in range(W):
        do_decode(i, lens_dec)
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    with torch.cuda.stream(side):
        torch.cuda._sleep(100_000_000)
    gate = torch.cuda.Event()
    gate.record(side)
    stream.wait_event(gate)
    ka = torch.cuda.Event(enable_timing=True)
    kb = torch.cuda.Event(enable_timing=True)
    ka.record(stream)
    for i in range(kp):
        do_decode(i, lens_dec)
    kb.record(stream)
    torch.cuda.synchronize()
    split_ms = [ka.elapsed_time(kb) / kp]
    assert int(status.item()) == 0, f"device status {int(status.item())}"

    ms_step = max_over_ranks(t_ms / K, pg, dev)
    value = ideal * world / (ms_step * 1e-3) / 1e9

    # End to end through the public API: every step copies its inputs (q, k_new, v_new) in
    # from pinned host memory and its result out to pinned host memory.
    hq = x["q"].pin_memory()
    hkn, hvn = x["k_new"].pin_memory(), x["v_new"].pin_memory()
    hout = torch.empty(tuple(q.shape), dtype=torch.float32).pin_memory()
    dq, dkn, dvn = torch.empty_like(q), torch.empty_like(kn), torch.empty_like(vn)
    h2d = hq.numel() * hq.element_size() + 2 * hkn.numel() * hkn.element_size()
    d2h = hout.numel() * 4

    def e2e_step(i, lens_row):
        dq.copy_(hq, non_blocking=True)
        dkn.copy_(hkn, non_blocking=True)
        dvn.copy_(hvn, non_blocking=True)
        step(i, lens_row, dq, dkn, dvn)
        hout.copy_(out, non_blocking=True)

    ke = min(K, 1000)
    lens_big = lens0.repeat(ke + W, 1).contiguous()
    for i in range(W):
        e2e_step(i, lens_big[ke + i])
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for i in range(ke):
        e2e_step(i, lens_big[i])
    b.record(stream)
    torch.cuda.synchronize()
    e2e_step_ms = max_over_ranks(a.elapsed_time(b) / ke, pg, dev)
    assert np.isfinite(hout.numpy()).all()
    assert int(status.item()) == 0, f"device status {int(status.item())}"
    Ke = ke

    split_avg = statistics.mean(split_ms)
    achieved = ideal / (split_avg * 1e-3) / 1e9
    peak, peak_kind = measured_peaks()
    result = None
    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            cpu = cpu_baseline(w, x, args.cpu_seconds)
        result = {
            "metric": METRIC,
            "value": round(value, 2),
            "unit": "GB/s",
            "n_gpus": world,
            "steps": K,
            "warmup": W,
            "ms_per_step": round(ms_step, 6),
            "us_per_step": round(ms_step * 1e3, 3),
            "tokens_per_s": round(w.B * w.queries * world / (ms_step * 1e-3), 1),
            "pct_of_measured_hbm": round(100 * value / world / peak, 2),
            "pct_of_8tbs_spec": round(100 * value / world / 8000.0, 2),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "e4m3" if w.fp8 else ("bf16" if w.dtype == torch.bfloat16 else "f32"),
            "data": "synthetic",
            "config": {
                "workload": w.name, "B": w.B, "H_q": w.H_q, "H_kv": w.H_kv, "d": w.d,
                "L_max": w.L_max, "seq_len": lengths[0] if w.length else "ragged",
                "window": w.window or None,
                "page_size": w.page_size or None,
                "query_tokens": w.queries,
                "sum_seq_lens": int(sum(lengths)),
                "kv_dtype": "e4m3 (per-head scales)" if w.fp8 else str(w.dtype).replace("torch.", ""),
                "accumulate": "f32", "ideal_kv_bytes_per_step": ideal,
                "parallelism": f"replicas x{world}",
                "l2": "inputs larger than L2: two cache copies alternate between steps "
                      f"({2 * caches[0][0].numel() * 2 * w.elem_bytes / 1e6:.0f} MB)",
            },
            "gpu_launches": 2 * K,
            "roofline": {
                "bound": "hbm", "kernel": "split_tc8_kernel" if w.fp8 else "split_tc_kernel",
                "achieved": round(achieved, 1),
                "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                "frac": round(achieved / peak, 4),
                "traffic": profiled_traffic(w.name, w.fp8),
                "algorithmic_bytes_per_launch": ideal,
                "avg_launch_us": round(split_avg * 1e3, 3),
                "launches_timed": kp,
            },
            "e2e": {
                "value": round(ideal * world / (e2e_step_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
                "ms_per_step": round(e2e_step_ms, 6),
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": Ke,
            },
            "clocks": clk,
            "cpu_baseline": cpu,
        }
    if pg is not None:
        pg.barrier()
        pg.destroy_process_group()
    return result


def cpu_baseline(w, x, budget_s, steps=None):
    """The oracle, as it stands, on whole sequences of the workload until the time budget is
    used (at least one sequence).  Returns the baseline object in the bench's unit (GB/s)."""
    import oracle
    from grouped_query_attention_decode_b200 import inputs

    o = oracle.get()
    B = w.B
    t0 = time.perf_counter()
    nbytes = 0
    done = []
    b = 0
    while True:
        xb = {k: (v[b:b + 1] if isinstance(v, torch.Tensor) and v.dim() > 0 and v.shape[0] == B else v)
              for k, v in x.items()}
        q = xb["q"].double().numpy()
        lens = xb["seq_lens_pre"].numpy().copy()
        if w.fp8:
            kc = xb["k_cache"].numpy().copy()
            vc = xb["v_cache"].numpy().copy()
            ksc, vsc = x["k_scale"].numpy(), x["v_scale"].numpy()
        else:
            kc = xb["k_cache"].double().numpy().copy()
            vc = xb["v_cache"].double().numpy().copy()
        ts = time.perf_counter()
        if w.fp8:
            o.kv_append_fp8(xb["k_new"].float().numpy(), xb["v_new"].float().numpy(), kc, vc, ksc, vsc, lens)
            o.decode_fp8(q, kc, vc, ksc, vsc, lens, x["scale"], window=w.window)
        elif w.queries > 1:
            for j in range(w.queries):  # the Q drafted rows, in order
                o.kv_append(xb["k_new"][:, j].double().numpy(), xb["v_new"][:, j].double().numpy(), kc, vc, lens)
            o.decode_multi(q, kc, vc, lens, x["scale"])
        else:
            o.kv_append(xb["k_new"].double().numpy(), xb["v_new"].double().numpy(), kc, vc, lens)
            if w.window > 0:
                o.decode_window(q, kc, vc, lens, w.window, x["scale"])
            else:
                o.decode(q, kc, vc, lens, x["scale"])
        done.append(time.perf_counter() - ts)
        nbytes += inputs.ideal_kv_bytes(w, lens.tolist())
        b = (b + 1) % B
        if (steps is not None and len(done) >= steps) or (steps is None and sum(done) >= budget_s):
            break
    secs = sum(done)
    return {"value": round(nbytes / secs / 1e9, 4), "unit": "GB/s", "cores": o.max_threads(),
            "kind": "oracle",
            "sample": f"{len(done)} whole sequence(s) of {w.name} (append + decode, fp64), "
                      f"{secs:.1f} s of CPU time, {time.perf_counter() - t0:.1f} s wall",
            "sec_per_sequence": round(secs / len(done), 4)}


def profile_run(args, local):
    """Plain append + decode steps through the public API, nothing else: what ncu captures."""
    import grouped_query_attention_decode_b200 as gqa
    from grouped_query_attention_decode_b200 import inputs

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = inputs.WORKLOADS[args.workload]
    x = inputs.make_inputs(w)
    q, kn, vn = x["q"].to(dev), x["k_new"].to(dev), x["v_new"].to(dev)
    kc, vc = x["k_cache"].to(dev), x["v_cache"].to(dev)
    block_table = None
    if w.page_size > 0:
        paged = inputs.make_paged(x, w.page_size)
        kc, vc = paged["k_pool"].to(dev), paged["v_pool"].to(dev)
        block_table = paged["block_table"].to(dev)
    lens_rows = x["seq_lens_pre"].to(dev).repeat(args.warmup + args.steps, 1).contiguous()
    out = torch.empty((w.B, w.H_q, w.d), dtype=torch.float32, device=dev)
    if w.fp8:
        ws = gqa.alloc_workspace_fp8(w.B, w.H_q, w.H_kv, w.d, device=dev)
        ks, vs = x["k_scale"].to(dev), x["v_scale"].to(dev)
    else:
        ws = gqa.alloc_workspace(w.B, w.H_q, w.H_kv, w.d, w.dtype, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    for i in range(args.warmup + args.steps):
        if w.fp8:
            if block_table is not None:
                gqa.kv_append_paged_fp8(kn, vn, kc, vc, ks, vs, block_table, lens_rows[i], status=status)
                gqa.decode_paged_fp8(q, kc, vc, ks, vs, block_table, lens_rows[i], x["scale"], out=out,
                                     workspace=ws, status=status)
            else:
                gqa.kv_append_fp8(kn, vn, kc, vc, ks, vs, lens_rows[i], status=status)
                gqa.decode_fp8(q, kc, vc, ks, vs, lens_rows[i], x["scale"], window=w.window, out=out,
                               workspace=ws, status=status)
            continue
        if block_table is not None:
            gqa.kv_append_paged(kn, vn, kc, vc, block_table, lens_rows[i], status=status)
            gqa.decode_paged(q, kc, vc, block_table, lens_rows[i], x["scale"], out=out,
                             workspace=ws, status=status)
            continue
        gqa.kv_append(kn, vn, kc, vc, lens_rows[i], status=status)
        if w.window > 0:
            gqa.decode_window(q, kc, vc, lens_rows[i], w.window, x["scale"], out=out,
                              workspace=ws, status=status)
        else:
            gqa.decode(q, kc, vc, lens_rows[i], x["scale"], out=out, workspace=ws, status=status)
    torch.cuda.synchronize()
    st = int(status.item())
    assert st == 0, f"device status {st}"
    return {"profile_run": w.name, "steps": args.steps, "warmup": args.warmup,
            "launches_per_step": 2}


def bench_reference(args, rank, world):
    """Reference arm: the CPU oracle on the host cores, one sequence of the workload per step."""
    if rank != 0:
        return None
    from grouped_query_attention_decode_b200 import inputs

    w = inputs.WORKLOADS[args.workload]
    x = inputs.make_inputs(w)
    # warm-up steps, then K timed steps; each step = one whole sequence of the workload
    _ = cpu_baseline(w, x, 0.0, steps=min(args.warmup, 3))
    t0 = time.perf_counter()
    cb = cpu_baseline(w, x, 0.0, steps=args.steps)
    wall = time.perf_counter() - t0
    lens = x["lengths"].tolist()
    per_seq = inputs.ideal_kv_bytes(w, lens) / w.B
    ms = cb["sec_per_sequence"] * 1e3
    value = cb["value"]
    return {
        "impl": "reference",
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H_q": w.H_q, "H_kv": w.H_kv, "d": w.d,
                   "L_max": w.L_max, "step": "one whole sequence (append + decode) per step",
                   "ideal_kv_bytes_per_step": int(per_seq)},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cb["cores"], "kind": "oracle",
                         "sample": cb["sample"]},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "wall_s": round(wall, 2),
    }


def main():
    args = parse()
    rank, world, local = dist_env()
    if args.gpus != world and world != 1:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {world}", file=sys.stderr)
    if args.profile_run:
        res = profile_run(args, local)
    elif args.impl == "reference":
        res = bench_reference(args, rank, world)
    else:
        res = bench_ours(args, rank, world, local)
    if rank == 0 and res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
