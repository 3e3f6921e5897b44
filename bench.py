#!/usr/bin/env python3
"""Benchmark of one GQA decode step (KV append + split-KV decode with its in-kernel merge) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

One step = the append and the decode of one batch of the workload, through the C ABI: one
gqa_kv_append_decode launch for a contiguous bf16 cache with one query token per sequence (the
lengths are read from one array and written to another), else gqa_kv_append then the
workload's decode call.
`value` is the whole-job KV-read throughput: ideal KV bytes (2 * sum(n_b) * H_kv * d * bytes) of
all steps on all ranks divided by the device-timed duration (CUDA events, max over ranks).
The KV cache is resident state; each rank runs an independent replica (the decode of one
sequence needs nothing from any other), so scaling is weak and there is no collective on the
data path.  Enough copies of the cache rotate between steps that every copy is touched again
only after at least twice the L2 size of other K/V bytes has streamed through: each step reads
its cache from HBM, also for workloads whose cache alone would fit in L2.

The same JSON line carries, under "also", the ragged long-context workload (the second
workload the >= 80 % target is stated on), timed the same way.

--gpus N without torchrun re-executes itself under torch.distributed.run with N local ranks.
--impl reference times the CPU oracle (test infrastructure) on the host cores on a bounded
sample of the same workload, as the reference arm.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import socket
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
ALSO_DEFAULT = "ragged_long"
PROFILE_DIR = os.path.join(ROOT, "profiles")
CSRC = os.path.join(ROOT, "grouped_query_attention_decode_b200", "csrc")
# GPU-side spin (clock cycles, ~0.2 ms) that holds the stream while the host queues a timed
# region's launches
HOST_GATE_CYCLES = 400_000
E2E_MIN_STEPS = 200
KERNEL_SOURCES = {
    "split_tc_kernel": ("decode_tc.cu", "device.cuh", "schedule.cuh"),
    "split_tc8_kernel": ("decode_tc8.cu", "device.cuh", "schedule.cuh"),
    "split_f32_kernel": ("decode_f32.cu", "device.cuh", "schedule.cuh"),
}


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--also", default=ALSO_DEFAULT,
                    help="second workload timed into the same line ('none' to skip)")
    ap.add_argument("--kernel-seconds", type=float, default=1.0,
                    help="the split-kernel leg runs at least this long ...")
    ap.add_argument("--kernel-launches", type=int, default=500,
                    help="... and at least this many launches, whatever --steps is")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="budget of each CPU-oracle baseline sample (all cores, one core)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--profile-run", action="store_true",
                    help="only run warmup + steps plain API steps (one cache copy, no timing "
                         "report): the command ncu captures")
    return ap.parse_args(argv)


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def launcher_argv(n: int, argv: list[str], port: int | None = None) -> list[str]:
    """The command that runs this script as n local ranks (one per GPU) under torchrun."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
            "--master-addr", "127.0.0.1", f"--master-port={port or _free_port()}",
            os.path.abspath(__file__), *argv]


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


def strip_comments(src: str) -> str:
    """C/C++/CUDA source without comments and blank space (string literals here hold no comment
    markers): two sources that differ only in comments or layout give the same text."""
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    src = re.sub(r"//[^\n]*", " ", src)
    return " ".join(src.split())


def kernel_source_hash(kernel: str) -> str:
    """sha256[:16] of a kernel's sources with comments and layout stripped."""
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(CSRC, name)) as f:
            h.update(strip_comments(f.read()).encode())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str, kernel: str):
    """DRAM bytes per launch of `kernel` from a committed ncu summary, when that capture was
    taken on the current code of the kernel (comments aside); else None."""
    p = os.path.join(PROFILE_DIR, f"{kernel.replace('_kernel', '')}_{workload}.json")
    if not os.path.exists(p) or kernel not in KERNEL_SOURCES:
        return None
    with open(p) as f:
        d = json.load(f)
    if d.get("kernel_source_hash") != kernel_source_hash(kernel):
        return None
    return d.get("dram_bytes_per_launch_full_size")


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


# A plain read-only stream for the roofline's read figure: every thread loads 16-byte vectors
# with a grid stride, four in flight, and folds them into one word that is stored only if it
# equals a value it never takes.  Compiled at run time with NVRTC for the device in use; it is
# a measuring stick for this script, not part of the library.
READ_STREAM_SRC = r"""
extern "C" __global__ void read_stream(const uint4 *__restrict__ p, unsigned long long n,
                                       unsigned int *out) {
    unsigned int acc = 0u;
    const unsigned long long stride = (unsigned long long)gridDim.x * blockDim.x;
    unsigned long long i = (unsigned long long)blockIdx.x * blockDim.x + threadIdx.x;
    for (; i + 3 * stride < n; i += 4 * stride) {
        const uint4 a = p[i], b = p[i + stride], c = p[i + 2 * stride], d = p[i + 3 * stride];
        acc ^= (a.x ^ a.y ^ a.z ^ a.w) ^ (b.x ^ b.y ^ b.z ^ b.w) ^ (c.x ^ c.y ^ c.z ^ c.w) ^
               (d.x ^ d.y ^ d.z ^ d.w);
    }
    for (; i < n; i += stride) {
        const uint4 a = p[i];
        acc ^= a.x ^ a.y ^ a.z ^ a.w;
    }
    if (acc == 0x9e3779b9u) out[0] = acc;
}
"""


def read_stream_gbs(dev, nbytes: int = 4 << 30, reps: int = 10) -> dict:
    """HBM read bandwidth of a plain streaming read (READ_STREAM_SRC) over a buffer far larger
    than L2: the best over a few launch shapes of the best of `reps` CUDA-event timings.
    Returns {"gbs": None, ...} when the kernel cannot be built here."""
    import ctypes

    try:
        from cuda.bindings import driver as cu, nvrtc
        major, minor = torch.cuda.get_device_capability(dev)
        err, prog = nvrtc.nvrtcCreateProgram(READ_STREAM_SRC.encode(), b"read_stream.cu", 0, [], [])
        opts = [f"--gpu-architecture=sm_{major}{minor}a".encode()]
        err, = nvrtc.nvrtcCompileProgram(prog, len(opts), opts)
        if err != nvrtc.nvrtcResult.NVRTC_SUCCESS:
            raise RuntimeError(f"nvrtc: {err}")
        err, size = nvrtc.nvrtcGetCUBINSize(prog)
        cubin = b" " * size
        err, = nvrtc.nvrtcGetCUBIN(prog, cubin)
        torch.cuda.synchronize(dev)
        err, mod = cu.cuModuleLoadData(cubin)
        if err != cu.CUresult.CUDA_SUCCESS:
            raise RuntimeError(f"cuModuleLoadData: {err}")
        err, fn = cu.cuModuleGetFunction(mod, b"read_stream")
    except Exception as e:  # noqa: BLE001 - the figure is optional context
        return {"gbs": None, "how": f"read-stream kernel unavailable: {type(e).__name__}: {e}"}
    x = torch.empty(nbytes // 4, dtype=torch.int32, device=dev).fill_(1)
    out = torch.zeros(1, dtype=torch.int32, device=dev)
    n16 = nbytes // 16
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    stream = cu.CUstream(torch.cuda.current_stream(dev).cuda_stream)
    types = (ctypes.c_void_p, ctypes.c_ulonglong, ctypes.c_void_p)

    def launch(grid, block):
        err, = cu.cuLaunchKernel(fn, grid, 1, 1, block, 1, 1, 0, stream,
                                 ((x.data_ptr(), n16, out.data_ptr()), types), 0)
        assert err == cu.CUresult.CUDA_SUCCESS, err

    best, shape = 0.0, None
    for per_sm, block in ((4, 512), (8, 256), (2, 1024), (16, 256)):
        for _ in range(2):
            launch(sms * per_sm, block)
        torch.cuda.synchronize(dev)
        for _ in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            launch(sms * per_sm, block)
            b.record()
            torch.cuda.synchronize(dev)
            g = nbytes / (a.elapsed_time(b) * 1e-3) / 1e9
            if g > best:
                best, shape = g, (sms * per_sm, block)
    cu.cuModuleUnload(mod)
    del x
    torch.cuda.empty_cache()
    return {"gbs": round(best, 1),
            "how": f"read-only stream of {nbytes >> 20} MiB (16-byte loads, grid {shape[0]} x "
                   f"{shape[1]}), best of {reps} CUDA-event timings per launch shape"}


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 100 ms in the background."""
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
                 "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.fh,
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


def cache_copies(l2_bytes: int, step_bytes: int) -> int:
    """Copies of the cache that rotate so that a copy is read again only after >= 2 x L2 of
    other K/V bytes: every step then reads HBM, not L2."""
    return max(2, min(1024, 1 + math.ceil(2 * l2_bytes / step_bytes)))


def percentile(v, p):
    s = sorted(v)
    if not s:
        return None
    k = (len(s) - 1) * p / 100.0
    lo, hi = math.floor(k), math.ceil(k)
    return s[lo] + (s[hi] - s[lo]) * (k - lo)


class Replica:
    """One rank's copy of a workload on its GPU and the timed loops over it.

    n_copies copies of the cache rotate (step i uses copy i % n_copies) so that a copy is
    touched again only after >= 2 x L2 of other K/V bytes: every step reads from HBM."""

    def __init__(self, w, dev, n_copies=None):
        import grouped_query_attention_decode_b200 as gqa
        from grouped_query_attention_decode_b200 import inputs

        self.gqa, self.w, self.dev = gqa, w, dev
        x = inputs.make_inputs(w)
        self.x = x
        self.lengths = x["lengths"].tolist()
        self.ideal = inputs.ideal_kv_bytes(w, self.lengths)
        self.l2_bytes = int(torch.cuda.get_device_properties(dev).L2_cache_size)
        self.n_copies = n_copies or cache_copies(self.l2_bytes, self.ideal)
        self.q = x["q"].to(dev)
        self.kn, self.vn = x["k_new"].to(dev), x["v_new"].to(dev)
        self.block_table = None
        if w.page_size > 0:
            paged = inputs.make_paged(x, w.page_size)
            self.block_table = paged["block_table"].to(dev)
            first = (paged["k_pool"].to(dev), paged["v_pool"].to(dev))
        else:
            first = (x["k_cache"].to(dev), x["v_cache"].to(dev))
        self.caches = [first] + [(first[0].clone(), first[1].clone()) for _ in range(self.n_copies - 1)]
        self.copy_bytes = 2 * first[0].numel() * first[0].element_size()
        self.lens0 = x["seq_lens_pre"].to(dev)
        self.lens_dec = x["lengths"].to(dev)
        self.out = torch.empty(tuple(self.q.shape), dtype=torch.float32, device=dev)
        if w.queries > 1:
            nws = gqa.load_library().gqa_decode_multi_workspace_size(
                w.B, w.queries, w.H_q, w.H_kv, w.d,
                gqa.DTYPE_BF16 if w.dtype == torch.bfloat16 else gqa.DTYPE_F32)
            self.ws = torch.zeros(nws, dtype=torch.uint8, device=dev)
        elif w.fp8:
            self.ws = gqa.alloc_workspace_fp8(w.B, w.H_q, w.H_kv, w.d, device=dev)
        else:
            self.ws = gqa.alloc_workspace(w.B, w.H_q, w.H_kv, w.d, w.dtype, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.ks = x["k_scale"].to(dev) if w.fp8 else None
        self.vs = x["v_scale"].to(dev) if w.fp8 else None

    @property
    def kernel(self) -> str:
        if self.w.fp8:
            return "split_tc8_kernel"
        return "split_tc_kernel" if self.w.dtype == torch.bfloat16 else "split_f32_kernel"

    @property
    def dtype_name(self) -> str:
        return "e4m3" if self.w.fp8 else ("bf16" if self.w.dtype == torch.bfloat16 else "f32")

    def l2_label(self) -> str:
        return (f"inputs larger than L2 in rotation: {self.n_copies} cache copies "
                f"({self.n_copies * self.copy_bytes / 1e6:.0f} MB allocated, {self.ideal / 1e6:.1f} MB "
                f"read per step) rotate so a copy is re-read only after "
                f"{(self.n_copies - 1) * self.ideal / 1e6:.0f} MB of other K/V, "
                f">= 2 x the {self.l2_bytes / 1e6:.0f} MB L2")

    # ---------------------------------------------------------------- one step, through the API
    def append(self, c, lens_row, kk=None, vv=None):
        gqa, w = self.gqa, self.w
        kk = self.kn if kk is None else kk
        vv = self.vn if vv is None else vv
        kc, vc = self.caches[c]
        st = self.status
        if w.fp8:
            if self.block_table is not None:
                gqa.kv_append_paged_fp8(kk, vv, kc, vc, self.ks, self.vs, self.block_table, lens_row, status=st)
            else:
                gqa.kv_append_fp8(kk, vv, kc, vc, self.ks, self.vs, lens_row, status=st)
        elif self.block_table is not None:
            gqa.kv_append_paged(kk, vv, kc, vc, self.block_table, lens_row, status=st)
        elif w.queries > 1:
            gqa.kv_append_multi(kk, vv, kc, vc, lens_row, status=st)
        else:
            gqa.kv_append(kk, vv, kc, vc, lens_row, status=st)

    def decode(self, c, lens_row, qq=None, out=None):
        gqa, w, x = self.gqa, self.w, self.x
        qq = self.q if qq is None else qq
        kc, vc = self.caches[c]
        kw = dict(out=self.out if out is None else out, workspace=self.ws, status=self.status)
        if w.fp8:
            if self.block_table is not None:
                gqa.decode_paged_fp8(qq, kc, vc, self.ks, self.vs, self.block_table, lens_row, x["scale"], **kw)
            else:
                gqa.decode_fp8(qq, kc, vc, self.ks, self.vs, lens_row, x["scale"], window=w.window, **kw)
        elif self.block_table is not None:
            gqa.decode_paged(qq, kc, vc, self.block_table, lens_row, x["scale"], **kw)
        elif w.queries > 1:
            gqa.decode_multi(qq, kc, vc, lens_row, x["scale"], **kw)
        elif w.window > 0:
            gqa.decode_window(qq, kc, vc, lens_row, w.window, x["scale"], **kw)
        else:
            gqa.decode(qq, kc, vc, lens_row, x["scale"], **kw)

    @property
    def fused(self) -> bool:
        """One launch per step: gqa_kv_append_decode covers a contiguous bf16 cache with one
        query token per sequence and no window."""
        w = self.w
        return (not w.fp8 and w.dtype == torch.bfloat16 and self.block_table is None and
                w.queries == 1 and w.window == 0)

    def step(self, c, lens_row, qq=None, kk=None, vv=None, out=None):
        """Append + decode on cache copy c.  lens_row holds the lengths before the append and
        is advanced (two calls), or (fused) receives the lengths after it, read from lens0."""
        if self.fused:
            kc, vc = self.caches[c]
            self.gqa.kv_append_decode(self.q if qq is None else qq, self.kn if kk is None else kk,
                                      self.vn if vv is None else vv, kc, vc, self.lens0, lens_row,
                                      self.x["scale"], out=self.out if out is None else out,
                                      workspace=self.ws, status=self.status)
            return
        self.append(c, lens_row, kk, vv)
        self.decode(c, lens_row, qq, out)

    def launches_per_step(self) -> int:
        return 1 if self.fused else 2

    def read_stream(self) -> dict:
        return read_stream_gbs(self.dev)

    def check(self):
        """One step, then the device status must be clean and the lengths advanced."""
        lens = self.lens0.clone()
        self.step(0, lens)
        torch.cuda.synchronize()
        assert int(self.status.item()) == 0, f"device status {int(self.status.item())}"
        assert torch.equal(lens.cpu(), self.x["lengths"]), "seq_lens after the append"

    # ---------------------------------------------------------------- timed loops
    def _capture(self, n, decode_only=False):
        """A CUDA graph of n steps (or n decode launches); step j uses cache copy
        j % n_copies.  Steps append into their own pre-set length rows, re-armed by one copy at
        the top of the graph."""
        rows = self.lens0.repeat(max(n, 1), 1).contiguous()
        init = rows.clone()
        g = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream()
        cap.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(cap):
            with torch.cuda.graph(g, stream=cap):
                if decode_only:
                    for j in range(n):
                        self.decode(j % self.n_copies, self.lens_dec)
                else:
                    if not self.fused:  # the fused step only writes its length rows
                        rows.copy_(init)
                    for j in range(n):
                        self.step(j % self.n_copies, rows[j])
        torch.cuda.current_stream().wait_stream(cap)
        torch.cuda.synchronize()
        return g, (rows, init)

    def time_steps(self, K: int, W: int, barrier=None) -> float:
        """Device time (ms) of exactly K steps, on the current stream, with a barrier (all
        ranks) and a synchronize before and after.  After the barrier, a GPU-side spin holds the
        stream while the host queues W untimed warm-up steps, the first event, the K timed steps
        and the last event: host launch latency stays outside the timed region, and the first
        timed step follows a step on a busy GPU exactly as every later one does."""
        ng = self.n_copies * max(1, 64 // self.n_copies)
        full, keep_full = self._capture(ng)
        tail = K % ng
        tail_g, keep_tail = self._capture(tail) if tail else (None, None)
        warm_g, keep_warm = self._capture(W)
        for _ in range(max(1, -(-W // ng))):
            full.replay()
        (barrier or torch.cuda.synchronize)()
        torch.cuda.synchronize()
        stream = torch.cuda.current_stream()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda._sleep(HOST_GATE_CYCLES)
        warm_g.replay()
        e0.record(stream)
        for _ in range(K // ng):
            full.replay()
        if tail_g is not None:
            tail_g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        (barrier or torch.cuda.synchronize)()
        assert int(self.status.item()) == 0, f"device status {int(self.status.item())}"
        del full, tail_g, warm_g, keep_full, keep_tail, keep_warm
        return e0.elapsed_time(e1)

    def time_kernel(self, min_launches: int, min_seconds: float) -> list[float]:
        """The split-KV kernel alone: a graph of kg back-to-back launches of it -- the fused
        append + decode launch when that is the whole step, else the decode launch (consecutive
        launches overlap only as programmatic dependent launch allows) -- replayed until at
        least min_launches launches and min_seconds; CUDA events around every replay.  Returns
        the average µs per launch of each replay."""
        kg = self.n_copies * max(1, -(-100 // self.n_copies))
        g, keep = self._capture(kg, decode_only=not self.fused)
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        g.replay()
        b.record()
        torch.cuda.synchronize()
        per = max(a.elapsed_time(b) * 1e-3, 1e-6)
        reps = max(-(-min_launches // kg), math.ceil(min_seconds / per), 5)
        reps = min(reps, max(5, 200000 // kg))
        stream = torch.cuda.current_stream()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(reps + 1)]
        torch.cuda._sleep(HOST_GATE_CYCLES)
        ev[0].record(stream)
        for i in range(reps):
            g.replay()
            ev[i + 1].record(stream)
        torch.cuda.synchronize()
        assert int(self.status.item()) == 0, f"device status {int(self.status.item())}"
        del g, keep
        return [ev[i].elapsed_time(ev[i + 1]) * 1e3 / kg for i in range(reps)]

    def time_e2e(self, K: int, W: int) -> dict:
        """End to end through the public API, no graph: every step copies its inputs (q, k_new,
        v_new) in from pinned host memory, runs append + decode, and copies the result out to
        pinned host memory.

        The reported loop is a two-deep pipeline, as a serving loop runs it: the inputs of step
        i + 1 travel over a copy stream while step i computes, and step i's result travels back
        while step i + 1 computes (two sets of device input/output buffers; events order every
        copy against the steps that use its buffer).  The inputs of a step are packed in one
        pinned buffer, so a step makes one host-to-device and one device-to-host copy.  The
        breakdown also times the same steps with every copy in line on one stream, the steps
        without copies, and the copies alone."""
        x = self.x
        parts = [x["q"], x["k_new"], x["v_new"]]
        offs, total = [], 0
        for t in parts:
            offs.append(total)
            total += -(-t.numel() * t.element_size() // 256) * 256
        hin = torch.zeros(total, dtype=torch.uint8).pin_memory()
        for t, o in zip(parts, offs):
            nb = t.numel() * t.element_size()
            hin[o:o + nb].copy_(t.contiguous().view(-1).view(torch.uint8))

        def views(buf):
            return [buf[o:o + t.numel() * t.element_size()].view(t.dtype).view(t.shape)
                    for t, o in zip(parts, offs)]

        sets = []
        for _ in range(2):
            din = torch.empty(total, dtype=torch.uint8, device=self.dev)
            sets.append((din, views(din), torch.empty_like(self.out),
                         torch.empty(tuple(self.out.shape), dtype=torch.float32).pin_memory()))
        h2d = sum(t.numel() * t.element_size() for t in parts)
        d2h = self.out.numel() * 4
        rows = self.lens0.repeat(K + W, 1).contiguous()
        comp = torch.cuda.current_stream()
        cs = torch.cuda.Stream(device=self.dev)
        in_ready = [torch.cuda.Event() for _ in range(2)]
        comp_done = [torch.cuda.Event() for _ in range(2)]
        out_read = [torch.cuda.Event() for _ in range(2)]

        def run_pipelined(first, n, rows_of):
            def issue_in(i):
                s = i & 1
                with torch.cuda.stream(cs):
                    if i - first >= 2:
                        cs.wait_event(comp_done[s])  # step i - 2 has finished with set s
                    sets[s][0].copy_(hin, non_blocking=True)
                    in_ready[s].record(cs)

            issue_in(first)
            for i in range(first, first + n):
                s = i & 1
                if i + 1 < first + n:
                    issue_in(i + 1)
                comp.wait_event(in_ready[s])
                if i - first >= 2:
                    comp.wait_event(out_read[s])  # step i - 2's result has left buffer s
                dq, dkn, dvn = sets[s][1]
                self.step(i % self.n_copies, rows_of(i), dq, dkn, dvn, out=sets[s][2])
                comp_done[s].record(comp)
                with torch.cuda.stream(cs):
                    cs.wait_event(comp_done[s])
                    sets[s][3].copy_(sets[s][2], non_blocking=True)
                    out_read[s].record(cs)
            comp.wait_stream(cs)

        dq0, dkn0, dvn0 = sets[0][1]
        dout0, hout0 = sets[0][2], sets[0][3]

        def serial(i, r):
            sets[0][0].copy_(hin, non_blocking=True)
            self.step(i % self.n_copies, r, dq0, dkn0, dvn0, out=dout0)
            hout0.copy_(dout0, non_blocking=True)

        def api_only(i, r):
            self.step(i % self.n_copies, r)

        def copies_only(i, r):
            sets[0][0].copy_(hin, non_blocking=True)
            hout0.copy_(dout0, non_blocking=True)

        res = {}
        # pipelined: W warm-up steps, then K timed ones; the copy stream joins the compute
        # stream before the closing event, so every copy is inside the timed region
        rows.copy_(self.lens0.repeat(K + W, 1))
        run_pipelined(0, W, lambda i: rows[K + i])
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(comp)
        cs.wait_stream(comp)
        run_pipelined(0, K, lambda i: rows[i])
        b.record(comp)
        torch.cuda.synchronize()
        res["pipelined"] = a.elapsed_time(b) / K
        for name, fn in (("serial", serial), ("api_only", api_only), ("copies_only", copies_only)):
            rows.copy_(self.lens0.repeat(K + W, 1))
            for i in range(W):
                fn(i, rows[K + i])
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(comp)
            for i in range(K):
                fn(i, rows[i])
            b.record(comp)
            torch.cuda.synchronize()
            res[name] = a.elapsed_time(b) / K
        for st in sets:
            assert torch.isfinite(st[3]).all()
        assert int(self.status.item()) == 0, f"device status {int(self.status.item())}"
        return {"ms_per_step": res["pipelined"], "serial_ms_per_step": res["serial"],
                "api_only_ms_per_step": res["api_only"],
                "copies_only_ms_per_step": res["copies_only"], "h2d": h2d, "d2h": d2h}


def summarize_kernel(rep: Replica, launch_us: list[float], peak: float, peak_kind: str) -> dict:
    avg = statistics.mean(launch_us)
    achieved = rep.ideal / (avg * 1e-6) / 1e9
    return {
        "bound": "hbm", "kernel": rep.kernel,
        "achieved": round(achieved, 1), "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
        "frac": round(achieved / peak, 4),
        "traffic": profiled_traffic(rep.w.name, rep.kernel),
        "algorithmic_bytes_per_launch": rep.ideal,
        "avg_launch_us": round(avg, 3),
        "p10_launch_us": round(percentile(launch_us, 10), 3),
        "p90_launch_us": round(percentile(launch_us, 90), 3),
        "launches_timed": len(launch_us) * (rep.n_copies * max(1, -(-100 // rep.n_copies))),
        "replays_timed": len(launch_us),
    }


def bench_ours(args, rank, world, local):
    assert torch.cuda.is_available(), "the ours arm needs a CUDA device"
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
        pg = dist
    result = run_replica(args, rank, world, local, dev, pg, Replica)
    if pg is not None:
        pg.barrier()
        pg.destroy_process_group()
    return result


def run_replica(args, rank, world, local, dev, pg, make_replica):
    """Every rank times its own replica; the numbers are the max over ranks.  Every rank takes
    the same collective steps in the same order."""
    from grouped_query_attention_decode_b200 import inputs

    K, W = args.steps, args.warmup
    assert W >= 3 and K >= 1
    w = inputs.WORKLOADS[args.workload]
    rep = make_replica(w, dev)
    rep.check()
    peak, peak_kind = measured_peaks()

    def barrier():
        if pg is not None:
            pg.barrier()
        if torch.cuda.is_available():
            torch.cuda.synchronize()

    clocks = ClockSampler(local, enabled=not args.no_clocks)
    # the kernel leg first (>= 1 s: the clocks settle and the sampler sees them), then the
    # K timed steps
    barrier()
    launch_us = rep.time_kernel(args.kernel_launches, args.kernel_seconds)
    t_ms = rep.time_steps(K, W, barrier)
    clk = clocks.stop()
    ms_step = max_over_ranks(t_ms / K, pg, dev)
    launch_us_max = max_over_ranks(statistics.mean(launch_us), pg, dev)
    value = rep.ideal * world / (ms_step * 1e-3) / 1e9
    # the end-to-end loop issues every step from the host: at least E2E_MIN_STEPS of them, so
    # one-time host costs do not dominate a short run
    e2e_k, e2e_w = max(K, E2E_MIN_STEPS), max(W, 10)
    e2e = rep.time_e2e(e2e_k, e2e_w)
    e2e_ms = max_over_ranks(e2e["ms_per_step"], pg, dev)
    roof = summarize_kernel(rep, launch_us, peak, peak_kind)
    roof["avg_launch_us_max_over_ranks"] = round(launch_us_max, 3)
    read_peak = rep.read_stream()
    roof["read_stream_gbs"] = read_peak
    roof["frac_of_read_stream"] = (round(roof["achieved"] / read_peak["gbs"], 4)
                                   if read_peak.get("gbs") else None)
    roof["frac_of_8tbs_spec"] = round(roof["achieved"] / 8000.0, 4)
    also = None
    if args.also and args.also != "none" and args.also != args.workload:
        also = time_also(args, rank, world, local, dev, pg, make_replica, peak, peak_kind, barrier)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, rep.x, args.cpu_seconds)
    if rank != 0:
        return None
    lengths = rep.lengths
    return {
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
        "dtype": rep.dtype_name,
        "data": "synthetic",
        "config": {
            "workload": w.name, "B": w.B, "H_q": w.H_q, "H_kv": w.H_kv, "d": w.d,
            "L_max": w.L_max, "seq_len": lengths[0] if w.length else "ragged",
            "window": w.window or None,
            "page_size": w.page_size or None,
            "query_tokens": w.queries,
            "sum_seq_lens": int(sum(lengths)),
            "kv_dtype": "e4m3 (per-head scales)" if w.fp8 else str(w.dtype).replace("torch.", ""),
            "accumulate": "f32", "ideal_kv_bytes_per_step": rep.ideal,
            "parallelism": f"replicas x{world}",
            "l2": rep.l2_label(),
        },
        "gpu_launches": rep.launches_per_step() * K,
        "roofline": roof,
        "e2e": {
            "value": round(rep.ideal * world / (e2e_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
            "ms_per_step": round(e2e_ms, 6),
            "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
            "steps": e2e_k, "warmup": e2e_w,
            "copies": "one packed host-to-device copy of q, k_new, v_new and one device-to-host "
                      "copy of out per step, on a copy stream that overlaps the neighbouring steps",
            "breakdown_ms_per_step": {
                "copies_in_line_on_one_stream": round(e2e["serial_ms_per_step"], 6),
                "api_calls_without_copies": round(e2e["api_only_ms_per_step"], 6),
                "copies_alone": round(e2e["copies_only_ms_per_step"], 6),
                "device_step_in_graph": round(ms_step, 6),
            },
        },
        "clocks": clk,
        "also": also,
        "cpu_baseline": cpu,
    }


def time_also(args, rank, world, local, dev, pg, make_replica, peak, peak_kind, barrier):
    """The second workload: the same step and kernel legs, reported under "also"."""
    from grouped_query_attention_decode_b200 import inputs

    w2 = inputs.WORKLOADS[args.also]
    torch.cuda.empty_cache()
    r2 = make_replica(w2, dev)
    r2.check()
    clocks = ClockSampler(local, enabled=not args.no_clocks)
    barrier()
    launch_us = r2.time_kernel(args.kernel_launches, args.kernel_seconds)
    t_ms = r2.time_steps(args.steps, args.warmup, barrier)
    clk = clocks.stop()
    ms_step = max_over_ranks(t_ms / args.steps, pg, dev)
    value = r2.ideal * world / (ms_step * 1e-3) / 1e9
    roof = summarize_kernel(r2, launch_us, peak, peak_kind)
    res = {
        "workload": w2.name, "value": round(value, 2), "unit": "GB/s",
        "us_per_step": round(ms_step * 1e3, 3), "steps": args.steps, "warmup": args.warmup,
        "pct_of_measured_hbm": round(100 * value / world / peak, 2),
        "pct_of_8tbs_spec": round(100 * value / world / 8000.0, 2),
        "dtype": r2.dtype_name,
        "config": {"B": w2.B, "H_q": w2.H_q, "H_kv": w2.H_kv, "d": w2.d, "L_max": w2.L_max,
                   "sum_seq_lens": int(sum(r2.lengths)), "ideal_kv_bytes_per_step": r2.ideal,
                   "l2": r2.l2_label()},
        "gpu_launches": r2.launches_per_step() * args.steps,
        "roofline": roof,
        "clocks": clk,
    }
    del r2
    torch.cuda.empty_cache()
    return res


def cpu_baseline(w, x, budget_s, steps=None, nthreads=0):
    """The oracle, as it stands, on whole sequences of the workload until the time budget is
    used (at least one sequence).  Returns the baseline object in the bench's unit (GB/s).
    nthreads = 0: all host cores (OpenMP over query heads); 1: one core."""
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
            o.decode_fp8(q, kc, vc, ksc, vsc, lens, x["scale"], window=w.window, nthreads=nthreads)
        elif w.queries > 1:
            for j in range(w.queries):  # the Q drafted rows, in order
                o.kv_append(xb["k_new"][:, j].double().numpy(), xb["v_new"][:, j].double().numpy(), kc, vc, lens)
            o.decode_multi(q, kc, vc, lens, x["scale"], nthreads=nthreads)
        else:
            o.kv_append(xb["k_new"].double().numpy(), xb["v_new"].double().numpy(), kc, vc, lens)
            if w.window > 0:
                o.decode_window(q, kc, vc, lens, w.window, x["scale"], nthreads=nthreads)
            else:
                o.decode(q, kc, vc, lens, x["scale"], nthreads=nthreads)
        done.append(time.perf_counter() - ts)
        nbytes += inputs.ideal_kv_bytes(w, lens.tolist())
        b = (b + 1) % B
        if (steps is not None and len(done) >= steps) or (steps is None and sum(done) >= budget_s):
            break
    secs = sum(done)
    cores = 1 if nthreads == 1 else o.max_threads()
    res = {"value": round(nbytes / secs / 1e9, 4), "unit": "GB/s", "cores": cores,
           "kind": "oracle",
           "sample": f"{len(done)} whole sequence(s) of {w.name} (append + decode, fp64), "
                     f"{secs:.1f} s of CPU time, {time.perf_counter() - t0:.1f} s wall",
           "sec_per_sequence": round(secs / len(done), 4),
           "cpu_model": cpu_model()}
    if nthreads == 0 and steps is None:
        one = cpu_baseline(w, x, budget_s, nthreads=1)
        res["single_thread"] = {k: one[k] for k in ("value", "unit", "cores", "sample", "sec_per_sequence")}
    return res


def profile_run(args, local):
    """Plain steps through the public API on one cache copy, nothing else: what ncu captures
    (the same calls as the timed step)."""
    from grouped_query_attention_decode_b200 import inputs

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = inputs.WORKLOADS[args.workload]
    rep = Replica(w, dev, n_copies=1)
    rows = rep.lens0.repeat(args.warmup + args.steps, 1).contiguous()
    for i in range(args.warmup + args.steps):
        rep.step(0, rows[i])
    torch.cuda.synchronize()
    st = int(rep.status.item())
    assert st == 0, f"device status {st}"
    return {"profile_run": w.name, "steps": args.steps, "warmup": args.warmup,
            "launches_per_step": rep.launches_per_step()}


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
                         "sample": cb["sample"], "cpu_model": cb["cpu_model"]},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "wall_s": round(wall, 2),
    }


def main(argv=None):
    argv = sys.argv[1:] if argv is None else argv
    args = parse(argv)
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ and not args.profile_run:
        # one process per GPU: re-run this command as N local ranks
        cmd = launcher_argv(args.gpus, argv)
        os.execv(cmd[0], cmd)
    rank, world, local = dist_env()
    if args.gpus != world:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {world}; reporting n_gpus = {world}",
              file=sys.stderr)
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
