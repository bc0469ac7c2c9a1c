#!/usr/bin/env python
"""Benchmark of the MXFP8 scale-factor rearrange (per-group 128x4 blocked layout).

One step = one pass of the hot path over one batch of synthetic scales: the
three production shapes of the pytorch/ao pages, each one C-ABI call:
  * M-groups (131072, 44), G=8  -- the DSV3-16b shape of #3708 (flat-row TMA path)
  * M-groups (131072, 224), G=8 -- data K = 7168 (TMA path)
  * K-groups (7168, 4096), G=8  -- data K = 131072 tokens (TMA path)
Metric: GB/s = (bytes of real scales read + exact padded bytes written) / time,
and the same as a fraction of the measured HBM copy bandwidth.

Timing: the K timed steps are captured in one CUDA graph (as the pages timed
their kernels), uploaded to the device, and replayed once between two CUDA
events right after the warm-up graph; inputs and outputs rotate over enough
buffer sets that one rotation spans more than 4x the L2, so every step reads
cold inputs.  Each call's own per-launch duration (the roofline figure) comes
from a graph of that call's launches alone, back to back over the same
rotation, at least --call-launches of them so that the figure is the steady
state whatever K is: one untimed replay, then one timed replay.
Multi-GPU: independent replicas, one process per GPU (torchrun), max time
over ranks.

--workload k_sweep times every point of the K-groups sweep (M x TotalK, 70
points) the same way, each beside a same-size device copy and the CPU oracle.

--impl reference times the CPU oracle (the plain C statement of the layout)
on this host on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import re
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

WORKLOADS = {
    "moe_step": ["m_skinny", "m_wide", "k_groups"],
    "m_tiny": ["m_tiny"],
    "m_skinny": ["m_skinny"],
    "m_wide": ["m_wide"],
    "k_groups": ["k_groups"],
}
WORKLOAD_DESC = {
    "m_tiny": "M-groups 1000x44 G=4 with one empty group, stride 44 B (flat-row TMA)",
    "moe_step": "M-groups 131072x44 G=8 (flat-row TMA) + M-groups 131072x224 G=8 (TMA) + K-groups 7168x4096 G=8 (TMA)",
    "m_skinny": "M-groups 131072x44 G=8, stride 44 B (flat-row TMA)",
    "m_wide": "M-groups 131072x224 G=8 (TMA)",
    "k_groups": "K-groups 7168x4096 G=8 (TMA)",
}
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0   # B200 HBM3e, nominal (the measured copy peak is the roofline's denominator)
L2_BYTES = 126 * 2**20
METRIC = "rearrange GB/s (read+padded write) and % of B200 HBM peak, 1 GPU"


# ------------------------------------------------------------------ sizes
def ceil_to(x: int, a: int) -> int:
    return -(-x // a) * a


def clamped_sizes(ends, limit):
    e = np.minimum(np.maximum.accumulate(np.maximum(np.asarray(ends, np.int64), 0)), limit)
    return np.diff(np.concatenate([[0], e])), int(e[-1])


def algorithmic_bytes(case) -> dict:
    """Real input bytes read, exact padded bytes written, and the allocation."""
    M = case.dim == 0
    sizes, used = clamped_sizes(case.ends, case.rows if M else case.cols)
    if M:
        read = used * case.cols
        written = sum(ceil_to(int(n), 128) for n in sizes) * ceil_to(case.cols, 4)
        alloc = (case.rows + 128 * case.num_groups) * ceil_to(case.cols, 4)
    else:
        read = case.rows * used
        written = ceil_to(case.rows, 128) * sum(ceil_to(int(n), 4) for n in sizes)
        alloc = ceil_to(case.rows, 128) * (case.cols + 4 * case.num_groups)
    return {"read": int(read), "written": int(written), "alloc": int(alloc)}


def make_cases(workload: str):
    from scale_factor_layout_b200 import synth

    if workload == "k_sweep":
        return [synth.k_sweep_point(i, k) for i, k in synth.sweep_points()]
    if workload.startswith("k_sweep_"):
        m, total_k = (int(v) for v in workload[len("k_sweep_"):].split("x"))
        return [synth.k_sweep_point(synth.SWEEP_ROWS.index(m), synth.SWEEP_TOTAL_K.index(total_k))]
    return [synth.NAMED[name]() for name in WORKLOADS[workload]]


def workload_desc(workload: str) -> str:
    if workload == "k_sweep":
        return "K-groups sweep: M in {128..28672} x TotalK in {2^10..2^19}, scales M x TotalK/32, G=8 (70 points)"
    if workload.startswith("k_sweep_"):
        m, total_k = (int(v) for v in workload[len("k_sweep_"):].split("x"))
        return f"K-groups sweep point M={m} TotalK={total_k}: scales {m}x{total_k // 32}, G=8 (TMA)"
    return WORKLOAD_DESC[workload]


def workload_arg(value: str) -> str:
    from scale_factor_layout_b200 import synth

    if value in WORKLOADS or value == "k_sweep":
        return value
    if value.startswith("k_sweep_"):
        try:
            m, total_k = (int(v) for v in value[len("k_sweep_"):].split("x"))
            if m in synth.SWEEP_ROWS and total_k in synth.SWEEP_TOTAL_K:
                return value
        except ValueError:
            pass
    raise argparse.ArgumentTypeError(f"unknown workload {value!r}: one of {sorted(WORKLOADS)} or k_sweep_<M>x<TotalK>")


# ------------------------------------------------------------------ environment
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


FORWARD_SOURCES = ("mx_device.cuh", "mx_rearrange.cu")   # what the rearrange kernels are built from
INVERSE_SOURCES = ("mx_device.cuh", "mx_inverse.cu")     # what the inverse kernels are built from
HOST_MARKER = b"// ------------------------------------------------------------------ host side"


def kernel_source_sha(root: str = ROOT, op: str = "rearrange") -> str:
    """sha256 prefix of the device code of the op's kernels (mx_device.cuh, and
    mx_rearrange.cu or mx_inverse.cu up to its host-side section), with `//`
    comments and blank lines left out so that comment edits keep the key."""
    h = hashlib.sha256()
    csrc = os.path.join(root, "scale_factor_layout_b200", "csrc")
    for name in FORWARD_SOURCES if op == "rearrange" else INVERSE_SOURCES:
        with open(os.path.join(csrc, name), "rb") as f:
            data = f.read()
        cut = data.find(HOST_MARKER)
        code = data if cut < 0 else data[:cut]
        lines = (re.sub(rb"//.*", b"", ln).rstrip() for ln in code.split(b"\n"))
        h.update(name.encode())
        h.update(b"\n".join(ln for ln in lines if ln))
    return h.hexdigest()[:16]


def ncu_traffic(call: str, op: str = "rearrange", root: str = ROOT, path: str | None = None,
                detail: bool = False):
    """DRAM bytes per launch recorded by an ncu capture (profiles/ncu_traffic.txt)
    of the op's kernel for this call, or None when absent or taken on different
    kernel sources.  With detail=True: {"read", "write", "l2_write"} (l2_write,
    the bytes the kernel wrote into L2, is None where the capture lacks it)."""
    path = path or os.path.join(root, "profiles", "ncu_traffic.txt")
    if not os.path.exists(path):
        return None
    sha = kernel_source_sha(root, op=op)
    for line in open(path):
        if line.startswith("#") or not line.strip():
            continue
        kv = dict(tok.split("=", 1) for tok in line.split() if "=" in tok)
        if kv.get("op", "rearrange") == op and kv.get("call") == call and kv.get("source_sha") == sha:
            if not detail:
                return int(float(kv["bytes_per_launch"]))
            l2w = kv.get("l2_write")
            return {"read": int(float(kv["read"])), "write": int(float(kv["write"])),
                    "l2_write": int(float(l2w)) if l2w is not None else None}
    return None


class ClockSampler:
    """Samples SM clocks and clock-event reasons through NVML while running."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, index: int, period_s: float = 0.005):
        self.samples, self.period, self.index = [], period_s, index
        self._stop = threading.Event()
        self.window = None
        try:
            import pynvml

            pynvml.nvmlInit()
            self.nvml = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nvml = None
            self.max_mhz = None

    def _run(self):
        n = self.nvml
        while not self._stop.is_set():
            try:
                mhz = n.nvmlDeviceGetClockInfo(self.h, n.NVML_CLOCK_SM)
                reasons = n.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((time.perf_counter(), mhz, reasons))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nvml:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self.nvml:
            self.t.join()

    def summary(self):
        if not self.nvml or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        t0, t1 = self.window if self.window else (self.samples[0][0], self.samples[-1][0])
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        if len(inside) < 3:  # a short timed region: take the samples nearest to it
            mid = 0.5 * (t0 + t1)
            inside = sorted(self.samples, key=lambda s: abs(s[0] - mid))[:5]
        bits = 0
        for s in inside:
            bits |= s[2]
        reasons = [name for b, name in self.REASONS.items() if bits & b and name != "gpu_idle"]
        return {"sm_mhz": statistics.median(s[1] for s in inside), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(inside)}


# ------------------------------------------------------------------ distributed
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def dist_init(world: int, backend: str):
    if world <= 1:
        return None
    import datetime

    import torch.distributed as dist

    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return dist


def max_over_ranks(value: float, dist, device=None) -> float:
    """Max of a per-rank float over all ranks (identity without a process group)."""
    if dist is None:
        return value
    import torch

    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(dist, device=None):
    if dist is not None:
        if device is not None:
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def aggregate_value(bytes_per_step: int, steps: int, n_gpus: int, seconds: float) -> float:
    """Whole-job GB/s: the bytes all replicas moved over the slowest rank's time."""
    return bytes_per_step * steps * n_gpus / seconds / 1e9


# ------------------------------------------------------------------ GPU arm
def device_copies(case, n, device, op="rearrange"):
    """n independent device copies of a case's inputs, each with its own output.
    For the inverse, the input is the blocked layout (made once here by the
    forward call) and the output a row-major (rows, cols) buffer."""
    import torch

    import scale_factor_layout_b200 as mxs

    out = []
    host_s = torch.from_numpy(np.ascontiguousarray(case.scales))
    host_e = torch.from_numpy(np.ascontiguousarray(case.ends, dtype=np.int32))
    size = mxs.mx_rearranged_size(case.dim, case.rows, case.cols, case.num_groups)
    for _ in range(n):
        s, e = host_s.to(device), host_e.to(device)
        if op == "inverse":
            blocked = mxs.rearrange(case.dim, s, e)
            out.append((case, blocked, e, torch.empty((case.rows, case.cols), dtype=torch.uint8, device=device)))
            del s
        else:
            out.append((case, s, e, torch.empty(size, dtype=torch.uint8, device=device)))
    return out


def rotation_count(case) -> int:
    """Copies needed so that one rotation of this call alone spans 4x the L2."""
    b = algorithmic_bytes(case)
    return max(2, math.ceil(4 * L2_BYTES / (b["read"] + b["alloc"])))


def launch(item, stream_handle, op="rearrange", path="auto"):
    from scale_factor_layout_b200 import _binding as B

    c, s, e, o = item
    if op == "inverse":
        fn = B.mx_unrearrange_m_groups if c.dim == 0 else B.mx_unrearrange_k_groups
        st = fn(s.data_ptr(), c.rows, c.cols, e.data_ptr(), c.num_groups, o.data_ptr(), c.cols, stream_handle)
    else:
        st = B.mx_rearrange_ex(c.dim, s.data_ptr(), c.rows, c.cols, c.cols, e.data_ptr(), c.num_groups,
                               o.data_ptr(), B.PATHS[path], stream_handle)
    if st != B.MX_OK:
        raise RuntimeError(f"{c.name}: {B.status_string(st)}")


_libcuda = None


def upload_graph(g, stream_handle: int) -> None:
    """Upload a captured graph's executable to the device ahead of its first
    replay (cuGraphUpload), so that no timed replay pays for the upload."""
    global _libcuda
    import ctypes

    if _libcuda is None:
        lib = ctypes.CDLL("libcuda.so.1")
        lib.cuGraphUpload.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
        lib.cuGraphUpload.restype = ctypes.c_int
        _libcuda = lib
    r = _libcuda.cuGraphUpload(ctypes.c_void_p(g.raw_cuda_graph_exec()), ctypes.c_void_p(stream_handle))
    if r != 0:
        raise RuntimeError(f"cuGraphUpload failed (CUresult {r})")


class GraphTimer:
    """CUDA graphs of launches on one stream, timed with CUDA events on that
    stream, barrier and synchronize on both sides, max over ranks."""

    def __init__(self, stream, dist, device):
        self.stream, self.dist, self.device = stream, dist, device
        self.handle = stream.cuda_stream

    def capture(self, fn_calls):
        """One graph holding the calls (each a zero-argument callable that
        enqueues work on the stream), uploaded to the device."""
        import torch

        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(self.stream):
            with torch.cuda.graph(g, stream=self.stream):
                for fn in fn_calls:
                    fn()
        upload_graph(g, self.handle)
        return g

    def replay(self, g):
        import torch

        with torch.cuda.stream(self.stream):
            g.replay()

    def time(self, g, pre=None) -> float:
        """Seconds of one replay of g (max over ranks); `pre` is replayed
        untimed right before, on the same stream."""
        import torch

        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        barrier(self.dist, self.device)
        torch.cuda.synchronize()
        with torch.cuda.stream(self.stream):
            if pre is not None:
                pre.replay()
            start.record(self.stream)
            g.replay()
            end.record(self.stream)
        torch.cuda.synchronize()
        barrier(self.dist, self.device)
        return max_over_ranks(start.elapsed_time(end) / 1e3, self.dist, self.device)

    def steady(self, g, n: int) -> float:
        """Average seconds per launch of a graph of n launches back to back:
        one untimed replay, then one timed replay."""
        self.replay(g)
        return self.time(g) / n


def per_launch_launches(steps: int, minimum: int) -> int:
    """Launches in each per-call timing graph: the timed step count, but at
    least `minimum`, so that the per-launch figure is the steady state of
    back-to-back launches whatever --steps is."""
    return max(steps, minimum)


def roofline_entry(kernel: str, case_name: str, bytes_moved: int, seconds: float, peak: float, peak_src: str,
                   traffic) -> dict:
    """The roofline object of the bench line for the dominant kernel."""
    achieved = bytes_moved / seconds / 1e9
    out = {"bound": "hbm", "kernel": f"{kernel} ({case_name})", "achieved": round(achieved, 1), "peak": peak,
           "unit": "GB/s", "frac": round(achieved / peak, 4), "peak_source": f"{peak_src} hbm_gbs",
           "nominal_peak": NOMINAL_HBM_GBS, "frac_of_nominal": round(achieved / NOMINAL_HBM_GBS, 4),
           "algorithmic_bytes": bytes_moved, "traffic": None}
    if traffic is not None:
        out["traffic"] = traffic["read"] + traffic["write"]
        out["traffic_read"] = traffic["read"]
        out["traffic_write"] = traffic["write"]
        if traffic.get("l2_write") is not None:
            out["traffic_l2_write"] = traffic["l2_write"]
        if traffic["write"] < 0.1 * (bytes_moved - traffic["read"]):
            out["traffic_note"] = ("read-dominated: the launch's output is still in L2 when it ends (written back "
                                   "to DRAM later); traffic_l2_write is what the kernel wrote to L2")
    return out


def inverse_kernel_name(case) -> str:
    """The inverse kernel the library picks for a case written to a dense,
    16-byte aligned row-major tensor (as the bench allocates it)."""
    if case.dim == 1:
        return "unrearrange_box_k_kernel" if case.cols >= 16 else "unrearrange_kernel<K, 8>"
    if case.cols <= 128 and case.cols % 4 == 0:
        return "unrearrange_kernel<M, 4>" if ceil_to(case.cols, 4) <= 48 else "unrearrange_kernel<M, 8>"
    return "unrearrange_tma_m_kernel" if case.cols % 16 == 0 else "unrearrange_kernel<M, 8>"


def run_ours(args, rank, world, local):
    import torch

    import scale_factor_layout_b200 as mxs
    from scale_factor_layout_b200 import _binding as B
    from scale_factor_layout_b200 import _build

    _build.build()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    dist = dist_init(world, "nccl")
    if args.workload == "k_sweep":
        return run_sweep(args, rank, world, device, dist)
    cases = make_cases(args.workload)
    per_call = [algorithmic_bytes(c) for c in cases]
    step_bytes = sum(b["read"] + b["written"] for b in per_call)
    step_bytes_pages = sum(b["read"] + b["alloc"] for b in per_call)

    rot = [device_copies(c, rotation_count(c), device, args.op) for c in cases]
    rot_bytes = sum(len(r) * (algorithmic_bytes(c)["read"] + algorithmic_bytes(c)["alloc"])
                    for c, r in zip(cases, rot))
    stream = torch.cuda.Stream(device)
    h = stream.cuda_stream
    ncalls = len(cases)
    timer = GraphTimer(stream, dist, device)

    def step_items(k):
        return [r[k % len(r)] for r in rot]

    with torch.cuda.stream(stream):
        for k in range(3):  # first calls set kernel attributes (outside capture) and warm caches
            for it in step_items(k):
                launch(it, h, args.op, args.path)
    torch.cuda.synchronize()

    def calls_of(items):
        return [lambda it=it: launch(it, h, args.op, args.path) for it in items]

    def steps_of(k0, n):
        return [it for k in range(k0, k0 + n) for it in step_items(k)]

    def copies_of(i, n):
        """The practical ceiling for call i: a D2D copy of its input bytes
        (read + write the same traffic), same rotation, same graph timing."""
        srcs = [it[1] for it in rot[i]]
        dsts = [torch.empty_like(x) for x in srcs]
        with torch.cuda.stream(stream):
            for a, b in zip(srcs, dsts):   # warm the copy path outside capture
                b.copy_(a)
        torch.cuda.synchronize()
        return [lambda a=srcs[k % len(srcs)], b=dsts[k % len(dsts)]: b.copy_(a) for k in range(n)], dsts

    warm_g = timer.capture(calls_of(steps_of(0, args.warmup)))
    timed_g = timer.capture(calls_of(steps_of(args.warmup, args.steps)))

    sampler = ClockSampler(local)
    with sampler:
        timer.replay(warm_g)
        t0 = time.perf_counter()
        seconds_max = timer.time(timed_g)
        t1 = time.perf_counter()
        sampler.window = (t0, t1)
        del timed_g
        # Each call's own per-launch duration: its launches back to back in a
        # graph of their own (same rotation, cold inputs), in steady state.
        n_call = per_launch_launches(args.steps, args.call_launches)
        avg, copy_avg = [], None
        for i in range(ncalls):
            g = timer.capture(calls_of([rot[i][k % len(rot[i])] for k in range(n_call)]))
            avg.append(timer.steady(g, n_call))
            del g
        if not args.no_copy_ceiling:
            copy_avg = []
            for i in range(ncalls):
                fns, dsts = copies_of(i, n_call)
                g = timer.capture(fns)
                copy_avg.append(timer.steady(g, n_call))
                del g, dsts
    del warm_g

    peak, peak_src = load_peaks()
    value = aggregate_value(step_bytes, args.steps, world, seconds_max)
    calls = []
    for ci, (c, b, t) in enumerate(zip(cases, per_call, avg)):
        gbs = (b["read"] + b["written"]) / t / 1e9
        path = (mxs.mx_select_path(c.dim, rot[ci][0][1].data_ptr(), c.rows, c.cols, c.cols)
                if args.path == "auto" else B.PATHS[args.path])
        calls.append({"case": c.name, "path": B.PATH_NAMES.get(path, "?"),
                      "us": round(t * 1e6, 3), "gbps": round(gbs, 1), "frac_of_peak": round(gbs / peak, 4),
                      "frac_of_nominal": round(gbs / NOMINAL_HBM_GBS, 4),
                      "read_bytes": b["read"], "written_bytes": b["written"], "alloc_bytes": b["alloc"],
                      "gbps_pages_convention": round((b["read"] + b["alloc"]) / t / 1e9, 1),
                      "launches_timed": n_call})
        if copy_avg is not None:
            cbytes = 2 * c.rows * c.cols   # the copy reads and writes the input's bytes
            cg = cbytes / copy_avg[ci] / 1e9
            calls[-1].update({"copy_us": round(copy_avg[ci] * 1e6, 3), "copy_gbps": round(cg, 1),
                              "frac_of_copy": round(gbs / cg, 4)})
    dom = max(range(ncalls), key=lambda i: avg[i])
    dc = calls[dom]
    kernel_names = {"tma": "rearrange_tma_m" if cases[dom].dim == 0 else "rearrange_tma_k",
                    "flat": "rearrange_flat_tma", "word": "rearrange_fallback", "byte": "rearrange_fallback"}
    kname = inverse_kernel_name(cases[dom]) if args.op == "inverse" else kernel_names.get(dc["path"], "?")
    traffic = ncu_traffic(dc["case"], args.op, detail=True) if args.path == "auto" else None
    roofline = roofline_entry(kname, dc["case"], dc["read_bytes"] + dc["written_bytes"], avg[dom], peak, peak_src,
                              traffic)

    if args.op == "inverse":
        for cl in calls:
            cl["path"] = "inverse"
    e2e = (run_e2e(args, cases, device, world, dist)
           if not args.no_e2e and args.op == "rearrange" and args.path == "auto" else None)
    result = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(seconds_max / args.steps * 1e3, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "u8",
        "data": "synthetic (seeded uniform E8M0 bytes, seeded group splits)",
        "config": {"workload": args.workload, "op": args.op, "path": args.path,
                   "description": workload_desc(args.workload),
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "bytes_per_step": step_bytes, "bytes_per_step_pages_convention": step_bytes_pages,
                   "l2": "inputs/outputs rotate per call over " + ", ".join(str(len(r)) for r in rot)
                         + f" copies ({rot_bytes / 1e6:.0f} MB); each call's rotation alone spans > 4x L2",
                   "timing": "the timed steps: one CUDA graph (uploaded beforehand) replayed once between two CUDA "
                             "events after the warm-up graph, max over ranks; per-call durations: each call's "
                             f"launches back to back in a graph of their own ({n_call} launches, same rotation), "
                             "one untimed replay, then one timed replay"},
        "frac_of_peak": round(value / world / peak, 4),
        "frac_of_nominal": round(value / world / NOMINAL_HBM_GBS, 4),
        "calls": calls,
        "roofline": roofline,
        "e2e": e2e,
        "gpu_launches": args.steps * ncalls,
        "clocks": sampler.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(cases, args.cpu_seconds)
    if dist is not None:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result))


SWEEP_MAX_COPIES = 64            # rotation cap per sweep point (small points stay L2-warm)
SWEEP_GRAPH_SECONDS = 0.02       # about this much work per timing graph
SWEEP_ORACLE_SINGLE_RUN = 256e6  # traffic above which the oracle is timed on one run


def sweep_launches(traffic_bytes: int) -> int:
    """Launches per timing graph of a sweep point: about SWEEP_GRAPH_SECONDS of
    work at an assumed 4 TB/s plus 3 us per launch, between 20 and 2000."""
    est = 3e-6 + traffic_bytes / 4e12
    return int(min(2000, max(20, SWEEP_GRAPH_SECONDS / est)))


def oracle_seconds(case, op: str = "rearrange") -> tuple[float, str]:
    """Single-thread CPU oracle time of one full call (the rearrange, or the
    inverse of the oracle's own blocked output): the median of 3 runs (each
    repeated to at least 20 ms for tiny points), or one run above
    SWEEP_ORACLE_SINGLE_RUN bytes of traffic."""
    import oracle

    oracle.load()
    if op == "inverse":
        blocked = oracle.rearrange(case.dim, case.scales, case.ends)

        def call():
            oracle.inverse(case.dim, blocked, case.rows, case.cols, case.ends)
    else:
        def call():
            oracle.rearrange(case.dim, case.scales, case.ends)
    b = algorithmic_bytes(case)
    if b["read"] + b["written"] > SWEEP_ORACLE_SINGLE_RUN:
        t0 = time.perf_counter()
        call()
        return time.perf_counter() - t0, "1 run"
    t0 = time.perf_counter()
    call()
    once = max(time.perf_counter() - t0, 1e-7)
    reps = max(1, int(math.ceil(0.02 / once)))
    runs = []
    for _ in range(3):
        t0 = time.perf_counter()
        for _ in range(reps):
            call()
        runs.append((time.perf_counter() - t0) / reps)
    return statistics.median(runs), f"median of 3 runs of {reps}"


def run_sweep(args, rank, world, device, dist):
    """Every point of the K-groups sweep, one after another (the rearrange, or
    with --op inverse the inverse): per point, its launches back to back in
    one uploaded graph over a rotation of input and output copies (one
    untimed replay, one timed), a device copy of the same input timed the
    same way, and the CPU oracle on the host."""
    import torch

    from scale_factor_layout_b200 import synth

    peak, peak_src = load_peaks()
    op = args.op
    stream = torch.cuda.Stream(device)
    h = stream.cuda_stream
    timer = GraphTimer(stream, dist, device)
    points, total_bytes, total_s, launches = [], 0, 0.0, 0
    sampler = ClockSampler(device.index)
    with sampler:
        t_start = time.perf_counter()
        for i_m, i_k in synth.sweep_points():
            case = synth.k_sweep_point(i_m, i_k)
            b = algorithmic_bytes(case)
            traffic = b["read"] + b["written"]
            per_copy = b["read"] + b["alloc"]
            n_rot = min(max(2, math.ceil(4 * L2_BYTES / per_copy)), SWEEP_MAX_COPIES)
            rot = device_copies(case, n_rot, device, op)
            with torch.cuda.stream(stream):
                launch(rot[0], h, op)
            n = sweep_launches(traffic)
            g = timer.capture([lambda it=rot[k % n_rot]: launch(it, h, op) for k in range(n)])
            t = timer.steady(g, n)
            del g
            srcs = [it[1] for it in rot]
            copy_bytes = 2 * srcs[0].numel()
            dsts = [torch.empty_like(x) for x in srcs]
            g = timer.capture([lambda a=srcs[k % n_rot], d=dsts[k % n_rot]: d.copy_(a) for k in range(n)])
            t_copy = timer.steady(g, n)
            del g, dsts, srcs, rot
            torch.cuda.empty_cache()
            entry = {"M": case.extra["M"], "TotalK": case.extra["TotalK"], "rows": case.rows, "cols": case.cols,
                     "us": round(t * 1e6, 3), "gbps": round(traffic / t / 1e9, 1),
                     "frac_of_peak": round(traffic / t / 1e9 / peak, 4),
                     "frac_of_nominal": round(traffic / t / 1e9 / NOMINAL_HBM_GBS, 4),
                     "gbps_pages_convention": round(per_copy / t / 1e9, 1),
                     "read_bytes": b["read"], "written_bytes": b["written"], "alloc_bytes": b["alloc"],
                     "copy_us": round(t_copy * 1e6, 3),
                     "frac_of_copy": round((traffic / t) / (copy_bytes / t_copy), 4),
                     "launches_timed": n, "rotation": n_rot, "l2_cold": n_rot * per_copy >= 4 * L2_BYTES}
            if rank == 0 and not args.no_cpu_baseline:
                ts, how = oracle_seconds(case, op)
                entry.update({"oracle_us": round(ts * 1e6, 1), "oracle_gbps": round(traffic / ts / 1e9, 3),
                              "oracle_runs": how})
            points.append(entry)
            total_bytes += traffic
            total_s += t
            launches += n
        sampler.window = (t_start, time.perf_counter())
    big = [p for p in points if p["read_bytes"] + p["written_bytes"] >= 32e6]
    result = {
        "metric": METRIC, "value": round(total_bytes / total_s / 1e9, 1), "unit": "GB/s", "n_gpus": world,
        "steps": 1, "warmup": args.warmup, "ms_per_step": round(total_s * 1e3, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "u8",
        "data": "synthetic (seeded uniform E8M0 bytes, seeded group splits)",
        "config": {"workload": "k_sweep", "op": op, "path": "auto",
                   "description": "K-groups sweep: M in {128..28672} x TotalK in {2^10..2^19}, scales M x TotalK/32, "
                                  "G=8 (70 points); a step is one pass over every point",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "bytes_per_step": total_bytes,
                   "l2": f"per point, inputs/outputs rotate over copies spanning >= 4x L2 where at most "
                         f"{SWEEP_MAX_COPIES} copies suffice (l2_cold), else over {SWEEP_MAX_COPIES} copies",
                   "timing": "per point: its launches back to back in one uploaded CUDA graph, one untimed replay, "
                             "one timed replay between CUDA events; value = all points' bytes / the sum of their "
                             "per-launch times"},
        "frac_of_peak": round(total_bytes / total_s / 1e9 / peak, 4),
        "points": points,
        "large_points_min_frac_of_peak": min((p["frac_of_peak"] for p in big), default=None),
        "roofline": roofline_entry("unrearrange_box_k_kernel" if op == "inverse" else "rearrange_tma_k",
                                   "k_sweep, all points", total_bytes, total_s, peak, peak_src, None),
        "e2e": None,
        "gpu_launches": launches,
        "clocks": sampler.summary(),
    }
    if rank == 0 and not args.no_cpu_baseline:
        t_cpu = sum(p["oracle_us"] for p in points) * 1e-6
        result["cpu_baseline"] = {"value": round(total_bytes / t_cpu / 1e9, 3), "unit": "GB/s", "cores": 1,
                                  "kind": "oracle",
                                  "sample": f"every sweep point once (median of 3 below {SWEEP_ORACLE_SINGLE_RUN/1e6:.0f} "
                                            f"MB of traffic), single thread, gcc -O2, {os.cpu_count()} host cores "
                                            f"({cpu_model()})"}
    if dist is not None:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result))


def run_e2e(args, cases, device, world, dist):
    """Through the public torch-level API: every step copies its inputs in from
    pinned host memory, rearranges them, and copies the output back.  The
    copies run on their own streams, double-buffered, so that one step's
    inputs go in while the previous step's output comes back (PCIe carries
    both directions at once); events order each buffer's reuse."""
    import torch

    import scale_factor_layout_b200 as mxs

    host_in = [(torch.from_numpy(np.ascontiguousarray(c.scales)).pin_memory(),
                torch.from_numpy(np.ascontiguousarray(c.ends, dtype=np.int32)).pin_memory()) for c in cases]
    sizes = [mxs.mx_rearranged_size(c.dim, c.rows, c.cols, c.num_groups) for c in cases]
    nbuf = 2
    dev_in = [[(torch.empty(s.shape, dtype=torch.uint8, device=device),
                torch.empty(e.shape, dtype=torch.int32, device=device)) for s, e in host_in] for _ in range(nbuf)]
    dev_out = [[torch.empty(n, dtype=torch.uint8, device=device) for n in sizes] for _ in range(nbuf)]
    host_out = [[torch.empty(n, dtype=torch.uint8).pin_memory() for n in sizes] for _ in range(nbuf)]
    steps = max(3, min(args.steps, args.e2e_steps))
    s_in, s_run, s_out = (torch.cuda.Stream(device) for _ in range(3))
    ncalls = len(cases)
    # per buffer and call: inputs consumed (rearrange done) and output drained (copied back)
    used = [[None] * ncalls for _ in range(nbuf)]
    drained = [[None] * ncalls for _ in range(nbuf)]

    def step(k):
        b = k % nbuf
        for i, c in enumerate(cases):
            (hs, he), (ds, de) = host_in[i], dev_in[b][i]
            with torch.cuda.stream(s_in):
                if used[b][i] is not None:
                    s_in.wait_event(used[b][i])
                ds.copy_(hs, non_blocking=True)
                de.copy_(he, non_blocking=True)
                loaded = torch.cuda.Event()
                loaded.record(s_in)
            with torch.cuda.stream(s_run):
                s_run.wait_event(loaded)
                if drained[b][i] is not None:
                    s_run.wait_event(drained[b][i])
                mxs.rearrange(c.dim, ds, de, out=dev_out[b][i])
                done = torch.cuda.Event()
                done.record(s_run)
                used[b][i] = done
            with torch.cuda.stream(s_out):
                s_out.wait_event(done)
                host_out[b][i].copy_(dev_out[b][i], non_blocking=True)
                out_ev = torch.cuda.Event()
                out_ev.record(s_out)
                drained[b][i] = out_ev

    main = torch.cuda.current_stream(device)

    def run(k0, n):
        for st in (s_in, s_run, s_out):
            st.wait_stream(main)
        for k in range(k0, k0 + n):
            step(k)
        for st in (s_in, s_run, s_out):
            main.wait_stream(st)

    run(0, 2)
    torch.cuda.synchronize()
    barrier(dist, device)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(main)
    run(2, steps)
    end.record(main)
    torch.cuda.synchronize()
    seconds = max_over_ranks(start.elapsed_time(end) / 1e3, dist, device)
    per_call = [algorithmic_bytes(c) for c in cases]
    step_bytes = sum(b["read"] + b["written"] for b in per_call)
    h2d = sum(s.numel() + e.numel() * 4 for s, e in host_in)
    d2h = sum(sizes)
    return {"value": round(aggregate_value(step_bytes, steps, world, seconds), 2), "unit": "GB/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "ms_per_step": round(seconds / steps * 1e3, 4),
            "note": "copies in and out on their own streams, double-buffered, overlapping across steps"}


# ------------------------------------------------------------------ CPU oracle
def cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_baseline(cases, budget_s: float) -> dict:
    """The CPU oracle as it stands (single-threaded C), on this host, over
    whole-call repetitions of the workload until about `budget_s` seconds."""
    import oracle

    oracle.load()
    per = [algorithmic_bytes(c) for c in cases]
    step_bytes = sum(b["read"] + b["written"] for b in per)
    reps, t_total = 0, 0.0
    while t_total < budget_s and reps < 1000:
        t0 = time.perf_counter()
        for c in cases:
            oracle.rearrange(c.dim, c.scales, c.ends)
        t_total += time.perf_counter() - t0
        reps += 1
    return {"value": round(step_bytes * reps / t_total / 1e9, 3), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"{reps} full steps ({'+'.join(c.name for c in cases)}), {t_total:.1f} s, "
                      f"single thread, gcc -O2, {os.cpu_count()} host cores ({cpu_model()})"}


def sample_cases(cases, fraction: float):
    """Leading row blocks of each case (offsets clamped by the layout's own rule)."""
    from scale_factor_layout_b200 import synth

    out = []
    for c in cases:
        rows = max(128, int(c.rows * fraction) // 128 * 128) if c.rows >= 128 else c.rows
        out.append(synth.Case(c.name, c.dim, c.scales[:rows], c.ends.copy(), c.seed))
    return out


def run_reference(args, rank, world):
    """The CPU oracle as the reference arm (rank 0 only; other ranks exit)."""
    if rank != 0:
        return
    import oracle

    oracle.load()
    cases = make_cases(args.workload)

    def runner(sample):
        """One step's oracle work: the rearrange, or for --op inverse the
        oracle's inverse of its own blocked output (made once, outside the timing)."""
        if args.op == "inverse":
            blocked = [oracle.rearrange(c.dim, c.scales, c.ends) for c in sample]
            return lambda: [oracle.inverse(c.dim, b, c.rows, c.cols, c.ends) for c, b in zip(sample, blocked)]
        return lambda: [oracle.rearrange(c.dim, c.scales, c.ends) for c in sample]

    full = runner(cases)
    t0 = time.perf_counter()
    full()
    full_step = time.perf_counter() - t0
    budget = 120.0
    fraction = min(1.0, budget / max(1e-9, full_step * (args.steps + args.warmup)))
    sample = cases if fraction >= 1.0 else sample_cases(cases, fraction)
    per = [algorithmic_bytes(c) for c in sample]
    step_bytes = sum(b["read"] + b["written"] for b in per)
    work = runner(sample)
    for _ in range(args.warmup):
        work()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        work()
    seconds = time.perf_counter() - t0
    value = step_bytes * args.steps / seconds / 1e9
    desc = "full workload" if fraction >= 1.0 else f"leading {fraction:.3f} of each case's rows"
    res = {"impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "GB/s", "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(seconds / args.steps * 1e3, 3),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "u8",
           "data": "synthetic (seeded uniform E8M0 bytes, seeded group splits)",
           "config": {"workload": args.workload, "op": args.op, "path": args.path,
                      "description": workload_desc(args.workload),
                      "parallelism": "single host thread"},
           "cpu_baseline": {"value": round(value, 3), "unit": "GB/s", "cores": 1, "kind": "oracle",
                            "sample": f"{desc}, single thread, gcc -O2, {cpu_model()}"},
           "e2e": {"value": round(value, 3), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(res))


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=4000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", type=workload_arg, default="moe_step",
                    help=f"one of {sorted(WORKLOADS)}, k_sweep (all 70 points of the K-groups sweep) "
                         "or k_sweep_<M>x<TotalK> (one point)")
    ap.add_argument("--op", choices=["rearrange", "inverse"], default="rearrange",
                    help="rearrange (row-major -> blocked, the hot path) or its inverse")
    ap.add_argument("--path", choices=["auto", "tma", "flat", "word", "byte"], default="auto",
                    help="force one kernel path of the rearrange, to measure the others (no e2e, no traffic)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=60)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-copy-ceiling", action="store_true",
                    help="skip timing a same-size device-to-device copy per call")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--call-launches", type=int, default=2000,
                    help="minimum launches in each per-call timing graph (steady-state per-launch duration)")
    args = ap.parse_args(argv)
    args.warmup = max(3, args.warmup)
    args.steps = max(1, args.steps)
    rank, world, local = dist_env()
    if args.impl == "reference":
        run_reference(args, rank, world)
    else:
        run_ours(args, rank, world, local)


if __name__ == "__main__":
    main()
