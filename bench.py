"""Benchmark of the B200 two-state optimizer step (Adam/AdamW, AdEMAMix).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload large_f32|transformer_bf16|small_collection]

One step is one optimizer update of the whole workload: one launch of the
persistent multi-tensor kernel through the C ABI (opt2s_step).  The default
workload is one fp32 tensor of 268,435,456 elements with Adam (28 algorithmic
bytes per element: grad, param, m, v read; param, m, v written), the
large-tensor case whose elements/s and HBM GB/s are the headline.  Its 7.5 GB
per step is far larger than the 126 MB L2, so no L2 flush is needed between
steps.  Gradients rotate through 4 pre-generated synthetic buffers.

Rank 0 prints one JSON line.  With N > 1 (torchrun) every rank steps its own
full-size workload on its own GPU (the update is elementwise, so shards of a
collection need no exchange): weak scaling, value = all ranks' elements per
second over the slowest rank's time.

--impl reference times the CPU oracle (the plain C restatement the tests check
the kernel against) on the host cores, each step a bounded sample of the same
workload; under torchrun only rank 0 runs it.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
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
METRIC = ("optimizer step: elements/s and HBM GB/s (% of B200 peak); "
          "µs per small-tensor step")
FALLBACK_HBM_GBS = 6650.0
BYTES_PER_ELEM = {("adam", "f32"): 28, ("ademamix", "f32"): 36,
                  ("adam", "f16"): 22, ("adam", "bf16"): 22,
                  ("ademamix", "f16"): 30, ("ademamix", "bf16"): 30}


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def workload(name, numel=0):
    from elementwise_optimizer_b200 import synth
    if name == "large_f32" and numel:
        return synth.large_f32(numel)
    return {"large_f32": synth.large_f32, "transformer_bf16": synth.transformer_bf16,
            "small_collection": synth.small_collection, "single_small": synth.single_small}[name]()


def algorithmic_bytes(w):
    return sum(BYTES_PER_ELEM[(w.algo, d)] * n for n, d in zip(w.sizes, w.dtypes))


# ---------------------------------------------------------------------------
# Clock sampling (nvidia-smi) during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu_index = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu_index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._t = threading.Thread(target=self._read, daemon=True)
            self._t.start()
        except Exception:
            self.proc = None
        time.sleep(0.25)
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        rows = []
        for l in self.lines:
            parts = [x.strip() for x in l.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append(dict(sm=float(parts[1]), max=float(parts[2]), power=float(parts[3]),
                                 hw=parts[5], hw_thermal=parts[6], sw_thermal=parts[7],
                                 power_cap=parts[8]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        loaded = [r for r in rows if r["power"] > 200] or rows
        reasons = set()
        for r in loaded:
            for k, name in (("hw", "hw_slowdown"), ("hw_thermal", "hw_thermal_slowdown"),
                            ("sw_thermal", "sw_thermal_slowdown"), ("power_cap", "sw_power_cap")):
                if r[k].lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in loaded),
                "sm_max_mhz": max(r["max"] for r in rows),
                "reasons": sorted(reasons), "samples": len(loaded),
                "power_w_max": max(r["power"] for r in rows)}


# ---------------------------------------------------------------------------
# Our arm
# ---------------------------------------------------------------------------

KERNEL_SOURCES = ("opt2s_kernel.cu", "opt2s_device.cuh", "opt2s_internal.h", "opt2s_api.cpp")


def strip_c_comments(text):
    """C/C++ source without its comments, every run of whitespace made one
    space: what the compiler sees, so that a comment edit does not count as a
    kernel change.  String and character literals are kept as they are."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c in "\"'":
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def kernel_source_sha256():
    """Hash of the sources that define the step kernel and its launch
    configuration (chunk length, block width), comments and whitespace
    aside."""
    h = hashlib.sha256()
    for name in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "elementwise_optimizer_b200", "csrc", name), encoding="utf-8") as f:
            h.update(strip_c_comments(f.read()).encode())
    return h.hexdigest()


def environment():
    """What the numbers were measured on: GPU, driver, CUDA runtime, nvcc,
    torch, the hash of the kernel sources and the command line."""
    import subprocess
    import torch
    env = {"torch": torch.__version__, "cuda_runtime": torch.version.cuda,
           "kernel_sources_sha256": kernel_source_sha256(), "command": " ".join(sys.argv)}
    if torch.cuda.is_available():
        env["gpu"] = torch.cuda.get_device_name()
    try:
        env["driver"] = subprocess.run(
            ["nvidia-smi", "--query-gpu=driver_version", "--format=csv,noheader"],
            capture_output=True, text=True, timeout=20).stdout.split("\n")[0].strip() or None
    except (OSError, subprocess.SubprocessError):
        env["driver"] = None
    try:
        out = subprocess.run(["nvcc", "--version"], capture_output=True, text=True, timeout=20).stdout
        env["nvcc"] = out.strip().splitlines()[-1] if out.strip() else None
    except (OSError, subprocess.SubprocessError):
        env["nvcc"] = None
    return env


def traffic_for(kernel_key, numel, path=None):
    """ncu DRAM bytes (read + written) per launch of `numel` elements, if the
    committed capture is of the kernel sources as they are now (else None).
    The capture is of a small case of the same kernel (16,777,216 elements,
    larger than L2, a few hundred MB on the device); the step moves a fixed
    number of bytes per element, so the figure is scaled by the element
    count."""
    path = path or os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        rec = json.load(open(path)).get(kernel_key)
        if rec and rec.get("kernel_source_sha256") == kernel_source_sha256():
            per_launch = float(rec["dram_bytes_read_per_launch"]) + float(rec["dram_bytes_write_per_launch"])
            return per_launch * numel / float(rec["captured_numel"])
    except Exception:
        pass
    return None


def max_over_ranks(value, device=None):
    """The largest `value` over all ranks of the default process group (the
    slowest rank's time); one all-reduce of a scalar, no data-path traffic."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def make_device_workload(w, device, n_grad_buffers):
    """Allocate param / grads / states for workload w on `device` and fill
    them with seeded synthetic values (made on the device: this is bench
    input, not a parity case)."""
    import torch
    from elementwise_optimizer_b200 import binding as B
    tdt = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}
    gen = torch.Generator(device=device)
    gen.manual_seed(w.seed)
    params, s1, s2 = [], [], []
    grads = [[] for _ in range(n_grad_buffers)]
    for n, d in zip(w.sizes, w.dtypes):
        p = torch.empty(n, dtype=torch.float32, device=device)
        p.normal_(0.0, w.param_std, generator=gen)
        params.append(p.to(tdt[d]))
        del p
        for k in range(n_grad_buffers):
            g = torch.empty(n, dtype=torch.float32, device=device)
            g.normal_(0.0, w.grad_std, generator=gen)
            grads[k].append(g.to(tdt[d]))
            del g
        s1.append(torch.zeros(2 * n if w.algo == "ademamix" else n, device=device))
        s2.append(torch.zeros(n, device=device))
    lists = [B.TensorList.from_tensors(params, grads[k], s1, s2) for k in range(n_grad_buffers)]
    hyper = B.make_hyper(w.algo, skip_zeros=w.skip_zeros, **w.hyper)
    return dict(params=params, grads=grads, s1=s1, s2=s2, lists=lists, hyper=hyper)


def small_collection_us(device, reps=200):
    """µs per step of the 2,000-tensor collection (one launch per step), L2
    flushed before every step by writing and then reading a 256 MB buffer."""
    import torch
    from elementwise_optimizer_b200 import binding as B
    w = workload("small_collection")
    d = make_device_workload(w, device, 1)
    flush = torch.empty(64 << 20, dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream()
    for t in range(1, 6):
        B.opt2s_step(d["lists"][0], d["hyper"], t)
    torch.cuda.synchronize()
    times = []
    launches0 = B.launch_count()
    for t in range(6, 6 + reps):
        # write a buffer larger than L2, then read it back so the dirty lines
        # drain before the timed launch rather than during it
        flush.fill_(float(t))
        flush.sum()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        B.opt2s_step(d["lists"][0], d["hyper"], t)
        b.record(stream)
        times.append((a, b))
    torch.cuda.synchronize()
    us = sorted(a.elapsed_time(b) * 1e3 for a, b in times)
    launches = B.launch_count() - launches0
    q = lambda f: us[min(len(us) - 1, int(f * len(us)))]
    # the protocol's floor: a one-element collection timed the same way (the
    # events, the launch and cold data and instruction caches after the flush)
    one = [torch.zeros(1, device=device) for _ in range(4)]
    tl1 = B.TensorList.from_tensors([one[0]], [one[1]], [one[2]], [one[3]])
    floor = []
    for t in range(1, 6 + reps):
        flush.fill_(float(t))
        flush.sum()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        B.opt2s_step(tl1, d["hyper"], t)
        b.record(stream)
        if t > 5:
            floor.append((a, b))
    torch.cuda.synchronize()
    fl = sorted(a.elapsed_time(b) * 1e3 for a, b in floor)
    return {"workload": w.name, "tensors": len(w.sizes), "numel": w.numel,
            "us_per_step_median": q(0.5), "us_per_step_p10": q(0.1), "us_per_step_p90": q(0.9),
            "launches_per_step": launches / reps, "l2": "flushed before each step (256 MB written, then read)",
            "protocol_floor_us_median": fl[len(fl) // 2],
            "protocol_floor": "a one-element collection, same flush and events"}


def single_small_us(device, reps=200):
    """µs per step of the single 1,024-element fp32 tensor (Adam): per call
    between CUDA events with L2 flushed before each step (as the collection),
    and the device time per launch of 200 steps replayed from a CUDA graph
    (no host dispatch between them)."""
    import torch
    from elementwise_optimizer_b200 import binding as B
    w = workload("single_small")
    d = make_device_workload(w, device, 1)
    flush = torch.empty(64 << 20, dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream()
    for t in range(1, 6):
        B.opt2s_step(d["lists"][0], d["hyper"], t)
    torch.cuda.synchronize()
    times = []
    launches0 = B.launch_count()
    for t in range(6, 6 + reps):
        flush.fill_(float(t))
        flush.sum()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        B.opt2s_step(d["lists"][0], d["hyper"], t)
        b.record(stream)
        times.append((a, b))
    torch.cuda.synchronize()
    launches = B.launch_count() - launches0
    us = sorted(a.elapsed_time(b) * 1e3 for a, b in times)
    plan = B.Plan(d["lists"][0], w.algo)
    plan.step(d["hyper"], 1000)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for _ in range(reps):
            plan.step(d["hyper"], 1000)
    graph.replay()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    graph.replay()
    b.record(stream)
    b.synchronize()
    graph_us = a.elapsed_time(b) * 1e3 / reps
    del graph
    plan.close()
    q = lambda f: us[min(len(us) - 1, int(f * len(us)))]
    nbytes = algorithmic_bytes(w)
    return {"workload": w.name, "numel": w.numel, "us_per_step_median": q(0.5),
            "us_per_step_p10": q(0.1), "us_per_step_p90": q(0.9),
            "device_us_per_launch_graph": graph_us, "launches_per_step": launches / reps,
            "algorithmic_bytes": nbytes,
            "l2": "flushed before each timed step (256 MB written, then read); graph replay: L2 warm",
            "bound": "launch latency (28,672 bytes a step)"}


def transformer_measure(device, steps=10, warmup=3, e2e_steps=3):
    """The 1.2 B-element bf16 AdEMAMix collection (24 layers, 240 tensors):
    ms per step, GB/s and fraction of the HBM peak over `steps` steps (CUDA
    events around each launch), plus the same metric end to end with host
    buffers (pinned grads in, params out, one slice per tensor)."""
    import torch
    from elementwise_optimizer_b200 import binding as B
    w = workload("transformer_bf16")
    d = make_device_workload(w, device, 2)
    stream = torch.cuda.current_stream()
    step = 0
    for _ in range(warmup):
        step += 1
        B.opt2s_step(d["lists"][step % 2], d["hyper"], step)
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
    ev[0].record(stream)
    for k in range(steps):
        step += 1
        B.opt2s_step(d["lists"][step % 2], d["hyper"], step)
        ev[k + 1].record(stream)
    torch.cuda.synchronize()
    per = [ev[k].elapsed_time(ev[k + 1]) for k in range(steps)]
    mean_s = statistics.mean(per) / 1e3
    peak, kind = measured_peak()
    nbytes = algorithmic_bytes(w)
    out = {"workload": w.name, "numel": w.numel, "tensors": len(w.sizes), "algo": w.algo,
           "storage": "bf16", "state": "f32", "steps": steps,
           "ms_per_step": statistics.mean(per), "ms_median": statistics.median(per),
           "elements_per_s": w.numel / mean_s, "hbm_gbs": nbytes / mean_s / 1e9,
           "roofline": {"bound": "hbm", "achieved": nbytes / mean_s / 1e9, "peak": peak,
                        "unit": "GB/s", "frac": nbytes / mean_s / 1e9 / peak,
                        "peak_source": kind, "algorithmic_bytes_per_launch": nbytes,
                        "bytes_per_element": nbytes / w.numel},
           "l2": f"inputs larger than L2 ({nbytes / 1e9:.1f} GB per step), no flush"}
    if e2e_steps > 0:
        try:
            out["e2e"] = e2e_measure(w, d, device, e2e_steps)
        except Exception as exc:  # reported, not hidden
            out["e2e_error"] = repr(exc)
    del d
    torch.cuda.empty_cache()
    return out


def norm_steps_measure(w, d, steps=20, warmup=3, max_unorm=1.0):
    """The bounded-update-norm step (max_unorm) and, for Adam, the LAMB step on
    the headline's own buffers: ms per step (CUDA events around each step of
    four launches), GB/s and fraction of the HBM peak against the plain step's
    bytes plus one more read of every input."""
    import torch
    from elementwise_optimizer_b200 import binding as B
    peak, kind = measured_peak()
    nbuf = len(d["lists"])
    legs = [("max_unorm", lambda k, t: B.opt2s_step_max_unorm(d["lists"][k % nbuf], d["hyper"], max_unorm, t))]
    if w.algo == "adam":
        legs.append(("lamb", lambda k, t: B.opt2s_step_lamb(d["lists"][k % nbuf], d["hyper"], t)))
    per_elem = algorithmic_bytes(w) / w.numel + {"adam": 16, "ademamix": 20}[w.algo]
    out = {"workload": w.name, "bytes_per_element": per_elem}
    for name, fn in legs:
        # warm-up steps touch every gradient buffer, so each descriptor's plan
        # (with its norm tables) is built before the timed steps
        nwarm = max(warmup, nbuf)
        for t in range(1, nwarm + 1):
            fn(t, t)
        torch.cuda.synchronize()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
        ev[0].record()
        for k in range(steps):
            fn(k, nwarm + 1 + k)
            ev[k + 1].record()
        torch.cuda.synchronize()
        ms = statistics.mean(ev[k].elapsed_time(ev[k + 1]) for k in range(steps))
        gbs = per_elem * w.numel / (ms / 1e3) / 1e9
        out[name] = {"ms_per_step": ms, "launches_per_step": 4,
                     "roofline": {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s",
                                  "frac": gbs / peak, "peak_source": kind}}
    return out


def shard_measure(device, world, rank, numel=268_435_456, steps=10, warmup=3):
    """The ZeRO-style sharded step across the N ranks of the run, over peer
    memory: every rank holds the whole flat fp32 param buffer (the same
    values) and its own gradient, maps the other ranks' buffers with CUDA IPC
    (shard.PeerBuffers), and steps its shard with opt2s_shard_step -- the
    rank-order gradient mean, the update and the param all-gather in one
    kernel, its remote loads and stores crossing NVLink.  Each step sits
    between two barriers; the time is the max over ranks of the CUDA-event
    time between them.  Every rank takes the same collective steps on every
    path: a rank that cannot set up reports it through one all-reduce, and
    then no rank steps.  Its results are checked against the oracle by
    tests/test_shard_ipc_gpu.py (two processes)."""
    import torch
    import torch.distributed as dist
    from elementwise_optimizer_b200 import binding as B
    from elementwise_optimizer_b200 import shard
    peers, err = None, None
    try:
        gen = torch.Generator(device=device)
        gen.manual_seed(0x0E0A0000 + 8)                 # the same params on every rank
        param = torch.empty(numel, device=device)
        param.normal_(0.0, 1.0, generator=gen)
        gen.manual_seed(0x0E0A0000 + 9 + rank)          # each rank its own gradient
        grad = torch.empty(numel, device=device)
        grad.normal_(0.0, 1e-2, generator=gen)
        peers = shard.PeerBuffers(param, grad)
        st = shard.ShardedStep(peers.params, peers.grads, rank, "adam")
        ok = 1
    except Exception as exc:  # reported, not hidden
        err, ok = repr(exc), 0
    flag = torch.tensor([ok], dtype=torch.int32, device=device)
    dist.all_reduce(flag, op=dist.ReduceOp.MIN)
    if int(flag.item()) == 0:
        if peers is not None:
            peers.close()
        return {"error": err or "another rank could not set up its peer mappings"}
    h = B.make_hyper("adam")
    times = []
    for t in range(1, warmup + steps + 1):
        dist.barrier()
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        st.step(h, t)
        b.record()
        torch.cuda.synchronize()
        dist.barrier()
        if t > warmup:
            times.append(a.elapsed_time(b))
    mean_ms = max_over_ranks(statistics.mean(times), device)
    torch.cuda.synchronize()
    dist.barrier()                                      # no rank unmaps while another steps
    peers.close()
    nbytes = (8 * world + 20) * numel
    nvlink_per_rank = 8 * (world - 1) * numel // world  # remote gradient reads + param writes
    return {"workload": f"flat fp32 Adam, {numel} elements sharded over {world} ranks",
            "ms_per_step": mean_ms, "elements_per_s": numel / (mean_ms / 1e3),
            "algorithmic_bytes_per_step": nbytes,
            "gbs_all_ranks": nbytes / (mean_ms / 1e3) / 1e9,
            "nvlink_bytes_per_rank": nvlink_per_rank,
            "nvlink_gbs_per_rank": nvlink_per_rank / (mean_ms / 1e3) / 1e9,
            "path": "CUDA IPC peer mappings; one opt2s_shard_step launch per rank per step "
                    "(plain peer loads and stores, no TMA, no multicast), barriers on both sides",
            "steps": steps}


def e2e_measure(w, d, device, steps, slices=8):
    """Same metric through the public call with host buffers: every step
    copies that step's gradient from pinned host memory to the device, runs
    the optimizer step, and reads the updated param back into pinned host
    memory.  The collection is cut into `slices` element ranges, each stepped
    through its own plan, so that host-to-device copies (one stream),
    steps (the compute stream) and device-to-host copies (a third stream)
    overlap: slice i+1 arrives while slice i is stepped and slice i-1 leaves."""
    import torch
    from elementwise_optimizer_b200 import binding as B
    params, grads, s1, s2 = d["params"], d["grads"][0], d["s1"], d["s2"]
    ranges = []                      # (tensor index, start, length) per slice
    for i, p in enumerate(params):
        n = p.numel()
        # AdEMAMix keeps [m1 | m2] per tensor: a slice is then a whole tensor
        k = 1 if w.algo == "ademamix" else max(1, min(slices, n // (1 << 20)))
        bounds = [n * j // k for j in range(k + 1)]
        ranges += [(i, bounds[j], bounds[j + 1] - bounds[j]) for j in range(k)]
    host_g = [g.cpu().pin_memory() for g in grads]
    host_p = [torch.empty(p.shape, dtype=p.dtype, pin_memory=True) for p in params]
    lists = []
    for i, a, n in ranges:
        n1 = s1[i].numel() // params[i].numel()      # 1 (Adam) or 2 (AdEMAMix: whole tensor)
        lists.append(B.TensorList.from_tensors([params[i][a:a + n]], [grads[i][a:a + n]],
                                               [s1[i][n1 * a:n1 * (a + n)]], [s2[i][a:a + n]]))
    plans = [B.Plan(tl, w.algo) for tl in lists]     # one explicit plan per slice
    compute = torch.cuda.current_stream()
    h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()
    h2d_bytes = sum(g.numel() * g.element_size() for g in host_g)
    d2h_bytes = sum(p.numel() * p.element_size() for p in host_p)

    prev_done = [None] * len(ranges)

    def one(t):
        arrived = []
        for k, (i, a, n) in enumerate(ranges):
            if prev_done[k] is not None:     # the previous step has used this slice's grad
                h2d.wait_event(prev_done[k])
            with torch.cuda.stream(h2d):
                grads[i][a:a + n].copy_(host_g[i][a:a + n], non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(h2d)
            arrived.append(ev)
        for k, (i, a, n) in enumerate(ranges):
            compute.wait_event(arrived[k])
            plans[k].step(d["hyper"], t, stream=compute)
            done = torch.cuda.Event()
            done.record(compute)
            prev_done[k] = done
            d2h.wait_event(done)
            with torch.cuda.stream(d2h):
                host_p[i][a:a + n].copy_(params[i][a:a + n], non_blocking=True)
        fin = torch.cuda.Event()
        fin.record(d2h)
        compute.wait_event(fin)          # the step ends when its result is on the host

    t0 = 1000
    for k in range(2):
        one(t0 + k)
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(compute)
    h2d.wait_stream(compute)
    for k in range(steps):
        one(t0 + 2 + k)
    b.record(compute)
    b.synchronize()
    sec = a.elapsed_time(b) / 1e3
    return {"value": w.numel * steps / sec, "unit": "elements/s", "h2d_bytes_per_step": h2d_bytes,
            "d2h_bytes_per_step": d2h_bytes, "steps": steps, "ms_per_step": sec * 1e3 / steps,
            "slices": len(ranges),
            "path": "pinned host grad -> device (stream 1), opt2s_plan_step per slice (stream 2), "
                    "device param -> pinned host (stream 3), slices overlapped"}


def run_ours(args, rank, world, local_rank):
    import torch
    from elementwise_optimizer_b200 import _build
    from elementwise_optimizer_b200 import binding as B
    if rank == 0 or not os.path.exists(B.LIB_PATH):
        _build.build()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    w = workload(args.workload, args.numel)
    d = make_device_workload(w, device, 4)
    stream = torch.cuda.current_stream()
    nbuf = len(d["lists"])

    step = 0
    for _ in range(args.warmup):
        step += 1
        B.opt2s_step(d["lists"][step % nbuf], d["hyper"], step)
    torch.cuda.synchronize()

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
        torch.cuda.synchronize()

    events = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    launches0 = B.launch_count()
    with ClockSampler(local_rank) as clocks:
        barrier()
        events[0].record(stream)
        for k in range(args.steps):
            step += 1
            B.opt2s_step(d["lists"][step % nbuf], d["hyper"], step)
            events[k + 1].record(stream)
        barrier()
    launches = B.launch_count() - launches0
    per_launch_ms = [events[k].elapsed_time(events[k + 1]) for k in range(args.steps)]
    total_ms = events[0].elapsed_time(events[-1])
    if world > 1:
        total_ms = max_over_ranks(total_ms, device)

    extras = {}
    if rank == 0 and world == 1 and not args.no_extras:
        extras["small_collection"] = small_collection_us(device)
        extras["single_small"] = single_small_us(device)
    if not args.no_extras:
        # every rank streams its own host buffers; the line reports all ranks'
        # elements over the slowest rank's time.  A rank whose leg fails still
        # joins the reduction (with an infinite time), so no rank waits forever.
        try:
            e2e = e2e_measure(w, d, device, args.e2e_steps)
            e2e_ms = e2e["ms_per_step"]
        except Exception as exc:  # reported, not hidden
            log(f"rank {rank}: e2e leg failed: {exc!r}")
            e2e, e2e_ms = None, float("inf")
        if world > 1:
            e2e_ms = max_over_ranks(e2e_ms, device)
        if e2e is not None and e2e_ms != float("inf"):
            e2e["ms_per_step"] = e2e_ms
            e2e["value"] = w.numel * world / (e2e_ms / 1e3)
            e2e["n_gpus"] = world
            extras["e2e"] = e2e
    if world > 1 and not args.no_extras:
        # every rank runs it (same collective steps); rank 0 reports it
        del d
        torch.cuda.empty_cache()
        d = None
        extras["shard"] = shard_measure(device, world, rank)
    if rank == 0 and world == 1 and not args.no_extras and args.workload == "large_f32":
        # the bounded-norm and LAMB steps on the same buffers, then the largest
        # configuration after the headline's buffers are freed (1.2 B
        # elements, 21.7 GB with two gradient buffers), then the 8-bit-state
        # step (268 M fp32 Adam, 16 B/element) and its mixed collection
        extras["norm_steps"] = norm_steps_measure(w, d)
        del d
        torch.cuda.empty_cache()
        extras["transformer_bf16"] = transformer_measure(device)
        torch.cuda.empty_cache()
        extras["eightbit"] = run_eightbit(steps=20, warmup=5, algos=(("adam", "f32"),), skip_zeros=False)
        extras["eightbit"].pop("env", None)
    cpu = None
    if rank == 0 and world == 1 and not args.no_extras:
        cpu = cpu_baseline(w, args.cpu_seconds)

    if rank != 0:
        return None
    sec = total_ms / 1e3
    elems = w.numel * args.steps * world
    algo_bytes = algorithmic_bytes(w)
    mean_launch_s = statistics.mean(per_launch_ms) / 1e3
    peak, peak_kind = measured_peak()
    achieved = algo_bytes / mean_launch_s / 1e9
    kernel_key = f"step_kernel/{'+'.join(sorted(set(w.dtypes)))}_{w.algo}"
    traffic = traffic_for(kernel_key, w.numel)
    dtype = sorted(set(w.dtypes))
    line = {
        "metric": METRIC,
        "value": elems / sec,
        "unit": "elements/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": total_ms / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32" if dtype == ["f32"] else f"{'+'.join(dtype)} storage, f32 math",
        "data": "synthetic",
        "config": {"workload": w.name, "numel_per_gpu": w.numel, "tensors": len(w.sizes),
                   "algo": w.algo, "storage": dtype, "state": "f32",
                   "bytes_per_element": algo_bytes / w.numel,
                   "l2": f"inputs larger than L2 ({algo_bytes / 1e9:.2f} GB per step), no flush",
                   "grad_buffers": nbuf,
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "hbm_gbs": algo_bytes * args.steps * world / sec / 1e9 / world,
        "hbm_frac_of_peak": algo_bytes * args.steps / sec / 1e9 / peak,
        "launch_ms": {"median": statistics.median(per_launch_ms),
                      "p10": float(np.percentile(per_launch_ms, 10)),
                      "p90": float(np.percentile(per_launch_ms, 90)),
                      "mean": statistics.mean(per_launch_ms)},
        "clocks": clocks.summary(),
        "gpu_launches": launches,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "traffic_source": ("ncu dram__bytes_read.sum + dram__bytes_write.sum of a "
                                        "16,777,216-element launch of the same kernel sources, scaled by "
                                        "elements (profiles/dram_traffic.json)") if traffic else None,
                     "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured" else "fallback 6.65 TB/s",
                     "kernel": "opt2s step_kernel", "algorithmic_bytes_per_launch": algo_bytes},
    }
    if "e2e" in extras:
        line["e2e"] = extras.pop("e2e")
    line.update(extras)
    line["env"] = environment()
    if cpu is not None:
        line["cpu_baseline"] = cpu
    return line


# ---------------------------------------------------------------------------
# The oracle on the host cores (cpu_baseline leg and --impl reference)
# ---------------------------------------------------------------------------

def _oracle_sample(w, n_sample):
    """A bounded sample of the workload's first tensor, as host arrays."""
    from elementwise_optimizer_b200 import synth
    d = w.dtypes[0]
    p = synth.to_storage(synth.normal(w.seed, (11,), n_sample, w.param_std), d)
    g = synth.to_storage(synth.normal(w.seed, (12,), n_sample, w.grad_std), d)
    s1 = np.zeros(2 * n_sample if w.algo == "ademamix" else n_sample, np.float32)
    s2 = np.zeros(n_sample, np.float32)
    return d, p, g, s1, s2


def _oracle_parallel_step(w, arrays, step, cores, pool):
    import oracle
    d, p, g, s1, s2 = arrays
    n = p.size
    bounds = np.linspace(0, n, cores + 1).astype(np.int64)

    def part(k):
        lo, hi = int(bounds[k]), int(bounds[k + 1])
        if hi <= lo:
            return
        if w.algo == "ademamix":
            # the oracle wants [m1 | m2] of its own slice contiguous
            s1k = np.concatenate([s1[lo:hi], s1[n + lo:n + hi]])
        else:
            s1k = s1[lo:hi]
        pk = p[lo:hi]
        s2k = s2[lo:hi]
        oracle.step_f32(pk, g[lo:hi], s1k, s2k, dtype=d, algo=w.algo, step=step,
                        skip_zeros=w.skip_zeros, **w.hyper)
        if w.algo == "ademamix":
            s1[lo:hi] = s1k[:hi - lo]
            s1[n + lo:n + hi] = s1k[hi - lo:]

    if pool is None:
        for k in range(cores):
            part(k)
    else:
        list(pool.map(part, range(cores)))


def cpu_baseline(w, seconds):
    """The oracle as it stands, on all host cores (one single-threaded oracle
    call per core on disjoint slices), on a bounded sample of the workload."""
    import oracle
    oracle.build()
    cores = os.cpu_count() or 1
    n_sample = 1 << 24
    arrays = _oracle_sample(w, n_sample)
    steps = 0
    with cf.ThreadPoolExecutor(max_workers=cores) as pool:
        _oracle_parallel_step(w, arrays, 1, cores, pool)           # warm-up
        t0 = time.perf_counter()
        while True:
            steps += 1
            _oracle_parallel_step(w, arrays, 1 + steps, cores, pool)
            el = time.perf_counter() - t0
            if el >= seconds:
                break
    # the same oracle on one core, on the first 1/cores of the sample, for about
    # a fifth of the time: the single-threaded figure beside the all-core one
    one = _oracle_sample(w, max(1, n_sample // cores))
    steps1 = 0
    t1 = time.perf_counter()
    while True:
        steps1 += 1
        _oracle_parallel_step(w, one, 1 + steps1, 1, None)
        el1 = time.perf_counter() - t1
        if el1 >= seconds / 5:
            break
    n1 = max(1, n_sample // cores)
    return {"value": n_sample * steps / el, "unit": "elements/s", "cores": cores,
            "kind": "oracle",
            "single_thread_value": n1 * steps1 / el1,
            "sample": f"first {n_sample} elements of {w.name}, {steps} steps, "
                      f"{el:.1f} s, {cores} threads x single-threaded oracle on disjoint slices; "
                      f"single_thread_value: the first {n1} elements on one thread, {steps1} steps, "
                      f"{el1:.1f} s"}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    import oracle
    oracle.build()
    w = workload(args.workload, args.numel)
    cores = os.cpu_count() or 1
    n_sample = 1 << 22
    arrays = _oracle_sample(w, n_sample)
    with cf.ThreadPoolExecutor(max_workers=cores) as pool:
        step = 0
        for _ in range(args.warmup):
            step += 1
            _oracle_parallel_step(w, arrays, step, cores, pool)
        t0 = time.perf_counter()
        for _ in range(args.steps):
            step += 1
            _oracle_parallel_step(w, arrays, step, cores, pool)
        sec = time.perf_counter() - t0
    value = n_sample * args.steps / sec
    sample = (f"each step: oracle over the first {n_sample} elements of {w.name} "
              f"on {cores} threads (disjoint slices)")
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "elements/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": sec * 1e3 / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": w.name, "numel_per_gpu": w.numel, "algo": w.algo,
                   "sample_elements_per_step": n_sample},
        "cpu_baseline": {"value": value, "unit": "elements/s", "cores": cores,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "elements/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


# ---------------------------------------------------------------------------
# Protocol of the bitsandbytes issue "Investigate a 256-thread SM103 path for
# small 32-bit optimizer tensors" (section "B300 benchmark and acceptance"):
# preallocated direct cells and eager collections, >= 20 warm-ups, 7
# interleaved rounds, medians with p10/p90.
# ---------------------------------------------------------------------------

CELL_SIZES = [1, 32, 64, 128, 256, 512, 768, 1023, 1024, 1025, 2048, 4096]


def _pct(xs, q):
    xs = sorted(xs)
    return xs[min(len(xs) - 1, int(q * len(xs)))]


def run_direct_cells(rounds=7, samples=200, warmup=20):
    """One tensor per call (opt2s_step), every (algo, dtype, n) cell; device
    time per call from CUDA events, host dispatch time from the wall clock of
    back-to-back calls.  torch.optim.AdamW(fused=True) on the same tensor is
    timed alongside for context."""
    import torch
    from elementwise_optimizer_b200 import binding as B
    dev = torch.device("cuda")
    tdt = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}
    cells = []
    for algo in ("adam", "ademamix"):
        for dt in ("f16", "bf16", "f32"):
            for n in CELL_SIZES:
                p = torch.randn(n, device=dev).to(tdt[dt])
                g = (torch.randn(n, device=dev) * 1e-2).to(tdt[dt])
                s1 = torch.zeros(2 * n if algo == "ademamix" else n, device=dev)
                s2 = torch.zeros(n, device=dev)
                h = B.make_hyper(algo, lr=1e-3, weight_decay=0.01, beta3=0.9999, alpha=5.0)
                tl = B.TensorList.from_tensors([p], [g], [s1], [s2])
                ref = None
                if algo == "adam":
                    rp = torch.nn.Parameter(p.clone())
                    rp.grad = g.clone()
                    ref = torch.optim.AdamW([rp], lr=1e-3, weight_decay=0.01, fused=True)
                cells.append(dict(algo=algo, dtype=dt, n=n, tl=tl, h=h, ref=ref, step=0,
                                  dev=[], host=[], torch_dev=[], graph=[],
                                  plan=B.Plan(tl, algo)))
    stream = torch.cuda.current_stream()
    for c in cells:
        for _ in range(warmup):
            c["step"] += 1
            B.opt2s_step(c["tl"], c["h"], c["step"])
            if c["ref"] is not None:
                c["ref"].step()
    torch.cuda.synchronize()
    for _ in range(rounds):
        for c in cells:                       # interleaved: every cell once per round
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(samples + 1)]
            ev[0].record(stream)
            for k in range(samples):
                c["step"] += 1
                B.opt2s_step(c["tl"], c["h"], c["step"])
                ev[k + 1].record(stream)
            torch.cuda.synchronize()
            c["dev"] += [ev[k].elapsed_time(ev[k + 1]) * 1e3 for k in range(samples)]
            t0 = time.perf_counter()
            for k in range(samples):
                c["step"] += 1
                B.opt2s_step(c["tl"], c["h"], c["step"])
            t1 = time.perf_counter()
            torch.cuda.synchronize()
            c["host"].append((t1 - t0) / samples * 1e6)
            if c["ref"] is not None:
                ev = [torch.cuda.Event(enable_timing=True) for _ in range(samples + 1)]
                ev[0].record(stream)
                for k in range(samples):
                    c["ref"].step()
                    ev[k + 1].record(stream)
                torch.cuda.synchronize()
                c["torch_dev"] += [ev[k].elapsed_time(ev[k + 1]) * 1e3 for k in range(samples)]
    # device-bound time per launch: 200 launches captured in a CUDA graph and
    # replayed (no host dispatch between them)
    for c in cells:
        graph = torch.cuda.CUDAGraph()
        c["plan"].step(c["h"], c["step"] + 1)
        torch.cuda.synchronize()
        with torch.cuda.graph(graph):
            for _ in range(samples):
                c["plan"].step(c["h"], c["step"] + 1)
        for _ in range(rounds):
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            graph.replay()
            b.record(stream)
            b.synchronize()
            c["graph"].append(a.elapsed_time(b) * 1e3 / samples)
        del graph
    out = []
    for c in cells:
        row = {"algo": c["algo"], "dtype": c["dtype"], "n": c["n"],
               "device_us_per_launch_graph": _pct(c["graph"], 0.5),
               "us_median": _pct(c["dev"], 0.5), "us_p10": _pct(c["dev"], 0.1),
               "us_p90": _pct(c["dev"], 0.9), "host_dispatch_us_median": _pct(c["host"], 0.5)}
        if c["torch_dev"]:
            row["torch_fused_adamw_us_median"] = _pct(c["torch_dev"], 0.5)
        out.append(row)
    return {"mode": "direct-cells", "rounds": rounds, "samples_per_round": samples,
            "warmup": warmup, "cells": out,
            "note": "us_*: time per call between CUDA events around back-to-back opt2s_step "
                    "calls from Python (bounded by host dispatch for small n); "
                    "host_dispatch_us: wall time per call (ctypes included); "
                    "device_us_per_launch_graph: 200 launches replayed from a CUDA graph"}


def run_eager_collection(rounds=7, steps=50, warmup=20):
    """optimizer.step() on a fixed collection: the 2,000 bias/norm/LoRA-like
    tensors (64..1,024 elements, fp32/bf16/fp16) plus 64 tensors of 4,096..
    65,536 elements (the ones the 8-bit classes keep in 8-bit state).  Wall
    time per step (host dispatch included, GPU drained at the end of each
    batch); a captured CUDA graph of the same step as a diagnostic control;
    torch.optim.AdamW(fused=True) for context."""
    import torch
    from elementwise_optimizer_b200 import optim, synth
    dev = torch.device("cuda")
    tdt = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}
    w = synth.small_collection()
    sizes = list(w.sizes) + [4096 * (1 << (i % 5)) for i in range(64)]
    dtypes = list(w.dtypes) + [("f32", "bf16", "f16")[i % 3] for i in range(64)]
    gen = torch.Generator(device=dev).manual_seed(1)

    def make():
        ps = []
        for n, d in zip(sizes, dtypes):
            p = torch.nn.Parameter(torch.randn(n, device=dev, generator=gen).to(tdt[d]))
            p.grad = (torch.randn(n, device=dev, generator=gen) * 1e-2).to(tdt[d])
            ps.append(p)
        return ps

    def timed(step_fn):
        for _ in range(warmup):
            step_fn()
        torch.cuda.synchronize()
        per = []
        for _ in range(rounds):
            t0 = time.perf_counter()
            for _ in range(steps):
                step_fn()
            torch.cuda.synchronize()
            per.append((time.perf_counter() - t0) / steps * 1e6)
        return {"us_per_step_median": _pct(per, 0.5), "us_p10": _pct(per, 0.1), "us_p90": _pct(per, 0.9)}

    res = {"mode": "eager-collection", "tensors": len(sizes), "numel": int(sum(sizes)),
           "rounds": rounds, "steps_per_round": steps}
    for name, cls, kw in (("AdamW32bit", optim.AdamW32bit, {}),
                          ("AdEMAMix32bit", optim.AdEMAMix32bit, {}),
                          ("AdamW8bit", optim.AdamW8bit, {}),
                          ("AdEMAMix8bit", optim.AdEMAMix8bit, {}),
                          ("AdamW32bit_flatten", optim.AdamW32bit, dict(flatten=True)),
                          ("AdEMAMix32bit_flatten", optim.AdEMAMix32bit, dict(flatten=True))):
        res[name] = timed(cls(make(), lr=1e-4, **kw).step)
    # graph-compatible control: the AdamW32bit step captured once, replayed
    opt = optim.AdamW32bit(make(), lr=1e-4, capturable=True, table_len=4096)
    opt.step()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        opt.step()
    res["AdamW32bit_graph_replay"] = timed(graph.replay)
    del graph
    ref = torch.optim.AdamW(make(), lr=1e-4, fused=True)
    res["torch_AdamW_fused_context"] = timed(ref.step)
    return res


def run_shard_emulated(numel=268_435_456, worlds=(1, 2, 4, 8), steps=20, warmup=5):
    """The fused sharded step with `world` emulated ranks on one GPU: every
    rank's param and grad buffer lives on this device, and one step is the
    world ranks' launches one after another.  Per element of the collection
    the step reads world gradients, the param and the fp32 state, and writes
    world params and the state: (8*world + 20) bytes for fp32 Adam.  On a real
    node the (world-1)/world remote share of those bytes crosses NVLink."""
    import torch
    from elementwise_optimizer_b200 import binding as B
    from elementwise_optimizer_b200 import shard
    dev = torch.device("cuda")
    peak, _ = measured_peak()
    res = {"mode": "shard-emulated", "numel": numel, "algo": "adam", "dtype": "f32", "rows": []}
    h = B.make_hyper("adam")
    for world in worlds:
        params = [torch.randn(numel, device=dev) for _ in range(world)]
        grads = [torch.randn(numel, device=dev) * 1e-2 for _ in range(world)]
        steppers = [shard.ShardedStep(params, grads, r, "adam") for r in range(world)]
        t = 0
        for _ in range(warmup):
            t += 1
            for st in steppers:
                st.step(h, t)
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(steps):
            t += 1
            for st in steppers:
                st.step(h, t)
        b.record()
        b.synchronize()
        ms = a.elapsed_time(b) / steps
        nbytes = (8 * world + 20) * numel
        res["rows"].append({"world": world, "ms_per_step": ms, "algorithmic_bytes": nbytes,
                            "gbs": nbytes / (ms / 1e3) / 1e9,
                            "frac_of_hbm_peak": nbytes / (ms / 1e3) / 1e9 / peak})
        del params, grads, steppers
        torch.cuda.empty_cache()
    return res


def run_roofline_table(numel=268_435_456, steps=50, warmup=10):
    """Every kernel variant on one tensor of `numel` elements: Adam and
    AdEMAMix, fp32/bf16/fp16 storage, with and without skip_zeros (grads
    without zeros, so both do the same work).  Algorithmic bytes per launch /
    mean launch time (CUDA events) against the measured HBM peak."""
    import torch
    from elementwise_optimizer_b200 import binding as B
    dev = torch.device("cuda")
    peak, kind = measured_peak()
    tdt = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}
    rows = []
    for algo in ("adam", "ademamix"):
        for dt in ("f32", "bf16", "f16"):
            for skip in (False, True):
                if skip and dt != "f32":
                    continue
                p = torch.randn(numel, device=dev).to(tdt[dt])
                grads = [(torch.randn(numel, device=dev) * 1e-2).to(tdt[dt]) for _ in range(2)]
                s1 = torch.zeros(2 * numel if algo == "ademamix" else numel, device=dev)
                s2 = torch.zeros(numel, device=dev)
                plans = [B.Plan(B.TensorList.from_tensors([p], [g], [s1], [s2]), algo) for g in grads]
                h = B.make_hyper(algo, weight_decay=0.01, beta3=0.9999, alpha=5.0, skip_zeros=skip)
                for t in range(1, warmup + 1):
                    plans[t % 2].step(h, t)
                torch.cuda.synchronize()
                ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
                ev[0].record()
                for k in range(steps):
                    plans[k % 2].step(h, warmup + 1 + k)
                    ev[k + 1].record()
                torch.cuda.synchronize()
                ms = [ev[k].elapsed_time(ev[k + 1]) for k in range(steps)]
                mean = sum(ms) / len(ms)
                nbytes = BYTES_PER_ELEM[(algo, dt)] * numel
                rows.append({"algo": algo, "dtype": dt, "skip_zeros": skip,
                             "bytes_per_elem": BYTES_PER_ELEM[(algo, dt)], "ms_mean": mean,
                             "gbs": nbytes / (mean / 1e3) / 1e9,
                             "frac": nbytes / (mean / 1e3) / 1e9 / peak})
                for x in plans:
                    x.close()
                del p, grads, s1, s2, plans
                torch.cuda.empty_cache()
    return {"mode": "roofline-table", "numel": numel, "peak_gbs": peak, "peak_source": kind,
            "rows": rows}


def run_max_unorm(numel=268_435_456, steps=50, warmup=10, max_unorm=1.0):
    """The bounded-update-norm step (opt2s_step_max_unorm: norm sums, scales,
    scaled update) on one tensor of `numel` elements, timed beside the plain
    step on the same buffers, and for Adam the LAMB step (opt2s_step_lamb, the
    same four launches).  Their algorithmic bytes are the plain step's plus
    one more read of every input (the norm pass reads g, p, m, v [, m2] and
    writes nothing)."""
    import torch
    from elementwise_optimizer_b200 import binding as B
    dev = torch.device("cuda")
    peak, kind = measured_peak()
    tdt = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}
    read_bytes = {("adam", "f32"): 16, ("ademamix", "f32"): 20,
                  ("adam", "bf16"): 12, ("ademamix", "bf16"): 16}
    rows = []
    for algo, dt in (("adam", "f32"), ("ademamix", "bf16")):
        p = torch.randn(numel, device=dev).to(tdt[dt])
        grads = [(torch.randn(numel, device=dev) * 1e-2).to(tdt[dt]) for _ in range(2)]
        s1 = torch.zeros(2 * numel if algo == "ademamix" else numel, device=dev)
        s2 = torch.zeros(numel, device=dev)
        lists = [B.TensorList.from_tensors([p], [g], [s1], [s2]) for g in grads]
        h = B.make_hyper(algo, weight_decay=0.01, beta3=0.9999, alpha=5.0)
        row = {"algo": algo, "dtype": dt, "max_unorm": max_unorm}
        legs = [("plain", lambda k, t: B.opt2s_step(lists[k % 2], h, t)),
                ("max_unorm", lambda k, t: B.opt2s_step_max_unorm(lists[k % 2], h, max_unorm, t))]
        if algo == "adam":
            legs.append(("lamb", lambda k, t: B.opt2s_step_lamb(lists[k % 2], h, t)))
        for name, fn in legs:
            for t in range(1, warmup + 1):
                fn(t, t)
            torch.cuda.synchronize()
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
            ev[0].record()
            for k in range(steps):
                fn(k, warmup + 1 + k)
                ev[k + 1].record()
            torch.cuda.synchronize()
            ms = sum(ev[k].elapsed_time(ev[k + 1]) for k in range(steps)) / steps
            per_elem = BYTES_PER_ELEM[(algo, dt)] + (read_bytes[(algo, dt)] if name != "plain" else 0)
            gbs = per_elem * numel / (ms / 1e3) / 1e9
            row[name] = {"ms_mean": ms, "bytes_per_elem": per_elem, "gbs": gbs, "frac": gbs / peak}
        row["time_ratio"] = row["max_unorm"]["ms_mean"] / row["plain"]["ms_mean"]
        row["byte_ratio"] = row["max_unorm"]["bytes_per_elem"] / row["plain"]["bytes_per_elem"]
        rows.append(row)
        del p, grads, s1, s2, lists
        B.opt2s_release_cache()
        torch.cuda.empty_cache()
    return {"mode": "max-unorm", "numel": numel, "peak_gbs": peak, "peak_source": kind,
            "rows": rows}


def eightbit_bytes_per_elem(algo, dt):
    """Algorithmic bytes per element of the 8-bit-state step: param and grad
    in their storage type, one byte per state quantity per element read and
    written, and each 2,048-element block's fp32 absmax per quantity read and
    written (8 bytes per quantity per block)."""
    es = 4 if dt == "f32" else 2
    q = 3 if algo == "ademamix" else 2
    return 3 * es + 2 * q + 8 * q / 2048


def run_eightbit(numel=268_435_456, steps=50, warmup=10, algos=(("adam", "f32"), ("ademamix", "bf16")),
                 skip_zeros=True):
    """The 8-bit blockwise-state step (opt2s_step_8bit) on one tensor of
    `numel` elements (by default fp32 Adam and bf16 AdEMAMix), timed beside
    the 32-bit step on the same param/grad, and with skip_zeros (a third
    gradient buffer with every seventh element zero) when `skip_zeros`; and
    the mixed AdamW collection of the eager protocol (2,000 tensors of
    64..1,024 elements with fp32 state plus 64 tensors of 4,096..65,536
    elements with 8-bit state) in one launch, L2 flushed before each step."""
    import torch
    from elementwise_optimizer_b200 import binding as B
    from elementwise_optimizer_b200 import synth
    dev = torch.device("cuda")
    peak, kind = measured_peak()
    tdt = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}
    rows = []
    for algo, dt in algos:
        two = algo == "ademamix"
        nb = (numel + 2047) // 2048
        p = torch.randn(numel, device=dev).to(tdt[dt])
        grads = [(torch.randn(numel, device=dev) * 1e-2).to(tdt[dt]) for _ in range(2)]
        q1 = torch.zeros((2 if two else 1) * numel, dtype=torch.uint8, device=dev)
        q2 = torch.zeros(numel, dtype=torch.uint8, device=dev)
        a1 = torch.zeros((2 if two else 1) * nb, device=dev)
        a2 = torch.zeros(nb, device=dev)
        lists = [B.TensorList8.from_tensors([p], [g], [q1], [q2], [a1], [a2]) for g in grads]
        h = B.make_hyper(algo, weight_decay=0.01, beta3=0.9999, alpha=5.0)
        row = {"algo": algo, "dtype": dt, "state": "8-bit blockwise"}
        ms = []
        for t in range(1, warmup + 1):
            B.opt2s_step_8bit(lists[t % 2], h, t)
        torch.cuda.synchronize()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
        ev[0].record()
        for k in range(steps):
            B.opt2s_step_8bit(lists[k % 2], h, warmup + 1 + k)
            ev[k + 1].record()
        torch.cuda.synchronize()
        ms = sum(ev[k].elapsed_time(ev[k + 1]) for k in range(steps)) / steps
        per = eightbit_bytes_per_elem(algo, dt)
        gbs = per * numel / (ms / 1e3) / 1e9
        row["eightbit"] = {"ms_mean": ms, "bytes_per_elem": per, "gbs": gbs, "frac": gbs / peak,
                           "elements_per_s": numel / (ms / 1e3)}
        if skip_zeros:
            gz = grads[0].clone()
            gz[::7] = 0
            lz = [lists[0], B.TensorList8.from_tensors([p], [gz], [q1], [q2], [a1], [a2])]
            hz = B.make_hyper(algo, weight_decay=0.01, beta3=0.9999, alpha=5.0, skip_zeros=True)
            t0 = warmup + steps
            for t in range(1, warmup + 1):
                B.opt2s_step_8bit(lz[t % 2], hz, t0 + t)
            torch.cuda.synchronize()
            ev[0].record()
            for k in range(steps):
                B.opt2s_step_8bit(lz[k % 2], hz, t0 + warmup + 1 + k)
                ev[k + 1].record()
            torch.cuda.synchronize()
            msz = sum(ev[k].elapsed_time(ev[k + 1]) for k in range(steps)) / steps
            row["eightbit_skip_zeros"] = {"ms_mean": msz, "grads": "alternately dense and every seventh zero"}
            del gz, lz
        del q1, q2, a1, a2, lists
        s1 = torch.zeros((2 if two else 1) * numel, device=dev)
        s2 = torch.zeros(numel, device=dev)
        plain = [B.TensorList.from_tensors([p], [g], [s1], [s2]) for g in grads]
        for t in range(1, warmup + 1):
            B.opt2s_step(plain[t % 2], h, t)
        torch.cuda.synchronize()
        ev[0].record()
        for k in range(steps):
            B.opt2s_step(plain[k % 2], h, warmup + 1 + k)
            ev[k + 1].record()
        torch.cuda.synchronize()
        ms32 = sum(ev[k].elapsed_time(ev[k + 1]) for k in range(steps)) / steps
        row["fp32_state"] = {"ms_mean": ms32, "bytes_per_elem": BYTES_PER_ELEM[(algo, dt)],
                             "frac": BYTES_PER_ELEM[(algo, dt)] * numel / (ms32 / 1e3) / 1e9 / peak}
        row["time_ratio_8_over_32"] = ms / ms32
        rows.append(row)
        del p, grads, s1, s2, plain
        B.opt2s_release_cache()
        torch.cuda.empty_cache()
    # the mixed collection
    w = synth.small_collection()
    sizes = list(w.sizes) + [4096 * (1 << (i % 5)) for i in range(64)]
    dtypes = list(w.dtypes) + [("f32", "bf16", "f16")[i % 3] for i in range(64)]
    gen = torch.Generator(device=dev).manual_seed(3)
    ps, gs, s1s, s2s, a1s, a2s = [], [], [], [], [], []
    for n, d in zip(sizes, dtypes):
        ps.append(torch.randn(n, device=dev, generator=gen).to(tdt[d]))
        gs.append((torch.randn(n, device=dev, generator=gen) * 1e-2).to(tdt[d]))
        if B.state_bits_for(n) == 8:
            s1s.append(torch.zeros(n, dtype=torch.uint8, device=dev))
            s2s.append(torch.zeros(n, dtype=torch.uint8, device=dev))
            a1s.append(torch.zeros((n + 2047) // 2048, device=dev))
            a2s.append(torch.zeros((n + 2047) // 2048, device=dev))
        else:
            s1s.append(torch.zeros(n, device=dev))
            s2s.append(torch.zeros(n, device=dev))
            a1s.append(None)
            a2s.append(None)
    tl = B.TensorList8.from_tensors(ps, gs, s1s, s2s, a1s, a2s)
    h = B.make_hyper("adam", weight_decay=0.01)
    flush = torch.empty(64 << 20, dtype=torch.float32, device=dev)
    for t in range(1, 6):
        B.opt2s_step_8bit(tl, h, t)
    torch.cuda.synchronize()
    launches0 = B.launch_count()
    times = []
    for t in range(6, 206):
        flush.fill_(float(t))
        flush.sum()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        B.opt2s_step_8bit(tl, h, t)
        b.record()
        times.append((a, b))
    torch.cuda.synchronize()
    us = sorted(a.elapsed_time(b) * 1e3 for a, b in times)
    n8 = sum(n for n in sizes if B.state_bits_for(n) == 8)
    mixed = {"tensors": len(sizes), "numel": int(sum(sizes)), "numel_8bit": int(n8),
             "tensors_8bit": sum(1 for n in sizes if B.state_bits_for(n) == 8),
             "us_median": _pct(us, 0.5), "us_p10": _pct(us, 0.1), "us_p90": _pct(us, 0.9),
             "launches_per_step": (B.launch_count() - launches0) / 200,
             "l2": "flushed before each step (256 MB written, then read)"}
    return {"mode": "eightbit", "numel": numel, "peak_gbs": peak, "peak_source": kind,
            "rows": rows, "mixed_adamw_collection": mixed}


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="large_f32",
                    choices=["large_f32", "transformer_bf16", "small_collection"])
    ap.add_argument("--numel", type=int, default=0,
                    help="size of the large_f32 tensor, and of the tensor of --mode max-unorm and "
                         "--mode roofline-table (default 268,435,456)")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the small-collection, e2e and cpu_baseline legs")
    ap.add_argument("--mode", choices=["headline", "direct-cells", "eager-collection", "max-unorm",
                                       "shard-emulated", "roofline-table", "eightbit"],
                    default="headline",
                    help="headline: the one-line bench; the others follow the issue's "
                         "direct-cell and eager-collection protocol and print their tables")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        log(f"note: WORLD_SIZE={world}, --gpus={args.gpus}; using WORLD_SIZE")

    if args.mode != "headline":
        import torch
        from elementwise_optimizer_b200 import _build
        _build.build()
        torch.cuda.set_device(local_rank)
        sized = {"roofline-table": run_roofline_table, "max-unorm": run_max_unorm,
                 "eightbit": run_eightbit}
        if args.mode in sized and args.numel:
            res = sized[args.mode](numel=args.numel)
        else:
            res = {"direct-cells": run_direct_cells, "eager-collection": run_eager_collection,
                   "shard-emulated": run_shard_emulated, **sized}[args.mode]()
        res["env"] = environment()
        print(json.dumps(res), flush=True)
        return

    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return

    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        line = run_ours(args, rank, world, local_rank)
        if line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
