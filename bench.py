"""Benchmark: FP8 paged decode attention, achieved HBM GB/s and us/step.

One step = the decode hot path for one layer of a synthetic serving batch:
the append of one new token per sequence, then decode attention over the
updated paged E4M3 cache -- by default one ``fp8_paged_decode_append_attention``
launch (append and split combine fused); ``--unfused`` runs ``fp8_kv_append``
and ``fp8_paged_decode_attention`` as two launches. Configs without an append
run the attention call alone. Inputs are resident in HBM when the timed
region starts; L2 is flushed between timed steps, outside each step's events.
``value`` = algorithmic bytes (attended K/V once per KV head + q + the
block-table entries read) / device time, summed over ranks.

The headline workload is the largest single-GPU one (long context, 8
sequences of 131,072 keys). At N = 1 the same JSON line also carries a
``configs`` object with the other serving workloads (Llama-like, gpt-oss-like
full and windowed, the mixed pool with one roofline per layer, long context
B = 1), each timed the same way.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]

With N > 1 every rank runs its own copy of the workload on its GPU
(independent sequences: no data-path collective); time is the max over ranks,
throughput the sum (weak scaling). Started without a launcher, ``--gpus N``
re-runs itself under ``torch.distributed.run`` with N ranks (and refuses when
fewer than N GPUs are visible). ``--impl reference`` times the float64 CPU
oracle on the same workload on every host core (rank 0 only).
"""

from __future__ import annotations

import argparse
import concurrent.futures
import json
import os
import platform
import socket
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "FP8 paged decode attention: achieved HBM GB/s and µs/step on 1 B200"
DEFAULT_CONFIG = "long_b8"
#: the other workloads timed beside the headline (N = 1 only)
SWEEP = ("llama", "gptoss_full", "gptoss_w128", "mixed", "long_b1")
WORKLOAD_TEXT = {
    "llama": "Llama-3-8B-like layer: B=32 Hq=32 Hkv=8 D=128 page=16 seq_len~U[512,4096] "
             "per-(page,head) scales, +1 appended token/seq",
    "tiny": "tiny: B=1 Hq=8 Hkv=2 D=64 page=16 L=256",
    "gptoss_full": "gpt-oss-like: B=64 Hq=64 Hkv=8 D=64 page=16 L=8192 sinks, full attention",
    "gptoss_w128": "gpt-oss-like: B=64 Hq=64 Hkv=8 D=64 page=16 L=8192 sinks, window=128",
    "mixed": "mixed pool: B=16 page=32 L~U[2048,16384]; sliding D=256 W=1024 + full D=512",
    "long_b1": "long context: B=1 Hq=64 Hkv=8 D=128 page=64 L=131072 per-KV-head scales, "
               "+1 appended token",
    "long_b8": "long context: B=8 Hq=64 Hkv=8 D=128 page=64 L=131072 per-KV-head scales, "
               "+1 appended token/seq",
}
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "dram_traffic_per_launch.txt")
KERNEL_NAME = {1: "decode_tma_kernel (split kernel, merge in the same launch)",
               3: "decode_tma_kernel (proportional splits, merge in the same launch)"}
UMMA_NAME = {1: "decode_umma_kernel (tcgen05, TMEM accumulators; split kernel, merge in the same "
                "launch)",
             3: "decode_umma_kernel (tcgen05, TMEM accumulators; proportional splits, merge in "
                "the same launch)"}
L2_TEXT = ("flushed between timed steps: 256 MiB write, then a 256 MiB read of another buffer "
           "(no dirty lines left), outside the step events")


def _peaks() -> dict:
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "source": "fallback"}


def _kernel_source_hash() -> str:
    import hashlib
    h = hashlib.sha256()
    for name in ("fp8pd_kernels.cu", "fp8pd_internal.h"):
        with open(os.path.join(ROOT, "fp8_paged_decode_split_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def _traffic(config: str, layer: int = 0):
    """DRAM bytes (read + write) per attention-kernel launch from the committed
    ncu summary, if it was taken on the current kernel source. Lines of that
    file: ``<workload>[:<layer>] <kernel source hash> <bytes> [how]``."""
    key = config if layer == 0 else f"{config}:{layer}"
    try:
        with open(PROFILE_TRAFFIC) as f:
            for line in f:
                parts = line.split()
                if len(parts) >= 3 and not line.startswith("#") and parts[0] == key \
                        and parts[1] == _kernel_source_hash():
                    return float(parts[2])
    except OSError:
        pass
    return None


class L2Flush:
    """Empties the 126 MB L2 between timed steps: a 256 MiB write, then a read
    of another 256 MiB buffer. The write alone would leave the L2 full of
    dirty lines whose write-back to HBM then lands inside the next timed
    step; after the read every line in the L2 is clean, so the step pays only
    for its own traffic."""

    def __init__(self, device: torch.device):
        self.w = torch.empty(256 << 20, dtype=torch.uint8, device=device)
        self.r = torch.ones(64 << 20, dtype=torch.float32, device=device)
        self.sink = torch.empty((), dtype=torch.float32, device=device)

    def fill_(self, v: int = 1) -> None:
        self.w.fill_(v & 0xFF)
        torch.sum(self.r, dim=0, out=self.sink)


class ClockSampler:
    """nvidia-smi samples during the timed region (SM clock, throttle reasons)."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: torch.device):
        try:
            self.index = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
        except Exception:
            self.index = str(device.index or 0)
        self.proc = None
        self.path = os.path.join(tempfile.gettempdir(), f"fp8pd_clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.f,
                stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def summary(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        try:
            with open(self.path) as f:
                for line in f:
                    parts = [p.strip() for p in line.split(",")]
                    if len(parts) >= 9:
                        rows.append(parts)
            os.remove(self.path)
        except Exception:
            pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


def _dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(values, device) -> list:
    """Element-wise maximum of per-rank timings over the process group (every
    rank gets the same result); the identity without a process group."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def whole_job_gbs(world: int, bytes_per_rank_step: int, ms_per_step: float) -> float:
    """Aggregate throughput of N weak-scaled replicas: every rank processes
    the same bytes per step; the step takes the slowest rank's time."""
    return world * bytes_per_rank_step / (ms_per_step * 1e-3) / 1e9


class Step:
    """One decode step of the workload through the library's public API: with
    an append, the fused call (append and attention in one launch) unless
    `fused` is off, then fp8_kv_append followed by the attention call.
    ``layers`` restricts the step to some layers (per-layer timing)."""

    def __init__(self, F, case: W.Case, fused: bool = True, layers=None):
        self.F = F
        self.case = case
        self.fused = fused and case.spec.append
        self.layers = list(range(len(case.layers))) if layers is None else list(layers)

    def run(self, stream=None):
        F, c = self.F, self.case
        for li in self.layers:
            layer = c.layers[li]
            if self.fused:
                F.fp8_paged_decode_append_attention(
                    layer.q, layer.k_new, layer.v_new, layer.k_pages, layer.v_pages,
                    layer.k_scale, layer.v_scale, layer.block_table, c.positions,
                    window=layer.window, sinks=layer.sinks, sm_scale=layer.sm_scale,
                    out=layer.out, stream=stream)
                continue
            if c.spec.append:
                F.fp8_kv_append(layer.k_new, layer.v_new, layer.k_pages, layer.v_pages,
                                layer.k_scale, layer.v_scale, layer.block_table, c.positions,
                                stream=stream)
            F.fp8_paged_decode_attention(layer.q, layer.k_pages, layer.v_pages, layer.k_scale,
                                         layer.v_scale, layer.block_table, c.attend_lens,
                                         window=layer.window, sinks=layer.sinks,
                                         sm_scale=layer.sm_scale, out=layer.out, stream=stream)


def _step_bytes(case: W.Case) -> int:
    return sum(W.algorithmic_bytes(case, i) for i in range(len(case.layers)))


def _config_dict(args, name: str, case_or_none=None, nbytes=None) -> dict:
    """The ``config`` object of a line: the same keys and values for both arms."""
    spec = W.spec_with(name, **_scale_override(args))
    if nbytes is None:
        # algorithmic bytes depend only on lengths and shapes: a CPU copy of
        # the workload's lengths is enough (no pools are built)
        nbytes = _spec_bytes(spec)
    world = _dist_env()[0]
    return {"workload": _workload_text(args, name), "name": name, "bytes_per_step": int(nbytes),
            "scales": _scales_text(spec),
            "l2": L2_TEXT, "parallelism": f"{world} independent replicas" if world > 1 else "1 GPU"}


def _spec_bytes(spec: W.Spec) -> int:
    """Algorithmic bytes of one step of ``spec`` from its lengths and shapes
    (the same count as workloads.algorithmic_bytes, without building pools)."""
    rng = np.random.default_rng(spec.seed)
    lens = W._lengths(spec, rng) + (1 if spec.append else 0)
    total = 0
    for L in spec.layers:
        for Lb in lens:
            lo = max(0, Lb - L.window) if L.window > 0 else 0
            n = max(0, Lb - lo)
            total += 2 * n * L.Hkv * L.D
            if n > 0:
                total += 4 * ((Lb - 1) // spec.ps - lo // spec.ps + 1)
            if spec.scale_mode == "token":
                total += 4 * n * L.Hkv * (spec.k_groups + 1)
            elif spec.scale_mode == "mx":
                total += 2 * n * L.Hkv * (L.D // 32)
        total += 2 * spec.B * L.Hq * L.D
    return int(total)


def time_case(F, case: W.Case, dev, args, flush: L2Flush, steps: int, warmup: int,
              clocks: bool = False) -> dict:
    """Device time of the workload's step as CUDA-graph replays (per-step
    events, L2 flushed between), then each layer's attention kernel alone from
    an eager pass (the library's events around its launch)."""
    stream = torch.cuda.current_stream(dev)
    step = Step(F, case, not args.unfused)
    for _ in range(warmup):
        step.run()
        flush.fill_(1)
    torch.cuda.synchronize(dev)
    if F.fp8pd_check_errors() != 0:
        raise RuntimeError("device error word set during warm-up")
    info0 = F.fp8pd_last_run_info()
    step.run()
    info1 = F.fp8pd_last_run_info()
    launches_per_step = int(info1["kernel_launches"] - info0["kernel_launches"])
    torch.cuda.synchronize(dev)

    # ---- the step as a CUDA graph (how a serving loop replays decode steps) --
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream(dev)
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        step.run()
    stream.wait_stream(side)
    with torch.cuda.graph(graph):
        step.run()
    for _ in range(warmup):
        graph.replay()
        flush.fill_(1)
    torch.cuda.synchronize(dev)

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    world = _dist_env()[0]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    sampler = ClockSampler(dev) if clocks else None
    if sampler:
        sampler.__enter__()
    try:
        for i in range(steps):
            ev[i][0].record(stream)
            graph.replay()
            ev[i][1].record(stream)
            flush.fill_(i & 0xFF)
        torch.cuda.synchronize(dev)
    finally:
        if sampler:
            sampler.__exit__()
    if world > 1:
        torch.distributed.barrier()
    total_ms = sum(a.elapsed_time(b) for a, b in ev)
    del graph

    # ---- per-layer kernel durations: eager, one layer at a time, the
    # library's events around each launch on the launching stream
    per_layer = []
    eager_ms = 0.0
    for li in range(len(case.layers)):
        lstep = Step(F, case, not args.unfused, layers=[li])
        F.fp8pd_timing_enable(True)
        F.fp8pd_timing_collect()
        ev2 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(steps)]
        torch.cuda.synchronize(dev)
        for i in range(steps):
            # a ~1 ms spin first, so the host has queued the whole step before
            # the GPU reaches it: the per-kernel events then hold device time
            # only, with no host launch gaps inside them
            torch.cuda._sleep(2_000_000)
            ev2[i][0].record(stream)
            lstep.run()
            ev2[i][1].record(stream)
            flush.fill_(i & 0xFF)
        torch.cuda.synchronize(dev)
        eager_ms += sum(a.elapsed_time(b) for a, b in ev2)
        kt = F.fp8pd_timing_collect()
        F.fp8pd_timing_enable(False)
        run = F.fp8pd_last_run_info()
        att_ms = kt["attention_ms"] / max(1, kt["attention_launches"])
        app_ms = kt["append_ms"] / kt["append_launches"] if kt["append_launches"] else None
        per_layer.append({"bytes": W.algorithmic_bytes(case, li), "kernel_ms": att_ms,
                          "append_ms": app_ms,
                          "plan": {k: run[k] for k in ("kernel", "schedule", "num_splits",
                                                       "head_groups", "grid_blocks", "combine")}})
    if F.fp8pd_check_errors() != 0:
        raise RuntimeError("device error word set during the timed region")
    return {"ms_per_step": total_ms / steps, "eager_ms_per_step": eager_ms / steps,
            "launches_per_step": launches_per_step, "layers": per_layer,
            "clocks": sampler.summary() if sampler else None, "fused": step.fused}


def _roofline(entry: dict, peaks: dict, fused: bool, traffic=None) -> dict:
    ms = entry["kernel_ms"]
    achieved = entry["bytes"] / (ms * 1e-3) / 1e9 if ms > 0 else None
    names = UMMA_NAME if entry["plan"].get("kernel") == 2 else KERNEL_NAME
    kernel = names.get(entry["plan"]["schedule"], "decode kernel") + \
        (", append fused" if fused else "")
    return {"bound": "hbm", "kernel": kernel,
            "achieved": round(achieved, 2) if achieved else None,
            "peak": peaks["hbm_gbs"], "peak_source": peaks["source"], "unit": "GB/s",
            "frac": round(achieved / peaks["hbm_gbs"], 4) if achieved else None,
            "traffic": traffic, "bytes_per_launch": int(entry["bytes"]),
            "us_per_launch": round(ms * 1e3, 3),
            "append_us_per_launch": round(entry["append_ms"] * 1e3, 3) if entry["append_ms"] else None,
            "plan": entry["plan"]}


def _build_case(name: str, dev, args) -> W.Case:
    case = W.make_case(name, dev, **_scale_override(args))
    for layer in case.layers:
        layer.out = torch.empty(layer.q.shape, dtype=torch.float32, device=dev)
    return case


def _set_options(F, args) -> None:
    F.fp8pd_set_option(F.OPT_K_DECODE, {"bits": 0, "cvt": 1, "mma8": 2}[args.k_decode])
    F.fp8pd_set_option(F.OPT_NUM_SPLITS, args.splits)
    F.fp8pd_set_option(F.OPT_SCHEDULE, args.schedule)
    F.fp8pd_set_option(F.OPT_COMPUTE, 1 if args.compute == "fp8" else 0)
    F.fp8pd_set_option(F.OPT_KERNEL, args.kernel)


def run_ours(args) -> dict | None:
    import fp8_paged_decode_split_b200 as F
    _set_options(F, args)
    world, rank, local = _dist_env()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    peaks = _peaks()
    flush = L2Flush(dev)

    case = _build_case(args.config, dev, args)
    nbytes = _step_bytes(case)
    t = time_case(F, case, dev, args, flush, args.steps, args.warmup, clocks=True)
    e2e = run_e2e(F, case, dev, flush, args)
    total_ms, e2e_ms = max_over_ranks([t["ms_per_step"] * args.steps, e2e["ms"]], dev)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(case, budget_s=args.cpu_seconds)
    del case
    torch.cuda.empty_cache()

    # ---- the other workloads (one GPU only: the scaling runs time the headline)
    sweep = {}
    if world == 1 and not args.no_sweep:
        for name in SWEEP:
            if name == args.config:
                continue
            c = _build_case(name, dev, args)
            ts = time_case(F, c, dev, args, flush, max(5, min(args.steps, 20)),
                           max(3, args.warmup))
            nb = _step_bytes(c)
            ent = {"workload": _workload_text(args, name),
                   "us_per_step": round(ts["ms_per_step"] * 1e3, 3),
                   "value": round(nb / (ts["ms_per_step"] * 1e-3) / 1e9, 2), "unit": "GB/s",
                   "bytes_per_step": nb,
                   "roofline": [_roofline(e, peaks, ts["fused"],
                                          _traffic(name, i) if args.scales == "workload" else None)
                                for i, e in enumerate(ts["layers"])]}
            if len(ent["roofline"]) == 1:
                ent["roofline"] = ent["roofline"][0]
            sweep[name] = ent
            del c
            torch.cuda.empty_cache()

    if world > 1:
        torch.distributed.destroy_process_group()
    if rank != 0:
        return None

    ms_per_step = total_ms / args.steps
    gbs = whole_job_gbs(world, nbytes, ms_per_step)
    # the dominant kernel: the layer whose launch takes longest
    hi = max(range(len(t["layers"])), key=lambda i: t["layers"][i]["kernel_ms"])
    head = t["layers"][hi]
    line = {
        "metric": METRIC,
        "value": round(gbs, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 6),
        "us_per_step": round(ms_per_step * 1e3, 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": ("e4m3 cache; f16 tensor-core MMA, f32 accumulate" if args.compute == "f32" else
                  "e4m3 cache; fp8 compute: q and P rounded to e4m3, e4m3 tensor-core MMA, "
                  "f32 accumulate"),
        "data": "synthetic (seeded), no dataset",
        "config": _config_dict(args, args.config, nbytes=nbytes),
        "timing": "device time of CUDA-graph replays of the step (per-step events); "
                  "per-kernel events from an eager pass of the same steps",
        "eager_ms_per_step": round(t["eager_ms_per_step"], 6),
        "roofline": _roofline(head, peaks, t["fused"],
                              _traffic(args.config, hi) if args.scales == "workload" else None),
        "gpu_launches": t["launches_per_step"] * args.steps,
        "e2e": {"value": round(whole_job_gbs(world, nbytes, e2e_ms / e2e["steps"]), 2),
                "unit": "GB/s", "ms_per_step": round(e2e_ms / e2e["steps"], 6),
                "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
                "copies": e2e["mode"]},
        "clocks": t["clocks"],
    }
    if world == 1:
        # the same copies without overlap: copy in, step, copy out, one stream
        line["e2e"]["serial"] = {
            "value": round(nbytes / (e2e["serial_ms"] / e2e["steps"] * 1e-3) / 1e9, 2),
            "ms_per_step": round(e2e["serial_ms"] / e2e["steps"], 6)}
    if len(t["layers"]) > 1:
        line["roofline"]["layer"] = hi
        line["roofline_layers"] = [
            _roofline(e, peaks, t["fused"],
                      _traffic(args.config, i) if args.scales == "workload" else None)
            for i, e in enumerate(t["layers"])]
    if cpu is not None:
        line["cpu_baseline"] = cpu
    if sweep:
        line["configs"] = sweep
    return line


def _e2e_fields(case: W.Case, step: "Step") -> list:
    """The per-step inputs a serving loop sends: (owner, attribute, tensor)."""
    fields = []
    for layer in case.layers:
        fields += [(layer, "q", layer.q), (layer, "block_table", layer.block_table)]
        if step.fused or case.spec.append:
            fields += [(layer, "k_new", layer.k_new), (layer, "v_new", layer.v_new)]
    if step.fused:
        fields.append((case, "positions", case.positions))
    else:
        fields.append((case, "attend_lens", case.attend_lens))
        if case.spec.append:
            fields.append((case, "positions", case.positions))
    return fields


def _stage(fields: list, dev, copies: int):
    """A pinned host staging buffer holding every field (256-byte aligned
    slots), ``copies`` device buffers of the same layout, and each device
    buffer's views of the fields."""
    offs, total = [], 0
    for _, _, t in fields:
        offs.append(total)
        total += (t.numel() * t.element_size() + 255) // 256 * 256
    host = torch.empty(total, dtype=torch.uint8).pin_memory()
    devs = [torch.empty(total, dtype=torch.uint8, device=dev) for _ in range(copies)]
    views = [[] for _ in range(copies)]
    for (_, _, t), off in zip(fields, offs):
        n = t.numel() * t.element_size()
        host[off:off + n].view(t.dtype).view(t.shape).copy_(t.cpu())
        for b in range(copies):
            views[b].append(devs[b][off:off + n].view(t.dtype).view(t.shape))
    return host, devs, views


def run_e2e(F, case: W.Case, dev, flush, args) -> dict:
    """The step through the public API with its inputs sent from and its
    outputs read back to pinned host memory, every step: q, the block table
    and the new K/V token of every layer and the positions or lengths go in
    as one host -> device copy of a packed staging buffer (the step reads its
    device side through views), and each layer's output comes back; the KV
    pools stay resident, as in serving. When a step's bytes exceed the L2,
    a serving loop's double buffering is used: step i + 1's inputs travel on
    one copy stream and step i - 1's outputs on another while step i runs,
    and the timed region runs from the end of the last untimed step to the
    end of the last timed step's output copy: K steps, K + 1 output copies
    and K - 1 input copies (the first timed step's inputs were copied while
    the step before it ran). Otherwise each step is copy in, step, copy out on
    one stream, timed per step with the L2 flushed between steps."""
    step = Step(F, case, not args.unfused)
    fields = _e2e_fields(case, step)
    h2d = sum(t.numel() * t.element_size() for _, _, t in fields)
    d2h = sum(layer.q.numel() * 4 for layer in case.layers)
    steps = max(3, min(args.steps, 20))
    l2 = getattr(torch.cuda.get_device_properties(dev), "L2_cache_size", 126 << 20)
    serial_ms = _e2e_serial(case, step, fields, dev, flush, steps)
    out = {"ms": serial_ms, "steps": steps, "h2d": int(h2d), "d2h": int(d2h),
           "mode": "serial: copy in, step, copy out on one stream; L2 flushed between steps",
           "serial_ms": serial_ms}
    if _step_bytes(case) > l2:
        out["ms"] = _e2e_pipelined(case, step, fields, dev, steps)
        out["mode"] = ("double-buffered: each step's inputs and outputs copied on their own "
                       "streams while the neighbouring steps run")
    return out


def _e2e_serial(case: W.Case, step: "Step", fields: list, dev, flush, steps: int) -> float:
    stream = torch.cuda.current_stream(dev)
    host_stage, (dev_stage,), (views,) = _stage(fields, dev, 1)
    host_out = [torch.empty(layer.q.shape, dtype=torch.float32).pin_memory() for layer in case.layers]
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    saved = [(obj, name, t) for obj, name, t in fields]
    try:
        for (obj, name, _), v in zip(fields, views):
            setattr(obj, name, v)
        for i in range(steps + 2):
            timed = i >= 2
            if timed:
                ev[i - 2][0].record(stream)
            dev_stage.copy_(host_stage, non_blocking=True)
            step.run()
            for h, layer in zip(host_out, case.layers):
                h.copy_(layer.out, non_blocking=True)
            if timed:
                ev[i - 2][1].record(stream)
            flush.fill_(3)
        torch.cuda.synchronize(dev)
    finally:
        for obj, name, t in saved:
            setattr(obj, name, t)
    return sum(a.elapsed_time(b) for a, b in ev)


def _e2e_pipelined(case: W.Case, step: "Step", fields: list, dev, steps: int) -> float:
    """Step i runs on the compute stream once its inputs (buffer i mod 2) are
    in and step i - 2's outputs (the same output buffers) have been read
    back; the input copy of step i + 1 waits only for step i - 1, the reader
    of its buffer."""
    compute = torch.cuda.current_stream(dev)
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    host_stage, dev_stage, views = _stage(fields, dev, 2)
    dev_out = [[torch.empty(layer.q.shape, dtype=torch.float32, device=dev) for layer in case.layers]
               for _ in range(2)]
    host_out = [[torch.empty(layer.q.shape, dtype=torch.float32).pin_memory()
                 for layer in case.layers] for _ in range(2)]
    ev_in = [torch.cuda.Event() for _ in range(2)]    # inputs of the buffer are in
    ev_done = [torch.cuda.Event() for _ in range(2)]  # the step using the buffer has run
    ev_read = [torch.cuda.Event() for _ in range(2)]  # its outputs have been read back
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    warm = 2
    n = warm + steps
    saved = [(obj, name, t) for obj, name, t in fields] + [(layer, "out", layer.out)
                                                           for layer in case.layers]

    def send(i: int) -> None:
        b = i & 1
        with torch.cuda.stream(up):
            if i >= 2:
                up.wait_event(ev_done[b])  # step i - 2 has read this buffer
            dev_stage[b].copy_(host_stage, non_blocking=True)
            ev_in[b].record(up)

    try:
        torch.cuda.synchronize(dev)
        send(0)
        for i in range(n):
            b = i & 1
            for (obj, name, _), v in zip(fields, views[b]):
                setattr(obj, name, v)
            for layer, o in zip(case.layers, dev_out[b]):
                layer.out = o
            compute.wait_event(ev_in[b])
            if i >= 2:
                compute.wait_event(ev_read[b])  # step i - 2's outputs are back
            step.run()
            ev_done[b].record(compute)
            if i == warm - 1:
                t0.record(compute)  # steady state: the timed steps start when this one ends
            if i + 1 < n:
                send(i + 1)
            with torch.cuda.stream(down):
                down.wait_event(ev_done[b])
                for h, o in zip(host_out[b], dev_out[b]):
                    h.copy_(o, non_blocking=True)
                ev_read[b].record(down)
        compute.wait_event(ev_read[(n - 1) & 1])
        t1.record(compute)
        torch.cuda.synchronize(dev)
    finally:
        for obj, name, t in saved:
            setattr(obj, name, t)
    return t0.elapsed_time(t1)


# ---------------------------------------------------------------------------
# The oracle on the host's cores
# ---------------------------------------------------------------------------

def host_threads() -> int:
    """Host cores this process may run on."""
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:
        return max(1, os.cpu_count() or 1)


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return platform.processor() or "unknown"


def _oracle_tasks(case_np: dict, lens) -> list:
    """The oracle's work as (layer, sequence, KV head, algorithmic bytes)
    tasks: the attended K and V bytes of that KV head, its block-table
    entries and the q rows of its query heads."""
    tasks = []
    for li, L in enumerate(case_np["layers"]):
        B, Hq, D = L["q"].shape
        ps, Hkv = L["k_pages"].shape[1], L["k_pages"].shape[2]
        G = Hq // Hkv
        for b in range(B):
            Lb = int(lens[b])
            lo = max(0, Lb - L["window"]) if L["window"] > 0 else 0
            n = max(0, Lb - lo)
            tok = sum(4 * n * (sc.shape[3] if sc.ndim == 4 else 1)
                      for sc in (L["k_scale"], L["v_scale"]) if sc.ndim >= 3)
            tbl = 4 * ((Lb - 1) // ps - lo // ps + 1) if n > 0 else 0
            for h in range(Hkv):  # the table row is read once per sequence
                tasks.append((li, b, h, 2 * n * D + tok + (tbl if h == 0 else 0) + 2 * G * D))
    return tasks


def _oracle_step(case_np: dict, lens, positions, append: bool, tasks, pool=None):
    """One step of the oracle over ``tasks``: the appends of their sequences
    (one token each, in order), then the attention of every task's
    (sequence, KV head) as its own job on ``pool`` (numpy releases the GIL
    inside its array kernels, so the jobs run on several cores at once)."""
    import oracle as O
    seqs = sorted({b for _, b, _, _ in tasks})
    if append:
        for L in case_np["layers"]:
            idx = np.array(seqs)
            O.kv_append(L["k_new"][idx], L["v_new"][idx], L["k_pages"], L["v_pages"],
                        L["k_scale"], L["v_scale"], L["block_table"][idx], positions[idx])
    jobs = []
    for li, b, h, _ in tasks:
        L = case_np["layers"][li]
        G = L["q"].shape[1] // L["k_pages"].shape[2]
        args = (L["q"], L["k_pages"], L["v_pages"], L["k_scale"], L["v_scale"],
                L["block_table"], lens)
        kw = dict(window=L["window"], sinks=L["sinks"], sm_scale=L["sm_scale"],
                  batch_heads=[(b, h * G + g) for g in range(G)])
        if pool is None:
            O.paged_decode_attention(*args, **kw)
        else:
            jobs.append(pool.submit(O.paged_decode_attention, *args, **kw))
    for j in jobs:
        j.result()


def _case_to_numpy(case: W.Case, seqs) -> tuple[dict, np.ndarray, np.ndarray | None]:
    """Host copy of the sequences ``seqs`` of a case (their pages only)."""
    out = {"layers": []}
    ps = case.spec.ps
    lens = case.attend_lens.cpu().numpy()[seqs]
    pos = case.positions.cpu().numpy()[seqs] if case.positions is not None else None
    for li, layer in enumerate(case.layers):
        tbl = layer.block_table.cpu().numpy()[seqs]
        npg = (lens + ps - 1) // ps
        ids = np.concatenate([tbl[i, :npg[i]] for i in range(len(seqs))]).astype(np.int64)
        new_tbl = np.full_like(tbl, -1)
        off = 0
        for i in range(len(seqs)):
            new_tbl[i, :npg[i]] = np.arange(off, off + npg[i])
            off += npg[i]
        idx = torch.as_tensor(ids, device=layer.k_pages.device)
        f = lambda t: t.detach().float().cpu().numpy().astype(np.float64)  # noqa: E731
        # per-page and per-token scales follow their pages; per-head ones do not
        pick = lambda sc: (sc[idx] if sc.dim() >= 2 else sc).cpu().numpy()  # noqa: E731
        out["layers"].append({
            "q": f(layer.q[list(seqs)]),
            "k_pages": layer.k_pages[idx].cpu().numpy(), "v_pages": layer.v_pages[idx].cpu().numpy(),
            "k_scale": pick(layer.k_scale), "v_scale": pick(layer.v_scale),
            "block_table": new_tbl, "window": layer.window, "sm_scale": layer.sm_scale,
            "sinks": layer.sinks.cpu().numpy() if layer.sinks is not None else None,
            "k_new": f(layer.k_new[list(seqs)]) if layer.k_new is not None else None,
            "v_new": f(layer.v_new[list(seqs)]) if layer.v_new is not None else None})
    return out, lens, pos


def _oracle_sample(case: W.Case, step_seconds: float, threads: int, pool):
    """A bounded sample of the workload for the oracle: the first sequences
    of the batch (their pages copied to the host), and as many of their
    (layer, sequence, KV head) tasks, in order, as the host's cores finish in
    about ``step_seconds`` (sized from one timed task; at least one task)."""
    B = case.spec.B
    per_seq = _step_bytes(case) / max(1, B)
    # enough sequences for the largest sample the time budget could take
    nseq = max(1, min(B, int(2e9 / max(1.0, per_seq)) + 1))
    seqs = list(range(nseq))
    case_np, lens, pos = _case_to_numpy(case, seqs)
    tasks = _oracle_tasks(case_np, lens)
    probe = tasks[:1]
    t0 = time.perf_counter()
    _oracle_step(case_np, lens, pos, case.spec.append, probe, None)
    one = max(1e-4, time.perf_counter() - t0)
    n = max(1, min(len(tasks), int(step_seconds * threads / one)))
    chosen = tasks[:n]
    # keep the host copy of the sequences the sample uses only
    used = sorted({b for _, b, _, _ in chosen})
    if len(used) < len(seqs):
        case_np, lens, pos = _case_to_numpy(case, used)
        remap = {b: i for i, b in enumerate(used)}
        chosen = [(li, remap[b], h, nb) for li, b, h, nb in chosen]
    nbytes = sum(nb for *_, nb in chosen)
    text = (f"{len(chosen)} of {len(tasks) * B // nseq} (layer, sequence, KV head) tasks over "
            f"{len(used)}/{B} sequences ({nbytes / 1e6:.1f} MB algorithmic per step), float64 "
            f"numpy, {threads} threads on {cpu_model()}")
    return case_np, lens, pos, chosen, nbytes, text


def cpu_baseline(case: W.Case, budget_s: float = 10.0) -> dict:
    """The oracle as it stands, timed on every core of this host on a bounded
    sample of the workload, repeated until about ``budget_s`` seconds, one
    BLAS thread per job."""
    from threadpoolctl import threadpool_limits
    threads = host_threads()
    with threadpool_limits(1), concurrent.futures.ThreadPoolExecutor(threads) as pool:
        case_np, lens, pos, tasks, nbytes, text = _oracle_sample(case, 1.5, threads, pool)
        reps, t_total = 0, 0.0
        while t_total < budget_s and reps < 1000:
            t0 = time.perf_counter()
            _oracle_step(case_np, lens, pos, case.spec.append, tasks, pool)
            t_total += time.perf_counter() - t0
            reps += 1
    return {"value": round(nbytes * reps / t_total / 1e9, 4), "unit": "GB/s", "cores": threads,
            "kind": "oracle", "sample": f"{reps} step(s) of {text}",
            "seconds": round(t_total, 2)}


def _scale_override(args) -> dict:
    """``--scales token``: the workload with one scale per stored token and KV
    head instead of its own scale form."""
    scales = getattr(args, "scales", "workload")
    if scales == "mx":
        return {"scale_mode": "mx"}
    if scales != "token":
        return {}
    return {"scale_mode": "token", "k_groups": getattr(args, "k_groups", 1)}


def _workload_text(args, name: str | None = None) -> str:
    name = name or args.config
    text = WORKLOAD_TEXT.get(name, name)
    if getattr(args, "scales", "workload") == "mx":
        return text + " (K and V stored as MXFP8: E8M0 scale per 32-entry block)"
    if getattr(args, "scales", "workload") != "token":
        return text
    groups = f", K in {args.k_groups} sub-row groups" if args.k_groups > 1 else ""
    return text + f" (scales replaced: per (token, KV head){groups})"


def _scales_text(spec) -> str:
    text = {"head": "per KV head", "page": "per (page, KV head)",
            "token": "per (token, KV head)",
            "mx": "MXFP8: E8M0 per (token, KV head, 32-entry block)"}[spec.scale_mode]
    if spec.scale_mode == "token" and spec.k_groups > 1:
        text += f"; K per (token, KV head, group of D/{spec.k_groups})"
    return text


def run_reference(args) -> dict | None:
    """The float64 CPU oracle on this host's cores: each step is one bounded
    sample of the workload (rank 0 only)."""
    world, rank, _ = _dist_env()
    if rank != 0:
        return None
    from threadpoolctl import threadpool_limits
    case = W.make_case(args.config, "cpu", **_scale_override(args))
    threads = host_threads()
    with threadpool_limits(1), concurrent.futures.ThreadPoolExecutor(threads) as pool:
        case_np, lens, pos, tasks, nbytes, text = _oracle_sample(case, 1.5, threads, pool)
        for _ in range(args.warmup):
            _oracle_step(case_np, lens, pos, case.spec.append, tasks, pool)
        t0 = time.perf_counter()
        for _ in range(args.steps):
            _oracle_step(case_np, lens, pos, case.spec.append, tasks, pool)
        total = time.perf_counter() - t0
    gbs = nbytes * args.steps / total / 1e9
    return {
        "impl": "reference", "metric": METRIC, "value": round(gbs, 4), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(total / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded), no dataset",
        "config": _config_dict(args, args.config),
        "cpu_baseline": {"value": round(gbs, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
                         "sample": text},
        "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


# ---------------------------------------------------------------------------
# Launching N ranks
# ---------------------------------------------------------------------------

def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def launch_ranks(argv: list, gpus: int, dry_run: bool, timeout_s: float = 1800.0) -> int:
    """Re-runs this script under ``torch.distributed.run`` with ``gpus`` ranks
    on this node (rendezvous on 127.0.0.1) and returns its exit code. Refuses,
    before starting anything, when fewer than ``gpus`` GPUs are visible
    (a dry run needs none)."""
    if not dry_run:
        visible = torch.cuda.device_count() if torch.cuda.is_available() else 0
        if visible < gpus:
            print(f"bench.py: --gpus {gpus} needs {gpus} visible GPUs, found {visible}",
                  file=sys.stderr)
            return 2
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={gpus}", "--master-addr=127.0.0.1",
           f"--master-port={_free_port()}", os.path.abspath(__file__), *argv]
    env = dict(os.environ)
    env.pop("WORLD_SIZE", None)
    try:
        return subprocess.run(cmd, env=env, timeout=timeout_s).returncode
    except subprocess.TimeoutExpired:
        print("bench.py: ranks did not finish in time", file=sys.stderr)
        return 3


def run_dry(args) -> dict | None:
    """Host logic of an N-rank run without a GPU: gloo ranks, a host-timed
    stand-in step, the max-over-ranks reduction and the weak-scaled total."""
    import datetime
    import torch.distributed as dist
    world, rank, _ = _dist_env()
    if world > 1:
        dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    nbytes = _spec_bytes(W.spec_with(args.config))
    t0 = time.perf_counter()
    for _ in range(args.steps):
        np.dot(np.ones(1 << 16), np.ones(1 << 16))
    ms = (time.perf_counter() - t0) * 1e3 / max(1, args.steps) + 1e-3 * (1 + rank)
    (ms_max,) = max_over_ranks([ms], torch.device("cpu"))
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return None
    return {"dry_run": True, "metric": METRIC, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_max,
            "value": round(whole_job_gbs(world, nbytes, ms_max), 2), "unit": "GB/s",
            "scaling": "weak", "config": _config_dict(args, args.config, nbytes=nbytes)}


def build_parser() -> argparse.ArgumentParser:
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default=DEFAULT_CONFIG, choices=sorted(W.SPECS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sweep", action="store_true",
                    help="time the headline workload only (no configs object)")
    ap.add_argument("--dry-run", action="store_true",
                    help="host logic of the N-rank run only (gloo, no GPU)")
    ap.add_argument("--unfused", action="store_true",
                    help="run fp8_kv_append and the attention call as two launches")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--k-decode", default="cvt", choices=["bits", "cvt", "mma8"],
                    help="QK contraction: K decoded to f16 by bit assembly or the hardware cvt, "
                         "or K's E4M3 bytes in E4M3 MMAs (mma8)")
    ap.add_argument("--splits", type=int, default=0, help="force a split count (0 = planner)")
    ap.add_argument("--scales", default="workload", choices=["workload", "token", "mx"],
                    help="token: per-token-per-head K/V scales instead of the workload's form; "
                         "mx: the MXFP8 cache (E8M0 scale per 32-entry block)")
    ap.add_argument("--k-groups", type=int, default=1,
                    help="with --scales token: K scales per sub-row group of D / k_groups entries")
    ap.add_argument("--compute", default="f32", choices=["f32", "fp8"],
                    help="numerical path: f32 (default, 1e-3) or the opt-in fp8 compute path "
                         "(q and P rounded once to E4M3; 1.5e-1)")
    ap.add_argument("--schedule", type=int, default=0, choices=[0, 1, 3],
                    help="0 = planner, 1 = uniform splits, 3 = proportional splits")
    ap.add_argument("--kernel", type=int, default=0, choices=[0, 1, 2],
                    help="0 = planner's choice, 1 = split kernel (mma.sync), "
                         "2 = tensor-memory kernel (tcgen05) where it applies")
    return ap


def main(argv=None) -> int:
    argv = sys.argv[1:] if argv is None else list(argv)
    ap = build_parser()
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.gpus < 1:
        ap.error("--gpus must be >= 1")
    world = _dist_env()[0]
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        return launch_ranks(argv, args.gpus, args.dry_run)
    if args.gpus != world:
        ap.error(f"--gpus {args.gpus} does not match WORLD_SIZE={world}")
    if args.dry_run:
        line = run_dry(args)
    elif args.impl == "reference":
        line = run_reference(args)
    else:
        line = run_ours(args)
    if line is not None:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
