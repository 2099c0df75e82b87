"""Benchmark: FP8 paged decode attention, achieved HBM GB/s and us/step.

One step = the decode hot path for one layer of a synthetic serving batch:
the append of one new token per sequence, then decode attention over the
updated paged E4M3 cache -- by default one ``fp8_paged_decode_append_attention``
launch (split kernel, append and combine fused); ``--unfused`` runs
``fp8_kv_append`` and ``fp8_paged_decode_attention`` as two launches.
Configs without an append run the attention call alone. Inputs are resident
in HBM when the timed region starts;
L2 is flushed between timed steps, outside each step's
events. ``value`` = algorithmic bytes (attended K/V once per KV head + q +
the block-table entries read) / device time, summed over ranks.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]

With N > 1 (torchrun, one process per GPU) every rank runs its own copy of
the workload on its GPU (independent sequences: no data-path collective);
time is the max over ranks, throughput the sum (weak scaling).
``--impl reference`` times the float64 CPU oracle on the same workload (rank
0 only).
"""

from __future__ import annotations

import argparse
import json
import os
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
DEFAULT_CONFIG = "llama"
WORKLOAD_TEXT = {
    "llama": "Llama-3-8B-like layer: B=32 Hq=32 Hkv=8 D=128 page=16 seq_len~U[512,4096] "
             "per-(page,head) scales, +1 appended token/seq",
    "tiny": "tiny: B=1 Hq=8 Hkv=2 D=64 page=16 L=256",
    "gptoss_full": "gpt-oss-like: B=64 Hq=64 Hkv=8 D=64 page=16 L=8192 sinks, full attention",
    "gptoss_w128": "gpt-oss-like: B=64 Hq=64 Hkv=8 D=64 page=16 L=8192 sinks, window=128",
    "mixed": "mixed pool: B=16 page=32 L~U[2048,16384]; sliding D=256 W=1024 + full D=512",
    "long_b1": "long context: B=1 Hq=64 Hkv=8 D=128 page=64 L=131072 +append",
    "long_b8": "long context: B=8 Hq=64 Hkv=8 D=128 page=64 L=131072 +append",
}
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "dram_traffic_per_launch.txt")
KERNEL_NAME = {1: "decode_tma_kernel (split kernel, merge in the same launch)",
               2: "decode_seg_kernel (balanced block ranges across sequences, merge in the same launch)",
               3: "decode_tma_kernel (proportional splits, merge in the same launch)"}


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


def _traffic(config: str):
    """DRAM bytes (read + write) per split-kernel launch from the committed ncu
    summary, if it was taken on the current kernel source and this workload.
    Lines of that file: ``<workload> <kernel source hash> <bytes>``."""
    try:
        with open(PROFILE_TRAFFIC) as f:
            for line in f:
                parts = line.split()
                if len(parts) == 3 and not line.startswith("#") and parts[0] == config \
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
    for its own traffic. FLUSH_MODE = "write" keeps the plain write."""
    MODE = os.environ.get("FP8PD_BENCH_FLUSH", "write+read")

    def __init__(self, device: torch.device):
        self.w = torch.empty(256 << 20, dtype=torch.uint8, device=device)
        self.r = torch.ones(64 << 20, dtype=torch.float32, device=device)
        self.sink = torch.empty((), dtype=torch.float32, device=device)

    def fill_(self, v: int = 1) -> None:
        if "write" in self.MODE:
            self.w.fill_(v & 0xFF)
        if "read" in self.MODE:
            torch.sum(self.r, dim=0, out=self.sink)

    def describe(self) -> str:
        return {"write": "256 MiB write", "read": "256 MiB read",
                "write+read": "256 MiB write, then a 256 MiB read of another buffer (no dirty "
                              "lines left)"}[self.MODE] + ", outside the step events"


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
    `fused` is off, then fp8_kv_append followed by the attention call."""

    def __init__(self, F, case: W.Case, fused: bool = True):
        self.F = F
        self.case = case
        self.fused = fused and case.spec.append

    def run(self, stream=None):
        F, c = self.F, self.case
        for layer in c.layers:
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


def run_ours(args) -> dict | None:
    import fp8_paged_decode_split_b200 as F
    F.fp8pd_set_option(F.OPT_K_DECODE, 1 if args.k_decode == "cvt" else 0)
    F.fp8pd_set_option(F.OPT_NUM_SPLITS, args.splits)
    F.fp8pd_set_option(F.OPT_SCHEDULE, args.schedule)
    world, rank, local = _dist_env()
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    case = W.make_case(args.config, dev, **_scale_override(args))
    for layer in case.layers:
        layer.out = torch.empty(layer.q.shape, dtype=torch.float32, device=dev)
    step = Step(F, case, not args.unfused)
    flush = L2Flush(dev)
    stream = torch.cuda.current_stream(dev)
    nbytes = _step_bytes(case)

    for _ in range(args.warmup):
        step.run()
        flush.fill_(1)
    torch.cuda.synchronize(dev)
    if F.fp8pd_check_errors() != 0:
        raise RuntimeError("device error word set during warm-up")
    info0 = F.fp8pd_last_run_info()
    step.run()
    plan_info = F.fp8pd_last_run_info()
    launches_per_step = int(plan_info["kernel_launches"] - info0["kernel_launches"])
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
    for _ in range(args.warmup):
        graph.replay()
        flush.fill_(1)
    torch.cuda.synchronize(dev)

    # ---- device-timed region: inputs resident, per-step events, L2 flushed between
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(dev) as clocks:
        for i in range(args.steps):
            ev[i][0].record(stream)
            graph.replay()
            ev[i][1].record(stream)
            flush.fill_(i & 0xFF)
        torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    total_ms = sum(a.elapsed_time(b) for a, b in ev)
    launches = launches_per_step * args.steps

    # ---- per-kernel durations: the same steps eagerly, the library's events
    # around each of its kernels on the launching stream, L2 flushed between
    F.fp8pd_timing_enable(True)
    F.fp8pd_timing_collect()
    ev2 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    torch.cuda.synchronize(dev)
    for i in range(args.steps):
        # a ~1 ms spin first, so the host has queued the whole step before the
        # GPU reaches it: the library's per-kernel events then hold device
        # time only, with no host launch gaps inside them
        torch.cuda._sleep(2_000_000)
        ev2[i][0].record(stream)
        step.run()
        ev2[i][1].record(stream)
        flush.fill_(i & 0xFF)
    torch.cuda.synchronize(dev)
    eager_ms = sum(a.elapsed_time(b) for a, b in ev2)
    kt = F.fp8pd_timing_collect()
    F.fp8pd_timing_enable(False)
    if F.fp8pd_check_errors() != 0:
        raise RuntimeError("device error word set during the timed region")
    del graph

    # ---- end to end through the public API with host buffers -----------------
    e2e = run_e2e(F, case, dev, flush, args)

    total_ms, e2e_ms = max_over_ranks([total_ms, e2e["ms"]], dev)
    if world > 1:
        torch.distributed.destroy_process_group()
    if rank != 0:
        return None

    ms_per_step = total_ms / args.steps
    gbs = whole_job_gbs(world, nbytes, ms_per_step)
    peaks = _peaks()
    att_ms = kt["attention_ms"] / max(1, kt["attention_launches"])
    app_ms = kt["append_ms"] / kt["append_launches"] if kt["append_launches"] else None
    layer_bytes = nbytes / max(1, len(case.layers))
    achieved = layer_bytes / (att_ms * 1e-3) / 1e9 if att_ms > 0 else None
    traffic = _traffic(args.config) if args.scales == "workload" else None
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
        "dtype": "e4m3 cache; f16 tensor-core MMA, f32 accumulate",
        "data": "synthetic (seeded), no dataset",
        "config": {"workload": _workload_text(args),
                   "name": args.config,
                   "bytes_per_step": nbytes, "k_decode": args.k_decode,
                   "scales": _scales_text(case),
                   "l2": "flushed between timed steps: " + flush.describe(),
                   "parallelism": f"{world} independent replicas" if world > 1 else "1 GPU"},
        "timing": "device time of CUDA-graph replays of the step (per-step events); "
                  "eager time and per-kernel events from an eager pass of the same steps",
        "eager_ms_per_step": round(eager_ms / args.steps, 6),
        "roofline": {"bound": "hbm",
                     "kernel": KERNEL_NAME[plan_info["schedule"]] +
                     (", append fused" if step.fused else ""),
                     "achieved": round(achieved, 2) if achieved else None,
                     "peak": peaks["hbm_gbs"], "peak_source": peaks["source"],
                     "unit": "GB/s",
                     "frac": round(achieved / peaks["hbm_gbs"], 4) if achieved else None,
                     "traffic": traffic,
                     "us_per_launch": round(att_ms * 1e3, 3),
                     "append_us_per_launch": round(app_ms * 1e3, 3) if app_ms else None},
        "gpu_launches": launches,
        "e2e": {"value": round(whole_job_gbs(world, nbytes, e2e_ms / e2e["steps"]), 2),
                "unit": "GB/s", "ms_per_step": round(e2e_ms / e2e["steps"], 6),
                "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"]},
        "clocks": clocks.summary(),
        "plan": {k: plan_info[k] for k in ("schedule", "num_splits", "head_groups", "grid_blocks",
                                           "combine")},
    }
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(case, budget_s=args.cpu_seconds)
    return line


def run_e2e(F, case: W.Case, dev, flush, args) -> dict:
    """Per step: one pinned host -> device copy of the step's inputs (q, the
    block table and the new K/V token of every layer, and the positions or
    lengths, packed into one staging buffer whose device side the step reads
    through views), the step, and a device -> host copy of each layer's
    output; timed with events on the step's stream. The KV pools stay
    resident, as in serving."""
    stream = torch.cuda.current_stream(dev)
    step = Step(F, case, not args.unfused)
    fields = []  # (owner, attribute, tensor)
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
    offs, total = [], 0
    for _, _, t in fields:
        offs.append(total)
        total += (t.numel() * t.element_size() + 255) // 256 * 256
    host_stage = torch.empty(total, dtype=torch.uint8).pin_memory()
    dev_stage = torch.empty(total, dtype=torch.uint8, device=dev)
    saved = []
    for (obj, name, t), off in zip(fields, offs):
        n = t.numel() * t.element_size()
        host_stage[off:off + n].view(t.dtype).view(t.shape).copy_(t.cpu())
        saved.append((obj, name, t))
        setattr(obj, name, dev_stage[off:off + n].view(t.dtype).view(t.shape))
    host_out = [torch.empty(layer.q.shape, dtype=torch.float32).pin_memory() for layer in case.layers]
    h2d = sum(t.numel() * t.element_size() for _, _, t in fields)
    d2h = sum(t.numel() * t.element_size() for t in host_out)
    steps = max(3, min(args.steps, 20))
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    try:
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
    ms = sum(a.elapsed_time(b) for a, b in ev)
    return {"ms": ms, "steps": steps, "h2d": int(h2d), "d2h": int(d2h)}


def _oracle_step(case_np: dict, lens, positions, append: bool):
    import oracle as O
    for L in case_np["layers"]:
        if append:
            O.kv_append(L["k_new"], L["v_new"], L["k_pages"], L["v_pages"], L["k_scale"],
                        L["v_scale"], L["block_table"], positions)
        O.paged_decode_attention(L["q"], L["k_pages"], L["v_pages"], L["k_scale"], L["v_scale"],
                                 L["block_table"], lens, window=L["window"], sinks=L["sinks"],
                                 sm_scale=L["sm_scale"])


def _case_to_numpy(case: W.Case, seqs) -> tuple[dict, np.ndarray, np.ndarray | None, int]:
    """Host copy of the sequences ``seqs`` of a case (their pages only)."""
    out = {"layers": []}
    ps = case.spec.ps
    lens = case.attend_lens.cpu().numpy()[seqs]
    pos = case.positions.cpu().numpy()[seqs] if case.positions is not None else None
    nbytes = 0
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
        d = {"q": f(layer.q[list(seqs)]),
             "k_pages": layer.k_pages[idx].cpu().numpy(), "v_pages": layer.v_pages[idx].cpu().numpy(),
             "k_scale": pick(layer.k_scale), "v_scale": pick(layer.v_scale),
             "block_table": new_tbl, "window": layer.window, "sm_scale": layer.sm_scale,
             "sinks": layer.sinks.cpu().numpy() if layer.sinks is not None else None,
             "k_new": f(layer.k_new[list(seqs)]) if layer.k_new is not None else None,
             "v_new": f(layer.v_new[list(seqs)]) if layer.v_new is not None else None}
        out["layers"].append(d)
        for b in range(len(seqs)):
            Lb = int(lens[b])
            lo = max(0, Lb - layer.window) if layer.window > 0 else 0
            n = Lb - lo
            nbytes += 2 * n * layer.spec.Hkv * layer.spec.D
            nbytes += sum(4 * n * layer.spec.Hkv * (sc.shape[3] if sc.dim() == 4 else 1)
                          for sc in (layer.k_scale, layer.v_scale) if sc.dim() >= 3)
            if n > 0:
                nbytes += 4 * ((Lb - 1) // ps - lo // ps + 1)
        nbytes += 2 * d["q"].size
    return out, lens, pos, nbytes


def cpu_baseline(case: W.Case, budget_s: float = 10.0) -> dict:
    """The oracle as it stands, timed on this host on a bounded sample of the
    workload: whole steps over the first sequences of the batch, repeated
    until about ``budget_s`` seconds, single BLAS thread."""
    from threadpoolctl import threadpool_limits
    B = case.spec.B
    total = _step_bytes(case)
    nseq = max(1, min(B, int(B * 160e6 / max(1, total))))   # ~1 s of oracle work per step
    seqs = list(range(nseq))
    case_np, lens, pos, nbytes = _case_to_numpy(case, seqs)
    reps, t_total = 0, 0.0
    with threadpool_limits(1):
        while t_total < budget_s and reps < 1000:
            t0 = time.perf_counter()
            _oracle_step(case_np, lens, pos, case.spec.append)
            t_total += time.perf_counter() - t0
            reps += 1
    return {"value": round(nbytes * reps / t_total / 1e9, 4), "unit": "GB/s", "cores": 1,
            "kind": "oracle",
            "sample": f"{reps} full step(s) over {nseq}/{B} sequences "
                      f"({nbytes / 1e6:.1f} MB/step algorithmic), float64 numpy, 1 thread",
            "seconds": round(t_total, 2)}


def _scale_override(args) -> dict:
    """``--scales token``: the workload with one scale per stored token and KV
    head instead of its own scale form."""
    if getattr(args, "scales", "workload") != "token":
        return {}
    return {"scale_mode": "token", "k_groups": getattr(args, "k_groups", 1)}


def _workload_text(args) -> str:
    text = WORKLOAD_TEXT.get(args.config, args.config)
    if getattr(args, "scales", "workload") != "token":
        return text
    groups = f", K in {args.k_groups} sub-row groups" if args.k_groups > 1 else ""
    return text + f" (scales replaced: per (token, KV head){groups})"


def _scales_text(case) -> str:
    text = {"head": "per KV head", "page": "per (page, KV head)",
            "token": "per (token, KV head)"}[case.spec.scale_mode]
    if case.spec.scale_mode == "token" and case.spec.k_groups > 1:
        text += f"; K per (token, KV head, group of D/{case.spec.k_groups})"
    return text


def run_reference(args) -> dict | None:
    """The float64 CPU oracle on this host: each step is one bounded sample of
    the workload (rank 0 only)."""
    world, rank, _ = _dist_env()
    if rank != 0:
        return None
    from threadpoolctl import threadpool_limits
    case = W.make_case(args.config, "cpu", **_scale_override(args))
    B = case.spec.B
    # bounded sample per step: as many whole sequences as fit in ~1.5 s
    seqs = list(range(B))
    case_np, lens, pos, nbytes = _case_to_numpy(case, seqs)
    with threadpool_limits(1):
        t0 = time.perf_counter()
        _oracle_step(case_np, lens, pos, case.spec.append)
        one = time.perf_counter() - t0
        if one > 1.5 and B > 1:
            keep = max(1, int(B * 1.5 / one))
            seqs = list(range(keep))
            case_np, lens, pos, nbytes = _case_to_numpy(case, seqs)
        for _ in range(args.warmup):
            _oracle_step(case_np, lens, pos, case.spec.append)
        t0 = time.perf_counter()
        for _ in range(args.steps):
            _oracle_step(case_np, lens, pos, case.spec.append)
        total = time.perf_counter() - t0
    gbs = nbytes * args.steps / total / 1e9
    sample = f"{len(seqs)}/{B} sequences per step ({nbytes / 1e6:.1f} MB algorithmic), float64 numpy"
    return {
        "impl": "reference", "metric": METRIC, "value": round(gbs, 4), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(total / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded), no dataset",
        "config": {"workload": _workload_text(args), "name": args.config,
                   "scales": _scales_text(case)},
        "cpu_baseline": {"value": round(gbs, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default=DEFAULT_CONFIG, choices=sorted(W.SPECS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--unfused", action="store_true",
                    help="run fp8_kv_append and the attention call as two launches")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--k-decode", default="cvt", choices=["bits", "cvt"],
                    help="E4M3 -> f16 decode of K: bit assembly or hardware cvt")
    ap.add_argument("--splits", type=int, default=0, help="force a split count (0 = planner)")
    ap.add_argument("--scales", default="workload", choices=["workload", "token"],
                    help="token: per-token-per-head K/V scales instead of the workload's form")
    ap.add_argument("--k-groups", type=int, default=1,
                    help="with --scales token: K scales per sub-row group of D / k_groups entries")
    ap.add_argument("--schedule", type=int, default=0, choices=[0, 1, 2, 3],
                    help="0 = planner, 1 = uniform splits, 2 = segment kernel, "
                         "3 = proportional splits")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world = _dist_env()[0]
    if world > 1 and args.gpus != world:
        ap.error(f"--gpus {args.gpus} does not match WORLD_SIZE={world}")
    line = run_reference(args) if args.impl == "reference" else run_ours(args)
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
