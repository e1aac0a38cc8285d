#!/usr/bin/env python
"""Throughput of the fused ZeRO-DP shard step on B200.

Default workload: GPT-2 1.5B-shaped parameters (48 layers, d = 1600, vocab
50257: Psi = 1,557,611,200) at data-parallel degree Nd = 8, stage-2 layout
(every simulated rank holds a full fp16 gradient), AdamW (wd 0.01), loss
scale 65536, speculative mode.  One step = the whole hot path over all
Nd owners: reduce-scatter sum of the 8 contributions, unscale, overflow check,
Adam on the fp32 master/momentum/variance and the fp16 cast into the
all-gathered parameter buffer.

Prints one JSON line (rank 0).  ``value`` is owned parameters updated per
second over all ranks with inputs resident in HBM; ``e2e`` repeats the
measurement through the C-ABI call with the step's gradients copied from
pinned host memory every step and the step's product (the updated 16-bit
parameters) and its result struct copied back; ``roofline``
reports the update kernel's algorithmic bytes per launch over its CUDA-event
duration against the measured HBM copy bandwidth; ``sustained`` repeats the
step back to back for a few seconds and reports the update kernel over the
last third, at the SM clock the power cap settles on; ``configs`` measures the
other named workloads and the sweep's >= 1B points in the same run;
``cpu_baseline`` times the CPU oracle on a bounded sample on this host.

``--peer`` runs the same step through peer tables with the Nd ranks' buffers
in this GPU's memory: each rank's gradient read through the table, every new
parameter stored into all Nd full parameter buffers (the all-gather by
stores), which adds 2 (Nd - 1) bytes per parameter.

``--dynamic-scale`` keeps the loss scale in the device optimizer state
(dynamic loss scaling) instead of the hyper-parameters; the step's bytes do
not change.

``--layer-gather`` measures the stage-3 schedule instead: the GPT-2
1.5B-shaped tensor list at Nd = 8, every layer gathered from the owners'
fp16 shards into a compact buffer while the previous one is in use, forward
then backward (2 Psi elements gathered per pass pair, 4 bytes each); then
the same schedule with a matrix product per layer as the layer's work, to
show how much of the gathering the prefetch hides; both with the copy kernel
and with the copy engines (``engine="dma"``).

``--retain`` runs the stage-2 variant with gradient retention: per step the
reduce-scatter keeps the owners' reduced gradients in 16 bits
(``zero_reduce_scatter``, 2 Nd + 2 bytes per parameter) and the step reads
that kept shard as its one contribution (28 bytes per parameter).

Multi-GPU (``torchrun --nproc-per-node N bench.py --gpus N``): the path has
no data exchange on one GPU, so N ranks run independent replicas (weak
scaling); the only collectives are the timing barrier and the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "fused ZeRO shard-step params/s and achieved HBM GB/s (fraction of B200 peak)"
UNIT = "params/s"
STORAGES = {"fp16": 0, "bf16": 1}   # the library's ZERO_STORAGE_* codes
FALLBACK_HBM_GBS = 6650.0  # used only if MEASURED_PEAKS.json is absent


def _workloads():
    from zero_dp_partitioned_shard_b200 import binding as B
    from zero_dp_partitioned_shard_b200 import synth
    return {
        "gpt2-1.5b-stage2-nd8": dict(
            desc="GPT-2 1.5B-shaped (48L d1600 vocab 50257, Psi=1,557,611,200), stage 2, Nd=8, "
                 "AdamW wd 0.01, loss scale 65536, speculative mode",
            sizes=synth.gpt2_xl_tensor_sizes, nd=8, stage=2, align=256, bucket=0, S=65536.0,
            wd=0.01, clip=0.0, mode=B.ZERO_MODE_SPECULATIVE, layout=B.ZERO_GRADS_FULL,
            owner_first=0, owner_count=None),
        "24l-d2048-stage2-nd16-clip": dict(
            desc="24-layer d2048 transformer (Psi=1,315,723,264), stage 2, Nd=16, 25M-element "
                 "buckets, global-norm clip 1.0, loss scale 65536, stash mode",
            sizes=synth.transformer_24l_d2048_tensor_sizes, nd=16, stage=2, align=256,
            bucket=25_000_000, S=65536.0, wd=0.0, clip=1.0, mode=B.ZERO_MODE_STASH,
            layout=B.ZERO_GRADS_FULL, owner_first=0, owner_count=None),
        "7.5b-nd64-stage3-owner0": dict(
            desc="stage-3 one-rank view of 7.5B params at Nd=64: owner 0's shard "
                 "(L=117,187,584) with 64 fp16 contributions, speculative mode",
            sizes=None, psi=7_500_000_000, nd=64, stage=3, align=256, bucket=0, S=1.0, wd=0.0,
            clip=0.0, mode=B.ZERO_MODE_SPECULATIVE, layout=B.ZERO_GRADS_PER_OWNER,
            owner_first=0, owner_count=1, assemble=True),
    }


def bytes_per_param(nd: int, mode: int) -> tuple[int, int]:
    """(algorithmic, moved-by-mode) bytes per owned parameter of one step."""
    alg = 2 * nd + 26  # Nd fp16 reads, master/m/v read+write (24), fp16 write (2)
    moved = {0: alg, 1: 4 * nd + 26, 2: 2 * nd + 34}[mode]
    return alg, moved


def pipeline_min_elems(nd: int, sms: int = 148) -> int:
    """Smallest launch (elements) with which the library's pipelined update
    gives every CTA 64 tiles, for 4 <= Nd <= 64: tiles of 256 x EPT elements,
    SMs x CTAs per SM CTAs (the shapes of the library's pipe_shape; the
    2-byte result region of the bulk-store shapes, Nd 5-11, still leaves room
    for 3 CTAs)."""
    if nd <= 16:
        ept, ctas = 4, (3 if nd <= 12 else 2)
    else:
        e = 12 + 2 * nd
        ept = 2 if 2 * (1024 + 2 * 256 * 2 * e + 1024) <= 228 * 1024 else 1
        smem = 1024 + 2 * 256 * ept * e
        ctas = 3
        while ctas > 1 and ctas * (smem + 1024) > 228 * 1024:
            ctas -= 1
    return 64 * 256 * ept * sms * ctas


def update_kernel_name(nd: int, mode: int, peer: bool = False, elems: int = 1 << 30) -> str:
    """The library's update kernel for this source: the bulk-copy pipeline for
    the stash, and for up to 64 contributions (up to 16 through peer tables;
    from Nd = 4 only for launches that give every CTA at least 64 tiles); the
    register path otherwise (larger Nd, small launches)."""
    max_nd = 16 if peer else 64
    if mode == 2 or nd <= 3 or (nd <= max_nd and elems >= pipeline_min_elems(nd)):
        return "zs_update_pipe_kernel"
    return "zs_update_kernel"


def launched_update_kernel(B, fallback: str) -> tuple:
    """The update kernel of the last step, from the library's launch record:
    (short name, mangled symbol, "launch record"), or (fallback, None, "shape
    rule") when the record holds no update kernel."""
    for sym in reversed(B.zero_recent_kernels(16)):
        for short in ("zs_update_pipe_kernel", "zs_update_kernel"):
            if short + "I" in sym or short + "<" in sym:
                return short, sym, "launch record"
    return fallback, None, "shape rule"


def update_launch_bytes(nd: int, mode: int, dests: int = 0) -> int:
    """Algorithmic bytes per parameter of the update kernel's own launch: the
    fused kernel reads the Nd contributions (speculative, two-pass) or the
    4-byte stash (stash), plus master/m/v read and write and the fp16 write
    (to the parameter buffer and to each of `dests` more)."""
    return (4 if mode == 2 else 2 * nd) + 26 + 2 * dests


def profiled_traffic(nd: int, mode: int, owned: int):
    """DRAM bytes (read + write) of one update-kernel launch, from a committed
    ncu summary under profiles/ that was captured on the current kernel source
    with the same Nd and mode, scaled to this launch by its parameters.  None
    when no such summary exists (for instance after the kernel changed)."""
    import glob
    import hashlib
    src = os.path.join(ROOT, "zero_dp_partitioned_shard_b200", "csrc", "kernels.cu")
    try:
        sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    except OSError:
        return None, None
    mode_name = {0: "speculative", 1: "two_pass", 2: "stash"}[mode]
    for path in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md"))):
        kv = {}
        for line in open(path):
            if ":" in line and not line.startswith(("|", " ", "#")):
                k, v = line.split(":", 1)
                kv[k.strip()] = v.strip()
        if (kv.get("kernels_cu_sha256_prefix") == sha and kv.get("traffic_nd") == str(nd)
                and kv.get("traffic_mode") == mode_name and "traffic_bytes_per_param" in kv):
            return float(kv["traffic_bytes_per_param"]) * owned, os.path.relpath(path, ROOT)
    return None, None


def measured_hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled in the background."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        self.t0 = time.time()

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for r in rows for k in range(4) if r[5 + k].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


class Bench:
    """Device buffers and the C-ABI arguments of one workload on one GPU."""

    def __init__(self, wl: dict, psi_override: int | None, seed: int, storage: int = 0, peer: bool = False,
                 retain: bool = False, dynamic_scale: bool = False):
        import torch
        from zero_dp_partitioned_shard_b200 import binding as B
        from zero_dp_partitioned_shard_b200 import synth
        self.B, self.torch = B, torch
        sizes = wl["sizes"]() if wl.get("sizes") else None
        psi = psi_override or (sum(sizes) if sizes else wl["psi"])
        if psi_override:
            sizes = None
        self.wl, self.psi, self.nd = wl, psi, wl["nd"]
        self.plan = B.zero_plan(psi, self.nd, stage=wl["stage"], align_elems=wl["align"],
                                bucket_elems=wl["bucket"], tensor_sizes=sizes)
        info = B.zero_plan_query(self.plan)
        L = self.L = info.shard_len
        o0 = wl["owner_first"]
        oc = self.nd if wl["owner_count"] is None else wl["owner_count"]
        self.o0, self.oc = o0, oc
        lo, hi = o0 * L, min((o0 + oc) * L, psi)
        self.owned = hi - lo
        n_state = oc * L
        dev = torch.device("cuda")
        spec = wl["mode"] == B.ZERO_MODE_SPECULATIVE
        self.storage = storage
        h16 = torch.bfloat16 if storage == B.ZERO_STORAGE_BF16 else torch.float16
        # gradient contributions
        if wl["layout"] == B.ZERO_GRADS_FULL:
            stride = info.psi_pad
            self.grads = torch.empty(self.nd * stride, dtype=h16, device=dev)
            for r in range(self.nd):
                row = self.grads[r * stride:(r + 1) * stride]
                synth.fill_normal_(row[:psi], seed=seed * 1000 + r, std=1e-3, scale=wl["S"])
                row[psi:].zero_()
        else:
            stride = L
            self.grads = torch.empty(oc * self.nd * L, dtype=h16, device=dev)
            synth.fill_normal_(self.grads, seed=seed * 1000, std=1e-3, scale=wl["S"])
        self.stride = stride
        self.grad_bytes = self.grads.numel() * 2
        f32 = lambda: torch.zeros(n_state, dtype=torch.float32, device=dev)
        self.master = [synth.fill_normal_(f32(), seed=seed * 1000 + 999, std=0.02),
                       f32() if spec else None]
        self.exp_avg = [f32(), f32() if spec else None]
        self.exp_avg_sq = [f32(), f32() if spec else None]
        self.stash = f32() if wl["mode"] == B.ZERO_MODE_STASH else None
        self.params = torch.zeros(psi, dtype=h16, device=dev)
        stream = torch.cuda.current_stream().cuda_stream
        B.zero_cast_params(self.plan, self.master[0].data_ptr(), self.params.data_ptr(), o0, oc, stream,
                           storage=storage)
        self.opt_state = torch.zeros(B.OPT_STATE_BYTES, dtype=torch.uint8, device=dev)
        self.result = torch.zeros(B.RESULT_BYTES, dtype=torch.uint8, device=dev)
        if dynamic_scale:    # the loss scale lives in the device optimizer state
            B.zero_opt_state_init_dynamic(self.opt_state.data_ptr(), wl["S"], 2.0, 0.5, 2000, stream)
        else:
            B.zero_opt_state_init(self.opt_state.data_ptr(), stream)
        self.hp = B.hparams(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=wl["wd"],
                            loss_scale=wl["S"], max_grad_norm=wl["clip"], mode=wl["mode"])
        ptr = lambda t: t.data_ptr() if t is not None else 0
        self.args = B.step_args(
            grads=self.grads.data_ptr(), grad_rank_stride=stride, grad_layout=wl["layout"],
            owner_first=o0, owner_count=oc, master=tuple(ptr(t) for t in self.master),
            exp_avg=tuple(ptr(t) for t in self.exp_avg),
            exp_avg_sq=tuple(ptr(t) for t in self.exp_avg_sq), params=self.params.data_ptr(),
            grad_stash=ptr(self.stash), opt_state=self.opt_state.data_ptr(),
            result=self.result.data_ptr(), storage=storage)
        # stage-3 view: after its own update the rank assembles the full fp16
        # buffer from the other owners' (seeded) parameter shards
        self.shards, self.shard_ptrs, self.assembled = None, None, 0
        if wl.get("assemble"):
            others = [r for r in range(self.nd) if not (o0 <= r < o0 + oc)]
            self.shards = torch.empty(len(others), L, dtype=h16, device=dev)
            for k, r in enumerate(others):
                synth.fill_normal_(self.shards[k], seed=seed * 1000 + 500 + r, std=0.02)
            self.shard_ptrs = [0] * self.nd
            for k, r in enumerate(others):
                self.shard_ptrs[r] = self.shards[k].data_ptr()
            self.assembled = sum(max(0, min(L, psi - r * L)) for r in others)
        # peer tables: rank r's gradient is row r, every rank has its own full
        # parameter buffer (the call's params plus Nd - 1 destinations)
        self.dests = []
        if peer:
            if wl["layout"] != B.ZERO_GRADS_FULL:
                raise ValueError("--peer needs a workload with full per-rank gradients")
            self.dests = [torch.zeros(psi, dtype=h16, device=dev) for _ in range(self.nd - 1)]
            rank_grads = [self.grads.data_ptr() + 2 * r * stride for r in range(self.nd)]
            B.attach_peers(self.args, B.peer_args(rank_grads, [t.data_ptr() for t in self.dests]))
        # stage-2 retention: the reduce-scatter reads the contributions, the
        # step reads the owners' kept 16-bit shards
        self.retain_args, self.kept = None, None
        if retain:
            if peer or wl.get("assemble"):
                raise ValueError("--retain runs the plain stage-2 layouts")
            self.kept = torch.empty(n_state, dtype=h16, device=dev)
            self.retain_args = B.step_args(
                grads=self.grads.data_ptr(), grad_rank_stride=stride, grad_layout=wl["layout"],
                owner_first=o0, owner_count=oc, master=(0, 0), exp_avg=(0, 0), exp_avg_sq=(0, 0),
                params=0, opt_state=0, storage=storage)
            self.args.grads = self.kept.data_ptr()
            self.args.grad_layout = B.ZERO_GRADS_REDUCED
            self.args.grad_rank_stride = 0
            self.reduce_events = None
        ws_bytes = B.zero_workspace_bytes(self.plan, self.hp, self.args)
        self.workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
        self.args.workspace = self.workspace.data_ptr()
        self.args.workspace_bytes = ws_bytes
        self.stream = stream
        torch.cuda.synchronize()

    def step(self, events=None):
        if events is not None:
            self.args.timing_events[0] = events[0].cuda_event
            self.args.timing_events[1] = events[1].cuda_event
        else:
            self.args.timing_events[0] = None
            self.args.timing_events[1] = None
        if self.retain_args is not None:
            if events is not None and len(events) > 2:
                events[2].record()
            self.B.zero_reduce_scatter(self.plan, self.retain_args, self.kept.data_ptr(), -1, self.stream)
            if events is not None and len(events) > 2:
                events[3].record()
        self.B.zero_shard_step(self.plan, self.hp, self.args, self.stream)
        if self.shard_ptrs is not None:
            self.B.zero_gather_params(self.plan, self.shard_ptrs, self.params.data_ptr(), self.stream)

    def close(self):
        self.B.zero_plan_destroy(self.plan)


def timed_steps(bench, steps: int, warmup: int, world: int, local: int, n_ev: int = 2,
                inject: dict | None = None) -> dict:
    """Warm-up, then ``steps`` steps timed on the device: CUDA events around the
    whole region (bracketed by a barrier and a synchronize on both sides) and
    around each step's update launches; SM clocks sampled during the region.
    inject: {step: (rank, flat index, value)} -- the value is planted in that
    rank's gradient before the step and the old value put back after it (a
    seeded overflow schedule: the step must be skipped).  Returns the region's
    ms, the per-step update-kernel ms of the applied steps, the skipped count,
    the library's launches and the clocks."""
    import torch
    from zero_dp_partitioned_shard_b200 import binding as B
    for _ in range(warmup):
        bench.step()
    k_events = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(n_ev)) for _ in range(steps)]
    for evs in k_events:    # create the CUDA events before handing their handles over
        for ev in evs:
            ev.record()
    inject = inject or {}
    if inject and bench.wl["layout"] != 0:
        raise ValueError("the injection schedule addresses the full per-rank gradient layout")
    planted = {}
    for k, (rank, i, val) in inject.items():
        if k < steps:
            flat = rank * bench.stride + i
            planted[k] = (flat, bench.grads[flat:flat + 1].clone(), val)
    skipped0 = B.opt_state_from_bytes(bench.opt_state.cpu().numpy().tobytes()).skipped
    torch.cuda.synchronize()
    _barrier(world)
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    launches0 = B.zero_launch_count()
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_start.record()
    for k in range(steps):
        hit = planted.get(k)
        if hit is not None:
            bench.grads[hit[0]] = hit[2]
        bench.step(k_events[k])
        if hit is not None:
            bench.grads[hit[0]:hit[0] + 1].copy_(hit[1])
    t_end.record()
    torch.cuda.synchronize()
    launches = B.zero_launch_count() - launches0
    clk = clocks.stop()
    _barrier(world)
    skipped = B.opt_state_from_bytes(bench.opt_state.cpu().numpy().tobytes()).skipped - skipped0
    return {"ms_total": t_start.elapsed_time(t_end), "launches": launches, "clocks": clk,
            "skipped": skipped, "injected": len(planted),
            "kernel_ms": [ev[0].elapsed_time(ev[1]) for k, ev in enumerate(k_events) if k not in planted],
            "reduce_ms": [ev[2].elapsed_time(ev[3]) for ev in k_events] if n_ev > 2 else []}


def _dist():
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(local)
    return world, rank, local


def max_over_ranks(x: float, world: int, device: str = "cuda") -> float:
    """Max of a per-rank scalar over all ranks (every rank gets it)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(owned: int, steps: int, ms_local: float, world: int, device: str = "cuda"):
    """Whole-job throughput: parameters updated by all ranks over the slowest
    rank's device time.  Returns (ms_max, params_per_second)."""
    ms_max = max_over_ranks(ms_local, world, device)
    return ms_max, world * owned * steps / (ms_max / 1e3)


def _barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def _draw_grads(storage: int):
    from zero_dp_partitioned_shard_b200 import synth
    return synth.grads_bf16 if storage == 1 else synth.grads_f16


def host_cpu() -> dict:
    """The host's logical CPU count and model name (from /proc/cpuinfo; None
    where it is not readable)."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"host_cpus": os.cpu_count(), "cpu_model": model}


def cpu_baseline(wl: dict, budget_s: float, sample_psi: int, threads: int, storage: int = 0) -> dict:
    """The CPU oracle, as it stands, on a bounded sample of the workload."""
    import oracle
    from zero_dp_partitioned_shard_b200 import synth
    nd = wl["nd"]
    G = _draw_grads(storage)(nd, sample_psi, seed=5, std=1e-3, scale=wl["S"])
    master = synth.normal_f32(sample_psi, seed=6, std=0.02)
    m = np.zeros(sample_psi, np.float32)
    v = np.zeros(sample_psi, np.float32)
    P = np.zeros(sample_psi, np.uint16)
    hp = oracle.HP(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=wl["wd"],
                   loss_scale=wl["S"], max_grad_norm=wl["clip"], storage=storage)
    opt = oracle.Opt()
    steps, t0 = 0, time.perf_counter()
    while True:
        oracle.step(G, master, m, v, P, hp, opt, threads=threads)
        steps += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    alg, _ = bytes_per_param(nd, 0)
    return {"value": sample_psi * steps / el, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{steps} oracle steps over {sample_psi:,} params x Nd={nd} "
                      f"(same hyper-parameters), {el:.1f} s, OpenMP threads={threads}",
            "gbs_alg": sample_psi * steps * alg / el / 1e9, **host_cpu()}


def run_reference(args, wl_name: str, wl: dict):
    """Reference arm: the CPU oracle timed on this host, on bounded samples."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    from zero_dp_partitioned_shard_b200 import synth
    threads = oracle.host_threads()
    nd = wl["nd"]
    sample = args.ref_sample
    storage = STORAGES[args.storage]
    G = _draw_grads(storage)(nd, sample, seed=5, std=1e-3, scale=wl["S"])
    master = synth.normal_f32(sample, seed=6, std=0.02)
    m = np.zeros(sample, np.float32)
    v = np.zeros(sample, np.float32)
    P = np.zeros(sample, np.uint16)
    hp = oracle.HP(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=wl["wd"],
                   loss_scale=wl["S"], max_grad_norm=wl["clip"], storage=storage)
    opt = oracle.Opt()
    for _ in range(args.warmup):
        oracle.step(G, master, m, v, P, hp, opt, threads=threads)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.step(G, master, m, v, P, hp, opt, threads=threads)
    el = time.perf_counter() - t0
    value = sample * args.steps / el
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": wl_name, "description": wl["desc"], "psi": _psi_of(wl),
                   "nd": nd, "storage": args.storage, "sample_params_per_step": sample},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": f"{args.steps} steps over {sample:,} params x Nd={nd}", **host_cpu()},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def step_alg_bytes(owned: int, assembled: int, nd: int, steps: int, skipped: int) -> int:
    """Algorithmic bytes of ``steps`` steps of which ``skipped`` were skipped on
    overflow: an applied step moves (2 Nd + 26) B per owned parameter plus 4 B
    per assembled one; a skipped step has still read every contribution
    (2 Nd B per owned parameter) and updates nothing."""
    return (steps - skipped) * (owned * (2 * nd + 26) + 4 * assembled) + skipped * owned * 2 * nd


def config_entry(name: str, wl: dict, args, world: int, local: int, peak: float, seed: int,
                 inject_rate: float = 0.0, min_ms: float = 400.0) -> dict:
    """One more workload measured in the same run as the headline: its step
    time, its update kernel's CUDA-event time against the kernel's own
    algorithmic bytes, and the whole step's fraction by the workload's
    algorithmic bytes (assembly included).  The timed steps are at least
    ``args.steps`` and enough for about ``min_ms`` of device time, so the clock
    sampler sees the region.  inject_rate > 0 plants a seeded overflow
    schedule (that share of steps, the first timed step always) in the timed
    region; skipped steps move only their gradient reads."""
    import torch
    from zero_dp_partitioned_shard_b200 import synth
    torch.cuda.empty_cache()
    bn = Bench(wl, None, seed=seed)
    try:
        for _ in range(args.warmup):
            bn.step()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        bn.step()
        b.record()
        torch.cuda.synchronize()
        one = max(a.elapsed_time(b), 1e-3)
        steps = max(args.steps, int(math.ceil(min_ms / one)))
        steps = int(max_over_ranks(float(steps), world))
        inject = None
        if inject_rate > 0:
            inject = synth.inject_schedule(steps, inject_rate, seed=seed * 7 + 1, nd=bn.nd, psi=bn.psi,
                                           force_step=0)
        tr = timed_steps(bn, steps, 3, world, local, inject=inject)
        k_name, k_sym, k_src = launched_update_kernel(bn.B, update_kernel_name(wl["nd"], wl["mode"], False, bn.owned))
        ms_max = max_over_ranks(tr["ms_total"], world)
        k_ms = max_over_ranks(statistics.mean(tr["kernel_ms"]), world)
        nd, mode = wl["nd"], wl["mode"]
        alg, moved = bytes_per_param(nd, mode)
        k_bytes = bn.owned * update_launch_bytes(nd, mode)
        step_bytes = step_alg_bytes(bn.owned, bn.assembled, nd, steps, tr["skipped"])
        achieved = k_bytes / (k_ms / 1e3) / 1e9
        step_gbs = step_bytes / (ms_max / 1e3) / 1e9
        return {
            "workload": name, "description": wl["desc"], "psi": bn.psi, "nd": nd, "stage": wl["stage"],
            "mode": {0: "speculative", 1: "two_pass", 2: "stash"}[mode], "owned_params": bn.owned,
            "assembled_params": bn.assembled, "steps": steps, "skipped_steps": tr["skipped"],
            "injected_steps": tr["injected"], "ms_per_step": ms_max / steps,
            "params_per_s": world * bn.owned * steps / (ms_max / 1e3),
            "bytes_per_param_alg": alg, "bytes_per_param_moved": moved,
            "update_kernel_ms": k_ms,
            "roofline": {"bound": "hbm", "kernel": k_name, "kernel_symbol": k_sym, "kernel_source": k_src,
                         "alg_bytes_per_launch": k_bytes,
                         "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak},
            "step": {"alg_bytes": step_bytes, "gbs": step_gbs, "frac": step_gbs / peak,
                     "bytes": "applied steps: owned x (2 Nd + 26) + 4 x assembled; skipped steps: "
                              "owned x 2 Nd"},
            "gpu_launches": tr["launches"], "clocks": tr["clocks"],
        }
    finally:
        bn.close()
        del bn
        torch.cuda.empty_cache()


CONFIG_SWEEP = [(1 << 30, 1), (1 << 30, 8), (1 << 30, 64), (2 << 30, 1), (2 << 30, 8), (2 << 30, 64)]


def run_configs(args, world: int, local: int, peak: float) -> list:
    """The other named workloads and the sweep's >= 1B points, each allocated,
    measured and freed in turn after the headline."""
    import torch
    wls = _workloads()
    out = [config_entry("7.5b-nd64-stage3-owner0", wls["7.5b-nd64-stage3-owner0"], args, world, local,
                        peak, seed=21),
           config_entry("24l-d2048-stage2-nd16-clip", wls["24l-d2048-stage2-nd16-clip"], args, world, local,
                        peak, seed=22, inject_rate=0.01)]
    for psi, nd in CONFIG_SWEEP:
        torch.cuda.empty_cache()
        free, _ = torch.cuda.mem_get_info()
        wl = sweep_workload(psi, nd, 1, int(max_over_ranks(-float(free), world) * -1))
        e = config_entry(f"sweep-psi{psi}-nd{nd}-stage1", wl, args, world, local, peak, seed=23 + nd)
        e["view"] = "owner0" if wl["owner_count"] == 1 else "all owners"
        out.append(e)
    return out


SWEEP_PSI = [1 << 20, 16 << 20, 256 << 20, 1 << 30, 2 << 30]
SWEEP_ND = [1, 2, 8, 64]


def sweep_workload(psi: int, nd: int, stage: int, free_bytes: int, mode: int = 0) -> dict:
    """One sweep point: speculative, no clipping; stage 1 = full gradients in one
    pass, stage 2 = the same in 8 buckets, stage 3 = per-owner contributions.
    All Nd owners are simulated when Psi*(2*Nd + 26) bytes fit in 80 % of free
    HBM; otherwise owner 0's view (the same bytes per parameter)."""
    from zero_dp_partitioned_shard_b200 import binding as B
    full_bytes = psi * (2 * nd + 26 + (4 if mode == B.ZERO_MODE_STASH else 0)) + (1 << 28)
    one_owner = full_bytes > 0.8 * free_bytes
    bucket = 0
    if stage == 2:
        bucket = -(-psi // (8 * 256)) * 256
    return dict(desc=f"sweep psi={psi} nd={nd} stage={stage}" + (" owner-0 view" if one_owner else ""),
                sizes=None, psi=psi, nd=nd, stage=stage, align=256, bucket=bucket, S=1.0, wd=0.0,
                clip=1.0 if mode != B.ZERO_MODE_SPECULATIVE else 0.0, mode=mode,
                # a one-owner view holds only its own slice of each rank's gradient
                layout=B.ZERO_GRADS_PER_OWNER if (stage == 3 or one_owner) else B.ZERO_GRADS_FULL,
                owner_first=0, owner_count=1 if one_owner else None)


def run_sweep(args) -> int:
    """Update-kernel GB/s against bytes per parameter over the sweep grid; one
    JSON line per point (measurement mode, not the benchmark line)."""
    import torch
    world, rank, local = _dist()
    peak, peak_kind = measured_hbm_peak()
    ints = lambda text, default: [int(x) for x in text.split(",")] if text else default
    modes = {"speculative": 0, "two_pass": 1, "stash": 2}
    for psi in ints(args.sweep_psi, SWEEP_PSI):
        for nd in ints(args.sweep_nd, SWEEP_ND):
          for mode_name in (args.sweep_mode or "speculative").split(","):
            for stage in ints(args.sweep_stage, [1, 2, 3]):
                torch.cuda.empty_cache()
                free, _ = torch.cuda.mem_get_info()
                wl = sweep_workload(psi, nd, stage, free, modes[mode_name])
                bn = Bench(wl, None, seed=7)
                for _ in range(args.warmup):
                    bn.step()
                ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                      for _ in range(args.steps)]
                for a, b in ev:
                    a.record()
                    b.record()
                t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                torch.cuda.synchronize()
                t0.record()
                for k in range(args.steps):
                    bn.step(ev[k])
                t1.record()
                torch.cuda.synchronize()
                k_ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
                step_ms = t0.elapsed_time(t1) / args.steps
                alg = update_launch_bytes(nd, wl["mode"])
                gbs = bn.owned * alg / (k_ms / 1e3) / 1e9
                if rank == 0:
                    print(json.dumps({"sweep": True, "psi": psi, "nd": nd, "stage": stage,
                                      "mode": mode_name,
                                      "view": "owner0" if wl["owner_count"] == 1 else "all owners",
                                      "owned": bn.owned, "bytes_per_param": alg,
                                      "kernel_ms": k_ms, "step_ms": step_ms, "gbs": gbs,
                                      "frac": gbs / peak, "peak": peak, "peak_kind": peak_kind,
                                      "params_per_s": bn.owned / (step_ms / 1e3)}), flush=True)
                bn.close()
                del bn
    return 0


def run_layer_gather(args) -> int:
    """Stage-3 on-demand gathering: forward + backward passes of the per-layer
    schedule over the GPT-2 1.5B-shaped tensor list at Nd = 8, with the copy
    kernel and with the copy engines (one JSON line, measurement mode)."""
    import torch
    from zero_dp_partitioned_shard_b200 import binding as B
    from zero_dp_partitioned_shard_b200 import synth
    from zero_dp_partitioned_shard_b200.stage3 import LayerGatherSchedule
    world, rank, local = _dist()
    sizes = synth.gpt2_xl_tensor_sizes()
    psi, nd = sum(sizes), 8
    peak, peak_kind = measured_hbm_peak()
    plan = B.zero_plan(psi, nd, stage=3, align_elems=256, tensor_sizes=sizes)
    try:
        L = B.zero_plan_query(plan).shard_len
        shards = torch.empty(nd, L, dtype=torch.float16, device="cuda")
        for o in range(nd):
            synth.fill_normal_(shards[o], seed=600 + o, std=0.02)
        per_layer = 12                                   # LN1, QKV, proj, LN2, MLP up and down (+ biases)
        n_layer = (len(sizes) - 4) // per_layer
        layers = [(i * per_layer, per_layer) for i in range(n_layer)] + [(n_layer * per_layer, 4)]
        order = list(range(len(layers))) + list(reversed(range(len(layers))))
        nothing = lambda layer, params: None             # no model: the data movement alone
        # the layer's work for the overlap measurement: an activation times the
        # layer's gathered QKV weight (a stand-in for its forward compute)
        d_model, qkv_off = 1600, 2 * 1600
        x = torch.randn(8192, d_model, dtype=torch.float16, device="cuda")
        y = torch.empty(8192, 3 * d_model, dtype=torch.float16, device="cuda")

        def use_mm(layer, params):
            off = qkv_off if layer < n_layer else 0
            torch.matmul(x, params[off:off + d_model * 3 * d_model].view(d_model, 3 * d_model), out=y)

        def timed(fn):
            for _ in range(args.warmup):
                fn()
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            for _ in range(args.steps):
                fn()
            b.record()
            torch.cuda.synchronize()
            return max_over_ranks(a.elapsed_time(b), world) / args.steps

        def measure(engine):
            sched = LayerGatherSchedule(plan, layers, [shards[o].data_ptr() for o in range(nd)], sizes,
                                        engine=engine)
            passes = lambda use: (sched.forward(use), sched.backward(use))
            gathered0 = sched.gathered
            passes(nothing)
            elems = (sched.gathered - gathered0) * world
            eager_ms = timed(lambda: passes(nothing))
            graphs = [sched.capture(range(len(layers)), nothing),
                      sched.capture(reversed(range(len(layers))), nothing)]
            graph_ms = timed(lambda: [gr.replay() for gr in graphs])
            del graphs
            fixed = sched.buffers[0][:max(sched.sizes)]
            compute_ms = timed(lambda: [use_mm(i, fixed) for i in order])
            both_ms = timed(lambda: passes(use_mm))
            frac = lambda t: elems * 4 / (t / 1e3) / 1e9 / peak
            return {"eager_ms": eager_ms, "eager_frac": frac(eager_ms), "graph_ms": graph_ms,
                    "graph_frac": frac(graph_ms), "elems": elems,
                    "overlap_with_compute": {"compute_only_ms": compute_ms, "both_ms": both_ms,
                                             "hidden_fraction_of_gather": (compute_ms + eager_ms - both_ms) / eager_ms}}

        _barrier(world)
        clocks = ClockSampler(local)
        clocks.start()
        time.sleep(0.3)
        launches0 = B.zero_launch_count()
        res = {engine: measure(engine) for engine in ("kernel", "dma")}
        launches = B.zero_launch_count() - launches0
        clk = clocks.stop()
        k = res["kernel"]
        if rank == 0:
            print(json.dumps({
                "mode": "layer_gather", "metric": "stage-3 gathered fp16 parameters per second",
                "value": k["elems"] / (k["eager_ms"] / 1e3), "unit": "params/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": k["eager_ms"], "higher_is_better": True,
                "config": {"workload": "gpt2-1.5b-stage3-nd8-layers", "psi": psi, "nd": nd, "layers": len(layers),
                           "step": "forward + backward pass of the gather schedule (2 Psi elements)",
                           "bytes_per_param": 4,
                           "use": "per layer: [8192, 1600] x [1600, 4800] fp16 matmul with the gathered QKV weight"},
                "roofline": {"bound": "hbm", "achieved": k["eager_frac"] * peak, "peak": peak, "unit": "GB/s",
                             "frac": k["eager_frac"], "peak_source": f"{peak_kind} hbm_gbs (copy)"},
                "gpu_launches": launches, "clocks": clk,
                "engines": res}), flush=True)
        del shards
    finally:
        B.zero_plan_destroy(plan)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


LINK_GBS = 770.0   # measured peer copy per direction over NVLink 5 on this part (900 nominal)


class HostTimer:
    """Wall clock of a region on the host (the CPU harness tests' timer)."""

    def start(self):
        self.t0 = time.perf_counter()

    def stop(self) -> float:
        return (time.perf_counter() - self.t0) * 1e3


class DeviceTimer:
    """CUDA events on the current stream around a region."""

    def __init__(self):
        import torch
        self.torch = torch
        self.a = torch.cuda.Event(enable_timing=True)
        self.b = torch.cuda.Event(enable_timing=True)

    def start(self):
        self.a.record()

    def stop(self) -> float:
        self.b.record()
        self.torch.cuda.synchronize()
        return self.a.elapsed_time(self.b)


def sharded_loop(step, steps: int, warmup: int, world: int, timer, sync=lambda: None,
                 device: str = "cuda") -> float:
    """Warm-up, then ``steps`` calls of ``step(k)`` timed by ``timer``,
    bracketed by a barrier and ``sync`` on both sides; returns the slowest
    rank's ms (every rank takes the same collective steps)."""
    for k in range(warmup):
        step(-1 - k)
    sync()
    _barrier(world)
    sync()
    timer.start()
    for k in range(steps):
        step(k)
    ms = timer.stop()
    _barrier(world)
    return max_over_ranks(ms, world, device)


def sharded_report(psi: int, world: int, L: int, steps: int, ms_max: float, k_ms_max: float | None,
                   transport: str, peak: float, comm: dict) -> dict:
    """What a step with one owner per process moves, against its bounds.

    Per process and step, the reduce-scatter's input sends (Nd-1) gradient
    slices of L elements and receives as many; the all-gather sends the own
    fp16 shard to the Nd-1 others and receives theirs: 2 (Nd-1) L elements,
    4 (Nd-1) L bytes, each way -- the 2 Psi of stages 1 and 2 on the ring,
    plus padding.  The link bound is those bytes at LINK_GBS per direction.
    comm: zero_state_bytes' report of the same Psi, Nd and stage."""
    elems = 2 * (world - 1) * L
    link_bytes = 2 * elems
    step_ms = ms_max / steps
    link_ms = link_bytes / (LINK_GBS * 1e9) * 1e3
    out = {
        "transport": transport, "owners": world, "shard_len": L,
        "exchange": {"elements_each_way": elems, "bytes_each_way": link_bytes,
                     "link_gbs": LINK_GBS, "link_bound_ms": link_ms,
                     "link_frac": (link_ms / step_ms) if step_ms > 0 else None},
        "accounting": {"comm_elems_pages": comm["comm_elems"], "comm_elems_ring": comm["comm_elems_ring"],
                       "exchanged_elems_each_way": elems,
                       "exchanged_over_ring": (elems / comm["comm_elems_ring"])
                       if comm["comm_elems_ring"] else None},
        "step_ms": step_ms,
    }
    if k_ms_max is not None:
        # the owner's update: Nd contributions in, master/m/v read and written, 16-bit out
        k_bytes = L * (2 * world + 26)
        gbs = k_bytes / (k_ms_max / 1e3) / 1e9
        out["update"] = {"kernel_ms": k_ms_max, "alg_bytes": k_bytes, "gbs": gbs, "frac_of_hbm": gbs / peak,
                         "note": "peer transport: the contributions of other ranks and the parameter "
                                 "stores cross NVLink inside this kernel" if transport == "peer" else
                                 "contributions already local after the exchange"}
    return out


def run_sharded(args) -> int:
    """--sharded {nccl,peer} (under torchrun, one process per GPU): the ZeRO-DP
    step with one owner per GPU -- ZeroDPStep (NCCL all-to-all, vote,
    all-gather) or ZeroDPPeerStep (the exchange inside the step's kernels over
    peer memory, no multicast).  Psi is fixed while the owners grow with the
    GPU count, so the scaling is strong."""
    import datetime

    import torch
    import torch.distributed as dist
    from zero_dp_partitioned_shard_b200 import binding as B
    from zero_dp_partitioned_shard_b200 import distributed as D
    from zero_dp_partitioned_shard_b200 import synth
    world, rank, local = _dist()
    if world == 1 and not dist.is_initialized():
        dist.init_process_group("nccl", store=dist.HashStore(), rank=0, world_size=1,
                                timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))
    wl = _workloads()[args.workload]
    if wl["layout"] != B.ZERO_GRADS_FULL:
        raise SystemExit("--sharded runs the workloads with full per-rank gradients")
    psi = args.psi or _psi_of(wl)
    hp = B.hparams(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=wl["wd"], loss_scale=wl["S"],
                   max_grad_norm=wl["clip"], mode=wl["mode"])
    cls = D.ZeroDPStep if args.sharded == "nccl" else D.ZeroDPPeerStep
    st = cls(psi, hp, stage=wl["stage"], bucket=wl["bucket"], align=wl["align"])
    try:
        master = torch.empty(psi, dtype=torch.float32, device="cuda")
        synth.fill_normal_(master, seed=999, std=0.02)
        st.load_master(master)
        del master
        grad = st.grads if args.sharded == "peer" else torch.empty(st.psi_pad, dtype=torch.float16,
                                                                     device="cuda")
        synth.fill_normal_(grad[:psi], seed=1000 + rank, std=1e-3, scale=wl["S"])
        grad[psi:].zero_()
        k_events = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                    for _ in range(args.steps)]
        for a, b in k_events:
            a.record()
            b.record()

        def one(k):
            evs = k_events[k] if k >= 0 else (None, None)
            st.args.timing_events[0] = evs[0].cuda_event if evs[0] is not None else None
            st.args.timing_events[1] = evs[1].cuda_event if evs[1] is not None else None
            if args.sharded == "nccl":
                st.step(grad)
            else:
                st.step()

        clocks = ClockSampler(local)
        clocks.start()
        launches0 = B.zero_launch_count()
        ms_max = sharded_loop(one, args.steps, args.warmup, world, DeviceTimer(), torch.cuda.synchronize)
        launches = B.zero_launch_count() - launches0
        clk = clocks.stop()
        k_ms_max = max_over_ranks(statistics.mean(a.elapsed_time(b) for a, b in k_events), world)
        peak, peak_kind = measured_hbm_peak()
        rep = sharded_report(psi, world, st.L, args.steps, ms_max, k_ms_max, args.sharded, peak,
                             B.zero_state_bytes(psi, world, wl["stage"], wl["align"]))
        res = B.step_result_from_bytes(st.result.cpu().numpy().tobytes())
        line = {
            "metric": METRIC, "value": psi * args.steps / (ms_max / 1e3), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max / args.steps,
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": {"workload": args.workload, "description": wl["desc"], "psi": psi, "nd": world,
                       "stage": wl["stage"], "sharded": args.sharded,
                       "parallelism": f"ZeRO-DP over {world} process(es), one owner shard per GPU",
                       "peak_source": f"{peak_kind} hbm_gbs (copy)"},
            "sharded": rep, "gpu_launches": launches, "clocks": clk,
            "last_step": {"overflow": res.overflow, "t": res.t},
        }
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        st.close()
        dist.destroy_process_group()
    return 0


def _psi_of(wl):
    return sum(wl["sizes"]()) if wl.get("sizes") else wl["psi"]


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="gpt2-1.5b-stage2-nd8")
    ap.add_argument("--psi", type=int, default=0, help="smaller Psi of the same workload (profiling)")
    ap.add_argument("--storage", choices=sorted(STORAGES), default="fp16",
                    help="16-bit format of gradients and parameters")
    ap.add_argument("--peer", action="store_true",
                    help="through peer tables, storing the parameters into all Nd ranks' buffers")
    ap.add_argument("--dynamic-scale", action="store_true",
                    help="dynamic loss scaling (the scale in the device optimizer state)")
    ap.add_argument("--layer-gather", action="store_true",
                    help="measure the stage-3 per-layer gather schedule (forward + backward)")
    ap.add_argument("--sharded", choices=["nccl", "peer"], default=None,
                    help="one owner per GPU under torchrun: NCCL exchange, or the exchange inside the "
                         "kernels over peer memory (not the default: the default runs replicas)")
    ap.add_argument("--retain", action="store_true",
                    help="stage-2 retention: reduce-scatter into kept 16-bit shards, then the step on them")
    ap.add_argument("--sustained-seconds", type=float, default=3.0,
                    help="after the timed steps, run the step back to back this long and report the update "
                         "kernel at the clock the power cap settles on (0: skip)")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the other named workloads and the >= 1B sweep points ('configs')")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--cpu-sample", type=int, default=1 << 22)
    ap.add_argument("--ref-sample", type=int, default=1 << 21)
    ap.add_argument("--sweep", action="store_true",
                    help="measure the Psi x Nd x stage grid (one JSON line per point)")
    ap.add_argument("--sweep-psi", default="", help="comma-separated Psi values (default: the grid)")
    ap.add_argument("--sweep-nd", default="", help="comma-separated Nd values")
    ap.add_argument("--sweep-stage", default="", help="comma-separated stages")
    ap.add_argument("--sweep-mode", default="", help="speculative,two_pass,stash (default speculative)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.sweep:
        return run_sweep(args)
    if args.layer_gather:
        return run_layer_gather(args)
    if args.sharded and args.impl == "ours":
        return run_sharded(args)
    wls = _workloads()
    if args.workload not in wls:
        ap.error(f"unknown workload {args.workload}; choose from {sorted(wls)}")
    wl = wls[args.workload]
    if args.impl == "reference":
        return run_reference(args, args.workload, wl)

    import torch
    from zero_dp_partitioned_shard_b200 import binding as B
    world, rank, local = _dist()
    bench = Bench(wl, args.psi or None, seed=1 + rank, storage=STORAGES[args.storage], peer=args.peer,
                  retain=args.retain, dynamic_scale=args.dynamic_scale)
    n_dests = len(bench.dests)
    k_nd = 1 if args.retain else wl["nd"]          # contributions the update kernel reads
    alg, moved = bytes_per_param(wl["nd"], wl["mode"])

    # --- device-resident timing ---
    tr = timed_steps(bench, args.steps, args.warmup, world, local, n_ev=4 if args.retain else 2)
    k_name, k_sym, k_src = launched_update_kernel(B, update_kernel_name(k_nd, wl["mode"], bool(n_dests), bench.owned))
    ms, launches, clk = tr["ms_total"], tr["launches"], tr["clocks"]
    ms_max, value = aggregate(bench.owned, args.steps, ms, world)
    k_ms = statistics.mean(tr["kernel_ms"])
    r_ms = statistics.mean(tr["reduce_ms"]) if args.retain else None
    k_ms_max = max_over_ranks(k_ms, world)
    k_ms_median = max_over_ranks(statistics.median(tr["kernel_ms"]), world)
    res = B.step_result_from_bytes(bench.result.cpu().numpy().tobytes())

    # --- sustained: the same step back to back for a few seconds, so that the
    # power cap sets the SM clock as it does inside a training job ---
    sustained = None
    if args.sustained_seconds > 0:
        n_sus = int(max_over_ranks(float(max(10, math.ceil(args.sustained_seconds * 1e3 / (ms / args.steps)))),
                                   world))
        ts = timed_steps(bench, n_sus, 0, world, local)
        k_all = ts["kernel_ms"]
        tail = k_all[len(k_all) * 2 // 3:]          # the last third: the settled clock
        k_sus = max_over_ranks(statistics.mean(tail), world)
        sus_bytes = bench.owned * update_launch_bytes(k_nd, wl["mode"], len(bench.dests))
        sustained = {"seconds": max_over_ranks(ts["ms_total"], world) / 1e3, "steps": n_sus,
                     "update_kernel_ms_last_third": k_sus,
                     "update_kernel_ms_all": max_over_ranks(statistics.mean(k_all), world),
                     "frac_last_third": sus_bytes / (k_sus / 1e3) / 1e9 / measured_hbm_peak()[0],
                     "clocks": ts["clocks"]}

    # --- end to end through the C ABI, host buffers ---
    e2e = None
    if not args.no_e2e:
        import psutil
        need = bench.grad_bytes + bench.params.numel() * 2
        # every rank on this node pins its own copy; all ranks must agree on
        # running the leg, since it holds collectives (barrier, max over ranks)
        n_local = int(os.environ.get("LOCAL_WORLD_SIZE", "1"))
        fits = psutil.virtual_memory().available > 2.5 * need * n_local
        fits = max_over_ranks(0.0 if fits else 1.0, world) == 0.0
        if fits:
            g_host = torch.empty(bench.grads.numel(), dtype=bench.grads.dtype, pin_memory=True)
            g_host.copy_(bench.grads)
            # the step's product: the updated 16-bit parameters (the all-gathered buffer)
            p_host = torch.empty(bench.params.numel(), dtype=bench.params.dtype, pin_memory=True)
            r_host = torch.empty(B.RESULT_BYTES, dtype=torch.uint8, pin_memory=True)
            main = torch.cuda.current_stream()
            side = torch.cuda.Stream()  # the parameter copy of step k beside the gradient copy of step k+1
            p_done = None
            torch.cuda.synchronize()
            for it in range(1 + args.e2e_steps):
                if it == 1:
                    _barrier(world)
                    e0 = torch.cuda.Event(enable_timing=True)
                    e1 = torch.cuda.Event(enable_timing=True)
                    e0.record()
                bench.grads.copy_(g_host, non_blocking=True)
                if p_done is not None:
                    main.wait_event(p_done)  # the step rewrites the parameters the last copy reads
                bench.step()
                r_host.copy_(bench.result, non_blocking=True)
                stepped = torch.cuda.Event()
                stepped.record(main)
                with torch.cuda.stream(side):
                    side.wait_event(stepped)
                    p_host.copy_(bench.params, non_blocking=True)
                    p_done = torch.cuda.Event()
                    p_done.record(side)
                main.synchronize()
                B.step_result_from_bytes(r_host.numpy().tobytes())  # the caller reads the result
            main.wait_event(p_done)  # the last step's parameters are on the host
            e1.record()
            torch.cuda.synchronize()
            e_ms, e_value = aggregate(bench.owned, args.e2e_steps, e0.elapsed_time(e1), world)
            e2e = {"value": e_value, "unit": UNIT,
                   "h2d_bytes_per_step": bench.grad_bytes,
                   "d2h_bytes_per_step": p_host.numel() * p_host.element_size() + B.RESULT_BYTES,
                   "steps": args.e2e_steps, "ms_per_step": e_ms / args.e2e_steps,
                   "copies": "rank gradients host->device, updated 16-bit parameters and the "
                             "result struct device->host, every step; the parameter copy of "
                             "step k runs on a second stream beside the gradient copy of step k+1"}
            del g_host, p_host
        else:
            e2e = {"value": None, "unit": UNIT,
                   "skipped": "host memory below 2.5x the gradient and parameter bytes of every rank "
                              "on the node"}

    peak, peak_kind = measured_hbm_peak()
    k_bytes = bench.owned * update_launch_bytes(k_nd, wl["mode"], n_dests)
    achieved = k_bytes / (k_ms_max / 1e3) / 1e9
    traffic, traffic_src = (profiled_traffic(wl["nd"], wl["mode"], bench.owned)
                            if not (n_dests or args.retain) else (None, None))
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": args.workload, "description": wl["desc"], "psi": bench.psi,
                   "nd": wl["nd"], "stage": wl["stage"], "storage": args.storage,
                   "peer_tables": bool(n_dests), "param_dests": n_dests,
                   "retention": bool(args.retain), "dynamic_loss_scale": bool(args.dynamic_scale),
                   "owned_params_per_gpu": bench.owned,
                   "mode": {0: "speculative", 1: "two_pass", 2: "stash"}[wl["mode"]],
                   "bytes_per_param_alg": alg, "bytes_per_param_moved": moved,
                   "assembled_params": bench.assembled,
                   "step_gbs_alg": (bench.owned * (alg + 2 * n_dests) + 4 * bench.assembled)
                                   / (ms_max / args.steps / 1e3) / 1e9,
                   "l2": "inputs larger than L2 (no flush): "
                         f"{bench.owned * moved / 1e9:.1f} GB moved per step",
                   "parallelism": f"{world} independent replica(s), Nd={wl['nd']} ranks simulated per GPU"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic, "traffic_source": traffic_src,
                     "kernel": k_name, "kernel_symbol": k_sym, "kernel_source": k_src,
                     "peak_source": f"{peak_kind} hbm_gbs (copy)",
                     "kernel_ms": k_ms_max,
                     "kernel_ms_median": k_ms_median,
                     "alg_bytes_per_launch": k_bytes},
        "e2e": e2e,
        "sustained": sustained,
        "gpu_launches": launches,
        "clocks": clk,
        "last_step": {"overflow": res.overflow, "t": res.t},
    }
    if args.retain:
        r_ms_max = max_over_ranks(r_ms, world)
        line["retention"] = {"reduce_kernel_ms": r_ms_max, "reduce_bytes_per_param": 2 * wl["nd"] + 2,
                             "reduce_gbs": bench.owned * (2 * wl["nd"] + 2) / (r_ms_max / 1e3) / 1e9}
        line["retention"]["reduce_frac"] = line["retention"]["reduce_gbs"] / peak
        line["config"]["step_gbs_alg"] = (bench.owned * (2 * wl["nd"] + 2 + update_launch_bytes(1, wl["mode"]))
                                          / (ms_max / args.steps / 1e3) / 1e9)
    bench.close()
    del bench
    torch.cuda.empty_cache()
    if not (args.no_configs or args.psi or args.peer or args.retain or args.dynamic_scale
            or args.storage != "fp16"):
        line["configs"] = run_configs(args, world, local, peak)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        line["cpu_baseline"] = cpu_baseline(wl, args.cpu_seconds, args.cpu_sample,
                                            oracle.host_threads(), STORAGES[args.storage])
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
