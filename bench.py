"""Benchmark: frames/s of the 24-block per-frame paged-KV prefill step on a
224x224, 320-frame stream (H=16, D=64, 256 patch + 6 special tokens, page 256,
8 scale frames, window 64), plus attention TFLOP/s and its roofline fraction.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 1]
    python bench.py --impl reference ...   # the CPU oracle, timed on host cores

One step = the whole stream: reset, then for each of the 320 frames
kv_begin_frame, kv_evict_frames, one kv_plan and 24 x kv_run_append through
the C-ABI (each one launch that appends the block's K/V and computes its
attention). Inputs come from a ring of 16 seeded frame sets already in HBM;
the 24 block pools (1.9 GB) exceed L2, so every call reads its K/V from HBM.
With --gpus N (torchrun) each rank runs an independent replica stream (the
path does not shard); value = frames of all ranks / max-over-ranks time.
"""
from __future__ import annotations

import argparse
import ctypes
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

import workload  # noqa: E402

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


TRAFFIC_PROFILE = os.path.join(ROOT, "profiles", "paged_prefill_attn_224x224_dram.txt")
KERNEL_SOURCES = ("paged_attn.cu", "sm100.cuh", "tmem_access.cuh", "kernels.h", "kv_layout.h", "merge.cuh",
                  "launch.cuh", "per_device.h")


def kernel_source_hash():
    import hashlib
    h = hashlib.sha256()
    for name in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "paged_kv_cache_frame_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def measured_traffic():
    """DRAM bytes per attention launch from the committed ncu summary, or None
    when that summary was taken on other kernel sources than the ones built."""
    if not os.path.exists(TRAFFIC_PROFILE):
        return None
    fields = {}
    for line in open(TRAFFIC_PROFILE):
        if ":" in line and not line.startswith("#"):
            k, v = line.split(":", 1)
            fields[k.strip()] = v.strip()
    if fields.get("kernel_sources_sha256_16") != kernel_source_hash():
        return None
    try:
        return float(fields["dram_bytes_per_launch_mean"])
    except (KeyError, ValueError):
        return None


def call_flops(T, lkv, H, D):
    """Tensor FLOPs of one attention call: Q K^T and P V, 2 per MAC."""
    return 4.0 * T * lkv * H * D


def call_kv_bytes(lkv, H, D, elt=2):
    """Algorithmic HBM bytes of one call: the visible K and V rows, read once."""
    return 2.0 * lkv * H * D * elt


# ------------------------------------------------------------------ ranks
def replica_seed(seed, rank):
    """Each rank runs an independent replica stream with its own inputs."""
    return seed + 1000 * rank


def max_over_ranks(x, world, device="cpu"):
    """The max of a per-rank number over all ranks (every rank gets it)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], device=device, dtype=torch.float64)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank, world, ms_max):
    """Units processed by all ranks per second of the slowest rank."""
    return units_per_rank * world / (ms_max / 1e3)


# ------------------------------------------------------------------ clocks
class ClockSampler:
    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}",
                 "--query-gpu=clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                 "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                 "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.15)
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

    def summary(self):
        if not self.path or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 8:
                continue
            try:
                sm.append(float(f[0]))
                smax.append(float(f[1]))
            except ValueError:
                continue
            for n, v in zip(names, f[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "samples": len(sm),
                "reasons": sorted(reasons)}


# ------------------------------------------------------------------ GPU arm
class HostIO:
    """End-to-end inputs and outputs: every frame step's Q/K/V (all blocks)
    go from pinned host memory to one of two device staging buffers on a copy
    stream, and its outputs from one of two device output buffers back to
    pinned host memory on another stream. Events order each buffer's reuse,
    so the copies of frame f+1 and f-1 run while frame f computes."""

    def __init__(self, runner):
        torch = runner.torch
        self.torch = torch
        self.hring = runner.ring.cpu().pin_memory()                 # [R, B, 3, rows, H, D]
        self.hout = torch.empty((runner.ring_n,) + tuple(runner.out.shape), dtype=runner.out.dtype).pin_memory()
        self.stage = [torch.empty_like(runner.ring[0]) for _ in range(2)]
        self.outb = [torch.empty_like(runner.out) for _ in range(2)]
        self.ptr = [[[st[b, i].data_ptr() for i in range(3)] for b in range(st.shape[0])] for st in self.stage]
        self.optr = [[o[b].data_ptr() for b in range(o.shape[0])] for o in self.outb]
        self.h2d = torch.cuda.Stream()
        self.d2h = torch.cuda.Stream()
        ev = lambda: [torch.cuda.Event() for _ in range(2)]
        self.copied, self.computed, self.drained = ev(), ev(), ev()
        self.used = [False, False]
        self.h2d_bytes = self.stage[0].numel() * self.stage[0].element_size()   # per frame step
        self.d2h_bytes = self.outb[0].numel() * self.outb[0].element_size()

    def begin_pass(self, compute):
        start = self.torch.cuda.Event()
        start.record(compute)
        self.h2d.wait_event(start)
        self.d2h.wait_event(start)
        self.used = [False, False]

    def inputs(self, f, r, compute):
        i = f % 2
        if self.used[i]:
            self.h2d.wait_event(self.computed[i])    # frame f-2 has read stage i
        with self.torch.cuda.stream(self.h2d):
            self.stage[i].copy_(self.hring[r], non_blocking=True)
            self.copied[i].record(self.h2d)
        compute.wait_event(self.copied[i])
        if self.used[i]:
            compute.wait_event(self.drained[i])      # frame f-2's outputs are back on the host
        return self.ptr[i], self.optr[i]

    def outputs(self, f, r, compute):
        i = f % 2
        self.computed[i].record(compute)
        self.d2h.wait_event(self.computed[i])
        with self.torch.cuda.stream(self.d2h):
            self.hout[r].copy_(self.outb[i], non_blocking=True)
            self.drained[i].record(self.d2h)
        self.used[i] = True

    def end_pass(self, compute):
        compute.wait_stream(self.h2d)
        compute.wait_stream(self.d2h)


class StreamRunner:
    """One replica of the workload's stream on the current GPU. A frame step
    is kv_begin_frame, kv_evict_frames, kv_plan, then kv_run_append for every
    block (one launch that appends the block's K/V and computes its
    attention), and the keyframe decision when frames are deferred."""

    def __init__(self, wl, seed, ring=16):
        import torch
        import paged_kv_cache_frame_b200 as pkv
        from paged_kv_cache_frame_b200 import capi
        self.torch, self.pkv, self.capi = torch, pkv, capi
        self.L = capi.lib()
        self.wl, self.ring_n = wl, ring
        self.stream = torch.cuda.current_stream()
        self.sp = self.stream.cuda_stream
        self.cache = pkv.PagedKVCache(wl.max_pages, wl.page_size, wl.H, wl.D, wl.S, wl.W,
                                      num_blocks=wl.blocks, num_special=wl.NS, dtype=wl.dtype,
                                      cross_frame_special=wl.cross_special)
        self.cache.allocate_pools("cuda")
        self.h = self.cache.handle
        self.cache_arr = (ctypes.c_void_p * 1)(self.h)
        self.ws = torch.empty(pkv.workspace_bytes([self.cache]), dtype=torch.uint8, device="cuda")
        self.ring = workload.qkv_ring_cuda(wl, seed, ring)            # [R, B, 3, T, H, D]
        self.out = torch.empty((wl.blocks, wl.T, wl.H, wl.D), dtype=wl.torch_dtype(), device="cuda")
        self.keep = workload.keyframe_mask(wl, seed)
        self.defer = wl.keyframes != "all"
        self.ptr = [[[self.ring[r, b, i].data_ptr() for i in range(3)] for b in range(wl.blocks)]
                    for r in range(ring)]
        self.optr = [self.out[b].data_ptr() for b in range(wl.blocks)]
        self.ws_ptr, self.ws_bytes = self.ws.data_ptr(), self.ws.numel()
        self.lkv = []            # per frame step of the last pass: visible tokens
        self.fused = []          # per frame step: the plan merged its splits in-kernel

    frames_per_pass = property(lambda self: self.wl.frames)
    steps_per_pass = property(lambda self: self.wl.frames)

    def _chk(self, rc, what):
        if rc != 0:
            raise self.capi.KVError(rc, what, self.L.kv_last_error().decode())

    def one_pass(self, io=None):
        """One pass over the stream; returns the library's kernel launches.
        io: a HostIO for the end-to-end variant. With self.pages_calls each
        block runs the pages' two calls, kv_append_frame then kv_run (a
        scatter launch and an attention launch), instead of kv_run_append."""
        if getattr(self, "pages_calls", False):
            return self.one_pass_pages(io)
        L, wl, h, sp = self.L, self.wl, self.h, self.sp
        self._chk(L.kv_reset(h), "kv_reset")
        plan = ctypes.c_void_p()
        st = self.capi.kv_plan_stats()
        self.lkv, self.fused = [], []
        launches = 0
        if io is not None:
            io.begin_pass(self.stream)
        for f in range(wl.frames):
            r = f % self.ring_n
            ptr, optr = io.inputs(f, r, self.stream) if io is not None else (self.ptr[r], self.optr)
            if self.defer:
                self._chk(L.kv_defer_eviction(h, 1), "defer")
            self._chk(L.kv_begin_frame(h), "begin_frame")
            self._chk(L.kv_evict_frames(h), "evict")
            if plan.value:
                L.kv_plan_free(plan)
            self._chk(L.kv_plan(ctypes.byref(plan), self.cache_arr, 1, 0, self.ws_ptr, self.ws_bytes, sp), "plan")
            L.kv_plan_get_stats(plan, ctypes.byref(st))
            launches += st.upload_launches + wl.blocks * st.run_launches
            self.lkv.append(st.visible_tokens)
            self.fused.append(st.fused_merge)
            for b in range(wl.blocks):
                q, k, v = ptr[b]
                self._chk(L.kv_run_append(plan, b, k, v, q, optr[b], sp), "run_append")
            if self.defer:
                if self.keep[f]:
                    self._chk(L.kv_commit_frame(h), "commit")
                else:
                    self._chk(L.kv_rollback_last_frame(h), "rollback")
            if io is not None:
                io.outputs(f, r, self.stream)
        if plan.value:
            L.kv_plan_free(plan)
        if io is not None:
            io.end_pass(self.stream)
        return launches


    def one_pass_pages(self, io=None):
        L, wl, h, sp = self.L, self.wl, self.h, self.sp
        self._chk(L.kv_reset(h), "kv_reset")
        plan = ctypes.c_void_p()
        st = self.capi.kv_plan_stats()
        self.lkv, self.fused = [], []
        launches = 0
        if io is not None:
            io.begin_pass(self.stream)
        for f in range(wl.frames):
            r = f % self.ring_n
            ptr, optr = io.inputs(f, r, self.stream) if io is not None else (self.ptr[r], self.optr)
            if self.defer:
                self._chk(L.kv_defer_eviction(h, 1), "defer")
            for b in range(wl.blocks):
                q, k, v = ptr[b]
                self._chk(L.kv_append_frame(h, b, k, v, sp), "append")
                if b == 0:
                    self._chk(L.kv_evict_frames(h), "evict")
                    if plan.value:
                        L.kv_plan_free(plan)
                    self._chk(L.kv_plan(ctypes.byref(plan), self.cache_arr, 1, 0, self.ws_ptr, self.ws_bytes, sp),
                              "plan")
                    L.kv_plan_get_stats(plan, ctypes.byref(st))
                    launches += st.upload_launches + wl.blocks * (1 + st.run_launches)
                    self.lkv.append(st.visible_tokens)
                    self.fused.append(st.fused_merge)
                self._chk(L.kv_run(plan, b, q, optr[b], sp), "run")
            if self.defer:
                if self.keep[f]:
                    self._chk(L.kv_commit_frame(h), "commit")
                else:
                    self._chk(L.kv_rollback_last_frame(h), "rollback")
            if io is not None:
                io.outputs(f, r, self.stream)
        if plan.value:
            L.kv_plan_free(plan)
        if io is not None:
            io.end_pass(self.stream)
        return launches


class BatchRunner:
    """Several streams of different ages planned together (one kv_plan over
    all caches per frame step, their query rows concatenated), as in the
    batched workload, sharing one pool per block. A pass is `steps` frame
    steps of every stream; the streams keep growing from pass to pass."""

    def __init__(self, wl, seed, steps, passes, ring=4):
        import torch
        import paged_kv_cache_frame_b200 as pkv
        from paged_kv_cache_frame_b200 import capi
        self.torch, self.pkv, self.capi = torch, pkv, capi
        self.L = capi.lib()
        self.wl, self.ring_n, self.steps = wl, ring, steps
        self.stream = torch.cuda.current_stream()
        self.sp = self.stream.cuda_stream
        self.ages = workload.stream_ages(wl, seed)
        span = int(self.ages.max()) + steps * passes
        sp_pages = max(1, math.ceil(wl.NS * span / wl.page_size))
        # one pool per block for all the streams (kv_init_group): common patch
        # pages, a special-page range per stream
        patch = wl.streams * wl.patch_pages
        self.caches = pkv.PagedKVCache.group(wl.streams, patch + wl.streams * sp_pages, wl.page_size, wl.H, wl.D,
                                             wl.S, wl.W, num_blocks=wl.blocks, num_special=wl.NS, dtype=wl.dtype,
                                             patch_pages=patch, special_pages=sp_pages)
        self.caches[0].allocate_pools("cuda")
        self.h = [c.handle for c in self.caches]
        self.cache_arr = (ctypes.c_void_p * wl.streams)(*self.h)
        self.ws = torch.empty(pkv.workspace_bytes(self.caches), dtype=torch.uint8, device="cuda")
        self.ring = workload.qkv_ring_cuda(wl, seed, ring)            # [R, B, 3, streams*T, H, D]
        self.out = torch.empty((wl.blocks, wl.streams * wl.T, wl.H, wl.D), dtype=wl.torch_dtype(), device="cuda")
        self.ptr = [[[self.ring[r, b, i].data_ptr() for i in range(3)] for b in range(wl.blocks)]
                    for r in range(ring)]
        self.optr = [self.out[b].data_ptr() for b in range(wl.blocks)]
        self.ws_ptr, self.ws_bytes = self.ws.data_ptr(), self.ws.numel()
        self.lkv, self.fused = [], []
        # warm every stream to its age: page state only (metadata appends)
        # (a frame step closes once every block has been appended)
        for h, age in zip(self.h, self.ages):
            for _ in range(int(age)):
                for b in range(wl.blocks):
                    self._chk(self.L.kv_append_frame(h, b, None, None, None), "warm append")
                self._chk(self.L.kv_evict_frames(h), "warm evict")

    frames_per_pass = property(lambda self: self.steps * self.wl.streams)
    steps_per_pass = property(lambda self: self.steps)

    def _chk(self, rc, what):
        if rc != 0:
            raise self.capi.KVError(rc, what, self.L.kv_last_error().decode())

    def one_pass(self, io=None):
        L, wl, sp = self.L, self.wl, self.sp
        plan = ctypes.c_void_p()
        st = self.capi.kv_plan_stats()
        self.lkv, self.fused = [], []
        launches = 0
        if io is not None:
            io.begin_pass(self.stream)
        for f in range(self.steps):
            r = f % self.ring_n
            ptr, optr = io.inputs(f, r, self.stream) if io is not None else (self.ptr[r], self.optr)
            for h in self.h:
                self._chk(L.kv_begin_frame(h), "begin_frame")
                self._chk(L.kv_evict_frames(h), "evict")
            if plan.value:
                L.kv_plan_free(plan)
            self._chk(L.kv_plan(ctypes.byref(plan), self.cache_arr, wl.streams, 0, self.ws_ptr,
                                self.ws_bytes, sp), "plan")
            L.kv_plan_get_stats(plan, ctypes.byref(st))
            launches += st.upload_launches + wl.blocks * st.run_launches
            self.lkv.append(st.visible_tokens)
            self.fused.append(st.fused_merge)
            for b in range(wl.blocks):
                q, k, v = ptr[b]
                self._chk(L.kv_run_append(plan, b, k, v, q, optr[b], sp), "run_append")
            if io is not None:
                io.outputs(f, r, self.stream)
        if plan.value:
            L.kv_plan_free(plan)
        if io is not None:
            io.end_pass(self.stream)
        return launches


def roofline_ms(wl, lkvs, peak_tf, hbm_gbs):
    """Sum over one pass of each attention call's roofline time
    max(FLOPs / tensor peak, K/V bytes / HBM bandwidth), in ms."""
    return sum(max(call_flops(wl.T, l, wl.H, wl.D) / (peak_tf * 1e12),
                   call_kv_bytes(l, wl.H, wl.D) / (hbm_gbs * 1e9)) for l in lkvs) * wl.blocks * 1e3


def run_gpu(args):
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)   # before the process group, so NCCL binds this GPU
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    from paged_kv_cache_frame_b200 import build
    build.build()
    wl = workload.WORKLOADS[args.workload]
    profiling_case = bool(args.frames or args.blocks)
    if profiling_case:
        import dataclasses
        wl = dataclasses.replace(wl, name=wl.name + "-profiling-case", frames=args.frames or wl.frames,
                                 blocks=args.blocks or wl.blocks)
    if wl.streams > 1:
        runner = BatchRunner(wl, seed=replica_seed(args.seed, rank), steps=wl.steps,
                             passes=args.warmup + 2 * args.steps + 3)
    else:
        runner = StreamRunner(wl, seed=replica_seed(args.seed, rank))
        runner.pages_calls = args.calls == "pages"
    torch.cuda.synchronize()

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local])

    for _ in range(args.warmup):
        runner.one_pass()
    torch.cuda.synchronize()

    # ---- timed region: K passes over the stream, inputs resident in HBM.
    # Nothing but the library's kernels runs on the stream inside it (one plan
    # upload per frame step, one kernel per block), so the region's time is
    # also the attention kernels' time, launch gaps included.
    barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    with clocks:
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record()
        launches = 0
        for _ in range(args.steps):
            launches += runner.one_pass()
        t1.record()
        torch.cuda.synchronize()
    barrier()
    ms_max = max_over_ranks(t0.elapsed_time(t1), world, "cuda")
    value = whole_job_rate(args.steps * runner.frames_per_pass, world, ms_max)
    ms_pass = ms_max / args.steps

    lkvs = list(runner.lkv)                            # per frame step of the last pass
    flops = sum(call_flops(wl.T, l, wl.H, wl.D) for l in lkvs) * wl.blocks
    kvbytes = sum(call_kv_bytes(l, wl.H, wl.D) for l in lkvs) * wl.blocks
    pk, pk_kind = peaks()
    burst_tf = pk["bf16_tflops"]
    sust_tf = pk.get("bf16_tflops_sustained", burst_tf)
    tflops = flops / (ms_pass / 1e3) / 1e12
    roof_sust = roofline_ms(wl, lkvs, sust_tf, pk["hbm_gbs"])
    roof_burst = roofline_ms(wl, lkvs, burst_tf, pk["hbm_gbs"])

    # ---- end to end: host (pinned) inputs copied in, outputs copied out, every frame step
    e2e = None
    if not args.no_e2e:
        io = HostIO(runner)
        runner.one_pass(io=io)
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(args.steps):
            runner.one_pass(io=io)
        b.record()
        torch.cuda.synchronize()
        barrier()
        ems = max_over_ranks(a.elapsed_time(b), world, "cuda")
        e2e = {"value": whole_job_rate(args.steps * runner.frames_per_pass, world, ems), "unit": "frames/s",
               "h2d_bytes_per_step": int(io.h2d_bytes * runner.steps_per_pass),
               "d2h_bytes_per_step": int(io.d2h_bytes * runner.steps_per_pass),
               "copies": "per frame step: H2D on a copy stream, D2H on another, double-buffered"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and wl.streams == 1:
        cpu = cpu_baseline(wl, args.seed, budget_s=args.cpu_budget, frames_sample=oracle_sample_frames(wl))

    if rank == 0:
        metric = metric_name(args.workload, wl)
        config = arm_config(wl, world, args.seed)
        if args.calls != "fused":
            config["calls"] = "kv_append_frame + kv_run"
        if wl.streams > 1:
            assert config["stream_ages"] == [int(x) for x in runner.ages]
        kernel_ms = ms_pass   # per pass: all library kernels of the timed region
        line = {
            "metric": metric,
            "profiling_case_not_a_bench_value": profiling_case or None,
            "value": round(value, 2), "unit": "frames/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_pass, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": wl.dtype,
            "data": f"synthetic (seeded N(0,1) Q/K/V, ring of {runner.ring_n} frame sets in HBM)",
            "config": config,
            "attention": {"tflops": round(tflops, 2), "kv_gbs": round(kvbytes / (kernel_ms / 1e3) / 1e9, 1),
                          "frac_of_sustained_roofline": round(roof_sust / kernel_ms, 4),
                          "frac_of_burst_roofline": round(roof_burst / kernel_ms, 4),
                          "roofline_ms_per_pass_sustained": round(roof_sust, 3),
                          "roofline_ms_per_pass_burst": round(roof_burst, 3),
                          "kernel_ms_per_pass": round(kernel_ms, 3),
                          "fused_merge_steps": int(sum(runner.fused)),
                          "steps_per_pass": len(lkvs)},
            "roofline": {"bound": "tensor", "achieved": round(tflops, 2),
                         "peak": sust_tf, "unit": "TFLOP/s",
                         "frac": round(roof_sust / kernel_ms, 4),
                         "frac_of_burst": round(roof_burst / kernel_ms, 4),
                         "traffic": measured_traffic() if args.workload == 1 else None,
                         "peak_kind": f"{pk_kind} bf16 dense sustained (kernel timed inside a long step); "
                                      f"burst {burst_tf} in frac_of_burst",
                         "kernel": "paged_prefill_attn (append + attention + split merge in one launch "
                                   "per block) and the per-frame plan upload: the whole timed region"},
            "gpu_launches": launches,
            "clocks": clocks.summary(),
            "e2e": e2e,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line))
    if world > 1:
        dist.destroy_process_group()


# ------------------------------------------------------------------ oracle arm
def oracle_threads():
    """Threads the oracle's numpy arithmetic can use (its einsum contractions
    run in the BLAS thread pool)."""
    try:
        import threadpoolctl
        n = [d["num_threads"] for d in threadpoolctl.threadpool_info() if d.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def metric_name(workload_id, wl):
    if workload_id == 1:
        return "frames/s (24-block stack) at 224x224, 320 frames"
    if wl.streams > 1:
        return f"frames/s ({wl.streams} streams x {wl.blocks}-block stack), {wl.name}"
    return f"frames/s ({wl.blocks}-block stack), {wl.name}"


def arm_config(wl, world, seed):
    """The config object of a bench line, identical in both arms: a batched
    workload adds rank 0's seeded stream ages (the ones BatchRunner draws)."""
    config = workload_config(wl, world)
    if wl.streams > 1:
        ages = workload.stream_ages(wl, replica_seed(seed, 0))
        config.update({"streams": wl.streams, "stream_ages": [int(x) for x in ages],
                       "frame_steps_per_pass": wl.steps, "frames": None})
    return config


def workload_config(wl, world):
    """The config object of a bench line (the same for both arms)."""
    return {"workload": wl.name, "frames": wl.frames, "blocks": wl.blocks, "H": wl.H,
            "D": wl.D, "tokens_per_frame": wl.T, "page_size": wl.page_size,
            "scale_frames": wl.S, "window": wl.W, "keyframes": wl.keyframes,
            "cross_frame_special": wl.cross_special,
            "parallelism": f"replicas x{world}",
            "l2": "inputs larger than L2 (one pool per block, all read every frame step)"}


def oracle_sample_frames(wl):
    """The frames both arms time the oracle on: the last frame of the
    window's ramp and the stream's last frame (0-based), all query rows of
    block 0."""
    n = max(1, wl.frames)
    return tuple(sorted({min(wl.S + wl.W, n) - 1, n - 1}))


def cpu_baseline(wl, seed, budget_s=20.0, frames_sample=(71, 319), rows=None):
    """Times the CPU oracle (float64 dense attention) on a bounded sample of
    the workload and extrapolates frames/s by FLOPs."""
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from oracle.stream import StreamOracle, bits16
    fr_cache = {}

    def fetch(f):
        if f not in fr_cache:
            fr_cache.clear()
            fr_cache[f] = tuple(bits16(x) for x in workload.frame_qkv(wl, seed, f, 0))
        return fr_cache[f]

    so = StreamOracle(wl.S, wl.W, wl.NS, wl.P, wl.dtype, fetch, cross_frame_special=wl.cross_special)
    rng = np.random.default_rng(seed)
    rows = wl.T if rows is None else rows   # all query rows by default (about 10-15 s on one core)
    sel = sorted(rng.choice(wl.T, size=min(rows, wl.T), replace=False).tolist())
    t_att, fl = 0.0, 0.0
    done = []
    for f in range(max(frames_sample) + 1):
        so.begin_frame(f)
        if f in frames_sample:
            t = time.perf_counter()
            so.expected(sel)
            dt = time.perf_counter() - t
            lkv = len(so.sim.attended_patch_frames()) * wl.P + len(so.sim.visible_specials())
            t_att += dt
            fl += call_flops(len(sel), lkv, wl.H, wl.D)
            done.append(f)
            if t_att > budget_s:
                break
    gflops = fl / t_att / 1e9
    # whole-workload FLOPs: every frame, every block
    sim_l = [min(n, wl.S + wl.W) * wl.P + wl.NS * (n if wl.cross_special else min(n, wl.S + wl.W))
             for n in range(1, wl.frames + 1)]
    total = sum(call_flops(wl.T, l, wl.H, wl.D) for l in sim_l) * wl.blocks
    fps = wl.frames / (total / (gflops * 1e9))
    return {"value": fps, "unit": "frames/s", "cores": oracle_threads(), "kind": "oracle",
            "gflops": round(gflops, 3),
            "sample": f"float64 oracle attention of block 0 at frames {[d + 1 for d in done]} for "
                      f"{len(sel)} of {wl.T} query rows ({t_att:.1f} s); frames/s extrapolated by "
                      f"the workload's {total / 1e12:.1f} TFLOP"}


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    arm = workload.WORKLOADS[args.workload]   # metric and config: the same as the GPU arm's
    wl = arm
    if wl.streams > 1:
        # the oracle runs one stream; a stream as old as the oldest in the batch
        import dataclasses
        wl = dataclasses.replace(wl, streams=1, frames=wl.age_hi)
    for _ in range(args.warmup):   # untimed: a small call to load and warm the oracle's code
        cpu_baseline(wl, args.seed, budget_s=1.0, frames_sample=(0,), rows=8)
    t = time.perf_counter()
    vals = []
    sample = oracle_sample_frames(wl)   # the GPU arm's cpu_baseline sample
    for _ in range(args.steps):
        vals.append(cpu_baseline(wl, args.seed, budget_s=args.cpu_budget, frames_sample=sample))
    el = time.perf_counter() - t
    v = statistics.median(x["value"] for x in vals)
    line = {
        "impl": "reference", "metric": metric_name(args.workload, arm),
        "value": v, "unit": "frames/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(el * 1e3 / max(1, args.steps), 1), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": arm_config(arm, world, args.seed),
        "cpu_baseline": {"value": v, "unit": "frames/s", "cores": oracle_threads(), "kind": "oracle",
                         "sample": vals[-1]["sample"]},
        "e2e": {"value": v, "unit": "frames/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", type=int, default=1, choices=[1, 2, 3, 4, 5])
    ap.add_argument("--seed", type=int, default=1)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--calls", default="fused", choices=["fused", "pages"],
                    help="per block: kv_run_append (fused) or the pages' kv_append_frame + kv_run")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=20.0)
    ap.add_argument("--frames", type=int, default=0,
                    help="profiling case: override the stream length (not a bench value)")
    ap.add_argument("--blocks", type=int, default=0,
                    help="profiling case: override the block count (not a bench value)")
    args = ap.parse_args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
