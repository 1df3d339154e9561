"""Benchmark: block top-k sparse decode over a paged KV cache on B200 (req-heads/s).

One step = one decode layer of the Qwen3-0.6B-like workload (B=32, Hq=16, Hkv=8, D=128,
page 16, contexts U[4096, 16384], 40,000-page shuffled pool, top-30 + 1 + 1 pages):
  vt_build_centroids  on the pages that fill at this step (requests whose length is a
                      multiple of 16),
  vt_sparse_decode_fused  group mean -> centroid scores -> exact top-k + reserved pages ->
                      attention over the selected pages, one launch of persistent CTAs
                      that schedule themselves (``--plan`` adds vt_plan_requests, the
                      longest-first order the cluster kernels take; the persistent kernel
                      does not need it).
Inputs are resident in HBM; steps rotate over ``--replicas`` copies of the inputs (pools,
centroids, q, page tables) whose combined footprint is far above the 126 MB L2, so no step
finds its data in L2.  Rank 0 prints one JSON line.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

``--impl reference`` times the fp64 CPU oracle on this host's cores on the same workload
(each step a bounded sample of requests) -- the only other place this script runs it is the
``cpu_baseline`` leg of the default arm.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import math
import os
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from paged_block_sparse_vt_b200.workloads import PAGE_SIZE, config, make_workload  # noqa: E402

CFG = 2
METRIC = "sparse-decode req-heads/s"
UNIT = "req-heads/s"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "fused_kernel_traffic.json")
FALLBACK_HBM_GBS = 6650.0


def log(*a):
    print(*a, file=sys.stderr, flush=True)


# ------------------------------------------------------------------------------------------
# algorithmic bytes (what the method must move; not the dense KV it avoids)
# ------------------------------------------------------------------------------------------
def algorithmic_bytes(c, seq_lens: torch.Tensor) -> dict:
    """Per step, from the generated lengths:
    fused   = sum_b [2 Hq D (q) + 2 Hq Dv (out) + 4 Hq (lse) + 4 n_b (page-table row)]
            + sum_{b,h} [4 D |C_b| (candidate centroids, sparse requests only)
                         + 2 (D + Dv) * tokens of the selected pages]
    build   = per filled page: 16 Hkv D * 2 (K read) + Hkv D * 4 (centroid write) + 4 (id)
    With eos >= 1 the (possibly partial) last page is always selected, so the selected tokens
    of a unit are 16 (min(n, kmax) - 1) + valid tokens of the last page.
    """
    assert c.eos >= 1
    L = seq_lens.long()
    n = (L + PAGE_SIZE - 1) // PAGE_SIZE
    last_valid = L - PAGE_SIZE * (n - 1)
    sparse = n > c.kmax
    cand = torch.where(sparse, n - c.bos - c.eos, torch.zeros_like(n))
    sel_pages = torch.minimum(n, torch.full_like(n, c.kmax))
    tokens = PAGE_SIZE * (sel_pages - 1) + last_valid
    per_req = 2 * c.Hq * c.D + 2 * c.Hq * c.Dv + 4 * c.Hq + 4 * n
    dv = 0 if c.mla else c.Dv  # MLA: V is the first Dv dims of the K row, read once
    per_unit = 4 * c.D * cand + 2 * (c.D + dv) * tokens
    fused = int(per_req.sum()) + c.Hkv * int(per_unit.sum())
    n_fill = int((L % PAGE_SIZE == 0).sum())
    build = n_fill * (PAGE_SIZE * c.Hkv * c.D * 2 + c.Hkv * c.D * 4 + 4)
    return dict(fused=fused, build=build, total=fused + build,
                centroid_bytes=c.Hkv * int((4 * c.D * cand).sum()),
                kv_bytes=c.Hkv * int((2 * (c.D + dv) * tokens).sum()))


def variant_bytes(c, seq_lens: torch.Tensor) -> dict:
    """Algorithmic bytes of the split calls, from the same lengths:
    select  = q + page-table rows + candidate centroids + sel/n_sel written
    decode  = q + out + lse + sel/n_sel read + one page-table entry per selected page
              + the selected K/V rows
    """
    L = seq_lens.long()
    n = (L + PAGE_SIZE - 1) // PAGE_SIZE
    last_valid = L - PAGE_SIZE * (n - 1)
    sparse = n > c.kmax
    cand = torch.where(sparse, n - c.bos - c.eos, torch.zeros_like(n))
    sel_pages = torch.minimum(n, torch.full_like(n, c.kmax))
    tokens = PAGE_SIZE * (sel_pages - 1) + last_valid
    dv = 0 if c.mla else c.Dv
    q = 2 * c.B * c.Hq * c.D
    selw = 4 * c.B * c.Hkv * (c.kmax + 1)
    select = q + 4 * int(n.sum()) + c.Hkv * int((4 * c.D * cand).sum()) + selw
    decode = (q + 2 * c.B * c.Hq * c.Dv + 4 * c.B * c.Hq + selw
              + c.Hkv * int((4 * sel_pages + 2 * (c.D + dv) * tokens).sum()))
    return dict(select=select, decode=decode)


def build_bytes(c, pages: int) -> int:
    """vt_build_centroids over `pages` pages: K rows read, fp32 centroid rows written, ids."""
    return pages * (PAGE_SIZE * c.Hkv * c.D * 2 + c.Hkv * c.D * 4 + 4)


NOMINAL_HBM_GBS = 8000.0


def read_peak_hbm():
    try:
        with open(PEAKS_FILE) as f:
            pk = json.load(f)
        return float(pk["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# the files the timed fused kernel is compiled from
FUSED_KERNEL_SOURCES = ("fused_persistent.cu", "gqa_attend.cuh", "topk.cuh", "common.cuh",
                        "centroid_chunk.cuh",
                        "decode_params.cuh")


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for name in FUSED_KERNEL_SOURCES:
        with open(os.path.join(ROOT, "paged_block_sparse_vt_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(cfg: int):
    """DRAM bytes per launch of the fused kernel from an ncu capture, if it was taken on this
    source and this workload."""
    try:
        with open(TRAFFIC_FILE) as f:
            rec = json.load(f)
        if rec.get("source_hash") == kernel_source_hash() and rec.get("config", CFG) == cfg:
            return rec.get("bytes_per_launch")
    except Exception:
        pass
    return None


# ------------------------------------------------------------------------------------------
# clocks sampled during the timed region
# ------------------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.lines = []
        self.t = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.t.join(timeout=5)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return None
        sm.sort()
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


# ------------------------------------------------------------------------------------------
# distributed plumbing (one process per GPU; the data path has no collective)
# ------------------------------------------------------------------------------------------
def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    elif n_gpus > 1:
        raise SystemExit("--gpus N > 1 needs torchrun (one process per GPU)")
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def aggregate_value(world: int, units_per_rank: int, steps: int, elapsed_s: float) -> float:
    """Whole-job throughput: every rank processed its own batch of units each step (weak
    scaling); the time is the slowest rank's."""
    return world * units_per_rank * steps / elapsed_s


def max_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------------------------------
# the reference arm: the CPU oracle
# ------------------------------------------------------------------------------------------
def oracle_prepare(w):
    import oracle
    oracle.build()
    c = w["config"]
    cent = torch.full((w["P"], c.Hkv, c.D), float("nan"))
    oracle.build_centroids(w["k_pool"], w["prebuilt_pages"], cent)
    return cent


def oracle_step(w, cent, reqs, kind="f64"):
    """One oracle decode step over the requests in ``reqs``: build the centroids of the pages
    that fill at this step, then select + attend."""
    import oracle
    c = w["config"]
    idx = torch.tensor(reqs, dtype=torch.long)
    L = w["seq_lens"][idx]
    n = (L + PAGE_SIZE - 1) // PAGE_SIZE
    fill = [int(w["page_table"][b, int(n[i]) - 1]) for i, b in enumerate(reqs)
            if int(L[i]) % PAGE_SIZE == 0]
    if fill:
        oracle.build_centroids(w["k_pool"], torch.tensor(fill, dtype=torch.int32), cent,
                               kind=kind)
    oracle.decode_step(w["q"][idx].contiguous(), w["k_pool"], w["v_pool"],
                       w["page_table"][idx].contiguous(), L.contiguous(), cent, c.topk, c.bos,
                       c.eos, c.sm_scale, head_dim_v=c.Dv, kind=kind)


def oracle_sample_size(w, cent, target_s: float) -> list:
    """Requests per oracle step so that one step takes about target_s seconds (>= 1)."""
    c = w["config"]
    t0 = time.perf_counter()
    oracle_step(w, cent, [0])
    dt = max(1e-4, time.perf_counter() - t0)
    k = max(1, min(c.B, int(target_s / dt)))
    return list(range(k))


def run_reference(args, world, rank):
    if rank != 0:
        return  # rank 0 alone runs the CPU reference
    import oracle
    c = config(args.config)
    w = make_workload(c, seed=1000 + args.config)
    cent = oracle_prepare(w)
    cores = oracle.get_threads()
    reqs = oracle_sample_size(w, cent, target_s=max(0.5, 60.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_step(w, cent, reqs)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(w, cent, reqs)
    dt = (time.perf_counter() - t0) / args.steps
    value = len(reqs) * c.Hq / dt
    sample = (f"{len(reqs)} of {c.B} requests ({len(reqs) * c.Hq} req-heads) per step, fp64 C "
              f"oracle, OpenMP over (request, KV head)")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(c, w, args),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def lengths_text(c) -> str:
    if c.lengths == "fixed":
        return f"{c.len_lo}"
    if c.lengths == "uniform":
        return f"U[{c.len_lo},{c.len_hi}]"
    return f"logU[{c.len_lo},{c.len_hi}]"


STEP_INPUTS = ("q", "page_table", "seq_lens", "fill_pages")  # what changes every step


def packed(tensors, device, pin: bool = False):
    """One byte buffer holding copies of the tensors, each at a 256-byte aligned offset, and
    views of it with the tensors' dtypes and shapes."""
    offs, total = [], 0
    for t in tensors:
        offs.append(total)
        total += (t.numel() * t.element_size() + 255) // 256 * 256
    buf = torch.empty(total, dtype=torch.uint8, device=device, pin_memory=pin)
    views = []
    for t, off in zip(tensors, offs):
        v = buf[off:off + t.numel() * t.element_size()].view(t.dtype).view(t.shape)
        v.copy_(t)
        views.append(v)
    return buf, views


def workload_config(c, w, args) -> dict:
    return {
        "workload": f"{c.name} sparse decode layer (B={c.B}, Hq={c.Hq}, Hkv={c.Hkv}, "
                    f"D={c.D}/{c.Dv}, page 16, context {lengths_text(c)}, "
                    f"top-{c.topk}+{c.bos}+{c.eos})",
        "B": c.B, "Hq": c.Hq, "Hkv": c.Hkv, "head_dim": c.D, "page_size": PAGE_SIZE,
        "topk": c.topk, "bos": c.bos, "eos": c.eos, "pool_pages": w["P"],
        "mean_pages_per_request": float(((w["seq_lens"].double() + 15) // 16).mean()),
        "parallelism": f"dp{args.gpus} (independent batches per GPU)",
        "l2": f"inputs rotate over {args.replicas} resident copies (>126 MB L2 between reuses)",
    }


# ------------------------------------------------------------------------------------------
# our arm
# ------------------------------------------------------------------------------------------
def run_ours(args, world, rank, local):
    import paged_block_sparse_vt_b200 as vt
    vt.load_library()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    c = config(args.config)
    w = make_workload(c, seed=1000 + args.config + 7919 * rank)
    nbytes = algorithmic_bytes(c, w["seq_lens"])
    stream = torch.cuda.current_stream(dev)

    # resident replicas of every per-step input; centroids of the full pages prebuilt
    reps = []
    for r in range(args.replicas):
        d = {k: w[k].to(dev) for k in ("k_pool", "prebuilt_pages")}
        # the per-step inputs as views of one device buffer, filled by one copy per step
        d["in_buf"], views = packed([w[k] for k in STEP_INPUTS], dev)
        d.update(zip(STEP_INPUTS, views))
        # MLA: V is a view of the K rows (one pool)
        d["v_pool"] = d["k_pool"] if w["v_pool"] is w["k_pool"] else w["v_pool"].to(dev)
        d["cent"] = torch.zeros((w["P"], c.Hkv, c.D), dtype=torch.float32, device=dev)
        vt.vt_build_centroids(d["k_pool"], d["prebuilt_pages"], d["cent"])
        # out and lse as views of one device buffer, read back by one copy per step
        d["out_buf"], (d["out"], d["lse"]) = packed(
            [torch.zeros((c.B, c.Hq, c.Dv), dtype=torch.bfloat16),
             torch.zeros((c.B, c.Hq), dtype=torch.float32)], dev)
        d["order"] = torch.empty((c.B,), dtype=torch.int32, device=dev)
        d["status"] = torch.zeros((1,), dtype=torch.int32, device=dev)
        d["ws"] = vt.fused_workspace(d["q"], d["k_pool"], d["v_pool"], d["page_table"],
                                     d["seq_lens"], d["cent"], c.topk, c.bos, c.eos,
                                     head_dim_v=c.Dv)
        reps.append(d)
    torch.cuda.synchronize(dev)

    def fused(d):
        vt.vt_sparse_decode_fused(d["q"], d["k_pool"], d["v_pool"], d["page_table"],
                                  d["seq_lens"], d["cent"], c.topk, c.bos, c.eos, c.sm_scale,
                                  out=d["out"], lse=d["lse"],
                                  order=d["order"] if args.plan else None, status=d["status"],
                                  workspace=d["ws"], head_dim_v=c.Dv)

    def one_launch(d):  # the build of this step's filled pages and the fused call, one launch
        vt.vt_sparse_decode_step(d["q"], d["k_pool"], d["v_pool"], d["page_table"],
                                 d["seq_lens"], d["cent"], c.topk, c.bos, c.eos, c.sm_scale,
                                 d["fill_pages"], out=d["out"], lse=d["lse"],
                                 order=d["order"] if args.plan else None, status=d["status"],
                                 workspace=d["ws"], head_dim_v=c.Dv)

    one = args.step_mode == "one-launch" and c.eos >= 1
    # Two-call mode: a page that fills at this step is its request's reserved last page
    # (eos >= 1) until the next step, so no score of this step reads its centroid: its build
    # runs on a second stream beside this step's fused call, and the stream joins again before
    # the next step.  One-launch mode folds the same build into the fused launch.
    side = torch.cuda.Stream(dev) if (c.eos >= 1 and not one) else None

    def build_call(d, prepared=False):
        if prepared:
            d["p_build"].run()
        else:
            vt.vt_build_centroids(d["k_pool"], d["fill_pages"], d["cent"], status=d["status"])

    def step(d, prepared=False, after_fused=None, overlap=True):
        if one:
            if args.plan:
                vt.vt_plan_requests(d["seq_lens"], d["order"])
            if prepared:
                d["p_step"].run()
            else:
                one_launch(d)
            if after_fused is not None:
                after_fused(d)
            return
        main = torch.cuda.current_stream(dev)
        if side is not None and overlap:
            side.wait_stream(main)  # this step's inputs are in place
            with torch.cuda.stream(side):
                build_call(d, prepared)
        else:
            build_call(d, prepared)
        if args.plan:
            vt.vt_plan_requests(d["seq_lens"], d["order"])
        if prepared:
            d["p_fused"].run()
        else:
            fused(d)
        if after_fused is not None:
            after_fused(d)
        if side is not None and overlap:
            main.wait_stream(side)  # the build is done before anything later on this stream

    launches_per_step = (1 if one else 2) + (1 if args.plan else 0)
    dominant = one_launch if one else fused  # the kernel the roofline is about
    for i in range(args.warmup):
        step(reps[i % args.replicas])
    torch.cuda.synchronize(dev)
    # The K timed steps (rotating over the input copies) are captured as one CUDA graph, as a
    # serving loop captures a whole decode pass (every layer's call) once and replays it, so
    # the timed region measures the GPU and not Python's per-call or per-graph launch overhead.
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for i in range(args.steps):
            step(reps[i % args.replicas])
    fused_graph = torch.cuda.CUDAGraph()  # the dominant kernel alone, the same sequence
    with torch.cuda.graph(fused_graph):
        for i in range(args.steps):
            dominant(reps[i % args.replicas])
    torch.cuda.synchronize(dev)
    graph.replay()  # untimed: the first replay of a graph uploads it
    fused_graph.replay()
    torch.cuda.synchronize(dev)
    barrier(world)

    clocks = ClockSampler(local) if rank == 0 else None
    if clocks:
        clocks.start()
        time.sleep(0.3)
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize(dev)
    t_start.record(stream)
    graph.replay()
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    elapsed = max_over_ranks(t_start.elapsed_time(t_end) / 1e3, world, dev)
    # average duration of one fused launch: the same launches back to back on the stream
    f_start, f_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f_start.record(stream)
    fused_graph.replay()
    f_end.record(stream)
    torch.cuda.synchronize(dev)
    fused_ms = f_start.elapsed_time(f_end) / args.steps

    # end to end through the public API: pinned host inputs in, results back, every step
    # (a serving loop stages a step's inputs in one pinned buffer and reads its results back
    # in one copy)
    in_h, _ = packed([w[k] for k in STEP_INPUTS], "cpu", pin=True)
    out_h = torch.empty(reps[0]["out_buf"].numel(), dtype=torch.uint8).pin_memory()
    h2d = in_h.numel()
    d2h = out_h.numel()

    # eager launches through the public API (no graph): each replica's two calls prepared
    # once (arguments checked and marshalled), as a serving loop does for its fixed buffers
    for d in reps:
        d["p_step"] = vt.prepare_sparse_decode_step(
            d["q"], d["k_pool"], d["v_pool"], d["page_table"], d["seq_lens"], d["cent"], c.topk,
            c.bos, c.eos, c.sm_scale, d["fill_pages"], out=d["out"], lse=d["lse"],
            order=d["order"] if args.plan else None, status=d["status"], head_dim_v=c.Dv,
            workspace=d["ws"])
        d["p_build"] = vt.prepare_build_centroids(d["k_pool"], d["fill_pages"], d["cent"],
                                                  status=d["status"])
        d["p_fused"] = vt.prepare_sparse_decode_fused(
            d["q"], d["k_pool"], d["v_pool"], d["page_table"], d["seq_lens"], d["cent"], c.topk,
            c.bos, c.eos, c.sm_scale, out=d["out"], lse=d["lse"],
            order=d["order"] if args.plan else None, status=d["status"], head_dim_v=c.Dv,
            workspace=d["ws"])

    # Every step copies its inputs in and reads its result back.  As a serving loop does, the
    # next step's input copy runs on a copy stream while this step computes (the steps rotate
    # over the input copies, so it never overwrites inputs still in use); the host then waits
    # for this step's result before it goes on.
    copy_stream = torch.cuda.Stream(dev)
    in_ready = [torch.cuda.Event() for _ in reps]
    res_ready = torch.cuda.Event()

    def copy_in(i):
        d = reps[i % args.replicas]
        with torch.cuda.stream(copy_stream):
            d["in_buf"].copy_(in_h, non_blocking=True)
            in_ready[i % args.replicas].record(copy_stream)

    def e2e_run(n):
        copy_in(0)
        for i in range(n):
            d = reps[i % args.replicas]
            stream.wait_event(in_ready[i % args.replicas])
            step(d, prepared=True, overlap=False,
                 after_fused=lambda d: out_h.copy_(d["out_buf"], non_blocking=True))
            res_ready.record(stream)
            if i + 1 < n:
                copy_in(i + 1)
            res_ready.synchronize()  # the host has this step's result

    e2e_run(args.warmup)
    barrier(world)
    torch.cuda.synchronize(dev)
    t0 = time.perf_counter()
    e2e_run(args.steps)
    e2e_s = max_over_ranks((time.perf_counter() - t0) / args.steps, world, dev)
    clk = clocks.stop() if clocks else None

    status = max(int(d["status"].item()) for d in reps)
    if status:
        raise SystemExit(f"device status {status}: an input was rejected by the kernels")
    graph.reset()
    fused_graph.reset()
    del reps, graph, fused_graph
    torch.cuda.empty_cache()

    peak, peak_kind = read_peak_hbm()
    per_config = None
    if world == 1 and not args.no_per_config:
        pc_clocks = ClockSampler(local)
        pc_clocks.start()
        per_config = {}
        for cfg in (1, 2, 3, 4, 5):
            t0 = time.perf_counter()
            per_config[str(cfg)] = measure_config(vt, cfg, dev, peak)
            log(f"config {cfg}: {time.perf_counter() - t0:.1f} s, fused "
                f"{per_config[str(cfg)]['fused']['us']} us")
        t0 = time.perf_counter()
        per_config["serving_pass"] = measure_serving_pass(vt, dev, peak)
        log(f"serving pass: {time.perf_counter() - t0:.1f} s, "
            f"{per_config['serving_pass']['pass_us']} us")
        per_config["clocks"] = pc_clocks.stop()
        per_config["timing"] = ("per row: 10 calls captured as one CUDA graph, one untimed "
                                "replay, one replay between CUDA events; us = per call")

    if rank != 0:
        return
    ms = elapsed / args.steps * 1e3
    units = c.B * c.Hq
    value = aggregate_value(world, units, args.steps, elapsed)
    launch_bytes = nbytes["total"] if one else nbytes["fused"]
    achieved = launch_bytes / (fused_ms / 1e3) / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": workload_config(c, w, args),
        "roofline": {
            "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
            "frac": achieved / peak, "frac_nominal_8000": achieved / NOMINAL_HBM_GBS,
            "frac_note": ("frac is against the measured copy peak (the roofline's denominator); "
                          "frac_nominal_8000 against the nominal ~8 TB/s HBM3e figure"),
            "traffic": recorded_traffic(args.config),
            "kernel": ("persist_mla_kernel" if c.mla else "persist_fused_kernel")
                      + (" (vt_sparse_decode_step: filled pages' build + select + attend)"
                         if one else " (vt_sparse_decode_fused)"),
            "algorithmic_bytes_per_launch": launch_bytes, "kernel_ms": fused_ms,
            "peak_source": f"{peak_kind} hbm_gbs (MEASURED_PEAKS.json)" if peak_kind == "measured"
            else "fallback 6650 GB/s",
        },
        "e2e": {"value": world * units / e2e_s, "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "how": "public API (prepared vt_sparse_decode_step), eager launches; each step "
                       "copies its inputs from pinned host memory (on a copy stream, while the "
                       "previous step computes) and the host waits for its result copied back; "
                       "wall clock per step"},
        "gpu_launches": launches_per_step * args.steps,
        "timing": "the K steps as one CUDA graph replayed once, CUDA events on the launching stream",
        "step": ("vt_sparse_decode_step: the centroid build of the pages filled this step "
                 "and the fused select + attend in one launch" if one else
                 "vt_build_centroids (pages filled this step) on a second stream beside "
                 "vt_sparse_decode_fused, joined before the next step (e2e: one stream)"
                 if side is not None else "vt_build_centroids then vt_sparse_decode_fused"),
        "clocks": clk,
        "step_bytes": nbytes,
    }
    if per_config is not None:
        line["per_config"] = per_config
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w)
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------------------------
# every workload of the hot-path table: fused launch, split calls, centroid builds
# ------------------------------------------------------------------------------------------
def graph_time_ms(calls, iters: int, dev) -> float:
    """Average ms of one call: `iters` calls (rotating over `calls`) captured as one CUDA graph,
    replayed once untimed, then once between CUDA events on the launching stream."""
    for i in range(2):
        calls[i % len(calls)]()
    torch.cuda.synchronize(dev)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(iters):
            calls[i % len(calls)]()
    g.replay()
    torch.cuda.synchronize(dev)
    stream = torch.cuda.current_stream(dev)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    g.replay()
    t1.record(stream)
    torch.cuda.synchronize(dev)
    ms = t0.elapsed_time(t1) / iters
    del g
    return ms


def measure_config(vt, cfg: int, dev, peak: float, iters: int = 10) -> dict:
    """One workload of the hot-path table on this GPU: the fused call (and, where the table
    asks for them, select-only, decode-only, select + decode back to back, the centroid build
    of the pages filled this step, and a build of every page of the pool).  Inputs whose
    per-call bytes are below 4x the 126 MB L2 rotate over copies so that no call finds its data
    in L2; the tiny workload is launch-bound and runs from L2."""
    c = config(cfg)
    w = make_workload(c, seed=1000 + cfg)
    nb = algorithmic_bytes(c, w["seq_lens"])
    vb = variant_bytes(c, w["seq_lens"])
    l2 = 126e6
    reps = 1 if (nb["fused"] >= 4 * l2 or nb["fused"] < 1e6) else min(3, 1 + int(4 * l2 // nb["fused"]))
    ds = []
    for _ in range(reps):
        d = {k: w[k].to(dev) for k in ("q", "k_pool", "page_table", "seq_lens", "prebuilt_pages",
                                       "fill_pages")}
        d["v_pool"] = d["k_pool"] if w["v_pool"] is w["k_pool"] else w["v_pool"].to(dev)
        d["cent"] = torch.zeros((w["P"], c.Hkv, c.D), dtype=torch.float32, device=dev)
        vt.vt_build_centroids(d["k_pool"], d["prebuilt_pages"], d["cent"])
        vt.vt_build_centroids(d["k_pool"], d["fill_pages"], d["cent"])
        d["out"] = torch.empty((c.B, c.Hq, c.Dv), dtype=torch.bfloat16, device=dev)
        d["lse"] = torch.empty((c.B, c.Hq), dtype=torch.float32, device=dev)
        d["sel"] = torch.empty((c.B, c.Hkv, c.kmax), dtype=torch.int32, device=dev)
        d["n_sel"] = torch.empty((c.B, c.Hkv), dtype=torch.int32, device=dev)
        d["status"] = torch.zeros((1,), dtype=torch.int32, device=dev)
        d["ws"] = vt.fused_workspace(d["q"], d["k_pool"], d["v_pool"], d["page_table"],
                                     d["seq_lens"], d["cent"], c.topk, c.bos, c.eos,
                                     head_dim_v=c.Dv)
        ds.append(d)
    torch.cuda.synchronize(dev)

    def fused(d):
        return lambda: vt.vt_sparse_decode_fused(
            d["q"], d["k_pool"], d["v_pool"], d["page_table"], d["seq_lens"], d["cent"], c.topk,
            c.bos, c.eos, c.sm_scale, out=d["out"], lse=d["lse"], status=d["status"],
            workspace=d["ws"], head_dim_v=c.Dv)

    def select(d):
        return lambda: vt.vt_select_pages(d["q"], d["k_pool"], d["v_pool"], d["page_table"],
                                          d["seq_lens"], d["cent"], c.topk, c.bos, c.eos,
                                          sel=d["sel"], n_sel=d["n_sel"], status=d["status"],
                                          head_dim_v=c.Dv)

    def select_ws(d):
        return lambda: vt.vt_select_pages(d["q"], d["k_pool"], d["v_pool"], d["page_table"],
                                          d["seq_lens"], d["cent"], c.topk, c.bos, c.eos,
                                          sel=d["sel"], n_sel=d["n_sel"], status=d["status"],
                                          head_dim_v=c.Dv, workspace=d["ws"])

    def decode_ws(d):
        return lambda: vt.vt_sparse_decode(d["q"], d["k_pool"], d["v_pool"], d["page_table"],
                                           d["seq_lens"], d["sel"], d["n_sel"], c.sm_scale,
                                           out=d["out"], lse=d["lse"], status=d["status"],
                                           head_dim_v=c.Dv, workspace=d["ws_dec"])

    def select_lossy(d):
        return lambda: vt.vt_select_pages_approx(d["q"], d["k_pool"], d["v_pool"], d["page_table"],
                                                 d["seq_lens"], d["cent"], c.topk, c.bos, c.eos,
                                                 0x5EED, sel=d["sel"], n_sel=d["n_sel"],
                                                 status=d["status"], head_dim_v=c.Dv)

    def decode(d):
        return lambda: vt.vt_sparse_decode(d["q"], d["k_pool"], d["v_pool"], d["page_table"],
                                           d["seq_lens"], d["sel"], d["n_sel"], c.sm_scale,
                                           out=d["out"], lse=d["lse"], status=d["status"],
                                           head_dim_v=c.Dv)

    def row(ms, nbytes):
        gbs = nbytes / (ms / 1e3) / 1e9
        return {"us": round(ms * 1e3, 2), "bytes": nbytes, "GB_s": round(gbs, 1),
                "frac": round(gbs / peak, 4), "frac_nominal_8000": round(gbs / NOMINAL_HBM_GBS, 4),
                "req_heads_per_s": c.B * c.Hq / (ms / 1e3)}

    res = {"workload": f"{c.name} (B={c.B}, Hq={c.Hq}, Hkv={c.Hkv}, D={c.D}/{c.Dv}, context "
                       f"{lengths_text(c)}, top-{c.topk}+{c.bos}+{c.eos}, pool {w['P']} pages)",
           "input_copies": reps}
    res["fused"] = row(graph_time_ms([fused(d) for d in ds], iters, dev), nb["fused"])
    if cfg in (2, 3, 5):
        res["select_only"] = row(graph_time_ms([select(d) for d in ds], iters, dev), vb["select"])
        res["select_only_workspace"] = row(graph_time_ms([select_ws(d) for d in ds], iters, dev),
                                           vb["select"])
        res["select_only_lossy"] = row(graph_time_ms([select_lossy(d) for d in ds], iters, dev),
                                       vb["select"])
    if cfg == 4:  # the MLA split calls: the cluster kernel, and the persistent kernel's modes
        res["select_only"] = row(graph_time_ms([select(d) for d in ds], iters, dev), vb["select"])
        res["select_only_workspace"] = row(graph_time_ms([select_ws(d) for d in ds], iters, dev),
                                           vb["select"])
    if cfg in (2, 3, 4):
        for d in ds:
            select(d)()
        res["decode_only"] = row(graph_time_ms([decode(d) for d in ds], iters, dev), vb["decode"])
        res["select_then_decode"] = row(
            graph_time_ms([(lambda d=d: (select(d)(), decode(d)())) for d in ds], iters, dev),
            vb["select"] + vb["decode"])
    if cfg in (2, 3, 4):
        for d in ds:
            d["ws_dec"] = vt.decode_workspace(d["q"], d["k_pool"], d["v_pool"], d["page_table"],
                                              d["seq_lens"], d["sel"], head_dim_v=c.Dv)
        res["decode_only_workspace"] = row(graph_time_ms([decode_ws(d) for d in ds], iters, dev),
                                           vb["decode"])
        res["select_then_decode_workspace"] = row(
            graph_time_ms([(lambda d=d: (select_ws(d)(), decode_ws(d)())) for d in ds], iters,
                          dev), vb["select"] + vb["decode"])
    n_fill = int(w["fill_pages"].numel())
    if n_fill:
        d = ds[0]
        res["build_filled_pages"] = dict(pages=n_fill, **row(graph_time_ms(
            [lambda: vt.vt_build_centroids(d["k_pool"], d["fill_pages"], d["cent"],
                                           status=d["status"])], iters, dev),
            build_bytes(c, n_fill)))
        res["build_filled_pages"].pop("req_heads_per_s")
    if cfg == 3:
        d = ds[0]
        allp = torch.arange(w["P"], dtype=torch.int32, device=dev)
        res["build_all_pages"] = dict(pages=w["P"], **row(graph_time_ms(
            [lambda: vt.vt_build_centroids(d["k_pool"], allp, d["cent"], status=d["status"])],
            5, dev), build_bytes(c, w["P"])))
        res["build_all_pages"].pop("req_heads_per_s")
    torch.cuda.synchronize(dev)
    if any(int(d["status"].item()) for d in ds):
        raise SystemExit(f"config {cfg}: device status set: an input was rejected by the kernels")
    del ds
    torch.cuda.empty_cache()
    return res


def measure_serving_pass(vt, dev, peak: float, L: int = 28, copies: int = 3) -> dict:
    """A serving-shaped decode pass over the Qwen3-0.6B-like batch: L layers, each one
    vt_sparse_decode_step launch (the build of the pages filled at this step, then select +
    attend), layer 0 dense (every page attended: the README runs its sparse attention with
    vortex_layers_skip = [0]), captured as one CUDA graph as a serving engine captures its
    decode step.  Layer l has its own query and reads K/V pool copy l % copies (each with its
    own centroid cache): the copies hold 3 x 2.6 GB, so no layer finds its data in L2."""
    c = config(2)
    w = make_workload(c, seed=1002)
    dense_topk = int(w["page_table"].shape[1])  # >= every request's candidates
    pools = []
    for r in range(copies):
        d = {k: w[k].to(dev) for k in ("k_pool", "v_pool", "page_table", "seq_lens",
                                       "prebuilt_pages", "fill_pages")}
        d["cent"] = torch.zeros((w["P"], c.Hkv, c.D), dtype=torch.float32, device=dev)
        vt.vt_build_centroids(d["k_pool"], d["prebuilt_pages"], d["cent"])
        pools.append(d)
    g = torch.Generator().manual_seed(77)
    layers = []
    for l in range(L):
        d = dict(pools[l % copies])
        d["q"] = torch.randn((c.B, c.Hq, c.D), generator=g).to(torch.bfloat16).to(dev)
        d["topk"] = dense_topk if l == 0 else c.topk
        d["out"] = torch.empty((c.B, c.Hq, c.Dv), dtype=torch.bfloat16, device=dev)
        d["lse"] = torch.empty((c.B, c.Hq), dtype=torch.float32, device=dev)
        d["status"] = torch.zeros((1,), dtype=torch.int32, device=dev)
        d["ws"] = vt.fused_workspace(d["q"], d["k_pool"], d["v_pool"], d["page_table"],
                                     d["seq_lens"], d["cent"], d["topk"], c.bos, c.eos)
        layers.append(d)
    torch.cuda.synchronize(dev)

    def layer_call(d):
        return lambda: vt.vt_sparse_decode_step(
            d["q"], d["k_pool"], d["v_pool"], d["page_table"], d["seq_lens"], d["cent"],
            d["topk"], c.bos, c.eos, c.sm_scale, d["fill_pages"], out=d["out"], lse=d["lse"],
            status=d["status"], workspace=d["ws"])

    calls = [layer_call(d) for d in layers]
    pass_us = graph_time_ms([lambda: [f() for f in calls]], 3, dev) * 1e3
    dense_us = graph_time_ms([calls[0]], 6, dev) * 1e3
    sparse_us = graph_time_ms(calls[1:], 3 * (L - 1), dev) * 1e3
    if any(int(d["status"].item()) for d in layers):
        raise SystemExit("serving pass: device status set")
    nb = algorithmic_bytes(c, w["seq_lens"])
    dense_cfg = dataclasses.replace(c, topk=dense_topk)
    nbd = algorithmic_bytes(dense_cfg, w["seq_lens"])
    # end to end: the step's host inputs (page tables, lengths, filled pages) in, the pass, the
    # last layer's output back, per pass (the queries of later layers come from the model on
    # the device)
    host = [w[k].pin_memory() for k in ("page_table", "seq_lens", "fill_pages")]
    out_h = torch.empty_like(layers[-1]["out"], device="cpu").pin_memory()
    gr = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gr):
        for f in calls:
            f()
    gr.replay()
    torch.cuda.synchronize(dev)
    stream = torch.cuda.current_stream(dev)
    h2d = sum(t.numel() * t.element_size() for t in host)

    def e2e_pass():
        for d in pools:
            for t, k in zip(host, ("page_table", "seq_lens", "fill_pages")):
                d[k].copy_(t, non_blocking=True)
        gr.replay()
        out_h.copy_(layers[-1]["out"], non_blocking=True)
        stream.synchronize()

    for _ in range(3):
        e2e_pass()
    t0 = time.perf_counter()
    reps = 10
    for _ in range(reps):
        e2e_pass()
    e2e_us = (time.perf_counter() - t0) / reps * 1e6
    res = {
        "workload": f"{L}-layer decode pass of the {c.name} batch (layer 0 dense, layers 1.."
                    f"{L - 1} top-{c.topk}+{c.bos}+{c.eos}), one vt_sparse_decode_step launch "
                    f"per layer, captured as one CUDA graph",
        "layers": L, "pass_us": round(pass_us, 1),
        "sparse_layer_us": round(sparse_us, 2), "dense_layer_us": round(dense_us, 2),
        "sparse_layer_frac": round(nb["total"] / (sparse_us / 1e6) / 1e9 / peak, 4),
        "dense_layer_frac": round(nbd["total"] / (dense_us / 1e6) / 1e9 / peak, 4),
        "tokens_per_s": c.B / (pass_us / 1e6),
        "e2e": {"pass_us": round(e2e_us, 1), "tokens_per_s": c.B / (e2e_us / 1e6),
                "h2d_bytes_per_pass": h2d * len(pools),
                "d2h_bytes_per_pass": out_h.numel() * out_h.element_size()},
    }
    del gr, layers, pools
    torch.cuda.empty_cache()
    return res


def cpu_baseline(w) -> dict:
    """The oracle, as it stands, on a bounded sample of the same workload (~10 s of CPU on all
    cores of the affinity mask), plus two labelled variants on smaller samples: the same C
    source built with fp32 arithmetic and -O3 -march=native (a timing-only copy), and the
    fp64 oracle on one thread."""
    import oracle
    c = w["config"]
    cent = oracle_prepare(w)

    def timed(reqs, kind, min_s, max_s):
        oracle_step(w, cent, reqs, kind=kind)  # warm
        t0 = time.perf_counter()
        reps = 0
        while reps < 2 or time.perf_counter() - t0 < min_s:
            oracle_step(w, cent, reqs, kind=kind)
            reps += 1
            if time.perf_counter() - t0 > max_s:
                break
        return (time.perf_counter() - t0) / reps, reps

    reqs = oracle_sample_size(w, cent, target_s=3.0)
    dt, reps = timed(reqs, "f64", 10.0, 30.0)
    res = {"value": len(reqs) * c.Hq / dt, "unit": UNIT, "cores": oracle.get_threads(),
           "kind": "oracle",
           "sample": f"{reps} oracle steps over requests 0..{len(reqs) - 1} of the same batch "
                     f"({len(reqs) * c.Hq} req-heads each; build of filled pages + select + "
                     f"attend), fp64"}
    variants = []
    dt32, reps32 = timed(reqs, "f32", 3.0, 10.0)
    variants.append({"value": len(reqs) * c.Hq / dt32, "unit": UNIT,
                     "cores": oracle.get_threads("f32"),
                     "kind": "oracle source built with fp32 arithmetic, gcc -O3 -march=native "
                             "(timing-only copy)",
                     "sample": f"{reps32} steps over requests 0..{len(reqs) - 1}"})
    oracle.set_threads(1)
    try:
        one = reqs[: max(1, len(reqs) // 8)]
        dt1, reps1 = timed(one, "f64", 3.0, 10.0)
    finally:
        oracle.set_threads(0)
    variants.append({"value": len(one) * c.Hq / dt1, "unit": UNIT, "cores": 1,
                     "kind": "oracle, one thread",
                     "sample": f"{reps1} steps over requests 0..{len(one) - 1}"})
    res["variants"] = variants
    return res


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--replicas", type=int, default=3)
    ap.add_argument("--config", type=int, default=CFG, choices=[1, 2, 3, 4, 5],
                    help="workload of the hot-path table (the headline line is config 2)")
    ap.add_argument("--plan", action="store_true",
                    help="add the vt_plan_requests launch to the step")
    ap.add_argument("--step-mode", choices=["one-launch", "two-call"], default="one-launch",
                    help="the step as one vt_sparse_decode_step launch, or vt_build_centroids "
                         "beside vt_sparse_decode_fused on two streams")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the per-workload rows (configs 1-5) of the default run")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    world, rank, local = dist_setup(args.gpus)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
