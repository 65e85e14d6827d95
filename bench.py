"""Benchmark of the VSA-H3 forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl vsa|reference] [--workload NAME]

One step = one whole VSA-H3 forward (gather + pool, pooled scores, top-k +
compression, block-sparse attention + gated epilogue) over one synthetic
input already resident in HBM, timed through the public call vsa_forward.
The per-stage times (and the attention time the roofline uses) come from a
second pass right after, through the step entry points.  The default workload is the 1344x768-shaped
one at sparsity 0.9 (56 heads, D=128, 73,728 video + 1,280 prefix tokens).

Metric: effective TFLOP/s counting only the selected (query tile, key tile)
pairs, 4*T*T*D FLOP each for T-token tiles (T = 64, or 128 for the
128-token-tile workload), per whole forward; ms per call is reported too.
Multi-GPU (torchrun), two modes:
  --mode ulysses (the default with more than one rank): ONE forward split over
      the ranks the way sequence parallelism holds it.  Rank r keeps tokens
      [r*L/N, (r+1)*L/N) of q, k, v, gate and out in its own HBM, maps the other
      ranks' parts through CUDA IPC, and runs vsa_forward_parts for heads
      [r*H/N, (r+1)*H/N): the gather kernel's loads and the epilogue's stores
      carry the two all-to-all exchanges over NVLink (plain peer loads and
      stores, no library kernel on peer memory).  value = one forward's FLOPs /
      the slowest rank's time ("scaling": "strong").
  --mode replicas: every rank runs its own whole forward on its own seeded
      input (no exchange); value = all ranks' FLOPs / the slowest rank's time
      ("scaling": "weak").
With one GPU both modes are the plain forward.

``--impl reference`` times the CPU oracle on a bounded sample of the same
workload on this host's cores (rank 0 only).
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "VSA-H3 fwd ms/call & effective TFLOPS (selected tiles) at 73.7k tok, 56 heads"
UNIT = "TFLOP/s"
L2_BYTES = 126 * 1024 * 1024


def tile_flops(D: int, tile: int = 64) -> int:
    return 4 * tile * tile * D


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return dict(source="measured", bf16_tflops=d["bf16_tflops"],
                    bf16_tflops_sustained=d.get("bf16_tflops_sustained", d["bf16_tflops"]), hbm_gbs=d["hbm_gbs"])
    return dict(source="fallback", bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, hbm_gbs=6650.0)


def attn_launches(w, heads):
    """Attention kernels of one bf16 tile-order forward over `heads` heads: with 128-token tiles the pair
    kernel alone; with 64-token tiles the video kernel, plus the pair kernel for the prefix query row
    blocks when their pairs, B * heads * ceil(P / 2), fill the SMs (the library's rule)."""
    import torch

    if w.tile == 128:
        return 1
    prefix_tiles = sum((n + 63) // 64 for n in w.segments)
    sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    return 1 + int(prefix_tiles > 0 and w.batch * heads * ((prefix_tiles + 1) // 2) >= sms)


def measured_attn_traffic():
    """DRAM bytes (read + write) of one attention launch from the committed ncu
    capture, or None when the kernel sources changed since it was taken."""
    import hashlib

    path = os.path.join(ROOT, "profiles", "vsa_attn_kernel_768p_s0.9_traffic.txt")
    if not os.path.exists(path):
        return None
    vals = {}
    with open(path) as f:
        for line in f:
            if line.startswith("#") or ":" not in line:
                continue
            k, v = line.split(":", 1)
            vals[k.strip()] = v.strip()
    h = hashlib.sha256()
    for rel in ("block_sparse_tiled_b200/csrc/attn_sm100.cuh", "block_sparse_tiled_b200/csrc/attn_pair_sm100.cuh",
                "block_sparse_tiled_b200/csrc/ptx.cuh"):
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    if vals.get("kernel_source_sha256") != h.hexdigest():
        return None
    return int(vals["dram_bytes_read"]) + int(vals["dram_bytes_write"])


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._t = threading.Thread(target=self._read, daemon=True)
            self._t.start()
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


def dist_setup(args):
    import torch

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        backend = "nccl" if (args.impl == "vsa" and torch.cuda.is_available()) else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def max_over_ranks(x: float, world: int, device=None) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


# ----------------------------------------------------------------------------- oracle (CPU) timing


def oracle_sample(w, every: int, seed: int = 0):
    """Time the CPU oracle on head 0 of the workload: full selection (pool,
    scores, top-k, compression) and the fine branch + output of every
    ``every``-th query tile.  Returns (seconds, selected-tile FLOPs, description)."""
    import numpy as np
    import torch

    import oracle
    import synth

    x = synth.make_inputs(dataclasses.replace(w, heads=1), seed=seed, device="cpu")
    xb = {n: synth.as_bits(x[n]) for n in ("q", "k", "v", "gate")}
    t0 = time.perf_counter()
    sel = oracle.selection(xb["q"], xb["k"], xb["v"], w.segments, w.grid, w.sparsity, tile=w.tile, cube=w.cube,
                           ref_segments=w.ref_segments, ref_keep=w.ref_keep)
    geo = sel["geo"]
    items = np.arange(0, geo.n_tiles, every, dtype=np.int64)
    of = oracle.fine_tiles(xb["q"], xb["k"], xb["v"], geo, sel["idx"], sel["topk"], sel["scale"], items)
    oracle.output_tiles(of, sel["o_c"], xb["gate"], geo, items, 1)
    dt = time.perf_counter() - t0
    pairs = sum((geo.n_tiles if i < geo.n_prefix else geo.n_prefix - geo.n_ref + sel["kr"] + sel["topk"])
                for i in items)
    flops = pairs * tile_flops(w.head_dim, w.tile)
    desc = (f"head 0 of 56: full selection (pool, fp32 scores, top-k, compression over {geo.n_tiles} tiles) "
            f"+ fine branch and output of every {every}th query tile ({len(items)} of {geo.n_tiles} tiles, "
            f"{pairs} selected tile pairs)")
    del torch
    return dt, flops, desc


def omp_threads():
    n = os.environ.get("OMP_NUM_THREADS")
    return int(n) if n else (os.cpu_count() or 1)


def run_reference(args, w, world, rank, mode="replicas"):
    """CPU oracle arm: rank 0 only."""
    if rank != 0:
        return
    every = args.ref_every
    for _ in range(args.warmup):
        oracle_sample(w, every)
    times, flops, desc = [], 0, ""
    for _ in range(args.steps):
        dt, flops, desc = oracle_sample(w, every)
        times.append(dt)
    ms = 1e3 * statistics.mean(times)
    value = flops / (ms * 1e-3) / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak" if mode == "replicas" else "strong", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded counter-based normal)",
        "config": config_dict(w, world=world, mode=mode),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": omp_threads(), "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- GPU arm


def config_dict(w, dims=None, world=1, mode="replicas"):
    import oracle

    geo = oracle.geometry(w.segments, w.grid, tile=w.tile, cube=w.cube, ref_segments=w.ref_segments) \
        if dims is None else None
    n_t = dims["n_tiles"] if dims else geo.n_tiles
    P = dims["n_prefix_tiles"] if dims else geo.n_prefix
    V = n_t - P
    k = dims["topk"] if dims else oracle.topk_count(w.sparsity, V)
    R = dims["n_ref_tiles"] if dims else geo.n_ref
    kr = dims["ref_topk"] if dims else (oracle.ref_count(w.ref_keep, R) if R and V else 0)
    pairs = V * (P - R + kr + k) + P * n_t
    return {
        "workload": w.name, "description": w.description, "batch": w.batch, "heads": w.heads,
        "head_dim": w.head_dim, "seq_len": w.seq_len, "prefix_segments": list(w.segments), "grid": list(w.grid),
        "tile_size": w.tile, "n_tiles": n_t, "n_prefix_tiles": P, "n_video_tiles": V, "sparsity": w.sparsity,
        "topk": k, **({"n_ref_tiles": R, "ref_keep": w.ref_keep, "ref_topk": kr} if R else {}),
        "selected_tile_pairs": pairs * w.batch * w.heads,
        "selected_tflop_per_call": pairs * w.batch * w.heads * tile_flops(w.head_dim, w.tile) / 1e12,
        "l2": "no flush: Q/K/V/out are %.1f GB per step, > 126 MB L2" % (4 * w.batch * w.seq_len * w.heads * w.head_dim * 2 / 1e9),
        "parallelism": (f"independent forward per GPU x{world}" if world == 1 or mode == "replicas"
                        else f"ulysses sequence parallel sp{world} (heads and token parts over {world} GPUs)"),
    }


def prep_roofline(w, dims, stage_ms, peaks, sm_mhz):
    """Achieved rates of the selection kernels against their own rooflines: HBM bytes for the gather
    and for top-k + compression (algorithmic bytes per launch, counted from the tensors each reads and
    writes), fp32 FMA throughput for the pooled scores (nominal: 128 FMA lanes per SM per clock at the
    sampled SM clock, no measured fp32 peak exists)."""
    B, H, D, L = w.batch, w.heads, w.head_dim, w.seq_len
    n_t, P, k, kr = dims["n_tiles"], dims["n_prefix_tiles"], dims["topk"], dims["ref_topk"]
    T = dims["tile_size"]
    V = n_t - P
    bh = B * H
    gather_bytes = (3 * B * L * H * D * 2            # q, k, v read (each token once)
                    + 3 * bh * n_t * T * D * 2         # tile-order copies written (pads included)
                    + 3 * bh * n_t * D * 4             # pooled tiles written
                    + bh * n_t * T * 4 + bh * 8)       # query row norms, key/value maxima
    scores_flop = 2 * bh * n_t * n_t * D
    scores_bytes = 2 * bh * n_t * D * 4 + bh * n_t * n_t * 4
    sel_bytes = bh * n_t * n_t * 4 + bh * n_t * D * 4 + bh * V * (k + kr) * 4 + bh * n_t * D * 4
    compress_flop = 2 * bh * n_t * n_t * D
    hbm = peaks["hbm_gbs"]
    fp32_nominal = 148 * 128 * 2 * (sm_mhz or 1965.0) * 1e6 / 1e12  # TFLOP/s

    def gbs(nbytes, ms):
        return nbytes / (ms * 1e-3) / 1e9

    g = gbs(gather_bytes, stage_ms["gather_pool"])
    t = gbs(sel_bytes, stage_ms["topk_compress"])
    sc = scores_flop / (stage_ms["scores"] * 1e-3) / 1e12
    return {
        "gather_pool": {"bound": "hbm", "bytes": gather_bytes, "achieved_gbs": g, "peak_gbs": hbm, "frac": g / hbm},
        "scores": {"bound": "alu", "flop": scores_flop, "bytes": scores_bytes, "achieved_tflops": sc,
                   "peak_tflops_nominal_fp32": fp32_nominal, "frac": sc / fp32_nominal,
                   "achieved_gbs": gbs(scores_bytes, stage_ms["scores"])},
        "topk_compress": {"bound": "hbm", "bytes": sel_bytes, "achieved_gbs": t, "peak_gbs": hbm, "frac": t / hbm,
                          "compress_flop": compress_flop,
                          "compress_tflops": compress_flop / (stage_ms["topk_compress"] * 1e-3) / 1e12},
        "peak_note": f"HBM: {peaks['source']} copy bandwidth; fp32: nominal, 148 SMs x 128 FMA/clk at the "
                     f"sampled median SM clock",
    }


def run_vsa(args, w, world, rank, local, mode="replicas"):
    import torch

    import block_sparse_tiled_b200 as vsa
    import synth

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    x = synth.make_inputs(w, seed=rank, device=dev)
    torch.cuda.synchronize()
    plan = vsa.vsa_plan_tiles(batch=w.batch, heads=w.heads, head_dim=w.head_dim, segments=w.segments, grid=w.grid,
                              sparsity=w.sparsity, tile_size=w.tile, cube=w.cube, ref_segments=w.ref_segments,
                              ref_keep=w.ref_keep)
    dims = plan.dims
    ws = vsa.alloc_workspace(plan, dev)
    v = vsa.workspace_views(plan, ws)
    out = torch.empty_like(x["q"])
    stream = torch.cuda.current_stream(dev)
    flops_call = dims["selected_pairs"] * w.batch * w.heads * tile_flops(w.head_dim, w.tile)

    def forward():
        vsa.vsa_forward(plan, x["q"], x["k"], x["v"], x["gate"], out=out, workspace=ws, stream=stream)

    for _ in range(args.warmup):
        forward()
    torch.cuda.synchronize()
    code, where = vsa.device_status(plan)
    if code != 0:
        raise RuntimeError(f"device status {code} at site {where} during warm-up")

    # ---- the timed region: K whole forwards through the public call, one per step
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record(stream)
        for _ in range(args.steps):
            forward()
        stop.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    elapsed_ms = start.elapsed_time(stop)
    elapsed_ms = max_over_ranks(elapsed_ms, world, dev)
    code, where = vsa.device_status(plan)
    if code != 0:
        raise RuntimeError(f"device status {code} at site {where} in the timed region")
    ms_step = elapsed_ms / args.steps
    value = world * flops_call / (ms_step * 1e-3) / 1e12
    clocks = clk.summary()

    # ---- stage pass, right after: the same forward through the four step entry points (the gather's
    # overflow-bound statistics passed on to the attention, as vsa_forward does), with an event between
    # stages; the attention's mean time here is the roofline's kernel time
    ev = {n: [] for n in ("t0", "t1", "t2", "t3", "t4")}
    for _ in range(args.steps):
        e = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
        e[0].record(stream)
        vsa.vsa_gather_tiles(plan, x["q"], x["k"], x["v"], v["q_t"], v["k_t"], v["v_t"], v["pq"], v["pk"], v["pv"],
                             q_norm=v["q_n"], kv_max=v["kv_max"], stream=stream)
        e[1].record(stream)
        vsa.vsa_pool_and_score(plan, None, None, None, v["pq"], v["pk"], v["pv"], v["scores"], stream=stream)
        e[2].record(stream)
        vsa.vsa_topk_select(plan, v["scores"], v["pv"], v["idx"], v["o_c"], stream=stream)
        e[3].record(stream)
        vsa.vsa_sparse_attn_fwd(plan, v["q_t"], v["k_t"], v["v_t"], v["idx"], v["o_c"], x["gate"], out,
                                q_norm=v["q_n"], kv_max=v["kv_max"], stream=stream)
        e[4].record(stream)
        for n, evt in zip(("t0", "t1", "t2", "t3", "t4"), e):
            ev[n].append(evt)
    torch.cuda.synchronize()

    def avg(a, b):
        return statistics.mean(x.elapsed_time(y) for x, y in zip(ev[a], ev[b]))

    stage_ms = {"gather_pool": avg("t0", "t1"), "scores": avg("t1", "t2"), "topk_compress": avg("t2", "t3"),
                "attention": avg("t3", "t4")}

    # end to end through the public call with host buffers (pinned), copies inside the timed region
    hx = {}
    for n in ("q", "k", "v", "gate"):  # pinned host copies, allocated once (no pageable intermediate)
        hx[n] = torch.empty(x[n].shape, dtype=x[n].dtype, pin_memory=True)
        hx[n].copy_(x[n])
    hout = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    # host inputs take the head-chunked pipeline: copies of one chunk overlap the forward of the next;
    # its device workspace is allocated by this first call and kept on the plan
    vsa.vsa_forward(plan, hx["q"], hx["k"], hx["v"], hx["gate"], out=hout)
    torch.cuda.synchronize()
    e2e_steps = max(1, min(args.steps, 3))
    barrier(world)
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s0.record(stream)
    for _ in range(e2e_steps):
        vsa.vsa_forward(plan, hx["q"], hx["k"], hx["v"], hx["gate"], out=hout)
    s1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(s0.elapsed_time(s1) / e2e_steps, world, dev)
    h2d = sum(t.numel() * t.element_size() for t in hx.values())
    d2h = hout.numel() * hout.element_size()

    peaks = load_peaks()
    attn_tflops = flops_call / (stage_ms["attention"] * 1e-3) / 1e12
    sm_mhz = clocks.get("sm_mhz")
    # clock-normalised: SM cycles per 64-query x 128-key block of the attention (per SM), and per launch
    blocks = flops_call / (2 * tile_flops(w.head_dim, 64))
    attn_cycles = stage_ms["attention"] * 1e-3 * sm_mhz * 1e6 if sm_mhz else None
    roofline = {
        "kernel": (f"attention stage: vsa_attn_pair_kernel<{w.head_dim}> (every 128-token query tile, its two "
                   f"64-row halves together)" if w.tile == 128 else
                   f"attention stage: vsa_attn_kernel<{w.head_dim}> (video query row blocks)" +
                   (f" and vsa_attn_pair_kernel<{w.head_dim}> (prefix query row blocks, two at a time)"
                    if attn_launches(w, w.heads) == 2 else "")),
        "bound": "tensor", "achieved": attn_tflops,
        "peak": peaks["bf16_tflops"], "unit": "TFLOP/s", "frac": attn_tflops / peaks["bf16_tflops"],
        "peak_kind": f"{peaks['source']} burst dense bf16 (cuBLAS)",
        "frac_of_sustained_peak": attn_tflops / peaks["bf16_tflops_sustained"],
        "kernel_time": "mean of the attention launches in the stage pass that follows the timed region",
        "algorithmic_flop_per_launch": flops_call,
        "attn_mcycles_per_launch": attn_cycles / 1e6 if attn_cycles else None,
        "cycles_per_block_per_sm": attn_cycles * 148 / blocks if attn_cycles else None,
        "traffic": measured_attn_traffic() if w.name == "768p_s0.9" else None,
        "traffic_unit": "bytes per launch (ncu dram__bytes_read.sum + dram__bytes_write.sum)",
    }
    # library kernels per timed step (one vsa_forward): gate check, gather+pool, scores, a top-k pass over
    # the reference candidates (with reference segments), top-k + compression in one kernel (rows of up to
    # 1280 tiles; longer rows take a top-k and a compression kernel), attention (one or two kernels)
    nv = dims["n_video_tiles"]
    fused = (dims["n_tiles"] + 31) // 32 <= 40
    launches = (4 + int(nv > 0 and dims["ref_topk"] > 0) + int(not fused) + attn_launches(w, w.heads)) * args.steps
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak" if mode == "replicas" else "strong",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded counter-based normal, structured tile offsets)",
        "config": config_dict(w, dims, world=world, mode=mode),
        "stage_ms": stage_ms, "roofline": roofline,
        "prep_roofline": prep_roofline(w, dims, stage_ms, peaks, sm_mhz),
        "e2e": {"value": world * flops_call / (e2e_ms * 1e-3) / 1e12, "unit": UNIT, "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "head_chunk": vsa.default_head_chunk(w.heads, w.head_dim)},
        "gpu_launches": launches,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        dt, fl, desc = oracle_sample(w, args.cpu_every)
        line["cpu_baseline"] = {"value": fl / dt / 1e12, "unit": UNIT, "cores": omp_threads(), "kind": "oracle",
                                "sample": desc, "seconds": dt}
    plan.destroy()
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_ulysses(args, w, world, rank, local):
    """Sequence-parallel forward over `world` ranks (see the module docstring)."""
    import torch
    import torch.distributed as dist
    from torch.multiprocessing.reductions import reduce_tensor

    import block_sparse_tiled_b200 as vsa
    import synth

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    L, H = w.seq_len, w.heads
    ls, hn, h0 = vsa.ulysses_partition(L, H, world, rank)
    # every rank draws the same seeded input and keeps its token part of it
    x = synth.make_inputs(w, seed=0, device=dev)
    mine = {n: x[n][:, rank * ls:(rank + 1) * ls].contiguous() for n in ("q", "k", "v", "gate")}
    mine["out"] = torch.empty_like(mine["q"])
    del x
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    # the other ranks' parts, mapped through CUDA IPC handles exchanged over the process group
    handles = {n: reduce_tensor(t) for n, t in mine.items()}
    every = [None] * world
    dist.all_gather_object(every, handles)
    parts = {n: [] for n in mine}
    for r in range(world):
        for n in mine:
            if r == rank:
                parts[n].append(mine[n])
            else:
                fn, fargs = every[r][n]
                parts[n].append(fn(*fargs))
    plan = vsa.vsa_plan_tiles(batch=w.batch, heads=hn, head_dim=w.head_dim, segments=w.segments, grid=w.grid,
                              sparsity=w.sparsity, tile_size=w.tile, cube=w.cube, ref_segments=w.ref_segments,
                              ref_keep=w.ref_keep)
    dims = plan.dims
    ws = vsa.alloc_workspace(plan, dev)
    stream = torch.cuda.current_stream(dev)
    flops_call = dims["selected_pairs"] * w.batch * H * tile_flops(w.head_dim, w.tile)  # the whole forward

    def step():
        vsa.vsa_forward_parts(plan, parts["q"], parts["k"], parts["v"], parts["gate"], parts["out"], h0,
                              workspace=ws, stream=stream)

    barrier(world)  # every part is written before any rank reads it
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    barrier(world)
    code, where = vsa.device_status(plan)
    if code != 0:
        raise RuntimeError(f"device status {code} at site {where} during warm-up")
    with ClockSampler(local) as clk:
        start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record(stream)
        for _ in range(args.steps):
            step()
        stop.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    ms_step = max_over_ranks(start.elapsed_time(stop) / args.steps, world, dev)
    value = flops_call / (ms_step * 1e-3) / 1e12

    # end to end: every rank copies its token part in from pinned host memory, the ranks meet, run the
    # forward, meet again (every out part complete) and copy their out part back
    hx = {n: torch.empty(mine[n].shape, dtype=mine[n].dtype, pin_memory=True) for n in ("q", "k", "v", "gate")}
    for n in hx:
        hx[n].copy_(mine[n])
    hout = torch.empty(mine["out"].shape, dtype=mine["out"].dtype, pin_memory=True)
    e2e_steps = max(1, min(args.steps, 3))
    torch.cuda.synchronize()
    barrier(world)
    s0 = time.perf_counter()
    for _ in range(e2e_steps):
        for n in hx:
            mine[n].copy_(hx[n], non_blocking=True)
        torch.cuda.synchronize()
        barrier(world)
        step()
        torch.cuda.synchronize()
        barrier(world)
        hout.copy_(mine["out"], non_blocking=True)
        torch.cuda.synchronize()
    e2e_ms = max_over_ranks((time.perf_counter() - s0) * 1e3 / e2e_steps, world, dev)
    h2d = sum(t.numel() * t.element_size() for t in hx.values())
    d2h = hout.numel() * hout.element_size()
    code, where = vsa.device_status(plan)
    if code != 0:
        raise RuntimeError(f"device status {code} at site {where}")
    B, D = w.batch, w.head_dim
    remote = (world - 1) / world
    exchange = {"q_k_v_read_from_peers": int(3 * B * L * hn * D * 2 * remote),
                "gate_read_from_peers": int(B * L * hn * 2 * remote),
                "out_written_to_peers": int(B * L * hn * D * 2 * remote)}
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "strong",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded counter-based normal, structured tile offsets)",
        "config": config_dict(w, dims=None, world=world, mode="ulysses"),
        "mode": "ulysses", "heads_per_rank": hn, "tokens_per_part": ls,
        "exchange_bytes_per_rank": exchange,
        "e2e": {"value": flops_call / (e2e_ms * 1e-3) / 1e12, "unit": UNIT, "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": h2d * world, "d2h_bytes_per_step": d2h * world,
                "timing": "wall clock per step around each rank's copies, barriers and forward; max over ranks"},
        # per rank and step: gather+pool, scores, select+compression, attention (no gate check over parts)
        "gpu_launches": (3 + attn_launches(w, hn)) * args.steps,
        "clocks": clk.summary(),
    }
    # release the peer mappings before any rank frees what they map
    parts = None
    torch.cuda.synchronize()
    barrier(world)
    plan.destroy()
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_ab(args, w, variants):
    """Side measurement (not the contract line): the whole vsa_forward under two plan variants of the
    same workload, alternating them over two rounds; prints one JSON line with the median forward times
    and the workspace sizes.  variants: name -> extra vsa_plan_tiles arguments."""
    import torch
    import synth
    import block_sparse_tiled_b200 as vsa

    torch.cuda.set_device(0)
    x = synth.make_inputs(w, seed=0, device="cuda")
    res = {"workload": w.name, "steps": args.steps, "warmup": args.warmup, "forward_ms": {}, "workspace_bytes": {}}
    for rnd in range(2):
        for key, extra in variants.items():
            plan = vsa.vsa_plan_tiles(batch=w.batch, heads=w.heads, head_dim=w.head_dim, segments=w.segments,
                                      grid=w.grid, sparsity=w.sparsity, tile_size=w.tile, cube=w.cube,
                                      ref_segments=w.ref_segments, ref_keep=w.ref_keep, **extra)
            ws = vsa.alloc_workspace(plan)
            out = torch.empty_like(x["q"])
            for _ in range(args.warmup):
                vsa.vsa_forward(plan, x["q"], x["k"], x["v"], x["gate"], out=out, workspace=ws)
            torch.cuda.synchronize()
            ts = []
            for _ in range(args.steps):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                vsa.vsa_forward(plan, x["q"], x["k"], x["v"], x["gate"], out=out, workspace=ws)
                e1.record()
                torch.cuda.synchronize()
                ts.append(e0.elapsed_time(e1))
            ts.sort()
            res["forward_ms"].setdefault(key, []).append(ts[len(ts) // 2])
            res["workspace_bytes"][key] = ws.numel()
            plan.destroy()
            del ws, out
            torch.cuda.empty_cache()
    print(json.dumps(res))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["vsa", "reference"], default="vsa")
    ap.add_argument("--mode", choices=["auto", "ulysses", "replicas"], default="auto",
                    help="with several ranks: one forward split over them (ulysses, the default) or one whole "
                         "forward per rank (replicas)")
    ap.add_argument("--workload", default="768p_s0.9")
    ap.add_argument("--sparsity", type=float, default=None)
    ap.add_argument("--heads", type=int, default=None,
                    help="override the workload's head count (a head slice of it, e.g. for profiling)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-every", type=int, default=1)
    ap.add_argument("--ref-every", type=int, default=16)
    ap.add_argument("--ab-seq-tiles", action="store_true",
                    help="side measurement: vsa_forward with tile-order copies against a seq_tiles plan")
    ap.add_argument("--ab-qk-fp8", action="store_true",
                    help="side measurement: vsa_forward with bf16 Q/K logits against 8-bit (E4M3) Q/K")
    ap.add_argument("--ab-prefix-fp8", action="store_true",
                    help="side measurement: vsa_forward with bf16 Q/K logits against the prefix split (8-bit Q/K "
                         "for the dense prefix query tiles only)")
    ap.add_argument("--ab-fp4", action="store_true",
                    help="side measurement: vsa_forward with bf16 Q/K logits, the prefix split, and the split with "
                         "FP4 Q and smoothed FP4 K for the video query tiles")
    args = ap.parse_args()
    import synth

    w = synth.workload(args.workload)
    if args.sparsity is not None:
        w = dataclasses.replace(w, sparsity=args.sparsity, name=f"{w.name}@s{args.sparsity}")
    if args.heads is not None:
        w = dataclasses.replace(w, heads=args.heads, name=f"{w.name}@h{args.heads}")
    if args.ab_seq_tiles:
        run_ab(args, w, {"tile_order": {}, "seq_tiles": {"seq_tiles": True}})
        return
    if args.ab_qk_fp8:
        run_ab(args, w, {"qk_bf16": {}, "qk_fp8": {"qk_fp8": True}})
        return
    if args.ab_prefix_fp8:
        run_ab(args, w, {"qk_bf16": {}, "qk_prefix_fp8": {"qk_fp8": "prefix"}})
        return
    if args.ab_fp4:
        run_ab(args, w, {"qk_bf16": {}, "qk_prefix_fp8": {"qk_fp8": "prefix"}, "qk_fp4_video": {"qk_fp8": "fp4"}})
        return
    world, rank, local = dist_setup(args)
    try:
        # auto: one forward split over the ranks (with one rank, the plain forward)
        mode = "ulysses" if args.mode == "auto" else args.mode
        if args.impl == "reference":
            run_reference(args, w, world, rank, mode)
        elif mode == "ulysses" and world > 1:
            run_ulysses(args, w, world, rank, local)
        else:
            run_vsa(args, w, world, rank, local, mode)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
