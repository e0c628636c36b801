"""Benchmark of the fused SS2D forward core on B200.

One step = one ss2d_forward_core call (CrossScan read by index arithmetic,
selective scan, CrossMerge into y) over the VMamba-T stage-1 workload
(B=32, D=192, 56x56, N=16; bf16 x/dts, fp32 B/C/y) with every input already
resident in device memory.  Throughput is scan elements B*4*D*L per second.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun each rank runs the same workload on its own GPU (independent
replicas, weak scaling), timed with CUDA events between barriers; the slowest
rank's time is used.  Rank 0 prints one JSON line.  With --shard the ranks split
the workload's batch instead (strong scaling: no exchange during the step) and
gather y's shards with one all_gather after the timed steps, timed apart.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from selective_scan_02_b200.inputs import (  # noqa: E402
    BLOCK_WORKLOADS, WORKLOADS, Workload, bf16_bits, make_block_inputs, make_inputs)

PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "scan2_kernel_traffic_vmamba_t_stage1.json")
KERNEL_SOURCES = [os.path.join(ROOT, "selective_scan_02_b200", "csrc", f) for f in ("scan2.cuh", "scan.cuh", "scan.cu", "common.cuh")]
FALLBACK_HBM_GBS = 6650.0
FALLBACK_SM_MHZ = 1965.0
SMS = 148
MUFU_PER_CLK_PER_SM = 16  # exp2 / log2 results per clock per SM (CUDA programming guide throughput table)


def load_peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p.get("sm_max_mhz", FALLBACK_SM_MHZ)), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_SM_MHZ, "fallback"


def max_over_ranks(ms: float, device=None) -> float:
    """The slowest rank's time (all_reduce MAX); the value itself on a single process."""
    import torch
    import torch.distributed as dist

    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size() == 1:
        return ms
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def shard_range(B: int, world: int, rank: int):
    """Images [b0, b1) of `rank` when a batch of B images is split over `world` ranks:
    contiguous shards, the first B % world ranks taking one image more."""
    base, extra = divmod(B, world)
    b0 = rank * base + min(rank, extra)
    return b0, b0 + base + (1 if rank < extra else 0)


def gather_shards(y_local, B: int, world: int):
    """All-gather the ranks' batch shards of y (rank r holds images shard_range(B, world, r))
    into the whole (B, ...) tensor on every rank.  Shards are padded to ceil(B / world) images
    for the collective (dist.all_gather over the process group: NCCL between GPUs, gloo in the
    CPU tests) and the padding is dropped again."""
    import torch
    import torch.distributed as dist

    per = -(-B // world)
    rest = tuple(y_local.shape[1:])
    pad = torch.zeros((per,) + rest, dtype=y_local.dtype, device=y_local.device)
    pad[: y_local.shape[0]] = y_local
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad)
    return torch.cat([parts[r][: shard_range(B, world, r)[1] - shard_range(B, world, r)[0]] for r in range(world)])


def weak_scaling_value(elements_per_rank: int, world: int, ms_per_step: float) -> float:
    """Whole-job throughput in Gelem/s: every rank processes its own replica of the workload."""
    return world * elements_per_rank / (ms_per_step * 1e-3) / 1e9


def kernel_source_hash() -> str:
    """Hash of the scan kernel's sources: recorded ncu traffic is reported only while it matches."""
    import hashlib
    hsh = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(f, "rb") as fh:
            hsh.update(fh.read())
    return hsh.hexdigest()[:16]


def recorded_traffic(wl):
    """DRAM bytes per launch of the fused scan kernel from a committed ncu capture, or None when the
    capture is missing, was taken on another workload, or predates the current kernel sources."""
    try:
        with open(TRAFFIC_FILE) as f:
            rec = json.load(f)
    except Exception:
        return None
    if rec.get("kernel_hash") != kernel_source_hash() or rec.get("workload") != wl.name:
        return None
    return float(rec["bytes_per_launch_full_size"])


def pipelined_e2e(hosts, run, outs_host, k_steps, barrier):
    """End-to-end ms per step through the public API with host buffers.

    Every step copies its inputs from pinned host memory to the device, makes the library call
    and copies its outputs back to pinned host memory.  Consecutive steps overlap on three
    streams: the upload of step k+1, the call of step k and the download of step k-1 (the
    two directions of the host link run at the same time).  Inputs and outputs are double
    buffered on the device; events order every reuse.  run(dev_inputs, slot, stream) makes
    the call and returns its device outputs, keyed like outs_host[slot].
    """
    import torch

    s_up, s_run, s_down = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    dev = [{k: torch.empty(v.shape, dtype=v.dtype, device="cuda") for k, v in hosts.items()} for _ in range(2)]
    up_done = [torch.cuda.Event() for _ in range(2)]
    run_done = [torch.cuda.Event() for _ in range(2)]
    down_done = [torch.cuda.Event() for _ in range(2)]

    def step(k):
        sl = k % 2
        with torch.cuda.stream(s_up):
            s_up.wait_event(run_done[sl])      # step k-2 has consumed this slot's inputs
            for key, h in hosts.items():
                dev[sl][key].copy_(h, non_blocking=True)
            up_done[sl].record(s_up)
        with torch.cuda.stream(s_run):
            s_run.wait_event(up_done[sl])
            s_run.wait_event(down_done[sl])    # step k-2's outputs of this slot are downloaded
            outs = run(dev[sl], sl, s_run)
            run_done[sl].record(s_run)
        with torch.cuda.stream(s_down):
            s_down.wait_event(run_done[sl])
            for key, t in outs.items():
                outs_host[sl][key].copy_(t, non_blocking=True)
            down_done[sl].record(s_down)

    for k in range(2):
        step(k)
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_up)
    for k in range(k_steps):
        step(k)
    e1.record(s_down)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / k_steps


def planned_segments(wl) -> int:
    """Segments the library plans for a whole-sequence scan of this workload's shape (one wave
    of sixteen-channel items: 12 one-warp CTAs per SM for bf16 u/dt, 11 for the projection
    form and 10 for fp32 u/dt, whose shared-memory layouts are larger; segments of whole
    32-step chunks, at least four chunks each), mirrored here to count the launches."""
    items = wl.B * 4 * ((wl.D + 15) // 16)
    target = 148 * (11 if wl.R > 0 else (12 if wl.x_dtype == "bf16" else 10))
    if wl.N != 16 or items >= target or wl.L < 8 * 32:
        return 1
    ns = min(target // items, wl.L // (4 * 32))
    if ns < 2:
        return 1
    seg = -(-wl.L // ns)
    seg = -(-seg // 32) * 32
    return -(-wl.L // seg)


def launches_per_step(wl, ws_bytes: int) -> int:
    """Kernels one core call launches: the zero-fill of y and the scan; the plane transpose of
    x when the workspace holds that copy (for bf16 x with even H and W the transpose also
    zeroes y, so there is no separate zero-fill); for a segmented scan its first pass and
    carry.  Projection form: the zero-fill of the GEMM's error word, the x_proj GEMM, the plane
    transpose of x (which zeroes y for even H and W; else y has its own zero-fill) and the scan;
    dt_ranks above 16 instead materialise dt_proj's output (no transpose) before the scan."""
    esize = 2 if wl.x_dtype == "bf16" else 4
    segmented = planned_segments(wl) > 1
    if wl.R > 0:
        if wl.R > 16:
            return 5
        transposed = wl.N == 16 and (wl.L * 2) % 16 == 0
        fused_zero = transposed and wl.H % 2 == 0 and wl.W % 2 == 0
        return 3 + (1 if transposed else 0) + (0 if fused_zero else 1) + (2 if segmented else 0)
    seg_bytes = 3 * wl.B * 4 * wl.D * planned_segments(wl) * 16 * 4 if segmented else 0
    transposed = ws_bytes - seg_bytes == wl.B * wl.D * wl.H * wl.W * esize
    fused_zero = transposed and wl.x_dtype == "bf16" and wl.H % 2 == 0 and wl.W % 2 == 0
    return 2 + (1 if transposed and not fused_zero else 0) + (2 if segmented else 0)


def time_standalone_scan(ss, wl, t, stream, args, barrier, hbm_peak):
    """The selective scan alone (ss2d_selective_scan) on the cross-scanned input materialised
    once, outside the timed region: u = CrossScan(x) and dts as (B, 4D, L), B and C as
    (B, 4, N, L), y (B, 4D, L) fp32.  Its algorithmic bytes are u, delta, B, C read and y
    written once."""
    import torch

    B, D, L, N = wl.B, wl.D, wl.L, wl.N
    xs = ss.cross_scan(t["x"], stream=stream).view(B, 4 * D, L)
    dts = t["dts"].view(B, 4 * D, L)
    ys = torch.empty((B, 4 * D, L), dtype=torch.float32, device="cuda")

    def sstep():
        ss.selective_scan(xs, dts, t["A_logs"], t["Bs"], t["Cs"], t["Ds"], t["dt_bias"], True, y=ys, stream=stream)

    for _ in range(args.warmup):
        sstep()
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        sstep()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms = max_over_ranks(e0.elapsed_time(e1), device="cuda") / args.steps
    esz = xs.element_size()
    nbytes = B * 4 * D * L * (esz + dts.element_size() + 4) + 2 * B * 4 * N * L * 4
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"ms_per_call": ms, "value": wl.elements / (ms * 1e-3) / 1e9, "unit": "Gelem/s",
            "hbm": {"achieved": gbs, "peak": hbm_peak, "unit": "GB/s", "frac": gbs / hbm_peak,
                    "algorithmic_bytes_per_call": nbytes},
            "note": "ss2d_selective_scan on materialised CrossScan(x), dts, B, C; y (B,4D,L) fp32"}


def algorithmic_bytes(wl) -> int:
    """Bytes the fused core must move at least once: x, dts, Bs, Cs read, y written (params negligible).
    Projection form, as designed (x_proj's output kept in HBM between its GEMM and the scan): x read
    twice, x_dbl (B, 4, R+2N, L) fp32 written and read once, y written."""
    xb = 2 if wl.x_dtype == "bf16" else 4
    db = 2 if wl.dt_dtype == "bf16" else 4
    L = wl.L
    if wl.R > 0:
        return 2 * wl.B * wl.D * L * xb + 2 * wl.B * 4 * (wl.R + 2 * wl.N) * L * 4 + wl.B * wl.D * L * 4
    return (wl.B * wl.D * L * xb + wl.B * 4 * wl.D * L * db + 2 * wl.B * 4 * wl.N * L * 4
            + wl.B * wl.D * L * 4 + 4 * wl.D * (wl.N + 2) * 4)


class ClockSampler:
    """nvidia-smi clock / throttle-reason sampling during the timed region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
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
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        out = {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        if self.proc is None:
            return out
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9 and parts[1].isdigit():
                    rows.append(parts)
        os.remove(self.path)
        if not rows:
            return out
        out["samples"] = len(rows)
        out["sm_mhz"] = statistics.median(float(r[1]) for r in rows)
        out["sm_max_mhz"] = max(float(r[2]) for r in rows)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        seen = set()
        for r in rows:
            for name, v in zip(names, r[5:9]):
                if v.lower().startswith("active"):
                    seen.add(name)
        out["reasons"] = sorted(seen)
        return out


def cpu_baseline(wl, seconds_target: float = 6.0):
    """Time the CPU oracle on bounded samples of the workload (the first nb batch elements with
    all of their channels, nb chosen from a one-element trial so each sample takes about
    seconds_target, never more than the whole batch):
      - the fp32 instantiation of the C oracle on one host thread;
      - the same on every host thread, the sample's batch elements split across threads (the
        C call releases the interpreter lock);
      - the fp64 instantiation (the parity oracle) on one host thread.
    The line's value is the all-threads fp32 figure; cores is the number of threads it used."""
    import concurrent.futures

    from oracle import oracle as orc

    inp = make_inputs(wl)

    def args_for(b0, b1):
        a = dict(x=inp["x"][b0:b1], A_logs=inp["A_logs"], Ds=inp["Ds"], dt_bias=inp["dt_bias"])
        if wl.R > 0:
            a.update(x_proj_weight=inp["x_proj_weight"], dt_projs_weight=inp["dt_projs_weight"])
        else:
            a.update(dts=inp["dts"][b0:b1], Bs=inp["Bs"][b0:b1], Cs=inp["Cs"][b0:b1])
        return a

    def run64(nb):
        t0 = time.perf_counter()
        orc.forward_core(**args_for(0, nb))
        return time.perf_counter() - t0

    def run32(b0, b1):
        a = args_for(b0, b1)
        orc.forward_core_f32(a["x"], a["A_logs"], a["Ds"], a["dt_bias"], a["dts"], a["Bs"], a["Cs"])

    def timed32(nb, threads):
        bounds = [(i * nb // threads, (i + 1) * nb // threads) for i in range(threads)]
        bounds = [bd for bd in bounds if bd[1] > bd[0]]
        t0 = time.perf_counter()
        if len(bounds) == 1:
            run32(*bounds[0])
        else:
            with concurrent.futures.ThreadPoolExecutor(len(bounds)) as ex:
                list(ex.map(lambda bd: run32(*bd), bounds))
        return time.perf_counter() - t0, len(bounds)

    orc.build()
    per_img = wl.elements // wl.B
    out = {"kind": "oracle", "unit": "Gelem/s"}
    t1 = run64(1)
    nb64 = int(max(1, min(wl.B, seconds_target / max(t1, 1e-6))))
    dt64 = run64(nb64) if nb64 > 1 else t1
    fp64 = {"value": nb64 * per_img / dt64 / 1e9, "threads": 1,
            "sample": f"batch elements 0..{nb64 - 1}, {dt64:.1f} s"}
    if wl.R > 0:  # the fp32 instantiation is timed for the dts/Bs/Cs form only
        out.update(value=fp64["value"], cores=1,
                   sample=f"batch elements 0..{nb64 - 1} with all channels ({nb64 * per_img} of {wl.elements} "
                          f"scan elements), fp64 sequential C oracle on one host thread, {dt64:.1f} s",
                   fp64_1thread=fp64)
        return out
    t1, _ = timed32(1, 1)
    nb32 = int(max(1, min(wl.B, seconds_target / max(t1, 1e-6))))
    dt32, _ = timed32(nb32, 1) if nb32 > 1 else (t1, 1)
    fp32_1 = {"value": nb32 * per_img / dt32 / 1e9, "threads": 1,
              "sample": f"batch elements 0..{nb32 - 1}, {dt32:.1f} s"}
    threads = os.cpu_count() or 1
    nbt = int(max(1, min(wl.B, nb32 * threads)))
    dtt, used = timed32(nbt, min(threads, nbt))
    out.update(value=nbt * per_img / dtt / 1e9, cores=used,
               sample=f"batch elements 0..{nbt - 1} with all channels ({nbt * per_img} of {wl.elements} scan "
                      f"elements), fp32 instantiation of the sequential C oracle, the batch split over {used} host "
                      f"threads ({os.cpu_count()} reported by the host), {dtt:.2f} s",
               fp32_1thread=fp32_1, fp64_1thread=fp64)
    return out


def other_workloads(ss, stream, hbm_peak, steps=20, warmup=3):
    """Device-timed fused core (and, for stage 1, its backward) on the other synthetic workloads,
    recorded beside the headline: each at its full size, inputs resident in HBM, CUDA events on
    the launching stream around each of `steps` calls after `warmup`, median of the call times.
    Before every timed call a 256 MB buffer (twice the L2) is written on the same stream, outside
    the events, so that no call finds its inputs in L2 (stage3_short's 71 MB would fit)."""
    import torch

    out = {}
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")

    def to_dev(a, dtype):
        if dtype == "bf16":
            return torch.from_numpy(bf16_bits(a).view(np.int16)).view(torch.bfloat16).cuda()
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()

    def timed(fn):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(steps):
            with torch.cuda.stream(stream):
                flush.fill_(1)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        return float(np.median(ts))

    for name in ("stage3_short", "hires_long", "proj"):
        wl = WORKLOADS[name]
        inp = make_inputs(wl)
        t = dict(x=to_dev(inp["x"], wl.x_dtype), A_logs=to_dev(inp["A_logs"], "f32"), Ds=to_dev(inp["Ds"], "f32"),
                 dt_bias=to_dev(inp["dt_bias"], "f32"))
        if wl.R > 0:
            t.update(x_proj_weight=to_dev(inp["x_proj_weight"], "bf16"),
                     dt_projs_weight=to_dev(inp["dt_projs_weight"], "f32"))
        else:
            t.update(dts=to_dev(inp["dts"], wl.dt_dtype), Bs=to_dev(inp["Bs"], "f32"), Cs=to_dev(inp["Cs"], "f32"))
        y = torch.empty((wl.B, wl.D, wl.H, wl.W), dtype=torch.float32, device="cuda")
        ws = torch.empty(max(ss.forward_core_workspace_size(**t), 1), dtype=torch.uint8, device="cuda")
        ms = timed(lambda: ss.forward_core(**t, y=y, workspace=ws, stream=stream))
        nbytes = algorithmic_bytes(wl)
        gbs = nbytes / (ms * 1e-3) / 1e9
        out[name] = {"ms_per_call": ms, "value": wl.elements / (ms * 1e-3) / 1e9, "unit": "Gelem/s",
                     "hbm": {"achieved": gbs, "frac": gbs / hbm_peak, "algorithmic_bytes_per_call": nbytes},
                     "config": {"B": wl.B, "D": wl.D, "H": wl.H, "W": wl.W, "N": wl.N, "R": wl.R,
                                "x_dtype": wl.x_dtype, "dts_dtype": wl.dt_dtype}}
        del t, y, ws
        torch.cuda.empty_cache()
    # the stage-1 core with the page-order merge (deterministic), and its backward
    # (ss2d_forward_core_backward with its own checkpoint pass)
    wl = WORKLOADS["vmamba_t_stage1"]
    inp = make_inputs(wl)
    t = dict(x=to_dev(inp["x"], "bf16"), A_logs=to_dev(inp["A_logs"], "f32"), Ds=to_dev(inp["Ds"], "f32"),
             dt_bias=to_dev(inp["dt_bias"], "f32"), dts=to_dev(inp["dts"], "bf16"), Bs=to_dev(inp["Bs"], "f32"),
             Cs=to_dev(inp["Cs"], "f32"))
    y = torch.empty((wl.B, wl.D, wl.H, wl.W), dtype=torch.float32, device="cuda")
    ws = torch.empty(max(ss.forward_core_workspace_size(**t, page_order=True), 1), dtype=torch.uint8, device="cuda")
    ms = timed(lambda: ss.forward_core(**t, y=y, workspace=ws, stream=stream, page_order=True))
    out["vmamba_t_stage1_page_order"] = {"ms_per_call": ms, "value": wl.elements / (ms * 1e-3) / 1e9,
                                         "unit": "Gelem/s",
                                         "note": "SS2D_MERGE_PAGE_ORDER: every direction stores its outputs once, "
                                                 "then one CrossMerge pass adds them in the article's order; "
                                                 "y bit-identical across runs"}
    del y, ws
    dy = torch.from_numpy(np.random.default_rng(wl.seed + 1).standard_normal(
        (wl.B, wl.D, wl.H, wl.W)).astype(np.float32)).cuda()
    grads = ss.forward_core_backward(**t, dy=dy, stream=stream)
    bws = torch.empty(ss.forward_core_backward_workspace_size(**t), dtype=torch.uint8, device="cuda")
    ms = timed(lambda: ss.forward_core_backward(**t, dy=dy, grads=grads, workspace=bws, stream=stream))
    out["vmamba_t_stage1_backward"] = {"ms_per_call": ms, "value": wl.elements / (ms * 1e-3) / 1e9,
                                       "unit": "Gelem/s", "note": "ss2d_forward_core_backward, all gradients"}
    del t, dy, grads, bws
    torch.cuda.empty_cache()
    # the whole SS2D block at stage 1 (input projection, convolution, core, gated norm, output projection)
    bwl = BLOCK_WORKLOADS["block_stage1"]
    binp = make_block_inputs(bwl)
    bt = {k: to_dev(v, "bf16" if k in ("x", "in_proj_weight", "x_proj_weight", "out_proj_weight") else "f32")
          for k, v in binp.items()}
    args = (bt["x"], bt["in_proj_weight"], bt["conv_weight"], bt["conv_bias"], bt["x_proj_weight"],
            bt["dt_projs_weight"], bt["dt_projs_bias"], bt["A_logs"], bt["Ds"], bt["out_norm_weight"],
            bt["out_norm_bias"], bt["out_proj_weight"])
    bout = torch.empty((bwl.B, bwl.H, bwl.W, bwl.d_model), dtype=torch.float32, device="cuda")
    bws = torch.empty(ss.block_forward_workspace_size(*args), dtype=torch.uint8, device="cuda")
    ms = timed(lambda: ss.block_forward(*args, out=bout, workspace=bws, stream=stream))
    nbytes = block_algorithmic_bytes(bwl)
    gbs = nbytes / (ms * 1e-3) / 1e9
    out["block_stage1"] = {"ms_per_call": ms, "value": bwl.elements / (ms * 1e-3) / 1e9, "unit": "Gelem/s",
                           "img_per_s": bwl.B / (ms * 1e-3),
                           "hbm": {"achieved": gbs, "frac": gbs / hbm_peak, "algorithmic_bytes_per_call": nbytes},
                           "config": {"B": bwl.B, "H": bwl.H, "W": bwl.W, "d_model": bwl.d_model, "D": bwl.D,
                                      "N": bwl.N, "R": bwl.R, "d_conv": bwl.d_conv},
                           "note": "ss2d_block_forward; value counts the core's scan elements B*4*D*L"}
    return out


def block_algorithmic_bytes(bwl) -> int:
    """Bytes the block moves at least once with its intermediates in HBM: the input projection
    reads x and writes xz (bf16), the convolution reads x_in and writes x_c (bf16), the core in
    its projection form (algorithmic_bytes of the same shape), the normalisation reads y (fp32)
    and z and writes g (bf16), the output projection reads g and writes out (fp32)."""
    M, D, dm = bwl.B * bwl.L, bwl.D, bwl.d_model
    core = algorithmic_bytes(Workload("block_core", bwl.B, D, bwl.H, bwl.W, bwl.N, bwl.R, "bf16", "bf16", 0))
    return (M * dm * 2 + M * 2 * D * 2) + (M * D * 2 + M * D * 2) + core + (M * D * 4 + M * D * 2 + M * D * 2) \
        + (M * D * 2 + M * dm * 4)


def reference_channels(wl):
    """Channels per direction in one step of the reference arm's sample (dts/Bs/Cs form): about
    3e5 scan elements, so a step takes tens of milliseconds and the per-call costs that do not
    grow with the channel count (B and C rows shared by a direction's channels) stay small."""
    return min(wl.D, max(2, 300_000 // (4 * wl.L)))


def run_reference(args):
    """The CPU oracle as the reference arm (rank 0 only)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    wl = WORKLOADS[args.workload]
    from oracle import oracle as orc

    orc.build()
    inp = make_inputs(wl)
    if wl.R > 0:
        # x_proj mixes every channel: one whole image per step
        sample = dict(x=inp["x"][:1], A_logs=inp["A_logs"], Ds=inp["Ds"], dt_bias=inp["dt_bias"],
                      x_proj_weight=inp["x_proj_weight"], dt_projs_weight=inp["dt_projs_weight"])
        elems = 4 * wl.D * wl.L
        what = "batch 0, all channels"
    else:
        ds = reference_channels(wl)
        chans = [k * wl.D + d for k in range(4) for d in range(ds)]
        sample = dict(x=inp["x"][:1, :ds], A_logs=inp["A_logs"][chans], Ds=inp["Ds"][chans],
                      dt_bias=inp["dt_bias"][chans], dts=inp["dts"][:1, :, :ds], Bs=inp["Bs"][:1], Cs=inp["Cs"][:1])
        elems = 4 * ds * wl.L
        what = f"batch 0, channels 0..{ds - 1} of every direction"
    for _ in range(args.warmup):
        orc.forward_core(**sample)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        orc.forward_core(**sample)
        times.append(time.perf_counter() - t0)
    total = sum(times)
    value = elems * args.steps / total / 1e9
    desc = f"{what} per step ({elems} scan elements), fp64 C oracle"
    line = {
        "impl": "reference", "metric": "SS2D core Gelem/s (B*4*D*L)", "value": value, "unit": "Gelem/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "description": wl.description, "sample": desc},
        "cpu_baseline": {"value": value, "unit": "Gelem/s", "cores": 1, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": "Gelem/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# MUFU operations per scan element of the forward: N decays and the exp2 of softplus (its
# log1p is a polynomial on the FMA pipe).
FWD_MUFU_EXTRA = 1
# MUFU operations per scan element of the backward: the checkpoint pass (16 decays, softplus's
# exp2), the rescan of each chunk (16 decays, softplus's exp2, the reciprocal of its sigmoid)
# and the reverse pass (16 decays recomputed per 4-step block).
BWD_MUFU_PER_ELEMENT = 17 + 18 + 16


def bwd_algorithmic_bytes(wl) -> int:
    """Bytes the backward must move at least once: x, dts, Bs, Cs, dy read; dx, ddts, dBs, dCs written.
    In the projection form dts, Bs and Cs are intermediates: x and dy read, dx written (the
    weights and their gradients are a few hundred KB)."""
    xb = 2 if wl.x_dtype == "bf16" else 4
    db = 2 if wl.dt_dtype == "bf16" else 4
    L, BD = wl.L, wl.B * wl.D
    if wl.R > 0:
        return BD * L * xb + BD * L * 4 + BD * L * 4
    return (BD * L * xb + 4 * BD * L * db + 2 * wl.B * 4 * wl.N * L * 4 + BD * L * 4
            + BD * L * 4 + 4 * BD * L * 4 + 2 * wl.B * 4 * wl.N * L * 4)


def bench_backward(args, wl, inp, t, world, rank, local, stream, barrier, train=False):
    """Times ss2d_forward_core_backward on the workload (dy resident in HBM) and prints its line.
    train: a step is the forward and then the backward, the forward keeping the checkpoints the
    backward reads (dts/Bs/Cs form; the projection form recomputes them)."""
    import torch

    import selective_scan_02_b200 as ss

    dy = torch.from_numpy(np.random.default_rng(wl.seed + 1).standard_normal(
        (wl.B, wl.D, wl.H, wl.W)).astype(np.float32)).cuda()
    grads = None
    if wl.R > 0:
        # projection form: the weight gradients, without copies of the intermediates' gradients
        f32 = dict(dtype=torch.float32, device="cuda")
        grads = dict(dx=torch.empty((wl.B, wl.D, wl.H, wl.W), **f32), dA_logs=torch.empty((4 * wl.D, wl.N), **f32),
                     dDs=torch.empty(4 * wl.D, **f32), ddt_bias=torch.empty(4 * wl.D, **f32),
                     dx_proj_weight=torch.empty((4, wl.R + 2 * wl.N, wl.D), **f32),
                     ddt_projs_weight=torch.empty((4, wl.D, wl.R), **f32))
    grads = ss.forward_core_backward(**t, dy=dy, grads=grads, stream=stream)
    ws = torch.empty(ss.forward_core_backward_workspace_size(**t), dtype=torch.uint8, device="cuda")
    keep = train and wl.R == 0
    ck = torch.empty(ss.checkpoint_shape(t["x"]), dtype=torch.float32, device="cuda") if keep else None
    y = torch.empty((wl.B, wl.D, wl.H, wl.W), dtype=torch.float32, device="cuda")
    fws = torch.empty(max(ss.forward_core_workspace_size(**t), 1), dtype=torch.uint8, device="cuda")

    def step():
        if train:
            ss.forward_core(**t, y=y, workspace=fws, stream=stream, ckpt=ck)
        ss.forward_core_backward(**t, dy=dy, grads=grads, workspace=ws, stream=stream, ckpt=ck)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    barrier()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(args.steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize()
    barrier()
    clocks = sampler.stop()
    ms_per_step = max_over_ranks(ev0.elapsed_time(ev1), device="cuda") / args.steps
    value = weak_scaling_value(wl.elements, world, ms_per_step)

    e2e = None
    if not args.no_e2e:
        hosts = {k: v.cpu().pin_memory() for k, v in t.items()}
        hosts["dy"] = dy.cpu().pin_memory()
        slot_grads = [grads, {k: torch.empty_like(v) if v is not None else None for k, v in grads.items()}]
        slot_y = [y, torch.empty_like(y)]
        slot_ck = [ck, torch.empty_like(ck) if ck is not None else None]
        outs = {k: v for k, v in grads.items() if v is not None}
        if train:
            outs["y"] = y
        outs_host = [{k: torch.empty(v.shape, dtype=v.dtype).pin_memory() for k, v in outs.items()} for _ in range(2)]
        h2d = sum(v.numel() * v.element_size() for v in hosts.values())
        d2h = sum(v.numel() * v.element_size() for v in outs_host[0].values())

        def run(dv, sl, st):
            res = {}
            if train:
                fw = {k: v for k, v in dv.items() if k != "dy"}
                res["y"] = ss.forward_core(**fw, y=slot_y[sl], workspace=fws, stream=st, ckpt=slot_ck[sl])
            g = ss.forward_core_backward(**dv, grads=slot_grads[sl], workspace=ws, stream=st, ckpt=slot_ck[sl])
            res.update({k: v for k, v in g.items() if v is not None})
            return res

        ms_e2e = pipelined_e2e(hosts, run, outs_host, max(3, min(args.steps, 10)), barrier)
        ems = max_over_ranks(ms_e2e, device="cuda")
        e2e = {"value": weak_scaling_value(wl.elements, world, ems), "unit": "Gelem/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "pipelined": "upload k+1 / call k / download k-1 on three streams"}

    hbm_peak, sm_max_mhz, peak_kind = load_peaks()
    bytes_step = bwd_algorithmic_bytes(wl) + (algorithmic_bytes(wl) if train else 0)
    # kept checkpoints: the forward's 17 MUFU ops per element replace the checkpoint pass's 17
    mufu_per_element = ((wl.N + FWD_MUFU_EXTRA + BWD_MUFU_PER_ELEMENT - (17 if keep else 0)) if train
                        else BWD_MUFU_PER_ELEMENT)
    mufu_achieved = wl.elements * mufu_per_element / (ms_per_step * 1e-3) / 1e9
    mufu_peak = MUFU_PER_CLK_PER_SM * SMS * sm_max_mhz * 1e6 / 1e9
    bf16 = wl.x_dtype == "bf16"
    fused_dt_adj = wl.D <= 256 and wl.R <= 16 and wl.L % 4 == 0
    proj_own_ckpt = (wl.L * 2) % 16 == 0 and planned_segments(wl) == 1
    bwd_launches = ((6 + 1 + 2 + 1 + 1 + 3 + 1 + (4 if fused_dt_adj else 5) + (1 if proj_own_ckpt else 0))
                    if wl.R > 0
                    else (6 + (2 if bf16 else 0) + 2 + (0 if keep else 1) + 1
                          + (1 if bf16 and not keep and (wl.L * 2) % 16 == 0 else 0)))
    if planned_segments(wl) > 1:
        # the adjoint's first pass and carry, and (unless kept) the checkpoint pass's first
        # pass and carry
        bwd_launches += 2 + (0 if keep else 2)
    fwd_launches = launches_per_step(wl, ss.forward_core_workspace_size(**t)) if train else 0
    metric = "SS2D core training step Gelem/s (B*4*D*L)" if train else "SS2D core backward Gelem/s (B*4*D*L)"
    note = (f"{mufu_per_element} MUFU ops per element (forward, then backward "
            f"{'reading the forward' + chr(39) + 's checkpoints' if keep else 'with its own checkpoint pass'}); "
            "duration = whole step") if train else (
            f"{BWD_MUFU_PER_ELEMENT} MUFU ops per element (checkpoint pass + chunk rescan + reverse pass); "
            "duration = whole backward call")
    line = {
        "metric": metric, "value": value, "unit": "Gelem/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": wl.name, "B": wl.B, "D": wl.D, "H": wl.H, "W": wl.W, "N": wl.N,
                   "x_dtype": wl.x_dtype, "dts_dtype": wl.dt_dtype, "R": wl.R,
                   "pass": "train" if train else "backward", "checkpoints_kept": keep,
                   "l2": "no flush: inputs and gradients exceed the 126 MB L2", "parallelism": f"replicas x{world}"},
        "roofline": {"bound": "alu", "achieved": mufu_achieved, "peak": mufu_peak, "unit": "Gop/s (MUFU ex2/rcp)",
                     "frac": mufu_achieved / mufu_peak, "traffic": None, "note": note},
        "hbm": {"achieved": bytes_step / (ms_per_step * 1e-3) / 1e9, "peak": hbm_peak, "unit": "GB/s",
                "frac": bytes_step / (ms_per_step * 1e-3) / 1e9 / hbm_peak, "algorithmic_bytes_per_step": bytes_step,
                "peak_source": peak_kind},
        "kernel_hash": kernel_source_hash(),
        "clocks": {"sm_mhz": clocks["sm_mhz"], "sm_max_mhz": clocks["sm_max_mhz"], "reasons": clocks["reasons"]},
        # backward: zero-fills of dx, dA_logs, dBs, dCs, dDs, ddt_bias; the checkpoint pass
        # (unless kept by the forward), which reads bf16 x and dts as they are plus a bf16
        # plane-transposed copy of x; two bf16 widenings; two plane transposes; the backward
        # scan; segmented, the first passes and carries.  Projection form: x widened once, plus
        # zero-fills of the dt_proj weight gradient and of the GEMM's error word, the x_proj
        # GEMM, dt_proj's expansion, the checkpoint pass's bf16 plane transpose of x (its pass
        # reads bf16 x and the fp32 dts) and four projection-gradient kernels (five where
        # dt_proj's adjoints run as two kernels).  train adds the forward's launches.
        "gpu_launches": (bwd_launches + fwd_launches) * args.steps,
        "e2e": e2e,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_backward(wl, train=train)
    if rank == 0:
        print(json.dumps(line), flush=True)


def cpu_baseline_backward(wl, seconds_target: float = 12.0, train=False):
    """The oracle's gradient (train: forward, then gradient) on a bounded sample: the first nb
    batch elements, all channels."""
    from oracle import oracle as orc

    inp = make_inputs(wl)
    dy = np.random.default_rng(wl.seed + 1).standard_normal((wl.B, wl.D, wl.H, wl.W)).astype(np.float32)

    def run(nb):
        t0 = time.perf_counter()
        if train:
            fw = dict(x=inp["x"][:nb], A_logs=inp["A_logs"], Ds=inp["Ds"], dt_bias=inp["dt_bias"])
            if wl.R > 0:
                fw.update(x_proj_weight=inp["x_proj_weight"], dt_projs_weight=inp["dt_projs_weight"])
            else:
                fw.update(dts=inp["dts"][:nb], Bs=inp["Bs"][:nb], Cs=inp["Cs"][:nb])
            orc.forward_core(**fw)
        if wl.R > 0:
            orc.forward_core_proj_bwd(inp["x"][:nb], inp["x_proj_weight"], inp["dt_projs_weight"], inp["A_logs"],
                                      inp["Ds"], inp["dt_bias"], dy[:nb])
        else:
            orc.forward_core_bwd(inp["x"][:nb], inp["A_logs"], inp["Ds"], inp["dt_bias"], inp["dts"][:nb],
                                 inp["Bs"][:nb], inp["Cs"][:nb], dy[:nb])
        return time.perf_counter() - t0

    orc.build()
    t1 = run(1)
    nb = int(max(1, min(wl.B, seconds_target / max(t1, 1e-6))))
    dt = run(nb) if nb > 1 else t1
    elems = nb * 4 * wl.D * wl.L
    return {"value": elems / dt / 1e9, "unit": "Gelem/s", "cores": 1, "kind": "oracle",
            "sample": f"{'forward and ' if train else ''}gradient of batch elements 0..{nb - 1} with all channels "
                      f"({elems} of {wl.elements} scan elements), fp64 sequential C oracle on one host core, "
                      f"{dt:.1f} s"}


def run_reference_backward(args, train=False):
    """The oracle's gradient (train: forward, then gradient) as the reference arm of --pass
    backward / train (rank 0 only)."""
    if int(os.environ.get("RANK", "0")) != 0:
        return
    wl = WORKLOADS[args.workload]
    from oracle import oracle as orc

    orc.build()
    inp = make_inputs(wl)
    if wl.R > 0:
        # x_proj mixes every channel: one whole image per step
        dy = np.random.default_rng(wl.seed + 1).standard_normal((1, wl.D, wl.H, wl.W)).astype(np.float32)
        sample = (inp["x"][:1], inp["x_proj_weight"], inp["dt_projs_weight"], inp["A_logs"], inp["Ds"],
                  inp["dt_bias"], dy)
        fn = orc.forward_core_proj_bwd
        fwd = dict(x=sample[0], x_proj_weight=sample[1], dt_projs_weight=sample[2], A_logs=sample[3],
                   Ds=sample[4], dt_bias=sample[5])
        elems = 4 * wl.D * wl.L
        what = "batch 0, all channels"
    else:
        ds = reference_channels(wl)
        chans = [k * wl.D + d for k in range(4) for d in range(ds)]
        dy = np.random.default_rng(wl.seed + 1).standard_normal((1, ds, wl.H, wl.W)).astype(np.float32)
        sample = (inp["x"][:1, :ds], inp["A_logs"][chans], inp["Ds"][chans], inp["dt_bias"][chans],
                  inp["dts"][:1, :, :ds], inp["Bs"][:1], inp["Cs"][:1], dy)
        fn = orc.forward_core_bwd
        fwd = dict(x=sample[0], A_logs=sample[1], Ds=sample[2], dt_bias=sample[3], dts=sample[4], Bs=sample[5],
                   Cs=sample[6])
        elems = 4 * ds * wl.L
        what = f"batch 0, channels 0..{ds - 1} of every direction"

    def one():
        if train:
            orc.forward_core(**fwd)
        fn(*sample)

    for _ in range(args.warmup):
        one()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        one()
    total = time.perf_counter() - t0
    value = elems * args.steps / total / 1e9
    desc = f"{'forward and ' if train else ''}gradient of {what} per step ({elems} scan elements), fp64 C oracle"
    metric = "SS2D core training step Gelem/s (B*4*D*L)" if train else "SS2D core backward Gelem/s (B*4*D*L)"
    print(json.dumps({
        "impl": "reference", "metric": metric, "value": value, "unit": "Gelem/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "pass": "train" if train else "backward", "sample": desc},
        "cpu_baseline": {"value": value, "unit": "Gelem/s", "cores": 1, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": "Gelem/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="vmamba_t_stage1", choices=sorted(WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-other-workloads", action="store_true",
                    help="skip the device-timed stage-3, 256x256, projection and backward results")
    ap.add_argument("--batch", type=int, default=0,
                    help="override the workload's batch size (smaller cases for profiling)")
    ap.add_argument("--shard", action="store_true",
                    help="under torchrun, split the workload's batch over the ranks (strong scaling: each rank "
                         "runs its shard_range images) and all-gather y after the timed steps; by default every "
                         "rank runs the whole workload (weak scaling)")
    ap.add_argument("--pass", dest="which", default="forward", choices=["forward", "backward", "train"],
                    help="time the fused core (default), its backward (ss2d_forward_core_backward), or a "
                         "training step (forward keeping the checkpoints, then backward)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    if args.impl == "reference":
        if args.which in ("backward", "train"):
            run_reference_backward(args, train=args.which == "train")
        else:
            run_reference(args)
        return

    import torch
    import torch.distributed as dist

    import selective_scan_02_b200 as ss

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))

    def barrier():
        if world > 1:
            dist.barrier()

    wl = WORKLOADS[args.workload]
    if args.batch > 0:
        import dataclasses
        wl = dataclasses.replace(wl, B=args.batch)
    inp = make_inputs(wl)
    # batch shards (strong scaling) or whole replicas (weak scaling) per rank
    sharded = args.shard and world > 1 and args.which == "forward"
    wl_run = wl
    if sharded:
        import dataclasses
        if wl.B < world:
            raise SystemExit(f"--shard: {wl.B} images cannot be split over {world} ranks")
        b0, b1 = shard_range(wl.B, world, rank)
        inp = {k: (np.ascontiguousarray(v[b0:b1]) if k in ("x", "dts", "Bs", "Cs") else v) for k, v in inp.items()}
        wl_run = dataclasses.replace(wl, B=b1 - b0)
    total_elements = wl.elements if sharded else world * wl.elements

    def to_dev(a, dtype):
        if dtype == "bf16":
            return torch.from_numpy(bf16_bits(a).view(np.int16)).view(torch.bfloat16).cuda()
        return torch.from_numpy(a).cuda()

    t = dict(x=to_dev(inp["x"], wl.x_dtype), A_logs=to_dev(inp["A_logs"], "f32"), Ds=to_dev(inp["Ds"], "f32"),
             dt_bias=to_dev(inp["dt_bias"], "f32"))
    if wl.R > 0:
        # projection form: x_proj (bf16 weights) and dt_proj (fp32 weights) inside the call
        t.update(x_proj_weight=to_dev(inp["x_proj_weight"], "bf16"),
                 dt_projs_weight=to_dev(inp["dt_projs_weight"], "f32"))
    else:
        t.update(dts=to_dev(inp["dts"], wl.dt_dtype), Bs=to_dev(inp["Bs"], "f32"), Cs=to_dev(inp["Cs"], "f32"))
    stream = torch.cuda.current_stream()
    if args.which in ("backward", "train"):
        bench_backward(args, wl, inp, t, world, rank, local, stream, barrier, train=args.which == "train")
        if world > 1:
            dist.destroy_process_group()
        return
    y = torch.empty((wl_run.B, wl.D, wl.H, wl.W), dtype=torch.float32, device="cuda")
    ws_bytes = ss.forward_core_workspace_size(**t)
    workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device="cuda")
    launches = launches_per_step(wl_run, ws_bytes)

    def step():
        ss.forward_core(**t, y=y, workspace=workspace, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    barrier()
    torch.cuda.synchronize()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(args.steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize()
    barrier()
    clocks = sampler.stop()
    ms = max_over_ranks(ev0.elapsed_time(ev1), device="cuda")
    ms_per_step = ms / args.steps
    value = total_elements / (ms_per_step * 1e-3) / 1e9
    gather = None
    if sharded:
        # the one collective of the sharded path: y's shards gathered on every rank, timed apart
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        y_all = gather_shards(y, wl.B, world)
        g1.record(stream)
        torch.cuda.synchronize()
        gather = {"ms": max_over_ranks(g0.elapsed_time(g1), device="cuda"), "bytes": int(y_all.numel() * 4),
                  "collective": "all_gather of the batch shards of y"}
        del y_all

    # End to end through the public API with host buffers: pinned host -> device copy of the
    # step's inputs, the core, and the device -> host copy of y, all inside the timed region.
    e2e = None
    if not args.no_e2e:
        hosts = {k: v.cpu().pin_memory() for k, v in t.items()}
        ys = [y, torch.empty_like(y)]
        outs_host = [{"y": torch.empty(y.shape, dtype=torch.float32).pin_memory()} for _ in range(2)]
        h2d = sum(v.numel() * v.element_size() for v in hosts.values())
        d2h = y.numel() * 4

        def run(dv, sl, st):
            return {"y": ss.forward_core(**dv, y=ys[sl], workspace=workspace, stream=st)}

        ms_e2e = pipelined_e2e(hosts, run, outs_host, max(3, min(args.steps, 10)), barrier)
        # the downloaded result is the call's result (the four merge additions may round differently)
        got, ref = outs_host[0]["y"], ys[0].cpu()
        if float((got - ref).abs().max()) > 1e-4 * float(ref.abs().max()):
            raise SystemExit("e2e: downloaded y differs from the device result")
        ems = max_over_ranks(ms_e2e, device="cuda")
        e2e = {"value": total_elements / (ems * 1e-3) / 1e9, "unit": "Gelem/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "pipelined": "upload k+1 / call k / download k-1 on three streams"}

    hbm_peak, sm_max_mhz, peak_kind = load_peaks()
    standalone = None
    if wl.R == 0:
        standalone = time_standalone_scan(ss, wl_run, t, stream, args, barrier, hbm_peak)
    # per-GPU rates: this rank's bytes and exponentials over the step time
    bytes_step = algorithmic_bytes(wl_run)
    hbm_achieved = bytes_step / (ms_per_step * 1e-3) / 1e9
    # The fused kernel is bounded by the exponential unit: N exp2 per scan element for the
    # decays plus the exp2 of softplus.
    mufu_ops = wl_run.elements * (wl.N + FWD_MUFU_EXTRA)
    mufu_achieved = mufu_ops / (ms_per_step * 1e-3) / 1e9
    mufu_peak = MUFU_PER_CLK_PER_SM * SMS * sm_max_mhz * 1e6 / 1e9

    line = {
        "metric": "SS2D core Gelem/s (B*4*D*L)",
        "value": value,
        "unit": "Gelem/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": "strong" if sharded else "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": wl.name, "B": wl.B, "D": wl.D, "H": wl.H, "W": wl.W, "N": wl.N, "R": wl.R,
                   "x_dtype": wl.x_dtype, "dts_dtype": wl.dt_dtype, "l2": "no flush: inputs+output "
                   f"{bytes_step / 1e6:.0f} MB per step exceed the 126 MB L2",
                   "parallelism": f"batch shards x{world}" if sharded else f"replicas x{world}"},
        "roofline": {"bound": "alu", "achieved": mufu_achieved, "peak": mufu_peak, "unit": "Gop/s (MUFU ex2)",
                     "frac": mufu_achieved / mufu_peak, "traffic": recorded_traffic(wl),
                     "note": f"MUFU peak = {MUFU_PER_CLK_PER_SM}/clk/SM x {SMS} SMs x {sm_max_mhz:.0f} MHz; "
                             "duration = whole step (all kernels of the core call)"},
        "hbm": {"achieved": hbm_achieved, "peak": hbm_peak, "unit": "GB/s", "frac": hbm_achieved / hbm_peak,
                "algorithmic_bytes_per_step": bytes_step, "peak_source": peak_kind},
        "kernel_hash": kernel_source_hash(),
        "clocks": {"sm_mhz": clocks["sm_mhz"], "sm_max_mhz": clocks["sm_max_mhz"], "reasons": clocks["reasons"]},
        "gpu_launches": launches * args.steps,
        "e2e": e2e,
        "standalone_scan": standalone,
    }
    if gather is not None:
        line["gather"] = gather
    if rank == 0 and world == 1 and not args.no_other_workloads and wl.name == "vmamba_t_stage1" and args.batch == 0:
        line["other_workloads"] = other_workloads(ss, stream, hbm_peak)
        line["other_workloads_timing"] = "median of 20 calls after 3 warm-up calls, L2 flushed (256 MB write) " \
                                         "before each, CUDA events on the launching stream"
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
