"""Benchmark of the SubMConv3d hot path on B200: neighbour-map build + bf16 forward.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload headline|dense|shell_bf16|batched]

One step = one pass of the whole hot path over one synthetic input: the
neighbour-map build (table init, insert, 27-lookup query + tile masks + x-run
layout) and the bf16 tcgen05 forward, for the headline workload (128^3 grid,
8 sphere shells, 329,839 voxels, 128 -> 128 channels) by default; with
--workload batched, the decoder stack (4 x 256^3 shell sets, 1,135,307
voxels, one map build + 64 -> 128 -> 128 -> 128 -> 64 with exact GELU
between).  Inputs are resident in HBM when the timed region starts; the L2 is
flushed (256 MB write) before every timed step; each step is timed with CUDA
events on the launching stream.

With N > 1 (torchrun, one process per GPU) there is no collective on the data
path.  headline / dense / shell_bf16: every rank runs its own replica on its
own features (weak scaling; `value` counts the voxels of all ranks).
batched: rank r takes batch elements r, r + N, ... of the one batch, the
weights replicated (strong scaling; `value` counts the batch's voxels).  The
job time is the max over ranks.

--impl reference times the CPU oracle (oracle/, C++ std::map + fp64 loops) on
the host cores, every step on the same bounded sample of the workload (a
raster-order prefix sized to the time budget), and prints the same line with
"impl": "reference".
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "SubMConv3d fwd voxels/s and TFLOP/s at 128^3/128ch bf16; % of B200 roofline"
L2_FLUSH_BYTES = 256 << 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# Kernels one map build launches: table init, insert, and the query, which
# also lays out the x-run positions and the E index table; the brick table
# adds its block allocation.
MAP_LAUNCHES = 3

# Algorithmic bytes of the map build per voxel: int32 (b,z,y,x) in + int32 [27] out.
MAP_BYTES_PER_VOXEL = 16 + 27 * 4


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def _profiled_traffic(workload: str):
    """DRAM bytes per forward launch from the committed ncu summary, when the
    forward kernel's source is unchanged since that capture (hash match) and
    the capture was of this workload; else None."""
    import hashlib
    import re
    if workload != "headline":
        return None
    prof = os.path.join(ROOT, "profiles", "fwd_bf16_runs_headline.md")
    csrc = os.path.join(ROOT, "sparse_voxel_conv_b200", "csrc")
    try:
        text = open(prof).read()
        h = hashlib.sha256()
        for f in ("forward_bf16_runs_sm100.cu", "ptx.cuh", "epilogue.cuh", "internal.h"):
            h.update(open(os.path.join(csrc, f), "rb").read())
    except OSError:
        return None
    sha = re.search(r"source_sha256_16:\s*([0-9a-f]{16})", text)
    traffic = re.search(r"traffic_bytes_per_launch:\s*(\d+)", text)
    if not sha or not traffic or sha.group(1) != h.hexdigest()[:16]:
        return None
    return int(traffic.group(1))


def _workload_config(wl, nnz_avg):
    """The workload keys of `config`, the same in both arms."""
    return {"workload": wl.name, "n_voxels": wl.n, "nnz_avg": nnz_avg, "cin": wl.channels[0],
            "cout": wl.channels[1], "channels": list(wl.channels), "grid_dim": wl.grid_dim,
            "batch": wl.batch}


def _workload(name):
    import workloads as WL
    return WL.make_workload(name)


def feature_seed(rank: int) -> int:
    """Seed of a replica's features: every rank convolves its own input."""
    return 1 + 1000 * rank


def max_over_ranks(value: float, device) -> float:
    """The job's time is the slowest rank's: all-reduce MAX of a float (a
    no-op without an initialised process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, device) -> float:
    """The job's total of a per-rank quantity (all-reduce SUM of a float; the
    value itself without an initialised process group).  Bookkeeping only,
    outside the timed region."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def job_rate(units_per_rank: int, world: int, job_seconds: float) -> float:
    """Weak-scaling throughput: the units every rank processed / the job time."""
    return units_per_rank * world / job_seconds


class ClockSampler:
    """Samples nvidia-smi clocks and throttle reasons in the background."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.device_index = device_index
        self.lines = []
        self.proc = None
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.device_index)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def _time_ms(fn, flush, reps=5, warm=2):
    """Median CUDA-event time of fn() over `reps` calls, L2 flushed before each."""
    import torch
    for _ in range(warm):
        fn()
    ts = []
    for _ in range(reps):
        flush.fill_(7)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b))
    return statistics.median(ts)


def fp32_forward_line(h, feats_f32, w_f32, flops, flush, sm_mhz):
    """The fp32 path (CUDA-core FMA) on the same map, forward and weight
    gradient, against the FP32 peak SMs x 128 lanes x 2 flop x SM clock."""
    import torch
    import sparse_voxel_conv_b200 as S
    out = torch.empty((h.n, w_f32.shape[0]), dtype=torch.float32, device=feats_f32.device)
    ms = _time_ms(lambda: S.forward(h, feats_f32, w_f32, out=out), flush)
    dy = torch.empty_like(out).normal_()
    dw = torch.empty(w_f32.shape, dtype=torch.float32, device=feats_f32.device)
    w_ms = _time_ms(lambda: S.backward_weight(h, feats_f32, dy, out=dw), flush, reps=3, warm=1)
    sms = torch.cuda.get_device_properties(feats_f32.device).multi_processor_count
    peak = sms * 128 * 2 * sm_mhz * 1e6 / 1e12
    achieved = flops / (ms / 1e3) / 1e12
    w_achieved = flops / (w_ms / 1e3) / 1e12
    return {"bound": "alu", "ms": ms, "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
            "frac": achieved / peak,
            "peak_source": f"{sms} SMs x 128 FP32 lanes x 2 x {sm_mhz:.0f} MHz",
            "weight_gradient": {"ms": w_ms, "achieved": w_achieved, "frac": w_achieved / peak}}


def per_offset_context(h, feats, weight, flush):
    """The pages' "obvious per-offset loop" in torch on this GPU, as context:
    27 x (index_select + matmul + index_add_) over this library's nbr, fp32
    accumulation.  Not part of the timed step."""
    import torch
    nbr = h.nbr.long()
    cout = weight.shape[0]
    w = weight.reshape(cout, 27, -1)
    acc = torch.empty((h.n, cout), dtype=torch.float32, device=feats.device)
    rows = [(nbr[:, k] >= 0).nonzero().squeeze(1) for k in range(27)]
    src = [nbr[r, k] for k, r in enumerate(rows)]

    def loop():
        acc.zero_()
        for k in range(27):
            part = feats.index_select(0, src[k]) @ w[:, k, :].t()
            acc.index_add_(0, rows[k], part.float())
        return acc.to(feats.dtype)

    ms = _time_ms(loop, flush, reps=3, warm=1)
    return {"ms": ms, "what": "27 x (index_select + bf16 matmul + index_add_) in torch, "
            "fp32 accumulation, indices precomputed from this library's nbr"}


def fused_epilogue_line(h, feats, weight, flops, flush, peak_tf, plain_ms):
    """The residual-block epilogue fused into the headline forward:
    out = silu(conv + bias) + residual, against the same tensor-core peak."""
    import torch
    import sparse_voxel_conv_b200 as S
    cout = weight.shape[0]
    bias = torch.linspace(-0.5, 0.5, cout, device=feats.device).to(feats.dtype)
    res = torch.empty((h.n, cout), dtype=feats.dtype, device=feats.device).normal_()
    out = torch.empty_like(res)
    ms = _time_ms(lambda: S.forward(h, feats, weight, act="silu", bias=bias, residual=res,
                                    out=out), flush)
    achieved = flops / (ms / 1e3) / 1e12
    return {"what": "silu(conv + bias) + residual in the forward's epilogue",
            "ms": ms, "plain_forward_ms": plain_ms, "achieved": achieved, "peak": peak_tf,
            "unit": "TFLOP/s", "frac": achieved / peak_tf,
            "extra_bytes": int(h.n) * cout * feats.element_size()}


def backward_line(h, feats, weight, flops, flush, peak_tf, fp32_peak):
    """The backward on the headline map: input gradient (a tensor-core forward
    with the transposed weight) and weight gradient (tcgen05 over the x-run
    layout, fp32 output); both against the bf16 tensor-core peak."""
    import torch
    import sparse_voxel_conv_b200 as S
    dy = torch.empty((h.n, weight.shape[0]), dtype=feats.dtype, device=feats.device).normal_()
    dx = torch.empty_like(feats)
    dw = torch.empty(weight.shape, dtype=torch.float32, device=feats.device)
    d_ms = _time_ms(lambda: S.backward_data(h, dy, weight, out=dx), flush)
    w_ms = _time_ms(lambda: S.backward_weight(h, feats, dy, out=dw), flush, reps=3, warm=1)
    d_tf = flops / (d_ms / 1e3) / 1e12
    w_tf = flops / (w_ms / 1e3) / 1e12
    return {"data": {"ms": d_ms, "achieved": d_tf, "peak": peak_tf, "unit": "TFLOP/s",
                     "frac": d_tf / peak_tf, "bound": "tensor"},
            "weight": {"ms": w_ms, "achieved": w_tf, "peak": peak_tf, "unit": "TFLOP/s",
                       "frac": w_tf / peak_tf, "bound": "tensor"}}


def resample_line(coords, feats, grid, flush, hbm_gbs):
    """Subdivide the headline set (8 children per voxel, features replicated) and
    mean-pool the result back (the fine map built beforehand); algorithmic bytes
    over time, against the HBM copy peak.  Pooling reads its parent count back
    to the host, so its time includes that one synchronisation."""
    import sparse_voxel_conv_b200 as S
    st = S.SparseTensor(coords, feats, grid, 1)
    n, c = feats.shape
    esz = feats.element_size()
    sub_ms = _time_ms(lambda: S.subdivide(st), flush)
    fine = S.subdivide(st)
    fine.get_map("subm0")
    pool_ms = _time_ms(lambda: S.downsample(fine, "mean"), flush)
    sub_bytes = n * (16 + c * esz) + 8 * n * (16 + c * esz)
    pool_bytes = 8 * n * (16 + c * esz) + n * (16 + c * esz)
    sub_gbs = sub_bytes / (sub_ms / 1e3) / 1e9
    pool_gbs = pool_bytes / (pool_ms / 1e3) / 1e9
    return {"subdivide": {"ms": sub_ms, "bytes": sub_bytes, "achieved": sub_gbs,
                          "peak": hbm_gbs, "unit": "GB/s", "frac": sub_gbs / hbm_gbs,
                          "bound": "hbm"},
            "downsample_mean": {"ms": pool_ms, "bytes": pool_bytes, "achieved": pool_gbs,
                                "peak": hbm_gbs, "unit": "GB/s", "frac": pool_gbs / hbm_gbs,
                                "bound": "hbm", "children": 8 * n}}


def decoder_stack_line(flush, peak_tf):
    """The decoder stack of the batched workload (4 x 256^3 sets, 1.14 M voxels,
    64 -> 128 -> 128 -> 128 -> 64 channels, exact GELU between layers): one map
    build and four fused layers on it, timed as one unit."""
    import torch
    import sparse_voxel_conv_b200 as S
    import workloads as WL
    wl = WL.make_workload("batched")
    dev = torch.device("cuda")
    coords = torch.from_numpy(wl.coords).to(dev)
    x0 = torch.from_numpy(WL.to_bf16_values(wl.features())).to(dev).to(torch.bfloat16)
    ws = [torch.from_numpy(w).to(dev).to(torch.bfloat16) for w in wl.weights()]
    n = wl.n
    outs = [torch.empty((n, w.shape[0]), dtype=torch.bfloat16, device=dev) for w in ws]
    nbr = torch.empty((n, 27), dtype=torch.int32, device=dev)
    ws_bytes = S._abi.subm3d_map_workspace_bytes(n, wl.grid_dim, wl.batch)
    work = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)

    def run():
        h = S.build_map(coords, wl.grid_dim, wl.batch, check=False, nbr=nbr, workspace=work)
        x = x0
        for li, w in enumerate(ws):
            x = S.forward(h, x, w, act="gelu" if li < len(ws) - 1 else None, out=outs[li])
        return x

    run()
    torch.cuda.synchronize()
    nnz = int((nbr >= 0).sum().item())
    ms = _time_ms(run, flush)
    flops = sum(2.0 * nnz * w.shape[0] * w.shape[-1] for w in ws)  # KRSC: Cout ... Cin
    tf = flops / (ms / 1e3) / 1e12
    # where the time goes: the map build and each layer alone (L2 flushed before each)
    h = S.build_map(coords, wl.grid_dim, wl.batch, check=False, nbr=nbr, workspace=work)
    parts = {"map_build": _time_ms(lambda: S.build_map(coords, wl.grid_dim, wl.batch,
                                                         check=False, nbr=nbr, workspace=work),
                                   flush)}
    ins = [x0] + outs[:-1]
    for li, w in enumerate(ws):
        act = "gelu" if li < len(ws) - 1 else None
        parts[f"layer{li} {w.shape[-1]}->{w.shape[0]}"] = _time_ms(
            lambda li=li, w=w, act=act: S.forward(h, ins[li], w, act=act, out=outs[li]), flush)
    table = {S._abi.SUBM3D_TABLE_DIRECT: "direct", S._abi.SUBM3D_TABLE_HASH: "hash",
             S._abi.SUBM3D_TABLE_BRICK: "brick"}[S._abi.subm3d_map_table(h)]
    return {"workload": wl.name, "n_voxels": n, "ms": ms, "voxels_per_s": n / (ms / 1e3),
            "flops": flops, "achieved": tf, "peak": peak_tf, "unit": "TFLOP/s",
            "frac": tf / peak_tf, "what": "one map build + 4 fused bf16 layers on it",
            "map_table": table, "parts_ms": parts}


def batch_elements(rank: int, world: int, batch: int) -> list:
    """Batch elements a rank takes when a batch is split over `world` ranks:
    rank, rank + world, rank + 2 world, ... (none when rank >= batch)."""
    return list(range(rank, batch, world))


def split_batch(coords: np.ndarray, elems) -> np.ndarray:
    """The rows of the given batch elements, in that order, their batch index
    renumbered 0, 1, ...: batch elements never share a neighbour, so each rank
    builds the map of its own elements alone."""
    parts = []
    for new_b, b in enumerate(elems):
        c = coords[coords[:, 0] == b].copy()
        c[:, 0] = new_b
        parts.append(c)
    return np.concatenate(parts) if parts else np.zeros((0, 4), np.int32)


class Job:
    """What one rank runs per step: its coordinate rows, features and layers.

    headline / dense / shell_bf16: every rank runs a replica of the whole set on
    its own features (weak scaling).  batched: the decoder-stack workload's
    batch elements are split over the ranks (batch_elements), W replicated,
    total work fixed (strong scaling); ranks past the batch size idle.  No
    collective on the data path either way."""

    def __init__(self, name: str, rank: int, world: int):
        import workloads as WL
        wl = WL.make_workload(name)
        self.wl = wl
        self.name = name
        if name == "batched":
            self.elems = batch_elements(rank, world, wl.batch)
            self.coords = split_batch(wl.coords, self.elems)
            self.batch = max(1, len(self.elems))
            self.units_job = wl.n
            self.scaling = "strong"
            self.parallelism = (f"batch split x{world}: rank r takes elements r, r+{world}, ... "
                                "(W replicated), no collective on the data path")
        else:
            self.elems = list(range(wl.batch))
            self.coords = wl.coords
            self.batch = wl.batch
            self.units_job = wl.n * world
            self.scaling = "weak"
            self.parallelism = f"replicas x{world}, no collective on the data path"
        self.n = int(self.coords.shape[0])
        self.grid = wl.grid_dim
        self.channels = list(wl.channels)
        n_layers = len(self.channels) - 1
        self.acts = ["gelu" if wl.gelu_between and li < n_layers - 1 else None
                     for li in range(n_layers)]
        self.weights = wl.weights()
        self.feats = WL.to_bf16_values(WL.make_features(self.n, self.channels[0],
                                                        feature_seed(rank)))

    def flops(self, nnz: int) -> float:
        """Algorithmic FLOPs of the layers over a map with nnz neighbour pairs."""
        return sum(2.0 * nnz * self.channels[li] * self.channels[li + 1]
                   for li in range(len(self.channels) - 1))

    def step_text(self, map_launches: int = MAP_LAUNCHES, table: str = "direct") -> str:
        layers = len(self.channels) - 1
        build = f"map build ({table} table, {map_launches} kernels)"
        if layers == 1:
            return f"{build} + bf16 x-run forward (1 kernel)"
        return f"{build} + {layers} bf16 forward layers on it (exact GELU between)"


def run_ours(args):
    import torch
    import torch.distributed as dist

    import sparse_voxel_conv_b200 as S
    from sparse_voxel_conv_b200 import _abi

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream()

    job = Job(args.workload, rank, world)
    wl = job.wl
    n = job.n
    cin, cout = job.channels[0], job.channels[-1]
    coords_h = torch.from_numpy(job.coords)
    feats_h = torch.from_numpy(job.feats)
    ws_h = [torch.from_numpy(w) for w in job.weights]
    coords = coords_h.to(dev)
    feats = feats_h.to(dev).to(torch.bfloat16)
    weights = [w.to(dev).to(torch.bfloat16) for w in ws_h]
    outs = [torch.empty((n, w.shape[0]), dtype=torch.bfloat16, device=dev) for w in weights]
    nbr = torch.empty((n, 27), dtype=torch.int32, device=dev)
    ws_bytes = max(1, _abi.subm3d_map_workspace_bytes(n, job.grid, job.batch))
    workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def compute(c, x0, ws, outs_, nbr_, work, ev_fwd=None, s=None):
        """The step's work on one buffer set: the map build, then every layer."""
        if n == 0:
            if ev_fwd is not None:
                ev_fwd[0].record(stream)
                ev_fwd[1].record(stream)
            return None
        h = S.build_map(c, job.grid, job.batch, check=False, nbr=nbr_, workspace=work, stream=s)
        if ev_fwd is not None:
            ev_fwd[0].record(stream)
        x = x0
        for li, w in enumerate(ws):
            x = S.forward(h, x, w, act=job.acts[li], out=outs_[li], stream=s)
        if ev_fwd is not None:
            ev_fwd[1].record(stream)
        return h

    def step(ev_fwd=None):
        return compute(coords, feats, weights, outs, nbr, workspace, ev_fwd)

    # correctness gate before timing: the map must be valid
    h0 = step()
    map_launches, table = MAP_LAUNCHES, "direct"
    if h0 is not None:
        assert S.map_status(h0) == 0, "map build reported a data error"
        kind = _abi.subm3d_map_table(h0)
        table = {_abi.SUBM3D_TABLE_DIRECT: "direct", _abi.SUBM3D_TABLE_HASH: "hash",
                 _abi.SUBM3D_TABLE_BRICK: "brick"}[kind]
        map_launches = MAP_LAUNCHES + (1 if kind == _abi.SUBM3D_TABLE_BRICK else 0)
    nnz_total = int((nbr >= 0).sum().item())
    assert _abi.subm3d_device_status() == 0
    for _ in range(args.warmup):
        flush.fill_(1)
        step()
    torch.cuda.synchronize()

    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(K)]
    evf = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(K)]
    visible = os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",")
    smi_index = visible[dev.index].strip() if len(visible) > dev.index and visible[0] else dev.index
    sampler = ClockSampler(smi_index)
    sampler.start()
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    for i in range(K):
        flush.fill_(i & 0xFF)
        ev[i][0].record(stream)
        step(evf[i])
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    assert _abi.subm3d_device_status() == 0
    step_ms = [a.elapsed_time(b) for a, b in ev]
    fwd_ms = [a.elapsed_time(b) for a, b in evf]
    map_ms = [s_ - f for s_, f in zip(step_ms, fwd_ms)]
    total_ms = max_over_ranks(float(sum(step_ms)), dev)

    # e2e through the public API with host buffers: every step copies its inputs
    # in from pinned memory, builds the map, runs the layers and copies the last
    # output back.  Steps are pipelined over two device buffer sets and three
    # streams (inputs in, compute, output out), ordered by events, so step k's
    # copies overlap the compute of its neighbours (PCIe is full duplex).  The
    # timed region runs from the first input copy to the last output copy.
    coords_p = coords_h.pin_memory()
    feats_p = feats_h.to(torch.bfloat16).pin_memory()
    ws_p = [w.to(torch.bfloat16).pin_memory() for w in ws_h]
    outs_p = [torch.empty((n, cout), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    h2d = coords_p.numel() * 4 + feats_p.numel() * 2 + sum(w.numel() * 2 for w in ws_p)
    d2h = outs_p[0].numel() * 2
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    bufs = [dict(coords=torch.empty_like(coords), feats=torch.empty_like(feats),
                 weights=[torch.empty_like(w) for w in weights],
                 outs=[torch.empty_like(o) for o in outs],
                 nbr=torch.empty_like(nbr), ws=torch.empty_like(workspace)) for _ in range(2)]
    mk = lambda: torch.cuda.Event()
    in_done, comp_done, out_done = [mk(), mk()], [mk(), mk()], [mk(), mk()]
    for e in in_done + comp_done + out_done:
        e.record(stream)

    def e2e_step(k):
        bset = k & 1
        B = bufs[bset]
        with torch.cuda.stream(s_in):
            s_in.wait_event(comp_done[bset])      # the previous user of this set has read it
            B["coords"].copy_(coords_p, non_blocking=True)
            B["feats"].copy_(feats_p, non_blocking=True)
            for dst, src in zip(B["weights"], ws_p):
                dst.copy_(src, non_blocking=True)
            in_done[bset].record(s_in)
        stream.wait_event(in_done[bset])
        stream.wait_event(out_done[bset])         # its output buffer has been copied out
        compute(B["coords"], B["feats"], B["weights"], B["outs"], B["nbr"], B["ws"], s=stream)
        comp_done[bset].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(comp_done[bset])
            outs_p[bset].copy_(B["outs"][-1], non_blocking=True)
            out_done[bset].record(s_out)

    for k in range(max(2, args.warmup)):
        e2e_step(k)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for k in range(K):
        e2e_step(k)
    e1.record(s_out)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dev)
    job_flops = sum_over_ranks(job.flops(nnz_total), dev)  # every rank's layers

    if rank == 0:
        peaks, peak_src = _peaks()
        flops = job.flops(nnz_total)
        fwd_avg_s = statistics.mean(fwd_ms) / 1e3
        map_avg_s = statistics.mean(map_ms) / 1e3
        achieved_tf = flops / fwd_avg_s / 1e12
        peak_tf = float(peaks["bf16_tflops"])
        map_gbs = n * MAP_BYTES_PER_VOXEL / map_avg_s / 1e9
        n_layers = len(job.weights)
        line = {
            "metric": METRIC,
            "value": job.units_job / (total_ms / 1e3 / K),
            "unit": "voxels/s",
            "n_gpus": world,
            "steps": K,
            "warmup": args.warmup,
            "ms_per_step": total_ms / K,
            "higher_is_better": True,
            "scaling": job.scaling,
            "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic",
            "config": {
                **_workload_config(wl, nnz_total / max(n, 1)),
                "step": job.step_text(map_launches, table),
                "l2": f"flushed before every timed step ({L2_FLUSH_BYTES >> 20} MB write)",
                "parallelism": job.parallelism,
            },
            "tflops_effective": job_flops / (total_ms / 1e3 / K) / 1e12,
            "roofline": {
                "kernel": "subm3d_fwd_bf16_runs_sm100" + (f" (x{n_layers} layers)"
                                                         if n_layers > 1 else ""),
                "bound": "tensor", "achieved": achieved_tf, "peak": peak_tf, "unit": "TFLOP/s",
                "frac": achieved_tf / peak_tf, "traffic": _profiled_traffic(args.workload),
                "traffic_unit": "bytes per launch (ncu dram read+write)",
                "peak_source": f"{peak_src} bf16 dense burst",
                "fwd_ms_avg": fwd_avg_s * 1e3,
            },
            "map_build": {
                "bound": "hbm", "achieved": map_gbs, "peak": float(peaks["hbm_gbs"]),
                "unit": "GB/s", "frac": map_gbs / float(peaks["hbm_gbs"]),
                "bytes_per_voxel": MAP_BYTES_PER_VOXEL, "ms_avg": map_avg_s * 1e3,
            },
            "e2e": {"value": job.units_job / (e2e_ms / 1e3 / K), "unit": "voxels/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": e2e_ms / K},
            "gpu_launches": (map_launches + n_layers) * K,
            "clocks": clocks,
        }
        if job.name == "batched":
            line["config"]["batch_elements_rank0"] = job.elems
        if world == 1 and not args.no_context and job.name == "headline":
            h_ctx = step()
            torch.cuda.synchronize()
            w0 = weights[0]
            line["fp32_forward"] = fp32_forward_line(
                h_ctx, feats.float(), w0.float(), flops, flush,
                float(clocks.get("sm_mhz") or clocks.get("sm_max_mhz") or 1965.0))
            line["fused_epilogue"] = fused_epilogue_line(h_ctx, feats, w0, flops, flush,
                                                         peak_tf, fwd_avg_s * 1e3)
            line["backward"] = backward_line(h_ctx, feats, w0, flops, flush, peak_tf,
                                             line["fp32_forward"]["peak"])
            line["resample"] = resample_line(coords, feats, wl.grid_dim, flush,
                                             float(peaks["hbm_gbs"]))
            line["decoder_stack"] = decoder_stack_line(flush, peak_tf)
            line["context_per_offset_torch"] = per_offset_context(h_ctx, feats, w0, flush)
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(job, args.cpu_budget_s)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def oracle_step(job, m: int) -> float:
    """One pass of the whole path through the oracle (oracle/, C++ std::map and
    fp64 loops) on a bounded sample of the job: the first m rows of its
    coordinate set in raster order -- their map, then every layer over them
    (GELU between where the workload has it, bf16 rounding after each layer).
    Returns the seconds it took."""
    from oracle import cpp as C
    c = job.coords[:m]
    t0 = time.perf_counter()
    nbr = C.build_map(c, job.grid, job.batch)
    x = job.feats[:m].astype(np.float64)
    for li, w in enumerate(job.weights):
        x = C.forward(nbr, x, w.astype(np.float64), act=job.acts[li], round_to_bf16=True)
    return time.perf_counter() - t0


def oracle_sample_rows(job, seconds: float) -> int:
    """Rows of a sample whose oracle_step takes about `seconds` (from a timed
    pass over 4,096 rows), at most the whole set."""
    m0 = min(job.n, 4096)
    if m0 == 0:
        return 0
    per_row = oracle_step(job, m0) / m0
    return int(max(m0, min(job.n, seconds / per_row)))


def cpu_baseline(job, budget_s: float, reps: int = 2):
    """The oracle as it stands on the host cores: `reps` passes of oracle_step
    over a raster-order prefix sized to about budget_s / reps seconds (all
    rows when they fit); voxels/s = rows / mean pass time."""
    from oracle import cpp as C
    m = oracle_sample_rows(job, budget_s / reps)
    ts = [oracle_step(job, m) for _ in range(reps)]
    what = "all rows" if m == job.n else f"the first {m} of {job.n} rows (raster order)"
    return {"value": m / statistics.mean(ts), "unit": "voxels/s",
            "cores": C.num_threads(), "kind": "oracle",
            "sample": f"{reps} x (map build + {len(job.weights)} fp64 layer(s)) over {what}, "
                      f"{statistics.mean(ts):.2f} s each"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from oracle import cpp as C
    job = Job(args.workload, 0, 1)
    wl = job.wl
    # every step is the same bounded sample, sized so that the K timed steps
    # take about --ref-budget-s seconds in all
    m = oracle_sample_rows(job, args.ref_budget_s / max(1, args.steps))
    nnz_avg = float((C.build_map(wl.coords, wl.grid_dim, wl.batch) >= 0).sum()) / wl.n
    for _ in range(min(args.warmup, 2)):
        oracle_step(job, min(m, 4096))
    t_start = time.perf_counter()
    ts = [oracle_step(job, m) for _ in range(args.steps)]
    wall = time.perf_counter() - t_start
    step_s = statistics.mean(ts)
    value = m / step_s
    what = "all rows" if m == job.n else f"the first {m} of {job.n} rows (raster order)"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "voxels/s",
        "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_s * 1e3,
        "higher_is_better": True, "scaling": job.scaling, "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {**_workload_config(wl, nnz_avg),
                   "step": f"map build + {len(job.weights)} fp64 layer(s) (C++ oracle)",
                   "parallelism": "host cores (OpenMP)"},
        "cpu_baseline": {"value": value, "unit": "voxels/s", "cores": C.num_threads(),
                         "kind": "oracle",
                         "sample": f"every step: map build + {len(job.weights)} fp64 layer(s) "
                                   f"over {what}; {args.steps} steps in {wall:.1f} s"},
        "e2e": {"value": value, "unit": "voxels/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="headline",
                    choices=["headline", "dense", "shell_bf16", "batched"])
    ap.add_argument("--cpu-budget-s", type=float, default=16.0,
                    help="host seconds the cpu_baseline passes may take in all")
    ap.add_argument("--ref-budget-s", type=float, default=60.0,
                    help="host seconds the reference arm's timed steps may take in all")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-context", action="store_true",
                    help="skip the fp32-path and per-offset-loop context measurements")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
