"""Benchmark of the SubMConv3d hot path on B200: neighbour-map build + bf16 forward.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload headline|dense|shell_bf16]

One step = one pass of the whole hot path over one synthetic input: the
neighbour-map build (hash-table init, insert, 27-probe query + tile masks) and
the bf16 tcgen05 forward, for the headline workload (128^3 grid, 8 sphere
shells, 329,839 voxels, 128 -> 128 channels).  Inputs are resident in HBM
when the timed region starts; the L2 is flushed (256 MB write) before every
timed step; each step is timed with CUDA events on the launching stream.

With N > 1 (torchrun, one process per GPU) every rank runs its own replica on
its own features (weak scaling, no collective on the data path); the job time
is the max over ranks and `value` counts the voxels of all ranks.

--impl reference times the CPU oracle (oracle/, C++ std::map + fp64 loop) on
the host cores, on bounded samples of the same workload, and prints the same
line with "impl": "reference".
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
# also lays out the x-run positions and the E index table.
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
        for f in ("forward_bf16_runs_sm100.cu", "ptx.cuh", "epilogue.cuh"):
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
            "cout": wl.channels[1], "grid_dim": wl.grid_dim, "batch": wl.batch}


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
    """The fp32 path (CUDA-core FMA) on the same map, against the FP32 peak
    SMs x 128 lanes x 2 flop x SM clock."""
    import torch
    import sparse_voxel_conv_b200 as S
    out = torch.empty((h.n, w_f32.shape[0]), dtype=torch.float32, device=feats_f32.device)
    ms = _time_ms(lambda: S.forward(h, feats_f32, w_f32, out=out), flush)
    sms = torch.cuda.get_device_properties(feats_f32.device).multi_processor_count
    peak = sms * 128 * 2 * sm_mhz * 1e6 / 1e12
    achieved = flops / (ms / 1e3) / 1e12
    return {"bound": "alu", "ms": ms, "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
            "frac": achieved / peak,
            "peak_source": f"{sms} SMs x 128 FP32 lanes x 2 x {sm_mhz:.0f} MHz"}


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
    return {"workload": wl.name, "n_voxels": n, "ms": ms, "voxels_per_s": n / (ms / 1e3),
            "flops": flops, "achieved": tf, "peak": peak_tf, "unit": "TFLOP/s",
            "frac": tf / peak_tf, "what": "one map build + 4 fused bf16 layers on it"}


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

    wl = _workload(args.workload)
    import workloads as WL
    cin, cout = wl.channels[0], wl.channels[1]
    n = wl.n
    coords_h = torch.from_numpy(wl.coords)
    feats_h = torch.from_numpy(WL.to_bf16_values(WL.make_features(n, cin, feature_seed(rank))))
    w_h = torch.from_numpy(wl.weights()[0])
    coords = coords_h.to(dev)
    feats = feats_h.to(dev).to(torch.bfloat16)
    weight = w_h.to(dev).to(torch.bfloat16)
    out = torch.empty((n, cout), dtype=torch.bfloat16, device=dev)
    nbr = torch.empty((n, 27), dtype=torch.int32, device=dev)
    ws_bytes = _abi.subm3d_map_workspace_bytes(n, wl.grid_dim, wl.batch)
    workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def step(ev_fwd=None):
        h = S.build_map(coords, wl.grid_dim, wl.batch, check=False, nbr=nbr, workspace=workspace)
        if ev_fwd is not None:
            ev_fwd[0].record(stream)
        S.forward(h, feats, weight, out=out)
        if ev_fwd is not None:
            ev_fwd[1].record(stream)
        return h

    # correctness gate before timing: the map must be valid
    h0 = step()
    assert S.map_status(h0) == 0, "map build reported a data error"
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
    map_ms = [s - f for s, f in zip(step_ms, fwd_ms)]
    total_ms = max_over_ranks(float(sum(step_ms)), dev)

    # e2e through the public API with host buffers: every step copies its inputs
    # in from pinned memory, builds the map, runs the forward and copies its
    # output back.  Steps are pipelined over two device buffer sets and three
    # streams (inputs in, compute, output out), ordered by events, so step k's
    # copies overlap the compute of its neighbours (PCIe is full duplex).  The
    # timed region runs from the first input copy to the last output copy.
    coords_p = coords_h.pin_memory()
    feats_p = feats_h.to(torch.bfloat16).pin_memory()
    w_p = w_h.to(torch.bfloat16).pin_memory()
    outs_p = [torch.empty((n, cout), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    h2d = coords_p.numel() * 4 + feats_p.numel() * 2 + w_p.numel() * 2
    d2h = outs_p[0].numel() * 2
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    bufs = [dict(coords=torch.empty_like(coords), feats=torch.empty_like(feats),
                 weight=torch.empty_like(weight), out=torch.empty_like(out),
                 nbr=torch.empty_like(nbr), ws=torch.empty_like(workspace)) for _ in range(2)]
    ev = lambda: torch.cuda.Event()
    in_done, comp_done, out_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    for e in in_done + comp_done + out_done:
        e.record(stream)

    def e2e_step(k):
        bset = k & 1
        B = bufs[bset]
        with torch.cuda.stream(s_in):
            s_in.wait_event(comp_done[bset])      # the previous user of this set has read it
            B["coords"].copy_(coords_p, non_blocking=True)
            B["feats"].copy_(feats_p, non_blocking=True)
            B["weight"].copy_(w_p, non_blocking=True)
            in_done[bset].record(s_in)
        stream.wait_event(in_done[bset])
        stream.wait_event(out_done[bset])         # its output buffer has been copied out
        h = S.build_map(B["coords"], wl.grid_dim, wl.batch, check=False, nbr=B["nbr"],
                        workspace=B["ws"], stream=stream)
        S.forward(h, B["feats"], B["weight"], out=B["out"], stream=stream)
        comp_done[bset].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(comp_done[bset])
            outs_p[bset].copy_(B["out"], non_blocking=True)
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

    if rank == 0:
        peaks, peak_src = _peaks()
        flops = 2.0 * nnz_total * cin * cout
        fwd_avg_s = statistics.mean(fwd_ms) / 1e3
        map_avg_s = statistics.mean(map_ms) / 1e3
        achieved_tf = flops / fwd_avg_s / 1e12
        peak_tf = float(peaks["bf16_tflops"])
        map_gbs = n * MAP_BYTES_PER_VOXEL / map_avg_s / 1e9
        voxels_total = n * world
        line = {
            "metric": METRIC,
            "value": job_rate(n, world, total_ms / 1e3 / K),
            "unit": "voxels/s",
            "n_gpus": world,
            "steps": K,
            "warmup": args.warmup,
            "ms_per_step": total_ms / K,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic",
            "config": {
                **_workload_config(wl, nnz_total / n),
                "step": f"map build ({MAP_LAUNCHES} kernels) + bf16 x-run forward (1 kernel)",
                "l2": f"flushed before every timed step ({L2_FLUSH_BYTES >> 20} MB write)",
                "parallelism": f"replicas x{world}, no collective on the data path",
            },
            "tflops_effective": flops * world / (total_ms / 1e3 / K) / 1e12,
            "roofline": {
                "kernel": "subm3d_fwd_bf16_runs_sm100",
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
            "e2e": {"value": job_rate(n, world, e2e_ms / 1e3 / K), "unit": "voxels/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": e2e_ms / K},
            "gpu_launches": (MAP_LAUNCHES + 1) * K,
            "clocks": clocks,
        }
        if world == 1 and not args.no_context:
            h_ctx = step()
            torch.cuda.synchronize()
            flops_alg = 2.0 * nnz_total * cin * cout
            line["fp32_forward"] = fp32_forward_line(
                h_ctx, feats.float(), weight.float(), flops_alg, flush,
                float(clocks.get("sm_mhz") or clocks.get("sm_max_mhz") or 1965.0))
            line["fused_epilogue"] = fused_epilogue_line(h_ctx, feats, weight, flops_alg, flush,
                                                         peak_tf, fwd_avg_s * 1e3)
            line["backward"] = backward_line(h_ctx, feats, weight, flops_alg, flush, peak_tf,
                                             line["fp32_forward"]["peak"])
            line["resample"] = resample_line(coords, feats, wl.grid_dim, flush,
                                             float(peaks["hbm_gbs"]))
            line["decoder_stack"] = decoder_stack_line(flush, peak_tf)
            line["context_per_offset_torch"] = per_offset_context(h_ctx, feats, weight, flush)
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(wl, args.cpu_rows)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def _oracle_inputs(wl):
    import workloads as WL
    x = WL.to_bf16_values(WL.make_features(wl.n, wl.channels[0], 1)).astype(np.float64)
    w = wl.weights()[0].astype(np.float64)
    return x, w


def _oracle_step(wl, x, w, rows):
    """One bounded oracle pass: the whole map (std::map) + the forward of `rows`."""
    from oracle import cpp as C
    t0 = time.perf_counter()
    nbr = C.build_map(wl.coords, wl.grid_dim, wl.batch)
    t1 = time.perf_counter()
    C.forward(nbr, x, w, rows=rows, round_to_bf16=True)
    t2 = time.perf_counter()
    return t1 - t0, t2 - t1


def cpu_baseline(wl, n_rows, reps=2):
    """The oracle as it stands on the host cores: map build of the full set plus
    the fp64 forward of `n_rows` evenly spaced rows (all rows when n_rows <= 0),
    `reps` times; voxels/s = 1 / mean(map_s / N + fwd_s / rows)."""
    from oracle import cpp as C
    n_rows = wl.n if n_rows <= 0 else min(n_rows, wl.n)
    rows = np.linspace(0, wl.n - 1, n_rows).astype(np.int64)
    x, w = _oracle_inputs(wl)
    per_voxel, map_t, fwd_t = [], [], []
    for _ in range(reps):
        map_s, fwd_s = _oracle_step(wl, x, w, rows)
        map_t.append(map_s)
        fwd_t.append(fwd_s)
        per_voxel.append(map_s / wl.n + fwd_s / rows.size)
    what = ("all rows" if rows.size == wl.n else f"{rows.size} evenly spaced rows")
    return {"value": 1.0 / statistics.mean(per_voxel), "unit": "voxels/s",
            "cores": C.num_threads(), "kind": "oracle",
            "sample": f"{reps} x (map build of all {wl.n} voxels, {statistics.mean(map_t):.2f} s "
                      f"+ fp64 forward of {what}, {statistics.mean(fwd_t):.2f} s)"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from oracle import cpp as C
    wl = _workload(args.workload)
    # rows per step shrink with K so that the whole run stays within minutes
    cap = wl.n if args.cpu_rows <= 0 else args.cpu_rows
    n_rows = max(256, min(cap, 2_000_000 // max(1, args.steps), wl.n))
    rows = np.linspace(0, wl.n - 1, n_rows).astype(np.int64)
    x, w = _oracle_inputs(wl)
    nnz_avg = float((C.build_map(wl.coords, wl.grid_dim, wl.batch) >= 0).sum()) / wl.n
    for _ in range(min(args.warmup, 3)):
        _oracle_step(wl, x, w, rows[:256])
    per_voxel = []
    t_start = time.perf_counter()
    for _ in range(args.steps):
        map_s, fwd_s = _oracle_step(wl, x, w, rows)
        per_voxel.append(map_s / wl.n + fwd_s / rows.size)
    wall = time.perf_counter() - t_start
    sec_per_voxel = statistics.mean(per_voxel)
    value = 1.0 / sec_per_voxel
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "voxels/s",
        "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": sec_per_voxel * wl.n * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {**_workload_config(wl, nnz_avg),
                   "step": "map build + fp64 forward (C++ oracle)",
                   "parallelism": "host cores (OpenMP)"},
        "cpu_baseline": {"value": value, "unit": "voxels/s", "cores": C.num_threads(),
                         "kind": "oracle",
                         "sample": f"per step: map build of all {wl.n} voxels + fp64 forward "
                                   f"of {rows.size} evenly spaced rows; ms_per_step extrapolates "
                                   f"to the full set; wall {wall:.1f} s"},
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
    ap.add_argument("--workload", default="headline", choices=["headline", "dense", "shell_bf16"])
    ap.add_argument("--cpu-rows", type=int, default=0,
                    help="rows of the cpu_baseline forward (0: all rows of the workload)")
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
