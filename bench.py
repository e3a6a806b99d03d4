#!/usr/bin/env python
"""Benchmark of the bit-packed VQ/RVQ hot path on B200 (one JSON line).

Step = one decode pass of the Llama-3-70B-shaped MLP at 2.0 bits per weight:
gate_proj and up_proj (28672 x 8192) and down_proj (8192 x 28672), d = 8, one
K = 2^16 fp16 codebook, per-row fp16 scale and bias, batch B = 1, through
vq_gemv_multi (gate_proj and up_proj, which read the same x, in one launch)
and vq_gemv (down_proj).  All three layers are stored in the tiled index
order (made by vq_repack_tile4 from the generated row-order streams, exactly
2.0 bits per weight like the row order) and run the lookup-table kernel.  Two copies of the three layers
(352 MB of index streams) are used in turn, so every step reads its weights
from HBM, not from the 126 MB L2.

value  = algorithmic bytes moved per step (packed indices + codebook + scale
         and bias + activations + outputs) x steps x ranks / timed region,
         in GB/s; the timed region is bracketed by a barrier and a device
         synchronise on both sides and is the max over ranks.
e2e    = the same metric through the public Python API with the activations
         in pinned host memory: each step copies the three layers' x to the
         device in one transfer, runs the layers and copies the three y back
         in one transfer.
gemm   = the prefill GEMM (x [2048, 8192] bf16, 8192 x 8192 layer, K = 2^16
         + residual K = 2^8, 3.0 bpw) through vq_gemm, in TFLOP/s.
encode = the nearest-centroid encoder (vq_encode) on a 4096 x 4096 matrix
         against one K = 2^16, d = 8 book, in (vector, centroid) pairs/s.
rht_gate = the 70B gate_proj in the rotated basis (vq_gemv_rht) beside the
         same layer through vq_gemv.
hessian = vq_hessian on 8192 tokens x 8192 features, in TFLOP/s.
sweep  = every other configuration of the measurement plan, one call each
         (tiny 512^2; 8B up_proj at B 1/4/16; 70B gate_proj and down_proj at
         B 2/8/16; 405B gate_proj at B 2/4/8/16 and prefill M=1024, 405B q_proj
         at M=1024; the 8192^2 prefill at M 512/4096).
roofline, cpu_baseline, clocks and gpu_launches are described beside the
keys they fill.  ``--impl reference`` times the CPU oracle on the same
metric instead (a bounded sample of the same workload per step).

Multi-GPU (torchrun): every rank runs its own copy of the step (the layer
rows shard with no exchange), so scaling is weak and no collective touches
the data path; NCCL is used only for the barrier and the max of the times.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402
from synth import WORKLOADS  # noqa: E402

METRIC = "VQ-GEMV µs/layer & achieved HBM GB/s (% of peak) at 2 bpw; GEMM TFLOP/s"
NOMINAL_HBM_GBS = 8000.0
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
DECODE = "llama3_70b_mlp"
PREFILL = "prefill_8192"
PREFILL_M = 2048
BATCH = 1
# Index order per decode layer (gate_proj, up_proj, down_proj): the layout
# whose batch-1 kernel measured faster on that shape (the tiled table kernel
# on all three: 89 / 89 / 140 us against 150 / 150 / 161 in row order).
LAYOUTS = ("tile4", "tile4", "tile4")
# Encoder workload (vq_encode): a 4096 x 4096 fp16 weight matrix ~ N(0, 0.02)
# against one K = 2^16, d = 8 codebook ~ N(0, 0.02) (2.0 bpw).
ENCODE_SHAPE = (4096, 4096, 8, [16])
ENCODE_STD = [0.02]
ENCODE_SEED = 11
# The Hessian-weighted encoder's H: 2 X^T X / n + 0.01 mean(diag) I of 1024
# synthetic bf16 tokens ~ N(0, 1) with 0.1 % outlier channels x20 (vq_hessian).
ENCODE_H_TOKENS = 1024
ENCODE_H_SEED = 14
RHT_SEED = 12           # sign bits of the rotated-basis measurement
HESSIAN_SHAPE = (8192, 8192)   # tokens, features
HESSIAN_SEED = 13


def kernel_sources_sha(files) -> str:
    """sha256 over the named source files (paths relative to the repo root)."""
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def profiled_traffic(kernel: str):
    """DRAM bytes per launch of `kernel` from the committed ncu record
    (profiles/traffic.json), or None when the kernel's sources changed since
    that capture."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as fh:
            rec = json.load(fh)[kernel]
        if kernel_sources_sha(rec["sources"]) != rec["sources_sha256"]:
            return None
        return rec
    except Exception:
        return None


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            p = json.load(fh)
        return {k: float(p[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except Exception:
        return dict(FALLBACK), "fallback"


def alg_bytes(spec, batch: int) -> float:
    """Bytes the layer must move once: packed indices (nvec * b bits per
    row), each codebook once, fp16 scale and bias, bf16 x and y."""
    idx = sum(spec.out_features * spec.nvec * b / 8.0 for b in spec.log2k)
    books = sum((1 << b) * spec.d * 2 for b in spec.log2k)
    affine = 2 * spec.out_features * (int(spec.scale_range is not None) + int(spec.bias_std is not None))
    return idx + books + affine + 2.0 * batch * spec.in_features + 2.0 * batch * spec.out_features


# -- distributed plumbing (timing only; no collective on the data path) ------

# The lookup-table GEMV's own attainable bound (2^16 book, d = 8, batch 1,
# tiled order): its two phases run one after the other on every SM.
#  - Table products: every (group of four vectors, slice) task streams its
#    slice of the codebook from L2 into the SM, so each layer moves the whole
#    book once per group; at best at the 31 TB/s that 148 SMs reading one
#    1 MiB buffer with coalesced 16-byte loads reach (probe; 24 TB/s low end).
#  - Lookups: every index is examined once per slice (LUT_SLICES), each
#    examination at least a field extract, the slice subtraction, the range
#    compare and one shared-memory load (4 instructions) at 4 warp
#    instructions per clock per SM; the HBM read of the index stream at the
#    measured copy bandwidth overlaps with it.
LUT_SLICES = 3
LUT_L2_TBS = (24.0, 31.0)
LUT_MIN_INSTR_PER_EXAM = 4
SM_COUNT = 148
SM_MAX_GHZ = 1.965


def lut_design_bound(specs, peak_hbm_gbs: float) -> dict:
    """Microseconds the table design cannot beat for one launch over `specs`
    (layers sharing x, batch 1)."""
    book_bytes = exams = 0
    for sp in specs:
        nvec = -(-sp.in_features // sp.d)
        groups = -(-nvec // 4)
        book_bytes += groups * (1 << sp.log2k[0]) * sp.d * 2
        exams += sp.out_features * nvec * LUT_SLICES
    a_us = [book_bytes / (tbs * 1e12) * 1e6 for tbs in LUT_L2_TBS]
    b_issue_us = exams * LUT_MIN_INSTR_PER_EXAM / 32 / (SM_COUNT * 4 * SM_MAX_GHZ * 1e9) * 1e6
    hbm_us = sum(alg_bytes(sp, 1) for sp in specs) / (peak_hbm_gbs * 1e9) * 1e6
    b_us = max(b_issue_us, hbm_us)
    return {"bound_us": a_us[1] + b_us, "bound_us_at_24tbs": a_us[0] + b_us,
            "codebook_l2_bytes": book_bytes, "table_phase_us": a_us[1],
            "slice_examinations": exams, "lookup_phase_issue_us": b_issue_us, "hbm_us": hbm_us}


def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init_dist(world: int, backend: str):
    if world <= 1:
        return None
    import torch.distributed as dist
    dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist


def reduce_max(value: float, dist_mod, device=None) -> float:
    """Max of a per-rank float over all ranks (identity on one rank)."""
    if dist_mod is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist_mod.all_reduce(t, op=dist_mod.ReduceOp.MAX)
    return float(t.item())


def whole_job_value(bytes_per_step: float, steps: int, world: int, ms_total_max: float) -> float:
    """GB/s of the whole job: every rank moves bytes_per_step per step; the
    time is the slowest rank's timed region."""
    return bytes_per_step * steps * world / (ms_total_max * 1e-3) / 1e9


def barrier(dist_mod, device=None):
    if dist_mod is not None:
        if device is not None:
            dist_mod.barrier(device_ids=[device.index])
        else:
            dist_mod.barrier()


# -- clocks during the timed region ------------------------------------------

class ClockSampler:
    """nvidia-smi clock / throttle-reason samples every 50 ms while active."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu = gpu_id
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.1)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        return False

    def summary(self):
        rows = []
        try:
            with open(self.path) as fh:
                for ln in fh:
                    parts = [p.strip() for p in ln.split(",")]
                    if len(parts) >= 9 and parts[1].replace(".", "").isdigit():
                        rows.append(parts)
        finally:
            if self.path and os.path.exists(self.path):
                os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        sm = [float(r[1]) for r in rows]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": float(rows[0][2]),
                "reasons": reasons, "samples": len(rows),
                "power_w_max": max(float(r[3]) for r in rows if r[3].replace(".", "").isdigit())}


# -- the oracle on the host (reference arm and cpu_baseline) ------------------

def oracle_rate(target_s: float, spec_seed_pairs, x_list):
    """Run the CPU oracle on a growing sample of output rows of the decode
    layers until one pass takes about target_s; return (GB/s, rows, seconds,
    threads).  Bytes are the algorithmic bytes of the rows processed."""
    import oracle
    datas = [synth.make_layer(spec, seed) for spec, seed in spec_seed_pairs]
    rows = 16
    while True:
        t0 = time.perf_counter()
        nbytes = 0.0
        for data, x in zip(datas, x_list):
            r = min(rows, data.spec.out_features)
            oracle.linear(data, x, rows=np.arange(r))
            nbytes += alg_bytes(data.spec, x.shape[0]) * r / data.spec.out_features
        dt = time.perf_counter() - t0
        if dt >= target_s or rows >= max(d.spec.out_features for d in datas):
            return nbytes / dt / 1e9, min(rows, max(d.spec.out_features for d in datas)), dt, \
                oracle.num_threads()
        rows = int(rows * min(8.0, max(1.5, 1.2 * target_s / max(dt, 1e-3))))


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    w = WORKLOADS[DECODE]
    xs = [synth.make_x(w.x_seed + i, BATCH, spec.in_features, w.outlier_frac)
          for i, (spec, _) in enumerate(w.layers)]
    per_step = max(0.02, min(6.0, 120.0 / max(1, args.steps + args.warmup)))
    gbs, rows, dt, cores = oracle_rate(per_step, w.layers, xs)
    import oracle
    datas = [synth.make_layer(spec, seed) for spec, seed in w.layers]
    for _ in range(args.warmup):
        for d, x in zip(datas, xs):
            oracle.linear(d, x, rows=np.arange(min(rows, d.spec.out_features)))
    t0 = time.perf_counter()
    nbytes = 0.0
    for _ in range(args.steps):
        for d, x in zip(datas, xs):
            r = min(rows, d.spec.out_features)
            oracle.linear(d, x, rows=np.arange(r))
            nbytes += alg_bytes(d.spec, BATCH) * r / d.spec.out_features
    dt = time.perf_counter() - t0
    value = nbytes / dt / 1e9
    sample = (f"first min({rows}, N) output rows of each of gate/up/down (B=1) per step, "
              f"oracle dequantise + fp64 dot products")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt / max(1, args.steps) * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": decode_config(),
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def decode_config():
    w = WORKLOADS[DECODE]
    return {
        "workload": "llama3_70b_mlp decode, B=1: gate_proj + up_proj 28672x8192, down_proj "
                    "8192x28672; d=8, one K=2^16 fp16 codebook (2.0 bpw), fp16 scale/bias",
        "batch": BATCH, "layers": [s.name for s, _ in w.layers], "bpw": 2.0,
        "index_order": dict(zip([s.name for s, _ in w.layers], LAYOUTS)),
        "x": "bf16 ~N(0,1), 0.1% outlier columns x20; gate_proj and up_proj read the same x",
        "l2": "inputs larger than L2: two copies of the three layers (352 MB of indices) used in turn",
        "parallelism": "replicas (each rank runs its own step; no collective on the data path)",
    }


# -- the GPU arm ----------------------------------------------------------------

def run_gpu(args):
    import torch
    from bit_packed_index_b200 import vq

    rank, world, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the CPU oracle runs with --impl reference)")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist_mod = init_dist(world, "nccl")
    peaks, peak_src = load_peaks()

    w = WORKLOADS[DECODE]
    specs = [s for s, _ in w.layers]
    copies = []
    for c in range(2):
        layers = []
        for (spec, seed), lay in zip(w.layers, LAYOUTS):
            layers.append(vq.Layer.from_synth(synth.make_layer(spec, seed + 1000 * c + 17 * rank), dev,
                                              layout=lay))
        copies.append(layers)
    # gate_proj and up_proj read the same x (the block's input); down_proj its own.
    xs_host = [synth.make_x(w.x_seed, BATCH, specs[0].in_features, w.outlier_frac),
               synth.make_x(w.x_seed + 2, BATCH, specs[2].in_features, w.outlier_frac)]
    xs = [torch.from_numpy(x.view(np.int16)).to(dev).view(torch.bfloat16) for x in xs_host]
    ys = [torch.empty((BATCH, s.out_features), dtype=torch.bfloat16, device=dev) for s in specs]
    need_gu = max(vq.gemv_multi_workspace_size(copies[c][:2], BATCH) for c in range(2))
    need_d = max(vq.gemv_workspace_size(copies[c][2], BATCH) for c in range(2))
    ws = [torch.empty(max(need_gu, 256), dtype=torch.uint8, device=dev),
          torch.empty(max(need_d, 256), dtype=torch.uint8, device=dev)]
    step_bytes = sum(alg_bytes(s, BATCH) for s in specs)

    def run_step(layers, x_gu, x_d, y_gu, y_d, events=None):
        """gate_proj + up_proj as one vq_gemv_multi call, then down_proj."""
        if events is not None:
            events[0][0].record()
        vq.gemv_multi(layers[:2], x_gu, outs=y_gu, workspace=ws[0])
        if events is not None:
            events[0][1].record()
            events[1][0].record()
        vq.gemv(layers[2], x_d, out=y_d, workspace=ws[1])
        if events is not None:
            events[1][1].record()

    def step(i, events=None):
        run_step(copies[i & 1], xs[0], xs[1], ys[:2], ys[2], events)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()

    evs = [[[torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)]
            for _ in range(2)] for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    uuid = str(getattr(torch.cuda.get_device_properties(local), "uuid", "") or "")
    gpu_id = ("GPU-" + uuid) if uuid and not uuid.startswith("GPU-") else (uuid or str(local))
    with ClockSampler(gpu_id) as clocks:
        barrier(dist_mod, dev)
        torch.cuda.synchronize()
        launches0 = vq.kernel_launches()
        t_start.record()
        for i in range(args.steps):
            step(i, evs[i])
        t_end.record()
        torch.cuda.synchronize()
        launches = vq.kernel_launches() - launches0
        barrier(dist_mod, dev)
    ms_total = reduce_max(t_start.elapsed_time(t_end), dist_mod, dev)
    ms_step = ms_total / args.steps
    value = whole_job_value(step_bytes, args.steps, world, ms_total)

    # Live roofline of the dominant kernel, the lookup-table GEMV, on its
    # fused gate_proj + up_proj launches (the workload of the committed ncu
    # capture): algorithmic bytes of one call / mean call time from CUDA
    # events on the launching stream.  A call is the table kernel plus its
    # per-block-sum reduction, so the figure slightly understates the kernel.
    call_ms = [statistics.mean(evs[i][k][0].elapsed_time(evs[i][k][1]) for i in range(args.steps))
               for k in range(2)]
    gu_bytes = alg_bytes(specs[0], BATCH) + alg_bytes(specs[1], BATCH)
    achieved = gu_bytes / (call_ms[0] * 1e-3) / 1e9
    rec = profiled_traffic("gemv_lut_kernel")
    lut_bound = lut_design_bound(specs[:2], peaks["hbm_gbs"])
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"],
                "traffic": rec["dram_bytes_per_launch"] if rec else None,
                "algorithmic_bytes_per_launch": gu_bytes,
                "kernel": "gemv_lut_kernel (+ gemv_lut_finalize)",
                "launch": "gate_proj + up_proj (2 x 28672x8192) in one vq_gemv_multi launch, B=1, "
                          "tiled index order",
                "peak_source": peak_src + " (HBM copy, kernel timed alone)",
                "per_call_us": {"gate_proj+up_proj": call_ms[0] * 1e3, "down_proj": call_ms[1] * 1e3},
                "frac_of_nominal_8tbs": achieved / NOMINAL_HBM_GBS,
                "row_order_gather_ceiling_us": 120.0,
                "design_bound": dict(lut_bound, frac=lut_bound["bound_us"] / (call_ms[0] * 1e3)),
                "note": "not HBM-bound: the table kernel is bound by instruction issue and "
                        "shared-memory lookups (3 slice tests per index), the row-order kernel "
                        "by random 16-byte centroid gathers through L1/L2 (0.84/clk/SM); "
                        "design_bound: the table design's own floor (codebook slices streamed "
                        "from L2 at 31 TB/s, then 4 instructions per slice examination of an "
                        "index or the HBM read, whichever is longer) and the fraction of it "
                        "the measured call reaches"}

    # e2e through the public API with pinned host activations and outputs:
    # each step copies all three layers' inputs to the device in one transfer,
    # runs the layers, and copies all outputs back in one transfer.
    xcat = np.concatenate([x.reshape(-1) for x in xs_host])
    xh = torch.from_numpy(xcat.view(np.int16)).view(torch.bfloat16).pin_memory()
    xd = torch.empty_like(xh, device=dev)
    xoff = np.cumsum([0] + [x.size for x in xs_host])
    xv = [xd[xoff[k]:xoff[k + 1]].view(BATCH, -1) for k in range(2)]
    ycat = sum(BATCH * s.out_features for s in specs)
    yh = torch.empty(ycat, dtype=torch.bfloat16).pin_memory()
    yd = torch.empty(ycat, dtype=torch.bfloat16, device=dev)
    yoff = np.cumsum([0] + [BATCH * s.out_features for s in specs])
    yv = [yd[yoff[k]:yoff[k + 1]].view(BATCH, -1) for k in range(3)]

    def e2e_step(i):
        xd.copy_(xh, non_blocking=True)
        run_step(copies[i & 1], xv[0], xv[1], yv[:2], yv[2])
        yh.copy_(yd, non_blocking=True)

    for i in range(args.warmup):
        e2e_step(i)
    torch.cuda.synchronize()
    barrier(dist_mod, dev)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for i in range(args.steps):
        e2e_step(i)
    b.record()
    torch.cuda.synchronize()
    barrier(dist_mod, dev)
    e2e_ms = reduce_max(a.elapsed_time(b), dist_mod, dev)
    e2e = {"value": whole_job_value(step_bytes, args.steps, world, e2e_ms), "unit": "GB/s",
           "h2d_bytes_per_step": xh.numel() * 2,
           "d2h_bytes_per_step": yh.numel() * 2,
           "ms_per_step": e2e_ms / args.steps}

    gemm = run_gemm(dev, peaks, peak_src, vq)
    sweep = run_sweep(dev, peaks, peak_src, vq, copies[0])
    decode_405b = run_decode_405b(dev, peaks, peak_src, vq)
    qkv_405b = run_405b_qkv(dev, peaks, peak_src, vq)
    rht = run_rht(dev, vq)
    hess = run_hessian(dev, peaks, peak_src, vq)
    encode = run_encode(dev, peaks, peak_src, vq,
                        with_oracle=rank == 0 and world == 1 and not args.no_cpu_baseline)
    encode_h = run_encode(dev, peaks, peak_src, vq,
                          with_oracle=rank == 0 and world == 1 and not args.no_cpu_baseline, hessian=True)

    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": decode_config(),
        "us_per_layer": ms_step * 1e3 / 3,
        "hbm_pct_of_measured": 100.0 * value / world / peaks["hbm_gbs"],
        "hbm_pct_of_nominal_8tbs": 100.0 * value / world / NOMINAL_HBM_GBS,
        "roofline": roofline,
        "e2e": e2e,
        "gpu_launches": int(launches),
        "clocks": clocks.summary(),
        "gemm": gemm,
        "sweep": sweep,
        "decode_405b_gate": decode_405b,
        "decode_405b_qkv": qkv_405b,
        "rht_gate": rht,
        "hessian": hess,
        "encode": encode,
        "encode_h": encode_h,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        gbs, rows, dt, cores = oracle_rate(10.0, w.layers, xs_host)
        line["cpu_baseline"] = {"value": gbs, "unit": "GB/s", "cores": cores, "kind": "oracle",
                                "sample": f"first min({rows}, N) output rows of each of gate/up/down "
                                          f"(B=1), {dt:.1f} s of oracle work"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist_mod is not None:
        dist_mod.destroy_process_group()
    return 0


def run_gemm(dev, peaks, peak_src, vq):
    """Prefill GEMM through vq_gemm, L2 flushed between timed calls."""
    import torch
    w = WORKLOADS[PREFILL]
    spec, seed = w.layers[0]
    layer = vq.Layer.from_synth(synth.make_layer(spec, seed), dev)
    x = torch.from_numpy(synth.make_x(w.x_seed, PREFILL_M, spec.in_features).view(np.int16)).to(dev)
    x = x.view(torch.bfloat16)
    y = torch.empty((PREFILL_M, spec.out_features), dtype=torch.bfloat16, device=dev)
    wsp = torch.empty(vq.gemm_workspace_size(layer, PREFILL_M), dtype=torch.uint8, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for _ in range(3):
        vq.gemm(layer, x, out=y, workspace=wsp)
    times = []
    for _ in range(10):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        vq.gemm(layer, x, out=y, workspace=wsp)
        b.record()
        b.synchronize()
        times.append(a.elapsed_time(b))
    torch.cuda.synchronize()
    status = int(wsp[:4].view(torch.int32).item())
    ms = statistics.median(times)
    flops = 2.0 * PREFILL_M * spec.out_features * spec.in_features
    tf = flops / (ms * 1e-3) / 1e12
    return {"workload": f"prefill_8192: x [{PREFILL_M},8192] bf16, W 8192x8192, d=8, K=2^16 + "
                        f"residual K=2^8 (3.0 bpw), fp16 operands, fp32 accumulate, bf16 out",
            "tflops": tf, "us": ms * 1e3, "device_status": status,
            "roofline": {"bound": "tensor", "achieved": tf, "peak": peaks["bf16_tflops"],
                         "unit": "TFLOP/s", "frac": tf / peaks["bf16_tflops"],
                         "peak_source": peak_src + " (bf16 burst; fp16 nominal rate is the same)"}}


def _median_us(fn, flush, reps=10, warm=3):
    """Median time of fn() in microseconds from CUDA events on the current
    stream, a 256 MB write between calls (L2 flushed), after warm-up calls."""
    import torch
    for _ in range(warm):
        fn()
    ts = []
    for _ in range(reps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        b.synchronize()
        ts.append(a.elapsed_time(b))
    return statistics.median(ts) * 1e3


def run_sweep(dev, peaks, peak_src, vq, layers70):
    """Every configuration of the measurement plan beside the headline, one
    call each, L2 flushed between calls: the decode GEMV per layer and batch
    (both index orders where the planner's kernels differ; the faster is
    reported first) and the prefill GEMM at the other row counts.  Decode:
    us, algorithmic GB/s and the fraction of the measured HBM peak; prefill:
    us, TFLOP/s and the fraction of the measured bf16 burst peak."""
    import torch
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    hbm = peaks["hbm_gbs"]
    out = {"protocol": "median of 10 calls, CUDA events, a 256 MB write between calls (L2 flushed)",
           "peak_source": peak_src, "decode": [], "prefill": []}

    def decode_entry(name, spec, layers_by_order, batches, x_seed, outlier):
        for bsz in batches:
            x = torch.from_numpy(synth.make_x(x_seed, bsz, spec.in_features, outlier).view(np.int16)).to(dev)
            x = x.view(torch.bfloat16)
            y = torch.empty((bsz, spec.out_features), dtype=torch.bfloat16, device=dev)
            res = {}
            for order, layer in layers_by_order.items():
                ws = torch.empty(max(256, vq.gemv_workspace_size(layer, bsz)), dtype=torch.uint8, device=dev)
                res[order] = _median_us(lambda: vq.gemv(layer, x, out=y, workspace=ws), flush)
                del ws
            best = min(res, key=res.get)
            gbs = alg_bytes(spec, bsz) / (res[best] * 1e-6) / 1e9
            out["decode"].append({"workload": name, "batch": bsz, "us": res[best], "index_order": best,
                                  "us_by_order": res, "gbs": gbs, "frac_of_measured_hbm": gbs / hbm})

    # tiny 512 x 512, one 2^16 book, B = 1
    w = WORKLOADS["tiny_512"]
    spec, seed = w.layers[0]
    rows = vq.Layer.from_synth(synth.make_layer(spec, seed), dev)
    decode_entry("tiny_512 512x512, d=8, K=2^16 (2.0 bpw)", spec,
                 {"rows": rows, "tile4": vq.repack_tile4(rows)}, (1,), w.x_seed, 0.0)
    # Llama-3-8B up_proj, 2^12 + 2^8 books, B in {1, 4, 16}
    w = WORKLOADS["llama3_8b_up"]
    spec, seed = w.layers[0]
    rows = vq.Layer.from_synth(synth.make_layer(spec, seed), dev)
    decode_entry("llama3_8b_up 14336x4096, d=8, K=2^12 + 2^8 (2.5 bpw)", spec,
                 {"rows": rows, "tile4": vq.repack_tile4(rows)}, (1, 4, 16), w.x_seed, 0.0)
    del rows
    # Llama-3-70B MLP layers (the step's tiled layers), B in {2, 8, 16}
    w = WORKLOADS[DECODE]
    for (spec, _), layer in zip(w.layers, layers70):
        if spec.name == "up_proj":
            continue                                    # the same shape as gate_proj
        decode_entry(f"llama3_70b {spec.name} {spec.out_features}x{spec.in_features}, d=8, K=2^16 (2.0 bpw)",
                     spec, {layer.layout: layer}, (2, 8, 16), w.x_seed, w.outlier_frac)
    # Llama-3.1-405B gate_proj, 2^12 + 2^4 books at d = 6, B in {2, 4, 8, 16}
    w = WORKLOADS["llama31_405b"]
    spec, seed = w.layers[4]
    rows = vq.Layer.from_synth(synth.make_layer(spec, seed), dev)
    decode_entry("llama31_405b gate_proj 53248x16384, d=6, K=2^12 + 2^4 (2.67 bpw)", spec,
                 {"rows": rows, "tile4": vq.repack_tile4(rows)}, (2, 4, 8, 16), w.x_seed + 4, 0.0)

    def prefill_entry(name, spec, layer, m, x_seed):
        x = torch.from_numpy(synth.make_x(x_seed, m, spec.in_features).view(np.int16)).to(dev).view(torch.bfloat16)
        y = torch.empty((m, spec.out_features), dtype=torch.bfloat16, device=dev)
        ws = torch.empty(vq.gemm_workspace_size(layer, m), dtype=torch.uint8, device=dev)
        us = _median_us(lambda: vq.gemm(layer, x, out=y, workspace=ws), flush)
        torch.cuda.synchronize()
        tf = 2.0 * m * spec.out_features * spec.in_features / (us * 1e-6) / 1e12
        out["prefill"].append({"workload": name, "m": m, "us": us, "tflops": tf,
                               "frac_of_measured_bf16": tf / peaks["bf16_tflops"],
                               "device_status": int(ws[:4].view(torch.int32).item())})

    # the 405B gate_proj at prefill M = 1024 (the layer above), then q_proj
    prefill_entry("llama31_405b gate_proj 53248x16384, M=1024", spec, rows, 1024, w.x_seed + 4)
    del rows
    qspec, qseed = w.layers[0]
    q = vq.Layer.from_synth(synth.make_layer(qspec, qseed), dev)
    prefill_entry("llama31_405b q_proj 16384x16384, M=1024", qspec, q, 1024, w.x_seed)
    del q
    # prefill 8192 x 8192 (2^16 + 2^8) at M = 512 and 4096 (2048 is the gemm object)
    w = WORKLOADS[PREFILL]
    spec, seed = w.layers[0]
    layer = vq.Layer.from_synth(synth.make_layer(spec, seed), dev)
    for m in (512, 4096):
        prefill_entry(f"prefill_8192 8192x8192, K=2^16 + 2^8 (3.0 bpw), M={m}", spec, layer, m, w.x_seed)
    del layer, flush
    torch.cuda.empty_cache()
    return out


def run_decode_405b(dev, peaks, peak_src, vq):
    """Beside the headline: the Llama-3.1-405B gate_proj (53248 x 16384, d = 6,
    K = 2^12 + 2^4, 2.67 bpw) at batch 1 in the tiled order, where the
    small-book lookup-table kernel runs; L2 flushed between timed calls."""
    import torch
    w = WORKLOADS["llama31_405b"]
    spec, seed = w.layers[4]
    layer = vq.Layer.from_synth(synth.make_layer(spec, seed), dev, layout="tile4")
    x = torch.from_numpy(synth.make_x(w.x_seed + 4, 1, spec.in_features).view(np.int16)).to(dev)
    x = x.view(torch.bfloat16)
    y = torch.empty((1, spec.out_features), dtype=torch.bfloat16, device=dev)
    ws = torch.empty(max(256, vq.gemv_workspace_size(layer, 1)), dtype=torch.uint8, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for _ in range(3):
        vq.gemv(layer, x, out=y, workspace=ws)
    times = []
    for _ in range(20):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        vq.gemv(layer, x, out=y, workspace=ws)
        b.record()
        b.synchronize()
        times.append(a.elapsed_time(b))
    ms = statistics.median(times)
    gbs = alg_bytes(spec, 1) / (ms * 1e-3) / 1e9
    return {"workload": "llama31_405b gate_proj 53248x16384, d=6, K=2^12 + residual K=2^4 (2.67 bpw), "
                        "B=1, tiled index order (small-book lookup-table kernel)",
            "us": ms * 1e3, "achieved_gbs": gbs, "frac_of_measured_hbm": gbs / peaks["hbm_gbs"],
            "algorithmic_bytes": alg_bytes(spec, 1), "peak_source": peak_src}


def run_405b_qkv(dev, peaks, peak_src, vq):
    """Beside the headline: the Llama-3.1-405B q/k/v projections (16384, 1024
    and 1024 rows x 16384, d = 6, K = 2^12 + 2^4) reading the same x, tiled, as
    one vq_gemv_multi call; L2 flushed between timed calls."""
    import torch
    w = WORKLOADS["llama31_405b"]
    specs = [w.layers[li][0] for li in (0, 1, 2)]
    layers = [vq.Layer.from_synth(synth.make_layer(*w.layers[li]), dev, layout="tile4") for li in (0, 1, 2)]
    x = torch.from_numpy(synth.make_x(w.x_seed, 1, specs[0].in_features).view(np.int16)).to(dev)
    x = x.view(torch.bfloat16)
    outs = [torch.empty((1, s.out_features), dtype=torch.bfloat16, device=dev) for s in specs]
    ws = torch.empty(max(256, vq.gemv_multi_workspace_size(layers, 1)), dtype=torch.uint8, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for _ in range(3):
        vq.gemv_multi(layers, x, outs=outs, workspace=ws)
    times = []
    for _ in range(20):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        vq.gemv_multi(layers, x, outs=outs, workspace=ws)
        b.record()
        b.synchronize()
        times.append(a.elapsed_time(b))
    ms = statistics.median(times)
    nbytes = sum(alg_bytes(s, 1) for s in specs)
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"workload": "llama31_405b q_proj + k_proj + v_proj (16384/1024/1024 x 16384), d=6, "
                        "K=2^12 + residual K=2^4, B=1, tiled, one vq_gemv_multi call",
            "us": ms * 1e3, "achieved_gbs": gbs, "frac_of_measured_hbm": gbs / peaks["hbm_gbs"],
            "algorithmic_bytes": nbytes, "peak_source": peak_src}


def run_encode(dev, peaks, peak_src, vq, with_oracle: bool, hessian: bool = False):
    """Beside the headline: the nearest-centroid encoder (vq_encode) on a
    4096 x 4096 fp16 matrix against one K = 2^16, d = 8 book (2M vectors x
    65536 centroids), L2 flushed between timed calls; the oracle's brute force
    on a sample of the same vectors for scale.  With ``hessian`` the
    Hessian-weighted distance, H from vq_hessian of synthetic activations."""
    import torch
    n, kin, d, log2k = ENCODE_SHAPE
    w, books = synth.make_encode_input(n, kin, d, log2k, ENCODE_STD, seed=ENCODE_SEED)
    W = torch.from_numpy(w.view(np.int16)).to(dev).view(torch.float16)
    B = [torch.from_numpy(b.view(np.int16)).to(dev).view(torch.float16) for b in books]
    H = None
    if hessian:
        xt = synth.make_x(ENCODE_H_SEED, ENCODE_H_TOKENS, kin, 0.001)
        H = vq.hessian(torch.from_numpy(xt.view(np.int16)).to(dev).view(torch.bfloat16))
    ws = torch.empty(vq.encode_workspace_size(n, kin, log2k, d, hessian=hessian), dtype=torch.uint8, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for _ in range(3):
        vq.encode(W, B, log2k, d, workspace=ws, hessian=H)
    times = []
    for _ in range(5):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        vq.encode(W, B, log2k, d, workspace=ws, hessian=H)
        b.record()
        b.synchronize()
        times.append(a.elapsed_time(b))
    ctrl = ws[:16].view(torch.int32).cpu().numpy()
    ms = statistics.median(times)
    nv = n * (kin // d)
    pairs = nv * sum(1 << b for b in log2k)
    rate = pairs / (ms * 1e-3)
    # ALU roofline: one minimum operation per (vector, centroid) pair at full
    # issue on every SM sub-partition (148 SMs x 4 x 32 lanes x max SM clock).
    alu_peak = 148 * 4 * 32 * 1.965e9
    what = ("Hessian-weighted (v-c)^T H_v (v-c), H of 1024 synthetic tokens with 0.1% outlier channels, "
            if hessian else "")
    out = {"workload": f"encode {what}{n}x{kin} fp16 W ~ N(0, {ENCODE_STD[0]}), d={d}, one K=2^{log2k[0]} book: "
                       f"{nv} vectors x {1 << log2k[0]} centroids",
           "ms": ms, "pairs_per_s": rate, "device_status": int(ctrl[0]),
           "exact_pass_vectors": int(ctrl[1]), "exact_pass_share": int(ctrl[1]) / nv,
           "roofline": {"bound": "alu", "achieved": rate, "peak": alu_peak, "unit": "pairs/s",
                        "frac": rate / alu_peak,
                        "peak_source": "derived: one ALU operation per pair at full issue, "
                                       "148 SMs x 128 lanes x 1965 MHz"},
           "tensor_tflops": 2.0 * (2 * d if hessian else d) * pairs / (ms * 1e-3) / 1e12}
    if hessian:
        out["roofline"]["note"] = ("the weighted epilogue spends two operations per pair (an fma adding "
                                   "c^T H_j c, then the minimum), so 0.5 of this peak is its ceiling")
    if not with_oracle:
        return out
    # CPU baseline: the oracle on a bounded sample of the same vectors (host cores)
    import oracle
    import time as _time
    sample = 256 if not hessian else 64
    v = oracle.f16_to_f32(w[:sample * d // kin + 1]).astype(np.float64).reshape(-1, d)[:sample]
    t0 = _time.perf_counter()
    if hessian:
        hb = oracle.hessian_blocks(H.double().cpu().numpy(), kin, d, sample * d // kin + 1)[0][:sample]
        t0 = _time.perf_counter()
        oracle.encode_h(v, hb, books[0])
    else:
        oracle.encode(v, books[0])
    dt = _time.perf_counter() - t0
    out["cpu_baseline"] = {"value": sample * (1 << log2k[0]) / dt, "unit": "pairs/s",
                           "cores": oracle.num_threads(), "kind": "oracle",
                           "sample": f"{sample} vectors x {1 << log2k[0]} centroids, {dt:.2f} s"}
    return out


def run_rht(dev, vq):
    """Beside the headline: the 70B gate_proj (tiled) in the rotated basis of
    QuIP#-style incoherence processing, y = U^T (W~ (V x)) through
    vq_gemv_rht, against the same layer through vq_gemv; L2 flushed."""
    import torch
    w = WORKLOADS[DECODE]
    spec, seed = w.layers[0]
    layer = vq.Layer.from_synth(synth.make_layer(spec, seed), dev, layout="tile4")
    x = torch.from_numpy(synth.make_x(w.x_seed, 1, spec.in_features, w.outlier_frac).view(np.int16)).to(dev)
    x = x.view(torch.bfloat16)
    rng = np.random.default_rng(RHT_SEED)
    s_in = torch.from_numpy(rng.integers(0, 2**31, size=(spec.in_features + 31) // 32, dtype=np.int64)
                            .astype(np.int32)).to(dev)
    s_out = torch.from_numpy(rng.integers(0, 2**31, size=(spec.out_features + 31) // 32, dtype=np.int64)
                             .astype(np.int32)).to(dev)
    y = torch.empty((1, spec.out_features), dtype=torch.bfloat16, device=dev)
    ws = torch.empty(max(256, vq.gemv_workspace_size(layer, 1)), dtype=torch.uint8, device=dev)
    wr = torch.empty(vq.gemv_rht_workspace_size(layer, 1), dtype=torch.uint8, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def med(fn):
        for _ in range(3):
            fn()
        ts = []
        for _ in range(20):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            b.synchronize()
            ts.append(a.elapsed_time(b))
        return statistics.median(ts) * 1e3

    plain = med(lambda: vq.gemv(layer, x, out=y, workspace=ws))
    rot = med(lambda: vq.gemv_rht(layer, s_in, s_out, x, out=y, workspace=wr))
    return {"workload": "llama3_70b_mlp gate_proj 28672x8192, tiled, B=1, in the rotated basis "
                        "(blocks of 8192 on x, 4096 on y)",
            "us": rot, "us_without_rotation": plain, "rotation_overhead_us": rot - plain,
            "achieved_gbs": alg_bytes(spec, 1) / (rot * 1e-6) / 1e9}


def run_hessian(dev, peaks, peak_src, vq):
    """Beside the headline: the Hessian of a layer's inputs (vq_hessian) for
    8192 bf16 activation tokens of 8192 features (X ~ N(0, 1), 0.1 % outlier
    columns x20), in TFLOP/s of the X^T X contraction."""
    import torch
    n, d = HESSIAN_SHAPE
    x = synth.make_x(HESSIAN_SEED, n, d, 0.001)
    xd = torch.from_numpy(x.view(np.int16)).to(dev).view(torch.bfloat16)
    out = torch.empty((d, d), dtype=torch.float32, device=dev)
    ws = torch.empty(max(256, vq.hessian_workspace_size(n, d)), dtype=torch.uint8, device=dev)
    for _ in range(3):
        vq.hessian(xd, out=out, workspace=ws)
    times = []
    for _ in range(10):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        vq.hessian(xd, out=out, workspace=ws)
        b.record()
        b.synchronize()
        times.append(a.elapsed_time(b))
    ms = statistics.median(times)
    tf = 2.0 * n * d * d / (ms * 1e-3) / 1e12
    return {"workload": f"hessian: {n} bf16 tokens x {d} features -> fp32 [{d}][{d}]",
            "ms": ms, "tflops": tf, "device_status": int(ws[:4].view(torch.int32).item()),
            "roofline": {"bound": "tensor", "achieved": tf, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": tf / peaks["bf16_tflops"], "peak_source": peak_src + " (bf16 burst)"}}


def run_profile(args):
    """A few launches of one call on its bench workload, nothing timed: the
    command the committed ncu summaries were captured from."""
    import torch
    from bit_packed_index_b200 import vq
    dev = torch.device("cuda", 0)
    if args.profile == "hessian":
        n, d = HESSIAN_SHAPE
        x = torch.from_numpy(synth.make_x(HESSIAN_SEED, n, d, 0.001).view(np.int16)).to(dev).view(torch.bfloat16)
        out = torch.empty((d, d), dtype=torch.float32, device=dev)
        ws = torch.empty(vq.hessian_workspace_size(n, d), dtype=torch.uint8, device=dev)
        for _ in range(args.profile_launches):
            vq.hessian(x, out=out, workspace=ws)
    elif args.profile == "encode":
        n, kin, d, log2k = ENCODE_SHAPE
        w, books = synth.make_encode_input(n, kin, d, log2k, ENCODE_STD, seed=ENCODE_SEED)
        W = torch.from_numpy(w.view(np.int16)).to(dev).view(torch.float16)
        B = [torch.from_numpy(b.view(np.int16)).to(dev).view(torch.float16) for b in books]
        ws = torch.empty(vq.encode_workspace_size(n, kin, log2k, d), dtype=torch.uint8, device=dev)
        for _ in range(args.profile_launches):
            vq.encode(W, B, log2k, d, workspace=ws)
    elif args.profile == "lut_gateup":
        w = WORKLOADS[DECODE]
        layers = [vq.Layer.from_synth(synth.make_layer(*w.layers[li]), dev, layout="tile4") for li in (0, 1)]
        x = torch.from_numpy(synth.make_x(w.x_seed, BATCH, layers[0].in_features, w.outlier_frac)
                             .view(np.int16)).to(dev).view(torch.bfloat16)
        outs = [torch.empty((BATCH, l.out_features), dtype=torch.bfloat16, device=dev) for l in layers]
        ws = torch.empty(vq.gemv_multi_workspace_size(layers, BATCH), dtype=torch.uint8, device=dev)
        for _ in range(args.profile_launches):
            vq.gemv_multi(layers, x, outs=outs, workspace=ws)
    elif args.profile in ("tc_gate16", "tcs_q16", "tcs_8b16"):
        # batch-16 decode on the tensor cores, tiled order: the 70B gate_proj
        # (2^16 book), the 405B q_proj and the 8B up_proj (small books)
        name, li = {"tc_gate16": (DECODE, 0), "tcs_q16": ("llama31_405b", 0),
                    "tcs_8b16": ("llama3_8b_up", 0)}[args.profile]
        w = WORKLOADS[name]
        spec, seed = w.layers[li]
        layer = vq.Layer.from_synth(synth.make_layer(spec, seed), dev, layout="tile4")
        x = torch.from_numpy(synth.make_x(w.x_seed, 16, spec.in_features, w.outlier_frac)
                             .view(np.int16)).to(dev).view(torch.bfloat16)
        out = torch.empty((16, spec.out_features), dtype=torch.bfloat16, device=dev)
        ws = torch.empty(max(256, vq.gemv_workspace_size(layer, 16)), dtype=torch.uint8, device=dev)
        for _ in range(args.profile_launches):
            vq.gemv(layer, x, out=out, workspace=ws)
    elif args.profile == "encode_h":
        n, kin, d, log2k = ENCODE_SHAPE
        w, books = synth.make_encode_input(n, kin, d, log2k, ENCODE_STD, seed=ENCODE_SEED)
        W = torch.from_numpy(w.view(np.int16)).to(dev).view(torch.float16)
        B = [torch.from_numpy(b.view(np.int16)).to(dev).view(torch.float16) for b in books]
        xt = synth.make_x(ENCODE_H_SEED, ENCODE_H_TOKENS, kin, 0.001)
        H = vq.hessian(torch.from_numpy(xt.view(np.int16)).to(dev).view(torch.bfloat16))
        ws = torch.empty(vq.encode_workspace_size(n, kin, log2k, d, hessian=True), dtype=torch.uint8, device=dev)
        for _ in range(args.profile_launches):
            vq.encode(W, B, log2k, d, workspace=ws, hessian=H)
    elif args.profile == "rht_gate":
        w = WORKLOADS[DECODE]
        spec, seed = w.layers[0]
        layer = vq.Layer.from_synth(synth.make_layer(spec, seed), dev, layout="tile4")
        x = torch.from_numpy(synth.make_x(w.x_seed, 1, spec.in_features, w.outlier_frac)
                             .view(np.int16)).to(dev).view(torch.bfloat16)
        rng = np.random.default_rng(RHT_SEED)
        s_in = torch.from_numpy(rng.integers(0, 2**31, size=(spec.in_features + 31) // 32, dtype=np.int64)
                                .astype(np.int32)).to(dev)
        s_out = torch.from_numpy(rng.integers(0, 2**31, size=(spec.out_features + 31) // 32, dtype=np.int64)
                                 .astype(np.int32)).to(dev)
        y = torch.empty((1, spec.out_features), dtype=torch.bfloat16, device=dev)
        wr = torch.empty(vq.gemv_rht_workspace_size(layer, 1), dtype=torch.uint8, device=dev)
        for _ in range(args.profile_launches):
            vq.gemv_rht(layer, s_in, s_out, x, out=y, workspace=wr)
    elif args.profile in ("gemv", "lut", "lut_down", "lut_small", "dequant"):
        w = WORKLOADS[DECODE if args.profile != "lut_small" else "llama31_405b"]
        spec, seed = w.layers[{"lut_small": 4, "lut_down": 2}.get(args.profile, 0)]
        layer = vq.Layer.from_synth(synth.make_layer(spec, seed), dev,
                                    layout="tile4" if args.profile.startswith("lut") else "rows")
        x = torch.from_numpy(synth.make_x(w.x_seed, BATCH, spec.in_features, w.outlier_frac)
                             .view(np.int16)).to(dev).view(torch.bfloat16)
        out = (torch.empty((spec.out_features, spec.in_features), dtype=torch.float16, device=dev)
               if args.profile == "dequant" else
               torch.empty((BATCH, spec.out_features), dtype=torch.bfloat16, device=dev))
        ws = torch.empty(max(256, vq.gemv_workspace_size(layer, BATCH)), dtype=torch.uint8, device=dev)
        for _ in range(args.profile_launches):
            if args.profile == "dequant":
                vq.dequant(layer, out=out)
            else:
                vq.gemv(layer, x, out=out, workspace=ws)
    else:
        w = WORKLOADS[PREFILL]
        spec, seed = w.layers[0]
        layer = vq.Layer.from_synth(synth.make_layer(spec, seed), dev)
        x = torch.from_numpy(synth.make_x(w.x_seed, PREFILL_M, spec.in_features).view(np.int16))
        x = x.to(dev).view(torch.bfloat16)
        y = torch.empty((PREFILL_M, spec.out_features), dtype=torch.bfloat16, device=dev)
        ws = torch.empty(vq.gemm_workspace_size(layer, PREFILL_M), dtype=torch.uint8, device=dev)
        for _ in range(args.profile_launches):
            vq.gemm(layer, x, out=y, workspace=ws)
    torch.cuda.synchronize()
    print(json.dumps({"profile": args.profile, "launches": args.profile_launches,
                      "kernel_launches": vq.kernel_launches()}))
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile", choices=["gemv", "lut", "lut_gateup", "lut_down", "lut_small", "gemm",
                                          "tc_gate16", "tcs_q16", "tcs_8b16", "encode_h", "rht_gate",
                                          "dequant", "encode", "hessian"],
                    help="run a few untimed launches of one call on its workload (for ncu): "
                         "gemv / lut = 70B gate_proj in row / tiled order, lut_gateup = 70B "
                         "gate_proj + up_proj in one vq_gemv_multi launch, lut_down = 70B "
                         "down_proj in tiled order, lut_small = 405B gate_proj in tiled order, "
                         "encode / hessian = the encoder / the Hessian on their bench workloads")
    ap.add_argument("--profile-launches", type=int, default=3)
    args = ap.parse_args(argv)
    if args.profile:
        return run_profile(args)
    if args.warmup < 3:
        raise SystemExit("--warmup must be at least 3")
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
