#!/usr/bin/env python
"""Benchmark of the TQ4_1S hot path on B200 (one JSON line on rank 0).

Workload (default): one Llama-3-8B-shaped decoder layer -- q,o 4096x4096,
k,v 1024x4096, gate,up 14336x4096, down 4096x14336 -- bf16 weights
~N(0, 0.02^2) with 1% of input columns replaced by 0.02*10*t(4) values,
batch-1 bf16 activations ~N(0,1).  Synthetic, seeded; no checkpoints.

A step is one pass of the whole path over the layer:
  quantise all seven matrices -> dequantise all seven (bf16) ->
  pre-rotate + fused GEMV for all seven (fp32 y).
The step is captured once in a CUDA graph and replayed.

Reported:
  value      GEMV weight GB/s = packed layer bytes (codes + scales) / GEMV
             phase time (one batched pre-rotation + fused-product pass over
             the seven matrices), steady state: 32 passes per graph replay
             (the 32 decoder layers of one Llama-3-8B token), alternating
             with an independent shadow layer so that every pass reads its
             packed weights from HBM; CUDA events on the stream;
  quantize   Gweights/s of the quantise phase (10 passes per replay);
  ms_per_step  the full step (10 steps per graph replay), inputs in HBM;
  e2e        the same GB/s metric through the public API with host buffers:
             every step copies the bf16 weights and activations from pinned
             host memory, runs the path and reads the outputs back;
  roofline   for the phase with the largest share of the step, against the
             measured HBM copy bandwidth; rooflines for every phase;
  cpu_baseline  the CPU oracle on a bounded row sample, rows split over all
             host cores (and on one core, beside it);
  prefill    the large-M tensor-core product on an 8192 x 8192 weight times
             2048 activation rows: whole call and product alone, TFLOP/s
             against the measured dense bf16 tensor peak;
  codec_comparison  NVFP4 next to TQ4_1S on the layer, and the TQ4_1S
             skinny sweep (1, 2, 4, 8, 16, 32 activation rows).

Multi-GPU (torchrun): every rank runs its own layer (independent problems,
no collective on the data path, weak scaling); times are the max over ranks.
"""
from __future__ import annotations

import argparse
import csv
import datetime
import io
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

import torch  # noqa: E402

METRIC = "TQ4_1S dequant-GEMV weight GB/s (% of HBM peak) at M=1; quantize Gweights/s"
UNIT = "GB/s"
FALLBACK_HBM_GBS = 6650.0


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------
def parse_args(argv=None):
    p = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=("ours", "reference"), default="ours")
    p.add_argument("--workload", choices=("llama3_8b_layer", "single_matrix", "ffn_70b"), default="llama3_8b_layer")
    p.add_argument("--skip-cpu-baseline", action="store_true")
    p.add_argument("--skip-e2e", action="store_true")
    p.add_argument("--skip-codec-comparison", action="store_true",
                   help="skip the NVFP4 vs TQ4_1S comparison on the Llama-3-8B layer shapes")
    p.add_argument("--skip-prefill", action="store_true", help="omit the large-M tensor-core product line")
    p.add_argument("--skip-ffn", action="store_true", help="omit the 70B-class FFN skinny sweep")
    p.add_argument("--skip-single", action="store_true", help="omit the single 2048x2048 matrix line")
    p.add_argument("--skip-comparators", action="store_true",
                   help="omit dequantise+matmul and dense bf16 GEMV on the same layer")
    p.add_argument("--no-graph", action="store_true", help="launch eagerly instead of replaying a CUDA graph")
    p.add_argument("--cpu-sample-rows", type=int, default=None,
                   help="rows per matrix for the CPU oracle sample (default: half of each matrix)")
    return p.parse_args(argv)


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# Operations the TQ4_1S codec defines per 32-element block when it quantises:
# sign flip 32, five butterfly stages 5 x 32, half-block RMS (32 squares, 2 x
# 15 adds, 2 x (scale by 1/16, square root, fp16 rounding)) 68, thresholds
# scaled by each half's scale 2 x 7, three threshold compares and the sign
# test per element 4 x 32, one nibble insert per element 32: 434 per block.
QUANT_OPS_PER_WEIGHT = 434 / 32
LANES_PER_SM = 128  # fp32 / integer lanes of one SM (4 partitions x 32)

PROFILE_FILES = {  # phase -> committed ncu summary and the sources its kernel is built from
    "quantize": ("quantize_kernel_llama3_8b_down.md", ("tq_device.cuh", "tq_codec.cu")),
    "dequantize": ("dequantize_kernel_llama3_8b_layer.md", ("tq_device.cuh", "tq_codec.cu")),
    "gemv": ("gemv_group_kernel_llama3_8b_layer.md", ("tq_device.cuh", "tq_gemv.cu")),
}


def profile_field(phase: str, field: str):
    """A `field: value` line of the phase's committed ncu summary, or None when
    the kernel source changed since the capture."""
    import hashlib

    name, sources = PROFILE_FILES[phase]
    try:
        text = open(os.path.join(ROOT, "profiles", name)).read()
        fields = dict(ln.split(": ", 1) for ln in text.splitlines() if ": " in ln)
        h = hashlib.sha256()
        for src in sources:
            with open(os.path.join(ROOT, "dequant_gemv_tq4_b200", "csrc", src), "rb") as f:
                h.update(f.read())
        if h.hexdigest()[:16] != fields["source_sha256"].strip():
            return None
        return fields[field].strip()
    except Exception:
        return None


def profile_traffic(phase: str, weights: int):
    """DRAM bytes (read + write) of one pass of `phase` from the committed ncu
    capture, scaled by the weights processed (traffic grows in proportion to
    the units), or None when the kernel source changed since the capture."""
    import hashlib

    name, sources = PROFILE_FILES[phase]
    try:
        text = open(os.path.join(ROOT, "profiles", name)).read()
        fields = dict(ln.split(": ", 1) for ln in text.splitlines() if ": " in ln and ln.split(": ", 1)[0] in
                      ("traffic_bytes_per_launch", "weights_per_launch", "source_sha256"))
        h = hashlib.sha256()
        for src in sources:
            with open(os.path.join(ROOT, "dequant_gemv_tq4_b200", "csrc", src), "rb") as f:
                h.update(f.read())
        if h.hexdigest()[:16] != fields["source_sha256"].strip():
            return None
        return int(round(int(fields["traffic_bytes_per_launch"]) * weights / int(fields["weights_per_launch"])))
    except Exception:
        return None


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms while active."""

    FIELDS = ["index", "pci.bus_id", "clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, device: int):
        props = torch.cuda.get_device_properties(device)
        self.bus = f"{getattr(props, 'pci_domain_id', 0):08X}:{getattr(props, 'pci_bus_id', 0):02X}:" \
                   f"{getattr(props, 'pci_device_id', 0):02X}.0"
        self.proc = None
        self.file = None

    def start(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={','.join(self.FIELDS)}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=self.file, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.file.flush()
        self.file.seek(0)
        rows = [r for r in csv.reader(io.StringIO(self.file.read())) if len(r) == len(self.FIELDS)]
        self.file.close()
        os.unlink(self.file.name)
        mine = [r for r in rows if r[1].strip().upper().endswith(self.bus[-12:].upper())] or rows
        sm = [float(r[2]) for r in mine if r[2].strip().replace(".", "").isdigit()]
        mx = [float(r[3]) for r in mine if r[3].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in mine for i in range(4) if r[6 + i].strip().lower() == "active"})
        loaded = [v for v in sm if mx and v > 0.5 * max(mx)] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(mine)}


# ---------------------------------------------------------------------------
# workloads
# ---------------------------------------------------------------------------
def make_workload(name: str, rank: int, device):
    from dequant_gemv_tq4_b200 import inputs

    mats = []  # (label, W, activation name)
    acts = {}
    if name == "llama3_8b_layer":
        weights, acts = inputs.llama3_8b_layer(seed=rank_seed(rank), device=device)
        for label, W in weights.items():
            mats.append((label, W, inputs.LLAMA3_8B_INPUTS[label]))
        desc = {"workload": "llama3_8b_layer", "shapes": {k: list(v) for k, v in inputs.LLAMA3_8B_LAYER.items()},
                "weights": "bf16 ~N(0,0.02^2), 1% outlier columns 0.2*t(4)", "x": "bf16 ~N(0,1)", "m": 1}
    elif name == "single_matrix":
        W, x = inputs.single_matrix(device=device)
        mats.append(("w", W, "x"))
        acts = {"x": x}
        desc = {"workload": "single_matrix_2048", "shapes": {"w": [2048, 2048]}, "weights": "fp32 ~N(0,0.02^2)",
                "x": "fp32 ~N(0,1)", "m": 1}
    else:
        for tid, (label, (n, k)) in enumerate(inputs.FFN_70B.items()):
            mats.append((label, inputs.gaussian_matrix(2 + rank_seed(rank), tid, n, k, 0.015, torch.bfloat16, device),
                         "x_" + label))
            acts["x_" + label] = inputs.gaussian_matrix(1, 200 + tid, 1, k, 1.0, torch.bfloat16, device)[0]
        desc = {"workload": "ffn_70b", "shapes": {k: list(v) for k, v in inputs.FFN_70B.items()},
                "weights": "bf16 ~N(0,0.015^2)", "x": "bf16 ~N(0,1)", "m": 1}
    return mats, acts, desc


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
class Path:
    """Buffers and launches of one step of the hot path."""

    def __init__(self, tq, mats, acts, device):
        self.tq = tq
        self.items = []
        for label, W, act in mats:
            n, k = W.shape
            codes = torch.empty(tq.tq_codes_bytes(n, k), dtype=torch.uint8, device=device)
            scales = torch.empty(tq.tq_scales_bytes(n, k) // 2, dtype=torch.int16, device=device)
            deq = torch.empty((n, k), dtype=torch.bfloat16, device=device)
            y = torch.empty((1, n), dtype=torch.float32, device=device)
            x = acts[act].view(1, -1)
            self.items.append(dict(label=label, W=W, x=x, n=n, k=k, codes=codes, scales=scales, deq=deq, y=y,
                                   ws=tq.workspace(1, n, k, device)))
        self.batch = [(it["codes"], it["scales"], it["n"], it["k"], it["x"], it["y"]) for it in self.items]
        self.descs = tq.batch_descs(self.batch)
        self.deq_batch = [(it["codes"], it["scales"], it["n"], it["k"], it["deq"]) for it in self.items]
        self.deq_descs = tq.dequant_descs(self.deq_batch)
        self.ws = tq.batch_workspace(self.batch, 1, device)

    def quantize(self):
        for it in self.items:
            self.tq.quantize(it["W"], it["codes"], it["scales"])

    def dequantize(self):
        """All matrices in one launch."""
        self.tq.dequantize_batch(self.deq_batch, descs=self.deq_descs)

    def gemv(self):
        """All matrices in one batch: one pre-rotation launch for the distinct
        inputs, one fused-product launch."""
        self.tq.gemm_batch(self.batch, m=1, ws=self.ws, descs=self.descs)

    def add_shadow(self, mats, acts, device):
        """A second, independent layer (packed once) so that timed GEMV passes
        can alternate between two layers whose packed weights together exceed
        the 126 MB L2: every pass then reads its weights from HBM."""
        self.shadow = []
        for label, W, act in mats:
            n, k = W.shape
            codes, scales = self.tq.quantize(W)
            self.shadow.append((codes, scales, n, k, acts[act].view(1, -1),
                                torch.empty((1, n), dtype=torch.float32, device=device)))
        self.shadow_descs = self.tq.batch_descs(self.shadow)
        self.shadow_ws = self.tq.batch_workspace(self.shadow, 1, device)

    def gemv_pair(self):
        """The layer's batched GEMV, then the shadow layer's."""
        self.gemv()
        self.tq.gemm_batch(self.shadow, m=1, ws=self.shadow_ws, descs=self.shadow_descs)

    def gemv_one(self, i):
        it = self.items[i]
        return lambda: self.tq.gemv(it["codes"], it["scales"], it["n"], it["k"], it["x"][0], out=it["y"][0],
                                    ws=it["ws"])

    def step(self):
        self.quantize()
        self.dequantize()
        self.gemv()

    # byte / weight accounting (algorithmic)
    def weights(self):
        return sum(it["n"] * it["k"] for it in self.items)

    def packed_bytes(self, i=None):
        its = self.items if i is None else [self.items[i]]
        return sum(it["codes"].numel() + 2 * it["scales"].numel() for it in its)

    def in_bytes(self):
        return sum(it["W"].numel() * it["W"].element_size() for it in self.items)

    def act_bytes(self):
        seen, total = set(), 0
        for it in self.items:
            if it["x"].data_ptr() not in seen:
                seen.add(it["x"].data_ptr())
                total += it["x"].numel() * it["x"].element_size()
        return total

    def out_bytes(self):
        return sum(it["y"].numel() * 4 for it in self.items)


def capture(fn, use_graph: bool, repeat: int = 1):
    """A callable that runs `fn` `repeat` times: one CUDA graph replay (or
    eager launches without graphs)."""
    def body():
        for _ in range(repeat):
            fn()

    if not use_graph:
        return body
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fn()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        body()
    return g.replay


def time_replays(run, reps: int, flush=None):
    """Sum of CUDA-event durations of `reps` calls on the current stream; the
    optional flush runs before each call, outside the timed interval."""
    stream = torch.cuda.current_stream()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(reps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(reps)]
    for i in range(reps):
        if flush is not None:
            flush()
        starts[i].record(stream)
        run()
        ends[i].record(stream)
    torch.cuda.synchronize()
    return sum(s.elapsed_time(e) for s, e in zip(starts, ends))


def replay_stats(run, reps: int, per_replay: int, flush=None):
    """CUDA-event time of each of `reps` calls of `run` (each `per_replay`
    passes), per pass in microseconds: (mean, median, min, max)."""
    stream = torch.cuda.current_stream()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(reps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(reps)]
    for i in range(reps):
        if flush is not None:
            flush()
        starts[i].record(stream)
        run()
        ends[i].record(stream)
    torch.cuda.synchronize()
    us = sorted(1e3 * s.elapsed_time(e) / per_replay for s, e in zip(starts, ends))
    return statistics.fmean(us), statistics.median(us), us[0], us[-1]


def rank_seed(rank: int) -> int:
    """Layer seed of a rank: every rank quantises and multiplies its own layer
    (independent problems, weak scaling, no collective on the data path)."""
    return 100 * rank


def max_over_ranks(values, world):
    """Element-wise max of per-rank timings (NCCL on GPU ranks, gloo on CPU)."""
    if world == 1:
        return list(values)
    import torch.distributed as dist

    dev = torch.device("cuda", torch.cuda.current_device()) if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor(values, dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def timed_launches(nmat: int, steps: int, passes: int, gemv_passes: int) -> dict:
    """Kernel launches of this library inside the timed regions of the main
    line, per phase: the step loop (a quantise launch per matrix, one batched
    dequantise, one pre-rotation and one fused product), the quantise and
    dequantise phases, the GEMV phase (pre-rotation and product per pass) and
    the per-matrix GEMV timings (one tq_gemv each: pre-rotation and product)."""
    per = {"step": (nmat + 3) * steps * passes, "quantize": nmat * steps * passes, "dequantize": steps * passes,
           "gemv": 2 * steps * gemv_passes, "gemv_single_matrix": 2 * steps * nmat}
    per["total"] = sum(per.values())
    return per


def job_gbs(bytes_per_rank: int, world: int, ms: float) -> float:
    """Whole-job throughput: the bytes all ranks processed / the slowest rank's time."""
    return world * bytes_per_rank / (ms * 1e-3) / 1e9


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()
    if torch.cuda.is_available():
        torch.cuda.synchronize()


CPU_SAMPLE_FRACTION = 8  # the CPU sample: the first 1/8 of every matrix's rows


def cpu_sample_rows(n: int, rows_per_matrix=None) -> int:
    return min(n, rows_per_matrix) if rows_per_matrix else max(16, n // CPU_SAMPLE_FRACTION)


def oracle_pass(mats, threads: int):
    """One pass of the CPU oracle, as it stands, over `mats` (list of
    (W fp32 numpy [r, k], x fp64 numpy [1, k])): quantise, dequantise and the
    fp64 GEMV.  With threads > 1 the rows are partitioned into `threads`
    slices (multiples of 16 rows) run concurrently (the oracle's C routines
    release the GIL); each slice is the oracle applied to those rows.
    Returns seconds per phase and the packed bytes produced."""
    from concurrent.futures import ThreadPoolExecutor

    import oracle

    def slices(r):
        per = max(16, -(-r // threads) // 16 * 16)
        return [(a, min(r, a + per)) for a in range(0, r, per)]

    tq_s = td_s = tg_s = 0.0
    packed = 0
    with ThreadPoolExecutor(max_workers=max(1, threads)) as ex:
        for W, x in mats:
            r, k = W.shape
            parts = slices(r)
            t0 = time.perf_counter()
            q = list(ex.map(lambda ab: oracle.quantize(np.ascontiguousarray(W[ab[0]:ab[1]])), parts))
            t1 = time.perf_counter()
            list(ex.map(lambda a: oracle.dequantize(a[1][0], a[1][1], a[0][1] - a[0][0], k), zip(parts, q)))
            t2 = time.perf_counter()
            list(ex.map(lambda a: oracle.gemm(a[1][0], a[1][1], a[0][1] - a[0][0], k, x), zip(parts, q)))
            t3 = time.perf_counter()
            tq_s += t1 - t0
            td_s += t2 - t1
            tg_s += t3 - t2
            packed += sum(c.nbytes + sc.nbytes for c, sc in q)
    return tq_s, td_s, tg_s, packed


def cpu_oracle_sample(path, rows_per_matrix=None):
    """The CPU oracle, as it stands, on the first rows of every matrix: one
    core, then the same rows partitioned over every host core."""
    import oracle

    oracle.build()
    mats = []
    weights = 0
    for it in path.items:
        n, k = it["n"], it["k"]
        r = cpu_sample_rows(n, rows_per_matrix)
        mats.append((it["W"][:r].float().cpu().numpy(),
                     it["x"].float().cpu().numpy().reshape(1, -1).astype(np.float64)))
        weights += r * k
    cores = os.cpu_count() or 1
    res = {}
    for label, threads in (("single_core", 1), ("all_cores", cores)):
        tq_s, td_s, tg_s, packed = oracle_pass(mats, threads)
        res[label] = {"threads": threads, "gemv_gbs": packed / tg_s / 1e9,
                      "quantize_gweights_per_s": weights / tq_s / 1e9,
                      "dequantize_gweights_per_s": weights / td_s / 1e9, "seconds": tq_s + td_s + tg_s}
    res["sample"] = (f"first {rows_per_matrix or f'1/{CPU_SAMPLE_FRACTION} of the'} rows of each of the "
                     f"{len(path.items)} matrices ({weights / 1e6:.1f} M weights): quantise, dequantise, GEMV")
    res["weights"] = weights
    return res


def run_ours(args, world, rank, local):
    import dequant_gemv_tq4_b200 as tq

    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    tq.load_library()  # raises: there is no CPU path
    mats, acts, desc = make_workload(args.workload, rank, device)
    path = Path(tq, mats, acts, device)
    smats, sacts, _ = make_workload(args.workload, rank + 1000, device)
    path.add_shadow(smats, sacts, device)
    del smats, sacts
    nmat = len(path.items)
    warmup = max(3, args.warmup)
    steps = max(1, args.steps)
    flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device=device)  # > 126 MB L2

    def flush():
        flush_buf.zero_()

    for _ in range(warmup):
        path.step()
    torch.cuda.synchronize()
    use_graph = not args.no_graph
    # Steady-state timing: R passes back to back inside one graph replay, so
    # the per-replay launch latency of the graph is amortised.  Quantise and
    # dequantise stream >400 MB per pass (far above L2); the GEMV passes
    # alternate between the layer and an independent shadow layer (together
    # 2 x 136 MB of packed weights), so every pass reads its weights from HBM.
    # A decode token runs the product over all 32 decoder layers of the
    # model, captured as one graph; the GEMV phase replays that many passes
    # per graph (the layer and the shadow layer alternating), so its time per
    # pass carries the graph boundary once per token, as decoding does.
    R = 10
    RG = 32
    try:
        step_run = capture(path.step, use_graph, R)
        q_run = capture(path.quantize, use_graph, R)
        d_run = capture(path.dequantize, use_graph, R)
        g_run = capture(path.gemv_pair, use_graph, RG // 2)
    except Exception as e:  # graph capture refused: launch eagerly
        print(f"[bench] CUDA graph capture failed ({e}); launching eagerly", file=sys.stderr)
        use_graph = False
        step_run, q_run, d_run, g_run = (capture(path.step, False, R), capture(path.quantize, False, R),
                                         capture(path.dequantize, False, R), capture(path.gemv_pair, False, RG // 2))
    for run in (step_run, q_run, d_run, g_run):
        for _ in range(warmup):
            run()
    torch.cuda.synchronize()

    sampler = ClockSampler(local)
    barrier(world)
    sampler.start()
    time.sleep(0.4)
    barrier(world)
    st_step = replay_stats(step_run, steps, R)
    barrier(world)
    st_q = replay_stats(q_run, steps, R, flush)
    st_d = replay_stats(d_run, steps, R, flush)
    # the GEMV passes alternate between two layers whose packed weights
    # together exceed L2, so they need no flush (a write flush would leave
    # 126 MB of dirty lines for the first pass to write back)
    st_g = replay_stats(g_run, steps, RG)
    t_step, t_q, t_d = (1e-3 * x[0] * steps * R for x in (st_step, st_q, st_d))
    t_g = 1e-3 * st_g[0] * steps * RG
    per_matrix = {}
    for i, it in enumerate(path.items):
        run_i = capture(path.gemv_one(i), use_graph)
        for _ in range(warmup):
            run_i()
        ms_i = time_replays(run_i, steps, flush) / steps
        per_matrix[it["label"]] = {"n": it["n"], "k": it["k"], "us": round(1e3 * ms_i, 2),
                                   "gbs": round(path.packed_bytes(i) / (ms_i * 1e-3) / 1e9, 1)}
    barrier(world)
    clocks = sampler.stop()
    t_step, t_q, t_d, t_g = max_over_ranks([t_step, t_q, t_d, t_g], world)

    ms_step = t_step / (steps * R)
    ms_q, ms_d, ms_g = t_q / (steps * R), t_d / (steps * R), t_g / (steps * RG)
    packed = path.packed_bytes()
    weights = path.weights()
    hbm, hbm_kind = measured_peaks()
    value = job_gbs(packed, world, ms_g)
    quant_gw = job_gbs(weights, world, ms_q)

    # algorithmic bytes per phase (one GPU)
    alg = {
        "quantize": (path.in_bytes() + packed, ms_q, nmat),
        "dequantize": (packed + 2 * weights, ms_d, 1),
        "gemv": (packed + path.act_bytes() + path.out_bytes(), ms_g, 2),
    }
    rooflines = {}
    for ph, (nbytes, ms, nl) in alg.items():
        ach = nbytes / (ms * 1e-3) / 1e9
        rooflines[ph] = {"bound": "hbm", "achieved": round(ach, 1), "peak": hbm, "unit": "GB/s",
                         "frac": round(ach / hbm, 4), "traffic": profile_traffic(ph, weights),
                         "bytes_per_step": nbytes, "ms": round(ms, 5), "launches": nl}
    dominant = max(("quantize", "dequantize", "gemv"), key=lambda ph: alg[ph][1])
    # the quantise kernel is bound by its arithmetic, not by HBM: its ALU
    # roofline counts the codec's defined operations against every lane of
    # every SM at the highest SM clock seen
    props = torch.cuda.get_device_properties(device)
    max_mhz = (clocks or {}).get("sm_max_mhz") or 1965.0
    alu_peak = props.multi_processor_count * LANES_PER_SM * max_mhz * 1e6 / 1e12
    alu_ach = QUANT_OPS_PER_WEIGHT * weights / (ms_q * 1e-3) / 1e12
    rooflines["quantize_alu"] = {"bound": "alu", "achieved": round(alu_ach, 3), "peak": round(alu_peak, 3),
                                 "unit": "Tops/s", "frac": round(alu_ach / alu_peak, 4),
                                 "traffic": rooflines["quantize"]["traffic"],
                                 "ops_per_weight": round(QUANT_OPS_PER_WEIGHT, 4), "ms": round(ms_q, 5),
                                 "peak_note": f"{props.multi_processor_count} SMs x {LANES_PER_SM} lanes x "
                                              f"{max_mhz:.0f} MHz, one operation per lane per cycle"}
    ipw = profile_field("quantize", "thread_instructions_per_weight")
    rooflines["quantize_alu"]["measured_instructions_per_weight"] = float(ipw) if ipw is not None else None
    rooflines["quantize_alu"]["instructions_note"] = (
        "ops_per_weight counts the codec's defined operations; measured_instructions_per_weight is ncu's "
        "thread-instruction count per weight for the same kernel (committed summary), null if the kernel "
        "changed since")
    top = rooflines["quantize_alu"] if dominant == "quantize" else rooflines[dominant]

    line = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": steps,
        "warmup": warmup, "ms_per_step": round(ms_step, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f16",
        "dtype_detail": "fused product: f16 tensor-core operands (centroids, pre-rotated x), f32 accumulate and "
                        "scales; codec: f32 (bit-exact order); inputs bf16",
        "data": "synthetic (seeded counter-based generator; no checkpoints)",
        "config": dict(desc, parallelism=f"replicas x{world}" if world > 1 else "single GPU",
                       l2="quantise / dequantise phases: flushed (256 MB write) before every replay; GEMV "
                          "phase and codec comparison: inputs > L2 (passes alternate between two layers, "
                          "2 x 136.5 MB packed), no flush; step loop: inputs > L2",
                       graph=use_graph, hbm_peak_source=hbm_kind),
        "pct_of_hbm_peak": round(100 * value / world / hbm, 2),
        "quantize_gweights_per_s": round(quant_gw, 2),
        "phases_ms": {"quantize": round(ms_q, 5), "dequantize": round(ms_d, 5), "gemv": round(ms_g, 5)},
        "gemv_single_matrix": per_matrix,
        "phase_stats_us": {ph: {"mean": round(v[0], 3), "median": round(v[1], 3), "min": round(v[2], 3),
                                "max": round(v[3], 3)}
                           for ph, v in (("step", st_step), ("quantize", st_q), ("dequantize", st_d),
                                         ("gemv", st_g))},
        "roofline": dict(top, kernel=dominant, **({} if dominant == "quantize" else
                                                  {"peak_note": f"{hbm_kind} HBM copy bandwidth"})),
        "rooflines": rooflines,
        "clocks": clocks,
        "gpu_launches": timed_launches(nmat, steps, R, RG)["total"],
        "gpu_launches_by_phase": timed_launches(nmat, steps, R, RG),
        "timing": {"passes_per_replay": R, "gemv_passes_per_replay": RG, "replays": steps,
                   "gemv": f"{RG} passes per graph replay (one token through the 32 decoder layers of Llama-3-8B), "
                           "alternating between the layer and an independent shadow layer (2 x packed bytes > L2)",
                   "single_matrix": "one tq_gemv per graph replay, L2 flushed before each; includes graph launch latency"},
    }

    if not args.skip_e2e:
        line["e2e"] = run_e2e(tq, path, steps=min(steps, 5), world=world)
    if args.workload == "llama3_8b_layer" and not args.skip_prefill:
        line["prefill"] = prefill_measure(tq, rank, device, min(steps, 10), warmup, flush)
    if args.workload == "llama3_8b_layer" and not args.skip_codec_comparison:
        line["codec_comparison"] = codec_comparison(tq, path, rank, device, min(steps, 10), warmup, flush, use_graph,
                                                    world)
    if args.workload == "llama3_8b_layer" and not args.skip_comparators:
        cmp = comparators(tq, path, device, min(steps, 10), warmup, use_graph, world, hbm)
        fused_us = 1e3 * ms_g
        for key in ("dequant_then_matmul", "dense_bf16_gemv"):
            cmp[key]["vs_fused"] = round(cmp[key]["us_mean"] / fused_us, 2)
        cmp["fused_us"] = round(fused_us, 2)
        line["comparators"] = cmp
    if args.workload == "llama3_8b_layer" and not args.skip_ffn:
        line["ffn_70b"] = ffn70b_sweep(tq, rank, device, min(steps, 10), warmup, use_graph, world, hbm)
    if args.workload == "llama3_8b_layer" and not args.skip_single:
        line["single_matrix"] = single_matrix_measure(tq, device, min(steps, 10), warmup, use_graph, hbm)
    if rank == 0 and world == 1 and not args.skip_cpu_baseline:
        cb = cpu_oracle_sample(path, args.cpu_sample_rows)
        allc, one = cb["all_cores"], cb["single_core"]
        line["cpu_baseline"] = {"value": round(allc["gemv_gbs"], 4), "unit": UNIT, "cores": allc["threads"],
                                "kind": "oracle", "sample": cb["sample"],
                                "quantize_gweights_per_s": round(allc["quantize_gweights_per_s"], 5),
                                "dequantize_gweights_per_s": round(allc["dequantize_gweights_per_s"], 5),
                                "seconds": round(allc["seconds"], 2),
                                "partition": "rows split into one slice per core (multiples of 16), the oracle "
                                             "as it stands applied to each slice on its own thread",
                                "single_core": {"value": round(one["gemv_gbs"], 4), "cores": 1,
                                                "quantize_gweights_per_s": round(one["quantize_gweights_per_s"], 5),
                                                "dequantize_gweights_per_s":
                                                    round(one["dequantize_gweights_per_s"], 5),
                                                "seconds": round(one["seconds"], 2)}}
    if rank == 0:
        print(json.dumps(line), flush=True)


def codec_comparison(tq, path, rank, device, steps, warmup, flush, use_graph, world):
    """NVFP4 next to TQ4_1S on the same layer: reconstruction rel-L2 over the
    layer, quantise Gweights/s and fused-product GB/s at M = 1 and M = 16
    (TQ4_1S also at M = 2, 4, 8 and 32: the skinny sweep)
    (steady state, passes alternating with a shadow layer as for the main
    metric).  GB/s counts each codec's own packed bytes."""
    from dequant_gemv_tq4_b200 import inputs

    R = 10
    smats, _, _ = make_workload("llama3_8b_layer", rank + 1000, device)
    x32 = {}
    for aid, act in enumerate(("attn", "attn_out", "ffn", "ffn_mid")):
        k = 14336 if act == "ffn_mid" else 4096
        x32[act] = inputs.gaussian_matrix(1, 300 + aid, 32, k, 1.0, torch.bfloat16, device)
    act_of = inputs.LLAMA3_8B_INPUTS

    def nv_pack(mats):
        return [tq.nvfp4_quantize(W) for _, W, _ in mats]

    layer_mats = [(it["label"], it["W"], None) for it in path.items]
    nv_layer, nv_shadow = nv_pack(layer_mats), nv_pack(smats)
    tq_shadow = [(c, s) for c, s, *_ in path.shadow]
    tq_layer = [(it["codes"], it["scales"]) for it in path.items]

    def items_tq(packs, mats, m):
        out = []
        for (c, s), (label, W, _) in zip(packs, mats):
            n, k = W.shape
            X = x32[act_of[label]][:m]
            out.append((c, s, n, k, X, torch.empty((m, n), dtype=torch.float32, device=device)))
        return out

    def items_nv(packs, mats, m):
        out = []
        for (c, s, t), (label, W, _) in zip(packs, mats):
            n, k = W.shape
            X = x32[act_of[label]][:m]
            out.append((c, s, t, n, k, X, torch.empty((m, n), dtype=torch.float32, device=device)))
        return out

    def timed(fn, passes, fl=None):
        run = capture(fn, use_graph, passes)
        for _ in range(warmup):
            run()
        torch.cuda.synchronize()
        return time_replays(run, steps, fl) / (steps * passes)

    result = {}
    for codec in ("tq4_1s", "nvfp4"):
        entry = {}
        if codec == "tq4_1s":
            packed = path.packed_bytes()
            entry["bits_per_weight"] = 5.0
        else:
            packed = sum(c.numel() + s.numel() + t.numel() * 4 for c, s, t in nv_layer)
            entry["bits_per_weight"] = 4.5
        # the skinny sweep (1..32 activation rows) for TQ4_1S, m = 1 and 16 for NVFP4
        for m in ((1, 2, 4, 8, 16, 32) if codec == "tq4_1s" else (1, 16)):
            if codec == "tq4_1s":
                a, b = items_tq(tq_layer, layer_mats, m), items_tq(tq_shadow, smats, m)
                da, db = tq.batch_descs(a), tq.batch_descs(b)
                wa, wb = tq.batch_workspace(a, m, device), tq.batch_workspace(b, m, device)

                def pair(a=a, b=b, da=da, db=db, wa=wa, wb=wb, m=m):
                    tq.gemm_batch(a, m=m, ws=wa, descs=da)
                    tq.gemm_batch(b, m=m, ws=wb, descs=db)
            else:
                a, b = items_nv(nv_layer, layer_mats, m), items_nv(nv_shadow, smats, m)
                da, db = tq.nvfp4_batch_descs(a), tq.nvfp4_batch_descs(b)
                wa, wb = tq.nvfp4_batch_workspace(a, m, device), tq.nvfp4_batch_workspace(b, m, device)

                def pair(a=a, b=b, da=da, db=db, wa=wa, wb=wb, m=m):
                    tq.nvfp4_gemm_batch(a, m=m, ws=wa, descs=da)
                    tq.nvfp4_gemm_batch(b, m=m, ws=wb, descs=db)
            ms = timed(pair, R // 2) / 2  # two layers alternate: packed bytes together > L2, no flush
            (ms,) = max_over_ranks([ms], world)
            entry[f"gemm_m{m}_us"] = round(1e3 * ms, 2)
            entry[f"gemm_m{m}_gbs"] = round(job_gbs(packed, world, ms), 1)
            entry[f"gemm_m{m}_tflops"] = round(2.0 * m * path.weights() * world / (ms * 1e-3) / 1e12, 2)
        if codec == "tq4_1s":
            qfn = path.quantize
        else:
            def qfn():
                for (c, s, t), it in zip(nv_layer, path.items):
                    n, k = it["W"].shape
                    st = tq.tq_nvfp4_quantize(it["W"].data_ptr(), tq.TQ_BF16, n, k, k, c.data_ptr(), s.data_ptr(),
                                              t.data_ptr(), torch.cuda.current_stream().cuda_stream)
                    if st != 0:
                        raise tq.TQError(st, "tq_nvfp4_quantize")
        ms_q = timed(qfn, R, flush)
        (ms_q,) = max_over_ranks([ms_q], world)
        entry["quantize_gweights_per_s"] = round(job_gbs(path.weights(), world, ms_q), 2)
        # reconstruction error over the layer: ||W~ - W|| / ||W||
        num = den = 0.0
        for i, it in enumerate(path.items):
            n, k = it["W"].shape
            if codec == "tq4_1s":
                Wd = tq.dequantize(it["codes"], it["scales"], n, k, dtype=torch.float32)
            else:
                c, s, t = nv_layer[i]
                Wd = tq.nvfp4_dequantize(c, s, t, n, k, dtype=torch.float32)
            Wf = it["W"].float()
            num += float(((Wd - Wf).double() ** 2).sum())
            den += float((Wf.double() ** 2).sum())
            del Wd, Wf
        entry["rel_l2_reconstruction"] = round((num / den) ** 0.5, 5)
        entry["packed_bytes"] = packed
        result[codec] = entry
    return result


def ffn70b_sweep(tq, rank, device, steps, warmup, use_graph, world, hbm):
    """The 70B-class FFN (gate, up 28672 x 8192; down 8192 x 28672; bf16
    ~N(0, 0.015^2)) at m = 1, 2, 4, 8, 16, 32 activation rows (bf16 ~N(0, 1)):
    one batched product over the three matrices per pass (gate and up share
    their input, down has its own), 440 MB of packed weights per pass (> L2,
    no flush needed), with the kernel the library picks for m; from m = 9 the
    mma.sync kernel forced by the test hook is timed beside it for context."""
    from dequant_gemv_tq4_b200 import inputs

    R = 5
    packs, shapes = [], []
    for tid, (label, (n, k)) in enumerate(inputs.FFN_70B.items()):
        W = inputs.gaussian_matrix(2 + rank_seed(rank), tid, n, k, 0.015, torch.bfloat16, device)
        packs.append(tq.quantize(W))
        shapes.append((label, n, k))
        del W
    packed = sum(c.numel() + 2 * s.numel() for c, s in packs)
    weights = sum(n * k for _, n, k in shapes)
    xs = {k: inputs.gaussian_matrix(1, 200 + i, 32, k, 1.0, torch.bfloat16, device)
          for i, k in enumerate(sorted({k for _, _, k in shapes}))}
    res = {"workload": "ffn_70b: gate, up 28672x8192 and down 8192x28672, bf16 ~N(0,0.015^2), X bf16 ~N(0,1)",
           "packed_bytes": packed, "passes_per_replay": R, "sweep": {}}
    for m in (1, 2, 4, 8, 16, 32):
        entry = {}
        for label, flag in (("default", 0), ("mma_sync", 8)):
            if label == "mma_sync" and m < 9:
                continue
            tq.tq_debug_set_flags(flag)
            try:
                items = [(c, s, n, k, xs[k][:m], torch.empty((m, n), dtype=torch.float32, device=device))
                         for (c, s), (_, n, k) in zip(packs, shapes)]
                descs = tq.batch_descs(items)
                ws = tq.batch_workspace(items, m, device)
                run = capture(lambda: tq.gemm_batch(items, m=m, ws=ws, descs=descs), use_graph, R)
                for _ in range(warmup):
                    run()
                mean, med, mn, mx = replay_stats(run, steps, R)
                st = tq.workspace_status(ws)
            finally:
                tq.tq_debug_set_flags(0)
            (mean,) = max_over_ranks([mean], world)
            gbs = job_gbs(packed, world, mean * 1e-3)
            entry[label] = {"us_mean": round(mean, 2), "us_median": round(med, 2), "us_min": round(mn, 2),
                            "us_max": round(mx, 2), "gbs": round(gbs, 1), "pct_of_hbm": round(100 * gbs / world / hbm, 1),
                            "tflops": round(2.0 * m * weights * world / (mean * 1e-6) / 1e12, 2), "status": int(st)}
            if label == "default":
                entry[label]["kernel"] = "tcgen05 (tensor memory)" if m >= 9 else "mma.sync"
        res["sweep"][f"m{m}"] = entry
    del packs
    return res


def single_matrix_measure(tq, device, steps, warmup, use_graph, hbm):
    """The single 2048 x 2048 fp32 matrix (~N(0, 0.02^2), seed 0) with an fp32
    activation (~N(0,1), seed 1): quantise, dequantise and the GEMV.  Its
    packed weights (2.6 MB) fit in L2, so the GEMV passes cycle through 64
    independently packed copies (168 MB > L2) to read from HBM; the quantise
    passes read the fp32 weights after a 256 MB L2 flush."""
    from dequant_gemv_tq4_b200 import inputs

    W, x = inputs.single_matrix(device=device)
    n, k = W.shape
    copies = []
    for i in range(64):
        Wi = W if i == 0 else (W * (1.0 + 2.0 ** -10 * i))
        copies.append(tq.quantize(Wi))
    ys = torch.empty((1, n), dtype=torch.float32, device=device)
    xs = x.view(1, -1)
    wss = [tq.workspace(1, n, k, device) for _ in range(8)]
    flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device=device)

    def gemv_all():
        for i, (c, s) in enumerate(copies):
            tq.gemm(c, s, n, k, xs, out=ys, ws=wss[i % 8])

    run = capture(gemv_all, use_graph)
    for _ in range(warmup):
        run()
    mean, med, mn, mx = replay_stats(run, steps, len(copies))
    packed = copies[0][0].numel() + 2 * copies[0][1].numel()
    codes, scales = tq.tq_codes_bytes(n, k), tq.tq_scales_bytes(n, k)
    c0 = torch.empty(codes, dtype=torch.uint8, device=device)
    s0 = torch.empty(scales // 2, dtype=torch.int16, device=device)
    qrun = capture(lambda: tq.quantize(W, c0, s0), use_graph)
    for _ in range(warmup):
        qrun()
    qmean, qmed, _, _ = replay_stats(qrun, steps, 1, flush=lambda: flush_buf.zero_())
    return {"workload": "single_matrix_2048: W 2048x2048 fp32 ~N(0,0.02^2) (seed 0), x fp32 ~N(0,1) (seed 1)",
            "gemv_us_mean": round(mean, 2), "gemv_us_median": round(med, 2), "gemv_us_min": round(mn, 2),
            "gemv_us_max": round(mx, 2), "gemv_gbs": round(packed / (mean * 1e-6) / 1e9, 1),
            "gemv_pct_of_hbm": round(100 * packed / (mean * 1e-6) / 1e9 / hbm, 1),
            "gemv_note": "one tq_gemm call per pass (pre-rotation + product), 64 packed copies cycled (> L2); "
                         "a 2.6 MB matrix is bound by launch latency, not HBM",
            "quantize_us": round(qmean, 2), "quantize_gweights_per_s": round(n * k / (qmean * 1e-6) / 1e9, 1)}


def comparators(tq, path, device, steps, warmup, use_graph, world, hbm):
    """Two ways to run the same batch-1 layer without the fused kernel
    (TQ4_1S page, TQ4_1S 是什么 / 解码速度 sections: the CUDA port converts
    TQ4_1S to q8_0 at load time and runs a plain kernel):
      * dequant_then_matmul: tq_dequantize_batch of every matrix to bf16
        (one launch), then a cuBLAS bf16 GEMV (torch.matmul) per matrix,
        every pass;
      * dense_bf16_gemv: cuBLAS bf16 GEMV on the unquantised bf16 weights
        (the weights converted once; 3.2 x the bytes of the packed form),
        alternating two copies of the layer (2 x 436 MB > L2).
    GB/s is counted for each method's own weight bytes; `vs_fused` is the
    method's time over the fused product's time on the same layer."""
    R = 4
    deq = [torch.empty((it["n"], it["k"]), dtype=torch.bfloat16, device=device) for it in path.items]
    outs = [torch.empty((1, it["n"]), dtype=torch.bfloat16, device=device) for it in path.items]

    dq_items = [(it["codes"], it["scales"], it["n"], it["k"], d) for it, d in zip(path.items, deq)]
    dq_descs = tq.dequant_descs(dq_items)

    def dq_mm():
        tq.dequantize_batch(dq_items, descs=dq_descs)
        for it, d, o in zip(path.items, deq, outs):
            torch.matmul(it["x"], d.t(), out=o)

    run = capture(dq_mm, use_graph, R)
    for _ in range(warmup):
        run()
    dq_mean, dq_med, dq_min, dq_max = replay_stats(run, steps, R)
    shadow_w = [it["W"].clone() for it in path.items]  # a second dense copy: two layers > L2

    def dense():
        for it, o in zip(path.items, outs):
            torch.matmul(it["x"], it["W"].t(), out=o)
        for it, w, o in zip(path.items, shadow_w, outs):
            torch.matmul(it["x"], w.t(), out=o)

    run2 = capture(dense, use_graph, R)
    for _ in range(warmup):
        run2()
    de_mean, de_med, de_min, de_max = replay_stats(run2, steps, 2 * R)
    del shadow_w
    packed, dense_bytes = path.packed_bytes(), path.in_bytes()
    return {"workload": "llama3_8b_layer at m = 1 (bf16 x, bf16 y)",
            "dequant_then_matmul": {"us_mean": round(dq_mean, 2), "us_median": round(dq_med, 2),
                                    "us_min": round(dq_min, 2), "us_max": round(dq_max, 2),
                                    "packed_gbs": round(packed / (dq_mean * 1e-6) / 1e9, 1)},
            "dense_bf16_gemv": {"us_mean": round(de_mean, 2), "us_median": round(de_med, 2),
                                "us_min": round(de_min, 2), "us_max": round(de_max, 2),
                                "bf16_gbs": round(dense_bytes / (de_mean * 1e-6) / 1e9, 1),
                                "pct_of_hbm": round(100 * dense_bytes / (de_mean * 1e-6) / 1e9 / hbm, 1)},
            "bytes": {"packed": packed, "bf16": dense_bytes}}


PREFILL_PROFILE = ("prefill_kernel_8192x8192_m2048.md", ("tq_device.cuh", "tq_prefill.cu"))


def prefill_measure(tq, rank, device, steps, warmup, flush):
    """The large-M product on its configured workload: an 8192 x 8192 weight
    (bf16 ~N(0, 0.02^2)) times 2048 activation rows (bf16 ~N(0, 1)), bf16 out.
    Times the whole call (plain pre-rotation + tensor-core product) and the
    product alone over a pre-rotated activation; the product's TFLOP/s is set
    against the measured dense bf16 tensor peak (fp16 operands run at the bf16
    rate).  cuBLAS bf16 on the dense weight of the same shape is context.
    Inputs total 74 MB (< L2), so L2 is flushed before every timed call."""
    import hashlib

    from dequant_gemv_tq4_b200 import inputs

    n = k = 8192
    m = 2048
    W = inputs.gaussian_matrix(rank_seed(rank), 40, n, k, 0.02, torch.bfloat16, device)
    X = inputs.gaussian_matrix(rank_seed(rank) + 1, 41, m, k, 1.0, torch.bfloat16, device)
    codes, scales = tq.quantize(W)
    ws = tq.prefill_workspace(m, k, device)
    hdr = torch.zeros(256, dtype=torch.uint8, device=device)
    xr = tq.prerotate_plain(X)
    Y = torch.empty((m, n), dtype=torch.bfloat16, device=device)
    full = lambda: tq.gemm_prefill(codes, scales, n, k, X, out=Y, ws=ws)
    prod = lambda: tq.gemm_prefill_xrot(codes, scales, n, k, xr, out=Y, ws=hdr)
    dense = lambda: torch.matmul(X, W.t(), out=Y)
    res = {}
    for name, fn in (("call", full), ("product", prod), ("cublas_bf16_dense", dense)):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        res[name] = time_replays(fn, steps, flush) / steps
    st = tq.workspace_status(ws) or tq.workspace_status(hdr)
    flops = 2.0 * m * n * k
    peaks = {}
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            peaks = json.load(f)
        peak, kind = float(peaks["bf16_tflops"]), "measured"
    except Exception:
        peak, kind = 1590.0, "fallback"
    ach = flops / (res["product"] * 1e-3) / 1e12
    traffic = None
    try:
        text = open(os.path.join(ROOT, "profiles", PREFILL_PROFILE[0])).read()
        fields = dict(ln.split(": ", 1) for ln in text.splitlines() if ": " in ln)
        h = hashlib.sha256()
        for src in PREFILL_PROFILE[1]:
            with open(os.path.join(ROOT, "dequant_gemv_tq4_b200", "csrc", src), "rb") as f:
                h.update(f.read())
        if h.hexdigest()[:16] == fields["source_sha256"].strip():
            traffic = int(fields["traffic_bytes_per_launch"])
    except Exception:
        traffic = None
    return {
        "workload": "8192x8192 TQ4_1S weight (bf16 source ~N(0,0.02^2)) x 2048 bf16 activation rows ~N(0,1), bf16 out",
        "ms_call": round(res["call"], 5), "tflops_call": round(flops / (res["call"] * 1e-3) / 1e12, 1),
        "ms_product": round(res["product"], 5),
        "roofline": {"bound": "tensor", "achieved": round(ach, 1), "peak": peak, "unit": "TFLOP/s",
                     "frac": round(ach / peak, 4), "traffic": traffic, "kernel": "prefill_kernel",
                     "peak_note": f"{kind} dense bf16 burst (fp16 operands, same nominal rate)",
                     "algorithmic": "2*m*n*k flops per launch"},
        "cublas_bf16_dense_ms": round(res["cublas_bf16_dense"], 5),
        "cublas_bf16_dense_tflops": round(flops / (res["cublas_bf16_dense"] * 1e-3) / 1e12, 1),
        "status": int(st), "l2": "flushed (256 MB write) before every timed call",
    }


def run_e2e(tq, path, steps, world):
    """Public API with host buffers: H2D of weights + activations from pinned
    memory, quantise/dequantise/GEMV, D2H of every y, per step."""
    host_w = [it["W"].cpu().pin_memory() for it in path.items]
    host_y = [torch.empty_like(it["y"], device="cpu").pin_memory() for it in path.items]
    dev_w = [torch.empty_like(it["W"]) for it in path.items]
    # one host/device buffer per distinct activation (matrices share inputs)
    xs = {}
    for it in path.items:
        xs.setdefault(it["x"].data_ptr(), (it["x"].cpu().pin_memory(), torch.empty_like(it["x"])))
    batch = [(it["codes"], it["scales"], it["n"], it["k"], xs[it["x"].data_ptr()][1], it["y"]) for it in path.items]
    descs = tq.batch_descs(batch)
    stream = torch.cuda.current_stream()

    def one():
        for i, it in enumerate(path.items):
            dev_w[i].copy_(host_w[i], non_blocking=True)
        for hx, dx in xs.values():
            dx.copy_(hx, non_blocking=True)
        for i, it in enumerate(path.items):
            tq.quantize(dev_w[i], it["codes"], it["scales"])
        for it in path.items:
            tq.dequantize(it["codes"], it["scales"], it["n"], it["k"], out=it["deq"])
        tq.gemm_batch(batch, m=1, ws=path.ws, descs=descs)
        for i, it in enumerate(path.items):
            host_y[i].copy_(it["y"], non_blocking=True)

    one()
    torch.cuda.synchronize()
    barrier(world)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(steps):
        one()
    end.record(stream)
    torch.cuda.synchronize()
    (ms,) = max_over_ranks([start.elapsed_time(end) / steps], world)
    return {"value": round(world * path.packed_bytes() / (ms * 1e-3) / 1e9, 2), "unit": UNIT,
            "h2d_bytes_per_step": path.in_bytes() + path.act_bytes(), "d2h_bytes_per_step": path.out_bytes(),
            "ms_per_step": round(ms, 4), "steps": steps}


# ---------------------------------------------------------------------------
# reference arm: the CPU oracle on the host cores
# ---------------------------------------------------------------------------
def run_reference(args, world, rank):
    """The reference arm: the CPU oracle, as it stands, on the host cores --
    the same row sample as the GPU line's cpu_baseline (the first 1/8 of every
    matrix's rows), partitioned over every core -- one oracle pass per step
    (quantise, dequantise, GEMV); the metric is the GEMV phase's GB/s of
    packed weights, as for the GPU line."""
    if rank != 0:
        return

    import oracle
    from dequant_gemv_tq4_b200 import inputs

    oracle.build()
    if args.workload == "llama3_8b_layer":
        shapes = [(lbl, n, k, seed) for seed, (lbl, (n, k)) in enumerate(inputs.LLAMA3_8B_LAYER.items())]
    elif args.workload == "single_matrix":
        shapes = [("w", 2048, 2048, 0)]
    else:
        shapes = [(lbl, n, k, tid) for tid, (lbl, (n, k)) in enumerate(inputs.FFN_70B.items())]
    mats = []
    weights = 0
    for lbl, n, k, seed in shapes:
        r = cpu_sample_rows(n, args.cpu_sample_rows)
        # the generator is row-major, so r rows are exactly the matrix's first r rows
        if args.workload == "llama3_8b_layer":
            W = inputs.llama_weight(seed, 0, r, k)
            x = inputs.gaussian_matrix(1, 7, 1, k, 1.0, torch.bfloat16)
        elif args.workload == "single_matrix":
            W = inputs.gaussian_matrix(0, 0, r, k, 0.02, torch.float32)
            x = inputs.gaussian_matrix(1, 0, 1, k, 1.0, torch.float32)
        else:
            W = inputs.gaussian_matrix(2, seed, r, k, 0.015, torch.bfloat16)
            x = inputs.gaussian_matrix(1, 7, 1, k, 1.0, torch.bfloat16)
        mats.append((W.float().numpy(), x.float().numpy().astype(np.float64)))
        weights += r * k
    cores = os.cpu_count() or 1
    for _ in range(max(3, args.warmup)):
        oracle_pass(mats, cores)
    tot_b = tot_t = tot_q = 0.0
    t0 = time.perf_counter()
    for _ in range(max(1, args.steps)):
        tq_s, td_s, tg_s, packed = oracle_pass(mats, cores)
        tot_b += packed
        tot_t += tg_s
        tot_q += tq_s
    wall = time.perf_counter() - t0
    value = tot_b / tot_t / 1e9
    sample = (f"first {args.cpu_sample_rows or f'1/{CPU_SAMPLE_FRACTION} of the'} rows of every matrix "
              f"({weights / 1e6:.1f} M weights) per step, rows split over {cores} threads: quantise, dequantise, GEMV")
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": UNIT, "n_gpus": args.gpus,
            "steps": max(1, args.steps), "warmup": max(3, args.warmup),
            "ms_per_step": round(1e3 * wall / max(1, args.steps), 2), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "dtype_detail": "CPU oracle: f32 codec in the codec order, f64 product",
            "data": "synthetic (seeded counter-based generator; no checkpoints)",
            "config": {"workload": args.workload, "sample": sample},
            "quantize_gweights_per_s": round(weights * max(1, args.steps) / tot_q / 1e9, 5),
            "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main(argv=None):
    args = parse_args(argv)
    world, rank, local = dist_env()
    if world > 1:
        import torch.distributed as dist

        if args.impl == "ours":
            torch.cuda.set_device(local)
        dist.init_process_group("nccl" if args.impl == "ours" else "gloo",
                                timeout=datetime.timedelta(seconds=300))
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
