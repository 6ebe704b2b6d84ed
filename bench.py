#!/usr/bin/env python
"""Benchmark: GPTQ quantization of one linear layer per step, end to end on the GPU.

A step is the whole hot path for one layer: H = 2 X^T X over all calibration tokens
(gptq_hessian_accumulate), damping + U = upper Cholesky factor of H^-1 (gptq_prepare_hinv), and
the column sweep with lazy updates writing the packed layer (gptq_quantize_pack_layer), all
through the C ABI. Default workload: the largest single-GPU layer, a Llama-70B-shaped down projection,
W 8192 x 28672 bf16 ~ N(0, 0.015^2), X 131072 x 28672 bf16 half-normal with lognormal(0, 1)
channel scales and 0.05 % outlier channels x30, 4-bit symmetric with one scale per row,
block 128, damp 0.01 (a 28672^2 fp32 Hessian). --workload selects another one.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0). Under torchrun each rank quantizes its own layer (independent
problems, no collective on the data path: weak scaling); the timed duration is the max over ranks.
--impl reference times the FP64 CPU oracle on bounded samples of the same workload.
Besides the headline the line reports the per-stage times (breakdown_ms) and each stage's
roofline (stages), the dominant kernel's roofline (roofline: the 3xTF32 GEMM at the step's
largest product, timed live) and the SYRK's (roofline_syrk), the end-to-end rate through the C
ABI from pinned host buffers (e2e: X streamed in chunks whose copies overlap the SYRK), the
oracle's rate on the host cores (cpu_baseline), the number of kernels launched in the timed
steps (counted from the recorded CUDA graphs), and the dequantizing GEMV and GEMM on a packed
8192 x 28672 int4 layer (dequant_gemv, dequant_gemm).
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "GPTQ layer quantize wall ms & weights/s (incl. XXᵀ); SYRK TFLOP/s; sweep GB/s"
UNIT = "weights/s"
DEFAULT_WORKLOAD = "llama70b_down_proj"
# TF32 peak from the measured bf16 peak by the nominal dense ratio (1.1 / 2.25 PFLOP/s).
TF32_PER_BF16 = 1.1 / 2.25


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--e2e-steps", type=int, default=5, help="end-to-end steps (at least 1)")
    ap.add_argument("--tokens", type=int, default=0,
                    help="calibration tokens instead of the workload's own count (smaller cases "
                         "for profiler captures; the config line reports the count used)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--eager", action="store_true",
                    help="call the C ABI directly in the timed steps instead of replaying the "
                         "CUDA graphs recorded from the same calls")
    return ap.parse_args()


def peaks():
    """(HBM GB/s, bf16 TFLOP/s burst, bf16 TFLOP/s sustained, source)."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return (float(p["hbm_gbs"]), float(p["bf16_tflops"]),
                float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), "measured")
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# ------------------------------------------------------------------------------------------
# Kernel launches of a step, counted from the CUDA graphs recorded from its C ABI calls
# ------------------------------------------------------------------------------------------

def new_graph():
    import torch
    try:
        return torch.cuda.CUDAGraph(keep_graph=True), True
    except TypeError:
        return torch.cuda.CUDAGraph(), False


def graph_kernel_nodes(gr):
    """Number of kernel nodes in a recorded graph (None when the graph is not inspectable)."""
    try:
        from cuda.bindings import runtime as rt
        handle = gr.raw_cuda_graph()
        err, _, n = rt.cudaGraphGetNodes(handle, 0)
        if int(err) != 0:
            return None
        err, nodes, n = rt.cudaGraphGetNodes(handle, n)
        if int(err) != 0:
            return None
        kern = 0
        for nd in nodes:
            err, t = rt.cudaGraphNodeGetType(nd)
            if int(err) == 0 and t == rt.cudaGraphNodeType.cudaGraphNodeTypeKernel:
                kern += 1
        return kern
    except Exception:
        return None


# ------------------------------------------------------------------------------------------
# Clock sampling during the timed region
# ------------------------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu_index = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.gpu_index)],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        rows = []
        try:
            for line in open(self.path):
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        except Exception:
            pass
        finally:
            if self.path and os.path.exists(self.path):
                os.remove(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        pw = [num(r[3]) for r in rows if num(r[3]) is not None]
        load = [s for s, p in zip(sm, pw) if p is not None and p > 250.0] or sm
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(load) if load else None,
                "sm_max_mhz": num(rows[0][2]), "reasons": reasons, "samples": len(rows),
                "samples_under_load": len(load)}


# ------------------------------------------------------------------------------------------
# Oracle timing (CPU baseline and the reference arm)
# ------------------------------------------------------------------------------------------

class OracleSample:
    """The FP64 oracle on a bounded sample of one layer of the workload. Both the cpu_baseline
    key of our arm and the reference arm use this one definition. A step times:
      * the oracle's H on the leading `hcols` channels of X over the first t1 and over the first
        t2 calibration tokens. The cost of H at a fixed width is a fixed part (allocating,
        mirroring and scaling the d x d result) plus a part linear in the tokens (the rank-k
        update), so the two timings give the line that is extrapolated to all N tokens; both
        parts grow with the entries of H, so the block's cost scales to the full d by
        (d / hcols)^2;
      * the blocked sweep and the pack at the full d of the first r1 and of the first r2 rows
        of W, with U from the prepare below; the sweep's cost is a fixed per-column part plus a
        part linear in the rows, so the two timings give the line that is extrapolated to all
        d_out rows.
    The prepare (act-order, dead columns, damping, U) runs once per process at the full d, on
    H over the first t2 tokens (its cost does not depend on the values), and is counted once.
    The whole layer's time is the sum of the three extrapolations."""

    def __init__(self, wl, tokens=(256, 1024), rows=(16, 64), hcols=7168):
        import torch

        import layer_inputs as li
        self.wl = wl
        lin = wl.linears[0]
        act = wl.act(lin.act)
        self.N, self.d, self.n = act.n_tokens, lin.d_in, lin.d_out
        self.t1, self.t2 = (min(t, act.n_tokens) for t in tokens)
        self.r1, self.r2 = (min(r, lin.d_out) for r in rows)
        self.hcols = min(hcols, lin.d_in)
        # The first rows of the full workload's X and W (same seeded streams, same order).
        self.X = li.activations(self.t2, act.d, chan_sigma=act.chan_sigma,
                                outlier_frac=act.outlier_frac, outlier_mult=act.outlier_mult,
                                half_normal=act.half_normal, dtype=torch.bfloat16, seed=act.seed)
        self.W = li.weight(self.r2, lin.d_in, lin.sigma, torch.bfloat16, lin.seed)
        self.P = None
        self.prepare_s = None

    @staticmethod
    def _fit(x1, y1, x2, y2, x):
        """Value at x of the line through (x1, y1) and (x2, y2); a negative slope (timing noise)
        counts as flat. With x1 == x2 (a workload smaller than both samples) plain scaling."""
        if x2 == x1:
            return y1 * x / x1
        slope = max((y2 - y1) / (x2 - x1), 0.0)
        return y2 + slope * (x - x2)

    def prepare_once(self):
        from oracle import hessian as hs
        from oracle import prepare as prep
        q = self.wl.quant
        H = hs.hessian(self.X)
        t0 = time.perf_counter()
        self.P = prep.prepare(H, self.W.double().numpy(), q.percdamp, act_order=q.act_order)
        self.prepare_s = time.perf_counter() - t0
        self.P.pop("H_inv", None)
        self.P.pop("H_damped", None)

    def step(self):
        """One sample step. Returns (seconds the step took, its parts)."""
        from oracle import hessian as hs
        from oracle import pack as pk
        from oracle import sweep as sw
        q = self.wl.quant
        parts = {}
        t_start = time.perf_counter()
        for key, t in (("h1", self.t1), ("h2", self.t2)):
            t0 = time.perf_counter()
            hs.hessian(self.X[:t, :self.hcols])
            parts[key] = time.perf_counter() - t0
        for key, r in (("s1", self.r1), ("s2", self.r2)):
            t0 = time.perf_counter()
            codes, S, Z, _ = sw.sweep_blocked(self.P["W"][:r], self.P["U"], q.bits, q.group_size,
                                              q.sym, q.block_size)
            pk.pack(codes, S, Z, q.bits)
            parts[key] = time.perf_counter() - t0
        return time.perf_counter() - t_start, parts

    def layer_seconds(self, parts):
        h = self._fit(self.t1, parts["h1"], self.t2, parts["h2"], self.N)
        h *= (self.d / self.hcols) ** 2
        sweep = self._fit(self.r1, parts["s1"], self.r2, parts["s2"], self.n)
        return h + self.prepare_s + sweep

    def describe(self):
        return (f"FP64 oracle: H on {self.hcols} of {self.d} channels over {self.t1} and "
                f"{self.t2} of {self.N} tokens (line in the token count, x{(self.d / self.hcols) ** 2:.0f} "
                f"for the full d x d), the full {self.d}x{self.d} prepare once per process "
                f"({self.prepare_s:.1f} s), blocked sweep and pack of {self.r1} and {self.r2} of "
                f"{self.n} rows at the full d (line in the row count); layer time = the sum")




def cpu_cores():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        if info:
            return int(max(i.get("num_threads", 1) for i in info))
    except Exception:
        pass
    return os.cpu_count() or 1


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    wl = workload(args)
    lin = wl.linears[0]
    smp = OracleSample(wl)
    smp.prepare_once()
    for _ in range(args.warmup):
        smp.step()
    step_s, layer_s = [], []
    for _ in range(args.steps):
        secs, parts = smp.step()
        step_s.append(secs)
        layer_s.append(smp.layer_seconds(parts))
    per_layer = statistics.mean(layer_s)
    value = lin.d_out * lin.d_in / per_layer
    # Same line as this bench's own arm (n_gpus and config of the launch); ms_per_step is the
    # time of a sample step as it ran, value the whole-layer rate extrapolated from it.
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": statistics.mean(step_s) * 1e3,
            "extrapolated_layer_ms": per_layer * 1e3,
            "oracle_prepare_ms_once": smp.prepare_s * 1e3,
            "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_dict(args, wl, world=args.gpus),
            "cpu_baseline": {"kind": "oracle", "value": value, "unit": UNIT, "cores": cpu_cores(),
                             "sample": smp.describe()},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def workload(args):
    """The named workload, with its calibration token count replaced when --tokens is given."""
    import dataclasses
    import layer_inputs as li
    wl = li.WORKLOADS[args.workload]
    if args.tokens > 0:
        acts = tuple(dataclasses.replace(a, n_tokens=args.tokens) for a in wl.acts)
        wl = dataclasses.replace(wl, acts=acts)
    return wl


def measure_gemm(L, dev, n, d, reps=5):
    """The product kernel (gemm_tf32x3_kernel through gptq_gemm_f32) at the shape of the step's
    largest lazy update, W[:, m:] -= Err[:, :m] U[:m, m:] with m = d / 2: M = n, N = K = d / 2.
    Random fp32 operands; CUDA events around each launch on the current stream."""
    import torch
    m = d // 2
    A = torch.randn((n, m), device=dev) * 1e-3
    B = torch.randn((m, m), device=dev)
    C = torch.randn((n, m), device=dev)
    for _ in range(2):
        L.gptq_gemm_f32(A, B, C, alpha=-1.0, beta=1.0)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(reps + 1)]
    torch.cuda.synchronize()
    # NVTX range bench_gemm marks these launches for profilers.
    torch.cuda.nvtx.range_push("bench_gemm")
    ev[0].record()
    for i in range(reps):
        L.gptq_gemm_f32(A, B, C, alpha=-1.0, beta=1.0)
        ev[i + 1].record()
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    ms = statistics.mean(ev[i].elapsed_time(ev[i + 1]) for i in range(reps))
    flops = 2.0 * n * m * m
    del A, B, C
    return {"M": n, "N": m, "K": m, "ms": ms, "flops": flops, "tflops": flops / (ms * 1e-3) / 1e12,
            "reps": reps}


def measure_pack(L, dev, Wd, U, perm, dead, p, codes, scales, zeros, g_idx, ws, status, qweight,
                 s16, z16, bits, reps=20):
    """gptq_pack alone on this layer's codes (one gptq_quantize_layer run outside the timing);
    CUDA events around each launch on the current stream. HBM-bound."""
    import torch
    L.gptq_quantize_layer(Wd, U, perm, dead, p, codes, scales, zeros, g_idx, ws, status)
    for _ in range(3):
        L.gptq_pack(codes, bits, scales, zeros, qweight, s16, z16)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(reps + 1)]
    torch.cuda.synchronize()
    ev[0].record()
    for i in range(reps):
        L.gptq_pack(codes, bits, scales, zeros, qweight, s16, z16)
        ev[i + 1].record()
    torch.cuda.synchronize()
    us = statistics.mean(ev[i].elapsed_time(ev[i + 1]) for i in range(reps)) * 1e3
    n, d = codes.shape
    G = scales.shape[1]
    nbytes = n * d + n * ((d * bits + 31) // 32) * 4 + n * G * 12
    return {"us": us, "bytes": nbytes}


def measure_gemv(L, dev, hbm_gbs):
    """Dequantizing matrix-vector product on a packed 8192 x 28672 int4 layer, g = 128 (the down
    projection of the 70B-shaped workload), batch 1 (the reported figure) and batch 8: HBM-bound.
    Two copies of the packed words (2 x 117 MB, more than L2) are used alternately; CUDA events
    on the current stream."""
    import torch
    n, d, bits, g = 8192, 28672, 4, 128
    ng = d // g
    qws = [torch.randint(-2 ** 31, 2 ** 31 - 1, (n, d * bits // 32), dtype=torch.int32,
                         device=dev) for _ in range(2)]
    s16 = (torch.rand((n, ng), device=dev) * 0.02 + 0.001).half()
    z16 = torch.randint(0, 2 ** bits, (n, ng), device=dev).half()
    reps = 20

    def timed(batch):
        x = torch.randn((batch, d), device=dev).half()
        y = torch.empty((batch, n), device=dev)
        for i in range(4):
            L.gptq_dequant_gemv(qws[i % 2], d, bits, s16, z16, g, None, x, y)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(reps + 1)]
        torch.cuda.synchronize()
        ev[0].record()
        for i in range(reps):
            L.gptq_dequant_gemv(qws[i % 2], d, bits, s16, z16, g, None, x, y)
            ev[i + 1].record()
        torch.cuda.synchronize()
        us = statistics.mean(ev[i].elapsed_time(ev[i + 1]) for i in range(reps)) * 1e3
        nbytes = n * d * bits // 8 + 2 * n * ng * 2 + batch * (d * 2 + n * 4)
        return us, nbytes

    us, nbytes = timed(1)
    us8, nbytes8 = timed(8)
    gbs = nbytes / (us * 1e-6) / 1e9
    return {"workload": f"{n} x {d} int4 g{g}, batch 1, fp16 x, fp32 y", "us": us,
            "bytes": nbytes, "achieved_gbs": gbs, "peak_gbs": hbm_gbs, "frac": gbs / hbm_gbs,
            "batch8_us": us8, "batch8_gbs": nbytes8 / (us8 * 1e-6) / 1e9,
            "launches": 2 * (reps + 4)}


def measure_dequant_gemm(L, dev, bf16_tflops, m=2048):
    """Dequantizing GEMM (prefill) on the same packed 8192 x 28672 int4 g128 layer with m fp16
    activation rows: tensor-bound (2 m n d flop). CUDA events over 10 calls."""
    import torch
    n, d, g = 8192, 28672, 128
    ng = d // g
    qw = torch.randint(-2 ** 31, 2 ** 31 - 1, (n, d // 8), dtype=torch.int32, device=dev)
    s16 = (torch.rand((n, ng), device=dev) * 0.02 + 0.001).half()
    z16 = torch.randint(0, 16, (n, ng), device=dev).half()
    x = torch.randn((m, d), device=dev).half()
    y = torch.empty((m, n), device=dev)
    for _ in range(3):
        L.gptq_dequant_gemm(qw, d, s16, z16, g, x, y)
    reps = 10
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record()
    for _ in range(reps):
        L.gptq_dequant_gemm(qw, d, s16, z16, g, x, y)
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / reps
    tflops = 2.0 * m * n * d / (ms * 1e-3) / 1e12
    return {"workload": f"{n} x {d} int4 g{g}, {m} fp16 activation rows, fp32 y", "ms": ms,
            "tflops": tflops, "peak_tflops": bf16_tflops, "frac": tflops / bf16_tflops,
            "peak_source": "measured bf16 burst (fp16 runs at the same rate)",
            "launches": reps + 3}


def config_dict(args, wl, world):
    lin = wl.linears[0]
    act = wl.act(lin.act)
    q = wl.quant
    return {"workload": f"{wl.name}: W {lin.d_out}x{lin.d_in} bf16, X {act.n_tokens}x{act.d} bf16 "
                        f"calibration tokens, {q.bits}-bit "
                        f"{'sym' if q.sym else 'asym'} g={q.group_size} block={q.block_size} "
                        f"damp={q.percdamp}{' act-order' if q.act_order else ''}",
            "d_out": lin.d_out, "d_in": lin.d_in, "n_tokens": act.n_tokens, "bits": q.bits,
            "group_size": q.group_size, "parallelism": f"{world} independent layer(s), one per GPU",
            "l2": f"X is {act.n_tokens * act.d * 2 / 2**30:.2f} GiB; a 256 MiB L2 flush between "
                  "timed steps"}


# ------------------------------------------------------------------------------------------
# Multi-rank plumbing (independent layers per rank; only timing crosses ranks)
# ------------------------------------------------------------------------------------------

def max_over_ranks(values, device):
    """Element-wise max over all ranks of a few host floats (identity when not distributed)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.cpu().tolist()


def rank_seed_offset(rank):
    """Each rank quantizes its own layer: same shapes and distributions, disjoint seeds."""
    return 100000 * rank


# ------------------------------------------------------------------------------------------
# Our arm
# ------------------------------------------------------------------------------------------

def run_ours(args):
    import torch
    import torch.distributed as dist

    import layer_inputs as li
    import post_weight_quantization_18_b200 as G
    from post_weight_quantization_18_b200 import _lib as L

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)

    wl = workload(args)
    lin = wl.linears[0]
    act = wl.act(lin.act)
    q = wl.quant
    n, d, N = lin.d_out, lin.d_in, act.n_tokens

    # Inputs: pinned host copies (for the end-to-end measurement) and device copies.
    import dataclasses
    act = dataclasses.replace(act, seed=act.seed + rank_seed_offset(rank))
    lin = dataclasses.replace(lin, seed=lin.seed + rank_seed_offset(rank))
    Xh = torch.empty((N, d), dtype=torch.bfloat16).pin_memory()
    act.make(out=Xh)
    Wh = lin.make().pin_memory()
    Xd = Xh.to(dev)
    Wd = Wh.to(dev)

    order = L.GPTQ_ORDER_DESC_ACT if q.act_order else L.GPTQ_ORDER_NATURAL
    p = L.make_params(q.bits, q.group_size, q.sym, order, q.block_size, q.percdamp)
    G_n = 1 if q.group_size == -1 else d // q.group_size
    H = torch.empty((d, d), dtype=torch.float32, device=dev)
    U = torch.empty((d, d), dtype=torch.float32, device=dev)
    perm = torch.empty(d, dtype=torch.int32, device=dev)
    dead = torch.empty(d, dtype=torch.uint8, device=dev)
    codes = torch.empty((n, d), dtype=torch.uint8, device=dev)
    scales = torch.empty((n, G_n), dtype=torch.float32, device=dev)
    zeros = torch.empty((n, G_n), dtype=torch.float32, device=dev)
    g_idx = torch.empty(d, dtype=torch.int32, device=dev)
    ws = torch.empty(L.gptq_workspace_size(n, d, p), dtype=torch.uint8, device=dev)
    qweight = torch.empty((n, (d * q.bits + 31) // 32), dtype=torch.int32, device=dev)
    s16 = torch.empty((n, G_n), dtype=torch.int16, device=dev)
    z16 = torch.empty((n, G_n), dtype=torch.int16, device=dev)
    status = torch.zeros(2, dtype=torch.int32, device=dev)
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device=dev)  # 256 MiB > L2
    outs_h = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in (qweight, s16, z16, g_idx)]

    ev = {k: [] for k in ("step", "syrk", "prep", "quant")}
    # The step: H, prepare, and the sweep writing the packed layer (codes are never stored).
    calls = [
        lambda X, W: L.gptq_hessian_accumulate(H, X, 2.0, False, status),
        lambda X, W: L.gptq_prepare_hinv(H, p, U, perm, dead, ws, status),
        lambda X, W: L.gptq_quantize_pack_layer(W, U, perm, dead, p, qweight, s16, z16, scales,
                                                zeros, g_idx, ws, status),
    ]

    def step(X, W, record, graphs=None):
        e = [torch.cuda.Event(enable_timing=True) for _ in range(4)] if record else None
        if record:
            e[0].record()
        for i, call in enumerate(calls):
            if graphs is not None:
                graphs[i].replay()
            else:
                call(X, W)
            if record:
                e[i + 1].record()
        if record:
            ev["step"].append((e[0], e[3]))
            ev["syrk"].append((e[0], e[1]))
            ev["prep"].append((e[1], e[2]))
            ev["quant"].append((e[2], e[3]))

    for _ in range(max(3, args.warmup)):
        step(Xd, Wd, False)
    torch.cuda.synchronize()
    st = status.cpu().tolist()
    if st[0] != 0:
        raise RuntimeError(f"device status after warm-up: {G.status_string(st[0])} index {st[1]}")

    # Record each C ABI call of the step once into a CUDA graph (the calls only enqueue
    # kernels on the current stream) and replay the graphs in the timed steps: the ~230
    # launches of a step then cost no host time and no launch gaps.
    # The same recording gives the number of kernels a step launches (kernel nodes).
    graphs = []
    launches = 0
    for call in calls:
        gr, kept = new_graph()
        with torch.cuda.graph(gr):
            call(Xd, Wd)
        k = graph_kernel_nodes(gr) if kept else None
        launches = None if (launches is None or k is None) else launches + k
        if kept and hasattr(gr, "instantiate"):
            gr.instantiate()
        graphs.append(gr)
    for gr in graphs:      # one untimed replay of the recorded step
        gr.replay()
    torch.cuda.synchronize()
    if args.eager:
        graphs = None

    with ClockSampler(local) as clk:
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        # An NVTX range marks the timed steps for profilers (ncu --nvtx-include bench_timed/).
        torch.cuda.nvtx.range_push("bench_timed")
        for _ in range(args.steps):
            flush.zero_()
            step(Xd, Wd, True, graphs)
        torch.cuda.nvtx.range_pop()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        # End to end: pinned host inputs -> device -> hot path -> packed result back to host,
        # through the public calls as a user streams calibration data: X arrives in chunks of
        # whole 8192-token ranges on a copy stream and H accumulates each chunk as it lands
        # (gptq_hessian_accumulate with accumulate = 1 after the first), so the host-to-device
        # copies overlap the SYRK; W's copy overlaps prepare, which does not read it.
        compute = torch.cuda.current_stream()
        copy_stream = torch.cuda.Stream(device=dev)
        chunk = max(8192, -(-N // (16 * 8192)) * 8192)
        bounds = [(t0, min(N, t0 + chunk)) for t0 in range(0, N, chunk)]
        e2e_ev = []
        for _ in range(args.e2e_steps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(compute)
            copy_stream.wait_event(a)
            landed = []
            with torch.cuda.stream(copy_stream):
                for t0, t1 in bounds:
                    Xd[t0:t1].copy_(Xh[t0:t1], non_blocking=True)
                    landed.append(torch.cuda.Event())
                    landed[-1].record(copy_stream)
                Wd.copy_(Wh, non_blocking=True)
                w_landed = torch.cuda.Event()
                w_landed.record(copy_stream)
            for i, (t0, t1) in enumerate(bounds):
                compute.wait_event(landed[i])
                L.gptq_hessian_accumulate(H, Xd[t0:t1], 2.0, i > 0, status)
            calls[1](Xd, Wd)
            compute.wait_event(w_landed)
            calls[2](Xd, Wd)
            for h, t in zip(outs_h, (qweight, s16, z16, g_idx)):
                h.copy_(t, non_blocking=True)
            b.record(compute)
            e2e_ev.append((a, b))
        torch.cuda.synchronize()
    st = status.cpu().tolist()
    if st[0] != 0:
        raise RuntimeError(f"device status: {G.status_string(st[0])} index {st[1]}")

    def ms(k):
        return [a.elapsed_time(b) for a, b in ev[k]]
    step_ms = ms("step")
    total_s = sum(step_ms) / 1e3
    e2e_ms = [a.elapsed_time(b) for a, b in e2e_ev]
    e2e_total_s = sum(e2e_ms) / 1e3
    total_s, e2e_total_s = max_over_ranks([total_s, e2e_total_s], dev)

    hbm, bf16, bf16_sus, peak_kind = peaks()
    tf32x3 = bf16 * TF32_PER_BF16 / 3.0   # fp32-accurate products: three TF32 MMAs each
    # Side measurements, after the timed steps (same stream, CUDA events):
    gemm = measure_gemm(L, dev, n, d)     # the dominant kernel at the step's largest product
    pack = measure_pack(L, dev, Wd, U, perm, dead, p, codes, scales, zeros, g_idx, ws, status,
                        qweight, s16, z16, q.bits)
    gemv = measure_gemv(L, dev, hbm)
    dgemm = measure_dequant_gemm(L, dev, bf16)
    if rank == 0:
        stage_ms = {k: statistics.mean(ms(k)) for k in ("syrk", "prep", "quant")}
        syrk_flops = float(d) * (d + 1) * N
        syrk_tflops = syrk_flops / (stage_ms["syrk"] * 1e-3) / 1e12
        # Sweep with packed output: W read, Err written and the packed bits written per weight;
        # fp32 and fp16 s, z per (row, group); the U diagonal blocks once. Its lazy updates are
        # n d^2 flops of 3xTF32 products.
        sweep_bytes = (n * d * 8 + n * ((d * q.bits + 31) // 32) * 4 + n * G_n * 12 +
                       (d // 128) * 128 * 128 * 4)
        sweep_flops = float(n) * d * d
        prep_flops = 2.0 / 3.0 * float(d) ** 3
        weights = n * d
        value = world * args.steps * weights / total_s
        e2e_value = world * args.e2e_steps * weights / e2e_total_s
        h2d = Xh.numel() * Xh.element_size() + Wh.numel() * Wh.element_size()
        d2h = sum(o.numel() * o.element_size() for o in outs_h)

        def stage(ms_, bound, work, unit, peak, peak_src, algo, **extra):
            t_roof = work / (peak * (1e12 if unit == "TFLOP/s" else 1e9))
            ach = work / (ms_ * 1e-3) / (1e12 if unit == "TFLOP/s" else 1e9)
            return dict(ms=ms_, bound=bound, achieved=ach, peak=peak, unit=unit,
                        frac=ach / peak, roof_ms=t_roof * 1e3, peak_source=peak_src,
                        algorithmic=algo, **extra)
        sweep_t = max(sweep_flops / (tf32x3 * 1e12), sweep_bytes / (hbm * 1e9))
        tf_src = f"{peak_kind} bf16 burst x 1.1/2.25 (TF32) / 3 (3xTF32)"
        stages = {
            "hessian_syrk": stage(stage_ms["syrk"], "tensor", syrk_flops, "TFLOP/s", bf16,
                                  f"{peak_kind} bf16 burst", f"d(d+1)N = {syrk_flops:.4g} flop"),
            "prepare": stage(stage_ms["prep"], "tensor", prep_flops, "TFLOP/s", tf32x3, tf_src,
                             f"2/3 d^3 = {prep_flops:.4g} flop (Cholesky and inverse)"),
            "quantize_sweep_pack": stage(stage_ms["quant"], "tensor", sweep_flops, "TFLOP/s",
                                         tf32x3, tf_src,
                                         f"n d^2 = {sweep_flops:.4g} flop of lazy updates",
                                         bytes=sweep_bytes,
                                         hbm_frac=sweep_bytes / (stage_ms["quant"] * 1e-3) /
                                         (hbm * 1e9),
                                         roof_ms_max_of_flops_and_bytes=sweep_t * 1e3),
            "pack_standalone": stage(pack["us"] * 1e-3, "hbm", pack["bytes"], "GB/s", hbm,
                                     f"{peak_kind} HBM copy",
                                     f"{pack['bytes']} B (codes read, words and fp16 s/z "
                                     "written, fp32 s/z read)",
                                     note="gptq_pack on this layer's codes, timed alone; the "
                                          "step packs inside the sweep instead"),
        }
        cpu = None
        if not args.no_cpu_baseline and world == 1:
            smp = OracleSample(wl)
            smp.prepare_once()
            _, parts = smp.step()
            cpu = {"value": weights / smp.layer_seconds(parts), "unit": UNIT,
                   "cores": cpu_cores(), "kind": "oracle", "sample": smp.describe()}
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": max(3, args.warmup), "ms_per_step": statistics.mean(step_ms),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": f"synthetic (seeded W ~ N(0, {lin.sigma}^2), X lognormal channel scales with "
                    "outliers)",
            "config": config_dict(args, wl, world),
            "breakdown_ms": {"hessian_syrk": stage_ms["syrk"], "prepare": stage_ms["prep"],
                             "quantize_sweep_pack": stage_ms["quant"]},
            "syrk_tflops": syrk_tflops,
            # the same time counted as the full 2 d^2 N product (upper and lower triangle)
            "syrk_tflops_2d2n_equivalent": 2.0 * d * d * N / (stage_ms["syrk"] * 1e-3) / 1e12,
            "sweep_gbs": sweep_bytes / (stage_ms["quant"] * 1e-3) / 1e9,
            "roofline": {"bound": "tensor", "kernel": "gemm_tf32x3_kernel",
                         "achieved": gemm["tflops"], "peak": tf32x3, "unit": "TFLOP/s",
                         "frac": gemm["tflops"] / tf32x3, "traffic": None,
                         "peak_source": tf_src,
                         "algorithmic": f"2 M N K = {gemm['flops']:.4g} flop per launch "
                                        f"(M={gemm['M']}, N={gemm['N']}, K={gemm['K']}: the "
                                        "step's largest lazy-update product)",
                         "avg_launch_ms": gemm["ms"], "launches_timed": gemm["reps"]},
            "roofline_syrk": {"bound": "tensor", "kernel": "syrk_bf16_tcgen05_kernel",
                              "achieved": syrk_tflops, "peak": bf16, "unit": "TFLOP/s",
                              "frac": syrk_tflops / bf16, "traffic": None,
                              "peak_source": f"{peak_kind} bf16 burst",
                              "frac_of_sustained": syrk_tflops / bf16_sus,
                              "algorithmic": f"d(d+1)N = {syrk_flops:.4g} flop per launch"},
            "stages": stages,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": statistics.mean(e2e_ms)},
            "gpu_launches": (launches * args.steps) if launches is not None else None,
            "gpu_launches_per_step": launches,
            "execution": "eager C ABI calls" if args.eager else
                         "CUDA graphs recorded from the C ABI calls, replayed",
            "clocks": clk.summary(),
            "cpu_baseline": cpu,
            "dequant_gemv": gemv,
            "dequant_gemm": dgemm,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def main():
    args = parse_args()
    args.e2e_steps = max(1, args.e2e_steps)
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
