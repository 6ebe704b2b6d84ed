#!/usr/bin/env python
"""Benchmark: GPTQ quantization of one linear layer per step, end to end on the GPU.

A step is the whole hot path for one layer: H = 2 X^T X over all calibration tokens
(gptq_hessian_accumulate), damping + U = upper Cholesky factor of H^-1 (gptq_prepare_hinv), the
column sweep with lazy updates (gptq_quantize_layer) and packing (gptq_pack), all through the C
ABI. Default workload: Llama-7B attention projection, W 4096 x 4096 bf16, X 262144 x 4096 bf16
(128 sequences x 2048 tokens, lognormal(0, 1) channel scales, 0.1 % outlier channels x20),
4-bit asymmetric, group 128, block 128, damp 0.01.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0). Under torchrun each rank quantizes its own layer (independent
problems, no collective on the data path: weak scaling); the timed duration is the max over ranks.
--impl reference times the FP64 CPU oracle on bounded samples of the same workload.
Outside the timed steps the line also reports the per-stage times (breakdown_ms), the SYRK
roofline, the end-to-end rate from pinned host buffers (e2e), the oracle's rate (cpu_baseline),
and the dequantizing GEMV on a packed 8192 x 28672 int4 layer (dequant_gemv).
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
DEFAULT_WORKLOAD = "llama7b_attn_proj"


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--tokens", type=int, default=0,
                    help="calibration tokens instead of the workload's own count (smaller cases "
                         "for profiler captures; the config line reports the count used)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--eager", action="store_true",
                    help="call the C ABI directly in the timed steps instead of replaying the "
                         "CUDA graphs recorded from the same calls")
    return ap.parse_args()


def syrk_traffic():
    """DRAM bytes per launch of the SYRK kernel from its committed ncu summary, or None when the
    kernel source has changed since the counters were taken (the summary records its hash)."""
    import hashlib
    import re
    try:
        with open(os.path.join(ROOT, "profiles", "syrk_bf16_llama7b_attn_proj.md")) as f:
            text = f.read()
        with open(os.path.join(ROOT, "post_weight_quantization_18_b200", "csrc",
                               "syrk_bf16.cu"), "rb") as f:
            digest = hashlib.sha256(f.read()).hexdigest()
    except OSError:
        return None
    want = re.search(r"kernel_source_sha256:\s*([0-9a-f]{64})", text)
    val = re.search(r"traffic_bytes_per_launch:\s*([0-9]+)", text)
    if not want or not val or want.group(1) != digest:
        return None
    return int(val.group(1))


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


# ------------------------------------------------------------------------------------------
# Launch accounting (mirrors the host recursions in csrc/api.cu)
# ------------------------------------------------------------------------------------------

def _split(n):
    m = ((n // 2) + 127) // 128 * 128
    if m >= n:
        m = n - 128
    if m <= 0:
        m = n // 2
    return m


def _rl_launches(n):
    """Right-looking node of nb blocks: per block a base block; below the last, the panel block
    and the diagonal update; below the last two, the rest of the panel and the trailing update
    (with the next block column); and two products of the inverse for every block but the
    last."""
    nb = (n + 127) // 128
    return nb + 2 * (nb - 1) + 2 * max(0, nb - 2) + 2 * (nb - 1)


def _prep_launches(n):
    if n <= 32 * 128:
        return _rl_launches(n)
    m = _split(n)
    return 4 + _prep_launches(m) + _prep_launches(n - m)


def _sweep_launches(n):
    if n <= 128:
        return 1
    m = _split(n)
    return 1 + _sweep_launches(m) + _sweep_launches(n - m)


def launches_per_step(d, q):
    hess = 2
    prep = (1 if not q.act_order else 3) + 2 + _prep_launches(d)
    quant = 1 + (1 if q.group_size == -1 else 0) + _sweep_launches(d) + \
        (1 if q.act_order else 0) + 1
    return hess + prep + quant + 2


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

def oracle_sample(wl, X_host, W_host, tok_sample, row_sample):
    """Time the FP64 oracle on a bounded sample of one layer and extrapolate to the whole layer.
    Returns (seconds for the full layer, description)."""
    import numpy as np

    import oracle
    from oracle import hessian as hs
    from oracle import prepare as prep
    from oracle import sweep as sw
    q = wl.quant
    N, d = X_host.shape
    n = W_host.shape[0]
    tok = min(N, tok_sample)
    rows = min(n, row_sample)
    Xs = X_host[:tok].double().numpy()
    t0 = time.perf_counter()
    H = hs.hessian(Xs)
    t_h = time.perf_counter() - t0
    W64 = W_host[:rows].double().numpy()
    t0 = time.perf_counter()
    P = prep.prepare(H, W64, q.percdamp, act_order=q.act_order)
    t_p = time.perf_counter() - t0
    t0 = time.perf_counter()
    sw.sweep_blocked(P["W"], P["U"], q.bits, q.group_size, q.sym, q.block_size)
    t_s = time.perf_counter() - t0
    total = t_h * (N / tok) + t_p + t_s * (n / rows)
    desc = (f"oracle on {tok} of {N} tokens (H, scaled x{N / tok:.0f}), full {d}x{d} prepare, "
            f"sweep of {rows} of {n} rows (scaled x{n / rows:.0f})")
    return total, desc, dict(hessian_s=t_h, prepare_s=t_p, sweep_s=t_s)


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
    import torch

    import layer_inputs as li
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    wl = workload(args)
    lin = wl.linears[0]
    act = wl.act(lin.act)
    tok_sample, row_sample = 4096, 32
    X = li.activations(tok_sample, act.d, chan_sigma=act.chan_sigma,
                       outlier_frac=act.outlier_frac, outlier_mult=act.outlier_mult,
                       half_normal=act.half_normal, dtype=torch.bfloat16, seed=act.seed)
    W = li.weight(row_sample, lin.d_in, lin.sigma, torch.bfloat16, lin.seed)

    class Full:  # shapes of the full workload for extrapolation
        shape = (act.n_tokens, act.d)

    def step():
        secs, desc, parts = oracle_sample(wl, X, W, tok_sample, row_sample)
        # scale from the generated sample shape to the full workload
        secs = parts["hessian_s"] * (act.n_tokens / tok_sample) + parts["prepare_s"] + \
            parts["sweep_s"] * (lin.d_out / row_sample)
        return secs, parts
    for _ in range(args.warmup):
        step()
    times = []
    for _ in range(args.steps):
        secs, parts = step()
        times.append(secs)
    per = statistics.mean(times)
    value = lin.d_out * lin.d_in / per
    sample = (f"each step: FP64 oracle H on {tok_sample} of {act.n_tokens} tokens (scaled), full "
              f"{act.d}x{act.d} prepare, blocked sweep of {row_sample} of {lin.d_out} rows (scaled)")
    # Same line as this bench's own arm (n_gpus and config of the launch); what actually ran,
    # the oracle on this host's cores, is described under cpu_baseline.
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": per * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_dict(args, wl, world=args.gpus),
            "cpu_baseline": {"kind": "oracle", "value": value, "unit": UNIT, "cores": cpu_cores(),
                             "sample": sample},
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

    ev = {k: [] for k in ("step", "syrk", "prep", "quant", "pack")}
    calls = [
        lambda X, W: L.gptq_hessian_accumulate(H, X, 2.0, False, status),
        lambda X, W: L.gptq_prepare_hinv(H, p, U, perm, dead, ws, status),
        lambda X, W: L.gptq_quantize_layer(W, U, perm, dead, p, codes, scales, zeros, g_idx, ws,
                                           status),
        lambda X, W: L.gptq_pack(codes, q.bits, scales, zeros, qweight, s16, z16),
    ]

    def step(X, W, record, graphs=None):
        e = [torch.cuda.Event(enable_timing=True) for _ in range(5)] if record else None
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
            ev["step"].append((e[0], e[4]))
            ev["syrk"].append((e[0], e[1]))
            ev["prep"].append((e[1], e[2]))
            ev["quant"].append((e[2], e[3]))
            ev["pack"].append((e[3], e[4]))

    for _ in range(max(3, args.warmup)):
        step(Xd, Wd, False)
    torch.cuda.synchronize()
    st = status.cpu().tolist()
    if st[0] != 0:
        raise RuntimeError(f"device status after warm-up: {G.status_string(st[0])} index {st[1]}")

    # Record each C ABI call of the step once into a CUDA graph (the calls only enqueue
    # kernels on the current stream) and replay the graphs in the timed steps: the ~230
    # launches of a step then cost no host time and no launch gaps.
    graphs = None
    if not args.eager:
        graphs = []
        for call in calls:
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr):
                call(Xd, Wd)
            graphs.append(gr)
        for gr in graphs:      # one untimed replay of the recorded step
            gr.replay()
        torch.cuda.synchronize()

    with ClockSampler(local) as clk:
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        for _ in range(args.steps):
            flush.zero_()
            step(Xd, Wd, True, graphs)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        # End to end: pinned host inputs -> device -> hot path -> packed result back to host.
        e2e_ev = []
        for _ in range(args.e2e_steps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            Xd.copy_(Xh, non_blocking=True)
            Wd.copy_(Wh, non_blocking=True)
            step(Xd, Wd, False)
            for h, t in zip(outs_h, (qweight, s16, z16, g_idx)):
                h.copy_(t, non_blocking=True)
            b.record()
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

    hbm, bf16, peak_kind = peaks()
    gemv = measure_gemv(L, dev, hbm)
    if rank == 0:
        syrk_ms = statistics.mean(ms("syrk"))
        quant_ms = statistics.mean(ms("quant"))
        syrk_flops = float(d) * (d + 1) * N
        syrk_tflops = syrk_flops / (syrk_ms * 1e-3) / 1e12
        sweep_bytes = n * d * 9 + n * G_n * 8 + d * d * 4
        weights = n * d
        value = world * args.steps * weights / total_s
        e2e_value = world * args.e2e_steps * weights / e2e_total_s
        h2d = Xh.numel() * Xh.element_size() + Wh.numel() * Wh.element_size()
        d2h = sum(o.numel() * o.element_size() for o in outs_h)
        cpu = None
        if not args.no_cpu_baseline and world == 1:
            secs, desc, _ = oracle_sample(wl, Xh, Wh, 8192, 64)
            cpu = {"value": weights / secs, "unit": UNIT, "cores": cpu_cores(), "kind": "oracle",
                   "sample": desc}
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": max(3, args.warmup), "ms_per_step": statistics.mean(step_ms),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded W ~ N(0, 0.02^2), X lognormal channel scales with outliers)",
            "config": config_dict(args, wl, world),
            "breakdown_ms": {"hessian_syrk": syrk_ms, "prepare": statistics.mean(ms("prep")),
                             "quantize_sweep": quant_ms, "pack": statistics.mean(ms("pack"))},
            "syrk_tflops": syrk_tflops,
            # the same time counted as the full 2 d^2 N product (upper and lower triangle)
            "syrk_tflops_2d2n_equivalent": 2.0 * d * d * N / (syrk_ms * 1e-3) / 1e12,
            "sweep_gbs": sweep_bytes / (quant_ms * 1e-3) / 1e9,
            "roofline": {"bound": "tensor", "kernel": "syrk_bf16_tcgen05_kernel",
                         "achieved": syrk_tflops, "peak": bf16, "unit": "TFLOP/s",
                         "frac": syrk_tflops / bf16,
                         "traffic": syrk_traffic() if act.n_tokens == 262144 and d == 4096 else None,
                         "peak_source": f"{peak_kind} bf16 burst",
                         "algorithmic": f"d(d+1)N = {syrk_flops:.4g} flop per launch"},
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": statistics.mean(e2e_ms)},
            "gpu_launches": launches_per_step(d, q) * args.steps,
            "execution": "eager C ABI calls" if args.eager else
                         "CUDA graphs recorded from the C ABI calls, replayed",
            "clocks": clk.summary(),
            "cpu_baseline": cpu,
            "dequant_gemv": gemv,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
