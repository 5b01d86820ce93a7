"""Benchmark of the chunk-causal 3D-RoPE attention path on B200.

One step = one DiT-layer attention call (dz_chunk_attn_forward) on the
single-layer inference workload: B=1, 40 heads, head_dim 128, a 464-token noisy
chunk (2 latent frames of 11x20 tokens + 24 action tokens) over a KV cache of 4
clean chunks plus itself (2320 keys).  The call fuses the token metadata, the
3D rotary of q and of the chunk's own k, the tile classification, QK^T, the
online softmax, PV and the split-KV combine.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Prints ONE JSON line on rank 0.  Timing: K calls replayed from CUDA graphs
that cycle through enough distinct input sets to exceed the 126 MB L2, timed
with CUDA events on the launching stream between barriers + synchronize, max
over ranks.  ``--impl reference`` times the CPU fp64 oracle instead (bounded
samples of the same workload per step).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from causal_video_diffusion_rope_b200 import synth  # noqa: E402

METRIC = ("chunk-causal attn TFLOP/s and % of B200 BF16 peak; "
          "µs per DiT-layer attention call")
DEFAULT_WORKLOAD = 1  # single DiT-layer inference step
L2_BYTES = 126 * 1024 * 1024
KERNEL_SOURCES = ["causal_video_diffusion_rope_b200/csrc/dz_attn.cu",
                  "causal_video_diffusion_rope_b200/csrc/dz_internal.cuh",
                  "causal_video_diffusion_rope_b200/csrc/dz_ptx.cuh"]


def visible_pairs(w: synth.Workload) -> int:
    """Visible (query, key) pairs of one batch item and head of a call (chunk rule)."""
    lay = w.layout
    L = lay.chunk_len
    if lay.mode == synth.MODE_DECODE:
        return L * (w.cache_tokens + L)
    if lay.mode == synth.MODE_CROSS:
        return lay.q_len * lay.kv_len
    if lay.mode == synth.MODE_PREFILL:
        return sum(L * (c + 1) * L for c in range(lay.num_chunks))
    N = lay.num_chunks
    clean = sum(L * (i + 1) * L for i in range(N))
    noisy = sum(L * (i * L + L) for i in range(N))
    return clean + noisy


def step_flops(w: synth.Workload) -> float:
    """Algorithmic FLOPs of one step: 4 * head_dim per visible (query, key) pair per head per
    batch item, for the self-attention call plus, in the long-cache workload, the
    cross-attention call (every key visible)."""
    f = 4.0 * w.head_dim * visible_pairs(w) * w.heads * w.layout.batch
    if w.cross_kv_len:
        f += 4.0 * w.head_dim * w.layout.chunk_len * w.cross_kv_len * w.heads * w.layout.batch
    return f


def step_bytes(w: synth.Workload) -> float:
    """Bytes one step must move at least once: q, k, v, cached K/V, out (bf16), and the
    cross-attention q, condition k/v and out."""
    lay = w.layout
    row = w.heads * w.head_dim * 2 * lay.batch
    n = 3 * lay.q_len + 2 * w.cache_tokens + lay.q_len
    if w.cross_kv_len:
        n += 2 * lay.chunk_len + 2 * w.cross_kv_len
    return row * n


def launches_per_step(w: synth.Workload) -> int:
    """Kernels of this library one step launches: the once-per-call rotation of q and k and
    the attention kernel, plus the cross-attention kernel in the long-cache workload."""
    return 2 + (1 if w.cross_kv_len else 0)


def sources_hash() -> str:
    """Hash of the attention kernel's code (comments and blank space left out, so that
    an edited comment does not retire a profile taken on the same code)."""
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, f), encoding="utf-8") as fh:
            text = fh.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        h.update(" ".join(text.split()).encode())
    return h.hexdigest()[:16]


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d.get("bf16_tflops", 1590.0), d.get("hbm_gbs", 6650.0), "measured"
    return 1590.0, 6650.0, "fallback"


def ncu_traffic():
    """Per-launch DRAM bytes of the attention kernel from the committed ncu summary,
    or None if it was taken on different kernel sources."""
    path = os.path.join(ROOT, "profiles", "attn_decode_b1_h40_q464_cache4.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    if d.get("sources_hash") != sources_hash():
        return None
    return d.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clock / throttle sampling in the background."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.t_on = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------------- CPU legs

def oracle_rate(w: synth.Workload, inp, rng, budget_s: float, rows_per_call: int):
    """Time the fp64 oracle on sampled query rows of workload ``w`` until ``budget_s`` passes.

    Returns (TFLOP/s, calls, seconds); FLOPs are counted like the GPU's (4*D per visible pair).
    """
    from oracle import dz_oracle as O
    lay = w.layout
    keys = visible_pairs(w) / lay.q_len  # mean visible keys of a query row
    flops = 0.0
    calls = 0
    t0 = time.perf_counter()
    while True:
        rows = [(int(rng.integers(lay.batch)), int(rng.integers(lay.q_len)),
                 int(rng.integers(w.heads))) for _ in range(rows_per_call)]
        O.attention_rows(inp["q"], inp["k"], inp["v"], rows, lay.mode, lay.frames_per_chunk,
                         lay.grid_h, lay.grid_w, lay.n_action, lay.num_chunks,
                         t_offset=lay.t_offset, cache_k_bits=inp.get("cache_k"),
                         cache_v_bits=inp.get("cache_v"), cache_len=w.cache_tokens)
        flops += 4.0 * w.head_dim * keys * rows_per_call
        calls += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    return flops / dt / 1e12, calls, dt


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def oracle_full_call_rate(w: synth.Workload, budget_s: float):
    """The oracle computing whole calls of ``w`` (all heads) for about ``budget_s``."""
    from oracle import dz_oracle as O
    lay = w.layout
    inp = synth.make_inputs(w, 0)
    t0 = time.perf_counter()
    n = 0
    heads_done = 0
    # whole calls if they fit the budget, else head slices of one call
    while time.perf_counter() - t0 < budget_s:
        h = heads_done % w.heads
        O.chunk_attn_forward(inp["q"], inp["k"], inp["v"], lay.mode, lay.frames_per_chunk,
                             lay.grid_h, lay.grid_w, lay.n_action, lay.num_chunks,
                             t_offset=lay.t_offset, cache_k_bits=inp.get("cache_k"),
                             cache_v_bits=inp.get("cache_v"), cache_len=w.cache_tokens,
                             heads=slice(h, h + 4))
        heads_done += 4
        n += 1
    dt = time.perf_counter() - t0
    self_flops = 4.0 * w.head_dim * visible_pairs(w) * w.layout.batch
    flops = self_flops * heads_done
    return flops / dt / 1e12, heads_done, dt


# ----------------------------------------------------------------------------------- ranks

def max_over_ranks(ms: float, world: int, device) -> float:
    """The slowest rank's time: every rank's elapsed milliseconds reduced with MAX."""
    if world <= 1:
        return ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(flops_per_step: float, steps: int, world: int, max_ms: float) -> float:
    """Whole-job TFLOP/s: every rank runs `steps` independent calls (weak scaling);
    the job takes as long as its slowest rank."""
    return flops_per_step * steps * world / (max_ms * 1e-3) / 1e12


def e2e_pipelined(dev, stream, dev_inputs: dict, dev_outputs: dict, call, n_steps: int,
                  world: int) -> dict:
    """End-to-end steps through the public calls: every step copies its inputs in from
    pinned host memory and its results back out.  Two slots: while step i runs on
    `stream`, the inputs of step i+1 and the results of step i-1 cross PCIe on their
    own streams (event-ordered).  Returns ms for n_steps (max over ranks) and bytes."""
    import torch
    host_in = {k: t.cpu().pin_memory() for k, t in dev_inputs.items()}
    host_out = [{k: torch.empty_like(t, device="cpu").pin_memory() for k, t in dev_outputs.items()}
                for _ in range(2)]
    dev_in = [{k: torch.empty_like(t) for k, t in dev_inputs.items()} for _ in range(2)]
    dev_out = [{k: torch.empty_like(t) for k, t in dev_outputs.items()} for _ in range(2)]
    h2d_stream = torch.cuda.Stream(device=dev)
    d2h_stream = torch.cuda.Stream(device=dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]    # inputs of the slot landed
    ev_comp = [torch.cuda.Event() for _ in range(2)]  # the call is done with the slot
    ev_out = [torch.cuda.Event() for _ in range(2)]   # the slot's results are on the host
    step_no = [0]

    def step():
        i = step_no[0]
        sl = i % 2
        step_no[0] += 1
        if i >= 2:
            h2d_stream.wait_event(ev_comp[sl])
        with torch.cuda.stream(h2d_stream):
            for k in host_in:
                dev_in[sl][k].copy_(host_in[k], non_blocking=True)
            ev_in[sl].record(h2d_stream)
        stream.wait_event(ev_in[sl])
        if i >= 2:
            stream.wait_event(ev_out[sl])
        call(dev_in[sl], dev_out[sl])
        ev_comp[sl].record(stream)
        d2h_stream.wait_event(ev_comp[sl])
        with torch.cuda.stream(d2h_stream):
            for k in host_out[sl]:
                host_out[sl][k].copy_(dev_out[sl][k], non_blocking=True)
            ev_out[sl].record(d2h_stream)

    for _ in range(3):
        step()
    torch.cuda.synchronize(dev)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    x0 = torch.cuda.Event(enable_timing=True)
    x1 = torch.cuda.Event(enable_timing=True)
    x0.record(h2d_stream)
    stream.wait_event(x0)
    d2h_stream.wait_event(x0)
    for _ in range(n_steps):
        step()
    stream.wait_event(ev_out[(step_no[0] - 1) % 2])
    stream.wait_event(ev_out[step_no[0] % 2])
    x1.record(stream)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(x0.elapsed_time(x1), world, dev)
    return {"unit": "TFLOP/s", "ms": ms, "steps_done": n_steps,
            "h2d_bytes_per_step": int(sum(t.numel() * t.element_size() for t in host_in.values())),
            "d2h_bytes_per_step": int(sum(t.numel() * t.element_size()
                                          for t in host_out[0].values())),
            "pipelined": "inputs of step i+1 and the results of step i-1 cross PCIe while "
                         "step i runs",
            "ms_per_step": round(ms / n_steps, 4), "steps": n_steps}


# ----------------------------------------------------------------------------------- GPU leg

def run_gpu(args, rank: int, world: int, local_rank: int):
    import torch
    import torch.distributed as dist
    from causal_video_diffusion_rope_b200 import dz

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = synth.WORKLOADS[args.workload]
    lay = w.layout
    B, H, D, L = lay.batch, w.heads, w.head_dim, lay.chunk_len
    per_set = step_bytes(w)
    n_sets = max(2, int(math.ceil(3 * L2_BYTES / per_set)))
    # q and the chunk's own k are rotated once per call (prerotate_tokens) before the
    # attention kernel; cache keys are stored rotated
    h = dz.dz_attn_create(dz.make_desc(num_heads=H, max_batch=B, max_q_tokens=lay.q_len,
                                       prerotate_tokens=lay.q_len))
    dl = dz.layout_from(lay)
    dlx = dz.layout_from(synth.cross_layout(w)) if w.cross_kv_len else None
    sets = []
    for i in range(n_sets):
        inp = synth.make_inputs(w, 1000 * rank + i)
        s = {k: torch.from_numpy(inp[k].view(np.int16)).to(dev).view(torch.bfloat16)
             for k in ("q", "k", "v", "cache_k", "cache_v", "q_x", "k_x", "v_x") if k in inp}
        s["out"] = torch.empty((B, lay.q_len, H, D), dtype=torch.bfloat16, device=dev)
        s["cache"] = (dz.make_cache(s["cache_k"], s["cache_v"], B, w.cache_tokens,
                                    w.cache_tokens, L) if "cache_k" in s else None)
        if w.cross_kv_len:
            s["out_x"] = torch.empty((B, L, H, D), dtype=torch.bfloat16, device=dev)
        sets.append(s)
    stream = torch.cuda.Stream(device=dev)

    def call(i):
        s = sets[i % n_sets]
        dz.dz_chunk_attn_forward(h, s["q"], s["k"], s["v"], s["cache"], dl, s["out"], stream)
        if dlx is not None:
            dz.dz_chunk_attn_forward(h, s["q_x"], s["k_x"], s["v_x"], None, dlx, s["out_x"],
                                     stream)

    # warm-up outside any graph
    with torch.cuda.stream(stream):
        for i in range(max(args.warmup, 3)):
            call(i)
    stream.synchronize()
    dz.dz_attn_sync_status(h, stream)

    # graphs of g calls cycling through the input sets
    g = n_sets * max(1, 240 // n_sets)
    graphs = {}

    def graph_of(n):
        if n not in graphs:
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr, stream=stream):
                for i in range(n):
                    call(i)
            graphs[n] = gr
        return graphs[n]

    full, rem = divmod(args.steps, g)
    if full:
        graph_of(g)
    if rem:
        graph_of(rem)
    # warm the graphs once
    with torch.cuda.stream(stream):
        if full:
            graphs[g].replay()
        if rem:
            graphs[rem].replay()
    stream.synchronize()

    sampler = ClockSampler(local_rank if "CUDA_VISIBLE_DEVICES" not in os.environ else 0)
    sampler.start()
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(full):
            graphs[g].replay()
        if rem:
            graphs[rem].replay()
        e1.record(stream)
    stream.synchronize()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    ms = e0.elapsed_time(e1)
    dz.dz_attn_sync_status(h, stream)
    ms = max_over_ranks(ms, world, dev)
    ms_per_step = ms / args.steps
    flops = step_flops(w)
    tflops_total = job_throughput(flops, args.steps, world, ms)

    # ---- end to end: host buffers in, result out, through the same C-ABI calls
    s0 = sets[0]
    in_keys = [k for k in ("q", "k", "v", "q_x", "k_x", "v_x") if k in s0]
    out_keys = [k for k in ("out", "out_x") if k in s0]

    def e2e_call(di, do):
        dz.dz_chunk_attn_forward(h, di["q"], di["k"], di["v"], s0["cache"], dl, do["out"], stream)
        if dlx is not None:
            dz.dz_chunk_attn_forward(h, di["q_x"], di["k_x"], di["v_x"], None, dlx,
                                     do["out_x"], stream)

    e2e = e2e_pipelined(dev, stream, {k: s0[k] for k in in_keys}, {k: s0[k] for k in out_keys},
                        e2e_call, max(3, min(args.steps, 200)), world)
    dz.dz_attn_sync_status(h, stream)
    e2e["value"] = round(job_throughput(flops, e2e.pop("steps_done"), world, e2e.pop("ms")), 3)

    for gr in graphs.values():
        del gr
    graphs.clear()
    dz.dz_attn_destroy(h)
    return ms_per_step, tflops_total, clocks, e2e


QKV_METRIC = ("fused QKV projection + 3D RoPE TFLOP/s and % of B200 BF16 peak; "
              "\u00b5s per DiT-layer projection of one chunk")
D_MODEL = 5120  # hidden size of the 14B DiT


def qkv_flops(w) -> float:
    lay = w.layout
    return 2.0 * lay.batch * lay.chunk_len * D_MODEL * 3 * w.heads * w.head_dim


def time_graph(stream, call, steps: int, warmup: int, world: int, dev, sampler=None):
    """Device time (ms, max over ranks) of `steps` calls replayed from CUDA graphs of up to
    240 calls, after `warmup` plain calls and one replay of each graph."""
    import torch
    with torch.cuda.stream(stream):
        for i in range(warmup):
            call(i)
    stream.synchronize()
    g = min(240, steps)
    full, rem = divmod(steps, g)
    graphs = {}
    for n in ([g] if full else []) + ([rem] if rem else []):
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=stream):
            for i in range(n):
                call(i)
        graphs[n] = gr
    with torch.cuda.stream(stream):
        for gr in graphs.values():
            gr.replay()
    stream.synchronize()
    if sampler:
        sampler.start()
        time.sleep(0.3)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(full):
            graphs[g].replay()
        if rem:
            graphs[rem].replay()
        e1.record(stream)
    stream.synchronize()
    clocks = sampler.stop() if sampler else None
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    graphs.clear()
    return ms, clocks


def run_qkv(args, rank: int, world: int, local_rank: int, config: dict):
    """Times dz_qkv_rope on one chunk of the workload (d_model 5120, random weights)."""
    import torch
    from causal_video_diffusion_rope_b200 import dz
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = synth.WORKLOADS[args.workload]
    lay = w.layout
    B, H, D, S = lay.batch, w.heads, w.head_dim, lay.chunk_len
    h = dz.dz_attn_create(dz.make_desc(num_heads=H, max_batch=B))
    dl = dz.layout_from(lay)
    first = lay.num_chunks if lay.mode == synth.MODE_DECODE else 0
    xs, W = [], None
    for i in range(2):
        xb, wb = synth.projection_inputs(1000 * rank + i, B, S, D_MODEL, H)
        xs.append(torch.from_numpy(xb.view(np.int16)).to(dev).view(torch.bfloat16))
        if W is None:
            W = torch.from_numpy(wb.view(np.int16)).to(dev).view(torch.bfloat16)
    q = torch.empty((B, S, H, D), dtype=torch.bfloat16, device=dev)
    k, v = torch.empty_like(q), torch.empty_like(q)
    stream = torch.cuda.Stream(device=dev)

    def call(i):
        dz.dz_qkv_rope(h, xs[i % 2], W, B, S, D_MODEL, dl, first, q, k, v, None, stream)

    sampler = ClockSampler(local_rank if "CUDA_VISIBLE_DEVICES" not in os.environ else 0)
    ms, clocks = time_graph(stream, call, args.steps, args.warmup, world, dev, sampler)
    dz.dz_attn_sync_status(h, stream)
    ms_per_step = ms / args.steps
    flops = qkv_flops(w)

    # context: cuBLAS (torch.matmul) on the same GEMM alone, no rotation, same timing
    x2 = [x.view(B * S, D_MODEL) for x in xs]
    y = torch.empty((B * S, 3 * H * D), dtype=torch.bfloat16, device=dev)

    def call_ref(i):
        torch.matmul(x2[i % 2], W.t(), out=y)

    ms_ref, _ = time_graph(stream, call_ref, min(args.steps, 2400), 3, world, dev)
    ref_us = 1e3 * ms_ref / min(args.steps, 2400)

    def e2e_call(di, do):
        dz.dz_qkv_rope(h, di["x"], W, B, S, D_MODEL, dl, first, do["q"], do["k"], do["v"],
                       None, stream)

    e2e = e2e_pipelined(dev, stream, {"x": xs[0]}, {"q": q, "k": k, "v": v}, e2e_call,
                        max(3, min(args.steps, 200)), world)
    e2e["value"] = round(job_throughput(flops, e2e.pop("steps_done"), world, e2e.pop("ms")), 3)
    dz.dz_attn_sync_status(h, stream)
    dz.dz_attn_destroy(h)
    if rank != 0:
        return
    peak_tf, _, peak_kind = measured_peaks()
    per_gpu = flops / (ms_per_step * 1e-3) / 1e12
    line = {"metric": QKV_METRIC, "value": round(job_throughput(flops, args.steps, world, ms), 3),
            "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms_per_step, 6), "us_per_call": round(ms_per_step * 1e3, 3),
            "pct_of_bf16_peak": round(100 * per_gpu / peak_tf, 2),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (x ~ N(0,1), random-init W ~ N(0, 1/5120))",
            "config": dict(config, op="qkv_rope", d_model=D_MODEL, tokens=B * S,
                           out_features=3 * H * D, flop_per_step=flops,
                           l2="the 157 MB weight alone exceeds the 126 MB L2",
                           parallelism=f"dp{world} (independent replicas of the call)"),
            "roofline": {"bound": "tensor", "achieved": round(per_gpu, 2), "peak": peak_tf,
                         "unit": "TFLOP/s", "frac": round(per_gpu / peak_tf, 4), "traffic": None,
                         "peak_kind": f"{peak_kind} bf16 (burst)", "kernel": "qkv_rope_kernel"},
            "context": {"cublas_same_gemm_us": round(ref_us, 3),
                        "cublas_same_gemm_tflops": round(flops / (ref_us * 1e-6) / 1e12, 2)},
            "cpu_baseline": None, "e2e": e2e, "gpu_launches": args.steps, "clocks": clocks}
    print(json.dumps(line), flush=True)


BWD_METRIC = ("chunk-causal attention backward TFLOP/s (dq, dk, dv; algorithmic 2.5x the "
              "forward's visible-pair FLOP) and % of B200 BF16 peak; \u00b5s per call")


def run_bwd(args, rank: int, world: int, local_rank: int, config: dict):
    """Times dz_chunk_attn_backward on a prefill / teacher-forcing workload."""
    import torch
    from causal_video_diffusion_rope_b200 import dz
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = synth.WORKLOADS[args.workload]
    lay = w.layout
    if lay.mode not in (synth.MODE_PREFILL, synth.MODE_TEACHER_FORCING):
        raise SystemExit("--op bwd needs a prefill or teacher-forcing workload (e.g. --workload 3)")
    B, H, D, S = lay.batch, w.heads, w.head_dim, lay.q_len
    h = dz.dz_attn_create(dz.make_desc(num_heads=H, max_batch=B, max_q_tokens=S,
                                       prerotate_tokens=S))
    dl = dz.layout_from(lay)
    rng = np.random.default_rng(1000 * rank + 7)

    def dev_bf16(a):
        return torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)

    q, k, v, dout = (dev_bf16(synth.normal_bf16(rng, (B, S, H, D))) for _ in range(4))
    out = torch.empty_like(q)
    lse = torch.empty((B, H, S), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    stream = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(stream):
        dz.dz_chunk_attn_forward_lse(h, q, k, v, dl, out, lse, stream)

    def call(i):
        dz.dz_chunk_attn_backward(h, q, k, v, out, dout, lse, dl, dq, dk, dv, stream)

    sampler = ClockSampler(local_rank if "CUDA_VISIBLE_DEVICES" not in os.environ else 0)
    ms, clocks = time_graph(stream, call, args.steps, args.warmup, world, dev, sampler)
    dz.dz_attn_sync_status(h, stream)
    ms_per_step = ms / args.steps
    flops = 2.5 * step_flops(w)

    def e2e_call(di, do):
        dz.dz_chunk_attn_backward(h, di["q"], di["k"], di["v"], di["out"], di["dout"], di["lse"],
                                  dl, do["dq"], do["dk"], do["dv"], stream)

    e2e = e2e_pipelined(dev, stream, {"q": q, "k": k, "v": v, "out": out, "dout": dout, "lse": lse},
                        {"dq": dq, "dk": dk, "dv": dv}, e2e_call, max(3, min(args.steps, 20)), world)
    e2e["value"] = round(job_throughput(flops, e2e.pop("steps_done"), world, e2e.pop("ms")), 3)
    dz.dz_attn_sync_status(h, stream)
    dz.dz_attn_destroy(h)
    if rank != 0:
        return
    peak_tf, _, peak_kind = measured_peaks()
    per_gpu = flops / (ms_per_step * 1e-3) / 1e12
    line = {"metric": BWD_METRIC, "value": round(job_throughput(flops, args.steps, world, ms), 3),
            "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms_per_step, 6), "us_per_call": round(ms_per_step * 1e3, 3),
            "pct_of_bf16_peak": round(100 * per_gpu / peak_tf, 2),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (q, k, v, dO ~ N(0,1))",
            "config": dict(config, op="backward", flop_per_step=flops,
                           l2=f"q, k, v, out, dO: {5 * B * S * H * D * 2 / 2**20:.0f} MiB > 126 MB L2",
                           parallelism=f"dp{world} (independent replicas of the call)"),
            "roofline": {"bound": "tensor", "achieved": round(per_gpu, 2), "peak": peak_tf,
                         "unit": "TFLOP/s", "frac": round(per_gpu / peak_tf, 4), "traffic": None,
                         "peak_kind": f"{peak_kind} bf16 (burst)",
                         "kernel": "bwd_dq_kernel + bwd_dkv_kernel"},
            "cpu_baseline": None, "e2e": e2e, "gpu_launches": 4 * args.steps, "clocks": clocks}
    print(json.dumps(line), flush=True)


CACHE_METRIC = "KV-cache chunk replace GB/s (keys + values read and written) and % of measured HBM copy bandwidth"


def run_cache(args, rank: int, world: int, local_rank: int, config: dict):
    """Times dz_kvcache_replace of one chunk (every batch item's K and V rows) on the
    workload's cache; the replaced chunk and the source set cycle, so the traffic
    (> L2 in all) goes to HBM."""
    import torch
    from causal_video_diffusion_rope_b200 import dz
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = synth.WORKLOADS[args.workload]
    lay = w.layout
    if not w.cache_tokens:
        raise SystemExit("--op cache needs a workload with a KV cache (e.g. --workload 2)")
    B, H, D, L = lay.batch, w.heads, w.head_dim, lay.chunk_len
    n_chunks = w.cache_tokens // L
    h = dz.dz_attn_create(dz.make_desc(num_heads=H, max_batch=B))
    ck = torch.zeros((B, w.cache_tokens, H, D), dtype=torch.bfloat16, device=dev)
    cv = torch.zeros_like(ck)
    cache = dz.make_cache(ck, cv, B, w.cache_tokens, w.cache_tokens, L)
    rng = np.random.default_rng(1000 * rank + 11)
    srcs = [tuple(torch.from_numpy(synth.normal_bf16(rng, (B, L, H, D)).view(np.int16)).to(dev)
                  .view(torch.bfloat16) for _ in range(2)) for _ in range(4)]
    stream = torch.cuda.Stream(device=dev)

    def call(i):
        k, v = srcs[i % len(srcs)]
        dz.dz_kvcache_replace(h, cache, i % n_chunks, k, v, stream)

    sampler = ClockSampler(local_rank if "CUDA_VISIBLE_DEVICES" not in os.environ else 0)
    ms, clocks = time_graph(stream, call, args.steps, args.warmup, world, dev, sampler)
    dz.dz_attn_sync_status(h, stream)
    bytes_per = 2 * 2 * B * L * H * D * 2  # K and V, read and written
    ms_per_step = ms / args.steps
    gbs = bytes_per / (ms_per_step * 1e-3) / 1e9

    def e2e_call(di, do):
        dz.dz_kvcache_replace(h, cache, n_chunks - 1, di["k"], di["v"], stream)
        with torch.cuda.stream(stream):
            do["k_row"].copy_(ck[:, -1, 0, :8])

    e2e = e2e_pipelined(dev, stream, {"k": srcs[0][0], "v": srcs[0][1]},
                        {"k_row": torch.empty((B, 8), dtype=torch.bfloat16, device=dev)},
                        e2e_call, max(3, min(args.steps, 200)), world)
    e2e_ms = e2e.pop("ms")
    e2e["value"] = round(bytes_per * e2e.pop("steps_done") * world / (e2e_ms * 1e-3) / 1e9, 2)
    e2e["unit"] = "GB/s"
    dz.dz_attn_destroy(h)
    if rank != 0:
        return
    _, peak_hbm, peak_kind = measured_peaks()
    line = {"metric": CACHE_METRIC, "value": round(gbs * world, 2), "unit": "GB/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms_per_step, 6), "us_per_call": round(ms_per_step * 1e3, 3),
            "pct_of_hbm_peak": round(100 * gbs / peak_hbm, 2), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16 (bit copy)",
            "data": "synthetic (N(0,1) bf16 observations)",
            "config": dict(config, op="kvcache_replace", bytes_per_step=bytes_per,
                           l2=f"cache {2 * B * w.cache_tokens * H * D * 2 / 2**20:.0f} MiB + "
                              f"4 source sets, replaced chunk cycling: > 126 MB L2",
                           parallelism=f"dp{world} (independent replicas of the call)"),
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peak_hbm,
                         "unit": "GB/s", "frac": round(gbs / peak_hbm, 4), "traffic": None,
                         "peak_kind": f"{peak_kind} copy", "kernel": "kv_copy_kernel"},
            "cpu_baseline": None, "e2e": e2e, "gpu_launches": args.steps, "clocks": clocks}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=48000)
    ap.add_argument("--warmup", type=int, default=240)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=15.0,
                    help="seconds of oracle CPU work for the cpu_baseline field")
    ap.add_argument("--op", default="attn", choices=["attn", "qkv", "bwd", "cache"],
                    help="attn: the chunk-causal attention call; qkv: the fused projection; "
                         "bwd: the backward of a prefill / teacher-forcing call; "
                         "cache: the KV-cache chunk replace")
    ap.add_argument("--workload", type=int, default=DEFAULT_WORKLOAD,
                    choices=range(len(synth.WORKLOADS)),
                    help="workload index (default: the single-layer inference step)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    w = synth.WORKLOADS[args.workload]
    config = {"workload": w.name, "batch": w.layout.batch, "heads": w.heads,
              "head_dim": w.head_dim, "q_tokens": w.layout.q_len,
              "keys": w.cache_tokens + w.layout.self_kv_len, "cache_tokens": w.cache_tokens,
              "mode": synth.MODE_NAMES[w.layout.mode],
              "cross_keys": w.cross_kv_len,
              "rope": "3d t/h/w 22/21/21 base 1e4; q and the chunk's k rotated once per call",
              "flop_per_step": step_flops(w)}

    if args.op in ("qkv", "bwd", "cache"):
        if args.impl == "reference":
            if rank == 0:
                print(json.dumps({"impl": "reference", "unavailable": "the reference arm times "
                                  "the attention call (--op attn) only"}), flush=True)
            return
        import torch.distributed as dist
        if world > 1:
            import datetime
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        {"qkv": run_qkv, "bwd": run_bwd, "cache": run_cache}[args.op](args, rank, world,
                                                                     local_rank, config)
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()
        return

    if args.impl == "reference":
        if rank != 0:
            return
        budget = 150.0 / (args.steps + args.warmup)
        # each step: the oracle on a bounded sample of query rows of the same call
        rows_per_step = 1
        rate = []
        t_all = time.perf_counter()
        inp = synth.make_inputs(w, 0)
        rng = np.random.default_rng(0)
        for i in range(args.warmup + args.steps):
            r, calls, dt = oracle_rate(w, inp, rng, budget, rows_per_step)
            if i >= args.warmup:
                rate.append((r, dt))
        elapsed = sum(dt for _, dt in rate)
        value = float(np.mean([r for r, _ in rate]))
        cores = blas_threads()
        line = {"impl": "reference", "metric": METRIC, "value": round(value, 6),
                "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": round(1e3 * elapsed / max(1, len(rate)), 3),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "config": dict(config, l2="n/a (CPU)"),
                "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": cores,
                                 "kind": "oracle",
                                 "sample": f"{rows_per_step} query row(s) of the call per step, "
                                           f"~{budget * 1e3:.1f} ms of oracle work per step"},
                "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0},
                "wall_s": round(time.perf_counter() - t_all, 1)}
        print(json.dumps(line), flush=True)
        return

    import torch
    import torch.distributed as dist
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    cpu = None
    if rank == 0 and world == 1 and args.cpu_budget > 0:
        # the oracle, timed on this host's cores before the GPU work starts
        r, heads_done, dt = oracle_full_call_rate(w, args.cpu_budget)
        cpu = {"value": round(r, 6), "unit": "TFLOP/s", "cores": blas_threads(),
               "kind": "oracle",
               "sample": f"{heads_done} of {w.heads} heads of the call (4-head slices), "
                         f"{dt:.1f} s of fp64 oracle work"}
    ms_per_step, tflops, clocks, e2e = run_gpu(args, rank, world, local_rank)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    peak_tf, peak_hbm, peak_kind = measured_peaks()
    per_gpu_tf = step_flops(w) / (ms_per_step * 1e-3) / 1e12
    roof = {"bound": "tensor", "achieved": round(per_gpu_tf, 2), "peak": peak_tf,
            "unit": "TFLOP/s", "frac": round(per_gpu_tf / peak_tf, 4),
            "traffic": ncu_traffic(), "peak_kind": f"{peak_kind} bf16 (burst)",
            "kernel": "chunk_attn_kernel",
            "hbm_frac": round(step_bytes(w) / (ms_per_step * 1e-3) / 1e9 / peak_hbm, 4)}
    n_sets = max(2, int(math.ceil(3 * L2_BYTES / step_bytes(w))))
    line = {"metric": METRIC, "value": round(tflops, 3), "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms_per_step, 6), "us_per_call": round(ms_per_step * 1e3, 3),
            "pct_of_bf16_peak": round(100 * per_gpu_tf / peak_tf, 2),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": dict(config, l2=f"inputs cycle through {n_sets} sets "
                                      f"({n_sets * step_bytes(w) / 2**20:.0f} MiB > 126 MB L2)",
                           parallelism=f"dp{world} (independent replicas of the call)"),
            "roofline": roof, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": args.steps * launches_per_step(w), "clocks": clocks}
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
