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
over ranks.  At N=1 the line also carries a `workloads` block with the other
full-size workloads (CFG decode with its cache replace, teacher forcing, long
cache + cross-attention, three-view decode) timed the same way.

With --gpus N and no launcher environment (WORLD_SIZE unset) the script starts
N rank processes itself, one per GPU.  Ranks share no data: on a workload whose
batch equals N (the CFG branches), rank r runs branch r's batch-1 calls against
its own half of the cache (the two-GPU CFG split); otherwise every rank runs
its own replica of the call.  ``--impl reference`` times the CPU fp64 oracle
instead (bounded samples of the same workload per step).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import socket
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
EXTRA_WORKLOADS = (2, 3, 4, 5)
L2_BYTES = 126 * 1024 * 1024
SPEC_BF16_TFLOPS = 2250.0  # B200 dense bf16, the figure the throughput aim is stated against
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


def self_flops(w: synth.Workload) -> float:
    """Algorithmic FLOPs of the self-attention call: 4 * head_dim per visible (query, key)
    pair per head per batch item."""
    return 4.0 * w.head_dim * visible_pairs(w) * w.heads * w.layout.batch


def cross_flops(w: synth.Workload) -> float:
    """Algorithmic FLOPs of the cross-attention call (every condition key visible)."""
    return 4.0 * w.head_dim * w.layout.chunk_len * w.cross_kv_len * w.heads * w.layout.batch


def step_flops(w: synth.Workload) -> float:
    """Algorithmic FLOPs of one step: the self-attention call plus, in the long-cache
    workload, the cross-attention call."""
    return self_flops(w) + (cross_flops(w) if w.cross_kv_len else 0.0)


def step_bytes(w: synth.Workload) -> float:
    """Bytes one step must move at least once: q, k, v, cached K/V, out (bf16), and the
    cross-attention q, condition k/v and out."""
    lay = w.layout
    row = w.heads * w.head_dim * 2 * lay.batch
    n = 3 * lay.q_len + 2 * w.cache_tokens + lay.q_len
    if w.cross_kv_len:
        n += 2 * lay.chunk_len + 2 * w.cross_kv_len
    return row * n


def launches_per_step(w: synth.Workload, rotation_pass: bool) -> int:
    """Kernels of this library one step launches: the attention kernel (plus the
    once-per-call rotation of q and k when it runs as its own pass), plus the
    cross-attention kernel in the long-cache workload."""
    return 1 + (1 if rotation_pass else 0) + (1 if w.cross_kv_len else 0)


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


def ncu_traffic(workload_name: str):
    """Per-launch DRAM bytes of the attention kernel on a workload from the committed ncu
    summary (profiles/attn_<workload>.json; the E4M3 variant's as attn_e4m3_<workload>),
    or None if there is none or it was taken on different kernel sources."""
    path = os.path.join(ROOT, "profiles", f"attn_{workload_name}.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    if d.get("sources_hash") != sources_hash():
        return None
    return d.get("dram_bytes_per_launch")


def cpu_info():
    """CPU model name and the cores this process may run on."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    try:
        cores = len(os.sched_getaffinity(0))
    except AttributeError:
        cores = os.cpu_count()
    return model, cores


def gpu_id(local_rank: int) -> str:
    """nvidia-smi --id of this rank's GPU: its UUID (the leased GPU, whatever
    CUDA_VISIBLE_DEVICES maps it to), else the CUDA_VISIBLE_DEVICES entry, else the index."""
    try:
        import torch
        u = str(torch.cuda.get_device_properties(local_rank).uuid)
        if u:
            return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        pass
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        entries = [e.strip() for e in vis.split(",") if e.strip()]
        if local_rank < len(entries):
            return entries[local_rank]
    return str(local_rank)


class ClockSampler:
    """nvidia-smi clock / throttle sampling of one GPU in the background."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu: str):
        self.gpu = gpu
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"],
                    "gpu": self.gpu}
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
                "reasons": sorted(reasons), "samples": len(sm), "gpu": self.gpu}


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


def cpu_baseline_fields(value: float, sample: str) -> dict:
    """cpu_baseline object: `cores` = the threads the oracle's matrix products ran on
    (the BLAS pool, bounded by this process's CPU affinity), with the affinity core
    count and the CPU model beside it."""
    model, avail = cpu_info()
    used = min(blas_threads(), avail) if avail else blas_threads()
    return {"value": round(value, 6), "unit": "TFLOP/s", "cores": used,
            "cores_available": avail, "cpu_model": model, "kind": "oracle", "sample": sample}


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
    flops = visible_pairs(w) * 4.0 * w.head_dim * w.layout.batch * heads_done
    return flops / dt / 1e12, heads_done, dt


# ----------------------------------------------------------------------------------- ranks

def free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def spawn_ranks(n: int, target, *args) -> None:
    """Run ``target(*args)`` in ``n`` fresh processes (spawn), one per GPU rank, with the
    launcher environment a rank expects (RANK, LOCAL_RANK, WORLD_SIZE, MASTER_ADDR,
    MASTER_PORT); raises if any rank fails."""
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    port = free_port()
    procs = [ctx.Process(target=_rank_entry, args=(r, n, port, target, args)) for r in range(n)]
    for p in procs:
        p.start()
    for p in procs:
        p.join()
    bad = [(r, p.exitcode) for r, p in enumerate(procs) if p.exitcode != 0]
    if bad:
        raise RuntimeError(f"rank processes failed: {bad}")


def _rank_entry(rank: int, world: int, port: int, target, args) -> None:
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    target(*args)


def rank_work(w: synth.Workload, rank: int, world: int):
    """What one rank runs of workload ``w``: ("cfg", r) -- branch r of a batch whose items
    are the CFG branches, one rank per branch (world == batch > 1) -- or ("replica", None),
    its own copy of the whole call."""
    if world > 1 and w.layout.batch == world:
        return "cfg", rank
    return "replica", None


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
    """Whole-job TFLOP/s: every rank runs `steps` calls of `flops_per_step` each; the job
    takes as long as its slowest rank."""
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
    torch.cuda.synchronize()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    clocks = sampler.stop() if sampler else None
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    graphs.clear()
    return ms, clocks


# ----------------------------------------------------------------------------------- GPU legs

class AttnSetup:
    """Handle, input sets and layouts of one workload's attention calls on this rank.

    Input sets cycle so that one pass over them exceeds the L2 (every call reads its
    q, k, v and cache from HBM).  ``branch`` selects one batch item of the workload
    (a CFG branch, with its own half of the cache); the seeds do not depend on the
    rank in that case, so the ranks together run exactly the batch-2 call."""

    def __init__(self, w: synth.Workload, dev, seed_base: int, rotation_pass: bool,
                 branch=None, max_sets=None):
        import torch
        from causal_video_diffusion_rope_b200 import dz
        self.dz = dz
        self.w_full = w
        self.w = w if branch is None else synth.branch_inputs(w, {}, branch)[0]
        lay = self.w.layout
        B, H, D, L = lay.batch, w.heads, w.head_dim, lay.chunk_len
        self.n_sets = max(2, int(math.ceil(3 * L2_BYTES / step_bytes(self.w))))
        if max_sets:
            self.n_sets = min(self.n_sets, max_sets)
        self.h = dz.dz_attn_create(dz.make_desc(num_heads=H, max_batch=B, max_q_tokens=lay.q_len,
                                                prerotate_tokens=lay.q_len if rotation_pass else 0))
        self.dl = dz.layout_from(lay)
        self.dlx = dz.layout_from(synth.cross_layout(self.w)) if w.cross_kv_len else None
        self.sets = []
        for i in range(self.n_sets):
            inp = synth.make_inputs(w, seed_base + i)
            if branch is not None:
                inp = synth.branch_inputs(w, inp, branch)[1]
            s = {k: torch.from_numpy(np.ascontiguousarray(inp[k]).view(np.int16)).to(dev)
                 .view(torch.bfloat16)
                 for k in ("q", "k", "v", "cache_k", "cache_v", "q_x", "k_x", "v_x") if k in inp}
            s["out"] = torch.empty((B, lay.q_len, H, D), dtype=torch.bfloat16, device=dev)
            s["cache"] = (dz.make_cache(s["cache_k"], s["cache_v"], B, self.w.cache_tokens,
                                        self.w.cache_tokens, L) if "cache_k" in s else None)
            if w.cross_kv_len:
                s["out_x"] = torch.empty((B, L, H, D), dtype=torch.bfloat16, device=dev)
            self.sets.append(s)

    def call(self, i, stream, part="step"):
        """One step on input set i: the self-attention call, plus the cross-attention call
        of the long-cache workload (part: "step" both, "self" or "cross" one of them)."""
        s = self.sets[i % self.n_sets]
        if part in ("step", "self"):
            self.dz.dz_chunk_attn_forward(self.h, s["q"], s["k"], s["v"], s["cache"], self.dl,
                                          s["out"], stream)
        if self.dlx is not None and part in ("step", "cross"):
            self.dz.dz_chunk_attn_forward(self.h, s["q_x"], s["k_x"], s["v_x"], None, self.dlx,
                                          s["out_x"], stream)

    def prepare_rotated(self, stream):
        """Rotated copies of every set's q and k (dz_rope3d, the rotation the call applies),
        for timing the attention kernel alone on DZ_MODE_ROTATED calls."""
        import torch
        lay = self.w.layout
        L, N = lay.chunk_len, lay.num_chunks
        self.dl_rot = self.dz.layout_from(lay)
        if lay.mode != synth.MODE_CROSS:
            self.dl_rot.mode = lay.mode | self.dz.DZ_MODE_ROTATED
        for s in self.sets:
            if lay.mode == synth.MODE_CROSS:
                s["qr"], s["kr"] = s["q"], s["k"]
                continue
            s["qr"], s["kr"] = torch.empty_like(s["q"]), torch.empty_like(s["k"])
            for x, y in ((s["q"], s["qr"]), (s["k"], s["kr"])):
                if lay.mode == synth.MODE_DECODE:
                    self.dz.dz_rope3d(self.h, x, y, lay.batch, L, self.dl, N, stream)
                elif lay.mode == synth.MODE_PREFILL:
                    self.dz.dz_rope3d(self.h, x, y, lay.batch, N * L, self.dl, 0, stream)
                else:  # teacher forcing: the noisy half sits at the clean half's positions
                    for b in range(lay.batch):
                        for h0 in (0, N * L):
                            self.dz.dz_rope3d(self.h, x[b:b + 1, h0:h0 + N * L],
                                              y[b:b + 1, h0:h0 + N * L], 1, N * L, self.dl, 0,
                                              stream)
        stream.synchronize()

    def kernel_call(self, i, stream):
        """The self-attention call on pre-rotated q, k: the attention kernel alone."""
        s = self.sets[i % self.n_sets]
        self.dz.dz_chunk_attn_forward(self.h, s["qr"], s["kr"], s["v"], s["cache"], self.dl_rot,
                                      s["out"], stream)

    def close(self):
        self.dz.dz_attn_sync_status(self.h)
        self.dz.dz_attn_destroy(self.h)
        self.sets.clear()


def extra_workload_block(wl: int, dev, stream, steps: int, peak_tf: float, peak_hbm: float,
                         rotation_pass: bool):
    """Timing of one more full-size workload (N=1), the headline's discipline: graphs of
    calls cycling input sets above L2, CUDA events on the launching stream."""
    import torch
    w = synth.WORKLOADS[wl]
    st = AttnSetup(w, dev, 2000 + 100 * wl, rotation_pass=rotation_pass, max_sets=3)
    n = max(20, min(steps, 240))
    res = {"workload": w.name, "mode": synth.MODE_NAMES[w.layout.mode],
           "batch": w.layout.batch, "q_tokens": w.layout.q_len,
           "keys": w.cache_tokens + w.layout.self_kv_len, "calls": n,
           "l2": f"{st.n_sets} input sets of {step_bytes(w) / 2**20:.0f} MiB cycle"}
    ms, _ = time_graph(stream, lambda i: st.call(i, stream), n, 3, 1, dev)
    us = 1e3 * ms / n
    tf = step_flops(w) / (us * 1e-6) / 1e12
    res.update(us_per_call=round(us, 3), tflops=round(tf, 2), frac=round(tf / peak_tf, 4),
               frac_of_spec=round(tf / SPEC_BF16_TFLOPS, 4), flop_per_call=step_flops(w),
               traffic=ncu_traffic(w.name))
    if w.cross_kv_len:
        for part, fl in (("self", self_flops(w)), ("cross", cross_flops(w))):
            ms, _ = time_graph(stream, lambda i, part=part: st.call(i, stream, part), n, 3, 1, dev)
            pus = 1e3 * ms / n
            ptf = fl / (pus * 1e-6) / 1e12
            res[part] = {"us_per_call": round(pus, 3), "tflops": round(ptf, 2),
                         "frac": round(ptf / peak_tf, 4), "flop_per_call": fl}
    if w.denoise_steps > 1 and st.sets[0]["cache"] is not None:
        # the request boundary: the observed chunk replaces the last cached chunk
        dz = st.dz
        lay = w.layout
        L = lay.chunk_len
        srcs = [(torch.randn((lay.batch, L, w.heads, w.head_dim), device=dev).to(torch.bfloat16),
                 torch.randn((lay.batch, L, w.heads, w.head_dim), device=dev).to(torch.bfloat16))
                for _ in range(4)]
        last = w.cache_tokens // L - 1

        def rep(i):
            s = st.sets[i % st.n_sets]
            k, v = srcs[i % len(srcs)]
            dz.dz_kvcache_replace(st.h, s["cache"], last, k, v, stream)

        ms, _ = time_graph(stream, rep, n, 3, 1, dev)
        rus = 1e3 * ms / n
        moved = 2 * 2 * lay.batch * L * w.heads * w.head_dim * 2  # K and V, read and written
        res["replace"] = {"us_per_call": round(rus, 3), "bytes": moved,
                          "gbs": round(moved / (rus * 1e-6) / 1e9, 1),
                          "frac_of_hbm": round(moved / (rus * 1e-6) / 1e9 / peak_hbm, 4)}
    st.close()
    del st
    torch.cuda.empty_cache()
    return res


E4M3_WORKLOADS = (1, 2, 3, 4, 5)
E4M3_METRIC = ("chunk-causal attention with E4M3 QK^T TFLOP/s and % of the B200 mixed "
               "E4M3/BF16 peak; \u00b5s per DiT-layer attention call")


class E4m3Setup:
    """Handle and input sets of workload w's self-attention in the FP8 variant: q, k and
    cached k as rotated E4M3 codes (synthetic, multipliers E4M3_Q_SCALE / E4M3_K_SCALE),
    v bf16; sets cycle so that one pass exceeds the L2."""

    def __init__(self, w: synth.Workload, dev, seed_base: int, max_sets: int = 4):
        import torch
        from causal_video_diffusion_rope_b200 import dz
        self.dz, self.w = dz, w
        lay = w.layout
        B, H, D, L = lay.batch, w.heads, w.head_dim, lay.chunk_len
        keys = w.cache_tokens + lay.self_kv_len
        self.set_bytes = B * H * D * (lay.q_len * (1 + 2) + keys * (1 + 2))
        self.n_sets = min(max_sets, max(2, int(math.ceil(3 * L2_BYTES / self.set_bytes))))
        self.h = dz.dz_attn_create(dz.make_desc(num_heads=H, max_batch=B, max_q_tokens=lay.q_len))
        self.dl = dz.layout_from(lay)
        self.sets = []
        for i in range(self.n_sets):
            inp = synth.make_inputs_e4m3(w, seed_base + i)
            st = {"q8": torch.from_numpy(inp["q8"]).to(dev), "k8": torch.from_numpy(inp["k8"]).to(dev),
                  "v": torch.from_numpy(inp["v"].view(np.int16)).to(dev).view(torch.bfloat16),
                  "out": torch.empty((B, lay.q_len, H, D), dtype=torch.bfloat16, device=dev),
                  "cache": None}
            if "cache_k8" in inp:
                st["ck8"] = torch.from_numpy(inp["cache_k8"]).to(dev)
                st["cv"] = torch.from_numpy(inp["cache_v"].view(np.int16)).to(dev).view(torch.bfloat16)
                st["cache"] = dz.make_cache(st["ck8"], st["cv"], B, w.cache_tokens, w.cache_tokens, L)
            self.sets.append(st)

    def call(self, i, stream, q8=None, k8=None, v=None, out=None):
        st = self.sets[i % self.n_sets]
        self.dz.dz_chunk_attn_forward_e4m3(
            self.h, st["q8"] if q8 is None else q8, st["k8"] if k8 is None else k8,
            st["v"] if v is None else v, st["cache"], self.dl, synth.E4M3_Q_SCALE,
            synth.E4M3_K_SCALE, st["out"] if out is None else out, stream)

    def close(self):
        self.dz.dz_attn_sync_status(self.h)
        self.dz.dz_attn_destroy(self.h)
        self.sets.clear()


def e4m3_block(wl: int, dev, stream, steps: int, peak_tf: float):
    """The FP8 variant (dz_chunk_attn_forward_e4m3) on workload wl's self-attention,
    timed like the headline (graphs of calls cycling input sets above L2, CUDA events
    on the launching stream).  Its QK^T runs at the E4M3 rate and PV at the bf16 rate,
    so the contraction's peak is taken as the bf16 peak x 4/3 (half the FLOPs at twice
    the rate)."""
    import torch
    w = synth.WORKLOADS[wl]
    st = E4m3Setup(w, dev, 3000 + 100 * wl)
    n = max(20, min(steps, 240))
    ms, _ = time_graph(stream, lambda i: st.call(i, stream), n, 3, 1, dev)
    st.close()
    us = 1e3 * ms / n
    tf = self_flops(w) / (us * 1e-6) / 1e12
    mixed = peak_tf * 4.0 / 3.0
    res = {"workload": w.name, "what": "attention kernel on E4M3 q, k (rotated, quantised "
           "beforehand), bf16 v", "calls": n,
           "l2": f"{st.n_sets} input sets of {st.set_bytes / 2**20:.0f} MiB cycle",
           "us_per_call": round(us, 3), "tflops": round(tf, 2), "flop_per_call": self_flops(w),
           "frac_of_bf16_peak": round(tf / peak_tf, 4), "mixed_peak": round(mixed, 1),
           "frac": round(tf / mixed, 4), "traffic": ncu_traffic("e4m3_" + w.name)}
    del st
    torch.cuda.empty_cache()
    return res


def run_e4m3(args, rank: int, world: int, local_rank: int, config: dict):
    """The FP8 variant as the headline: K calls of dz_chunk_attn_forward_e4m3 on the
    workload's self-attention (E4M3 q, k and cached k; bf16 v), then the end-to-end leg
    with q8, k8, v copied in from pinned host memory and out copied back."""
    import torch
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = synth.WORKLOADS[args.workload]
    st = E4m3Setup(w, dev, 3000 + 1000 * rank)
    stream = torch.cuda.Stream(device=dev)
    sampler = ClockSampler(gpu_id(local_rank))
    ms, clocks = time_graph(stream, lambda i: st.call(i, stream), args.steps, max(args.warmup, 3),
                            world, dev, sampler)
    st.dz.dz_attn_sync_status(st.h, stream)
    ms_per_step = ms / args.steps
    fl = self_flops(w)
    tf = fl / (ms_per_step * 1e-3) / 1e12
    s0 = st.sets[0]

    def e2e_call(di, do):
        st.call(0, stream, di["q8"], di["k8"], di["v"], do["out"])

    e2e = e2e_pipelined(dev, stream, {k: s0[k] for k in ("q8", "k8", "v")}, {"out": s0["out"]},
                        e2e_call, max(3, min(args.steps, 200)), world)
    e2e["value"] = round(job_throughput(fl, e2e.pop("steps_done"), world, e2e.pop("ms")), 3)
    n_sets, set_bytes = st.n_sets, st.set_bytes
    # a decode call from bf16 q and k: rotation and quantisation of q and the chunk's k
    # in one pass each (dz_rope3d_e4m3), then the attention on the E4M3 cache
    whole = None
    lay = w.layout
    if lay.mode == synth.MODE_DECODE:
        B, H, D = lay.batch, w.heads, w.head_dim
        rng = np.random.default_rng(5000 + rank)
        bf = [{x: torch.from_numpy(synth.normal_bf16(rng, (B, lay.q_len, H, D)).view(np.int16))
               .to(dev).view(torch.bfloat16) for x in ("q", "k")} for _ in range(n_sets)]
        q8b = torch.empty((B, lay.q_len, H, D), dtype=torch.uint8, device=dev)
        k8b = torch.empty_like(q8b)

        def whole_call(i):
            b = bf[i % n_sets]
            st.dz.dz_rope3d_e4m3(st.h, b["q"], q8b, B, lay.q_len, st.dl, lay.num_chunks,
                                 synth.E4M3_Q_SCALE, stream)
            st.dz.dz_rope3d_e4m3(st.h, b["k"], k8b, B, lay.q_len, st.dl, lay.num_chunks,
                                 synth.E4M3_K_SCALE, stream)
            st.call(i, stream, q8=q8b, k8=k8b)

        nw = max(20, min(args.steps, 2400))
        wms, _ = time_graph(stream, whole_call, nw, 3, world, dev)
        st.dz.dz_attn_sync_status(st.h, stream)
        wus = 1e3 * wms / nw
        whole = {"what": "dz_rope3d_e4m3 of q and of the chunk's k, then the E4M3 attention",
                 "us_per_call": round(wus, 3), "tflops": round(fl / (wus * 1e-6) / 1e12, 2),
                 "launches_per_call": 3}
        del bf, q8b, k8b
    # the quantisation that feeds the variant (dz_quantize_e4m3), HBM-bound: 64 Mi bf16
    # values (128 MiB read, 64 MiB written) per call, two buffers alternating
    nq = 64 << 20
    xs = [torch.randn(nq, device=dev).to(torch.bfloat16) for _ in range(2)]
    ys = [torch.empty(nq, dtype=torch.uint8, device=dev) for _ in range(2)]
    nqc = max(10, min(args.steps, 100))
    qms, _ = time_graph(stream, lambda i: st.dz.dz_quantize_e4m3(st.h, xs[i % 2], ys[i % 2], nq,
                                                                   synth.E4M3_Q_SCALE, stream),
                        nqc, 3, world, dev)
    st.dz.dz_attn_sync_status(st.h, stream)
    del xs, ys
    st.close()
    if rank != 0:
        return
    peak_tf, peak_hbm, peak_kind = measured_peaks()
    qus = 1e3 * qms / nqc
    qgbs = 3 * nq / (qus * 1e-6) / 1e9
    quant = {"what": "dz_quantize_e4m3 of 64 Mi bf16 values", "us_per_call": round(qus, 3),
             "bytes": 3 * nq, "gbs": round(qgbs, 1), "frac_of_hbm": round(qgbs / peak_hbm, 4)}
    mixed = peak_tf * 4.0 / 3.0
    line = {"metric": E4M3_METRIC, "value": round(tf * world, 3), "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms_per_step, 6), "us_per_call": round(ms_per_step * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "e4m3 q/k, bf16 v/p/out, fp32 accumulation",
            "data": "synthetic (E4M3 codes of N(0,1) q, k; N(0,1) bf16 v)",
            "config": dict(config, op="attention_e4m3", q_scale=synth.E4M3_Q_SCALE,
                           rope="q and k arrive rotated as E4M3 codes (call_from_bf16: rotated "
                                "and quantised by dz_rope3d_e4m3 inside the timed call)",
                           k_scale=synth.E4M3_K_SCALE,
                           l2=f"inputs cycle through {n_sets} sets "
                              f"({n_sets * set_bytes / 2**20:.0f} MiB > 126 MB L2)",
                           parallelism=f"dp{world} (independent replicas of the call)"),
            "roofline": {"bound": "tensor", "achieved": round(tf, 2), "peak": round(mixed, 1),
                         "unit": "TFLOP/s", "frac": round(tf / mixed, 4),
                         "traffic": ncu_traffic("e4m3_" + w.name),
                         "peak_kind": f"{peak_kind} bf16 (burst) x 4/3: QK^T at the E4M3 rate "
                                      "(2x bf16), PV at the bf16 rate",
                         "frac_of_bf16_peak": round(tf / peak_tf, 4),
                         "kernel": "chunk_attn_kernel (E4M3 instantiation)",
                         "kernel_us": round(ms_per_step * 1e3, 3)},
            "quantize": quant, "call_from_bf16": whole,
            "cpu_baseline": None, "e2e": e2e, "gpu_launches": args.steps, "clocks": clocks}
    print(json.dumps(line), flush=True)


def run_attention(args, rank: int, world: int, local_rank: int):
    """The headline: K steps of the attention call on this rank, timed with CUDA events
    (max over ranks); then the end-to-end leg through the same C-ABI call with host
    buffers.  Returns (ms_per_step, job TFLOP/s, clocks, e2e, what this rank ran)."""
    import torch
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = synth.WORKLOADS[args.workload]
    kind, branch = rank_work(w, rank, world)
    seed_base = 1000 if kind == "cfg" else 1000 * rank
    rotation_pass = args.rotation == "pass"
    st = AttnSetup(w, dev, seed_base, rotation_pass, branch=branch)
    stream = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(stream):
        for i in range(max(args.warmup, 3)):
            st.call(i, stream)
    stream.synchronize()
    st.dz.dz_attn_sync_status(st.h, stream)
    sampler = ClockSampler(gpu_id(local_rank))
    ms, clocks = time_graph(stream, lambda i: st.call(i, stream), args.steps, 0, world, dev,
                            sampler)
    st.dz.dz_attn_sync_status(st.h, stream)
    ms_per_step = ms / args.steps
    flops_rank = step_flops(st.w)  # this rank's share of one step
    tflops_total = job_throughput(flops_rank, args.steps, world, ms)

    # ---- the attention kernel alone (its launch duration, for the roofline): the same
    # calls on q, k rotated beforehand, timed the same way
    st.prepare_rotated(stream)
    n_k = min(args.steps, 2400)
    kms, _ = time_graph(stream, lambda i: st.kernel_call(i, stream), n_k, 3, world, dev)
    st.dz.dz_attn_sync_status(st.h, stream)
    kernel_ms = kms / n_k

    # ---- end to end: host buffers in, result out, through the same C-ABI calls
    s0 = st.sets[0]
    in_keys = [k for k in ("q", "k", "v", "q_x", "k_x", "v_x") if k in s0]
    out_keys = [k for k in ("out", "out_x") if k in s0]

    def e2e_call(di, do):
        st.dz.dz_chunk_attn_forward(st.h, di["q"], di["k"], di["v"], s0["cache"], st.dl,
                                    do["out"], stream)
        if st.dlx is not None:
            st.dz.dz_chunk_attn_forward(st.h, di["q_x"], di["k_x"], di["v_x"], None, st.dlx,
                                        do["out_x"], stream)

    e2e = e2e_pipelined(dev, stream, {k: s0[k] for k in in_keys}, {k: s0[k] for k in out_keys},
                        e2e_call, max(3, min(args.steps, 200)), world)
    st.dz.dz_attn_sync_status(st.h, stream)
    e2e["value"] = round(job_throughput(flops_rank, e2e.pop("steps_done"), world, e2e.pop("ms")), 3)
    ran = {"kind": kind, "branch": branch, "batch_per_rank": st.w.layout.batch,
           "n_sets": st.n_sets, "set_bytes": step_bytes(st.w), "kernel_ms": kernel_ms}
    st.close()
    extra = None
    if world == 1 and args.extra:
        peak_tf, peak_hbm, _ = measured_peaks()
        extra = [extra_workload_block(x, dev, stream, args.steps, peak_tf, peak_hbm, rotation_pass)
                 for x in EXTRA_WORKLOADS if x != args.workload]
        extra = {"bf16": extra, "e4m3": [e4m3_block(x, dev, stream, args.steps, peak_tf)
                                         for x in E4M3_WORKLOADS]}
    return ms_per_step, tflops_total, clocks, e2e, ran, extra


QKV_METRIC = ("fused QKV projection + 3D RoPE TFLOP/s and % of B200 BF16 peak; "
              "\u00b5s per DiT-layer projection of one chunk")
D_MODEL = 5120  # hidden size of the 14B DiT


def qkv_flops(w) -> float:
    lay = w.layout
    return 2.0 * lay.batch * lay.chunk_len * D_MODEL * 3 * w.heads * w.head_dim


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

    sampler = ClockSampler(gpu_id(local_rank))
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

    # the rotation the unfused path adds after that GEMM: q and k through dz_rope3d
    qr, kr = torch.empty_like(q), torch.empty_like(k)

    def call_rot(i):
        dz.dz_rope3d(h, q, qr, B, S, dl, first, stream)
        dz.dz_rope3d(h, k, kr, B, S, dl, first, stream)

    ms_rot, _ = time_graph(stream, call_rot, min(args.steps, 2400), 3, world, dev)
    rot_us = 1e3 * ms_rot / min(args.steps, 2400)

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
                        "cublas_same_gemm_tflops": round(flops / (ref_us * 1e-6) / 1e12, 2),
                        "rotation_pass_us": round(rot_us, 3),
                        "unfused_us": round(ref_us + rot_us, 3)},
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

    sampler = ClockSampler(gpu_id(local_rank))
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

    sampler = ClockSampler(gpu_id(local_rank))
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


def reference_line(args, w, config) -> dict:
    """The reference arm: the CPU fp64 oracle as it stands, on bounded samples of the
    same workload (one sampled query row per step)."""
    budget = 150.0 / (args.steps + args.warmup)
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
    sample = (f"{rows_per_step} query row(s) of the call per step, "
              f"~{budget * 1e3:.1f} ms of oracle work per step")
    return {"impl": "reference", "metric": METRIC, "value": round(value, 6),
            "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(1e3 * elapsed / max(1, len(rate)), 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": dict(config, l2="n/a (CPU)"),
            "cpu_baseline": cpu_baseline_fields(value, sample),
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
            "wall_s": round(time.perf_counter() - t_all, 1)}


def parse_args(argv):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=48000)
    ap.add_argument("--warmup", type=int, default=240)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=15.0,
                    help="seconds of oracle CPU work for the cpu_baseline field")
    ap.add_argument("--op", default="attn", choices=["attn", "qkv", "bwd", "cache", "e4m3"],
                    help="attn: the chunk-causal attention call; qkv: the fused projection; "
                         "bwd: the backward of a prefill / teacher-forcing call; "
                         "cache: the KV-cache chunk replace; e4m3: the attention call with "
                         "E4M3 q and k")
    ap.add_argument("--workload", type=int, default=DEFAULT_WORKLOAD,
                    choices=range(len(synth.WORKLOADS)),
                    help="workload index (default: the single-layer inference step)")
    ap.add_argument("--rotation", default="pass", choices=["kernel", "pass"],
                    help="kernel: q and the chunk's k rotated as the attention kernel loads "
                         "them; pass: rotated once per call by a separate kernel first")
    ap.add_argument("--no-extra", dest="extra", action="store_false",
                    help="skip the other workloads' block of the headline line")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3
    return args


def rank_main(argv) -> None:
    """One rank's work (rank, world and local rank come from the launcher environment)."""
    args = parse_args(argv)
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    w = synth.WORKLOADS[args.workload]
    config = {"workload": w.name, "batch": w.layout.batch, "heads": w.heads,
              "head_dim": w.head_dim, "q_tokens": w.layout.q_len,
              "keys": w.cache_tokens + w.layout.self_kv_len, "cache_tokens": w.cache_tokens,
              "mode": synth.MODE_NAMES[w.layout.mode],
              "cross_keys": w.cross_kv_len,
              "rope": ("3d t/h/w 22/21/21 base 1e4; q and the chunk's k rotated " +
                       ("as the attention kernel loads them" if args.rotation == "kernel"
                        else "once per call by a separate kernel")),
              "flop_per_step": step_flops(w)}

    if args.impl == "reference":
        # rank 0 alone runs the oracle; other ranks exit without work
        if rank == 0:
            if args.op != "attn":
                print(json.dumps({"impl": "reference", "unavailable": "the reference arm times "
                                  "the attention call (--op attn) only"}), flush=True)
            else:
                print(json.dumps(reference_line(args, w, config)), flush=True)
        return

    import torch.distributed as dist
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        if args.op in ("qkv", "bwd", "cache", "e4m3"):
            {"qkv": run_qkv, "bwd": run_bwd, "cache": run_cache,
             "e4m3": run_e4m3}[args.op](args, rank, world, local_rank, config)
            return
        cpu = None
        if rank == 0 and world == 1 and args.cpu_budget > 0:
            # the oracle, timed on this host's cores before the GPU work starts
            r, heads_done, dt = oracle_full_call_rate(w, args.cpu_budget)
            cpu = cpu_baseline_fields(r, f"{heads_done} of {w.heads} heads of the call "
                                         f"(4-head slices), {dt:.1f} s of fp64 oracle work")
        ms_per_step, tflops, clocks, e2e, ran, extra = run_attention(args, rank, world,
                                                                     local_rank)
    finally:
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()
    if rank != 0:
        return
    peak_tf, peak_hbm, peak_kind = measured_peaks()
    # this rank's share of a step: the whole call (replicas) or one CFG branch of it
    w_rank = synth.branch_inputs(w, {}, 0)[0] if ran["kind"] == "cfg" else w
    per_gpu_tf = step_flops(w_rank) / (ms_per_step * 1e-3) / 1e12
    rotation_pass = args.rotation == "pass"
    # the dominant kernel: the attention kernel's algorithmic FLOPs over its own launch
    # duration (timed on pre-rotated q, k); the whole call (with the rotation pass) beside it
    kernel_ms = ran["kernel_ms"]
    kernel_tf = self_flops(w_rank) / (kernel_ms * 1e-3) / 1e12
    roof = {"bound": "tensor", "achieved": round(kernel_tf, 2), "peak": peak_tf,
            "unit": "TFLOP/s", "frac": round(kernel_tf / peak_tf, 4),
            "traffic": ncu_traffic(w.name),
            "peak_kind": f"{peak_kind} bf16 (burst)",
            "frac_of_spec": round(kernel_tf / SPEC_BF16_TFLOPS, 4),
            "spec_peak": SPEC_BF16_TFLOPS,
            "kernel": "chunk_attn_kernel", "kernel_us": round(kernel_ms * 1e3, 3),
            "hbm_frac": round(step_bytes(w_rank) / (kernel_ms * 1e-3) / 1e9 / peak_hbm, 4),
            "call": {"what": "the whole call: " + ("rotation pass + attention kernel"
                                                  if rotation_pass else "attention kernel"),
                     "us": round(ms_per_step * 1e3, 3), "tflops": round(per_gpu_tf, 2),
                     "frac": round(per_gpu_tf / peak_tf, 4),
                     "frac_of_spec": round(per_gpu_tf / SPEC_BF16_TFLOPS, 4)}}
    scaling = "strong" if ran["kind"] == "cfg" else "weak"
    parallelism = (f"cfg{world} (rank r runs CFG branch r: batch 1 with its own cache half)"
                   if ran["kind"] == "cfg" else f"dp{world} (independent replicas of the call)")
    line = {"metric": METRIC, "value": round(tflops, 3), "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms_per_step, 6), "us_per_call": round(ms_per_step * 1e3, 3),
            "pct_of_bf16_peak": round(100 * per_gpu_tf / peak_tf, 2),
            "pct_of_spec_bf16_peak": round(100 * per_gpu_tf / SPEC_BF16_TFLOPS, 2),
            "higher_is_better": True, "scaling": scaling, "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": dict(config, l2=f"inputs cycle through {ran['n_sets']} sets "
                                      f"({ran['n_sets'] * ran['set_bytes'] / 2**20:.0f} MiB > "
                                      f"126 MB L2)",
                           parallelism=parallelism),
            "roofline": roof, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": args.steps * launches_per_step(w, rotation_pass), "clocks": clocks}
    if extra is not None:
        line["workloads"] = extra["bf16"]
        line["e4m3"] = extra["e4m3"]
    print(json.dumps(line), flush=True)


def main() -> None:
    argv = sys.argv[1:]
    args = parse_args(argv)
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ and args.impl == "ours":
        spawn_ranks(args.gpus, rank_main, argv)
        return
    rank_main(argv)


if __name__ == "__main__":
    main()
