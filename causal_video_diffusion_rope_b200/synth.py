"""Seeded synthetic inputs shared by the CUDA path's tests/bench and by the oracle.

This module holds shapes and random draws only: no attention, rotary or mask
arithmetic lives here.  Every tensor is drawn as float32 standard normals from
``numpy.random.default_rng(seed)`` and rounded to bfloat16 (round to nearest,
ties to even), so the same bytes go to the GPU and to the CPU oracle; the FP8
variant's q and k are the same kind of draws cast to E4M3 codes by torch's
float8_e4m3fn conversion.

Workloads follow the DreamZero pages (Causal WAN DiT: 40 heads, head_dim 128,
dim 5120 -- "DreamZero_Architecture", section 5 hyper-parameter table; chunked
autoregressive denoising with a KV cache of clean chunks -- arXiv 2602.15922
summary, "Method"; 24 action tokens per chunk -- section 5 table; 8x spatial
VAE stride -- section 2.2).  The 11x20 token grid per latent frame (176x320
frame, 8x VAE, 2x2 patch) and the 22/21/21 rotary split are the workload's
stated shapes.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import numpy as np

# dz_mode values (must match include/dz.h)
MODE_DECODE = 0
MODE_TEACHER_FORCING = 1
MODE_PREFILL = 2
MODE_CROSS = 3

MODE_NAMES = {
    MODE_DECODE: "decode",
    MODE_TEACHER_FORCING: "teacher_forcing",
    MODE_PREFILL: "prefill",
    MODE_CROSS: "cross",
}


@dataclasses.dataclass(frozen=True)
class Layout:
    """Chunk layout of one attention call (mirrors ``dz_chunk_layout``)."""

    mode: int
    batch: int
    frames_per_chunk: int
    grid_h: int
    grid_w: int
    n_action: int
    num_chunks: int
    t_offset: int = 0
    kv_len: int = 0

    @property
    def chunk_len(self) -> int:
        return self.frames_per_chunk * self.grid_h * self.grid_w + self.n_action

    @property
    def q_len(self) -> int:
        L = self.chunk_len
        if self.mode == MODE_DECODE:
            return L
        if self.mode == MODE_TEACHER_FORCING:
            return 2 * self.num_chunks * L
        return self.num_chunks * L  # PREFILL, CROSS

    @property
    def self_kv_len(self) -> int:
        """Keys held in the call's own k/v tensors (excludes the cache)."""
        if self.mode == MODE_CROSS:
            return self.kv_len
        return self.q_len


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    heads: int
    layout: Layout
    cache_tokens: int = 0          # DECODE: tokens already in the KV cache
    cross_kv_len: int = 0          # extra cross-attention call (text + image keys)
    k_boost: float = 1.0           # K scaled by this factor on a subset of heads
    k_boost_frac: float = 0.0      # fraction of heads boosted
    denoise_steps: int = 1
    description: str = ""

    @property
    def head_dim(self) -> int:
        return 128


# The workloads; index i is "workload i" in tests and the benchmark.
WORKLOADS = [
    Workload(
        "tiny_prefill_b1_h2_3x36", heads=2,
        layout=Layout(MODE_PREFILL, batch=1, frames_per_chunk=1, grid_h=4, grid_w=8,
                      n_action=4, num_chunks=3),
        description="3 chunks x (1 latent frame of 4x8 + 4 action tokens) = 108 tokens, "
                    "block-causal over chunks"),
    Workload(
        "decode_b1_h40_q464_cache4", heads=40,
        layout=Layout(MODE_DECODE, batch=1, frames_per_chunk=2, grid_h=11, grid_w=20,
                      n_action=24, num_chunks=4),
        cache_tokens=4 * 464,
        description="464-token noisy chunk over a cache of 4 clean chunks + itself (2320 keys)"),
    Workload(
        "cfg_decode_b2_h40_q464_cache8_x16", heads=40,
        layout=Layout(MODE_DECODE, batch=2, frames_per_chunk=2, grid_h=11, grid_w=20,
                      n_action=24, num_chunks=8),
        cache_tokens=8 * 464, denoise_steps=16,
        description="CFG batch 2, cache of 8 chunks (4176 keys incl. self), 16 denoising "
                    "steps, last chunk replaced between requests"),
    Workload(
        "teacher_forcing_b1_h40_8x2x464", heads=40,
        layout=Layout(MODE_TEACHER_FORCING, batch=1, frames_per_chunk=2, grid_h=11,
                      grid_w=20, n_action=24, num_chunks=8),
        description="8 clean + 8 noisy chunks of 464 tokens (7424 tokens), teacher-forcing mask"),
    Workload(
        "long_cache_cross_b2_h40_cache32", heads=40,
        layout=Layout(MODE_DECODE, batch=2, frames_per_chunk=2, grid_h=11, grid_w=20,
                      n_action=24, num_chunks=32),
        cache_tokens=32 * 464, cross_kv_len=512 + 257, k_boost=3.0, k_boost_frac=0.05,
        description="cache of 32 chunks (15312 keys incl. self) + cross-attention to "
                    "512 text + 257 image keys; K x3 on 5% of heads"),
    Workload(
        "decode_b1_h40_3view_q1784_cache4", heads=40,
        layout=Layout(MODE_DECODE, batch=1, frames_per_chunk=2, grid_h=22, grid_w=40,
                      n_action=24, num_chunks=4),
        cache_tokens=4 * 1784,
        description="three camera views tiled to 352x640 (22x40 = 880 tokens per latent "
                    "frame): 1784-token chunk over a cache of 4 chunks + itself (8920 keys)"),
]


def bf16_bits_from_f32(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest, ties to even); returns uint16 bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    nan = np.isnan(x)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)
    r[nan] = 0x7FC0
    return r


def f32_from_bf16_bits(b: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bits to float32 (exact)."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def normal_bf16(rng: np.random.Generator, shape, scale: Optional[np.ndarray] = None) -> np.ndarray:
    """Standard normals drawn in float32, optionally scaled per head, rounded to bf16 bits.

    ``scale`` (if given) has length = shape[2] (heads) and is applied in float32
    before the rounding.
    """
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if scale is not None:
        x = x * scale.astype(np.float32)[None, None, :, None]
    return bf16_bits_from_f32(x)


def boosted_heads(rng: np.random.Generator, heads: int, frac: float) -> np.ndarray:
    n = int(round(heads * frac))
    if n == 0:
        return np.zeros(0, dtype=np.int64)
    return np.sort(rng.choice(heads, size=n, replace=False))


def projection_inputs(seed: int, B: int, S: int, d_model: int, heads: int, head_dim: int = 128):
    """Hidden states x [B, S, d_model] ~ N(0, 1) and projection weights
    w [3 * heads * head_dim, d_model] ~ N(0, 1 / d_model) (random init: no trained
    weights), both drawn in fp32 and rounded to bf16; returns uint16 bit arrays."""
    rng = np.random.default_rng(seed)
    x = bf16_bits_from_f32(rng.standard_normal((B, S, d_model), dtype=np.float32))
    w = bf16_bits_from_f32(rng.standard_normal((3 * heads * head_dim, d_model), dtype=np.float32)
                           * np.float32(1.0 / np.sqrt(d_model)))
    return x, w


def make_inputs(w: Workload, seed: int, cache_capacity: Optional[int] = None) -> Dict[str, np.ndarray]:
    """Draw one call's inputs for workload ``w`` as bf16 bit arrays (uint16), BSHD layout.

    Draw order (fixed): boosted heads, q, k, v, cache_k, cache_v, then for a
    cross-attention workload q_x, k_x, v_x.  Cache tensors have
    ``cache_capacity`` rows (default: exactly the cached tokens); rows past the
    cached tokens are filled with a NaN pattern so that any read of them shows.
    """
    rng = np.random.default_rng(seed)
    lay = w.layout
    B, H, D = lay.batch, w.heads, w.head_dim
    heads_x = boosted_heads(rng, H, w.k_boost_frac)
    kscale = np.ones(H, dtype=np.float32)
    kscale[heads_x] = w.k_boost
    out: Dict[str, np.ndarray] = {"boosted_heads": heads_x}
    out["q"] = normal_bf16(rng, (B, lay.q_len, H, D))
    out["k"] = normal_bf16(rng, (B, lay.self_kv_len, H, D), kscale)
    out["v"] = normal_bf16(rng, (B, lay.self_kv_len, H, D))
    if lay.mode == MODE_DECODE:
        n = w.cache_tokens
        cap = n if cache_capacity is None else cache_capacity
        ck = np.full((B, cap, H, D), 0x7FC1, dtype=np.uint16)
        cv = np.full((B, cap, H, D), 0x7FC1, dtype=np.uint16)
        ck[:, :n] = normal_bf16(rng, (B, n, H, D), kscale)
        cv[:, :n] = normal_bf16(rng, (B, n, H, D))
        out["cache_k"], out["cache_v"] = ck, cv
    if w.cross_kv_len:
        out["q_x"] = normal_bf16(rng, (B, lay.chunk_len, H, D))
        out["k_x"] = normal_bf16(rng, (B, w.cross_kv_len, H, D), kscale)
        out["v_x"] = normal_bf16(rng, (B, w.cross_kv_len, H, D))
    return out


# Multipliers of the E4M3 operands (one per tensor, powers of two): |q| stays
# below ~6 and |k| below ~18 on the K x 3 heads, so the codes stay under 448.
E4M3_Q_SCALE = 64.0
E4M3_K_SCALE = 16.0


def normal_e4m3(rng: np.random.Generator, shape, multiplier: float,
                scale: Optional[np.ndarray] = None) -> np.ndarray:
    """Standard normals drawn in float32 (optionally scaled per head), times
    ``multiplier``, cast to float8_e4m3fn by torch (nearest, ties to even);
    returns the uint8 codes.  Values are clipped to +-440 first (the cast gives
    NaN past the format's range)."""
    import torch

    x = rng.standard_normal(size=shape, dtype=np.float32)
    if scale is not None:
        x = x * scale.astype(np.float32)[None, None, :, None]
    x = np.clip(x * np.float32(multiplier), -440.0, 440.0).astype(np.float32)
    return torch.from_numpy(np.ascontiguousarray(x)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def make_inputs_e4m3(w: Workload, seed: int,
                     cache_capacity: Optional[int] = None) -> Dict[str, np.ndarray]:
    """Inputs of the FP8 attention variant for workload ``w``: q and k (the call's
    own and the cached keys) as E4M3 codes standing for already rotated operands
    (multipliers E4M3_Q_SCALE, E4M3_K_SCALE), v and cached v as bf16 bits.  Same
    shapes, K x 3 heads and draw order as ``make_inputs``; cache rows past the
    cached tokens hold NaN codes."""
    rng = np.random.default_rng(seed)
    lay = w.layout
    B, H, D = lay.batch, w.heads, w.head_dim
    heads_x = boosted_heads(rng, H, w.k_boost_frac)
    kscale = np.ones(H, dtype=np.float32)
    kscale[heads_x] = w.k_boost
    out: Dict[str, np.ndarray] = {"boosted_heads": heads_x}
    out["q8"] = normal_e4m3(rng, (B, lay.q_len, H, D), E4M3_Q_SCALE)
    out["k8"] = normal_e4m3(rng, (B, lay.self_kv_len, H, D), E4M3_K_SCALE, kscale)
    out["v"] = normal_bf16(rng, (B, lay.self_kv_len, H, D))
    if lay.mode == MODE_DECODE:
        n = w.cache_tokens
        cap = n if cache_capacity is None else cache_capacity
        ck = np.full((B, cap, H, D), 0x7F, dtype=np.uint8)
        cv = np.full((B, cap, H, D), 0x7FC1, dtype=np.uint16)
        ck[:, :n] = normal_e4m3(rng, (B, n, H, D), E4M3_K_SCALE, kscale)
        cv[:, :n] = normal_bf16(rng, (B, n, H, D))
        out["cache_k8"], out["cache_v"] = ck, cv
    return out


def cross_layout(w: Workload) -> Layout:
    """Layout of the cross-attention call of workload ``w`` (one query chunk)."""
    lay = w.layout
    return dataclasses.replace(lay, mode=MODE_CROSS, num_chunks=1, kv_len=w.cross_kv_len,
                               t_offset=0)


def fresh_chunk(rng: np.random.Generator, w: Workload) -> Dict[str, np.ndarray]:
    """New noisy-chunk q, k, v for one denoising step (same shapes as ``make_inputs``)."""
    lay = w.layout
    B, H, D = lay.batch, w.heads, w.head_dim
    return {
        "q": normal_bf16(rng, (B, lay.q_len, H, D)),
        "k": normal_bf16(rng, (B, lay.self_kv_len, H, D)),
        "v": normal_bf16(rng, (B, lay.self_kv_len, H, D)),
    }


def branch_inputs(w: Workload, inp: Dict[str, np.ndarray], branch: int):
    """One batch item (a CFG branch) of a workload and its inputs: the workload with
    batch 1 and every batched tensor sliced to item ``branch`` (its own cache half)."""
    lay = dataclasses.replace(w.layout, batch=1)
    wb = dataclasses.replace(w, layout=lay)
    out = {k: (v[branch:branch + 1] if k != "boosted_heads" else v) for k, v in inp.items()}
    return wb, out

