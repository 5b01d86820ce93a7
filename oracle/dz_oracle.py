"""CPU fp64 oracle for chunk-causal 3D-RoPE attention and the KV-cache operations.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import this module:
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
reference leg of ``bench.py`` use it.  It shares no code with the CUDA
library; both sides only consume the seeded bf16 inputs drawn by
``causal_video_diffusion_rope_b200.synth`` (which holds no method arithmetic).

Everything here is the plain definition, written for reading, not for speed:
inputs are the exact bf16 values widened to float64, nothing is rounded in
between, softmax is the textbook ``exp(s - max) / sum`` over an explicit
boolean visibility matrix, and the rotary embedding is an explicit 2x2
rotation of each adjacent pair.  Library matmuls (numpy, float64) are used
for the contractions.

Sources (page title, section):
  * Causal WAN DiT: 40 heads, head_dim 128, dim 5120, causal self-attention,
    RoPE on the video latent sequence -- "DreamZero (WAM) 模型架构", §2.3 block
    diagram and §5 hyper-parameter table.
  * Chunked autoregression; each chunk holds a fixed number of latent frames;
    the current noisy chunk sees the clean context of earlier chunks and no
    future token (teacher forcing) -- "World Action Models are Zero-shot
    Policies" (hyper.ai summary), section "方法" (method), paragraph 3; the
    walkthrough of the same paper, training objective paragraph (Fig. 14).
  * KV cache of clean chunks; after a chunk executes, its predicted frames in
    the cache are replaced by the real observation -- hyper.ai summary,
    "方法" paragraph 4; "DreamZero 单卡推理", "架构" table (DiT runner keeps the
    attention KV) and "连续请求" (frame position and KV carried across requests).
  * 24 action tokens per chunk -- "DreamZero (WAM) 模型架构", §5 table
    (action horizon 24) and §2.4.
  * Cross-attention to the concatenated visual + language conditioning --
    "DreamZero (WAM) 模型架构", §2.1 (fusion diagram) and §2.3 block diagram.

Readings taken where the pages are silent:
  * mask granularity is the chunk; inside a chunk attention is bidirectional;
    action tokens follow their chunk's rule;
  * teacher forcing: clean chunk i sees clean chunks <= i; noisy chunk i sees
    clean chunks < i and noisy chunk i; clean never sees noisy;
  * rotary: 64 adjacent (interleaved) pairs, pairs 0..21 rotate by the t
    position, 22..42 by h, 43..63 by w; per-axis frequency ladder
    omega_{a,j} = base^(-2j/d_a) with d_a = 2 * pairs_a, base 10000;
  * token order inside a chunk: frame-major, then row, then column, then the
    action tokens; a video token of frame f, row r, column c in chunk n has
    position (t_offset + n*F + f, r, c); an action token has
    (t_offset + n*F, 0, 0); noisy chunk i in teacher forcing takes the
    positions of clean chunk i;
  * cache K is stored already rotated (the cache holds post-RoPE keys);
  * softmax scale 1/sqrt(head_dim);
  * cross-attention: one softmax over all condition keys, no rotary, no mask.

Parity pins: see tests/test_oracle.py (brute force, library SDPA, closed forms,
invariants, golden fixtures) and tests/test_oracle_e4m3.py (the E4M3 format
against torch's float8_e4m3fn, brute force, scale invariance).  No function
here is "parity unpinned".
"""
from __future__ import annotations

import dataclasses
import functools
import math
from typing import Optional, Tuple

import numpy as np

DECODE, TEACHER_FORCING, PREFILL, CROSS = 0, 1, 2, 3


@dataclasses.dataclass(frozen=True)
class RopeSpec:
    """3D rotary parameters: pairs per axis (t, h, w) and the frequency base."""

    pairs_t: int = 22
    pairs_h: int = 21
    pairs_w: int = 21
    base: float = 10000.0

    @property
    def head_dim(self) -> int:
        return 2 * (self.pairs_t + self.pairs_h + self.pairs_w)


def widen_bf16(bits: np.ndarray) -> np.ndarray:
    """Exact value of bfloat16 bit patterns as float64."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# ---------------------------------------------------------------------------
# Token metadata: chunk index and (t, h, w) grid position of every token.
# ---------------------------------------------------------------------------

def chunk_len(F: int, gh: int, gw: int, n_action: int) -> int:
    return F * gh * gw + n_action


def token_position(s: int, F: int, gh: int, gw: int, n_action: int, t_offset: int,
                   first_chunk: int) -> Tuple[int, int, int]:
    """(t, h, w) of token s of a run of whole chunks that starts at chunk ``first_chunk``.

    Token s lies in chunk ``n = first_chunk + s // L`` at offset ``o = s % L``.
    Offsets below F*gh*gw are video tokens, frame-major then row then column,
    at (t_offset + n*F + frame, row, column); the remaining ``n_action`` offsets
    are action tokens at (t_offset + n*F, 0, 0).
    """
    L = chunk_len(F, gh, gw, n_action)
    n = first_chunk + s // L
    o = s % L
    per_frame = gh * gw
    if o < F * per_frame:
        f, rem = divmod(o, per_frame)
        r, c = divmod(rem, gw)
        return t_offset + n * F + f, r, c
    return t_offset + n * F, 0, 0


@functools.lru_cache(maxsize=64)
def token_positions(n_tokens: int, F: int, gh: int, gw: int, n_action: int,
                    t_offset: int, first_chunk: int) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Arrays (t, h, w) of ``token_position`` for tokens 0..n_tokens-1 (read-only)."""
    pos = np.array([token_position(s, F, gh, gw, n_action, t_offset, first_chunk)
                    for s in range(n_tokens)], dtype=np.int64).reshape(n_tokens, 3)
    pos.setflags(write=False)
    return pos[:, 0], pos[:, 1], pos[:, 2]


# ---------------------------------------------------------------------------
# 3D rotary embedding
# ---------------------------------------------------------------------------

def rope_angles(t: np.ndarray, h: np.ndarray, w: np.ndarray, spec: RopeSpec) -> np.ndarray:
    """Rotation angle of each (token, pair): shape [S, 64].

    Pair j < pairs_t turns by t * omega_t[j]; the next pairs_h pairs by
    h * omega_h[j']; the last pairs_w pairs by w * omega_w[j''], where
    omega_a[j] = base ** (-2 j / (2 * pairs_a)).
    """
    parts = []
    for pos, npairs in ((t, spec.pairs_t), (h, spec.pairs_h), (w, spec.pairs_w)):
        d_a = 2 * npairs
        omega = spec.base ** (-2.0 * np.arange(npairs, dtype=np.float64) / d_a)
        parts.append(pos.astype(np.float64)[:, None] * omega[None, :])
    return np.concatenate(parts, axis=1)


def rotate_pairs(x: np.ndarray, theta: np.ndarray) -> np.ndarray:
    """Rotate adjacent pairs (x[2j], x[2j+1]) of x [B, S, H, D] by theta [S, D/2]."""
    x0 = x[..., 0::2]
    x1 = x[..., 1::2]
    c = np.cos(theta)[None, :, None, :]
    s = np.sin(theta)[None, :, None, :]
    y = np.empty_like(x)
    y[..., 0::2] = x0 * c - x1 * s
    y[..., 1::2] = x0 * s + x1 * c
    return y


def rope3d(x: np.ndarray, F: int, gh: int, gw: int, n_action: int, t_offset: int,
           first_chunk: int, spec: RopeSpec = RopeSpec()) -> np.ndarray:
    """dz_rope3d: rotate x [B, S, H, D] (float64) by each token's (t, h, w) position."""
    S = x.shape[1]
    t, h, w = token_positions(S, F, gh, gw, n_action, t_offset, first_chunk)
    return rotate_pairs(x, rope_angles(t, h, w, spec))


def qkv_rope(x_bits: np.ndarray, w_bits: np.ndarray, heads: int, F: int, gh: int, gw: int,
             n_action: int, t_offset: int, first_chunk: int, spec: RopeSpec = RopeSpec()):
    """dz_qkv_rope: the attention inputs of a run of chunk tokens.

    The causal self-attention of a DiT block projects the block's hidden state
    [B, T, 5120] to q, k, v ("DreamZero (WAM) 模型架构", §2.3 block diagram) and
    RoPE acts on the latent sequence.  Here [q | k | v] = x W^T (no bias: the
    pages give none) from the exact bf16 values in float64, split into heads of
    128 features (feature n of a section belongs to head n // 128), then q and k
    are rotated at their tokens' positions by ``rope3d``.  Returns float64
    q, k, v, each [B, S, heads, 128].
    """
    x = widen_bf16(x_bits)                 # [B, S, d_model]
    w = widen_bf16(w_bits)                 # [3 * heads * D, d_model]
    D = spec.head_dim
    B, S = x.shape[0], x.shape[1]
    y = x @ w.T                            # [B, S, 3 * heads * D]
    HD = heads * D
    q = y[..., :HD].reshape(B, S, heads, D)
    k = y[..., HD:2 * HD].reshape(B, S, heads, D)
    v = y[..., 2 * HD:].reshape(B, S, heads, D)
    q = rope3d(q, F, gh, gw, n_action, t_offset, first_chunk, spec)
    k = rope3d(k, F, gh, gw, n_action, t_offset, first_chunk, spec)
    return q, k, v


# ---------------------------------------------------------------------------
# Visibility (the chunk mask)
# ---------------------------------------------------------------------------

def visibility(mode: int, L: int, num_chunks: int, cache_len: int = 0,
               kv_len: int = 0) -> np.ndarray:
    """Boolean [Sq, Sk]: may query i attend to key j.

    DECODE: keys are cache[0:cache_len] followed by the chunk's own L keys; the
      chunk sees all of them (no future token exists).
    PREFILL: num_chunks chunks; a query in chunk c sees keys of chunks <= c.
    TEACHER_FORCING: 2*num_chunks chunks, clean 0..N-1 then noisy 0..N-1;
      clean i sees clean <= i; noisy i sees clean < i and noisy i.
    CROSS: num_chunks query chunks against kv_len condition keys, all visible.
    """
    if mode == DECODE:
        return np.ones((L, cache_len + L), dtype=bool)
    if mode == CROSS:
        return np.ones((num_chunks * L, kv_len), dtype=bool)
    if mode == PREFILL:
        n = num_chunks * L
        cq = np.arange(n) // L
        return cq[:, None] >= cq[None, :]
    if mode == TEACHER_FORCING:
        N = num_chunks
        n = 2 * N * L
        c = np.arange(n) // L
        noisy = c >= N
        idx = np.where(noisy, c - N, c)
        qn, kn = noisy[:, None], noisy[None, :]
        qi, ki = idx[:, None], idx[None, :]
        clean_q = (~qn) & (~kn) & (ki <= qi)
        noisy_q_clean_k = qn & (~kn) & (ki < qi)
        noisy_q_same = qn & kn & (ki == qi)
        return clean_q | noisy_q_clean_k | noisy_q_same
    raise ValueError(f"unknown mode {mode}")


# ---------------------------------------------------------------------------
# Masked softmax attention
# ---------------------------------------------------------------------------

def softmax_probs(scores: np.ndarray, visible: np.ndarray) -> np.ndarray:
    """Row softmax over the visible entries; invisible entries get probability 0."""
    s = np.where(visible, scores, -np.inf)
    m = s.max(axis=-1, keepdims=True)
    e = np.exp(s - m)
    return e / e.sum(axis=-1, keepdims=True)


def masked_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray,
                     visible: np.ndarray) -> np.ndarray:
    """softmax(q k^T / sqrt(D), restricted to ``visible``) v for every (batch, head).

    q [B, Sq, H, D], k and v [B, Sk, H, D] (float64) -> [B, Sq, H, D].
    """
    B, Sq, H, D = q.shape
    out = np.empty((B, Sq, H, D), dtype=np.float64)
    scale = 1.0 / math.sqrt(D)
    for b in range(B):
        for hh in range(H):
            scores = (q[b, :, hh, :] @ k[b, :, hh, :].T) * scale
            p = softmax_probs(scores, visible)
            out[b, :, hh, :] = p @ v[b, :, hh, :]
    return out


def rotated_operands(q_bits: np.ndarray, k_bits: np.ndarray, v_bits: np.ndarray,
                     mode: int, F: int, gh: int, gw: int, n_action: int, num_chunks: int,
                     t_offset: int = 0, cache_k_bits: Optional[np.ndarray] = None,
                     cache_v_bits: Optional[np.ndarray] = None, cache_len: int = 0,
                     spec: RopeSpec = RopeSpec(), heads: Optional[slice] = None,
                     batch: Optional[slice] = None):
    """The call's q, keys and values as float64, rotated, keys in the call's order.

    Rotary is applied to q and to the call's own k: DECODE at the positions of
    chunk ``num_chunks``; PREFILL from chunk 0; TEACHER_FORCING with clean chunk
    i and noisy chunk i both at chunk i's positions; never in CROSS.  Cache keys
    are stored rotated and are used as they are, placed before the chunk's own
    keys.  ``heads`` / ``batch`` optionally select a slice of heads / batch items.
    """
    L = chunk_len(F, gh, gw, n_action)
    hs = slice(None) if heads is None else heads
    bs = slice(None) if batch is None else batch
    q = widen_bf16(q_bits[bs, :, hs, :])
    k = widen_bf16(k_bits[bs, :, hs, :])
    v = widen_bf16(v_bits[bs, :, hs, :])
    if mode == DECODE:
        q = rope3d(q, F, gh, gw, n_action, t_offset, num_chunks, spec)
        k = rope3d(k, F, gh, gw, n_action, t_offset, num_chunks, spec)
        if cache_len > 0:
            ck = widen_bf16(cache_k_bits[bs, :cache_len, hs, :])
            cv = widen_bf16(cache_v_bits[bs, :cache_len, hs, :])
            k = np.concatenate([ck, k], axis=1)
            v = np.concatenate([cv, v], axis=1)
    elif mode == PREFILL:
        q = rope3d(q, F, gh, gw, n_action, t_offset, 0, spec)
        k = rope3d(k, F, gh, gw, n_action, t_offset, 0, spec)
    elif mode == TEACHER_FORCING:
        half = num_chunks * L
        q = np.concatenate([rope3d(q[:, :half], F, gh, gw, n_action, t_offset, 0, spec),
                            rope3d(q[:, half:], F, gh, gw, n_action, t_offset, 0, spec)], axis=1)
        k = np.concatenate([rope3d(k[:, :half], F, gh, gw, n_action, t_offset, 0, spec),
                            rope3d(k[:, half:], F, gh, gw, n_action, t_offset, 0, spec)], axis=1)
    elif mode != CROSS:
        raise ValueError(f"unknown mode {mode}")
    return q, k, v


def chunk_attn_forward(q_bits: np.ndarray, k_bits: np.ndarray, v_bits: np.ndarray,
                       mode: int, F: int, gh: int, gw: int, n_action: int,
                       num_chunks: int, t_offset: int = 0, kv_len: int = 0,
                       cache_k_bits: Optional[np.ndarray] = None,
                       cache_v_bits: Optional[np.ndarray] = None, cache_len: int = 0,
                       spec: RopeSpec = RopeSpec(),
                       heads: Optional[slice] = None) -> np.ndarray:
    """dz_chunk_attn_forward on bf16 bit arrays; returns float64 [B, Sq, H, D].

    ``heads`` optionally restricts the computation to a slice of heads (the
    result then holds only those heads).
    """
    L = chunk_len(F, gh, gw, n_action)
    q, k, v = rotated_operands(q_bits, k_bits, v_bits, mode, F, gh, gw, n_action, num_chunks,
                               t_offset, cache_k_bits, cache_v_bits, cache_len, spec, heads)
    vis = visibility(mode, L, num_chunks, cache_len=cache_len, kv_len=kv_len)
    assert vis.shape == (q.shape[1], k.shape[1]), (vis.shape, q.shape, k.shape)
    return masked_attention(q, k, v, vis)


def chunk_attn_backward_f64(q: np.ndarray, k: np.ndarray, v: np.ndarray, do: np.ndarray,
                            mode: int, F: int, gh: int, gw: int, n_action: int, num_chunks: int,
                            t_offset: int = 0, spec: RopeSpec = RopeSpec()):
    """Gradients of sum(dO * O) for the PREFILL / TEACHER_FORCING self-attention call,
    with respect to its unrotated q, k and v (float64 [B, S, H, D] each).

    The forward is O = softmax(qr kr^T / sqrt(D) over the visible pairs) v with
    qr = R q and kr = R k, R the per-token 3D rotation (an orthogonal map: a 2x2
    rotation per pair).  By the chain rule, with P the probabilities:
        dv  = P^T dO,   dP = dO v^T,   dS = P * (dP - rowsum(P * dP)),
        dqr = dS kr / sqrt(D),   dkr = dS^T qr / sqrt(D),
        dq = R^T dqr,   dk = R^T dkr   (R^T turns each pair back by -theta).
    Training form of the same chunk mask (hyper.ai summary, "方法": teacher
    forcing; the walkthrough's training objective, Fig. 14).
    """
    if mode not in (PREFILL, TEACHER_FORCING):
        raise ValueError("the backward covers PREFILL and TEACHER_FORCING")
    B, S, H, D = q.shape
    L = chunk_len(F, gh, gw, n_action)
    if mode == PREFILL:
        theta = rope_angles(*token_positions(S, F, gh, gw, n_action, t_offset, 0), spec)
    else:
        half = num_chunks * L
        th = rope_angles(*token_positions(half, F, gh, gw, n_action, t_offset, 0), spec)
        theta = np.concatenate([th, th], axis=0)
    qr = rotate_pairs(q, theta)
    kr = rotate_pairs(k, theta)
    visible = visibility(mode, L, num_chunks)
    scale = 1.0 / math.sqrt(D)
    dq = np.empty_like(q)
    dk = np.empty_like(k)
    dv = np.empty_like(v)
    for b in range(B):
        for hh in range(H):
            P = softmax_probs((qr[b, :, hh] @ kr[b, :, hh].T) * scale, visible)
            g = do[b, :, hh]
            dv[b, :, hh] = P.T @ g
            dP = g @ v[b, :, hh].T
            dS = P * (dP - (P * dP).sum(axis=1, keepdims=True))
            dq[b, :, hh] = dS @ kr[b, :, hh] * scale
            dk[b, :, hh] = dS.T @ qr[b, :, hh] * scale
    dq = rotate_pairs(dq, -theta)
    dk = rotate_pairs(dk, -theta)
    return dq, dk, dv


def chunk_attn_backward(q_bits, k_bits, v_bits, do_bits, mode: int, F: int, gh: int, gw: int,
                        n_action: int, num_chunks: int, t_offset: int = 0,
                        heads: Optional[slice] = None, spec: RopeSpec = RopeSpec()):
    """``chunk_attn_backward_f64`` on bf16 bit arrays (optionally a slice of heads)."""
    hs = slice(None) if heads is None else heads
    return chunk_attn_backward_f64(widen_bf16(q_bits[:, :, hs]), widen_bf16(k_bits[:, :, hs]),
                                   widen_bf16(v_bits[:, :, hs]), widen_bf16(do_bits[:, :, hs]),
                                   mode, F, gh, gw, n_action, num_chunks, t_offset, spec)


def attention_rows(q_bits, k_bits, v_bits, rows, mode: int, F: int, gh: int, gw: int,
                   n_action: int, num_chunks: int, t_offset: int = 0, kv_len: int = 0,
                   cache_k_bits=None, cache_v_bits=None, cache_len: int = 0,
                   spec: RopeSpec = RopeSpec()):
    """Outputs of selected (b, s, h) rows only, each from the plain definition.

    ``rows`` is a sequence of (b, s, h).  Returns float64 [len(rows), D].  Used
    to check full-size GPU results on a sample of rows.
    """
    L = chunk_len(F, gh, gw, n_action)
    D = q_bits.shape[-1]
    out = np.empty((len(rows), D), dtype=np.float64)
    vis = visibility(mode, L, num_chunks, cache_len=cache_len, kv_len=kv_len)
    groups = {}
    for n, (b, s, h) in enumerate(rows):
        groups.setdefault((b, h), []).append((n, s))
    for (b, h), items in groups.items():
        q, k, v = rotated_operands(q_bits, k_bits, v_bits, mode, F, gh, gw, n_action, num_chunks,
                                   t_offset, cache_k_bits, cache_v_bits, cache_len, spec,
                                   heads=slice(h, h + 1), batch=slice(b, b + 1))
        for n, s in items:
            out[n] = masked_attention(q[:, s:s + 1], k, v, vis[s:s + 1])[0, 0, 0]
    return out


# ---------------------------------------------------------------------------
# KV cache
# ---------------------------------------------------------------------------

def kvcache_append(cache_k: np.ndarray, cache_v: np.ndarray, len_tokens: int,
                   k: np.ndarray, v: np.ndarray) -> int:
    """Copy the chunk's keys/values into cache rows [len, len + L); returns the new length."""
    L = k.shape[1]
    cache_k[:, len_tokens:len_tokens + L] = k
    cache_v[:, len_tokens:len_tokens + L] = v
    return len_tokens + L


def kvcache_replace(cache_k: np.ndarray, cache_v: np.ndarray, chunk_index: int,
                    chunk_len_: int, k: np.ndarray, v: np.ndarray) -> None:
    """Overwrite cache rows [c*L, (c+1)*L) (chunk c) with the observed chunk's keys/values."""
    a = chunk_index * chunk_len_
    cache_k[:, a:a + chunk_len_] = k
    cache_v[:, a:a + chunk_len_] = v


# ---------------------------------------------------------------------------
# FP8 (E4M3) variant of the attention.  The walkthrough's system optimisations
# section: on Blackwell the authors run parts of the DiT in FP8 / NVFP4 and keep
# the rotary embedding in higher precision.  Here the scores QK^T take rotated q
# and k as E4M3 codes with one multiplier per tensor (code = E4M3(x * scale));
# values, probabilities and the output stay as in the bf16 path.
#
# E4M3 (the 8-bit floating-point format with 4 exponent and 3 mantissa bits):
# sign bit, exponent field e (bias 7), mantissa field m; e = 0 encodes the
# subnormals m/8 * 2^-6; e = 15 with m = 7 is NaN; there are no infinities, so
# the largest finite magnitude is 1.75 * 2^8 = 448.
# ---------------------------------------------------------------------------

def e4m3_value(codes: np.ndarray) -> np.ndarray:
    """Exact value of E4M3 codes (uint8) as float64; NaN for the two NaN codes."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c >> 7, -1.0, 1.0)
    e = (c >> 3) & 15
    m = c & 7
    mag = np.where(e == 0, (m / 8.0) * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return sign * mag


def quantize_e4m3(x: np.ndarray, scale: float) -> np.ndarray:
    """E4M3 codes of float32(x * scale): the product is formed in float32 (round to
    nearest even), then rounded to the nearest finite E4M3 value, ties to the even
    code, magnitudes past 448 saturating to 448; the sign is kept (so negative
    values that round to zero give -0); NaN gives the NaN code."""
    y = (np.asarray(x, dtype=np.float32) * np.float32(scale)).astype(np.float32)
    a = np.abs(y.astype(np.float64))
    grid = e4m3_value(np.arange(127, dtype=np.uint8))  # codes 0..126: 0, ..., 448
    hi = np.clip(np.searchsorted(grid, a, side="left"), 0, 126)
    lo = np.clip(hi - 1, 0, 126)
    d_lo = a - grid[lo]
    d_hi = grid[hi] - a
    pick = np.where(d_lo < d_hi, lo, np.where(d_hi < d_lo, hi, np.where(lo % 2 == 0, lo, hi)))
    pick = np.where(a >= 448.0, 126, pick)
    code = pick.astype(np.uint8) | (np.signbit(y).astype(np.uint8) << 7)
    return np.where(np.isnan(y), np.uint8(0x7F) | (np.signbit(y).astype(np.uint8) << 7),
                    code).astype(np.uint8)


def chunk_attn_forward_e4m3(q8: np.ndarray, k8: np.ndarray, v_bits: np.ndarray, mode: int,
                            F: int, gh: int, gw: int, n_action: int, num_chunks: int,
                            q_scale: float, k_scale: float, kv_len: int = 0,
                            cache_k8: Optional[np.ndarray] = None,
                            cache_v_bits: Optional[np.ndarray] = None, cache_len: int = 0,
                            heads: Optional[slice] = None) -> np.ndarray:
    """dz_chunk_attn_forward_e4m3: q and k (and the cache keys) arrive rotated, as E4M3
    codes with multipliers q_scale and k_scale; each operand is its code's value
    divided by its multiplier.  No rotary is applied.  Returns float64 [B, Sq, H, D]."""
    L = chunk_len(F, gh, gw, n_action)
    hs = slice(None) if heads is None else heads
    q = e4m3_value(q8[:, :, hs, :]) / q_scale
    k = e4m3_value(k8[:, :, hs, :]) / k_scale
    v = widen_bf16(v_bits[:, :, hs, :])
    if mode == DECODE and cache_len > 0:
        k = np.concatenate([e4m3_value(cache_k8[:, :cache_len, hs, :]) / k_scale, k], axis=1)
        v = np.concatenate([widen_bf16(cache_v_bits[:, :cache_len, hs, :]), v], axis=1)
    vis = visibility(mode, L, num_chunks, cache_len=cache_len, kv_len=kv_len)
    assert vis.shape == (q.shape[1], k.shape[1]), (vis.shape, q.shape, k.shape)
    return masked_attention(q, k, v, vis)
