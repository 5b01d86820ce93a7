"""A second, independent statement of the attention, used only to pin the oracle.

Pure-Python loops over single (query, key) pairs, for tiny inputs only.  It
shares no helper with ``oracle/dz_oracle.py``: visibility is decided from
per-token metadata (chunk number and role) by a predicate written from the
rules directly; the rotary embedding is written as multiplication of the
complex number x[2j] + i*x[2j+1] by exp(i*theta) (the textbook RoFormer form)
rather than as a 2x2 rotation; softmax uses ``math.exp``.
"""
from __future__ import annotations

import cmath
import math
from typing import List, Sequence, Tuple

DECODE, TEACHER_FORCING, PREFILL, CROSS = 0, 1, 2, 3

# token roles
CACHE, SELF, CLEAN, NOISY, COND = "cache", "self", "clean", "noisy", "cond"


def _frequencies(npairs: int, base: float) -> List[float]:
    # RoFormer: theta_j = base^{-2j/d} over the d = 2 * npairs dimensions of the axis
    d = 2 * npairs
    return [1.0 / (base ** (2 * j / d)) for j in range(npairs)]


def _grid_pos(offset_in_chunk: int, chunk_for_position: int, F: int, gh: int, gw: int,
              t_offset: int) -> Tuple[int, int, int]:
    frame_tokens = gh * gw
    if offset_in_chunk >= F * frame_tokens:        # an action token
        return (t_offset + chunk_for_position * F, 0, 0)
    frame = offset_in_chunk // frame_tokens
    row = (offset_in_chunk % frame_tokens) // gw
    col = offset_in_chunk % gw
    return (t_offset + chunk_for_position * F + frame, row, col)


def rotate_token(x: Sequence[float], pos: Tuple[int, int, int], pairs=(22, 21, 21),
                 base: float = 10000.0) -> List[float]:
    freqs = []
    axis_of = []
    for a, n in enumerate(pairs):
        freqs += _frequencies(n, base)
        axis_of += [a] * n
    out = [0.0] * len(x)
    for j in range(len(x) // 2):
        z = complex(x[2 * j], x[2 * j + 1]) * cmath.exp(1j * pos[axis_of[j]] * freqs[j])
        out[2 * j], out[2 * j + 1] = z.real, z.imag
    return out


def token_table(mode: int, L: int, num_chunks: int, F: int, gh: int, gw: int,
                t_offset: int, cache_len: int = 0, kv_len: int = 0):
    """Per-token (role, chunk number, position) lists for queries and keys."""
    queries, keys = [], []
    if mode == DECODE:
        for s in range(L):
            pos = _grid_pos(s, num_chunks, F, gh, gw, t_offset)
            queries.append((SELF, num_chunks, pos))
        for s in range(cache_len):
            keys.append((CACHE, s // L, None))      # stored rotated: no position
        keys += queries
    elif mode == PREFILL:
        for s in range(num_chunks * L):
            c = s // L
            queries.append((CLEAN, c, _grid_pos(s % L, c, F, gh, gw, t_offset)))
        keys = list(queries)
    elif mode == TEACHER_FORCING:
        for s in range(2 * num_chunks * L):
            c = s // L
            if c < num_chunks:
                queries.append((CLEAN, c, _grid_pos(s % L, c, F, gh, gw, t_offset)))
            else:
                i = c - num_chunks
                queries.append((NOISY, i, _grid_pos(s % L, i, F, gh, gw, t_offset)))
        keys = list(queries)
    elif mode == CROSS:
        for s in range(num_chunks * L):
            queries.append((SELF, s // L, None))
        for s in range(kv_len):
            keys.append((COND, 0, None))
    return queries, keys


def may_attend(mode: int, qtok, ktok) -> bool:
    qrole, qc, _ = qtok
    krole, kc, _ = ktok
    if mode == CROSS:
        return True
    if mode == DECODE:
        # the current chunk is the newest: every cached chunk and itself are in the past/present
        return krole in (CACHE, SELF)
    if mode == PREFILL:
        return kc <= qc
    if mode == TEACHER_FORCING:
        if qrole == CLEAN:
            return krole == CLEAN and kc <= qc
        if krole == CLEAN:
            return kc < qc
        return kc == qc
    raise ValueError(mode)


def attention(q, k, v, mode: int, L: int, num_chunks: int, F: int, gh: int, gw: int,
              t_offset: int = 0, cache_k=None, cache_v=None, cache_len: int = 0,
              kv_len: int = 0, pairs=(22, 21, 21), base: float = 10000.0,
              rotate: bool = True):
    """q, k, v: nested lists [B][S][H][D] of floats. Returns [B][Sq][H][D].
    With ``rotate`` false, q and k are taken as already rotated."""
    queries, keys = token_table(mode, L, num_chunks, F, gh, gw, t_offset, cache_len, kv_len)
    B, H, D = len(q), len(q[0][0]), len(q[0][0][0])
    out = [[[None] * H for _ in range(len(queries))] for _ in range(B)]
    for b in range(B):
        for h in range(H):
            # key vectors in the order of ``keys``
            kvecs, vvecs = [], []
            if mode == DECODE:
                for s in range(cache_len):
                    kvecs.append(list(cache_k[b][s][h]))
                    vvecs.append(list(cache_v[b][s][h]))
                for s in range(L):
                    kvecs.append(rotate_token(k[b][s][h], keys[cache_len + s][2], pairs, base)
                                 if rotate else list(k[b][s][h]))
                    vvecs.append(list(v[b][s][h]))
            else:
                for s, tok in enumerate(keys):
                    kk = k[b][s][h]
                    kvecs.append(list(kk) if tok[2] is None or not rotate
                                 else rotate_token(kk, tok[2], pairs, base))
                    vvecs.append(list(v[b][s][h]))
            for i, qt in enumerate(queries):
                qq = q[b][i][h]
                qv = list(qq) if qt[2] is None or not rotate else rotate_token(qq, qt[2], pairs, base)
                scores = []
                for j, kt in enumerate(keys):
                    if may_attend(mode, qt, kt):
                        dot = sum(a * c for a, c in zip(qv, kvecs[j]))
                        scores.append((j, dot / math.sqrt(D)))
                top = max(sc for _, sc in scores)
                weights = [(j, math.exp(sc - top)) for j, sc in scores]
                z = sum(wt for _, wt in weights)
                row = [0.0] * D
                for j, wt in weights:
                    for d in range(D):
                        row[d] += wt * vvecs[j][d]
                out[b][i][h] = [x / z for x in row]
    return out
