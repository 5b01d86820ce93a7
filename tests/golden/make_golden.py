"""Write closed-form attention examples to attention_closed_form.json.

The pages print no worked example of the attention, so these fixtures are
built from closed forms: every input is a sparse combination of unit vectors
with bf16-exact coefficients, positions are small integers, and the expected
output is written down with ``math`` from the definitions

  * score(i, j) = <R(p_i) q_i, R(p_j) k_j> / sqrt(128), where R(p) turns the
    complex number x[2m] + i x[2m+1] by exp(i * p_axis(m) * omega_m) and
    omega_m = 10000^(-2 m' / d_axis) (m' = index of the pair inside its axis);
    for unit vectors this reduces to a single cos or sin of one angle;
  * out_i = sum_j exp(score_ij) v_j / sum_j exp(score_ij) over visible j
    (softmax over the visible keys, "DreamZero (WAM) 模型架构" §2.3 block
    diagram; chunk visibility from the paper's method section).

It does not import the oracle or the CUDA library.  Run from the repo root:
    python tests/golden/make_golden.py
"""
import json
import math
import os

D = 128
SQ = math.sqrt(D)


def omega(axis_pairs, m):
    return 10000.0 ** (-2.0 * m / (2 * axis_pairs))


def softmax_combine(scores, vs):
    top = max(scores)
    w = [math.exp(s - top) for s in scores]
    z = sum(w)
    out = [0.0] * D
    for wi, v in zip(w, vs):
        for idx, val in v:
            out[idx] += wi * val / z
    return out


def sparse(*pairs):
    return [list(p) for p in pairs]


cases = []

# A: t-axis pair 0 (omega = 1); the sign of sin is pinned by k0 = e1.
# PREFILL, chunks of one token (F=1, 1x1 grid, no action token): token s sits at t = s.
s10 = math.sin(1.0) / SQ
s11 = 1.0 / SQ
v0, v1 = sparse((3, 1.0)), sparse((4, 1.0))
cases.append(dict(
    name="t_axis_pair0_sin_sign", mode=2, F=1, gh=1, gw=1, n_action=0, num_chunks=2,
    t_offset=0, q=[sparse((0, 1.0)), sparse((0, 1.0))], k=[sparse((1, 1.0)), sparse((0, 1.0))],
    v=[v0, v1], expected={"0": softmax_combine([0.0], [v0]),
                          "1": softmax_combine([s10, s11], [v0, v1])}))

# B: h axis, first h pair (pair 22 -> elements 44, 45), one chunk of 1 frame of 2x1 tokens.
# token 0 at (0,0,0), token 1 at (0,1,0); both in the same chunk, so both see both keys.
v0, v1 = sparse((7, 2.0)), sparse((8, -1.0))
q0 = sparse((44, 1.0))
q1 = sparse((44, 1.0))
k0 = sparse((45, 1.0))
k1 = sparse((44, 1.0))
# row 0 at h=0: <e44, e45> = 0 ; <e44, R_h(1) e44> = cos(1)
# row 1 at h=1: <R_h(1) e44, e45> = sin(1) ; <R_h(1) e44, R_h(1) e44> = 1
cases.append(dict(
    name="h_axis_first_pair", mode=2, F=1, gh=2, gw=1, n_action=0, num_chunks=1, t_offset=0,
    q=[q0, q1], k=[k0, k1], v=[v0, v1],
    expected={"0": softmax_combine([0.0, math.cos(1.0) / SQ], [v0, v1]),
              "1": softmax_combine([math.sin(1.0) / SQ, 1.0 / SQ], [v0, v1])}))

# C: w axis, second w pair (pair 44 -> elements 88, 89), omega = 10000^(-2/42).
w1 = omega(21, 1)
v0, v1 = sparse((0, 1.0), (1, 1.0)), sparse((127, 4.0))
cases.append(dict(
    name="w_axis_second_pair", mode=2, F=1, gh=1, gw=2, n_action=0, num_chunks=1, t_offset=0,
    q=[sparse((88, 2.0)), sparse((88, 2.0))], k=[sparse((89, 2.0)), sparse((88, 1.0))],
    v=[v0, v1],
    expected={"0": softmax_combine([0.0, 2.0 * math.cos(w1) / SQ], [v0, v1]),
              "1": softmax_combine([4.0 * math.sin(w1) / SQ, 2.0 / SQ], [v0, v1])}))

# D: t axis pair 5 (elements 10, 11), omega = 10000^(-10/44); t_offset 3 (positions 3, 4).
w5 = omega(22, 5)
v0, v1 = sparse((20, 1.0)), sparse((21, 1.0))
cases.append(dict(
    name="t_axis_pair5_offset", mode=2, F=1, gh=1, gw=1, n_action=0, num_chunks=2, t_offset=3,
    q=[sparse((10, 4.0)), sparse((10, 4.0))], k=[sparse((11, 8.0)), sparse((10, 2.0), (11, 2.0))],
    v=[v0, v1],
    expected={"0": softmax_combine([0.0], [v0]),
              "1": softmax_combine([32.0 * math.sin(w5) / SQ, 8.0 / SQ], [v0, v1])}))

# E: teacher forcing, N = 1 clean + 1 noisy chunk of one token: clean sees itself,
# noisy sees only itself (no earlier clean chunk).
v0, v1 = sparse((9, 1.5)), sparse((9, -2.5))
cases.append(dict(
    name="teacher_forcing_single", mode=1, F=1, gh=1, gw=1, n_action=0, num_chunks=1, t_offset=0,
    q=[sparse((0, 1.0)), sparse((0, 1.0))], k=[sparse((0, 1.0)), sparse((0, 1.0))],
    v=[v0, v1], expected={"0": softmax_combine([0.0], [v0]), "1": softmax_combine([0.0], [v1])}))

# F: decode. Cache of 2 one-token chunks holding keys already rotated (used as stored);
# the current chunk is chunk 2 at t = 2; its q and k are rotated by t = 2.
# scores: <R(2)e0, e1> = sin 2 ; <R(2)e0, 3 e0> = 3 cos 2 ; <R(2)e0, R(2)e0> = 1
vc0, vc1, vs = sparse((5, 1.0)), sparse((6, 1.0)), sparse((7, 1.0))
cases.append(dict(
    name="decode_cache_unrotated", mode=0, F=1, gh=1, gw=1, n_action=0, num_chunks=2, t_offset=0,
    q=[sparse((0, 1.0))], k=[sparse((0, 1.0))], v=[vs],
    cache_k=[sparse((1, 1.0)), sparse((0, 3.0))], cache_v=[vc0, vc1],
    expected={"0": softmax_combine([math.sin(2.0) / SQ, 3.0 * math.cos(2.0) / SQ, 1.0 / SQ],
                                   [vc0, vc1, vs])}))

# G: cross attention: no rotary, every key visible.
v0, v1, v2 = sparse((1, 1.0)), sparse((2, 1.0)), sparse((3, 1.0))
cases.append(dict(
    name="cross_unmasked", mode=3, F=1, gh=1, gw=1, n_action=0, num_chunks=1, t_offset=0,
    kv_len=3, q=[sparse((0, 2.0))], k=[sparse((0, 1.0)), sparse((0, -1.0)), []], v=[v0, v1, v2],
    expected={"0": softmax_combine([2.0 / SQ, -2.0 / SQ, 0.0], [v0, v1, v2])}))

doc = {
    "source": "Closed forms of softmax(q k^T / sqrt(d)) v with 3D RoPE and the chunk mask "
              "('DreamZero (WAM) 模型架构' §2.3; 'World Action Models are Zero-shot Policies', "
              "method section). Written by tests/golden/make_golden.py with math only.",
    "head_dim": D,
    "cases": cases,
}
path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "attention_closed_form.json")
with open(path, "w") as f:
    json.dump(doc, f, indent=1)
print("wrote", path, len(cases), "cases")
