"""CPU check of the backward's per-element error model (tests/bwd_error_model.py).

The kernels' declared rounding points are simulated in float64 numpy: rotated q
and k rounded to bf16, the forward's probabilities rounded to bf16 for PV and its
output to bf16, the backward's P (for dV) and dS (for dQ, dK) rounded to bf16, the
results rounded to bf16.  Against the exact oracle, the simulated gradients must
stay inside |sim - ref| <= 2^-8 |ref| + 8 sigma element by element, and sigma must
not be vacuous: the simulated errors' RMS must be a sizeable fraction of the
model's, and a gradient with one corrupted row must fail the bound.
"""
import math

import numpy as np
import pytest

from causal_video_diffusion_rope_b200 import synth
from oracle import dz_oracle as O

import bwd_error_model as M


def bf16(x):
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)
    return np.ldexp(np.round(np.ldexp(m, 8)), e - 8)


def simulate(q_bits, k_bits, v_bits, do_bits, mode, F, gh, gw, na, N, t0):
    """dq, dk, dv [B, S, H, D] with the kernels' rounding points, in float64."""
    L = O.chunk_len(F, gh, gw, na)
    B, S, H, D = q_bits.shape
    qr, kr, v = O.rotated_operands(q_bits, k_bits, v_bits, mode, F, gh, gw, na, N, t0)
    qr, kr = bf16(qr), bf16(kr)
    g = O.widen_bf16(do_bits)
    vis = O.visibility(mode, L, N)
    dqr, dkr, dv = (np.empty((B, S, H, D)) for _ in range(3))
    for b in range(B):
        for h in range(H):
            s = np.where(vis, qr[b, :, h] @ kr[b, :, h].T / math.sqrt(D), -np.inf)
            m = s.max(axis=1, keepdims=True)
            p = np.exp(s - m)
            l = p.sum(axis=1, keepdims=True)
            out = bf16((bf16(p) @ v[b, :, h]) / l)          # forward: bf16 P operand, bf16 O
            P = p / l                                         # backward's recomputed P
            dP = g[b, :, h] @ v[b, :, h].T
            Dv = (g[b, :, h] * out).sum(axis=1, keepdims=True)
            dS = bf16(P * (dP - Dv))
            dv[b, :, h] = bf16(bf16(P).T @ g[b, :, h])
            dqr[b, :, h] = dS @ kr[b, :, h] / math.sqrt(D)
            dkr[b, :, h] = dS.T @ qr[b, :, h] / math.sqrt(D)
    # turn the rotated gradients back (the oracle's own rotation, with minus the angles)
    if mode == O.PREFILL:
        th = O.rope_angles(*O.token_positions(S, F, gh, gw, na, t0, 0), O.RopeSpec())
    else:
        half = O.rope_angles(*O.token_positions(N * L, F, gh, gw, na, t0, 0), O.RopeSpec())
        th = np.concatenate([half, half], axis=0)
    dq = bf16(O.rotate_pairs(dqr, -th))
    dk = bf16(O.rotate_pairs(dkr, -th))
    return dq, dk, dv


CASES = [
    (O.TEACHER_FORCING, 1, 2, 1, 4, 8, 4, 3, 0, 1.0),
    (O.PREFILL, 1, 2, 1, 5, 7, 6, 3, 2, 1.0),
    (O.TEACHER_FORCING, 1, 1, 1, 4, 8, 4, 2, 1, 3.0),   # wider scores (q, k std 3)
]


@pytest.mark.parametrize("mode,B,H,F,gh,gw,na,N,t0,scale", CASES)
def test_error_model_covers_simulated_roundings(mode, B, H, F, gh, gw, na, N, t0, scale):
    rng = np.random.default_rng(90 + N + H)
    L = O.chunk_len(F, gh, gw, na)
    S = (2 if mode == O.TEACHER_FORCING else 1) * N * L
    q = synth.bf16_bits_from_f32(rng.standard_normal((B, S, H, 128)).astype(np.float32) * scale)
    k = synth.bf16_bits_from_f32(rng.standard_normal((B, S, H, 128)).astype(np.float32) * scale)
    v, do = (synth.normal_bf16(rng, (B, S, H, 128)) for _ in range(2))
    ref = O.chunk_attn_backward(q, k, v, do, mode, F, gh, gw, na, N, t0)
    sim = simulate(q, k, v, do, mode, F, gh, gw, na, N, t0)
    vis = O.visibility(mode, L, N)
    for b in range(B):
        for h in range(H):
            sig = M.sigmas(*M.operands(q, k, v, do, mode, F, gh, gw, na, N, t0, b, h), vis)
            for name, s, r, sg in zip(("dq", "dk", "dv"), sim, ref, sig):
                got, want = s[b, :, h], r[b, :, h]
                M.check(got, want, sg, f"{name} b{b} h{h}")
                # not vacuous: the simulated error is a sizeable part of the modelled one
                e_rms = math.sqrt(float(np.mean((got - want) ** 2)))
                s_rms = math.sqrt(float(np.mean(sg ** 2)))
                assert 0.05 < e_rms / s_rms < 3.0, (name, e_rms, s_rms)
                # a corrupted row fails the bound
                bad = got.copy()
                bad[S // 2] *= 0.5
                with pytest.raises(AssertionError):
                    M.check(bad, want, sg, "planted")
