"""Per-element error scale of the backward kernels' declared arithmetic.

The backward of the chunk attention (dq, dk, dv for the prefill / teacher-forcing
forms) rounds to bf16, as tensor-core operands: the rotated q and k, the
probabilities P (for dV = P^T dO), the score gradients dS (for dQ = dS K and
dK = dS^T Q), the forward's output O (for D = rowsum(dO * O)), and finally each
result.  Everything else is fp32.  A bf16 rounding (8 significant bits, nearest)
moves x by at most U|x|, U = 2^-8; modelled as uniform within that, its variance
is at most (U x)^2 / 3.

First-order propagation, roundings independent (per batch item and head; S the
scores, qr, kr the rotated operands, g = dO, D the head dimension):
  score error        Var dS_ij   = 2 (U^2/3) sum_d qr_id^2 kr_jd^2 / D
  probabilities      Var dP_ij   = P_ij^2 (Var dS_ij + sum_j' P_ij'^2 Var dS_ij')
                     (the second term: the row normaliser moves with the scores)
  D_i                Var dD_i    = 4 sum_d g_id^2 (U O_id)^2 / 3
                     (bf16 rounding of O, and the forward's own error, of the same size)
  score gradients    A_ij        = Var dP_ij (dP_ij - D_i)^2 + (U dS_ij)^2 / 3
  dq (rotated)       sum_j A_ij kr_jd^2 / D + sum_j dS_ij^2 (U kr_jd)^2/(3D)
                       + Var dD_i (sum_j P_ij kr_jd)^2 / D
  dk (rotated)       sum_i A_ij qr_id^2 / D + sum_i dS_ij^2 (U qr_id)^2/(3D)
                       + sum_i Var dD_i P_ij^2 qr_id^2 / D
  dv                 sum_i (Var dP_ij + (U P_ij)^2 / 3) g_id^2
dq and dk are then turned back by R^T, which mixes the two features of a pair: their
variances are added pairwise.  The bound used by the tests is
  |gpu - ref| <= U |ref| + 8 sigma
(U |ref|: the rounding of the result itself).  The model is checked on the CPU
(tests/test_bwd_error_model.py) against a simulation of those roundings.
"""
import math

import numpy as np

from oracle import dz_oracle as O

U = 2.0 ** -8
SIGMAS = 8.0


def var_round(x):
    return (U * x) ** 2 / 3.0


def pair_sum(x):
    """Per feature, the sum over its rotation pair (features 2p and 2p + 1)."""
    return np.repeat(x[..., 0::2] + x[..., 1::2], 2, axis=-1)


def intermediates(qr, kr, v, g, visible):
    """Exact (fp64) scores, probabilities, output, dP, D and dS of one batch item and head."""
    D = qr.shape[-1]
    P = O.softmax_probs(qr @ kr.T / math.sqrt(D), visible)
    out = P @ v
    dP = g @ v.T
    Dv = (g * out).sum(axis=1)
    dS = P * (dP - Dv[:, None])
    return P, out, dP, Dv, dS


def sigmas(qr, kr, v, g, visible):
    """Standard deviations of the rounding errors of dq, dk, dv ([S, D] each) of one batch
    item and head, from float64 rotated operands qr, kr, values v and output gradient g."""
    D = qr.shape[-1]
    P, out, dP, Dv, dS = intermediates(qr, kr, v, g, visible)
    f = np.float32  # an error scale needs no more precision
    qr2, kr2 = (qr ** 2).astype(f), (kr ** 2).astype(f)
    P, dP, dS, Dv = P.astype(f), dP.astype(f), dS.astype(f), Dv.astype(f)
    var_s = f(2.0 * U * U / 3.0 / D) * (qr2 @ kr2.T)
    P2 = P * P
    var_p = P2 * (var_s + (P2 * var_s).sum(axis=1, keepdims=True))
    del var_s
    var_d = (4.0 * ((g ** 2) * var_round(out)).sum(axis=1)).astype(f)
    A = var_p * (dP - Dv[:, None]) ** 2 + var_round(dS)
    dS2 = dS * dS
    c = f(U * U / 3.0)
    var_dq = (A @ kr2 + dS2 @ (c * kr2)) / D + var_d[:, None] * (P @ kr.astype(f)) ** 2 / D
    var_dk = (A.T @ qr2 + dS2.T @ (c * qr2) + (P2 * var_d[:, None]).T @ qr2) / D
    var_dv = (var_p + var_round(P)).T @ (g.astype(f) ** 2)
    return (np.sqrt(pair_sum(var_dq)).astype(np.float64), np.sqrt(pair_sum(var_dk)).astype(np.float64),
            np.sqrt(var_dv).astype(np.float64))


def operands(q_bits, k_bits, v_bits, do_bits, mode, F, gh, gw, na, N, t0, b, h):
    """Rotated q, k, values and dO (float64 [S, D]) of batch item b and head h."""
    qr, kr, v = O.rotated_operands(q_bits, k_bits, v_bits, mode, F, gh, gw, na, N, t0,
                                   heads=slice(h, h + 1), batch=slice(b, b + 1))
    g = O.widen_bf16(do_bits[b, :, h])
    return qr[0, :, 0], kr[0, :, 0], v[0, :, 0], g


def check(got, ref, sigma, what):
    """Element-wise |got - ref| <= U |ref| + 8 sigma; returns the largest ratio of error to
    bound and the median bound relative to the reference's RMS."""
    err = np.abs(got - ref)
    bound = U * np.abs(ref) + SIGMAS * sigma
    ratio = err / bound
    worst = np.unravel_index(np.argmax(ratio), ratio.shape)
    assert (err <= bound).all(), (f"{what}: |err| {err[worst]:.3e} > bound {bound[worst]:.3e} "
                                  f"at {worst} (ref {ref[worst]:.3e})")
    rms = math.sqrt(float(np.mean(ref ** 2)))
    return float(ratio.max()), float(np.median(bound)) / max(rms, 1e-300)
