"""GPU parity of the training-form forward (per-row log2 normaliser) and of the
backward of the prefill / teacher-forcing attention against the fp64 oracle.

Bounds.  lse: |gpu - ref| <= 2e-2 in log2 units (the rotated q, k are rounded to
bf16 before the fp32 scores, which moves unit-variance scores by ~1.6e-3 rms).
Gradients, element by element: |gpu - ref| <= 2^-8 |ref| + 8 sigma, sigma the
per-element standard deviation that the kernels' declared roundings give
(tests/bwd_error_model.py: bf16 rotated q and k, through P and dS; P and dS as
bf16 tensor-core operands; D from the bf16 forward output; the bf16 result), and
over each of dq, dk, dv a relative L2 error <= 1e-2.  The oracle uses exact
probabilities and the exact output.
"""
import numpy as np
import pytest
import torch

from causal_video_diffusion_rope_b200 import dz, synth
from causal_video_diffusion_rope_b200.synth import MODE_DECODE, MODE_PREFILL, MODE_TEACHER_FORCING
from gpu_util import Handle, log_errors, to_dev, to_f64
from oracle import dz_oracle as O

import bwd_error_model as M

pytestmark = pytest.mark.gpu

D = 128


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dz.load()


def _rel(got, ref, what=""):
    r = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))
    if what:
        log_errors(what, float(np.abs(got - ref).max()), r, got.size)
    return r


def _run(h, lay, heads, q, k, v, dout):
    B, S = q.shape[0], q.shape[1]
    qd, kd, vd, dod = to_dev(q), to_dev(k), to_dev(v), to_dev(dout)
    out = torch.empty((B, S, heads, D), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, heads, S), dtype=torch.float32, device="cuda")
    dz.dz_chunk_attn_forward_lse(h, qd, kd, vd, lay, out, lse)
    dq, dk, dv = torch.empty_like(qd), torch.empty_like(kd), torch.empty_like(vd)
    dz.dz_chunk_attn_backward(h, qd, kd, vd, out, dod, lse, lay, dq, dk, dv)
    dz.dz_attn_sync_status(h)
    return to_f64(out), lse.double().cpu().numpy(), to_f64(dq), to_f64(dk), to_f64(dv)


def _lse_ref(q, k, v, mode, F, gh, gw, na, N, t0, heads=None):
    qr, kr, _ = O.rotated_operands(q, k, v, mode, F, gh, gw, na, N, t0, heads=heads)
    L = O.chunk_len(F, gh, gw, na)
    vis = O.visibility(mode, L, N)
    B, S, H, _ = qr.shape
    out = np.empty((B, H, S))
    for b in range(B):
        for hh in range(H):
            s = np.where(vis, (qr[b, :, hh] @ kr[b, :, hh].T) / np.sqrt(D), -np.inf)
            m = s.max(axis=1, keepdims=True)
            out[b, hh] = (m[:, 0] + np.log(np.exp(s - m).sum(axis=1))) / np.log(2.0)
    return out


@pytest.mark.parametrize("mode,B,H,F,gh,gw,na,N,t0", [
    (MODE_TEACHER_FORCING, 1, 2, 1, 8, 8, 8, 2, 0),    # 288 tokens: 3 tiles, ragged
    (MODE_PREFILL, 2, 3, 1, 4, 8, 4, 3, 5),             # 108 tokens: one partial tile
    (MODE_TEACHER_FORCING, 1, 2, 2, 5, 7, 6, 3, 2),     # L = 76: chunks across tile edges
])
def test_backward_small(mode, B, H, F, gh, gw, na, N, t0):
    rng = np.random.default_rng(60 + N)
    L = F * gh * gw + na
    S = (2 if mode == MODE_TEACHER_FORCING else 1) * N * L
    q, k, v, dout = (synth.normal_bf16(rng, (B, S, H, D)) for _ in range(4))
    h = Handle(H, max_batch=B, prerotate_tokens=8192)
    try:
        lay = dz.make_layout(mode, B, F, gh, gw, na, N, t0)
        out, lse, dq, dk, dv = _run(h.h, lay, H, q, k, v, dout)
    finally:
        h.close()
    ref_lse = _lse_ref(q, k, v, mode, F, gh, gw, na, N, t0)
    log_errors(f"lse mode {mode} N {N}", float(np.abs(lse - ref_lse).max()), 0.0, lse.size)
    assert np.abs(lse - ref_lse).max() <= 2e-2
    rq, rk, rv = O.chunk_attn_backward(q, k, v, dout, mode, F, gh, gw, na, N, t0)
    for name, got, ref in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
        assert np.isfinite(got).all(), name
        r = _rel(got, ref, f"backward mode {mode} N {N} {name}")
        assert r <= 1e-2, f"{name}: rel L2 {r:.3e}"
    _elementwise(q, k, v, dout, mode, F, gh, gw, na, N, t0, (dq, dk, dv), (rq, rk, rv),
                 [(b, hh) for b in range(B) for hh in range(H)], f"mode {mode} N {N}")


def _elementwise(q, k, v, dout, mode, F, gh, gw, na, N, t0, gots, refs, items, what,
                 ref_heads=None):
    """Every element of dq, dk, dv of the given (batch, head) items within
    2^-8 |ref| + 8 sigma (refs indexed by position in ref_heads when given)."""
    L = O.chunk_len(F, gh, gw, na)
    vis = O.visibility(mode, L, N)
    for b, hh in items:
        hr = hh if ref_heads is None else ref_heads.index(hh)
        sig = M.sigmas(*M.operands(q, k, v, dout, mode, F, gh, gw, na, N, t0, b, hh), vis)
        for name, got, ref, sg in zip(("dq", "dk", "dv"), gots, refs, sig):
            worst, med = M.check(got[b, :, hh], ref[b, :, hr], sg, f"{what} b{b} h{hh} {name}")
            log_errors(f"backward {what} b{b} h{hh} {name} err/bound", worst, med, sg.size)


TF_HEADS = [3, 31] + sorted(int(x) for x in np.random.default_rng(64).choice(
    [hh for hh in range(40) if hh not in (3, 31)], size=6, replace=False))


def test_backward_teacher_forcing_workload_shape():
    """The teacher-forcing training shape (8 clean + 8 noisy chunks of 464 tokens,
    40 heads); eight heads (3, 31 and six drawn from a fixed seed) are compared with
    the oracle element by element over every row -- all 16 chunks, both the clean and
    the noisy half, every 464-token chunk edge inside the 128-row tiles."""
    w = synth.WORKLOADS[3]
    lay = w.layout
    rng = np.random.default_rng(63)
    B, S, H = lay.batch, lay.q_len, w.heads
    q, k, v, dout = (synth.normal_bf16(rng, (B, S, H, D)) for _ in range(4))
    h = Handle(H, max_batch=B, prerotate_tokens=8192)
    try:
        out, lse, dq, dk, dv = _run(h.h, dz.layout_from(lay), H, q, k, v, dout)
    finally:
        h.close()
    args = (lay.mode, lay.frames_per_chunk, lay.grid_h, lay.grid_w, lay.n_action,
            lay.num_chunks, lay.t_offset)
    for hh in TF_HEADS:
        hs = slice(hh, hh + 1)
        rq, rk, rv = O.chunk_attn_backward(q, k, v, dout, *args, heads=hs)
        for name, got, ref in (("dq", dq[:, :, hs], rq), ("dk", dk[:, :, hs], rk),
                               ("dv", dv[:, :, hs], rv)):
            assert np.isfinite(got).all(), name
            r = _rel(got, ref, f"backward teacher forcing 8x2x464 head {hh} {name}")
            assert r <= 1e-2, f"head {hh} {name}: rel L2 {r:.3e}"
        _elementwise(q, k, v, dout, *args, (dq, dk, dv), (rq, rk, rv), [(0, hh)],
                     "teacher forcing 8x2x464", ref_heads=[hh])


def test_backward_argument_errors():
    h = Handle(2, max_batch=1, prerotate_tokens=0)
    try:
        x = torch.zeros((1, 72, 2, D), dtype=torch.bfloat16, device="cuda")
        lse = torch.zeros((1, 2, 72), dtype=torch.float32, device="cuda")
        lay = dz.make_layout(MODE_PREFILL, 1, 1, 8, 8, 8, 1)
        with pytest.raises(dz.DzError) as e:        # no rotation workspace in this handle
            dz.dz_chunk_attn_backward(h.h, x, x, x, x, x, lse, lay, x, x, x)
        assert e.value.status == dz.DZ_ERR_CAPACITY
        dec = dz.make_layout(MODE_DECODE, 1, 1, 8, 8, 8, 1)
        with pytest.raises(dz.DzError) as e:
            dz.dz_chunk_attn_backward(h.h, x, x, x, x, x, lse, dec, x, x, x)
        assert e.value.status == dz.DZ_ERR_UNSUPPORTED
        with pytest.raises(dz.DzError) as e:
            dz.dz_chunk_attn_forward_lse(h.h, x, x, x, dec, x, lse)
        assert e.value.status == dz.DZ_ERR_UNSUPPORTED
    finally:
        h.close()
