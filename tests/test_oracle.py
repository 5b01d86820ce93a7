"""Pins of the CPU oracle against things other than itself (no GPU needed).

Each ``pin_*`` function checks the oracle against a fact fixed by the pages or
by mathematics: hand-written golden tables, closed forms, an independent
brute-force statement (tests/brute_force.py), a library routine
(torch float64 scaled_dot_product_attention), and invariants.  The planted-
mistake tests at the end break the oracle on purpose (on the CPU, in this
process only) and check that some pin fails.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import brute_force as bf
from oracle import dz_oracle as O
from causal_video_diffusion_rope_b200 import synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
D = 128


def _read_table(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append([c == "1" for c in line])
    return np.array(rows, dtype=bool)


def _dense(spvec):
    x = np.zeros(D)
    for i, v in spvec:
        x[i] = v
    return x


def _bits(x):
    """float array whose values are bf16-exact -> bf16 bits."""
    b = synth.bf16_bits_from_f32(np.asarray(x, dtype=np.float32))
    assert np.array_equal(O.widen_bf16(b), np.asarray(x, dtype=np.float64)), "not bf16-exact"
    return b


def _rand_bits(rng, shape, scale=1.0):
    return synth.bf16_bits_from_f32(rng.standard_normal(shape).astype(np.float32) * scale)


def _to_lists(bits):
    return O.widen_bf16(bits).tolist()


# ---------------------------------------------------------------------------
# pins
# ---------------------------------------------------------------------------

def pin_visibility_golden():
    L = 2
    assert np.array_equal(O.visibility(O.PREFILL, L, 3), _read_table("visibility_prefill_3x2.txt"))
    assert np.array_equal(O.visibility(O.TEACHER_FORCING, L, 2),
                          _read_table("visibility_teacher_forcing_2x2.txt"))
    assert O.visibility(O.DECODE, L, 2, cache_len=4).all()
    assert O.visibility(O.DECODE, L, 2, cache_len=4).shape == (2, 6)


def pin_positions_golden():
    with open(os.path.join(GOLDEN, "token_positions.json")) as f:
        doc = json.load(f)
    for case in doc["cases"]:
        n = max(s for s, _ in case["tokens"]) + 1
        t, h, w = O.token_positions(n, case["F"], case["gh"], case["gw"], case["n_action"],
                                    case["t_offset"], case["first_chunk"])
        for s, (et, eh, ew) in case["tokens"]:
            assert (t[s], h[s], w[s]) == (et, eh, ew), (case, s, (t[s], h[s], w[s]))


def pin_attention_closed_forms():
    with open(os.path.join(GOLDEN, "attention_closed_form.json")) as f:
        doc = json.load(f)
    for c in doc["cases"]:
        q = _bits(np.array([_dense(x) for x in c["q"]])[None, :, None, :])
        k = _bits(np.array([_dense(x) for x in c["k"]])[None, :, None, :])
        v = _bits(np.array([_dense(x) for x in c["v"]])[None, :, None, :])
        kw = {}
        if "cache_k" in c:
            kw["cache_k_bits"] = _bits(np.array([_dense(x) for x in c["cache_k"]])[None, :, None, :])
            kw["cache_v_bits"] = _bits(np.array([_dense(x) for x in c["cache_v"]])[None, :, None, :])
            kw["cache_len"] = len(c["cache_k"])
        out = O.chunk_attn_forward(q, k, v, c["mode"], c["F"], c["gh"], c["gw"], c["n_action"],
                                   c["num_chunks"], t_offset=c["t_offset"],
                                   kv_len=c.get("kv_len", 0), **kw)
        for row, expected in c["expected"].items():
            np.testing.assert_allclose(out[0, int(row), 0], np.array(expected), rtol=0,
                                       atol=1e-14, err_msg=c["name"])


def pin_rope_invariants():
    rng = np.random.default_rng(1)
    x = O.widen_bf16(_rand_bits(rng, (1, 36, 2, D)))
    spec = O.RopeSpec()
    # positions all zero: identity
    z = np.zeros(36, dtype=np.int64)
    assert np.array_equal(O.rotate_pairs(x, O.rope_angles(z, z, z, spec)), x)
    # norm of every pair is preserved
    y = O.rope3d(x, 1, 4, 8, 4, 7, 2, spec)
    n0 = x[..., 0::2] ** 2 + x[..., 1::2] ** 2
    n1 = y[..., 0::2] ** 2 + y[..., 1::2] ** 2
    np.testing.assert_allclose(n1, n0, rtol=1e-13, atol=1e-13)
    # the t-only position reduces to textbook 1-D RoPE (complex form) on the first
    # 22 pairs and leaves the h/w pairs untouched
    t = np.arange(36, dtype=np.int64) * 3
    y = O.rotate_pairs(x, O.rope_angles(t, z, z, spec))
    inv = 1.0 / (10000.0 ** (np.arange(0, 44, 2) / 44.0))
    zc = (x[..., 0:44:2] + 1j * x[..., 1:44:2]) * np.exp(1j * t[None, :, None, None] * inv)
    np.testing.assert_allclose(y[..., 0:44:2], zc.real, rtol=0, atol=1e-12)
    np.testing.assert_allclose(y[..., 1:44:2], zc.imag, rtol=0, atol=1e-12)
    assert np.array_equal(y[..., 44:], x[..., 44:])
    # h-only and w-only rotate only their own pairs
    hh = np.arange(36, dtype=np.int64) % 11
    y = O.rotate_pairs(x, O.rope_angles(z, hh, z, spec))
    assert np.array_equal(y[..., :44], x[..., :44]) and np.array_equal(y[..., 86:], x[..., 86:])
    y = O.rotate_pairs(x, O.rope_angles(z, z, hh, spec))
    assert np.array_equal(y[..., :86], x[..., :86])


def pin_rope_relative():
    """Shifting every t position by the same offset leaves every score unchanged."""
    rng = np.random.default_rng(2)
    q = _rand_bits(rng, (1, 72, 2, D))
    k = _rand_bits(rng, (1, 72, 2, D))
    qa = O.rope3d(O.widen_bf16(q), 1, 4, 8, 4, 0, 0)
    ka = O.rope3d(O.widen_bf16(k), 1, 4, 8, 4, 0, 0)
    qb = O.rope3d(O.widen_bf16(q), 1, 4, 8, 4, 17, 0)
    kb = O.rope3d(O.widen_bf16(k), 1, 4, 8, 4, 17, 0)
    sa = np.einsum("bshd,bthd->bhst", qa, ka)
    sb = np.einsum("bshd,bthd->bhst", qb, kb)
    np.testing.assert_allclose(sa, sb, rtol=0, atol=1e-11)


TINY = [
    # mode, F, gh, gw, n_action, num_chunks, t_offset, cache_len, kv_len
    (O.PREFILL, 1, 2, 3, 2, 3, 0, 0, 0),
    (O.PREFILL, 2, 1, 2, 1, 2, 4, 0, 0),
    (O.TEACHER_FORCING, 1, 2, 2, 1, 2, 1, 0, 0),
    (O.TEACHER_FORCING, 1, 1, 3, 0, 3, 0, 0, 0),
    (O.DECODE, 1, 2, 2, 2, 3, 2, 18, 0),
    (O.DECODE, 2, 1, 2, 1, 0, 0, 0, 0),
    (O.CROSS, 1, 2, 2, 1, 2, 0, 0, 7),
]


def _tiny_inputs(case, seed, B=2, H=2):
    mode, F, gh, gw, na, nc, toff, clen, kvl = case
    L = O.chunk_len(F, gh, gw, na)
    Sq = {O.DECODE: L, O.PREFILL: nc * L, O.TEACHER_FORCING: 2 * nc * L, O.CROSS: nc * L}[mode]
    Sk = kvl if mode == O.CROSS else Sq
    rng = np.random.default_rng(seed)
    q = _rand_bits(rng, (B, Sq, H, D))
    k = _rand_bits(rng, (B, Sk, H, D))
    v = _rand_bits(rng, (B, Sk, H, D))
    ck = _rand_bits(rng, (B, clen, H, D)) if clen else None
    cv = _rand_bits(rng, (B, clen, H, D)) if clen else None
    return L, q, k, v, ck, cv


def pin_brute_force():
    for n, case in enumerate(TINY):
        mode, F, gh, gw, na, nc, toff, clen, kvl = case
        L, q, k, v, ck, cv = _tiny_inputs(case, 10 + n)
        got = O.chunk_attn_forward(q, k, v, mode, F, gh, gw, na, nc, t_offset=toff, kv_len=kvl,
                                   cache_k_bits=ck, cache_v_bits=cv, cache_len=clen)
        ref = bf.attention(_to_lists(q), _to_lists(k), _to_lists(v), mode, L, nc, F, gh, gw,
                           t_offset=toff, cache_k=None if ck is None else _to_lists(ck),
                           cache_v=None if cv is None else _to_lists(cv), cache_len=clen,
                           kv_len=kvl)
        ref = np.array(ref)
        err = np.abs(got - ref).max() / np.abs(ref).max()
        assert err < 1e-12, (case, err)


def pin_library_sdpa():
    for n, case in enumerate(TINY):
        mode, F, gh, gw, na, nc, toff, clen, kvl = case
        L, q, k, v, ck, cv = _tiny_inputs(case, 40 + n)
        got = O.chunk_attn_forward(q, k, v, mode, F, gh, gw, na, nc, t_offset=toff, kv_len=kvl,
                                   cache_k_bits=ck, cache_v_bits=cv, cache_len=clen)
        # rotate with the brute-force complex form, then torch float64 SDPA with a bool mask
        queries, keys = bf.token_table(mode, L, nc, F, gh, gw, toff, clen, kvl)
        qq = O.widen_bf16(q)
        kk = O.widen_bf16(k)
        vv = O.widen_bf16(v)
        if mode == O.DECODE:
            kk = np.concatenate([O.widen_bf16(ck), kk], axis=1) if clen else kk
            vv = np.concatenate([O.widen_bf16(cv), vv], axis=1) if clen else vv
        qr = np.array([[[bf.rotate_token(qq[b, i, h], queries[i][2]) if queries[i][2] else qq[b, i, h]
                         for h in range(qq.shape[2])] for i in range(qq.shape[1])]
                       for b in range(qq.shape[0])])
        kr = np.array([[[bf.rotate_token(kk[b, j, h], keys[j][2]) if keys[j][2] else kk[b, j, h]
                         for h in range(kk.shape[2])] for j in range(kk.shape[1])]
                       for b in range(kk.shape[0])])
        mask = np.array([[bf.may_attend(mode, qt, kt) for kt in keys] for qt in queries])
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(qr).permute(0, 2, 1, 3), torch.from_numpy(kr).permute(0, 2, 1, 3),
            torch.from_numpy(vv).permute(0, 2, 1, 3), attn_mask=torch.from_numpy(mask))
        ref = ref.permute(0, 2, 1, 3).numpy()
        err = np.abs(got - ref).max() / np.abs(ref).max()
        assert err < 1e-12, (case, err)


def pin_softmax_rows():
    rng = np.random.default_rng(3)
    s = rng.standard_normal((50, 70)) * 5
    vis = O.visibility(O.TEACHER_FORCING, 5, 7)[:50, :70].copy()
    vis[:, 0] = True
    p = O.softmax_probs(s, vis)
    assert (p >= 0).all()
    assert np.all(p[~vis] == 0)
    np.testing.assert_allclose(p.sum(axis=1), 1.0, rtol=0, atol=1e-12)


def pin_single_visible_key():
    rng = np.random.default_rng(4)
    # chunks of one token: query 0 sees only key 0 -> output is v0 exactly
    q = _rand_bits(rng, (1, 5, 3, D))
    k = _rand_bits(rng, (1, 5, 3, D))
    v = _rand_bits(rng, (1, 5, 3, D))
    out = O.chunk_attn_forward(q, k, v, O.PREFILL, 1, 1, 1, 0, 5)
    assert np.array_equal(out[:, 0], O.widen_bf16(v)[:, 0])
    # teacher forcing: noisy chunk 0 sees only itself
    q = _rand_bits(rng, (1, 6, 3, D))
    k = _rand_bits(rng, (1, 6, 3, D))
    v = _rand_bits(rng, (1, 6, 3, D))
    out = O.chunk_attn_forward(q, k, v, O.TEACHER_FORCING, 1, 1, 1, 0, 3)
    assert np.array_equal(out[:, 3], O.widen_bf16(v)[:, 3])
    assert np.array_equal(out[:, 0], O.widen_bf16(v)[:, 0])


def pin_equal_scores():
    rng = np.random.default_rng(5)
    L = 6
    q = np.zeros((1, 3 * L, 2, D), dtype=np.uint16)    # q = 0: all scores equal
    k = _rand_bits(rng, (1, 3 * L, 2, D))
    v = _rand_bits(rng, (1, 3 * L, 2, D))
    out = O.chunk_attn_forward(q, k, v, O.PREFILL, 1, 2, 2, 2, 3)
    vv = O.widen_bf16(v)
    for c in range(3):
        mean = vv[:, :(c + 1) * L].mean(axis=1)
        for i in range(c * L, (c + 1) * L):
            np.testing.assert_allclose(out[:, i], mean, rtol=0, atol=1e-14)


def pin_causality():
    rng = np.random.default_rng(6)
    L, N = 6, 3
    # prefill: perturbing chunks > c leaves chunk c's outputs bit-identical
    q = _rand_bits(rng, (1, N * L, 2, D))
    k = _rand_bits(rng, (1, N * L, 2, D))
    v = _rand_bits(rng, (1, N * L, 2, D))
    base = O.chunk_attn_forward(q, k, v, O.PREFILL, 1, 2, 2, 2, N)
    for c in range(N - 1):
        k2, v2 = k.copy(), v.copy()
        k2[:, (c + 1) * L:] = _rand_bits(rng, k2[:, (c + 1) * L:].shape)
        v2[:, (c + 1) * L:] = _rand_bits(rng, v2[:, (c + 1) * L:].shape)
        out = O.chunk_attn_forward(q, k2, v2, O.PREFILL, 1, 2, 2, 2, N)
        assert np.array_equal(out[:, :(c + 1) * L], base[:, :(c + 1) * L])
        assert not np.array_equal(out[:, (c + 1) * L:], base[:, (c + 1) * L:])
    # teacher forcing: noisy chunk i's output ignores noisy chunks != i and clean chunks >= i
    q = _rand_bits(rng, (1, 2 * N * L, 2, D))
    k = _rand_bits(rng, (1, 2 * N * L, 2, D))
    v = _rand_bits(rng, (1, 2 * N * L, 2, D))
    base = O.chunk_attn_forward(q, k, v, O.TEACHER_FORCING, 1, 2, 2, 2, N)
    for i in range(N):
        rows = slice((N + i) * L, (N + i + 1) * L)
        k2, v2 = k.copy(), v.copy()
        for c in list(range(i, N)) + [N + j for j in range(N) if j != i]:
            k2[:, c * L:(c + 1) * L] = _rand_bits(rng, (1, L, 2, D))
            v2[:, c * L:(c + 1) * L] = _rand_bits(rng, (1, L, 2, D))
        out = O.chunk_attn_forward(q, k2, v2, O.TEACHER_FORCING, 1, 2, 2, 2, N)
        assert np.array_equal(out[:, rows], base[:, rows])
        # and the clean chunks never see noisy ones
        assert np.array_equal(out[:, :i * L], O.chunk_attn_forward(
            q, k2, v2, O.TEACHER_FORCING, 1, 2, 2, 2, N)[:, :i * L])


def pin_decode_equals_prefill():
    """DECODE over a cache of pre-rotated chunks 0..n-1 == the last chunk's rows of PREFILL."""
    rng = np.random.default_rng(7)
    F, gh, gw, na, n = 1, 2, 3, 2, 3
    L = O.chunk_len(F, gh, gw, na)
    q = _rand_bits(rng, (2, (n + 1) * L, 2, D))
    k = _rand_bits(rng, (2, (n + 1) * L, 2, D))
    v = _rand_bits(rng, (2, (n + 1) * L, 2, D))
    full = O.chunk_attn_forward(q, k, v, O.PREFILL, F, gh, gw, na, n + 1, t_offset=3)
    # the cache holds rotated keys; they are exact in float64 but the API takes bf16,
    # so compare through the float64 path: rotate, then run the DECODE visibility
    kr = O.rope3d(O.widen_bf16(k[:, :n * L]), F, gh, gw, na, 3, 0)
    qd = O.rope3d(O.widen_bf16(q[:, n * L:]), F, gh, gw, na, 3, n)
    kd = O.rope3d(O.widen_bf16(k[:, n * L:]), F, gh, gw, na, 3, n)
    keys = np.concatenate([kr, kd], axis=1)
    vals = O.widen_bf16(v)
    dec = O.masked_attention(qd, keys, vals, O.visibility(O.DECODE, L, n, cache_len=n * L))
    np.testing.assert_allclose(dec, full[:, n * L:], rtol=0, atol=1e-13)


def pin_qkv_identity_blocks():
    """With W = [I; 2I; -I] (d_model = H*128) the projection copies x: q is x rotated,
    k is 2x rotated, v is -x unrotated; fixes the q/k/v section order, the head
    layout of the features and which sections turn."""
    rng = np.random.default_rng(41)
    H, F, gh, gw, na = 2, 1, 2, 3, 2
    L = O.chunk_len(F, gh, gw, na)
    S = 2 * L
    x = _rand_bits(rng, (1, S, H * D))
    eye = np.eye(H * D)
    w = _bits(np.concatenate([eye, 2 * eye, -eye]))
    q, k, v = O.qkv_rope(x, w, H, F, gh, gw, na, 5, 1)
    xs = O.widen_bf16(x).reshape(1, S, H, D)
    for s in range(S):
        pos = bf._grid_pos(s % L, 1 + s // L, F, gh, gw, 5)
        for h in range(H):
            ref = bf.rotate_token(xs[0, s, h].tolist(), pos)
            np.testing.assert_allclose(q[0, s, h], ref, rtol=0, atol=1e-12)
            np.testing.assert_allclose(k[0, s, h], 2 * np.array(ref), rtol=0, atol=1e-12)
    np.testing.assert_array_equal(v, -xs)


def pin_qkv_brute_force():
    """One token's q, k, v by explicit sums over d_model and the complex-number
    rotation, against the oracle's matmul + 2x2 rotation."""
    rng = np.random.default_rng(42)
    H, dm, F, gh, gw, na = 1, 64, 2, 2, 2, 1
    L = O.chunk_len(F, gh, gw, na)
    x = _rand_bits(rng, (1, L, dm))
    w = _rand_bits(rng, (3 * H * D, dm), 0.2)
    q, k, v = O.qkv_rope(x, w, H, F, gh, gw, na, 0, 2)
    xf, wf = O.widen_bf16(x), O.widen_bf16(w)
    for s in (0, 5, L - 1):
        y = [math.fsum(xf[0, s, c] * wf[n, c] for c in range(dm)) for n in range(3 * D)]
        pos = bf._grid_pos(s, 2, F, gh, gw, 0)
        np.testing.assert_allclose(q[0, s, 0], bf.rotate_token(y[:D], pos), rtol=0, atol=1e-11)
        np.testing.assert_allclose(k[0, s, 0], bf.rotate_token(y[D:2 * D], pos), rtol=0, atol=1e-11)
        np.testing.assert_allclose(v[0, s, 0], y[2 * D:], rtol=0, atol=1e-11)


def _forward_f64(q, k, v, mode, F, gh, gw, na, N, t0):
    """The oracle's forward on float64 inputs (rotation + masked attention)."""
    L = O.chunk_len(F, gh, gw, na)
    if mode == O.PREFILL:
        qr = O.rope3d(q, F, gh, gw, na, t0, 0)
        kr = O.rope3d(k, F, gh, gw, na, t0, 0)
    else:
        h = N * L
        qr = np.concatenate([O.rope3d(q[:, :h], F, gh, gw, na, t0, 0),
                             O.rope3d(q[:, h:], F, gh, gw, na, t0, 0)], axis=1)
        kr = np.concatenate([O.rope3d(k[:, :h], F, gh, gw, na, t0, 0),
                             O.rope3d(k[:, h:], F, gh, gw, na, t0, 0)], axis=1)
    return O.masked_attention(qr, kr, v, O.visibility(mode, L, N))


def pin_backward_finite_differences():
    """Central differences of sum(dO * O) against the backward, for elements of q, k
    and v in clean and noisy chunks (teacher forcing) and in prefill."""
    rng = np.random.default_rng(51)
    F, gh, gw, na, N, t0 = 1, 2, 2, 1, 2, 3
    L = O.chunk_len(F, gh, gw, na)
    for mode, S in ((O.TEACHER_FORCING, 2 * N * L), (O.PREFILL, N * L)):
        q, k, v, do = (rng.standard_normal((1, S, 1, D)) for _ in range(4))
        dq, dk, dv = O.chunk_attn_backward_f64(q, k, v, do, mode, F, gh, gw, na, N, t0)
        h = 1e-6
        for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
            for (s, d) in ((0, 0), (L + 1, 37), (S - 1, 101), (S // 2, 64)):
                xp, xm = x.copy(), x.copy()
                xp[0, s, 0, d] += h
                xm[0, s, 0, d] -= h
                def f(xx):
                    qq, kk, vv = (xx if name == "q" else q, xx if name == "k" else k,
                                  xx if name == "v" else v)
                    return float((_forward_f64(qq, kk, vv, mode, F, gh, gw, na, N, t0) * do).sum())
                fd = (f(xp) - f(xm)) / (2 * h)
                assert abs(fd - g[0, s, 0, d]) <= 1e-6 * (1 + abs(fd)), (mode, name, s, d, fd, g[0, s, 0, d])


def pin_backward_autograd():
    """torch float64 autograd through rotation, masked softmax and PV against the
    closed-form backward (two heads, batch 2, teacher forcing)."""
    rng = np.random.default_rng(52)
    F, gh, gw, na, N, t0 = 1, 2, 3, 2, 2, 1
    L = O.chunk_len(F, gh, gw, na)
    S = 2 * N * L
    q, k, v, do = (rng.standard_normal((2, S, 2, D)) for _ in range(4))
    dq, dk, dv = O.chunk_attn_backward_f64(q, k, v, do, O.TEACHER_FORCING, F, gh, gw, na, N, t0)
    th = O.rope_angles(*O.token_positions(N * L, F, gh, gw, na, t0, 0), O.RopeSpec())
    theta = torch.from_numpy(np.concatenate([th, th], axis=0))
    c, sn = torch.cos(theta)[None, :, None, :], torch.sin(theta)[None, :, None, :]
    vis = torch.from_numpy(O.visibility(O.TEACHER_FORCING, L, N))
    tq, tk, tv = (torch.from_numpy(a).requires_grad_() for a in (q, k, v))

    def rot(x):
        x0, x1 = x[..., 0::2], x[..., 1::2]
        return torch.stack([x0 * c - x1 * sn, x0 * sn + x1 * c], dim=-1).flatten(-2)

    qr, kr = rot(tq), rot(tk)
    scores = torch.einsum("bshd,bthd->bhst", qr, kr) / math.sqrt(D)
    p = torch.softmax(scores.masked_fill(~vis, float("-inf")), dim=-1)
    out = torch.einsum("bhst,bthd->bshd", p, tv)
    (out * torch.from_numpy(do)).sum().backward()
    for got, ref in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad)):
        np.testing.assert_allclose(got, ref.numpy(), rtol=0, atol=1e-11)


ALL_PINS = [pin_visibility_golden, pin_positions_golden, pin_attention_closed_forms,
            pin_rope_invariants, pin_rope_relative, pin_brute_force, pin_library_sdpa,
            pin_softmax_rows, pin_single_visible_key, pin_equal_scores, pin_causality,
            pin_decode_equals_prefill, pin_qkv_identity_blocks, pin_qkv_brute_force,
            pin_backward_finite_differences, pin_backward_autograd]


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda f: f.__name__)
def test_oracle_pin(pin):
    pin()


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(8)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 3,
                        np.array([0.0, -0.0, 1e-40, 65504.0, 3.3895e38, np.inf, -np.inf],
                                 dtype=np.float32)])
    ours = synth.bf16_bits_from_f32(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_attention_rows_match_full():
    w = synth.WORKLOADS[0]
    lay = w.layout
    inp = synth.make_inputs(w, 3)
    full = O.chunk_attn_forward(inp["q"], inp["k"], inp["v"], lay.mode, lay.frames_per_chunk,
                                lay.grid_h, lay.grid_w, lay.n_action, lay.num_chunks)
    rows = [(0, 0, 0), (0, 35, 1), (0, 36, 0), (0, 107, 1), (0, 70, 0)]
    got = O.attention_rows(inp["q"], inp["k"], inp["v"], rows, lay.mode, lay.frames_per_chunk,
                           lay.grid_h, lay.grid_w, lay.n_action, lay.num_chunks)
    for n, (b, s, h) in enumerate(rows):
        np.testing.assert_allclose(got[n], full[b, s, h], rtol=0, atol=1e-13)


def test_attention_rows_teacher_forcing_and_decode():
    rng = np.random.default_rng(9)
    for case in [(O.TEACHER_FORCING, 1, 2, 2, 1, 3, 2, 0, 0), (O.DECODE, 1, 2, 2, 2, 3, 2, 18, 0),
                 (O.CROSS, 1, 2, 2, 1, 2, 0, 0, 7)]:
        mode, F, gh, gw, na, nc, toff, clen, kvl = case
        L, q, k, v, ck, cv = _tiny_inputs(case, int(rng.integers(1000)))
        full = O.chunk_attn_forward(q, k, v, mode, F, gh, gw, na, nc, t_offset=toff, kv_len=kvl,
                                    cache_k_bits=ck, cache_v_bits=cv, cache_len=clen)
        rows = [(b, s, h) for b in range(2) for s in range(q.shape[1]) for h in range(2)][::3]
        got = O.attention_rows(q, k, v, rows, mode, F, gh, gw, na, nc, t_offset=toff,
                               kv_len=kvl, cache_k_bits=ck, cache_v_bits=cv, cache_len=clen)
        for n, (b, s, h) in enumerate(rows):
            np.testing.assert_allclose(got[n], full[b, s, h], rtol=0, atol=1e-13)


def test_cache_ops_are_copies():
    rng = np.random.default_rng(11)
    ck = np.zeros((2, 20, 3, D), dtype=np.uint16)
    cv = np.zeros((2, 20, 3, D), dtype=np.uint16)
    k = _rand_bits(rng, (2, 5, 3, D))
    v = _rand_bits(rng, (2, 5, 3, D))
    n = O.kvcache_append(ck, cv, 5, k, v)
    assert n == 10
    assert np.array_equal(ck[:, 5:10], k) and np.array_equal(cv[:, 5:10], v)
    assert not ck[:, :5].any() and not ck[:, 10:].any()
    k2 = _rand_bits(rng, (2, 5, 3, D))
    v2 = _rand_bits(rng, (2, 5, 3, D))
    O.kvcache_replace(ck, cv, 1, 5, k2, v2)
    assert np.array_equal(ck[:, 5:10], k2) and np.array_equal(cv[:, 5:10], v2)


# ---------------------------------------------------------------------------
# planted mistakes: each must make at least one pin fail
# ---------------------------------------------------------------------------

def _fails_some_pin():
    for pin in ALL_PINS:
        try:
            pin()
        except Exception:
            return True
    return False


def _wrong_sign_rotate(x, theta):
    y = np.empty_like(x)
    c = np.cos(theta)[None, :, None, :]
    s = np.sin(theta)[None, :, None, :]
    y[..., 0::2] = x[..., 0::2] * c + x[..., 1::2] * s
    y[..., 1::2] = -x[..., 0::2] * s + x[..., 1::2] * c
    return y


def _swapped_axes_angles(t, h, w, spec):
    return _orig_angles(t, w, h, spec)


_orig_angles = O.rope_angles


def _split_21_22_21(t, h, w, spec):
    return _orig_angles(t, h, w, O.RopeSpec(21, 22, 21, spec.base))


def _global_ladder(t, h, w, spec):
    omega = spec.base ** (-2.0 * np.arange(64) / 128.0)
    pos = np.concatenate([np.repeat(t[:, None], spec.pairs_t, 1), np.repeat(h[:, None], spec.pairs_h, 1),
                          np.repeat(w[:, None], spec.pairs_w, 1)], axis=1)
    return pos * omega[None, :]


_orig_vis = O.visibility


def _tf_noisy_sees_own_clean(mode, L, num_chunks, cache_len=0, kv_len=0):
    v = _orig_vis(mode, L, num_chunks, cache_len, kv_len)
    if mode == O.TEACHER_FORCING:
        v = v.copy()
        N = num_chunks
        for i in range(N):
            v[(N + i) * L:(N + i + 1) * L, i * L:(i + 1) * L] = True
    return v


def _prefill_strict(mode, L, num_chunks, cache_len=0, kv_len=0):
    v = _orig_vis(mode, L, num_chunks, cache_len, kv_len)
    if mode == O.PREFILL:
        c = np.arange(num_chunks * L) // L
        v = (c[:, None] > c[None, :]) | (np.arange(num_chunks * L)[:, None] == np.arange(num_chunks * L)[None, :])
    return v


_orig_masked = O.masked_attention


def _no_scale_attention(q, k, v, visible):
    return _orig_masked(q * math.sqrt(q.shape[-1]), k, v, visible)


_orig_positions = O.token_positions


def _action_at_last_frame(n_tokens, F, gh, gw, n_action, t_offset, first_chunk):
    t, h, w = _orig_positions(n_tokens, F, gh, gw, n_action, t_offset, first_chunk)
    L = F * gh * gw + n_action
    o = np.arange(n_tokens) % L
    t = np.where(o >= F * gh * gw, t + F - 1, t)
    return t, h, w


def _row_major_frames(n_tokens, F, gh, gw, n_action, t_offset, first_chunk):
    t, h, w = _orig_positions(n_tokens, F, gh, gw, n_action, t_offset, first_chunk)
    return t, w % gh if gh > 1 else h, h % gw if gw > 1 else w


_orig_qkv = O.qkv_rope


def _qkv_rotates_v(x_bits, w_bits, heads, F, gh, gw, n_action, t_offset, first_chunk,
                   spec=O.RopeSpec()):
    q, k, v = _orig_qkv(x_bits, w_bits, heads, F, gh, gw, n_action, t_offset, first_chunk, spec)
    return q, k, O.rope3d(v, F, gh, gw, n_action, t_offset, first_chunk, spec)


def _qkv_sections_swapped(x_bits, w_bits, heads, F, gh, gw, n_action, t_offset, first_chunk,
                          spec=O.RopeSpec()):
    q, k, v = _orig_qkv(x_bits, w_bits, heads, F, gh, gw, n_action, t_offset, first_chunk, spec)
    return k, q, v


_orig_bwd = O.chunk_attn_backward_f64


def _bwd_without_rowsum(q, k, v, do, mode, F, gh, gw, n_action, num_chunks, t_offset=0,
                        spec=O.RopeSpec()):
    # dS = P * dP (the rowsum(P * dP) term dropped): recompute everything by hand
    L = O.chunk_len(F, gh, gw, n_action)
    S = q.shape[1]
    if mode == O.PREFILL:
        theta = O.rope_angles(*O.token_positions(S, F, gh, gw, n_action, t_offset, 0), spec)
    else:
        th = O.rope_angles(*O.token_positions(num_chunks * L, F, gh, gw, n_action, t_offset, 0), spec)
        theta = np.concatenate([th, th], axis=0)
    qr, kr = O.rotate_pairs(q, theta), O.rotate_pairs(k, theta)
    vis = O.visibility(mode, L, num_chunks)
    dq, dk, dv = np.empty_like(q), np.empty_like(k), np.empty_like(v)
    sc = 1.0 / math.sqrt(q.shape[-1])
    for b in range(q.shape[0]):
        for hh in range(q.shape[2]):
            P = O.softmax_probs((qr[b, :, hh] @ kr[b, :, hh].T) * sc, vis)
            dv[b, :, hh] = P.T @ do[b, :, hh]
            dS = P * (do[b, :, hh] @ v[b, :, hh].T)
            dq[b, :, hh] = dS @ kr[b, :, hh] * sc
            dk[b, :, hh] = dS.T @ qr[b, :, hh] * sc
    return O.rotate_pairs(dq, -theta), O.rotate_pairs(dk, -theta), dv


def _bwd_rotates_forward(q, k, v, do, mode, F, gh, gw, n_action, num_chunks, t_offset=0,
                         spec=O.RopeSpec()):
    # the gradients turned by +theta twice more instead of back by -theta
    dq, dk, dv = _orig_bwd(q, k, v, do, mode, F, gh, gw, n_action, num_chunks, t_offset, spec)
    L = O.chunk_len(F, gh, gw, n_action)
    S = q.shape[1]
    if mode == O.PREFILL:
        theta = O.rope_angles(*O.token_positions(S, F, gh, gw, n_action, t_offset, 0), spec)
    else:
        th = O.rope_angles(*O.token_positions(num_chunks * L, F, gh, gw, n_action, t_offset, 0), spec)
        theta = np.concatenate([th, th], axis=0)
    return O.rotate_pairs(dq, 2 * theta), O.rotate_pairs(dk, 2 * theta), dv


PLANTED = [
    ("chunk_attn_backward_f64", _bwd_without_rowsum),
    ("chunk_attn_backward_f64", _bwd_rotates_forward),
    ("qkv_rope", _qkv_rotates_v),
    ("qkv_rope", _qkv_sections_swapped),
    ("rotate_pairs", _wrong_sign_rotate),
    ("rope_angles", _swapped_axes_angles),
    ("rope_angles", _split_21_22_21),
    ("rope_angles", _global_ladder),
    ("visibility", _tf_noisy_sees_own_clean),
    ("visibility", _prefill_strict),
    ("masked_attention", _no_scale_attention),
    ("token_positions", _action_at_last_frame),
    ("token_positions", _row_major_frames),
]


@pytest.mark.parametrize("name,fn", PLANTED, ids=[f.__name__ for _, f in PLANTED])
def test_planted_mistake_is_caught(monkeypatch, name, fn):
    monkeypatch.setattr(O, name, fn)
    assert _fails_some_pin(), f"no pin caught the planted mistake {fn.__name__}"
