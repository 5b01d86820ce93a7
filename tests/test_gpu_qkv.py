"""GPU parity of the fused QKV projection + rotation (+ cache append) against the
fp64 oracle, and of attention on inputs given already rotated.

Projection bound per element: |gpu - ref| <= 2^-8 |ref| + 2^-12 A, where A is the
sum over d_model of |x_c w_nc| for the feature (for a rotated pair, of both
features of the pair): one bf16 rounding of the output (half an ulp is 2^-9
relative) plus fp32 accumulation of d_model products.  Over each output tensor
the relative L2 error must also stay below 3e-3 (bf16 rounding alone gives about
2^-9 / sqrt(3) = 1.1e-3).
"""
import numpy as np
import pytest
import torch

from causal_video_diffusion_rope_b200 import dz, synth
from causal_video_diffusion_rope_b200.synth import MODE_DECODE, MODE_PREFILL
from gpu_util import Handle, to_bits, to_dev, to_f64
from oracle import dz_oracle as O

pytestmark = pytest.mark.gpu

D = 128


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dz.load()


def _abs_sums(x_bits, w_bits, heads):
    """A per output feature [B, S, 3, heads, D], pairs merged for the q and k sections."""
    xa = np.abs(O.widen_bf16(x_bits))
    wa = np.abs(O.widen_bf16(w_bits))
    B, S = xa.shape[:2]
    a = (xa @ wa.T).reshape(B, S, 3, heads, D)
    pair = a[..., 0::2] + a[..., 1::2]
    a[:, :, :2, :, 0::2] = pair[:, :, :2]
    a[:, :, :2, :, 1::2] = pair[:, :, :2]
    return a


def _check(got, ref, A, what):
    err = np.abs(got - ref)
    bound = 2.0 ** -8 * np.abs(ref) + 2.0 ** -12 * A
    worst = np.unravel_index(np.argmax(err - bound), err.shape)
    assert (err <= bound).all(), f"{what}: |err| {err[worst]:.3e} > bound {bound[worst]:.3e} at {worst}"
    rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert rel <= 3e-3, f"{what}: rel L2 {rel:.3e}"


def _run(h, heads, B, S, dm, lay, first_chunk, seed, cache=None):
    x, w = synth.projection_inputs(seed, B, S, dm, heads)
    q = torch.empty((B, S, heads, D), dtype=torch.bfloat16, device="cuda")
    k, v = torch.empty_like(q), torch.empty_like(q)
    dz.dz_qkv_rope(h, to_dev(x), to_dev(w), B, S, dm, lay, first_chunk, q, k, v, cache)
    dz.dz_attn_sync_status(h)
    return x, w, q, k, v


@pytest.mark.parametrize("B,heads,dm,F,gh,gw,na,n_chunks,first,t0", [
    (1, 2, 256, 1, 8, 8, 8, 1, 1, 3),        # one partial M tile, 3 N tiles
    (2, 4, 512, 2, 11, 20, 24, 1, 0, 0),     # 928 tokens: 8 M tiles with a ragged tail
    (1, 3, 192, 1, 4, 5, 3, 3, 2, 7),        # odd head count: a tile straddles q/k/v
])
def test_qkv_rope_elementwise(B, heads, dm, F, gh, gw, na, n_chunks, first, t0):
    h = Handle(heads, max_batch=B)
    try:
        L = F * gh * gw + na
        S = n_chunks * L
        lay = dz.make_layout(MODE_PREFILL, B, F, gh, gw, na, n_chunks, t0)
        x, w, q, k, v = _run(h.h, heads, B, S, dm, lay, first, 100 + dm)
        rq, rk, rv = O.qkv_rope(x, w, heads, F, gh, gw, na, t0, first)
        A = _abs_sums(x, w, heads)
        for name, got, ref, a in (("q", q, rq, A[:, :, 0]), ("k", k, rk, A[:, :, 1]),
                                  ("v", v, rv, A[:, :, 2])):
            _check(to_f64(got), ref, a, name)
    finally:
        h.close()


def test_qkv_rope_decode_size_with_cache_append():
    """The DiT layer's projection for one 464-token chunk (d_model 5120, 40 heads:
    240 output tiles, so CTAs take two tiles and both TMEM buffers), appending the
    rotated k and v to a cache of 4 chunks."""
    heads, B, dm = 40, 1, 5120
    w1 = synth.WORKLOADS[1]
    lay = w1.layout
    L = lay.chunk_len
    h = Handle(heads, max_batch=1)
    try:
        cap = 6 * L
        ck = torch.zeros((B, cap, heads, D), dtype=torch.bfloat16, device="cuda")
        cv = torch.zeros_like(ck)
        cache = dz.make_cache(ck, cv, B, cap, 4 * L, L)
        dl = dz.layout_from(lay)
        x, w, q, k, v = _run(h.h, heads, B, L, dm, dl, lay.num_chunks, 7, cache)
        assert cache.len_tokens == 5 * L
        rq, rk, rv = O.qkv_rope(x, w, heads, lay.frames_per_chunk, lay.grid_h, lay.grid_w,
                                lay.n_action, lay.t_offset, lay.num_chunks)
        A = _abs_sums(x, w, heads)
        _check(to_f64(q), rq, A[:, :, 0], "q")
        _check(to_f64(k), rk, A[:, :, 1], "k")
        _check(to_f64(v), rv, A[:, :, 2], "v")
        # the appended rows are the same bits as k and v; nothing else was written
        assert np.array_equal(to_bits(ck[:, 4 * L:5 * L]), to_bits(k))
        assert np.array_equal(to_bits(cv[:, 4 * L:5 * L]), to_bits(v))
        assert not to_bits(ck[:, :4 * L]).any() and not to_bits(ck[:, 5 * L:]).any()
        assert not to_bits(cv[:, :4 * L]).any() and not to_bits(cv[:, 5 * L:]).any()
    finally:
        h.close()


def test_attention_on_given_rotated_inputs_is_bit_identical():
    """DZ_MODE_ROTATED with q, k rotated by dz_rope3d gives the same bits as the
    call that rotates them itself."""
    w1 = synth.WORKLOADS[1]
    lay = w1.layout
    inp = synth.make_inputs(w1, 11)
    h = Handle(w1.heads, prerotate_tokens=8192)
    try:
        B, L, H = lay.batch, lay.chunk_len, w1.heads
        qd, kd, vd = to_dev(inp["q"]), to_dev(inp["k"]), to_dev(inp["v"])
        ck, cv = to_dev(inp["cache_k"]), to_dev(inp["cache_v"])
        cache = dz.make_cache(ck, cv, B, inp["cache_k"].shape[1], w1.cache_tokens, L)
        out_a = torch.empty((B, L, H, D), dtype=torch.bfloat16, device="cuda")
        out_b = torch.empty_like(out_a)
        dz.dz_chunk_attn_forward(h.h, qd, kd, vd, cache, dz.layout_from(lay), out_a)
        qr, kr = torch.empty_like(qd), torch.empty_like(kd)
        rl = dz.make_layout(MODE_PREFILL, B, lay.frames_per_chunk, lay.grid_h, lay.grid_w,
                            lay.n_action, 1, lay.t_offset)
        dz.dz_rope3d(h.h, qd, qr, B, L, rl, lay.num_chunks)
        dz.dz_rope3d(h.h, kd, kr, B, L, rl, lay.num_chunks)
        lr = dz.layout_from(lay)
        lr.mode = MODE_DECODE | dz.DZ_MODE_ROTATED
        dz.dz_chunk_attn_forward(h.h, qr, kr, vd, cache, lr, out_b)
        dz.dz_attn_sync_status(h.h)
        assert torch.equal(out_a.view(torch.int16), out_b.view(torch.int16))
    finally:
        h.close()


def test_qkv_rope_argument_errors():
    h = Handle(2, max_batch=1)
    try:
        lay = dz.make_layout(MODE_PREFILL, 1, 1, 4, 4, 4, 1)
        S = 20
        x, w = synth.projection_inputs(3, 1, S, 128, 2)
        xd, wd = to_dev(x), to_dev(w)
        q = torch.zeros((1, S, 2, D), dtype=torch.bfloat16, device="cuda")
        k, v = torch.zeros_like(q), torch.zeros_like(q)
        with pytest.raises(dz.DzError) as e:
            dz.dz_qkv_rope(h.h, xd, wd, 1, S, 96, lay, 0, q, k, v)          # d_model % 64
        assert e.value.status == dz.DZ_ERR_SHAPE
        with pytest.raises(dz.DzError) as e:
            dz.dz_qkv_rope(h.h, xd, wd, 2, S, 128, lay, 0, q, k, v)         # batch > handle
        assert e.value.status == dz.DZ_ERR_CAPACITY
        ck = torch.zeros((1, 2 * S, 2, D), dtype=torch.bfloat16, device="cuda")
        cv = torch.zeros_like(ck)
        full = dz.make_cache(ck, cv, 1, 2 * S, 2 * S, S)
        with pytest.raises(dz.DzError) as e:
            dz.dz_qkv_rope(h.h, xd, wd, 1, S, 128, lay, 0, q, k, v, full)   # cache full
        assert e.value.status == dz.DZ_ERR_CAPACITY
        wrong = dz.make_cache(ck, cv, 1, 2 * S, 0, S + 1)
        with pytest.raises(dz.DzError) as e:
            dz.dz_qkv_rope(h.h, xd, wd, 1, S, 128, lay, 0, q, k, v, wrong)  # S != chunk_len
        assert e.value.status == dz.DZ_ERR_INVALID_ARG
        torch.cuda.synchronize()
        for t in (q, k, v, ck, cv):
            assert not t.view(torch.int16).any()
        assert full.len_tokens == 2 * S and wrong.len_tokens == 0
    finally:
        h.close()
