"""The seeded input recipe (no method arithmetic): determinism, shapes, the NaN fill
past the cached tokens, the K scaling on a fraction of heads, and the projection
inputs' scale."""
import numpy as np

from causal_video_diffusion_rope_b200 import synth
from causal_video_diffusion_rope_b200.synth import Layout, MODE_DECODE, Workload


def _small_decode(**kw):
    return Workload("small_decode", heads=40,
                    layout=Layout(MODE_DECODE, batch=2, frames_per_chunk=1, grid_h=2, grid_w=3,
                                  n_action=2, num_chunks=3),
                    cache_tokens=3 * 8, **kw)


def test_inputs_are_deterministic_and_shaped():
    w = _small_decode()
    a, b = synth.make_inputs(w, 7), synth.make_inputs(w, 7)
    c = synth.make_inputs(w, 8)
    L = w.layout.chunk_len
    assert L == 8
    for k in ("q", "k", "v", "cache_k", "cache_v"):
        assert a[k].dtype == np.uint16 and np.array_equal(a[k], b[k])
        assert not np.array_equal(a[k], c[k])
    assert a["q"].shape == (2, L, 40, 128) and a["cache_k"].shape == (2, 24, 40, 128)


def test_rows_past_the_cached_tokens_hold_nan():
    w = _small_decode()
    inp = synth.make_inputs(w, 1, cache_capacity=40)
    tail = synth.f32_from_bf16_bits(inp["cache_k"][:, 24:])
    assert np.isnan(tail).all()
    assert np.isfinite(synth.f32_from_bf16_bits(inp["cache_k"][:, :24])).all()


def test_k_scaled_on_the_drawn_heads_only():
    w = _small_decode(k_boost=3.0, k_boost_frac=0.05)
    inp = synth.make_inputs(w, 3)
    hx = inp["boosted_heads"]
    assert len(hx) == 2 and len(set(hx.tolist())) == 2
    ck = synth.f32_from_bf16_bits(inp["cache_k"])
    others = np.setdiff1d(np.arange(40), hx)
    assert abs(ck[:, :, hx].std() / ck[:, :, others].std() - 3.0) < 0.15
    v = synth.f32_from_bf16_bits(inp["cache_v"])
    assert abs(v[:, :, hx].std() / v[:, :, others].std() - 1.0) < 0.1


def test_projection_inputs_scale():
    x, w = synth.projection_inputs(0, 1, 64, 512, 2)
    assert x.shape == (1, 64, 512) and w.shape == (3 * 2 * 128, 512)
    wf = synth.f32_from_bf16_bits(w)
    assert abs(wf.std() * np.sqrt(512) - 1.0) < 0.02
    assert abs(synth.f32_from_bf16_bits(x).std() - 1.0) < 0.02
