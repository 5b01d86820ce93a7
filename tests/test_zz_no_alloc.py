"""The allocation-free attention entry point (dz_chunk_attn_forward_noalloc).

Some callers cannot call cudaMalloc (stream capture in global mode, runtimes
that own all device memory through their own pool, fixed-budget plug-ins), so
the library offers attention whose scratch memory is a static device array.
Its output must agree with the handle-based dz_chunk_attn_forward within the
parity tolerance of the other tests, on two calls in a row (the second call
finds the static arrays holding the first call's contents).  This file is
collected last so that a failure here does not hide the other tests.
"""
import ctypes

import pytest
import torch

from causal_video_diffusion_rope_b200 import dz, synth
from gpu_util import assert_close, to_dev, to_f64

pytestmark = pytest.mark.gpu


def _run(w, seed):
    lay = w.layout
    inp = synth.make_inputs(w, seed)
    q, k, v = to_dev(inp["q"]), to_dev(inp["k"]), to_dev(inp["v"])
    cache = None
    keep = []
    if "cache_k" in inp:
        ck, cv = to_dev(inp["cache_k"]), to_dev(inp["cache_v"])
        keep += [ck, cv]
        cache = dz.make_cache(ck, cv, lay.batch, w.cache_tokens, w.cache_tokens, lay.chunk_len)
    desc = dz.make_desc(num_heads=w.heads, max_batch=lay.batch, max_q_tokens=lay.q_len)
    dl = dz.layout_from(lay)
    shape = (lay.batch, lay.q_len, w.heads, 128)

    h = dz.dz_attn_create(desc)
    try:
        ref = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
        dz.dz_chunk_attn_forward(h, q, k, v, cache, dl, ref)
        dz.dz_attn_sync_status(h)
    finally:
        dz.dz_attn_destroy(h)
    outs = []
    for _ in range(2):  # two calls in a row on the same static arrays
        out = torch.full(shape, float("nan"), dtype=torch.bfloat16, device="cuda")
        dz.dz_chunk_attn_forward_noalloc(desc, q, k, v, cache, dl, out)
        torch.cuda.synchronize()
        outs.append(to_f64(out))
    return to_f64(ref), outs


@pytest.mark.parametrize("wi", [1, 0, 3])
def test_noalloc_matches_handle_path(wi):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    w = synth.WORKLOADS[wi]
    ref, outs = _run(w, 5 + wi)
    for n, got in enumerate(outs):
        assert_close(got, ref, f"noalloc call {n + 1} vs handle path, {w.name}")


def test_noalloc_rejects_sizes_beyond_its_arrays():
    lib = dz.load()
    lay = dz.make_layout(dz.DZ_MODE_DECODE, 1, 1, 4, 8, 4, 0)
    big = dz.make_desc(num_heads=40, max_batch=64, max_q_tokens=16384)  # 64*40*64*2 counters
    st = lib.dz_chunk_attn_forward_noalloc(ctypes.byref(big), 16, 16, 16, None, ctypes.byref(lay),
                                           16, None)
    assert st == dz.DZ_ERR_CAPACITY
    wide = dz.make_desc(num_heads=2, max_pos_t=1 << 16)
    st = lib.dz_chunk_attn_forward_noalloc(ctypes.byref(wide), 16, 16, 16, None,
                                           ctypes.byref(lay), 16, None)
    assert st == dz.DZ_ERR_CAPACITY
