"""The allocation-free attention entry point (dz_chunk_attn_forward_noalloc).

Some callers cannot call cudaMalloc (stream capture in global mode, runtimes
that own all device memory through their own pool, fixed-budget plug-ins), so
the library offers attention whose scratch memory is a static device array.
Its output must agree with the handle-based dz_chunk_attn_forward within the
parity tolerance of the other tests, on two calls in a row (the second call
finds the static arrays holding the first call's contents), and with the fp64
oracle itself.  It keeps its own rotary tables: a call with a different rotary
configuration rebuilds them only once the earlier calls are done.  Its device
timeouts are read with dz_attn_sync_status(NULL, stream).  This file is
collected last so that a failure here does not hide the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

from causal_video_diffusion_rope_b200 import build, dz, synth
from gpu_util import assert_close, to_dev, to_f64
from oracle import dz_oracle as O

pytestmark = pytest.mark.gpu


def _inputs(w, seed):
    inp = synth.make_inputs(w, seed)
    lay = w.layout
    q, k, v = to_dev(inp["q"]), to_dev(inp["k"]), to_dev(inp["v"])
    cache = None
    keep = []
    if "cache_k" in inp:
        ck, cv = to_dev(inp["cache_k"]), to_dev(inp["cache_v"])
        keep += [ck, cv]
        cache = dz.make_cache(ck, cv, lay.batch, w.cache_tokens, w.cache_tokens, lay.chunk_len)
    return inp, (q, k, v), cache, keep


def _oracle(w, inp):
    lay = w.layout
    return O.chunk_attn_forward(inp["q"], inp["k"], inp["v"], lay.mode, lay.frames_per_chunk,
                                lay.grid_h, lay.grid_w, lay.n_action, lay.num_chunks,
                                t_offset=lay.t_offset, cache_k_bits=inp.get("cache_k"),
                                cache_v_bits=inp.get("cache_v"), cache_len=w.cache_tokens)


def _run(w, seed):
    lay = w.layout
    inp, (q, k, v), cache, keep = _inputs(w, seed)
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
    dz.dz_attn_sync_status(None)  # no device wait ran out on the allocation-free path
    return inp, to_f64(ref), outs


@pytest.mark.parametrize("wi", [1, 0, 3])
def test_noalloc_matches_handle_path(wi):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    w = synth.WORKLOADS[wi]
    inp, ref, outs = _run(w, 5 + wi)
    for n, got in enumerate(outs):
        assert_close(got, ref, f"noalloc call {n + 1} vs handle path, {w.name}")
    if wi in (0, 1):
        exact = _oracle(w, inp)
        for n, got in enumerate(outs):
            assert_close(got, exact, f"noalloc call {n + 1} vs oracle, {w.name}")


def test_noalloc_rotary_config_change_on_one_stream():
    """Two calls with different rotary tables (max_pos_t) queued back to back on one
    non-blocking stream: the second call's table rebuild must not overwrite the
    tables under the first call's kernel."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    w = synth.WORKLOADS[1]
    lay = w.layout
    inp, (q, k, v), cache, keep = _inputs(w, 77)
    exact = _oracle(w, inp)
    dl = dz.layout_from(lay)
    shape = (lay.batch, lay.q_len, w.heads, 128)
    stream = torch.cuda.Stream()  # non-blocking with respect to the legacy stream
    outs = []
    for max_pos_t in (4096, 1024, 4096):
        desc = dz.make_desc(num_heads=w.heads, max_batch=lay.batch, max_q_tokens=lay.q_len,
                            max_pos_t=max_pos_t)
        out = torch.full(shape, float("nan"), dtype=torch.bfloat16, device="cuda")
        dz.dz_chunk_attn_forward_noalloc(desc, q, k, v, cache, dl, out, stream)
        outs.append(out)
    stream.synchronize()
    dz.dz_attn_sync_status(None, stream)
    for n, out in enumerate(outs):
        assert_close(to_f64(out), exact, f"noalloc call {n + 1} after a rotary table change")


def test_noalloc_timeout_is_reported():
    """With the test build (20 ms device waits) and split counters preset so that a
    merge can never complete, the allocation-free call's timeout is reported by
    dz_attn_sync_status(NULL, stream), which clears it; the next call is correct."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib = dz.bind(ctypes.CDLL(build.TEST_LIB))
    lib.dz_test_fill_split_counters.argtypes = [ctypes.c_int32]
    lib.dz_test_fill_split_counters.restype = None
    w = synth.WORKLOADS[1]  # 80 units over at most 63 CTAs: always split
    lay = w.layout
    inp, (q, k, v), cache, keep = _inputs(w, 78)
    desc = dz.make_desc(num_heads=w.heads, max_batch=lay.batch, max_q_tokens=lay.q_len)
    dl = dz.layout_from(lay)
    out = torch.full((lay.batch, lay.q_len, w.heads, 128), float("nan"), dtype=torch.bfloat16,
                     device="cuda")

    def call():
        return lib.dz_chunk_attn_forward_noalloc(ctypes.byref(desc), q.data_ptr(), k.data_ptr(),
                                                 v.data_ptr(), ctypes.byref(cache),
                                                 ctypes.byref(dl), out.data_ptr(), None)
    try:
        assert call() == dz.DZ_OK  # first call on the device: set-up outside the hook
        assert lib.dz_attn_sync_status(None, None) == dz.DZ_OK
        lib.dz_test_fill_split_counters(0x40000000)
        assert call() == dz.DZ_OK
        assert lib.dz_attn_sync_status(None, None) == dz.DZ_ERR_TIMEOUT
        assert lib.dz_attn_sync_status(None, None) == dz.DZ_OK
        lib.dz_test_fill_split_counters(0)
        out.fill_(float("nan"))
        assert call() == dz.DZ_OK
        assert lib.dz_attn_sync_status(None, None) == dz.DZ_OK
        assert_close(to_f64(out), _oracle(w, inp), "noalloc call after a timeout")
    finally:
        lib.dz_test_fill_split_counters(0)


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
