"""Device-side bounded waits end with DZ_ERR_TIMEOUT instead of hanging.

libdz_test.so is the library built from the same sources with a 20 ms limit on
every device wait and one test-only call, dz_test_fill_split_counters(value):
while it is set, every attention call presets its split counters to `value`
before the kernel runs.  With 0x40000000 (zero low half, nonzero high half) the
pieces of a split unit still count their arrivals as usual, but the piece that
merges the others waits for a publication count that can never be reached.  At
that wait the merging piece has finished all of its own tiles, so no TMA copy or
tensor-core product of its CTA is in flight: the wait runs out after 20 ms, the
kernel records the timeout in the status word and returns.  dz_attn_sync_status
then reports DZ_ERR_TIMEOUT and clears the word and the counters, and the next
call on the same handle must agree with the oracle again.
"""
import ctypes

import numpy as np
import pytest
import torch

from causal_video_diffusion_rope_b200 import build, dz, synth
from gpu_util import assert_close, to_dev, to_f64
from oracle import dz_oracle as O

pytestmark = pytest.mark.gpu

NEVER = 0x40000000
D = 128
# DECODE over a 300-token cache with 160 heads: 160 work units of 4 key tiles, more
# units than SMs, so the call splits units across CTAs on any B200.
H, F, GH, GW, NA, CHUNK, CACHE = 160, 1, 4, 8, 4, 9, 300


def load_test_lib():
    lib = dz.bind(ctypes.CDLL(build.TEST_LIB))
    lib.dz_test_fill_split_counters.argtypes = [ctypes.c_int32]
    lib.dz_test_fill_split_counters.restype = None
    return lib


def inputs(seed):
    rng = np.random.default_rng(seed)
    L = F * GH * GW + NA
    return tuple(synth.normal_bf16(rng, (1, n, H, D)) for n in (L, L, L, CACHE, CACHE))


def oracle(q, k, v, ck, cv):
    return O.chunk_attn_forward(q, k, v, dz.DZ_MODE_DECODE, F, GH, GW, NA, CHUNK,
                                cache_k_bits=ck, cache_v_bits=cv, cache_len=CACHE)


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def test_merge_wait_times_out_then_next_call_is_clean():
    lib = load_test_lib()
    q, k, v, ck, cv = inputs(41)
    qd, kd, vd, ckd, cvd = (to_dev(x) for x in (q, k, v, ck, cv))
    cache = dz.make_cache(ckd, cvd, 1, CACHE, CACHE, F * GH * GW + NA)
    lay = dz.make_layout(dz.DZ_MODE_DECODE, 1, F, GH, GW, NA, CHUNK)
    desc = dz.make_desc(num_heads=H, max_batch=1, max_q_tokens=64)
    h = ctypes.c_void_p()
    assert lib.dz_attn_create(ctypes.byref(h), ctypes.byref(desc)) == dz.DZ_OK
    out = torch.full_like(qd, float("nan"))
    try:
        lib.dz_test_fill_split_counters(NEVER)
        st = lib.dz_chunk_attn_forward(h, qd.data_ptr(), kd.data_ptr(), vd.data_ptr(),
                                       ctypes.byref(cache), ctypes.byref(lay), out.data_ptr(), None)
        assert st == dz.DZ_OK  # the launch itself succeeds
        assert lib.dz_attn_sync_status(h, None) == dz.DZ_ERR_TIMEOUT
        # the word was cleared by the read
        assert lib.dz_attn_sync_status(h, None) == dz.DZ_OK
        lib.dz_test_fill_split_counters(0)
        out.fill_(float("nan"))
        st = lib.dz_chunk_attn_forward(h, qd.data_ptr(), kd.data_ptr(), vd.data_ptr(),
                                       ctypes.byref(cache), ctypes.byref(lay), out.data_ptr(), None)
        assert st == dz.DZ_OK
        assert lib.dz_attn_sync_status(h, None) == dz.DZ_OK
        assert_close(to_f64(out), oracle(q, k, v, ck, cv), "call after a timeout")
    finally:
        lib.dz_test_fill_split_counters(0)
        lib.dz_attn_destroy(h)
