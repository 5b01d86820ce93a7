"""Every kernel's global indexes stay inside their buffers.

libdz_test.so is built with DZ_DEBUG_BOUNDS: each kernel checks the index of every
global store, of the split workspace and counter accesses and of the rotary-table
reads against the extent of the buffer; a failed check skips the access and sets
DZ_ERR_BOUNDS in the handle's status word, which dz_attn_sync_status reports and
dz_attn_sync_status / dz_attn_destroy count on the host (dz_test_bounds_faults).
This stands in for a memory checker, which is not run on these GPUs: the parity
cases of the other GPU test files are run again through the bounds-checked library
(same kernels, same launch shapes) and must agree with the oracle with no fault.
A planted fault, an output extent stated a few tokens short of the real one, must
be reported, with the tokens past the stated extent left unwritten.
"""
import ctypes

import numpy as np
import pytest
import torch

from causal_video_diffusion_rope_b200 import build, dz, synth
from gpu_util import Handle, assert_close, to_dev, to_f64
from oracle import dz_oracle as O

pytestmark = pytest.mark.gpu

D = 128


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def cases(fn):
    """Argument tuples of a test function's parametrize mark (one empty tuple if none)."""
    for m in getattr(fn, "pytestmark", []):
        if m.name == "parametrize":
            out = []
            for v in m.args[1]:
                v = v.values if hasattr(v, "values") else v
                out.append(tuple(v) if isinstance(v, (tuple, list)) else (v,))
            return out
    return [()]


@pytest.fixture(scope="module")
def checked():
    """The dz binding routed to the bounds-checked library for this module's tests."""
    import test_gpu_e4m3 as E
    import test_gpu_parity as P
    product = dz.load()
    P.teardown_module(P)  # handles of the product library, if any are cached
    E.teardown_module(E)
    lib = dz.bind(ctypes.CDLL(build.TEST_LIB))
    lib.dz_test_shrink_out.argtypes = [ctypes.c_int64]
    lib.dz_test_shrink_out.restype = None
    lib.dz_test_bounds_faults.argtypes = []
    lib.dz_test_bounds_faults.restype = ctypes.c_int64
    dz._lib = lib
    lib.dz_test_bounds_faults()
    try:
        yield lib
    finally:
        lib.dz_test_shrink_out(0)
        P.teardown_module(P)  # handles made with the checked library
        E.teardown_module(E)
        dz._lib = product


def run_all(fn, lib):
    for args in cases(fn):
        fn(*args)
    assert lib.dz_test_bounds_faults() == 0, f"{fn.__name__}: index fault"


def test_attention_small_cases_in_bounds(checked):
    import test_gpu_parity as P
    run_all(P.test_attention_elementwise, checked)
    run_all(P.test_attention_elementwise_rotation_in_kernel, checked)
    run_all(P.test_attention_wide_scores, checked)
    run_all(P.test_single_visible_key_exact, checked)


def test_attention_workloads_in_bounds(checked):
    import test_gpu_parity as P
    for fn in (P.test_workload0_tiny_prefill, P.test_workload1_decode_full_elementwise,
               P.test_workload3_teacher_forcing_full_elementwise,
               P.test_workload4_long_cache_and_cross, P.test_workload5_three_view_grid_decode):
        run_all(fn, checked)


def test_rotation_and_cache_ops_in_bounds(checked):
    import test_gpu_parity as P
    run_all(P.test_rope3d_matches_oracle, checked)
    run_all(P.test_kvcache_append_replace_bit_exact, checked)


def test_projection_in_bounds(checked):
    import test_gpu_qkv as Q
    run_all(Q.test_qkv_rope_elementwise, checked)
    run_all(Q.test_qkv_rope_decode_size_with_cache_append, checked)


def test_backward_in_bounds(checked):
    import test_gpu_bwd as B
    run_all(B.test_backward_small, checked)


def test_e4m3_in_bounds(checked):
    import test_gpu_e4m3 as E
    run_all(E.test_e4m3_attention_elementwise, checked)
    E.test_e4m3_workload_full_elementwise(1)
    E.test_e4m3_workload_full_elementwise(3)
    assert checked.dz_test_bounds_faults() == 0, "e4m3 workloads: index fault"


def test_planted_extent_fault_is_reported(checked):
    """The attention is told that its output holds 5 tokens fewer than it does: the
    stores of those tokens fail their check, are skipped (the NaN fill stays) and the
    call reports DZ_ERR_BOUNDS; every other token agrees with the oracle, and the next
    call, with the true extent, is clean."""
    lib = checked
    w = synth.WORKLOADS[0]
    lay, H = w.layout, w.heads
    inp = synth.make_inputs(w, 0)
    ref = O.chunk_attn_forward(inp["q"], inp["k"], inp["v"], lay.mode, lay.frames_per_chunk,
                               lay.grid_h, lay.grid_w, lay.n_action, lay.num_chunks)
    h = Handle(H, prerotate_tokens=0)
    try:
        qd, kd, vd = (to_dev(inp[x]) for x in ("q", "k", "v"))
        out = torch.full((lay.batch, lay.q_len, H, D), float("nan"), dtype=torch.bfloat16,
                         device="cuda")
        short = 5
        lib.dz_test_shrink_out(short * H * D)
        dz.dz_chunk_attn_forward(h.h, qd, kd, vd, None, dz.layout_from(lay), out)
        with pytest.raises(dz.DzError) as e:
            dz.dz_attn_sync_status(h.h)
        assert e.value.status == dz.DZ_ERR_BOUNDS
        assert lib.dz_test_bounds_faults() == 1
        got = to_f64(out)
        keep = lay.q_len - short
        assert np.isnan(got[:, keep:]).all()
        assert_close(got[:, :keep], ref[:, :keep], "tokens inside the stated extent")
        lib.dz_test_shrink_out(0)
        out.fill_(float("nan"))
        dz.dz_chunk_attn_forward(h.h, qd, kd, vd, None, dz.layout_from(lay), out)
        dz.dz_attn_sync_status(h.h)
        assert_close(to_f64(out), ref, "call with the true extent")
    finally:
        lib.dz_test_shrink_out(0)
        h.close()
    assert lib.dz_test_bounds_faults() == 0
