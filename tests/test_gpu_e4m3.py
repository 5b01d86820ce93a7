"""GPU parity of the FP8 (E4M3) variant against the fp64 oracle.

* dz_quantize_e4m3: bit-exact against the oracle's quantize_e4m3.  Both take the
  rounding decision from the same fp32 product bf16(x) * scale, so the codes must
  agree exactly: ties (power-of-two scales make exact midpoints), E4M3 subnormals,
  saturation, signed zeros and infinities included, with ragged lengths.
* dz_chunk_attn_forward_e4m3: the oracle reads the same E4M3 codes, whose values
  are exact in float64, so the kernel differs from it only by its own roundings
  (fp32 accumulation of the E4M3 products, P to bf16, fp32 PV accumulation, bf16
  output) -- the bf16 path's bounds apply unchanged: max |gpu - ref| <= 2e-2 and
  rel-L2 <= 5e-3 per call.
* dz_rope3d_e4m3: the bytes of dz_rope3d followed by dz_quantize_e4m3, and the
  oracle's codes of its own rotation rounded to bf16 except at bf16 rounding
  boundaries (neighbouring codes there).
* The quantisation's own effect (rotation and E4M3 by dz_rope3d_e4m3, then the FP8
  attention, against the oracle on the unquantised bf16 operands):
  E4M3 keeps 3 mantissa bits, so each operand carries a relative rounding error of
  rms eps (about 2.7% for normally distributed values, at most 2^-4); a score
  q.k/sqrt(128) over independent normal entries then moves by about sqrt(2) * eps of
  its own spread, and the output, a softmax average over many keys, by about the
  same fraction: sqrt(2) * 2.7% = 3.8% relative L2.  The test allows 6% (and a max
  abs of 5e-2).
"""
import zlib

import numpy as np
import pytest
import torch

from causal_video_diffusion_rope_b200 import dz, synth
from causal_video_diffusion_rope_b200.synth import (Layout, MODE_CROSS, MODE_DECODE, MODE_PREFILL,
                                                    MODE_TEACHER_FORCING, WORKLOADS)
from gpu_util import Handle, assert_close, to_dev, to_f64
from oracle import dz_oracle as O

pytestmark = pytest.mark.gpu

D = 128
QS, KS = synth.E4M3_Q_SCALE, synth.E4M3_K_SCALE


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dz.load()


_handles = {}


def handle(heads):
    if heads not in _handles:
        _handles[heads] = Handle(heads)
    return _handles[heads].h


def teardown_module(module):
    for h in _handles.values():
        h.close()
    _handles.clear()


def u8_dev(codes: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8)).cuda()


# ------------------------------------------------------------------ quantisation

def _quantize_inputs(rng, n):
    x = rng.standard_normal(n).astype(np.float32) * np.exp2(rng.integers(-16, 4, n)).astype(np.float32)
    bits = synth.bf16_bits_from_f32(x)
    special = np.array([0x0000, 0x8000, 0x7F80, 0xFF80, 0x0001, 0x8001, 0x3F80, 0xBF80, 0x4780,
                        0xC780], dtype=np.uint16)  # +-0, +-inf, +-tiny, +-1, +-65536
    bits[: min(n, special.size)] = special[: min(n, special.size)]
    return bits


@pytest.mark.parametrize("n", [1_000_003, 16, 5, 4096 * 3 + 15])
@pytest.mark.parametrize("scale", [64.0, 57.3, 1.0 / 1024])
def test_quantize_bit_exact(n, scale):
    rng = np.random.default_rng(n * 7 + int(scale * 1000))
    bits = _quantize_inputs(rng, n)
    h = handle(2)
    y = torch.full((n + 32,), 0xAA, dtype=torch.uint8, device="cuda")
    dz.dz_quantize_e4m3(h, to_dev(bits), y, n, scale)
    dz.dz_attn_sync_status(h)
    got = y.cpu().numpy()
    ref = O.quantize_e4m3(synth.f32_from_bf16_bits(bits), scale)
    bad = np.nonzero(got[:n] != ref)[0]
    assert bad.size == 0, f"{bad.size} codes differ, first at {bad[:5]}: got {got[bad[:5]]} ref {ref[bad[:5]]}"
    assert np.all(got[n:] == 0xAA), "wrote past n"


def test_quantize_argument_errors():
    h = handle(2)
    x = torch.zeros(64, dtype=torch.bfloat16, device="cuda")
    y = torch.zeros(64, dtype=torch.uint8, device="cuda")
    for bad in (0.0, -1.0, float("inf"), float("nan")):
        with pytest.raises(dz.DzError) as e:
            dz.dz_quantize_e4m3(h, x, y, 64, bad)
        assert e.value.status == dz.DZ_ERR_INVALID_ARG
    with pytest.raises(dz.DzError) as e:
        dz.dz_quantize_e4m3(h, x, y[1:], 63, 1.0)
    assert e.value.status == dz.DZ_ERR_ALIGNMENT
    dz.dz_quantize_e4m3(h, x, y, 0, 1.0)  # empty: nothing to do


# ------------------------------------------------------------------ rotation + quantisation in one pass

@pytest.mark.parametrize("B,S,H,F,gh,gw,na,t0,first,scale", [
    (1, 108, 2, 1, 4, 8, 4, 0, 0, 64.0),
    (1, 464, 40, 2, 11, 20, 24, 0, 4, 16.0),
    (2, 928, 3, 2, 11, 20, 24, 5, 31, 57.3),
    (1, 37, 1, 1, 1, 1, 0, 100, 0, 1.0 / 8),
])
def test_rope3d_e4m3(B, S, H, F, gh, gw, na, t0, first, scale):
    """dz_rope3d_e4m3 gives the bytes of dz_rope3d followed by dz_quantize_e4m3, and the
    oracle's codes of its own rotation rounded to bf16 (nearest even) everywhere except
    where that rotation lies within fp32 rounding of a bf16 rounding boundary: there the
    two codes may be neighbours."""
    from gpu_util import bf16_round
    rng = np.random.default_rng(11 + S)
    x = synth.bf16_bits_from_f32(rng.standard_normal((B, S, H, D)).astype(np.float32) * 2.0)
    h = handle(H)
    lay = dz.make_layout(0, B, F, gh, gw, na, 0, t0)
    xd = to_dev(x)
    y8 = torch.full((B, S, H, D), 0xAA, dtype=torch.uint8, device="cuda")
    dz.dz_rope3d_e4m3(h, xd, y8, B, S, lay, first, scale)
    y16 = torch.empty_like(xd)
    dz.dz_rope3d(h, xd, y16, B, S, lay, first)
    q8 = torch.empty_like(y8)
    dz.dz_quantize_e4m3(h, y16, q8, q8.numel(), scale)
    dz.dz_attn_sync_status(h)
    got = y8.cpu().numpy()
    assert np.array_equal(got, q8.cpu().numpy()), "fused pass differs from the two calls"
    ref = O.quantize_e4m3(bf16_round(O.rope3d(O.widen_bf16(x), F, gh, gw, na, t0, first))
                          .astype(np.float32), scale)
    bad = np.nonzero(got != ref)
    assert bad[0].size <= max(2, got.size // 100000), bad[0].size
    g, r = got[bad].astype(np.int64), ref[bad].astype(np.int64)
    assert np.all((g & 0x80) == (r & 0x80)) and np.all(np.abs((g & 0x7F) - (r & 0x7F)) <= 1)


def test_rope3d_e4m3_argument_errors():
    h = handle(2)
    lay = dz.make_layout(0, 1, 1, 4, 8, 4, 0, 0)
    x = torch.zeros((1, 36, 2, D), dtype=torch.bfloat16, device="cuda")
    y = torch.zeros((1, 36, 2, D), dtype=torch.uint8, device="cuda")
    for bad in (0.0, -2.0, float("nan")):
        with pytest.raises(dz.DzError) as e:
            dz.dz_rope3d_e4m3(h, x, y, 1, 36, lay, 0, bad)
        assert e.value.status == dz.DZ_ERR_INVALID_ARG
    with pytest.raises(dz.DzError) as e:
        dz.dz_rope3d_e4m3(h, x, x, 1, 36, lay, 0, 1.0)
    assert e.value.status == dz.DZ_ERR_INVALID_ARG


# ------------------------------------------------------------------ attention on E4M3 q, k

def run_e4m3(lay: Layout, heads: int, q8, k8, v, cache_k8=None, cache_v=None, cache_len=0):
    h = handle(heads)
    keep = []
    cache = None
    if lay.mode == MODE_DECODE and cache_k8 is not None:
        ck, cv = u8_dev(cache_k8), to_dev(cache_v)
        keep += [ck, cv]
        cache = dz.make_cache(ck, cv, lay.batch, cache_k8.shape[1], cache_len, lay.chunk_len)
    out = torch.empty((lay.batch, lay.q_len, heads, D), dtype=torch.bfloat16, device="cuda")
    dz.dz_chunk_attn_forward_e4m3(h, u8_dev(q8), u8_dev(k8), to_dev(v), cache, dz.layout_from(lay),
                                  QS, KS, out)
    dz.dz_attn_sync_status(h)
    return to_f64(out)


def oracle_e4m3(lay: Layout, q8, k8, v, cache_k8=None, cache_v=None, cache_len=0):
    return O.chunk_attn_forward_e4m3(q8, k8, v, lay.mode, lay.frames_per_chunk, lay.grid_h,
                                     lay.grid_w, lay.n_action, lay.num_chunks, QS, KS,
                                     kv_len=lay.kv_len, cache_k8=cache_k8, cache_v_bits=cache_v,
                                     cache_len=cache_len)


def L_(mode, B, F, gh, gw, na, N, t0=0, kv=0):
    return Layout(mode, B, F, gh, gw, na, N, t0, kv)


SMALL_CASES = [
    # name, layout, heads, cache_len
    ("tiny_prefill_c0", WORKLOADS[0].layout, 2, 0),
    ("decode_L464_cache1856_h4", L_(MODE_DECODE, 1, 2, 11, 20, 24, 4), 4, 1856),
    ("decode_no_cache", L_(MODE_DECODE, 1, 2, 11, 20, 24, 0), 3, 0),
    ("decode_L36_cache300_b2", L_(MODE_DECODE, 2, 1, 4, 8, 4, 9, 3), 3, 300),
    ("tf_N3_L36", L_(MODE_TEACHER_FORCING, 1, 1, 4, 8, 4, 3), 2, 0),
    ("tf_N2_L464", L_(MODE_TEACHER_FORCING, 1, 2, 11, 20, 24, 2), 2, 0),
    ("prefill_L1_N130", L_(MODE_PREFILL, 1, 1, 1, 1, 0, 130), 1, 0),
    ("cross_464x769_b2", L_(MODE_CROSS, 2, 2, 11, 20, 24, 1, 0, 769), 2, 0),
    ("cross_kv1", L_(MODE_CROSS, 1, 1, 4, 8, 4, 2, 0, 1), 2, 0),
]


@pytest.mark.parametrize("name,lay,heads,cache_len", SMALL_CASES, ids=[c[0] for c in SMALL_CASES])
def test_e4m3_attention_elementwise(name, lay, heads, cache_len):
    rng = np.random.default_rng(zlib.crc32(("e4m3" + name).encode()))
    B = lay.batch
    q8 = synth.normal_e4m3(rng, (B, lay.q_len, heads, D), QS)
    k8 = synth.normal_e4m3(rng, (B, lay.self_kv_len, heads, D), KS)
    v = synth.normal_bf16(rng, (B, lay.self_kv_len, heads, D))
    ck8 = cv = None
    if lay.mode == MODE_DECODE and cache_len > 0:
        cap = cache_len + 77
        ck8 = np.full((B, cap, heads, D), 0x7F, dtype=np.uint8)     # NaN codes past the rows
        cv = np.full((B, cap, heads, D), 0x7FC1, dtype=np.uint16)
        ck8[:, :cache_len] = synth.normal_e4m3(rng, (B, cache_len, heads, D), KS)
        cv[:, :cache_len] = synth.normal_bf16(rng, (B, cache_len, heads, D))
    got = run_e4m3(lay, heads, q8, k8, v, ck8, cv, cache_len)
    assert_close(got, oracle_e4m3(lay, q8, k8, v, ck8, cv, cache_len), "e4m3 " + name)


@pytest.mark.parametrize("wi", [1, 2, 3, 5])
def test_e4m3_workload_full_elementwise(wi):
    w = WORKLOADS[wi]
    lay = w.layout
    inp = synth.make_inputs_e4m3(w, 100 + wi)
    ck8, cv = inp.get("cache_k8"), inp.get("cache_v")
    clen = w.cache_tokens if lay.mode == MODE_DECODE else 0
    got = run_e4m3(lay, w.heads, inp["q8"], inp["k8"], inp["v"], ck8, cv, clen)
    assert_close(got, oracle_e4m3(lay, inp["q8"], inp["k8"], inp["v"], ck8, cv, clen),
                 "e4m3 " + w.name)


def test_e4m3_argument_errors():
    h = handle(2)
    lay = dz.make_layout(MODE_PREFILL, 1, 1, 4, 8, 4, 2)
    q = torch.zeros((1, 72, 2, D), dtype=torch.uint8, device="cuda")
    v = torch.zeros((1, 72, 2, D), dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(v)
    for qs, ks in ((0.0, 1.0), (1.0, -2.0), (float("nan"), 1.0), (1.0, float("inf"))):
        with pytest.raises(dz.DzError) as e:
            dz.dz_chunk_attn_forward_e4m3(h, q, q, v, None, lay, qs, ks, out)
        assert e.value.status == dz.DZ_ERR_INVALID_ARG


def test_e4m3_pipeline_quantisation_error():
    """Workload 1 through the FP8 path from bf16 q, k, v: dz_rope3d_e4m3 (rotation and
    quantisation in one pass) for q and the chunk's k, dz_quantize_e4m3 for the cached
    (already rotated) keys, then the E4M3 attention, against the oracle on the
    unquantised operands."""
    w = WORKLOADS[1]
    lay = w.layout
    B, H, L = lay.batch, w.heads, lay.chunk_len
    inp = synth.make_inputs(w, 11)
    h = handle(H)
    dl = dz.layout_from(lay)
    q8 = torch.empty((B, L, H, D), dtype=torch.uint8, device="cuda")
    k8 = torch.empty_like(q8)
    cap = w.cache_tokens
    ck8 = torch.empty((B, cap, H, D), dtype=torch.uint8, device="cuda")
    dz.dz_rope3d_e4m3(h, to_dev(inp["q"]), q8, B, L, dl, lay.num_chunks, QS)
    dz.dz_rope3d_e4m3(h, to_dev(inp["k"]), k8, B, L, dl, lay.num_chunks, KS)
    dz.dz_quantize_e4m3(h, to_dev(inp["cache_k"]), ck8, ck8.numel(), KS)
    cv = to_dev(inp["cache_v"])
    cache = dz.make_cache(ck8, cv, B, cap, w.cache_tokens, L)
    out = torch.empty((B, L, H, D), dtype=torch.bfloat16, device="cuda")
    dz.dz_chunk_attn_forward_e4m3(h, q8, k8, to_dev(inp["v"]), cache, dl, QS, KS, out)
    dz.dz_attn_sync_status(h)
    got = to_f64(out)
    ref = O.chunk_attn_forward(inp["q"], inp["k"], inp["v"], lay.mode, lay.frames_per_chunk,
                               lay.grid_h, lay.grid_w, lay.n_action, lay.num_chunks,
                               t_offset=lay.t_offset, cache_k_bits=inp["cache_k"],
                               cache_v_bits=inp["cache_v"], cache_len=w.cache_tokens)
    assert_close(got, ref, "e4m3 pipeline vs unquantised oracle", max_abs_tol=5e-2, rel_tol=6e-2)
