"""Pins of the oracle's FP8 (E4M3) functions against things other than themselves.

* Decoding: every one of the 256 codes against torch's float8_e4m3fn (a library
  routine), plus the format's closed forms (1, 2, 448, the smallest subnormal and
  normal, signed zero, NaN).
* Rounding: random float32 across the whole exponent range, every midpoint between
  neighbouring codes (exact ties) and signed zeros against torch's cast to
  float8_e4m3fn; the cast does not saturate (it gives NaN past 448 + 16), so values
  beyond the range are pinned by the saturating reading itself: the largest finite
  code, sign kept.
* Attention on E4M3 operands: the brute-force statement (tests/brute_force.py, no
  shared helper) on operands decoded by torch and divided by their multipliers;
  and an exact invariance: doubling every q value (code exponent + 1) while
  doubling q's multiplier leaves the output bit-identical.
Each planted mistake below must make at least one pin fail.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import brute_force as bf
from oracle import dz_oracle as O
from causal_video_diffusion_rope_b200 import synth

D = 128


def _torch_decode(codes):
    return torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8)).view(
        torch.float8_e4m3fn).to(torch.float64).numpy()


def _torch_cast(x32):
    return torch.from_numpy(np.ascontiguousarray(x32, dtype=np.float32)).to(
        torch.float8_e4m3fn).view(torch.uint8).numpy()


def pin_decode_library():
    codes = np.arange(256, dtype=np.uint8)
    got, ref = O.e4m3_value(codes), _torch_decode(codes)
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])
    assert np.array_equal(np.signbit(got[ok]), np.signbit(ref[ok]))


def pin_decode_closed_forms():
    v = O.e4m3_value(np.array([0x38, 0x40, 0x7E, 0x01, 0x07, 0x08, 0xB8, 0x80, 0x7F, 0xFF],
                              dtype=np.uint8))
    assert v[0] == 1.0 and v[1] == 2.0 and v[2] == 448.0
    assert v[3] == 2.0 ** -9 and v[4] == 7 * 2.0 ** -9 and v[5] == 2.0 ** -6
    assert v[6] == -1.0 and v[7] == 0.0 and np.signbit(v[7])
    assert np.isnan(v[8]) and np.isnan(v[9])
    finite = O.e4m3_value(np.arange(127, dtype=np.uint8))
    assert np.all(np.diff(finite) > 0)


def pin_round_library():
    rng = np.random.default_rng(5)
    n = 200_000
    x = rng.standard_normal(n).astype(np.float32) * np.exp2(rng.integers(-14, 8, n)).astype(np.float32)
    x = np.clip(x, -440.0, 440.0).astype(np.float32)
    grid = O.e4m3_value(np.arange(127, dtype=np.uint8))
    mids = ((grid[:-1] + grid[1:]) / 2).astype(np.float32)
    assert np.array_equal(mids.astype(np.float64), (grid[:-1] + grid[1:]) / 2)  # exact ties
    x = np.concatenate([x, mids, -mids, np.array([0.0, -0.0, 1e-30, -1e-30], np.float32)])
    assert np.array_equal(O.quantize_e4m3(x, 1.0), _torch_cast(x))


def pin_round_saturates():
    x = np.array([448.0, 463.9, 464.0, 500.0, 1e30, -470.0, -1e30], np.float32)
    assert O.quantize_e4m3(x, 1.0).tolist() == [0x7E] * 5 + [0xFE] * 2
    assert O.quantize_e4m3(np.array([np.nan], np.float32), 1.0)[0] & 0x7F == 0x7F


def pin_round_trip_and_scale():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    assert np.array_equal(O.quantize_e4m3(O.e4m3_value(codes).astype(np.float32), 1.0), codes)
    rng = np.random.default_rng(6)
    x = rng.standard_normal(50_000).astype(np.float32)
    s = np.float32(57.3)
    assert np.array_equal(O.quantize_e4m3(x, s), _torch_cast(np.clip(x * s, -440, 440)))


TINY = [  # mode, F, gh, gw, n_action, num_chunks, cache_len, kv_len
    (O.PREFILL, 1, 2, 3, 1, 3, 0, 0),
    (O.TEACHER_FORCING, 1, 1, 3, 0, 2, 0, 0),
    (O.DECODE, 1, 2, 2, 2, 3, 18, 0),
    (O.CROSS, 1, 2, 2, 1, 2, 0, 7),
]


def _tiny_e4m3(case, seed, B=2, H=2):
    mode, F, gh, gw, na, nc, clen, kvl = case
    L = O.chunk_len(F, gh, gw, na)
    Sq = {O.DECODE: L, O.PREFILL: nc * L, O.TEACHER_FORCING: 2 * nc * L, O.CROSS: nc * L}[mode]
    Sk = kvl if mode == O.CROSS else Sq
    rng = np.random.default_rng(seed)
    q8 = synth.normal_e4m3(rng, (B, Sq, H, D), 48.0)
    k8 = synth.normal_e4m3(rng, (B, Sk, H, D), 40.0)
    v = synth.normal_bf16(rng, (B, Sk, H, D))
    ck8 = synth.normal_e4m3(rng, (B, clen, H, D), 40.0) if clen else None
    cv = synth.normal_bf16(rng, (B, clen, H, D)) if clen else None
    return L, q8, k8, v, ck8, cv


def pin_attention_brute_force():
    for n, case in enumerate(TINY):
        mode, F, gh, gw, na, nc, clen, kvl = case
        L, q8, k8, v, ck8, cv = _tiny_e4m3(case, 70 + n)
        got = O.chunk_attn_forward_e4m3(q8, k8, v, mode, F, gh, gw, na, nc, 48.0, 40.0, kv_len=kvl,
                                        cache_k8=ck8, cache_v_bits=cv, cache_len=clen)
        ref = bf.attention((_torch_decode(q8) / 48.0).tolist(), (_torch_decode(k8) / 40.0).tolist(),
                           O.widen_bf16(v).tolist(), mode, L, nc, F, gh, gw,
                           cache_k=None if ck8 is None else (_torch_decode(ck8) / 40.0).tolist(),
                           cache_v=None if cv is None else O.widen_bf16(cv).tolist(),
                           cache_len=clen, kv_len=kvl, rotate=False)
        ref = np.array(ref)
        assert np.abs(got - ref).max() / np.abs(ref).max() < 1e-12, case


def pin_attention_scale_invariance():
    case = TINY[2]
    mode, F, gh, gw, na, nc, clen, kvl = case
    L, q8, k8, v, ck8, cv = _tiny_e4m3(case, 90)
    e = (q8 >> 3) & 15
    q8 = np.where((e >= 1) & (e <= 13), q8, np.uint8(0x38) | (q8 & 0x80)).astype(np.uint8)
    q8x2 = (q8 + 8).astype(np.uint8)  # exponent + 1: every value doubles
    assert np.array_equal(_torch_decode(q8x2), 2 * _torch_decode(q8))
    a = O.chunk_attn_forward_e4m3(q8, k8, v, mode, F, gh, gw, na, nc, 48.0, 40.0,
                                  cache_k8=ck8, cache_v_bits=cv, cache_len=clen)
    b = O.chunk_attn_forward_e4m3(q8x2, k8, v, mode, F, gh, gw, na, nc, 96.0, 40.0,
                                  cache_k8=ck8, cache_v_bits=cv, cache_len=clen)
    assert np.array_equal(a, b)


E4M3_PINS = [pin_decode_library, pin_decode_closed_forms, pin_round_library, pin_round_saturates,
             pin_round_trip_and_scale, pin_attention_brute_force, pin_attention_scale_invariance]


@pytest.mark.parametrize("pin", E4M3_PINS, ids=lambda f: f.__name__)
def test_e4m3_pin(pin):
    pin()


# ---------------------------------------------------------------------------
# planted mistakes
# ---------------------------------------------------------------------------

_orig_value = O.e4m3_value
_orig_attn = O.chunk_attn_forward_e4m3


def _bias_8(codes):
    return _orig_value(codes) / 2.0


def _ties_away(x, scale):
    y = (np.asarray(x, np.float32) * np.float32(scale)).astype(np.float32)
    a = np.abs(y.astype(np.float64))
    grid = _orig_value(np.arange(127, dtype=np.uint8))
    hi = np.clip(np.searchsorted(grid, a, side="left"), 0, 126)
    lo = np.clip(hi - 1, 0, 126)
    pick = np.where(a - grid[lo] < grid[hi] - a, lo, hi)
    pick = np.where(a >= 448.0, 126, pick)
    return (pick.astype(np.uint8) | (np.signbit(y).astype(np.uint8) << 7)).astype(np.uint8)


def _truncating(x, scale):
    y = (np.asarray(x, np.float32) * np.float32(scale)).astype(np.float32)
    a = np.abs(y.astype(np.float64))
    grid = _orig_value(np.arange(127, dtype=np.uint8))
    lo = np.clip(np.searchsorted(grid, a, side="right") - 1, 0, 126)
    return (lo.astype(np.uint8) | (np.signbit(y).astype(np.uint8) << 7)).astype(np.uint8)


def _multiplies_by_scale(q8, k8, v_bits, mode, F, gh, gw, na, nc, q_scale, k_scale, **kw):
    return _orig_attn(q8, k8, v_bits, mode, F, gh, gw, na, nc, 1.0 / q_scale, 1.0 / k_scale, **kw)


def _drops_cache(q8, k8, v_bits, mode, F, gh, gw, na, nc, q_scale, k_scale, **kw):
    if kw.get("cache_len", 0):
        L = O.chunk_len(F, gh, gw, na)
        return _orig_attn(q8, k8, v_bits, O.PREFILL, F, gh, gw, na, 1, q_scale, k_scale,
                          heads=kw.get("heads"))
    return _orig_attn(q8, k8, v_bits, mode, F, gh, gw, na, nc, q_scale, k_scale, **kw)


PLANTED = [
    ("e4m3_value", _bias_8),
    ("quantize_e4m3", _ties_away),
    ("quantize_e4m3", _truncating),
    ("chunk_attn_forward_e4m3", _multiplies_by_scale),
    ("chunk_attn_forward_e4m3", _drops_cache),
]


def _fails_some_pin():
    for pin in E4M3_PINS:
        try:
            pin()
        except Exception:
            return True
    return False


@pytest.mark.parametrize("name,fn", PLANTED, ids=[f.__name__ for _, f in PLANTED])
def test_planted_mistake_is_caught(monkeypatch, name, fn):
    monkeypatch.setattr(O, name, fn)
    assert _fails_some_pin(), f"no pin caught the planted mistake {fn.__name__}"
