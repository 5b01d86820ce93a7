"""The attention kernel's work split (host side), through the test library's
dz_test_plan_schedule: for a call whose (batch, head) pairs each have query groups
with the given key-tile counts, CTA c first takes whole units c + k * grid for
k < waves (head-major order), then the flattened key tiles [tb[c], tb[c + 1]) of
the remaining units; units of equal size get no waves and tb[c] = c * W / grid.
Checked without a GPU: every key tile of every unit is covered exactly once, the
ranges are ordered, the whole-unit waves leave a tail of at least half a wave, and
the estimated work per CTA is balanced.  The tile
counts of the real workloads are counted here from the oracle's visibility matrix."""
import ctypes

import numpy as np
import pytest

from causal_video_diffusion_rope_b200 import build, synth
from oracle import dz_oracle as O

MAX_GRID = 256
SWITCH = 2  # estimated start-up cost of a whole unit, in key tiles (as in the planner)


@pytest.fixture(scope="module")
def lib():
    build.build()
    lib = ctypes.CDLL(build.TEST_LIB)
    lib.dz_test_plan_schedule.argtypes = [ctypes.POINTER(ctypes.c_int32), ctypes.c_int32,
                                          ctypes.c_int64, ctypes.c_int32,
                                          ctypes.POINTER(ctypes.c_int32),
                                          ctypes.POINTER(ctypes.c_int32),
                                          ctypes.POINTER(ctypes.c_uint32)]
    lib.dz_test_plan_schedule.restype = ctypes.c_int32
    return lib


def plan(lib, tiles, bh, sms):
    t = (ctypes.c_int32 * len(tiles))(*tiles)
    g, w = ctypes.c_int32(), ctypes.c_int32()
    tb = (ctypes.c_uint32 * (MAX_GRID + 1))()
    lib.dz_test_plan_schedule(t, len(tiles), bh, sms, ctypes.byref(g), ctypes.byref(w), tb)
    return g.value, w.value, list(tb[:g.value + 1])


def group_tiles(w):
    """Key tiles each 256-row query group of a workload can see (128-key tiles, the
    call's key order: cache first), counted from the oracle's visibility matrix."""
    lay = w.layout
    if lay.mode == synth.MODE_CROSS:
        vis = np.ones((lay.q_len, lay.kv_len), dtype=bool)
    else:
        vis = O.visibility(lay.mode, lay.chunk_len, lay.num_chunks, cache_len=w.cache_tokens)
    nk = vis.shape[1]
    if lay.mode == synth.MODE_DECODE and w.cache_tokens:
        # cache tiles and own-key tiles are separate (the cache need not be tile aligned)
        bounds = list(range(0, w.cache_tokens, 128)) + list(range(w.cache_tokens, nk, 128))
    else:
        bounds = list(range(0, nk, 128))
    bounds.append(nk)
    out = []
    for q0 in range(0, lay.q_len, 256):
        rows = vis[q0:q0 + 256]
        out.append(sum(1 for a, b in zip(bounds[:-1], bounds[1:]) if rows[:, a:b].any()))
    return out


def check(tiles, bh, sms, g, waves, tb):
    tiles = list(tiles)
    n_qg = len(tiles)
    units = bh * n_qg
    W = sum(tiles) * bh
    assert 1 <= g <= min(sms, MAX_GRID)
    start = np.cumsum([0] + [tiles[u % n_qg] for u in range(units)])  # flattened starts
    covered = np.zeros(W, dtype=np.int32)
    load = np.zeros(g)
    for c in range(g):
        for k in range(waves):
            u = c + k * g
            if u < units:
                covered[start[u]:start[u + 1]] += 1
                load[c] += tiles[u % n_qg] + SWITCH
    assert all(a <= b for a, b in zip(tb[:-1], tb[1:]))
    assert tb[g] == W
    if waves:
        assert waves * g <= units
        assert tb[0] == start[min(waves * g, units)]
    for c in range(g):
        covered[tb[c]:tb[c + 1]] += 1
        load[c] += tb[c + 1] - tb[c]
    assert (covered == 1).all()
    return load


@pytest.mark.parametrize("wi", range(len(synth.WORKLOADS)))
def test_real_workloads(lib, wi):
    w = synth.WORKLOADS[wi]
    tiles = group_tiles(w)
    bh = w.layout.batch * w.heads
    g, waves, tb = plan(lib, tiles, bh, 148)
    load = check(tiles, bh, 148, g, waves, tb)
    if waves and tb[0] < tb[g]:
        # whole units plus tail share: balanced within one unit and one tile
        assert load.max() - load.mean() <= max(tiles) + SWITCH + 1


def test_teacher_forcing_uses_whole_unit_waves(lib):
    w = synth.WORKLOADS[3]
    tiles = group_tiles(w)
    g, waves, tb = plan(lib, tiles, w.heads, 148)
    assert g == 148 and waves >= 1
    assert 40 * len(tiles) - waves * g >= g // 2  # a tail of at least half a wave


def test_decode_few_units_one_per_cta(lib):
    # 8 equal units of 3 tiles on 148 SMs: one CTA per unit through the plain split
    g, waves, tb = plan(lib, [3, 3], 4, 148)
    assert g == 8 and waves == 0 and tb == [3 * c for c in range(9)]
    check([3, 3], 4, 148, g, waves, tb)


def test_ragged_few_units_one_per_cta(lib):
    # 8 units of 3 or 4 tiles: one whole-unit wave, no tail
    g, waves, tb = plan(lib, [3, 4], 4, 148)
    assert g == 8 and waves == 1 and tb == [28] * 9  # W = 4 pairs x 7 tiles
    check([3, 4], 4, 148, g, waves, tb)


@pytest.mark.parametrize("wi", range(len(synth.WORKLOADS)))
def test_equal_units_never_use_waves(lib, wi):
    # decode and cross-attention units all see the same key tiles: the plain split
    w = synth.WORKLOADS[wi]
    tiles = group_tiles(w)
    if len(set(tiles)) != 1:
        pytest.skip("ragged units")
    g, waves, tb = plan(lib, tiles, w.layout.batch * w.heads, 148)
    W = sum(tiles) * w.layout.batch * w.heads
    assert waves == 0 and tb == [c * W // g for c in range(g + 1)]


@pytest.mark.parametrize("seed", range(6))
def test_random_tile_lists(lib, seed):
    rng = np.random.default_rng(seed)
    n_qg = int(rng.integers(1, 40))
    tiles = [int(x) for x in rng.integers(1, 60, n_qg)]
    bh = int(rng.integers(1, 90))
    sms = int(rng.choice([7, 63, 132, 148]))
    g, waves, tb = plan(lib, tiles, bh, sms)
    check(tiles, bh, sms, g, waves, tb)
