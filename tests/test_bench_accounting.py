"""The bench's algorithmic work per call (visible query-key pairs, FLOP, bytes) against
independent counts: the oracle's explicit visibility matrix and the tensor sizes."""
import numpy as np
import pytest

import bench
from causal_video_diffusion_rope_b200 import synth
from oracle import dz_oracle as O


@pytest.mark.parametrize("wi", range(len(synth.WORKLOADS)))
def test_visible_pairs_match_oracle_mask(wi):
    w = synth.WORKLOADS[wi]
    lay = w.layout
    L = lay.chunk_len
    vis = O.visibility(lay.mode, L, lay.num_chunks, cache_len=w.cache_tokens, kv_len=lay.kv_len)
    assert vis.shape == (lay.q_len, w.cache_tokens + lay.self_kv_len)
    assert bench.visible_pairs(w) == int(vis.sum())


def test_flop_and_byte_accounting():
    w1 = synth.WORKLOADS[1]
    # 464 queries x 2320 keys, 4 * 128 FLOP per pair, 40 heads
    assert bench.step_flops(w1) == 4 * 128 * 464 * 2320 * 40
    # q, k, v, out of the chunk and the 1856 cached K and V rows, bf16, 40 heads of 128
    assert bench.step_bytes(w1) == (4 * 464 + 2 * 1856) * 40 * 128 * 2
    w4 = synth.WORKLOADS[4]
    cross = 4 * 128 * 464 * (512 + 257) * 40 * 2
    assert bench.step_flops(w4) == 4 * 128 * 464 * (14848 + 464) * 40 * 2 + cross
    # the projection: 2 * tokens * d_model * 3 * 5120
    assert bench.qkv_flops(w1) == 2.0 * 464 * 5120 * 3 * 40 * 128
    # the backward counts five products per visible pair (2.5x the forward)
    w3 = synth.WORKLOADS[3]
    vis = O.visibility(w3.layout.mode, w3.layout.chunk_len, w3.layout.num_chunks)
    assert bench.step_flops(w3) == 4 * 128 * int(vis.sum()) * 40
    assert np.isclose(bench.step_flops(w3) / (4 * 128 * 7424 * 7424 * 40), 0.28125)
