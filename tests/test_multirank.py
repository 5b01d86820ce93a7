"""Multi-rank host logic of bench.py on CPU (gloo, world size 2).

* every rank's time is reduced with MAX, and the job throughput counts all ranks'
  steps over that time;
* bench.spawn_ranks (what ``bench.py --gpus N`` runs without a launcher) starts N
  processes with the launcher environment, and reports a failing rank;
* the two-GPU CFG split: with world size 2 on a batch-2 workload, rank r runs
  branch r's batch-1 call against its own half of the cache.  Pushed through the
  oracle, the branches gathered from the ranks are exactly the batch-2 call's
  output (the walkthrough's system optimisations: CFG's two branches on two GPUs).
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from causal_video_diffusion_rope_b200 import synth
from oracle import dz_oracle as O

# a small batch-2 decode workload (two CFG branches) over a two-chunk cache
CFG_W = synth.Workload(
    "cfg_decode_small", heads=2,
    layout=synth.Layout(synth.MODE_DECODE, batch=2, frames_per_chunk=1, grid_h=4, grid_w=8,
                        n_action=4, num_chunks=2),
    cache_tokens=2 * 36)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = [12.5, 20.0][rank]
        got = bench.max_over_ranks(ms, world, torch.device("cpu"))
        out[rank] = (got, bench.job_throughput(1e12, 10, world, got))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_gloo():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, join=True,
                       start_method="spawn")
    for r in range(world):
        ms, tf = out[r]
        assert ms == 20.0                      # the slowest rank
        assert tf == pytest.approx(1e12 * 10 * 2 / 20e-3 / 1e12)


def test_single_rank_passthrough():
    assert bench.max_over_ranks(3.0, 1, None) == 3.0
    assert bench.job_throughput(2e12, 5, 1, 10.0) == pytest.approx(1000.0)


def _oracle_call(w, inp):
    lay = w.layout
    return O.chunk_attn_forward(inp["q"], inp["k"], inp["v"], lay.mode, lay.frames_per_chunk,
                                lay.grid_h, lay.grid_w, lay.n_action, lay.num_chunks,
                                t_offset=lay.t_offset, cache_k_bits=inp.get("cache_k"),
                                cache_v_bits=inp.get("cache_v"), cache_len=w.cache_tokens)


def test_rank_work_partition():
    # batch 2 on two ranks: one CFG branch each; otherwise every rank runs a replica
    assert [bench.rank_work(CFG_W, r, 2) for r in range(2)] == [("cfg", 0), ("cfg", 1)]
    assert bench.rank_work(CFG_W, 0, 1) == ("replica", None)
    assert bench.rank_work(CFG_W, 3, 4) == ("replica", None)
    assert bench.rank_work(synth.WORKLOADS[1], 1, 2) == ("replica", None)


def test_cfg_branch_split_reproduces_batch_call():
    inp = synth.make_inputs(CFG_W, 9)
    full = _oracle_call(CFG_W, inp)
    for b in range(2):
        wb, ib = synth.branch_inputs(CFG_W, inp, b)
        assert wb.layout.batch == 1 and ib["cache_k"].shape[0] == 1
        assert np.array_equal(_oracle_call(wb, ib)[0], full[b])


def _spawned_cfg_rank(result_dir):
    """Target of bench.spawn_ranks: the launcher environment is set; run this rank's CFG
    branch through the oracle and gather the branches on rank 0."""
    rank, world = int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"])
    assert os.environ["LOCAL_RANK"] == str(rank) and os.environ["MASTER_ADDR"] == "127.0.0.1"
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        kind, branch = bench.rank_work(CFG_W, rank, world)
        assert kind == "cfg" and branch == rank
        inp = synth.make_inputs(CFG_W, 9)          # the same call on every rank
        wb, ib = synth.branch_inputs(CFG_W, inp, branch)
        mine = torch.from_numpy(_oracle_call(wb, ib))
        parts = [torch.zeros_like(mine) for _ in range(world)]
        dist.all_gather(parts, mine)
        slowest = bench.max_over_ranks([5.0, 7.0][rank], world, torch.device("cpu"))
        if rank == 0:
            got = torch.cat(parts, dim=0).numpy()
            np.save(os.path.join(result_dir, "gathered.npy"), got)
            with open(os.path.join(result_dir, "slowest.txt"), "w") as f:
                f.write(repr(slowest))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _failing_rank():
    if int(os.environ["RANK"]) == 1:
        raise SystemExit(3)


def test_spawn_ranks_runs_cfg_split(tmp_path):
    bench.spawn_ranks(2, _spawned_cfg_rank, str(tmp_path))
    got = np.load(tmp_path / "gathered.npy")
    assert np.array_equal(got, _oracle_call(CFG_W, synth.make_inputs(CFG_W, 9)))
    assert float((tmp_path / "slowest.txt").read_text()) == 7.0


def test_spawn_ranks_reports_a_failing_rank():
    with pytest.raises(RuntimeError, match="rank processes failed"):
        bench.spawn_ranks(2, _failing_rank)
