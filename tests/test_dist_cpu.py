"""The multi-rank bench path on the CPU: two gloo ranks, no GPU.

Each (sequence, KV head) unit of the eviction is independent, so ranks shard the work
by layer with no data-path collective; the only exchange is the max of the elapsed
times after the timed region. These checks cover that host-side logic: every rank gets
its own inputs, the max over ranks is the slowest rank's time, and the whole-job time
per layer counts every rank's layers. Each rank also evicts its own layer (with the CPU
oracle, which stands in for the GPU path here): the kept positions each rank finds
equal a single-process eviction of that rank's layer, and no data crosses ranks.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        wl = synth.WORKLOADS["tiny"]
        inp = synth.make_inputs(wl, layer=bench.rank_layer(rank))
        # the slowest rank's time wins; every rank sees the same result
        elapsed = 10.0 + 5.0 * rank
        slowest = bench.max_over_ranks(elapsed, "cpu", world)
        per_layer = bench.job_ms_per_layer(slowest, steps=4, world=world)
        digest = float(np.frombuffer(inp.k.tobytes()[:4096], dtype=np.uint16).sum())
        np.save(os.path.join(out_dir, f"rank{rank}.npy"),
                np.array([slowest, per_layer, digest, inp.k.shape[2]], dtype=np.float64))
        import oracle
        kept = oracle.oracle_layer(inp.q_win, inp.k, inp.v, wl.window, wl.budget)["idx"]
        np.save(os.path.join(out_dir, f"idx{rank}.npy"), kept)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_by_layer_and_take_the_slowest_time(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    r0 = np.load(tmp_path / "rank0.npy")
    r1 = np.load(tmp_path / "rank1.npy")
    assert r0[0] == r1[0] == 15.0                 # max over ranks, seen by both
    assert r0[1] == r1[1] == 15.0 / (4 * world)   # 8 layers done in 15 ms
    assert r0[3] == r1[3] == synth.WORKLOADS["tiny"].seq_len
    assert r0[2] != r1[2]                         # distinct seeds: distinct inputs
    # every rank's eviction is the single-process eviction of that rank's own layer
    import oracle
    wl = synth.WORKLOADS["tiny"]
    for rank in range(world):
        inp = synth.make_inputs(wl, layer=bench.rank_layer(rank))
        want = oracle.oracle_layer(inp.q_win, inp.k, inp.v, wl.window, wl.budget)["idx"]
        assert np.array_equal(np.load(tmp_path / f"idx{rank}.npy"), want)
    assert not np.array_equal(np.load(tmp_path / "idx0.npy"), np.load(tmp_path / "idx1.npy"))


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.5, "cpu", 1) == 3.5
    assert bench.job_ms_per_layer(12.0, steps=6, world=1) == 2.0
    assert bench.rank_layer(0) != bench.rank_layer(1)
