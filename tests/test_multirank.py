"""The multi-GPU host path of bench.py, on CPU with the gloo backend and two
ranks: the max-over-ranks step time, the barrier, the disjoint per-rank
sequence batches (weak scaling: no collective on the data path) and the
whole-job rate."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import synth

WORLD = 2


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=WORLD)
    try:
        # step times that differ per rank: every rank must see the slowest
        t = bench.max_over_ranks(1.5 + rank, WORLD, device="cpu")
        bench.barrier(WORLD, rank, backend="gloo")
        # this rank's batch of the tiny workload, two sequences per rank
        w = synth.WORKLOADS["tiny_f32"].with_(batch=2)
        K, V, runs = synth.cache_arrays(w, 300, seq_offset=bench.rank_sequences(rank, w.batch))
        np.savez(os.path.join(out_dir, f"rank{rank}.npz"), t=t, K=K, V=V,
                 rate=bench.aggregate_rate(WORLD, w.batch, 10, t))
    finally:
        dist.destroy_process_group()


def test_two_ranks_gloo(tmp_path):
    mp.spawn(_rank_main, args=(_free_port(), str(tmp_path)), nprocs=WORLD, join=True)
    res = [np.load(tmp_path / f"rank{r}.npz") for r in range(WORLD)]
    assert [float(r["t"]) for r in res] == [2.5, 2.5]
    assert [float(r["rate"]) for r in res] == [WORLD * 2 * 10 / 2.5] * 2
    # the ranks' batches are the global batch's sequences 0-1 and 2-3
    w4 = synth.WORKLOADS["tiny_f32"].with_(batch=4)
    K4, V4, _ = synth.cache_arrays(w4, 300)
    for r in range(WORLD):
        assert np.array_equal(res[r]["K"], K4[2 * r:2 * r + 2])
        assert np.array_equal(res[r]["V"], V4[2 * r:2 * r + 2])
    assert not np.array_equal(res[0]["K"], res[1]["K"])


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.0, 1) == 3.0
    bench.barrier(1, 0)
    assert bench.rank_sequences(3, 4) == 12
    assert bench.aggregate_rate(1, 4, 8, 2.0) == 16.0
