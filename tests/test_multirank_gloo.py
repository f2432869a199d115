"""The N > 1 path on the CPU: two gloo ranks split the batch with
shard_range, each computes its slice (with the oracle, standing in for its
GPU), and the slices gathered together equal the single-process result;
the timing reduction returns the slowest rank's time."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from vision_sliding_window_b200.dist import max_over_ranks, shard_range


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_shard_range_partitions_exactly():
    for units in range(0, 40):
        for world in range(1, 9):
            spans = [shard_range(units, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == units
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            sizes = [e - b for b, e in spans]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard_range(4, 2, 2)


def _worker(rank, world, port, result_path):
    import oracle
    from vision_sliding_window_b200.inputs import make_inputs

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q, k, v, rpb = make_inputs(5, 2, 9, 11, 16, 5, "f32", seed=77)
        b0, b1 = shard_range(q.shape[0], rank, world)
        mine = oracle.forward(q[b0:b1], k[b0:b1], v[b0:b1], rpb, 5, nthreads=1)
        parts = [None] * world
        dist.all_gather_object(parts, (b0, b1, mine))
        slowest = max_over_ranks(1.0 + rank)
        if rank == 0:
            full = np.concatenate([p[2] for p in sorted(parts, key=lambda p: p[0])], axis=0)
            np.save(result_path, full)
            assert slowest == float(world)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reassemble_the_batch(tmp_path):
    import oracle
    from vision_sliding_window_b200.inputs import make_inputs

    world, port = 2, _free_port()
    out = str(tmp_path / "gathered.npy")
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
    q, k, v, rpb = make_inputs(5, 2, 9, 11, 16, 5, "f32", seed=77)
    np.testing.assert_array_equal(np.load(out), oracle.forward(q, k, v, rpb, 5, nthreads=1))
