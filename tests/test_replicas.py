"""Multi-process (world size 2, gloo, CPU) tests of the replica host logic used by
bench.py for N > 1: batch sharing, per-rank seeds, the max-over-ranks time and the
whole-job throughput."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from vision_transformer_encoder_vit_b200 import replicas as R


def test_split_batch_covers_every_image_once():
    for gb in (0, 1, 7, 8, 9, 64):
        for world in (1, 2, 3, 8):
            seen = []
            for r in range(world):
                first, count = R.split_batch(gb, world, r)
                seen += list(range(first, first + count))
            assert seen == list(range(gb))
    with pytest.raises(ValueError):
        R.split_batch(8, 2, 2)


def test_throughput_and_seeds():
    assert R.job_throughput(8, 10, 200.0, 4) == pytest.approx(4 * 8 * 10 / 0.2)
    assert len({R.replica_seed(2, r) for r in range(8)}) == 8
    assert R.max_over_ranks(3.5) == 3.5  # no process group: identity


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        r, w, lr = R.rank_env()
        assert (r, w, lr) == (rank, world, rank)
        my_ms = 100.0 + 50.0 * rank          # rank 1 is slower
        m = R.max_over_ranks(my_ms)
        first, count = R.split_batch(16, world, rank)
        dist.barrier()
        out[rank] = (m, first, count, R.job_throughput(count, 5, m, world))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_max_time_and_shares():
    world = 2
    port = _free_port()
    manager = mp.get_context("spawn").Manager()
    out = manager.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    assert out[0][0] == out[1][0] == 150.0
    assert (out[0][1], out[0][2]) == (0, 8) and (out[1][1], out[1][2]) == (8, 8)
    assert out[0][3] == pytest.approx(2 * 8 * 5 / 0.15)
