"""The benchmark's multi-rank host logic on CPU (gloo, world size 2): requests shard across
ranks with no data-path collective; only the timing reduction crosses ranks."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    from draft_tree_verification_masked_b200 import workload as W
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    # each rank draws its own batch (same shapes, different seeded requests)
    wl = W.generate("tiny", seed=W.config_seed("tiny") + 7919 * rank, B=2, hidden=64, vocab=64)
    step_s, e2e_s, tok = 0.5 + rank, 2.0 - rank, 10 * (rank + 1)
    res = bench.reduce_over_ranks(step_s, e2e_s, tok, world, "cpu")
    out[rank] = (res, int(wl.tokens.sum()))
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_reduction_is_max_time_and_summed_tokens():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world,
                       start_method="spawn", join=True)
    (r0, t0), (r1, t1) = out[0], out[1]
    assert r0 == r1 == (1.5, 2.0, 30.0)
    assert t0 != t1                    # the ranks verified different requests


def test_single_rank_passes_through():
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    assert bench.reduce_over_ranks(0.25, 0.5, 7, 1, "cpu") == (0.25, 0.5, 7.0)
