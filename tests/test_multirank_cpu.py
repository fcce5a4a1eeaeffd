"""The multi-process path of bench.py on CPU: two gloo ranks share rank 0's seeded inputs through
/dev/shm and agree on the max-over-ranks step time.  No GPU is involved."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import torch.distributed as dist
    from datetime import timedelta

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    import bench
    from block_sparse_attention_blocks_b200 import workloads as W

    w = W.get("pr1_1k")
    q, k, v = bench.make_inputs(w, rank, world)
    digest = float(np.asarray(q, np.float64).sum() + 3 * np.asarray(v, np.float64).sum())
    t = bench.max_over_ranks(10.0 + rank)
    out[rank] = (digest, t)
    dist.barrier()
    dist.destroy_process_group()


def test_two_ranks_share_inputs_and_max_time():
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as man:  # no fork of this threaded process
        out = man.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    from block_sparse_attention_blocks_b200 import workloads as W

    q, k, v = W.make_qkv(W.get("pr1_1k"))
    want = float(np.asarray(q, np.float64).sum() + 3 * np.asarray(v, np.float64).sum())
    assert res[0][0] == want and res[1][0] == want
    assert res[0][1] == res[1][1] == 11.0
