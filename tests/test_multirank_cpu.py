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


def _split_worker(rank, world, port, out):
    import torch.distributed as dist
    from datetime import timedelta

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    import bench
    import oracle
    from block_sparse_attention_blocks_b200 import workloads as W

    w = W.get("stress_mixed")
    from dataclasses import replace

    w = replace(w, N=1024, grid=(4, 16, 16))  # small: 2 x 16 heads of 1024 tokens
    heads = bench.shard_heads(w.B * w.H, rank, world)
    q, k, v = W.make_qkv(w, heads=heads)
    o = _oracle_path(oracle, w, q[0], k[0], v[0])
    gathered = [None] * world
    dist.all_gather_object(gathered, (heads, o))
    if rank == 0:
        out["parts"] = gathered
    dist.barrier()
    dist.destroy_process_group()


def _oracle_path(oracle, w, q, k, v):
    """Pooling, hybrid selection and masked attention of every query block of heads [h, N, d]
    (the computation one rank performs on its slice), through the fp64 oracle."""
    import math

    BH, N, d = q.shape
    qp = oracle.pool_blocks(q, w.bs)
    kp = oracle.pool_blocks(k, w.bs)
    sel = oracle.select(qp, kp, w.topk, w.topp, 1 / math.sqrt(d))
    return oracle.masked_attention(q, k, v, sel.mask.reshape(BH, w.nb, w.nb), w.bs, 1 / math.sqrt(d))


def test_head_split_equals_one_rank():
    # The heads of one call split over two gloo ranks (contiguous slices, bench.shard_heads):
    # each rank generates only its heads and runs the path on them; the gathered slices, in rank
    # order, equal the single-process result over all heads.  This is the partition bench.py uses
    # with --split heads (untested on several GPUs here: the pool gives one GPU per call).
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as man:
        out = man.dict()
        mp.spawn(_split_worker, args=(world, port, out), nprocs=world, join=True)
        parts = out["parts"]
    import bench
    import oracle
    from dataclasses import replace
    from block_sparse_attention_blocks_b200 import workloads as W

    w = replace(W.get("stress_mixed"), N=1024, grid=(4, 16, 16))
    n = w.B * w.H
    assert [h for hs, _ in parts for h in hs] == list(range(n))
    assert all(len(hs) in (n // world, n // world + 1) for hs, _ in parts)
    q, k, v = W.make_qkv(w)
    full = _oracle_path(oracle, w, q.reshape(n, w.N, w.d), k.reshape(n, w.N, w.d),
                        v.reshape(n, w.N, w.d))
    split = np.concatenate([o for _, o in parts], axis=0)
    assert split.shape == full.shape
    assert np.array_equal(split, full)
    assert bench.shard_heads(5, 0, 2) == [0, 1] and bench.shard_heads(5, 1, 2) == [2, 3, 4]
