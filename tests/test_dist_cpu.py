"""Multi-rank plumbing on CPU: two gloo ranks (world_size 2) shard the examples of a workload
with no data exchange, keep the weights replicated, and reduce the per-rank device time with a
max, exactly as bench.py does under torchrun on GPUs."""
import os
import socket

import numpy as np
import torch.multiprocessing as mp

from wukong_hstu_cross_b200 import dist as D
from wukong_hstu_cross_b200 import inputs as I


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    r, wsz, lr = D.rank_env()
    w = D.shard_workload(I.WORKLOADS["stack_d128"].replace(batch=4), r, wsz)
    lengths = I.draw_lengths(w)
    tok0 = I.tokens_of_example(w, 0)
    wq = I.make_layer_weights(w, 0)["w_q"]
    t = D.max_over_ranks(10.0 + rank, wsz)
    # gather what each rank holds (test-side only) to check disjointness / replication
    objs = [None] * wsz
    dist.all_gather_object(objs, (lengths.tolist(), float(tok0.sum()), float(wq.sum()), t))
    if rank == 0:
        out.put(objs)
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_shard_examples_and_reduce_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (len0, tok0, wq0, t0), (len1, tok1, wq1, t1) = res
    assert t0 == t1 == 11.0                       # max over ranks
    assert wq0 == wq1                             # weights replicated
    assert tok0 != tok1 and len0 != len1          # each rank its own examples
    # rank 0 of an N-rank run processes the single-GPU batch
    w = I.WORKLOADS["stack_d128"].replace(batch=4)
    assert len0 == I.draw_lengths(w).tolist()
    assert np.isclose(tok0, float(I.tokens_of_example(w, 0).sum()))


def test_single_process_defaults():
    w = I.WORKLOADS["stack_d128"]
    assert D.shard_workload(w, 0, 1) is w
    assert D.max_over_ranks(3.5, 1) == 3.5
