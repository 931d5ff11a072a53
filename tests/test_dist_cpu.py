"""Multi-rank plumbing on CPU: two gloo ranks (world_size 2) shard the examples of a workload
with no data exchange, keep the weights replicated, and reduce the per-rank device time with a
max, exactly as bench.py does under torchrun on GPUs. One batch split across the ranks by
history rows (shard_batch) and run through the oracle on each rank gives, gathered, bitwise the
unsharded result."""
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


def _shard_worker(rank, world, port, out):
    import torch.distributed as dist
    from oracle import whale_oracle as O
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    w = I.WORKLOADS["stack_d128"].replace(batch=7, n_layers=2, lengths=("uniform", 1, 120))
    L = I.draw_lengths(w)
    L[3] = 0
    off = I.offsets_of(L)
    tokens = I.make_tokens(w)
    states = np.stack([I.make_states_layer(w, l, L, threads=1) for l in range(w.n_layers)])
    lws = I.make_all_weights(w, gains="random")
    tok_r, st_r, off_r, (b0, b1) = D.shard_batch(tokens, states, off, rank, world)
    y = O.fusion_stack(tok_r, st_r, off_r, lws, w.n_heads, w.eps) if b1 > b0 else np.zeros((0, w.n_tokens, w.d))
    objs = [None] * world
    dist.all_gather_object(objs, (b0, b1, int(st_r.shape[1]), y))
    if rank == 0:
        full = O.fusion_stack(tokens, states, off, lws, w.n_heads, w.eps)
        out.put((objs, full, L.tolist()))
    dist.barrier()
    dist.destroy_process_group()


def test_one_batch_sharded_by_history_rows_equals_unsharded():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    objs, full, L = q.get(timeout=180)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (a0, a1, rows0, y0), (c0, c1, rows1, y1) = objs
    assert (a0, a1, c1) == (0, c0, len(L))                 # contiguous, covering the batch
    assert rows0 + rows1 == sum(L) and abs(rows0 - rows1) <= max(L)   # balanced within one example
    assert np.array_equal(np.concatenate([y0, y1]), full)  # bitwise the unsharded oracle


def test_balanced_ranges_edge_cases():
    assert D.balanced_ranges([5, 5, 5, 5], 2) == [(0, 2), (2, 4)]
    assert D.balanced_ranges([100, 1, 1, 1], 2) == [(0, 1), (1, 4)]
    assert D.balanced_ranges([3], 4) == [(0, 0), (0, 1), (1, 1), (1, 1)] or \
        sum(b - a for a, b in D.balanced_ranges([3], 4)) == 1
    assert D.balanced_ranges([], 2) == [(0, 0), (0, 0)]
    assert D.balanced_ranges([0, 0, 7, 0], 1) == [(0, 4)]
    # every example lands in exactly one range, ranges in order
    rng = np.random.default_rng(0)
    for world in (2, 3, 8):
        L = rng.integers(0, 5000, size=37)
        rr = D.balanced_ranges(L, world)
        assert rr[0][0] == 0 and rr[-1][1] == 37 and all(rr[k][1] == rr[k + 1][0] for k in range(world - 1))
        loads = [int(L[a:b].sum()) for a, b in rr]
        assert max(loads) - min(loads) <= 2 * int(L.max())


def _cand_worker(rank, world, port, out):
    import torch.distributed as dist
    from oracle import whale_oracle as O
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    # a reduced serving request: one shared history, 7 candidates x 4 tokens (7 does not divide by 2)
    w = I.WORKLOADS["serve_15k"].replace(n_tokens=7 * 4, candidates=7, d=64, n_heads=2, n_layers=2,
                                         lengths=("fixed", 150))
    L = I.draw_lengths(w)
    off = I.offsets_of(L)
    tokens = I.make_tokens(w)
    states = np.stack([I.make_states_layer(w, l, L, threads=1) for l in range(w.n_layers)])
    lws = I.make_all_weights(w, gains="random")
    tok_r, (c0, c1) = D.shard_candidates(tokens, 4, rank, world)
    y = O.fusion_stack(tok_r, states, off, lws, w.n_heads, w.eps)     # the history replicated
    objs = [None] * world
    dist.all_gather_object(objs, (c0, c1, y))
    if rank == 0:
        out.put((objs, O.fusion_stack(tokens, states, off, lws, w.n_heads, w.eps)))
    dist.barrier()
    dist.destroy_process_group()


def test_serving_request_sharded_by_candidates_equals_unsharded():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_cand_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    objs, full = q.get(timeout=180)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (a0, a1, y0), (c0, c1, y1) = objs
    assert (a0, a1, c0, c1) == (0, 4, 4, 7)
    got = np.concatenate([y0, y1], axis=1)
    assert got.shape == full.shape
    # each token's result depends on its own row and the shared history only; the fp64 products of
    # fewer rows may be blocked differently by BLAS, so agreement is to fp64 rounding, not bitwise
    assert np.allclose(got, full, rtol=1e-12, atol=1e-12), float(np.abs(got - full).max())


def test_candidate_ranges():
    assert [D.candidate_range(1024, r, 8) for r in (0, 7)] == [(0, 128), (896, 1024)]
    assert [D.candidate_range(7, r, 3) for r in range(3)] == [(0, 3), (3, 5), (5, 7)]
    assert [D.candidate_range(2, r, 4) for r in range(4)] == [(0, 1), (1, 2), (2, 2), (2, 2)]
    x = np.zeros((1, 12, 3))
    assert D.shard_candidates(x, 4, 1, 2)[0].shape == (1, 4, 3)
    try:
        D.shard_candidates(x, 5, 0, 2)
        raise AssertionError("12 tokens are not whole candidates of 5")
    except ValueError:
        pass
