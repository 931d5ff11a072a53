"""The fp64 oracle over whole examples of a seeded workload, in a pool of worker processes.

Test infrastructure: each worker regenerates its example's inputs from the workload's seeds
(wukong_hstu_cross_b200.inputs) and runs oracle.whale_oracle.fusion_stack_example on them, so the
full-size workloads can be checked example by example in seconds. Workers are started with `spawn`
(the parent process holds a CUDA context: a forked worker would hang), each with one BLAS thread.
"""
from __future__ import annotations

import multiprocessing as mp
import os
from concurrent.futures import ProcessPoolExecutor

_WEIGHTS = {}


def _setup(key):
    from wukong_hstu_cross_b200 import inputs as I
    if key not in _WEIGHTS:
        name, overrides, gains, shared_kv, tied_gate = key
        w = I.WORKLOADS[name].replace(**dict(overrides))
        _WEIGHTS[key] = (w, I.make_all_weights(w, gains=gains, shared_kv=shared_kv, tied_gate=tied_gate))
    return _WEIGHTS[key]


def _one(task):
    from oracle import whale_oracle as O
    from wukong_hstu_cross_b200 import inputs as I
    key, b, length, t0, t1 = task
    w, lws = _setup(key)
    x = I.tokens_of_example(w, b)[t0:t1]
    slabs = [I.states_of_example(w, l, b, length) for l in range(w.n_layers)]
    _, _, _, shared_kv, tied_gate = key
    return b, t0, O.fusion_stack_example(x, slabs, lws, w.n_heads, w.eps, shared_kv=shared_kv, tied_gate=tied_gate)


def workers() -> int:
    return max(1, min(32, len(os.sched_getaffinity(0))))


def oracle_outputs(name, lengths, gains="ones", overrides=(), shared_kv=False, tied_gate=False, token_chunk=None):
    """Oracle output of every token of every example: yields (b, first token, [tokens, d] float64).
    token_chunk splits each example's tokens into independent tasks (tokens of one example do not
    interact given its history), for the many-candidate serving workload."""
    from wukong_hstu_cross_b200 import inputs as I
    key = (name, tuple(sorted(dict(overrides).items())), gains, shared_kv, tied_gate)
    w = I.WORKLOADS[name].replace(**dict(overrides))
    step = token_chunk or w.n_tokens
    tasks = [(key, b, int(lengths[b]), t0, min(w.n_tokens, t0 + step))
             for b in range(w.batch) for t0 in range(0, w.n_tokens, step)]
    # longest first: the pool ends with short tasks
    tasks.sort(key=lambda t: -t[2] * (t[4] - t[3]))
    env = {k: os.environ.get(k) for k in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS")}
    for k in env:
        os.environ[k] = "1"
    try:
        with ProcessPoolExecutor(workers(), mp_context=mp.get_context("spawn")) as ex:
            for res in ex.map(_one, tasks, chunksize=1):
                yield res
    finally:
        for k, v in env.items():
            if v is None:
                os.environ.pop(k, None)
            else:
                os.environ[k] = v


def _one_bwd(task):
    from oracle import whale_backward as OB
    from wukong_hstu_cross_b200 import inputs as I
    key, b, length, dy_b = task
    w, lws = _setup(key)
    _, _, _, shared_kv, tied_gate = key
    x = I.tokens_of_example(w, b)
    s = I.states_of_example(w, 0, b, length)
    dx, ds, dlw = OB.fusion_layer_backward(x, s, lws[0], w.n_heads, w.eps, dy_b, shared_kv=shared_kv,
                                           tied_gate=tied_gate)
    return b, dx, ds, dlw


def oracle_layer_backward(name, lengths, dy, gains="ones", overrides=(), shared_kv=False, tied_gate=False):
    """The fp64 VJP of layer 0 for every example (upstream gradient dy [B, N, d]): yields (b, d_tokens,
    d_states [L_b, d], {parameter: this example's share of its gradient})."""
    from wukong_hstu_cross_b200 import inputs as I
    key = (name, tuple(sorted(dict(overrides).items())), gains, shared_kv, tied_gate)
    w = I.WORKLOADS[name].replace(**dict(overrides))
    tasks = [(key, b, int(lengths[b]), dy[b]) for b in range(w.batch)]
    tasks.sort(key=lambda t: -t[2])  # longest first
    env = {k: os.environ.get(k) for k in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS")}
    for k in env:
        os.environ[k] = "1"
    try:
        with ProcessPoolExecutor(workers(), mp_context=mp.get_context("spawn")) as ex:
            for res in ex.map(_one_bwd, tasks, chunksize=1):
                yield res
    finally:
        for k, v in env.items():
            if v is None:
                os.environ.pop(k, None)
            else:
                os.environ[k] = v
