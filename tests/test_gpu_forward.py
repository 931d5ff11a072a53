"""Whole-layer and whole-stack parity of the CUDA path against the fp64 oracle through
whale_fusion_forward / whale_fusion_layer_forward / whale_fusion_forward_host: every example
of reduced copies of the workloads (ragged lengths, an empty history, every variant flag),
then the full-size workloads in the benchmark's launch configuration, checked on every example
and every token against the oracle run per example in a process pool. Also batch-reordering
invariance and the debug offset check."""
import json
import os

import numpy as np
import pytest
import torch

from oracle import whale_oracle as O
from tests.gpu_util import BF16_TOL, assert_parity
from wukong_hstu_cross_b200 import inputs as I

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from wukong_hstu_cross_b200 import build
    build.build()
    from wukong_hstu_cross_b200 import harness as Hn
    from wukong_hstu_cross_b200 import whale as W


def _oracle_all(p, examples=None, token_idx=None):
    w = p.w
    flags = p.flags
    res = {}
    for b in (range(w.batch) if examples is None else examples):
        x = I.tokens_of_example(w, b)
        if token_idx is not None:
            x = x[token_idx]
        res[b] = O.fusion_stack_example(x, Hn.states_of_example_host(p, b), p.host_weights, w.n_heads, w.eps, **flags)
    return res


def _check(p, out, examples=None, token_idx=None, rms_rel=2e-2):
    ref = _oracle_all(p, examples, token_idx)
    o = out.float().cpu().numpy()
    for b, r in ref.items():
        g = o[b] if token_idx is None else o[b][token_idx]
        assert_parity(g, r, p.w.dtype, rms_rel=rms_rel if p.w.dtype == "bf16" else None, what=f"example {b}")


REDUCED = {
    "tiny_fp32": dict(),
    "tiny_as_bf16": dict(dtype="bf16"),
    "stack_d128": dict(batch=6, lengths=("uniform", 1, 700)),
    "stack_d256": dict(batch=4, lengths=("uniform", 100, 1500)),
    "hist15k_d512": dict(batch=3, n_layers=2, lengths=("lognormal", 1500.0, 0.5, 64, 3000)),
    "serve_15k": dict(n_tokens=16 * 64, n_layers=2, lengths=("fixed", 3000)),
}


@pytest.mark.parametrize("name", list(REDUCED))
def test_stack_reduced_workloads(name):
    base = "tiny_fp32" if name.startswith("tiny") else name
    w = I.WORKLOADS[base].replace(**REDUCED[name])
    L = I.draw_lengths(w)
    if name == "stack_d128":
        L[2] = 0  # an empty history inside the batch
    p = Hn.build_problem(w, gains="random", lengths=L)
    out = Hn.run_forward(p)
    torch.cuda.synchronize()
    if name == "serve_15k":
        idx = np.random.default_rng(0).choice(w.n_tokens, 64, replace=False)
        _check(p, out, token_idx=idx)
    else:
        _check(p, out)


@pytest.mark.parametrize("shared_kv,tied_gate,fusion_mult", [(True, False, 2), (False, True, 2), (True, True, 0),
                                                              (False, False, 0)])
def test_variants(shared_kv, tied_gate, fusion_mult):
    w = I.WORKLOADS["stack_d256"].replace(batch=3, n_layers=2, lengths=("uniform", 1, 900), fusion_mult=fusion_mult)
    p = Hn.build_problem(w, gains="random", shared_kv=shared_kv, tied_gate=tied_gate)
    out = Hn.run_forward(p)
    torch.cuda.synchronize()
    _check(p, out)


def test_fp32_variants():
    w = I.WORKLOADS["tiny_fp32"].replace(batch=3, n_layers=2, fusion_mult=0)
    p = Hn.build_problem(w, gains="random", shared_kv=True, tied_gate=True)
    out = Hn.run_forward(p)
    torch.cuda.synchronize()
    _check(p, out)


def test_layer_entry_point_and_batch_reordering():
    w = I.WORKLOADS["stack_d128"].replace(batch=5, n_layers=1, lengths=("uniform", 1, 800))
    p = Hn.build_problem(w, gains="random")
    y = torch.empty_like(p.tokens)
    W.whale_fusion_layer_forward(p.cfg, p.tokens, p.states[0], p.offsets_t, p.weights[0], y, p.hint, p.workspace)
    out = Hn.run_forward(p)
    torch.cuda.synchronize()
    assert torch.equal(y, out)
    _check(p, y)
    # reorder the examples (same total and max length): each example's output follows it. The
    # attention's load-balanced split points depend on where an example sits in the batch, so the
    # order of the fp32 partial merges (not the result) may change: compare within 1e-2*(1+|y|).
    perm = np.array([3, 0, 4, 2, 1])
    L2 = p.lengths[perm]
    off2 = I.offsets_of(L2)
    rows = [p.states[0, p.offsets[b]:p.offsets[b + 1]] for b in perm]
    states2 = torch.cat(rows).unsqueeze(0).contiguous()
    tok2 = p.tokens[torch.from_numpy(perm).cuda()].contiguous()
    y2 = torch.empty_like(tok2)
    W.whale_fusion_forward(p.cfg, tok2, states2, torch.from_numpy(off2).cuda(), p.weights, y2, p.hint, p.workspace)
    torch.cuda.synchronize()
    ref = out[torch.from_numpy(perm).cuda()].float()
    assert bool(((y2.float() - ref).abs() <= 1e-2 * (1 + ref.abs())).all())


def test_prepared_weights_match_per_call_fold():
    w = I.WORKLOADS["stack_d256"].replace(batch=3, n_layers=2, lengths=("uniform", 1, 900))
    for tied in (False, True):
        p = Hn.build_problem(w, gains="random", tied_gate=tied)
        ref = Hn.run_forward(p).clone()
        buf = torch.empty(W.whale_prepared_weights_size(p.cfg), dtype=torch.uint8, device="cuda")
        pw = W.whale_prepare_weights(p.cfg, p.weights, buf)
        cfg = W.make_config(p.cfg.n_layers, p.cfg.d, p.cfg.n_heads, p.cfg.n_tokens, p.cfg.ffn_hidden,
                            p.cfg.fusion_hidden, p.cfg.dtype, p.cfg.flags | W.WHALE_PREPARED_WEIGHTS, p.cfg.eps)
        out = torch.empty_like(p.out)
        W.whale_fusion_forward(cfg, p.tokens, p.states, p.offsets_t, pw, out, p.hint, p.workspace)
        torch.cuda.synchronize()
        assert torch.equal(out, ref)


def test_prepared_weights_outlive_the_raw_weight_list():
    """Prepared weights point into the caller's raw w_f1, w_f2, w_down and gains: once the problem's
    weight list is replaced by the prepared array, those tensors must stay alive. Repeated forwards
    with allocations and a cache flush in between give bitwise the same output (a dangling pointer
    here once made later forwards read freed memory)."""
    w = I.WORKLOADS["stack_d128"].replace(batch=4, n_layers=2, lengths=("uniform", 1, 400))
    p = Hn.build_problem(w, gains="random")
    Hn.prepare_weights(p)
    ref = Hn.run_forward(p).clone()
    torch.cuda.synchronize()
    _check(p, ref)
    for _ in range(3):
        junk = [torch.full((1 << 20,), 7.0, device="cuda") for _ in range(8)]  # reuse freed memory, if any
        del junk
        torch.cuda.empty_cache()
        out = Hn.run_forward(p)
        torch.cuda.synchronize()
        assert torch.equal(out, ref)


def test_cuda_graph_replay_matches_stream_launches():
    """One forward of the absorbed 15k-history path (prepared weights) captured in a CUDA graph: the
    programmatic-dependent launches become graph edges; replays give bitwise the stream result."""
    w = I.WORKLOADS["hist15k_d512"].replace(**REDUCED["hist15k_d512"])
    p = Hn.build_problem(w, gains="random")
    Hn.prepare_weights(p)
    st = torch.cuda.Stream()
    with torch.cuda.stream(st):
        for _ in range(2):
            Hn.run_forward(p, st)
    torch.cuda.synchronize()
    ref = p.out.clone()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=st):
        Hn.run_forward(p, st)
    torch.cuda.synchronize()
    for _ in range(3):
        p.out.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(p.out, ref)
    del g
    _check(p, ref)


def test_host_buffer_entry_point_matches_device_entry_point():
    w = I.WORKLOADS["stack_d256"].replace(batch=4, n_layers=3, lengths=("uniform", 10, 1200))
    p = Hn.build_problem(w, gains="random")
    out = Hn.run_forward(p).clone()
    hs = p.states.cpu().pin_memory()
    ht = p.tokens.cpu().pin_memory()
    ho = torch.empty_like(ht).pin_memory()
    hoff = torch.from_numpy(p.offsets).pin_memory()
    ws = torch.empty(W.whale_host_workspace_size(p.cfg, p.hint), dtype=torch.uint8, device="cuda")
    for _ in range(2):
        ho.zero_()
        W.whale_fusion_forward_host(p.cfg, ht, hs, hoff, p.weights, ho, p.hint, ws)
        torch.cuda.synchronize()
        assert torch.equal(ho, out.cpu())


def test_debug_mode_flags_bad_offsets():
    w = I.WORKLOADS["stack_d128"].replace(batch=3, n_layers=1, lengths=("uniform", 10, 50))
    p = Hn.build_problem(w, debug=True)
    Hn.run_forward(p)
    assert W.whale_get_device_error() == 0
    bad = torch.tensor([0, 40, 20, int(p.offsets[-1])], dtype=torch.int32, device="cuda")  # decreasing: invalid
    W.whale_fusion_forward(p.cfg, p.tokens, p.states, bad, p.weights, p.out, p.hint, p.workspace)
    assert W.whale_get_device_error() & W.WHALE_DEVERR_OFFSETS
    assert W.whale_get_device_error() == 0  # cleared by the read


# ------------------------------------------------------------------------------------------
# full-size workloads, as the benchmark launches them: every example, every token
# ------------------------------------------------------------------------------------------
def _report(entry):
    """Append one config's worst error to the JSON-lines file named by WHALE_PARITY_REPORT (if set)."""
    path = os.environ.get("WHALE_PARITY_REPORT")
    if path:
        with open(path, "a") as fh:
            fh.write(json.dumps(entry) + "\n")


@pytest.mark.parametrize("gains", ["ones", "random"])
@pytest.mark.parametrize("name", ["stack_d128", "stack_d256", "hist15k_d512", "serve_15k"])
def test_full_size_every_example(name, gains):
    """The full-size workloads in the benchmark's launch configuration (weights prepared once, gains
    folded in) against the fp64 oracle on every output element: all B examples x all N tokens (all
    16 384 candidate tokens of the serving request), with the workload's gains (ones) and with random
    gains. The oracle runs per example in a process pool."""
    from tests import oracle_pool
    w = I.WORKLOADS[name]
    p = Hn.build_problem(w, gains=gains)
    Hn.prepare_weights(p)
    out = Hn.run_forward(p)
    torch.cuda.synchronize()
    o = out.float().cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(o))
    worst, checked = 0.0, 0
    chunk = 1024 if w.candidates else None
    for b, t0, ref in oracle_pool.oracle_outputs(name, p.lengths, gains=gains, token_chunk=chunk):
        g = o[b, t0:t0 + ref.shape[0]]
        err = np.abs(g - ref)
        worst = max(worst, float((err / (BF16_TOL * (1.0 + np.abs(ref)))).max()))
        checked += ref.size
        assert_parity(g, ref, "bf16", what=f"{name} gains={gains} example {b} tokens {t0}..")
    assert checked == o.size
    _report({"workload": name, "gains": gains, "elements": checked, "max_err_over_bound": worst,
             "bound": "2e-2*(1+|oracle|)", "weights": "prepared (whale_prepare_weights)"})
    # determinism: two more runs give bitwise the same output
    out2 = Hn.run_forward(p).clone()
    torch.cuda.synchronize()
    out3 = Hn.run_forward(p)
    torch.cuda.synchronize()
    assert torch.equal(out2, out3)


def test_kernel_profile_records_every_launch():
    """whale_profile_begin/end (the benchmark's per-kernel timing): one profiled forward of a
    two-layer absorbed stack returns one record per launch, in launch order, each a kernel of this
    library with a positive CUDA-event duration; profiling off again afterwards."""
    w = I.WORKLOADS["hist15k_d512"].replace(**REDUCED["hist15k_d512"])
    p = Hn.build_problem(w, device="cuda:0")
    Hn.prepare_weights(p)
    Hn.run_forward(p)  # first use outside the profile
    torch.cuda.synchronize()
    W.whale_profile_begin()
    Hn.run_forward(p)
    torch.cuda.synchronize()
    recs = W.whale_profile_end()
    names = [n for n, _ in recs]
    assert len(recs) > 0 and all(ms > 0.0 for _, ms in recs)
    assert all("whale" in n for n in names), names[:5]
    # per layer: the absorbed passes run once each, in order
    a = [i for i, n in enumerate(names) if "abs_scores_kernel" in n]
    b = [i for i, n in enumerate(names) if "abs_values_kernel" in n]
    assert len(a) == len(b) == w.n_layers and all(x < y for x, y in zip(a, b))
    # nothing is recorded once profiling has ended
    Hn.run_forward(p)
    torch.cuda.synchronize()
    W.whale_profile_begin()
    assert W.whale_profile_end() == []
