"""Parity of the absorbed cross-attention path (K and V folded into the queries) against the fp64
oracle, through whale_fusion_forward: ragged lengths around the 256-row unit (1, 255, 256, 257,
513), empty histories, batches whose examples are split across CTA pairs and pairs holding many
short examples, histories whose later rows raise pass A's softmax reference (so pass B rescales
its accumulator), both widths the path takes (d = 512 with 8 heads, d = 256 with 4 heads), shared
K = V, prepared weights and agreement with the materialising path."""
import numpy as np
import pytest
import torch

from oracle import whale_oracle as O
from tests.gpu_util import assert_parity
from wukong_hstu_cross_b200 import inputs as I

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from wukong_hstu_cross_b200 import build
    build.build()
    from wukong_hstu_cross_b200 import harness as Hn
    from wukong_hstu_cross_b200 import whale as W


def _workload(d, batch, n_layers=1, fusion_mult=2):
    if d == 512:
        return I.WORKLOADS["hist15k_d512"].replace(batch=batch, n_layers=n_layers, fusion_mult=fusion_mult)
    # d = 256 with d_head = 64: 4 heads, 64 tokens -> 256 absorbed queries
    return I.WORKLOADS["stack_d256"].replace(batch=batch, n_layers=n_layers, n_heads=4, n_tokens=64,
                                             fusion_mult=fusion_mult)


def _oracle_check(p, out, examples=None):
    o = out.float().cpu().numpy()
    for b in (range(p.w.batch) if examples is None else examples):
        ref = O.fusion_stack_example(I.tokens_of_example(p.w, b), Hn.states_of_example_host(p, b), p.host_weights,
                                     p.w.n_heads, p.w.eps, **p.flags)
        assert_parity(o[b], ref, "bf16", rms_rel=2e-2, what=f"example {b}")


def _with_flags(p, extra):
    cfg = W.make_config(p.cfg.n_layers, p.cfg.d, p.cfg.n_heads, p.cfg.n_tokens, p.cfg.ffn_hidden,
                        p.cfg.fusion_hidden, p.cfg.dtype, p.cfg.flags | extra, p.cfg.eps)
    ws = torch.empty(W.whale_workspace_size(cfg, p.hint), dtype=torch.uint8, device="cuda")
    return cfg, ws


def _scale_query_gain(p, factor):
    """Multiply g_q of every layer (device and oracle copies): larger score ranges."""
    for l in range(p.w.n_layers):
        p.weights[l]["g_q"].mul_(factor)
        p.host_weights[l]["g_q"] = p.host_weights[l]["g_q"] * np.float32(factor)


@pytest.mark.parametrize("d", [512, 256])
def test_absorbed_ragged_units(d):
    L = np.array([1, 255, 256, 257, 0, 513, 1800, 40])
    w = _workload(d, len(L))
    p = Hn.build_problem(w, gains="random", lengths=L)
    out = Hn.run_forward(p)
    torch.cuda.synchronize()
    _oracle_check(p, out)


def test_absorbed_two_layers_many_pairs():
    # 40 short and long histories: ranges cut inside examples and ranges holding several examples
    w = _workload(512, 40, n_layers=2).replace(lengths=("uniform", 1, 2500))
    L = I.draw_lengths(w)
    L[7] = 0
    p = Hn.build_problem(w, gains="random", lengths=L)
    out = Hn.run_forward(p)
    torch.cuda.synchronize()
    _oracle_check(p, out, examples=[0, 7, 13, 21, 39])


@pytest.mark.parametrize("d", [512, 256])
def test_absorbed_reference_raised_mid_history(d):
    # The first 256 rows of every history repeat one row, so the first unit's tile maximum is a
    # single score; with query gains x2 (log2-scores of spread ~4) the maximum over the later
    # random rows exceeds it by more than the lazy headroom for most queries: pass A raises its
    # reference mid-history and pass B rescales its accumulator.
    L = np.array([3000, 2100, 700])
    w = _workload(d, len(L))
    p = Hn.build_problem(w, gains="random", lengths=L)
    _scale_query_gain(p, 2.0)
    states = []
    for b in range(len(L)):
        per_layer = Hn.states_of_example_host(p, b)
        for l, h in enumerate(per_layer):
            h[:256] = h[0]
            rows = torch.from_numpy(I.bf16_bits(h[:256]).view(np.int16)).view(torch.bfloat16)
            p.states[l, int(p.offsets[b]):int(p.offsets[b]) + 256].copy_(rows.cuda())
        states.append(per_layer)
    out = Hn.run_forward(p)
    torch.cuda.synchronize()
    o = out.float().cpu().numpy()
    for b in range(len(L)):
        ref = O.fusion_stack_example(I.tokens_of_example(p.w, b), states[b], p.host_weights, p.w.n_heads, p.w.eps,
                                     **p.flags)
        assert_parity(o[b], ref, "bf16", rms_rel=2e-2, what=f"example {b}")


@pytest.mark.parametrize("shared_kv,tied_gate", [(True, False), (True, True)])
def test_absorbed_variants(shared_kv, tied_gate):
    w = _workload(512, 3, n_layers=2).replace(lengths=("uniform", 100, 1200))
    p = Hn.build_problem(w, gains="random", shared_kv=shared_kv, tied_gate=tied_gate)
    out = Hn.run_forward(p)
    torch.cuda.synchronize()
    _oracle_check(p, out)


def test_absorbed_matches_materialized_path():
    w = _workload(512, 4, n_layers=2).replace(lengths=("uniform", 300, 2000))
    p = Hn.build_problem(w, gains="random")
    out = Hn.run_forward(p).clone()
    cfg, ws = _with_flags(p, W.WHALE_MATERIALIZED_KV)
    out_m = torch.empty_like(p.out)
    W.whale_fusion_forward(cfg, p.tokens, p.states, p.offsets_t, p.weights, out_m, p.hint, ws)
    torch.cuda.synchronize()
    _oracle_check(p, out)
    _oracle_check(p, out_m)
    a, b = out.float(), out_m.float()
    assert bool(((a - b).abs() <= 2e-2 * (1 + b.abs())).all())


def test_absorbed_prepared_weights():
    w = _workload(512, 3, n_layers=2).replace(lengths=("uniform", 1, 900))
    p = Hn.build_problem(w, gains="random")
    ref = Hn.run_forward(p).clone()
    buf = torch.empty(W.whale_prepared_weights_size(p.cfg), dtype=torch.uint8, device="cuda")
    pw = W.whale_prepare_weights(p.cfg, p.weights, buf)
    assert all(pw[l].w_kabs for l in range(w.n_layers))
    cfg, _ = _with_flags(p, W.WHALE_PREPARED_WEIGHTS)
    out = torch.empty_like(p.out)
    W.whale_fusion_forward(cfg, p.tokens, p.states, p.offsets_t, pw, out, p.hint, p.workspace)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)  # same folds from the same inputs
    # prepared weights without the absorbed keys: formed per call from the folded W_K
    for l in range(w.n_layers):
        pw[l].w_kabs = None
    out2 = torch.empty_like(p.out)
    W.whale_fusion_forward(cfg, p.tokens, p.states, p.offsets_t, pw, out2, p.hint, p.workspace)
    torch.cuda.synchronize()
    _oracle_check(p, out2)


def test_absorbed_deterministic_and_all_empty():
    w = _workload(256, 5).replace(lengths=("uniform", 1, 1500))
    p = Hn.build_problem(w, gains="random")
    a = Hn.run_forward(p).clone()
    b = Hn.run_forward(p).clone()
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    # every history empty: A = 0 for every query
    L0 = np.zeros(3, dtype=np.int64)
    p0 = Hn.build_problem(_workload(512, 3), gains="random", lengths=L0)
    out0 = Hn.run_forward(p0)
    torch.cuda.synchronize()
    _oracle_check(p0, out0)


def _states_host(p, b):
    """Per-layer history rows of example b as they sit on the device (bf16 values, exact in fp64)."""
    o0, o1 = int(p.offsets[b]), int(p.offsets[b + 1])
    return [p.states[l, o0:o1].float().cpu().numpy() for l in range(p.w.n_layers)]


def test_absorbed_long_history_of_identical_rows():
    """A 15 000-row history whose rows are all equal (every score ties: the softmax is an average
    over 59 units split across CTA pairs, each unit's weights exactly 1), next to a one-row and a
    4 000-row copy-of-one-row history; checked against the oracle on the device's states."""
    w = _workload(512, 3)
    p = Hn.build_problem(w, lengths=np.array([15000, 1, 4000]), gains="random")
    for b in (0, 2):
        o0, o1 = int(p.offsets[b]), int(p.offsets[b + 1])
        p.states[:, o0:o1] = p.states[:, o0:o0 + 1]
    Hn.prepare_weights(p)
    out = Hn.run_forward(p)
    torch.cuda.synchronize()
    o = out.float().cpu().numpy()
    for b in range(3):
        ref = O.fusion_stack_example(I.tokens_of_example(w, b), _states_host(p, b), p.host_weights, w.n_heads,
                                     w.eps, **p.flags)
        assert_parity(o[b], ref, "bf16", rms_rel=2e-2, what=f"example {b}")


def test_absorbed_history_permutation_invariance_full_lengths():
    """Permuting the rows of every example's history (the same permutation in every layer) leaves
    the output unchanged up to summation order, at the 15k workload's length mix: the scores move
    across units, CTA pairs and partial segments."""
    w = _workload(512, 8, n_layers=2)
    p = Hn.build_problem(w)
    Hn.prepare_weights(p)
    out1 = Hn.run_forward(p).clone()
    rng = np.random.default_rng(11)
    for b in range(w.batch):
        o0, o1 = int(p.offsets[b]), int(p.offsets[b + 1])
        perm = torch.from_numpy(rng.permutation(o1 - o0) + o0).to(p.states.device)
        p.states[:, o0:o1] = p.states[:, perm]
    out2 = Hn.run_forward(p)
    torch.cuda.synchronize()
    assert_parity(out2.float().cpu().numpy(), out1.float().cpu().numpy().astype(np.float64), "bf16", rms_rel=2e-2,
                  what="permuted history")
