"""Host-side checks of the seeded input generators (CPU only)."""
import numpy as np

from wukong_hstu_cross_b200 import inputs as I


def test_bf16_rounding_is_round_to_nearest_even():
    one = np.float32(1.0)
    ulp = np.float32(2.0 ** -7)          # bf16 spacing at 1.0
    cases = {
        float(one + ulp / 2): 1.0,            # tie -> even (1.0)
        float(one + 3 * ulp / 2): float(one + 2 * ulp),   # tie -> even (1 + 2 ulp)
        float(one + ulp / 2 + 2 ** -20): float(one + ulp),   # above the tie -> up
        -2.5: -2.5, 0.0: 0.0,
    }
    for x, want in cases.items():
        assert I.bf16_round(np.array([x], np.float32))[0] == np.float32(want), x
    x = np.random.default_rng(0).standard_normal(10000).astype(np.float32)
    r = I.bf16_round(x)
    assert np.all(I.bf16_round(r) == r)
    assert np.max(np.abs(r - x) / np.abs(x)) <= 2.0 ** -8
    np.testing.assert_array_equal(I.from_bf16_bits(I.bf16_bits(x)), r)


def test_lengths_follow_their_distributions_and_are_deterministic():
    for name in I.ORDER:
        w = I.WORKLOADS[name]
        L = I.draw_lengths(w)
        assert len(L) == w.batch
        np.testing.assert_array_equal(L, I.draw_lengths(w))
        kind = w.lengths[0]
        if kind == "uniform":
            assert L.min() >= w.lengths[1] and L.max() <= w.lengths[2]
        elif kind == "lognormal":
            assert L.min() >= w.lengths[3] and L.max() <= w.lengths[4]
        else:
            assert np.all(L == w.lengths[1])
    hist = I.draw_lengths(I.WORKLOADS["hist15k_d512"])
    assert 4500 < np.median(hist) < 8000


def test_slices_regenerate_alone():
    w = I.small_workload("stack_d128", batch=3, d=32, n_heads=2, lengths=("uniform", 2, 9))
    L = I.draw_lengths(w)
    off = I.offsets_of(L)
    slab = I.make_states_layer(w, 1, L, threads=2)
    for b in range(3):
        np.testing.assert_array_equal(slab[off[b]:off[b + 1]], I.states_of_example(w, 1, b, L[b]))
    bits = I.make_states_layer(w, 1, L, threads=1, as_bits=True)
    np.testing.assert_array_equal(I.from_bf16_bits(bits), slab)
    lw = I.make_layer_weights(w, 0)
    assert lw["w_kv"].shape == (2 * w.d, w.d) and lw["w_upgate"].shape == (2 * w.ffn_hidden, w.d)
    assert lw["w_f1"].shape == (w.fusion_hidden, 2 * w.d) and lw["w_f2"].shape == (w.d, w.fusion_hidden)
    a = np.sqrt(6.0 / (w.d + w.d))
    assert np.abs(lw["w_q"]).max() <= a * (1 + 2.0 ** -8)   # bf16 rounding may step one ulp out
