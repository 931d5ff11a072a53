"""The C-ABI library loads, exports every function include/whale_fusion.h declares, and its
host-side checks return the documented status codes. No GPU work: every call below
returns before any CUDA call is made."""
import ctypes

from wukong_hstu_cross_b200 import build

build.build()
from wukong_hstu_cross_b200 import whale as W  # noqa: E402
from wukong_hstu_cross_b200 import inputs as I  # noqa: E402
from wukong_hstu_cross_b200 import harness as Hn  # noqa: E402

EXPECTED = {
    "whale_status_string", "whale_workspace_size", "whale_fusion_forward", "whale_host_workspace_size",
    "whale_fusion_forward_host", "whale_fusion_layer_forward", "whale_project_queries", "whale_project_kv",
    "whale_cross_attention", "whale_fusion_mlp", "whale_swiglu_ffn", "whale_get_device_error",
    "whale_attend_states", "whale_prepare_weights", "whale_prepared_weights_size", "whale_cross_attention_noalloc",
    "whale_profile_begin", "whale_profile_end", "whale_test_bounded_waits", "whale_backward_workspace_size",
    "whale_fusion_layer_backward", "whale_fusion_backward",
}


def test_library_exports_every_declared_symbol():
    declared = set(W.header_functions())
    assert EXPECTED <= declared, EXPECTED - declared
    lib = ctypes.CDLL(W.LIB_PATH)
    for name in declared:
        assert hasattr(lib, name), name


def test_backward_workspace_size_and_supported_shapes():
    # the training workloads are supported; the many-candidate serving shape (N = 16384) is not
    for name in ("tiny_fp32", "stack_d128", "stack_d256", "hist15k_d512"):
        w, cfg = _cfg(name)
        assert W.whale_backward_workspace_size(cfg, W.make_hint(w.batch, 3000, w.batch * 3000)) > 0, name
    w, cfg = _cfg("serve_15k")
    assert W.whale_backward_workspace_size(cfg, W.make_hint(1, 15000, 15000)) == 0
    # prepared (gain-folded, re-packed) weights are not accepted: the backward needs the raw ones
    w, cfg = _cfg("stack_d128")
    prep = W.make_config(cfg.n_layers, cfg.d, cfg.n_heads, cfg.n_tokens, cfg.ffn_hidden, cfg.fusion_hidden, cfg.dtype,
                         cfg.flags | W.WHALE_PREPARED_WEIGHTS, cfg.eps)
    assert W.whale_backward_workspace_size(prep, W.make_hint(4, 100, 400)) == 0
    # the workspace grows with the history (K|V, its gradient, the states' gradient terms)
    small = W.whale_backward_workspace_size(cfg, W.make_hint(4, 100, 400))
    large = W.whale_backward_workspace_size(cfg, W.make_hint(4, 100, 40000))
    assert large - small >= (40000 - 400) * cfg.d * (2 * 2 + 2 * 2 + 4 + 2)


def test_stack_backward_keeps_each_layers_activations():
    # bf16: every layer past the first adds its own forward activations to the stack's workspace
    # (its K|V pair over the history above all: 4 bytes per K|V element), so that the stack runs each
    # layer's forward once; fp32 adds only the layer's input (it recomputes inside each layer)
    T, B = 40000, 4
    for name in ("stack_d128", "tiny_fp32"):
        _, cfg = _cfg(name)
        kvw = 2 * cfg.d
        sizes = []
        for nl in (1, 2, 3):
            c = W.make_config(nl, cfg.d, cfg.n_heads, cfg.n_tokens, cfg.ffn_hidden, cfg.fusion_hidden, cfg.dtype,
                              cfg.flags, cfg.eps)
            sizes.append(W.whale_backward_workspace_size(c, W.make_hint(B, T // B, T)))
        step = sizes[2] - sizes[1]
        assert step == sizes[1] - sizes[0], name  # the same for every added layer
        rows = B * cfg.n_tokens
        if cfg.dtype == W.WHALE_BF16:
            assert step >= T * kvw * 4 + rows * cfg.d * (4 + 2 + 2), name
        else:
            assert rows * cfg.d * 4 <= step < T * kvw * 4, name
    # the SwiGLU backward takes 8 hidden columns per thread: other hidden sizes are not supported
    w, cfg = _cfg("stack_d128")
    odd = W.make_config(cfg.n_layers, cfg.d, cfg.n_heads, cfg.n_tokens, cfg.ffn_hidden + 4, cfg.fusion_hidden,
                        W.WHALE_FP32, cfg.flags, cfg.eps)
    assert W.whale_backward_workspace_size(odd, W.make_hint(4, 100, 400)) == 0


def test_backward_host_side_errors():
    w, cfg = _cfg("stack_d128")
    hint = W.make_hint(2, 10, 20)
    fake = 1 << 20  # never dereferenced: every call below fails its checks first
    lw = dict.fromkeys(["g_q", "g_kv", "w_q", "w_kv", "w_f1", "w_f2", "g_ffn", "w_upgate", "w_down"], fake)
    gr = dict(lw)
    nbytes = W.whale_backward_workspace_size(cfg, hint)
    # workspace too small (for one layer, and for the stack)
    assert W.whale_fusion_layer_backward(cfg, fake, fake, fake, lw, fake, fake, fake, gr, hint, fake, 1024,
                                         stream=0, raw=True) == 4
    assert W.whale_fusion_backward(cfg, fake, fake, fake, [lw] * cfg.n_layers, fake, fake, fake, [gr] * cfg.n_layers,
                                   hint, fake, nbytes - 1, stream=0, raw=True) == 4
    # a missing gradient buffer
    bad = dict(gr, w_down=None)
    assert W.whale_fusion_layer_backward(cfg, fake, fake, fake, lw, fake, fake, fake, bad, hint, fake, nbytes,
                                         stream=0, raw=True) == 1
    # unsupported: more than 32 tokens per example in bf16
    w2, cfg2 = _cfg("stack_d128", n_tokens=64)
    assert W.whale_fusion_layer_backward(cfg2, fake, fake, fake, lw, fake, fake, fake, gr, hint, fake, 1 << 30,
                                         stream=0, raw=True) == 2


def test_bounded_wait_self_test_rejects_limits_out_of_range():
    # 1 us .. 2 s; out-of-range limits are refused on the host before any launch
    assert W.whale_test_bounded_waits(999, stream=0, raw=True) == 1
    assert W.whale_test_bounded_waits(2_000_000_001, stream=0, raw=True) == 1


def test_status_strings():
    for code in range(6):
        assert W.whale_status_string(code) and W.whale_status_string(code) != "unknown status"
    assert W.whale_status_string(99) == "unknown status"


def _cfg(name, **kw):
    w = I.WORKLOADS[name].replace(**kw) if kw else I.WORKLOADS[name]
    return w, Hn.config_of(w)


def test_workspace_size_scales_and_rejects_invalid():
    w, cfg = _cfg("stack_d256")
    small = W.whale_workspace_size(cfg, W.make_hint(4, 100, 400))
    large = W.whale_workspace_size(cfg, W.make_hint(128, 6000, 576000))
    assert 0 < small < large
    # K|V buffer alone (total_L x 2d bf16) must fit
    assert large > 576000 * 2 * w.d * 2
    bad = Hn.config_of(w.replace(n_heads=3))           # d % heads != 0
    assert W.whale_workspace_size(bad, W.make_hint(4, 100, 400)) == 0
    unsup = Hn.config_of(w.replace(d=96, n_heads=3))   # bf16 needs d % 64 == 0
    assert W.whale_workspace_size(unsup, W.make_hint(4, 100, 400)) == 0
    assert W.whale_workspace_size(cfg, W.make_hint(-1, 100, 400)) == 0


def test_host_side_errors_are_reported_without_gpu_work():
    w, cfg = _cfg("stack_d128")
    hint = W.make_hint(2, 10, 20)
    ws = W.whale_workspace_size(cfg, hint)
    fake = 1 << 20  # never dereferenced: every call below fails validation first
    wts = [dict.fromkeys(["g_q", "g_kv", "w_q", "w_kv", "w_f1", "w_f2", "g_ffn", "w_upgate", "w_down"], fake)] * 4
    # null tokens
    assert W.whale_fusion_forward(cfg, None, fake, fake, wts, fake, hint, fake, ws, stream=0, raw=True) == 1
    # workspace too small / null
    assert W.whale_fusion_forward(cfg, fake, fake, fake, wts, fake, hint, fake, ws - 1, stream=0, raw=True) == 4
    assert W.whale_fusion_forward(cfg, fake, fake, fake, wts, fake, hint, None, ws, stream=0, raw=True) == 4
    # missing weight pointer
    wts2 = [dict(wts[0], w_down=None)] + wts[1:]
    assert W.whale_fusion_forward(cfg, fake, fake, fake, wts2, fake, hint, fake, ws, stream=0, raw=True) == 1
    # invalid config / unsupported shape
    bad = Hn.config_of(w.replace(n_heads=3))
    assert W.whale_fusion_forward(bad, fake, fake, fake, wts, fake, hint, fake, ws, stream=0, raw=True) == 1
    unsup = Hn.config_of(w.replace(d=128, n_heads=1))   # d_head 128 not in the bf16 path
    assert W.whale_fusion_forward(unsup, fake, fake, fake, wts, fake, hint, fake, ws, stream=0, raw=True) == 2
    # bad hint
    assert W.whale_fusion_forward(cfg, fake, fake, fake, wts, fake, W.make_hint(2, 10, -5), fake, ws, stream=0,
                                  raw=True) == 1
    # misaligned tokens pointer
    assert W.whale_fusion_forward(cfg, fake + 2, fake, fake, wts, fake, hint, fake, ws, stream=0, raw=True) == 1
    # step entry points
    assert W.whale_project_kv(cfg, 10, None, fake, fake, fake, fake, 1 << 20, stream=0, raw=True) == 1
    assert W.whale_project_kv(cfg, 10, fake, fake, fake, fake, fake, 16, stream=0, raw=True) == 4
    assert W.whale_cross_attention(cfg, fake, fake, None, fake, hint, fake, 1 << 30, stream=0, raw=True) == 1
    assert W.whale_swiglu_ffn(cfg, 10, fake, fake, fake, fake, fake, None, 0, stream=0, raw=True) == 4


def test_empty_batch_is_a_no_op():
    w, cfg = _cfg("stack_d128")
    hint = W.make_hint(0, 0, 0)
    ws = W.whale_workspace_size(cfg, hint)
    assert ws > 0
    fake = 1 << 20
    wts = [dict.fromkeys(["g_q", "g_kv", "w_q", "w_kv", "w_f1", "w_f2", "g_ffn", "w_upgate", "w_down"], fake)] * 4
    assert W.whale_fusion_forward(cfg, fake, fake, fake, wts, fake, hint, fake, ws, stream=0, raw=True) == 0


def test_absorbed_path_selection_and_step_checks():
    fake = 1 << 20
    lw = dict.fromkeys(["g_q", "g_kv", "w_q", "w_kv", "w_f1", "w_f2", "g_ffn", "w_upgate", "w_down"], fake)
    # 15k workload: N*h = 256, d_head = 64 -> absorbed; its workspace holds no K|V tensor
    w, cfg = _cfg("hist15k_d512")
    hint = W.make_hint(64, 15000, 403481)
    cfg_m = W.make_config(cfg.n_layers, cfg.d, cfg.n_heads, cfg.n_tokens, cfg.ffn_hidden, cfg.fusion_hidden,
                          cfg.dtype, cfg.flags | W.WHALE_MATERIALIZED_KV, cfg.eps)
    ws_abs, ws_mat = W.whale_workspace_size(cfg, hint), W.whale_workspace_size(cfg_m, hint)
    assert ws_abs > 0 and ws_mat > 403481 * 2 * w.d * 2
    assert W.whale_attend_states(cfg, None, fake, fake, lw, fake, hint, fake, ws_abs, stream=0, raw=True) == 1
    assert W.whale_attend_states(cfg, fake, fake, fake, lw, fake, hint, fake, ws_abs - 1, stream=0, raw=True) == 4
    assert W.whale_attend_states(cfg_m, fake, fake, fake, lw, fake, hint, fake, ws_mat, stream=0, raw=True) == 2
    # shapes outside the absorbed path: d_head 32 (stack_d256), fp32
    for name in ("stack_d256", "tiny_fp32"):
        w2, cfg2 = _cfg(name)
        h2 = W.make_hint(2, 10, 20)
        ws2 = W.whale_workspace_size(cfg2, h2)
        assert W.whale_attend_states(cfg2, fake, fake, fake, lw, fake, h2, fake, ws2, stream=0, raw=True) == 2
    # prepared weights carry the absorbed keys only where the path applies
    assert W.whale_prepared_weights_size(cfg) > W.whale_prepared_weights_size(
        Hn.config_of(w.replace(n_tokens=16)))


def test_profile_records_nothing_without_launches():
    assert W._lib.whale_profile_begin(0) == 1          # max_kernels must be positive
    W.whale_profile_begin(16)
    assert W.whale_profile_end() == []                  # no kernel launched: no records, no CUDA call
    n = ctypes.c_int(-1)
    assert W._lib.whale_profile_end(None, 4, ctypes.byref(n)) == 1   # records requested into a null buffer


def test_host_buffer_forward_checks_before_any_copy():
    # the host-buffer forward checks its layer count and workspace before it enqueues a copy
    w, cfg = _cfg("stack_d128")
    hint = W.make_hint(2, 10, 20)
    fake = 1 << 20
    lw = dict.fromkeys(["g_q", "g_kv", "w_q", "w_kv", "w_f1", "w_f2", "g_ffn", "w_upgate", "w_down"], fake)
    deep = W.make_config(65, cfg.d, cfg.n_heads, cfg.n_tokens, cfg.ffn_hidden, cfg.fusion_hidden, cfg.dtype,
                         cfg.flags, cfg.eps)
    ws = W.whale_host_workspace_size(deep, hint)
    assert ws > W.whale_workspace_size(deep, hint)          # the staging buffers come first
    assert W.whale_fusion_forward_host(deep, fake, fake, fake, [lw] * 65, fake, hint, fake, ws, stream=0,
                                       raw=True) == 2        # more than 64 layers
    ws4 = W.whale_host_workspace_size(cfg, hint)
    assert W.whale_fusion_forward_host(cfg, fake, fake, fake, [lw] * 4, fake, hint, fake, ws4 - 1, stream=0,
                                       raw=True) == 4
    assert W.whale_fusion_forward_host(cfg, None, fake, fake, [lw] * 4, fake, hint, fake, ws4, stream=0,
                                       raw=True) == 1


def test_fp32_head_sizes():
    # fp32 mode takes d_head 8, 16, 32, 64 or 128 (any d those divide); other head sizes are refused
    hint = W.make_hint(2, 10, 20)
    for d, h, ok in ((64, 8, True), (24, 3, True), (64, 1, True), (128, 1, True), (96, 2, False), (256, 1, False)):
        cfg = W.make_config(1, d, h, 8, 4 * d, 2 * d, W.WHALE_FP32, 0, 1e-6)
        assert (W.whale_workspace_size(cfg, hint) > 0) == ok, (d, h)


def test_bf16_head_counts():
    # bf16 mode: d_head 32 or 64 with 2, 4 or a multiple of 8 heads
    hint = W.make_hint(2, 10, 20)
    for h in range(1, 33):
        for dh in (32, 64):
            d = h * dh
            if d % 64:
                continue
            cfg = W.make_config(1, d, h, 8, 4 * d, 2 * d, W.WHALE_BF16, 0, 1e-6)
            assert (W.whale_workspace_size(cfg, hint) > 0) == (h in (2, 4) or h % 8 == 0), (h, dh)


def test_backward_shapes():
    hint = W.make_hint(2, 10, 20)
    cases = [  # (dtype, d, heads, n_tokens, ffn_hidden, supported)
        (W.WHALE_BF16, 512, 8, 32, 2048, True), (W.WHALE_BF16, 128, 4, 16, 512, True),
        (W.WHALE_BF16, 1024, 16, 32, 4096, True), (W.WHALE_BF16, 2048, 32, 32, 8192, False),   # d > 1024
        (W.WHALE_BF16, 512, 8, 33, 2048, False), (W.WHALE_BF16, 192, 2, 16, 768, False),     # N > 32; d % 128
        (W.WHALE_FP32, 64, 2, 8, 256, True), (W.WHALE_FP32, 96, 12, 8, 384, True),
        (W.WHALE_FP32, 128, 1, 8, 512, False), (W.WHALE_FP32, 48, 6, 8, 192, False),          # d_head 128; d % 32
        (W.WHALE_FP32, 64, 2, 8, 260, False),                                               # ffn_hidden % 8
    ]
    for dt, d, h, n, ffn, ok in cases:
        cfg = W.make_config(1, d, h, n, ffn, 2 * d, dt, 0, 1e-6)
        assert (W.whale_backward_workspace_size(cfg, hint) > 0) == ok, (dt, d, h, n, ffn)
