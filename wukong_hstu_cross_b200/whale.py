"""Thin ctypes binding of libwhale_fusion.so (include/whale_fusion.h), same names.

Argument marshalling only: every step of the forward runs in the library's CUDA kernels.
Tensors are torch tensors (device memory and streams come from PyTorch); a plain int is
taken as a raw pointer. Importing this module loads the library and raises ImportError
if it has not been built (python -m wukong_hstu_cross_b200.build) — there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
import re
from ctypes import POINTER, c_float, c_int, c_longlong, c_size_t, c_uint, c_void_p

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libwhale_fusion.so")
HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "whale_fusion.h")

WHALE_FP32, WHALE_BF16 = 0, 1
WHALE_SHARED_KV, WHALE_TIED_GATE, WHALE_DEBUG, WHALE_PREPARED_WEIGHTS = 1, 2, 4, 8
WHALE_MATERIALIZED_KV = 16
WHALE_DEVERR_TIMEOUT, WHALE_DEVERR_OFFSETS = 1, 2
WHALE_NOALLOC_SCRATCH_BYTES = 32 << 20
STATUS = {0: "WHALE_OK", 1: "WHALE_ERR_INVALID_ARG", 2: "WHALE_ERR_UNSUPPORTED", 3: "WHALE_ERR_CUDA",
          4: "WHALE_ERR_WORKSPACE", 5: "WHALE_ERR_DEVICE_CHECK"}


class whale_config(ctypes.Structure):
    _fields_ = [("n_layers", c_int), ("d", c_int), ("n_heads", c_int), ("n_tokens", c_int),
                ("ffn_hidden", c_int), ("fusion_hidden", c_int), ("dtype", c_int), ("flags", c_uint),
                ("eps", c_float)]


_WNAMES = ("g_q", "g_kv", "w_q", "w_kv", "w_f1", "w_f2", "g_ffn", "w_upgate", "w_down", "w_kabs")


class whale_layer_weights(ctypes.Structure):
    _fields_ = [(n, c_void_p) for n in _WNAMES]


_GNAMES = ("g_q", "g_kv", "w_q", "w_kv", "w_f1", "w_f2", "g_ffn", "w_upgate", "w_down")


class whale_layer_grads(ctypes.Structure):
    _fields_ = [(n, c_void_p) for n in _GNAMES]


class whale_shape_hint(ctypes.Structure):
    _fields_ = [("B", c_int), ("max_L", c_int), ("total_L", c_longlong)]


class whale_kernel_time(ctypes.Structure):
    _fields_ = [("kernel", ctypes.c_char_p), ("ms", c_float)]


class WhaleError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {STATUS.get(status, status)}")
        self.status = status


if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m wukong_hstu_cross_b200.build`")
_lib = ctypes.CDLL(LIB_PATH)

_P = c_void_p
_SIGS = {
    "whale_status_string": ([c_int], ctypes.c_char_p),
    "whale_profile_begin": ([c_int], c_int),
    "whale_profile_end": ([POINTER(whale_kernel_time), c_int, POINTER(c_int)], c_int),
    "whale_workspace_size": ([POINTER(whale_config), POINTER(whale_shape_hint)], c_size_t),
    "whale_host_workspace_size": ([POINTER(whale_config), POINTER(whale_shape_hint)], c_size_t),
    "whale_fusion_forward": ([POINTER(whale_config), _P, _P, _P, POINTER(whale_layer_weights), _P,
                              POINTER(whale_shape_hint), _P, c_size_t, _P], c_int),
    "whale_fusion_forward_host": ([POINTER(whale_config), _P, _P, _P, POINTER(whale_layer_weights), _P,
                                   POINTER(whale_shape_hint), _P, c_size_t, _P], c_int),
    "whale_fusion_layer_forward": ([POINTER(whale_config), _P, _P, _P, POINTER(whale_layer_weights), _P,
                                    POINTER(whale_shape_hint), _P, c_size_t, _P], c_int),
    "whale_project_queries": ([POINTER(whale_config), c_longlong, _P, _P, _P, _P, _P, c_size_t, _P], c_int),
    "whale_project_kv": ([POINTER(whale_config), c_longlong, _P, _P, _P, _P, _P, c_size_t, _P], c_int),
    "whale_cross_attention": ([POINTER(whale_config), _P, _P, _P, _P, POINTER(whale_shape_hint), _P, c_size_t,
                               _P], c_int),
    "whale_attend_states": ([POINTER(whale_config), _P, _P, _P, POINTER(whale_layer_weights), _P,
                             POINTER(whale_shape_hint), _P, c_size_t, _P], c_int),
    "whale_fusion_mlp": ([POINTER(whale_config), c_longlong, _P, _P, _P, _P, _P, _P, c_size_t, _P], c_int),
    "whale_swiglu_ffn": ([POINTER(whale_config), c_longlong, _P, _P, _P, _P, _P, _P, c_size_t, _P], c_int),
    "whale_get_device_error": ([_P, POINTER(c_int)], c_int),
    "whale_prepared_weights_size": ([POINTER(whale_config)], c_size_t),
    "whale_prepare_weights": ([POINTER(whale_config), POINTER(whale_layer_weights), _P, c_size_t,
                               POINTER(whale_layer_weights), _P], c_int),
    "whale_cross_attention_noalloc": ([POINTER(whale_config), _P, _P, _P, _P, POINTER(whale_shape_hint), _P], c_int),
    "whale_test_bounded_waits": ([ctypes.c_ulonglong, _P], c_int),
    "whale_backward_workspace_size": ([POINTER(whale_config), POINTER(whale_shape_hint)], c_size_t),
    "whale_fusion_layer_backward": ([POINTER(whale_config), _P, _P, _P, POINTER(whale_layer_weights), _P, _P, _P,
                                     POINTER(whale_layer_grads), POINTER(whale_shape_hint), _P, c_size_t, _P], c_int),
    "whale_fusion_backward": ([POINTER(whale_config), _P, _P, _P, POINTER(whale_layer_weights), _P, _P, _P,
                               POINTER(whale_layer_grads), POINTER(whale_shape_hint), _P, c_size_t, _P], c_int),
}
for _name, (_args, _res) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.argtypes, _f.restype = _args, _res


def header_functions() -> list:
    """Names of the functions include/whale_fusion.h declares."""
    with open(HEADER) as fh:
        text = fh.read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\**\s+\**(whale_\w+)\s*\(", text, flags=re.M)))


# ------------------------------------------------------------------------------------------------
# marshalling helpers
# ------------------------------------------------------------------------------------------------
def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, where: str) -> None:
    if status != 0:
        raise WhaleError(status, where)


def make_config(n_layers, d, n_heads, n_tokens, ffn_hidden, fusion_hidden, dtype, flags=0, eps=1e-6) -> whale_config:
    return whale_config(n_layers, d, n_heads, n_tokens, ffn_hidden, fusion_hidden, dtype, flags, eps)


def make_hint(B, max_L, total_L) -> whale_shape_hint:
    return whale_shape_hint(int(B), int(max_L), int(total_L))


def layer_weights(lw) -> whale_layer_weights:
    """A whale_layer_weights from a dict of tensors (None allowed for w_f1)."""
    if isinstance(lw, whale_layer_weights):
        return lw
    return whale_layer_weights(*[_ptr(lw.get(n)) for n in _WNAMES])


def weights_array(layers) -> ctypes.Array:
    arr = (whale_layer_weights * len(layers))()
    for i, lw in enumerate(layers):
        arr[i] = layer_weights(lw)
    return arr


# ------------------------------------------------------------------------------------------------
# entry points (same names as the C ABI)
# ------------------------------------------------------------------------------------------------
def whale_status_string(status: int) -> str:
    return _lib.whale_status_string(status).decode()


def whale_workspace_size(cfg: whale_config, hint: whale_shape_hint) -> int:
    return int(_lib.whale_workspace_size(ctypes.byref(cfg), ctypes.byref(hint)))


def whale_host_workspace_size(cfg: whale_config, hint: whale_shape_hint) -> int:
    return int(_lib.whale_host_workspace_size(ctypes.byref(cfg), ctypes.byref(hint)))


def _ws_bytes(workspace, nbytes):
    if nbytes is not None:
        return int(nbytes)
    if workspace is None:
        return 0
    return workspace.numel() * workspace.element_size()


def whale_prepared_weights_size(cfg: whale_config) -> int:
    return int(_lib.whale_prepared_weights_size(ctypes.byref(cfg)))


def whale_prepare_weights(cfg, weights, prepared, prepared_bytes=None, stream=None, raw=False):
    """Fold gains / pack up|gate once; returns the ctypes array of prepared layer weights (use it
    with cfg.flags | WHALE_PREPARED_WEIGHTS). The array points into `prepared` and, for the matrices
    that are not re-packed (w_f1, w_f2, w_down, the gains), into the caller's original tensors: it
    keeps references to both, so neither is freed while the array is alive."""
    w = weights if isinstance(weights, ctypes.Array) else weights_array(weights)
    out = (whale_layer_weights * len(w))()
    st = _lib.whale_prepare_weights(ctypes.byref(cfg), w, _ptr(prepared), _ws_bytes(prepared, prepared_bytes), out,
                                    _stream(stream))
    if raw:
        return st
    _check(st, "whale_prepare_weights")
    out._keepalive = (weights, w, prepared)
    return out


def whale_fusion_forward(cfg, wukong_tokens, seq_states, seq_offsets, weights, out, hint, workspace,
                         workspace_bytes=None, stream=None, raw=False):
    w = weights if isinstance(weights, ctypes.Array) else weights_array(weights)
    st = _lib.whale_fusion_forward(ctypes.byref(cfg), _ptr(wukong_tokens), _ptr(seq_states), _ptr(seq_offsets), w,
                                   _ptr(out), ctypes.byref(hint), _ptr(workspace),
                                   _ws_bytes(workspace, workspace_bytes), _stream(stream))
    if raw:
        return st
    _check(st, "whale_fusion_forward")


def whale_fusion_forward_host(cfg, host_tokens, host_seq_states, host_offsets, weights, host_out, hint, workspace,
                              workspace_bytes=None, stream=None, raw=False):
    w = weights if isinstance(weights, ctypes.Array) else weights_array(weights)
    st = _lib.whale_fusion_forward_host(ctypes.byref(cfg), _ptr(host_tokens), _ptr(host_seq_states),
                                        _ptr(host_offsets), w, _ptr(host_out), ctypes.byref(hint), _ptr(workspace),
                                        _ws_bytes(workspace, workspace_bytes), _stream(stream))
    if raw:
        return st
    _check(st, "whale_fusion_forward_host")


def whale_fusion_layer_forward(cfg, tokens_in, layer_states, seq_offsets, layer_weights_, tokens_out, hint, workspace,
                               workspace_bytes=None, stream=None, raw=False):
    lw = layer_weights(layer_weights_)
    st = _lib.whale_fusion_layer_forward(ctypes.byref(cfg), _ptr(tokens_in), _ptr(layer_states), _ptr(seq_offsets),
                                         ctypes.byref(lw), _ptr(tokens_out), ctypes.byref(hint), _ptr(workspace),
                                         _ws_bytes(workspace, workspace_bytes), _stream(stream))
    if raw:
        return st
    _check(st, "whale_fusion_layer_forward")


def whale_project_queries(cfg, rows, x, g_q, w_q, q, workspace, workspace_bytes=None, stream=None, raw=False):
    st = _lib.whale_project_queries(ctypes.byref(cfg), int(rows), _ptr(x), _ptr(g_q), _ptr(w_q), _ptr(q),
                                    _ptr(workspace), _ws_bytes(workspace, workspace_bytes), _stream(stream))
    if raw:
        return st
    _check(st, "whale_project_queries")


def whale_project_kv(cfg, rows, s, g_kv, w_kv, kv, workspace, workspace_bytes=None, stream=None, raw=False):
    st = _lib.whale_project_kv(ctypes.byref(cfg), int(rows), _ptr(s), _ptr(g_kv), _ptr(w_kv), _ptr(kv),
                               _ptr(workspace), _ws_bytes(workspace, workspace_bytes), _stream(stream))
    if raw:
        return st
    _check(st, "whale_project_kv")


def whale_cross_attention(cfg, q, kv, seq_offsets, a, hint, workspace, workspace_bytes=None, stream=None, raw=False):
    st = _lib.whale_cross_attention(ctypes.byref(cfg), _ptr(q), _ptr(kv), _ptr(seq_offsets), _ptr(a),
                                    ctypes.byref(hint), _ptr(workspace), _ws_bytes(workspace, workspace_bytes),
                                    _stream(stream))
    if raw:
        return st
    _check(st, "whale_cross_attention")


def whale_attend_states(cfg, q, layer_states, seq_offsets, weights, a, hint, workspace, workspace_bytes=None,
                        stream=None, raw=False):
    """S2 + S3 in absorbed form (no K|V tensor): `weights` is one layer's dict or whale_layer_weights."""
    lw = layer_weights(weights)
    st = _lib.whale_attend_states(ctypes.byref(cfg), _ptr(q), _ptr(layer_states), _ptr(seq_offsets),
                                  ctypes.byref(lw), _ptr(a), ctypes.byref(hint), _ptr(workspace),
                                  _ws_bytes(workspace, workspace_bytes), _stream(stream))
    if raw:
        return st
    _check(st, "whale_attend_states")


def whale_cross_attention_noalloc(cfg, q, kv, seq_offsets, a, hint, stream=None, raw=False):
    """Eq. (4) without a workspace: the partials live in the library's fixed device array
    (WHALE_NOALLOC_SCRATCH_BYTES); see include/whale_fusion.h."""
    st = _lib.whale_cross_attention_noalloc(ctypes.byref(cfg), _ptr(q), _ptr(kv), _ptr(seq_offsets), _ptr(a),
                                            ctypes.byref(hint), _stream(stream))
    if raw:
        return st
    _check(st, "whale_cross_attention_noalloc")


def whale_fusion_mlp(cfg, rows, a, x, w_f1, w_f2, f, workspace, workspace_bytes=None, stream=None, raw=False):
    st = _lib.whale_fusion_mlp(ctypes.byref(cfg), int(rows), _ptr(a), _ptr(x), _ptr(w_f1), _ptr(w_f2), _ptr(f),
                               _ptr(workspace), _ws_bytes(workspace, workspace_bytes), _stream(stream))
    if raw:
        return st
    _check(st, "whale_fusion_mlp")


def whale_swiglu_ffn(cfg, rows, f, g_ffn, w_upgate, w_down, y, workspace, workspace_bytes=None, stream=None,
                     raw=False):
    st = _lib.whale_swiglu_ffn(ctypes.byref(cfg), int(rows), _ptr(f), _ptr(g_ffn), _ptr(w_upgate), _ptr(w_down),
                               _ptr(y), _ptr(workspace), _ws_bytes(workspace, workspace_bytes), _stream(stream))
    if raw:
        return st
    _check(st, "whale_swiglu_ffn")


def whale_profile_begin(max_kernels: int = 4096) -> None:
    _check(_lib.whale_profile_begin(max_kernels), "whale_profile_begin")


def whale_profile_end(capacity: int = 4096) -> list:
    """[(kernel name, ms), ...] in launch order (see include/whale_fusion.h)."""
    buf = (whale_kernel_time * capacity)()
    n = c_int(0)
    _check(_lib.whale_profile_end(buf, capacity, ctypes.byref(n)), "whale_profile_end")
    return [((buf[i].kernel or b"?").decode(), float(buf[i].ms)) for i in range(min(n.value, capacity))]


def whale_backward_workspace_size(cfg: whale_config, hint: whale_shape_hint) -> int:
    return int(_lib.whale_backward_workspace_size(ctypes.byref(cfg), ctypes.byref(hint)))


def layer_grads(g) -> whale_layer_grads:
    """A whale_layer_grads from a dict of fp32 tensors (w_f1 may be absent or None)."""
    if isinstance(g, whale_layer_grads):
        return g
    return whale_layer_grads(*[_ptr(g.get(n)) for n in _GNAMES])


def whale_fusion_layer_backward(cfg, tokens_in, layer_states, seq_offsets, layer_weights_, d_out, d_tokens, d_states,
                                grads, hint, workspace, workspace_bytes=None, stream=None, raw=False):
    """Gradients of one fusion layer (see include/whale_fusion.h); `grads` is a dict of fp32 tensors."""
    lw = layer_weights(layer_weights_)
    gr = layer_grads(grads)
    st = _lib.whale_fusion_layer_backward(ctypes.byref(cfg), _ptr(tokens_in), _ptr(layer_states), _ptr(seq_offsets),
                                          ctypes.byref(lw), _ptr(d_out), _ptr(d_tokens), _ptr(d_states),
                                          ctypes.byref(gr), ctypes.byref(hint), _ptr(workspace),
                                          _ws_bytes(workspace, workspace_bytes), _stream(stream))
    if raw:
        return st
    _check(st, "whale_fusion_layer_backward")


def whale_fusion_backward(cfg, wukong_tokens, seq_states, seq_offsets, weights, d_out, d_tokens, d_states, grads,
                          hint, workspace, workspace_bytes=None, stream=None, raw=False):
    """Gradients of the whole stack (see include/whale_fusion.h): `weights` one dict per layer (raw),
    `grads` one dict of fp32 tensors per layer."""
    w = weights if isinstance(weights, ctypes.Array) else weights_array(weights)
    g = (whale_layer_grads * len(grads))(*[layer_grads(x) for x in grads])
    st = _lib.whale_fusion_backward(ctypes.byref(cfg), _ptr(wukong_tokens), _ptr(seq_states), _ptr(seq_offsets), w,
                                    _ptr(d_out), _ptr(d_tokens), _ptr(d_states), g, ctypes.byref(hint),
                                    _ptr(workspace), _ws_bytes(workspace, workspace_bytes), _stream(stream))
    if raw:
        return st
    _check(st, "whale_fusion_backward")


def whale_test_bounded_waits(limit_ns: int, stream=None, raw=False):
    """Enqueue the self-test of the bounded device waits (see include/whale_fusion.h)."""
    st = _lib.whale_test_bounded_waits(int(limit_ns), _stream(stream))
    if raw:
        return st
    _check(st, "whale_test_bounded_waits")


def whale_get_device_error(stream=None) -> int:
    code = c_int(0)
    st = _lib.whale_get_device_error(_stream(stream), ctypes.byref(code))
    if st not in (0, 5):
        _check(st, "whale_get_device_error")
    return code.value
