"""Device placement of the seeded synthetic inputs and one-call runners over the C ABI.

Used by the tests, the smoke check and the benchmark. Nothing here computes any part of
the method: inputs come from `inputs`, every step of the forward runs in libwhale_fusion.so.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch

from . import inputs as I
from . import whale as W


def torch_dtype(w: I.Workload):
    return torch.bfloat16 if w.dtype == "bf16" else torch.float32


def to_device(a: np.ndarray, w: I.Workload, device) -> torch.Tensor:
    """float32 host array (already stored-type rounded) -> device tensor of the storage type."""
    if a is None:
        return None
    if w.dtype == "bf16":
        bits = I.bf16_bits(a)
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)


def gain_to_device(g: np.ndarray, device) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(g, dtype=np.float32)).to(device)


def weights_to_device(lws, w: I.Workload, device) -> list:
    out = []
    for lw in lws:
        out.append({k: (gain_to_device(v, device) if k.startswith("g_") else to_device(v, w, device))
                    for k, v in lw.items()})
    return out


def flags_of(shared_kv=False, tied_gate=False, debug=False, materialized_kv=False) -> int:
    return (W.WHALE_SHARED_KV if shared_kv else 0) | (W.WHALE_TIED_GATE if tied_gate else 0) | \
        (W.WHALE_DEBUG if debug else 0) | (W.WHALE_MATERIALIZED_KV if materialized_kv else 0)


def absorbed_applies(w: I.Workload, materialized_kv: bool = False) -> bool:
    """Whether the library takes the absorbed attention path for this workload (whale_config)."""
    return (w.dtype == "bf16" and not materialized_kv and w.n_tokens * w.n_heads == 256 and w.d_head == 64
            and w.d in (256, 512))


def config_of(w: I.Workload, flags: int = 0) -> W.whale_config:
    return W.make_config(w.n_layers, w.d, w.n_heads, w.n_tokens, w.ffn_hidden, w.fusion_hidden,
                         W.WHALE_BF16 if w.dtype == "bf16" else W.WHALE_FP32, flags, w.eps)


@dataclasses.dataclass
class Problem:
    w: I.Workload
    lengths: np.ndarray
    offsets: np.ndarray
    host_weights: list          # float32 numpy per layer (for the oracle)
    tokens: torch.Tensor        # [B, N, d]
    states: torch.Tensor        # [n_layers, total_L, d]
    offsets_t: torch.Tensor     # int32 [B+1]
    weights: list               # per-layer dicts of device tensors
    cfg: W.whale_config
    hint: W.whale_shape_hint
    out: torch.Tensor
    workspace: torch.Tensor
    flags: dict
    prepared_buf: torch.Tensor | None = None
    raw_weights: list | None = None     # the unprepared weights (kept alive once prepared)

    @property
    def total_L(self) -> int:
        return int(self.offsets[-1])


def build_problem(w: I.Workload, device="cuda", gains="ones", shared_kv=False, tied_gate=False, debug=False,
                  lengths: np.ndarray | None = None, threads: int = 16, materialized_kv=False) -> Problem:
    L = I.draw_lengths(w) if lengths is None else np.asarray(lengths, dtype=np.int64)
    off = I.offsets_of(L)
    total = int(off[-1])
    lws = I.make_all_weights(w, gains=gains, shared_kv=shared_kv, tied_gate=tied_gate)
    tdt = torch_dtype(w)
    states = torch.empty((w.n_layers, max(total, 1), w.d), dtype=tdt, device=device)
    for l in range(w.n_layers):
        if total == 0:
            continue
        if w.dtype == "bf16":
            bits = I.make_states_layer(w, l, L, threads=threads, as_bits=True)
            states[l, :total].copy_(torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16))
        else:
            states[l, :total].copy_(torch.from_numpy(I.make_states_layer(w, l, L, threads=threads)))
    tokens = to_device(I.make_tokens(w), w, device)
    fl = flags_of(shared_kv, tied_gate, debug, materialized_kv)
    cfg = config_of(w, fl)
    hint = W.make_hint(w.batch, int(L.max()) if len(L) else 0, total)
    ws_bytes = W.whale_workspace_size(cfg, hint)
    if ws_bytes == 0:
        raise ValueError("unsupported configuration for the library")
    workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=device)
    out = torch.empty_like(tokens)
    return Problem(w, L, off, lws, tokens, states, torch.from_numpy(off).to(device), weights_to_device(lws, w, device),
                   cfg, hint, out, workspace, {"shared_kv": shared_kv, "tied_gate": tied_gate})


def prepare_weights(p: Problem) -> None:
    """Fold the gains into the weights once (whale_prepare_weights) and switch the problem's
    config to WHALE_PREPARED_WEIGHTS (bf16 only): what a deployment does at load time."""
    if p.w.dtype != "bf16":
        return
    p.prepared_buf = torch.empty(W.whale_prepared_weights_size(p.cfg), dtype=torch.uint8, device=p.out.device)
    # the prepared array still points at the raw w_f1, w_f2, w_down and gains: keep them alive
    p.raw_weights = p.weights
    p.weights = W.whale_prepare_weights(p.cfg, p.weights, p.prepared_buf)
    p.cfg = W.make_config(p.cfg.n_layers, p.cfg.d, p.cfg.n_heads, p.cfg.n_tokens, p.cfg.ffn_hidden,
                          p.cfg.fusion_hidden, p.cfg.dtype, p.cfg.flags | W.WHALE_PREPARED_WEIGHTS, p.cfg.eps)


def run_forward(p: Problem, stream=None) -> torch.Tensor:
    W.whale_fusion_forward(p.cfg, p.tokens, p.states, p.offsets_t, p.weights, p.out, p.hint, p.workspace,
                           stream=stream)
    return p.out


def states_of_example_host(p: Problem, b: int) -> list:
    """Per-layer H_s rows of example b, regenerated on the host (float32)."""
    return [I.states_of_example(p.w, l, b, int(p.lengths[b])) for l in range(p.w.n_layers)]


def run_layer_backward(p: Problem, layer: int, d_out: torch.Tensor, stream=None) -> dict:
    """Gradients of layer `layer` for the upstream gradient d_out (fp32 [B, N, d]) through
    whale_fusion_layer_backward, with the layer's raw weights; the layer's input is the problem's
    tokens. Returns {"d_tokens", "d_states", and one fp32 tensor per parameter}."""
    w = p.w
    lw = (p.raw_weights or p.weights)[layer]
    dev = p.tokens.device
    grads = {k: torch.empty(tuple(v.shape), dtype=torch.float32, device=dev) for k, v in lw.items()
             if v is not None and k != "w_kabs"}
    cfg = config_of(w, flags_of(p.flags.get("shared_kv", False), p.flags.get("tied_gate", False)))
    nbytes = W.whale_backward_workspace_size(cfg, p.hint)
    if nbytes == 0:
        raise ValueError("shape not supported by the backward pass")
    ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    d_tokens = torch.empty(p.tokens.shape, dtype=torch.float32, device=dev)
    d_states = torch.empty(p.states.shape[1:], dtype=p.states.dtype, device=dev)
    W.whale_fusion_layer_backward(cfg, p.tokens, p.states[layer], p.offsets_t, lw, d_out, d_tokens, d_states, grads,
                                  p.hint, ws, stream=stream)
    return {"d_tokens": d_tokens, "d_states": d_states, **grads}


def run_stack_backward(p: Problem, d_out: torch.Tensor, stream=None) -> dict:
    """Gradients of the whole stack for d_out (fp32 [B, N, d]) through whale_fusion_backward, with the
    raw weights. Returns {"d_tokens", "d_states" [n_layers, total_L, d], "grads": one dict per layer}."""
    w = p.w
    dev = p.tokens.device
    raw = p.raw_weights or p.weights
    grads = [{k: torch.empty(tuple(v.shape), dtype=torch.float32, device=dev) for k, v in lw.items()
              if v is not None and k != "w_kabs"} for lw in raw]
    cfg = config_of(w, flags_of(p.flags.get("shared_kv", False), p.flags.get("tied_gate", False)))
    nbytes = W.whale_backward_workspace_size(cfg, p.hint)
    if nbytes == 0:
        raise ValueError("shape not supported by the backward pass")
    ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    d_tokens = torch.empty(p.tokens.shape, dtype=torch.float32, device=dev)
    d_states = torch.empty(p.states.shape, dtype=p.states.dtype, device=dev)
    W.whale_fusion_backward(cfg, p.tokens, p.states, p.offsets_t, raw, d_out, d_tokens, d_states, grads, p.hint, ws,
                            stream=stream)
    return {"d_tokens": d_tokens, "d_states": d_states, "grads": grads}
