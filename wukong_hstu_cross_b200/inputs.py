"""Seeded synthetic inputs for the WHALE fusion forward.

This module is shared by the CPU oracle's tests and by the CUDA path's tests and
benchmark. It holds none of the method's arithmetic: it only draws numbers
(history lengths, token and state values, weights) and rounds them to the
storage type. The five workloads below restate, as shapes and distributions,
the operating points the WHALE pages describe:

* N non-sequence (Wukong) tokens per example, width d, heads, stacked layers
  (pith.science paper page, "Axiom & Free-Parameter Ledger": depth 8, D = 256,
  N = 64, 15k history cap; paper-daily.com digest, section 2: depth 2-8,
  width 64-512, history 3k-15k);
* jagged per-user behavior histories of irregular length
  (paper-daily.com digest, section 2, "irregular lengths");
* a serving workload in which one request's history is shared by many
  candidates whose K/V projections are amortised once per request
  (pith.science verdict, skeptic critique on footnote 1 / M-FALCON).

The pages' own data set (80B/4B samples of a short-video platform) is
proprietary; these synthetic inputs stand in for it.

Every draw comes from numpy's PCG64 through a SeedSequence keyed by
(seed, stream, layer, example, ...), so any slice (one example of one layer)
can be regenerated alone, and the oracle can rebuild a sampled example of a
full-size workload without drawing the rest.
"""
from __future__ import annotations

import dataclasses
import math
from concurrent.futures import ThreadPoolExecutor

import numpy as np

# Stream identifiers for SeedSequence keys (kept distinct so draws never overlap).
_S_TOKENS, _S_STATES, _S_WEIGHTS, _S_LENGTHS, _S_GAINS = 0, 1, 2, 3, 4

# Weight matrix identifiers inside one layer.
_W_IDS = {"w_q": 0, "w_k": 1, "w_v": 2, "w_f1": 3, "w_f2": 4, "w_up": 5, "w_gate": 6, "w_down": 7}
_G_IDS = {"g_q": 0, "g_kv": 1, "g_ffn": 2}


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shapes and distributions of one synthetic workload.

    lengths: ("uniform", lo, hi) integer uniform on [lo, hi];
             ("lognormal", median, sigma, lo, hi) rounded, rejection-resampled
             into [lo, hi]; ("fixed", L).
    """

    name: str
    batch: int            # B: examples (requests)
    n_tokens: int         # N: Wukong tokens (queries) per example
    d: int                # model width
    n_heads: int
    n_layers: int
    dtype: str            # "fp32" or "bf16": storage type of tokens/states/weights
    lengths: tuple
    seed: int
    ffn_mult: int = 4     # SwiGLU hidden = ffn_mult * d
    fusion_mult: int = 2  # Fusion MLP hidden = fusion_mult * d (0: single linear)
    candidates: int = 0   # serving workload: candidates per request (N = candidates * tokens)
    eps: float = 1e-6
    weight_seed: int | None = None   # weights' seed when it differs from `seed` (per-rank shards)

    @property
    def d_head(self) -> int:
        return self.d // self.n_heads

    @property
    def ffn_hidden(self) -> int:
        return self.ffn_mult * self.d

    @property
    def fusion_hidden(self) -> int:
        return self.fusion_mult * self.d

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five operating points. Names state the sizes.
WORKLOADS = {
    "tiny_fp32": Workload("tiny_fp32 (B2 N8 d64 h2 1 layer, L~U[1,256])", 2, 8, 64, 2, 1, "fp32",
                          ("uniform", 1, 256), seed=1),
    "stack_d128": Workload("stack_d128 (B64 N16 d128 h4 4 layers, L~U[1500,3000])", 64, 16, 128, 4, 4,
                           "bf16", ("uniform", 1500, 3000), seed=2),
    "stack_d256": Workload("stack_d256 (B128 N32 d256 h8 4 layers, L~U[3000,6000])", 128, 32, 256, 8, 4,
                           "bf16", ("uniform", 3000, 6000), seed=3),
    "hist15k_d512": Workload("hist15k_d512 (B64 N32 d512 h8 8 layers, L~lognormal(6000,0.5) in [64,15000])",
                             64, 32, 512, 8, 8, "bf16", ("lognormal", 6000.0, 0.5, 64, 15000), seed=4),
    "serve_15k": Workload("serve_15k (1 request, L=15000 shared, 1024 candidates x 16 tokens, d256 h8 4 layers)",
                          1, 1024 * 16, 256, 8, 4, "bf16", ("fixed", 15000), seed=5, candidates=1024),
}
ORDER = ["tiny_fp32", "stack_d128", "stack_d256", "hist15k_d512", "serve_15k"]


def _rng(*key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(k) for k in key])))


# ----------------------------------------------------------------------------------------------
# Storage rounding (round-to-nearest-even to bfloat16), done with integer bit operations.
# ----------------------------------------------------------------------------------------------
def bf16_bits(x: np.ndarray) -> np.ndarray:
    """uint16 bfloat16 bit patterns of float32 values, round-to-nearest-even (no NaN inputs)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_round(x: np.ndarray) -> np.ndarray:
    """float32 array whose values are exactly the bfloat16 rounding of x."""
    return (bf16_bits(x).astype(np.uint32) << np.uint32(16)).view(np.float32)


def from_bf16_bits(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _store(x: np.ndarray, dtype: str) -> np.ndarray:
    x = np.asarray(x, dtype=np.float32)
    return bf16_round(x) if dtype == "bf16" else x


# ----------------------------------------------------------------------------------------------
# Lengths and offsets
# ----------------------------------------------------------------------------------------------
def draw_lengths(w: Workload) -> np.ndarray:
    """History length of every example (int64 [B])."""
    kind = w.lengths[0]
    rng = _rng(w.seed, _S_LENGTHS)
    if kind == "fixed":
        return np.full(w.batch, int(w.lengths[1]), dtype=np.int64)
    if kind == "uniform":
        lo, hi = int(w.lengths[1]), int(w.lengths[2])
        return rng.integers(lo, hi + 1, size=w.batch, dtype=np.int64)
    if kind == "lognormal":
        median, sigma, lo, hi = float(w.lengths[1]), float(w.lengths[2]), int(w.lengths[3]), int(w.lengths[4])
        out = np.empty(w.batch, dtype=np.int64)
        for i in range(w.batch):
            while True:
                v = int(round(float(rng.lognormal(math.log(median), sigma))))
                if lo <= v <= hi:
                    out[i] = v
                    break
        return out
    raise ValueError(f"unknown length distribution {kind!r}")


def offsets_of(lengths: np.ndarray) -> np.ndarray:
    """int32 [B+1] prefix offsets: example b owns history rows [off[b], off[b+1])."""
    off = np.zeros(len(lengths) + 1, dtype=np.int64)
    off[1:] = np.cumsum(lengths)
    if off[-1] >= 2**31:
        raise ValueError("total history rows exceed int32 offsets")
    return off.astype(np.int32)


# ----------------------------------------------------------------------------------------------
# Values
# ----------------------------------------------------------------------------------------------
def tokens_of_example(w: Workload, b: int) -> np.ndarray:
    """Wukong tokens H_w of example b: float32 [N, d], N(0,1), stored-type rounded."""
    return _store(_rng(w.seed, _S_TOKENS, b).standard_normal((w.n_tokens, w.d), dtype=np.float32), w.dtype)


def states_of_example(w: Workload, layer: int, b: int, length: int) -> np.ndarray:
    """HSTU states H_s of example b in layer `layer`: float32 [length, d], N(0,1), stored-type rounded."""
    return _store(_rng(w.seed, _S_STATES, layer, b).standard_normal((int(length), w.d), dtype=np.float32),
                  w.dtype)


def make_tokens(w: Workload) -> np.ndarray:
    """float32 [B, N, d]."""
    return np.stack([tokens_of_example(w, b) for b in range(w.batch)]) if w.batch else \
        np.zeros((0, w.n_tokens, w.d), np.float32)


def make_states_layer(w: Workload, layer: int, lengths: np.ndarray, threads: int = 8,
                      out: np.ndarray | None = None, as_bits: bool = False) -> np.ndarray:
    """One layer's jagged state slab, float32 [sum(L), d] (or bf16 bit patterns if as_bits)."""
    off = offsets_of(lengths).astype(np.int64)
    total = int(off[-1])
    if out is None:
        out = np.empty((total, w.d), dtype=np.uint16 if as_bits else np.float32)

    def fill(b: int) -> None:
        s = states_of_example(w, layer, b, int(lengths[b]))
        out[off[b]:off[b + 1]] = bf16_bits(s) if as_bits else s

    if threads > 1 and w.batch > 1:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(fill, range(w.batch)))
    else:
        for b in range(w.batch):
            fill(b)
    return out


def xavier_uniform(rng: np.random.Generator, fan_out: int, fan_in: int) -> np.ndarray:
    """[fan_out, fan_in] float32 drawn from U(-a, a), a = sqrt(6 / (fan_in + fan_out))."""
    a = math.sqrt(6.0 / (fan_in + fan_out))
    return rng.uniform(-a, a, size=(fan_out, fan_in)).astype(np.float32)


def make_layer_weights(w: Workload, layer: int, gains: str = "ones", shared_kv: bool = False,
                       tied_gate: bool = False) -> dict:
    """All weights of one fusion layer as float32 arrays (stored-type rounded).

    Matrices follow the nn.Linear convention [out, in]. Concatenated matrices:
      w_kv     = [W_K ; W_V]      [2d, d]   (just W_K, [d, d], when shared_kv)
      w_upgate = [W_up ; W_gate]  [2H, d]   (just W_up, [H, d], when tied_gate)
    w_f1 [Fh, 2d] reads the concatenation [A ; H_w]; w_f2 [d, Fh]. With fusion_hidden 0 the
    Fusion MLP is one linear map and w_f1 is absent, w_f2 is [d, 2d].
    Gains g_q, g_kv, g_ffn are float32 [d]: ones, or U[0.5, 1.5] when gains == "random".
    """
    d, H, Fh = w.d, w.ffn_hidden, w.fusion_hidden
    wseed = w.seed if w.weight_seed is None else w.weight_seed

    def mat(name: str, fan_out: int, fan_in: int) -> np.ndarray:
        return _store(xavier_uniform(_rng(wseed, _S_WEIGHTS, layer, _W_IDS[name]), fan_out, fan_in), w.dtype)

    def gain(name: str) -> np.ndarray:
        if gains == "ones":
            return np.ones(d, dtype=np.float32)
        return _rng(wseed, _S_GAINS, layer, _G_IDS[name]).uniform(0.5, 1.5, size=d).astype(np.float32)

    lw = {"g_q": gain("g_q"), "g_kv": gain("g_kv"), "g_ffn": gain("g_ffn"), "w_q": mat("w_q", d, d)}
    wk = mat("w_k", d, d)
    lw["w_kv"] = wk if shared_kv else np.concatenate([wk, mat("w_v", d, d)], axis=0)
    if Fh > 0:
        lw["w_f1"] = mat("w_f1", Fh, 2 * d)
        lw["w_f2"] = mat("w_f2", d, Fh)
    else:
        lw["w_f1"] = None
        lw["w_f2"] = mat("w_f2", d, 2 * d)
    wu = mat("w_up", H, d)
    lw["w_upgate"] = wu if tied_gate else np.concatenate([wu, mat("w_gate", H, d)], axis=0)
    lw["w_down"] = mat("w_down", d, H)
    return lw


def make_all_weights(w: Workload, **kw) -> list:
    return [make_layer_weights(w, l, **kw) for l in range(w.n_layers)]


def small_workload(base: str = "stack_d128", **overrides) -> Workload:
    """A reduced copy of a named workload for tests (same distributions, smaller sizes)."""
    return WORKLOADS[base].replace(**overrides)
