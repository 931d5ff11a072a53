"""Benchmark of the WHALE attention-fusion forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

A step is one pass of the whole hot path (every layer of the stack: RMSNorm + projections,
split-L cross-attention, Fusion MLP, SwiGLU FFN) over one batch of synthetic inputs that are
already resident in HBM. The default workload is the 15k-history stack (B=64 examples,
N=32 Wukong tokens, d=512, 8 heads, 8 layers, lognormal history lengths in [64, 15000]).
Every layer reads its own 0.4 GB state slab, larger than the 126 MB L2, so no L2 flush is
needed between steps. Under torchrun each rank runs its own batch (weak scaling, examples are
independent: no data-path collective); the step time is the max over ranks.

Prints one JSON line (rank 0). `--impl reference` times the fp64 CPU oracle instead (the
reference arm of this repository), on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import re
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from wukong_hstu_cross_b200 import inputs as I  # noqa: E402

METRIC = "WHALE fusion-layer examples/s @15k jagged history; % of HBM/TC roofline"
# DRAM bytes per launch measured by ncu (dram__bytes_read.sum + dram__bytes_write.sum), per
# history row: one capture of the 2-SM K|V projection GEMM at d = 512 on 109 605 rows. Reported
# only for that width; null otherwise.
KV_TRAFFIC_BYTES_PER_ROW_D512 = (113.378816e6 + 169.603840e6) / 109605

# DRAM bytes per history row of the absorbed path's pass A kernel (abs_scores_kernel<2>): one ncu
# capture at d = 512 on the full 403 481-row batch (444.77 MB read + 174.42 MB written per launch).
# Two-kernel path only (the default).
ABS_PASSA_BYTES_PER_ROW_D512 = (444.77e6 + 174.42e6) / 403481
# ... and of a whole whale_attend_states call (its six kernels: 1121.52 MB read + 191.63 MB written)
ABS_TRAFFIC_BYTES_PER_ROW_D512 = (1121.52e6 + 191.63e6) / 403481

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0}


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as fh:
            p = json.load(fh)
        return p, "measured"
    except Exception:
        return PEAKS_FALLBACK, "fallback"


def tensor_peak(peaks: dict, clocks) -> tuple:
    """The bf16 tensor peak that applies to kernels timed in this run: the burst figure when the SM
    clock sampled during the timed region stayed near its maximum (a short run, below the power
    cap), else the sustained figure (a long run that settled under the power cap)."""
    burst, sus = peaks["bf16_tflops"], peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    mx = peaks.get("sm_max_mhz", 1965.0)
    if clocks and clocks.get("sm_mhz") and clocks["sm_mhz"] < 0.95 * mx:
        return sus, f"bf16 sustained (median SM clock {clocks['sm_mhz']:.0f} of {mx:.0f} MHz under load)"
    return burst, (f"bf16 burst (median SM clock {clocks['sm_mhz']:.0f} of {mx:.0f} MHz under load)" if clocks
                   and clocks.get("sm_mhz") else "bf16 burst (no clock samples)")


def roofline_of(flops: float, nbytes: float, t_ms: float, tc_peak: float, hbm_peak: float) -> dict:
    """Roofline position of a kernel from its algorithmic work: the bound is the larger of its FLOP
    time at the tensor peak and its byte time at the copy bandwidth; achieved and peak are in that
    bound's unit, so frac = (bound's algorithmic time) / (measured time)."""
    t_flop = flops / (tc_peak * 1e12)
    t_byte = nbytes / (hbm_peak * 1e9)
    t = t_ms * 1e-3
    if t_flop >= t_byte:
        return {"bound": "tensor", "achieved": flops / t / 1e12, "peak": tc_peak, "unit": "TFLOP/s",
                "frac": t_flop / t, "t_flop_us": t_flop * 1e6, "t_byte_us": t_byte * 1e6,
                "tensor_frac": t_flop / t, "hbm_frac": t_byte / t}
    return {"bound": "hbm", "achieved": nbytes / t / 1e9, "peak": hbm_peak, "unit": "GB/s", "frac": t_byte / t,
            "t_flop_us": t_flop * 1e6, "t_byte_us": t_byte * 1e6, "tensor_frac": t_flop / t, "hbm_frac": t_byte / t}


# ------------------------------------------------------------------------------------------------
# algorithmic work per step (bf16 storage)
# ------------------------------------------------------------------------------------------------
def step_work(w: I.Workload, total_L: int, shared_kv: bool = False, tied_gate: bool = False,
              absorbed: bool = False) -> dict:
    """FLOPs and bytes per kernel family for one layer (no re-reads, no partials; the hi/lo
    operand halves of the token-side GEMMs are not counted: algorithmic work only).

    absorbed: S2 + S3 with K and V folded into the queries (one family): the scores of the N*h
    absorbed queries against every history row and the weighted row sums, 2 x (2 N h L d), plus the
    per-head query and output GEMMs (2 rows d d_head h = 2 rows d^2 each); its algorithmic bytes
    are the states read once plus q, A and the two weight matrices."""
    B, N, d, H, Fh = w.batch, w.n_tokens, w.d, w.ffn_hidden, w.fusion_hidden
    rows = B * N
    e = 2
    kvw = d if shared_kv else 2 * d
    ugw = H if tied_gate else 2 * H
    if absorbed:
        nq = N * w.n_heads
        history = {"attention_absorbed": {"flops": 4.0 * nq * total_L * d + 4.0 * rows * d * d,
                                          "bytes": e * (total_L * d + 2 * rows * d + 2 * d * d)}}
    else:
        history = {
            "kv_proj": {"flops": 2.0 * total_L * d * kvw, "bytes": e * (total_L * d + total_L * kvw + kvw * d)},
            "attention": {"flops": 4.0 * N * total_L * d,   # q k^T and p v: 2 x (2 N L d) per example
                          "bytes": e * (total_L * kvw + 2 * rows * d)},
        }
    return {
        **history,
        "q_proj": {"flops": 2.0 * rows * d * d, "bytes": e * (2 * rows * d + d * d)},
        "fusion_mlp": {"flops": 2.0 * rows * (2 * d * Fh + Fh * d), "bytes": e * (3 * rows * d + 2 * rows * Fh + 3 * d * Fh)},
        "swiglu_ffn": {"flops": 2.0 * rows * (d * ugw + H * d), "bytes": e * (3 * rows * d + 2 * rows * H + (ugw + H) * d)},
    }


def kernel_name(mangled: str) -> str:
    """Readable name of one of the library's kernels: `_ZN5whale17abs_scores_kernelE...` ->
    `abs_scores_kernel`, with integer / bool template arguments as `<64,2,0,1>`."""
    m = re.match(r"_ZN5whale(\d+)", mangled)
    if not m:
        return mangled
    n = int(m.group(1))
    rest = mangled[m.end():]
    name, rest = rest[:n], rest[n:]
    if rest.startswith("I"):
        args = re.findall(r"L[ib](-?\d+)E", rest.split("EE")[0] + "E")
        if args:
            name += "<" + ",".join(args) + ">"
    return name


def launches_per_step(w: I.Workload, fold_per_call: bool, absorbed: bool) -> int:
    # once: residual-stream set-up (+ unit starts of the absorbed path); per layer: [weight fold,]
    # Q GEMM, then either K|V GEMM + attention (split merge fused in) or absorbed-query GEMM + pass A +
    # pass B + merge + W_V GEMM; Fusion GEMM(s), up|gate GEMM, down GEMM
    history = 5 if absorbed else 2
    return 1 + (1 if absorbed else 0) + w.n_layers * (
        1 + history + 3 + (1 if fold_per_call else 0) + (1 if w.fusion_hidden > 0 else 0))


# ------------------------------------------------------------------------------------------------
# clocks sampled while the timed region runs
# ------------------------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"whale_clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.fh,
                                         stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.fh.close()

    def summary(self):
        if self.proc is None:
            return None
        try:
            rows = [r.split(",") for r in open(self.path).read().strip().splitlines() if r.strip()]
        except Exception:
            return None
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
                for k, v in zip(names, r[5:9]):
                    if v.strip() == "Active":
                        reasons.add(k)
            except Exception:
                continue
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------------------------------------
# CPU baseline: the oracle on a bounded sample of the workload
# ------------------------------------------------------------------------------------------------
class OracleSampler:
    """The fp64 oracle timed on whole examples of the workload, walking the batch in order (and
    round again): lengths and weights are drawn once; each example's inputs are generated before
    its timed region (not concurrently: a generator thread beside the oracle's BLAS threads
    oversubscribes the cores and slows the oracle down)."""

    def __init__(self, w: I.Workload):
        self.w = w
        self.L = I.draw_lengths(w)
        self.lws = I.make_all_weights(w)
        # serving workload: time 64 of the request's candidate tokens, scale per example
        self.sample_tokens = 64 if w.candidates else w.n_tokens
        self.next_b = 0
        self.done, self.toks, self.t = 0, 0, 0.0
        self.step_s = []

    def _inputs(self, b: int):
        w = self.w
        x = I.tokens_of_example(w, b)[:self.sample_tokens]
        slabs = [I.states_of_example(w, l, b, int(self.L[b])) for l in range(w.n_layers)]
        return x, slabs

    def run(self, budget_s: float, max_examples: int = None, count: bool = True) -> float:
        """Examples from the rolling index on until budget_s of oracle time (at least one); returns
        the oracle time spent."""
        from oracle import whale_oracle as O
        w = self.w
        t_run, n = 0.0, 0
        while True:
            x, slabs = self._inputs(self.next_b)
            self.next_b = (self.next_b + 1) % w.batch
            t0 = time.perf_counter()
            O.fusion_stack_example(x, slabs, self.lws, w.n_heads, w.eps)
            dt = time.perf_counter() - t0
            t_run += dt
            n += 1
            if count:
                self.t += dt
                self.done += 1
                self.toks += self.sample_tokens
            if t_run >= budget_s or (max_examples is not None and n >= max_examples):
                break
        if count:
            self.step_s.append(t_run)
        return t_run

    def value(self) -> float:
        w = self.w
        if w.candidates:  # per-token cost: the sampled tokens share the K/V projections (as in serving)
            return 1.0 / (self.t * (w.n_tokens / self.toks))
        return self.done / self.t

    def summary(self, what: str) -> dict:
        w = self.w
        cores = len(os.sched_getaffinity(0))
        if w.candidates:
            desc = f"{self.done} request(s), {self.sample_tokens} of {w.n_tokens} candidate tokens timed, scaled per request"
        else:
            desc = (f"{what}: {self.done} examples timed, walking the batch in order from example 0 "
                    f"(all {w.n_layers} layers, all {w.n_tokens} tokens each)")
        return {"value": self.value(), "unit": "examples/s", "cores": cores, "kind": "oracle",
                "sample": desc + f"; fp64 numpy on {cores} host threads, {self.t:.1f} s of oracle time"}


def oracle_sample(w: I.Workload, budget_s: float = 15.0, max_examples: int = 64):
    s = OracleSampler(w)
    s.run(budget_s, max_examples=min(w.batch, max_examples))
    return s.summary("cpu baseline")


def workload_config(w: I.Workload, total_L: int, max_L: int, world: int, args) -> dict:
    """The `config` object of the JSON line (the same for both arms)."""
    return {"workload": w.name, "batch": w.batch, "n_tokens": w.n_tokens, "d": w.d, "heads": w.n_heads,
            "layers": w.n_layers, "total_L": int(total_L), "max_L": int(max_L),
            "parallelism": f"dp{world} (independent examples per rank, no collective)",
            "variant": ("shared K=V " if args.shared_kv else "") + ("tied gate" if args.tied_gate else "")
                       or "separate W_K, W_V; untied up|gate",
            "weights": ("gains folded per forward" if args.fold_per_call else
                        "gains folded into the weights once at load (whale_prepare_weights)"),
            "l2": "inputs larger than L2 (each layer reads its own "
                  f"{total_L * w.d * 2 / 1e6:.0f} MB state slab), no flush"}


# ------------------------------------------------------------------------------------------------
def dist_setup(n_gpus):
    import torch
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    else:
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    from wukong_hstu_cross_b200 import dist as D
    return D.max_over_ranks(x, world, device="cuda")


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = I.WORKLOADS[args.workload]
    t0 = time.time()
    steps = max(args.steps, 1)
    sampler = OracleSampler(w)
    for _ in range(max(args.warmup, 0)):   # untimed: one example each
        sampler.run(0.0, count=False)
    # the whole run is bounded: each step gets an equal share of --ref-total seconds of oracle time
    # (at least one whole example), walking the batch in order from where the warm-up stopped
    per_step = max(0.2, args.ref_total / steps)
    for _ in range(steps):
        sampler.run(per_step)
    cb = sampler.summary("reference arm")
    value = cb["value"]
    ms_step = 1e3 * statistics.mean(sampler.step_s)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "examples/s", "n_gpus": args.gpus,
            "steps": steps, "warmup": max(args.warmup, 0), "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(w, int(sampler.L.sum()), int(sampler.L.max()), args.gpus, args),
            "step": f"a bounded sample of the workload: {per_step:.1f} s of oracle time per step, whole examples",
            "cpu_baseline": cb, "e2e": {"value": value, "unit": "examples/s", "h2d_bytes_per_step": 0,
                                        "d2h_bytes_per_step": 0},
            "wall_s": time.time() - t0}
    print(json.dumps(line), flush=True)
    return 0


def run_kernel_case(args):
    """One step entry point (K|V projection, attention, absorbed attention, SwiGLU FFN or Fusion MLP)
    on one layer, for ncu captures.
    Prints the average device time per launch; not a benchmark line."""
    import torch
    from wukong_hstu_cross_b200 import build
    build.build()
    from wukong_hstu_cross_b200 import harness as Hn
    from wukong_hstu_cross_b200 import whale as Wb
    w = I.WORKLOADS[args.workload].replace(n_layers=1)
    if args.batch:
        w = w.replace(batch=args.batch)
    p = Hn.build_problem(w, device="cuda")
    lw = p.weights[0]
    if args.kernel_case == "backward":  # one layer's backward (all of its kernels)
        import torch
        res = time_backward(p, p.weights, w, p.total_L, load_peaks()[0], None, torch.cuda.current_stream(),
                            reps=args.steps)
        print(json.dumps({"kernel_case": "backward", "workload": w.name, "total_L": p.total_L,
                          "ms_per_layer": res.get("ms_per_layer")}), flush=True)
        return 0
    if args.kernel_case == "absorbed":
        Hn.prepare_weights(p)   # as the forward runs it: gains folded, absorbed keys formed at load
    T = p.total_L
    kv = torch.empty(T, 2 * w.d, dtype=torch.bfloat16, device="cuda")
    q = torch.empty(w.batch * w.n_tokens, w.d, dtype=torch.bfloat16, device="cuda")
    a = torch.empty_like(q)
    raw = Hn.config_of(w)
    Wb.whale_project_queries(raw, q.shape[0], p.tokens, lw["g_q"], lw["w_q"], q, p.workspace)
    if args.kernel_case != "absorbed":
        Wb.whale_project_kv(p.cfg, T, p.states[0], lw["g_kv"], lw["w_kv"], kv, p.workspace)

    rows = w.batch * w.n_tokens
    f_out = torch.empty_like(q)

    def step():
        if args.kernel_case == "kv":
            Wb.whale_project_kv(p.cfg, T, p.states[0], lw["g_kv"], lw["w_kv"], kv, p.workspace)
        elif args.kernel_case == "attn":
            Wb.whale_cross_attention(p.cfg, q, kv, p.offsets_t, a, p.hint, p.workspace)
        elif args.kernel_case == "absorbed":  # S2 + S3 without K|V: query GEMM, pass A, pass B, merge, W_V GEMM
            Wb.whale_attend_states(p.cfg, q, p.states[0], p.offsets_t, p.weights[0], a, p.hint, p.workspace)
        elif args.kernel_case == "ffn":     # up|gate GEMM (SwiGLU epilogue) + down GEMM
            Wb.whale_swiglu_ffn(p.cfg, rows, q, lw["g_ffn"], lw["w_upgate"], lw["w_down"], f_out, p.workspace)
        else:                               # Fusion MLP: two GEMMs
            Wb.whale_fusion_mlp(p.cfg, rows, a, q, lw["w_f1"], lw["w_f2"], f_out, p.workspace)
    step()  # compile / first-use work outside the timed loop
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    work = step_work(w, T, absorbed=args.kernel_case == "absorbed")[
        {"kv": "kv_proj", "attn": "attention", "ffn": "swiglu_ffn", "fusion": "fusion_mlp",
         "absorbed": "attention_absorbed"}[args.kernel_case]]
    print(json.dumps({"kernel_case": args.kernel_case, "workload": w.name, "total_L": T, "ms_per_launch": ms,
                      "tflops": work["flops"] / ms / 1e9, "gbs": work["bytes"] / ms / 1e6}), flush=True)
    return 0


def time_backward(p, raw_weights, w, total_L, peaks, clocks, stream, reps=10):
    """One layer's backward (whale_fusion_layer_backward, raw weights, an N(0,1) upstream gradient)
    timed with CUDA events over `reps` calls, its kernels from the library's per-kernel events, and
    the roofline of its attention kernel (KV-parallel: reads K|V and writes dK|dV once, plus the
    example's queries per history chunk: HBM-bound at N <= 32)."""
    import torch
    from wukong_hstu_cross_b200 import harness as Hn
    from wukong_hstu_cross_b200 import whale as Wb
    cfg = Hn.config_of(w, Hn.flags_of(p.flags.get("shared_kv", False), p.flags.get("tied_gate", False)))
    nbytes = Wb.whale_backward_workspace_size(cfg, p.hint)
    if nbytes == 0:
        return {"unsupported": "shape outside the backward pass's support"}
    lw = raw_weights[0]
    dev = p.tokens.device
    grads = {k: torch.empty(tuple(v.shape), dtype=torch.float32, device=dev) for k, v in lw.items()
             if v is not None and k != "w_kabs"}
    ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    d_out = torch.randn(p.tokens.shape, dtype=torch.float32, device=dev, generator=torch.Generator(dev).manual_seed(1))
    d_tok = torch.empty(p.tokens.shape, dtype=torch.float32, device=dev)
    d_st = torch.empty(p.states.shape[1:], dtype=p.states.dtype, device=dev)

    def call():
        Wb.whale_fusion_layer_backward(cfg, p.tokens, p.states[0], p.offsets_t, lw, d_out, d_tok, d_st, grads, p.hint,
                                       ws, stream=stream)
    for _ in range(2):
        call()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        call()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    Wb.whale_profile_begin(4096)
    call()
    recs = Wb.whale_profile_end()
    kern = {}
    for name, kms in recs:
        e = kern.setdefault(kernel_name(name), [0, 0.0])
        e[0] += 1
        e[1] += kms
    tot = sum(v[1] for v in kern.values()) or 1.0
    kernels = {n: {"launches": c, "avg_ms": t / c, "share": t / tot}
               for n, (c, t) in sorted(kern.items(), key=lambda x: -x[1][1])}
    out = {"entry_point": "whale_fusion_layer_backward (one layer, its forward recomputed inside)", "ms_per_layer": ms,
           "reps": reps, "kernels": kernels,
           "launch_order": [[kernel_name(n), round(t, 4)] for n, t in recs]}
    abk = next((k for k in kernels if k.split("<")[0] in ("attn_bwd_tc_kernel", "attn_bwd_kernel")), None)
    ab = kernels[abk] if abk else None
    if ab:
        kvw = w.d if p.flags.get("shared_kv") else 2 * w.d
        nb = 2.0 * total_L * kvw * 2          # K|V read once, dK|dV written once (bf16)
        fl = 10.0 * w.n_tokens * total_L * w.d  # S, dP, dV, dK, dQ: five contractions of 2 N L d
        tc, tc_src = tensor_peak(peaks, clocks)
        what = ("tcgen05, TMEM accumulators" if abk.startswith("attn_bwd_tc") else "mma.sync")
        out["roofline"] = {"kernel": f"{abk} (KV-parallel attention backward, {what})",
                           **roofline_of(fl, nb, ab["avg_ms"], tc, peaks["hbm_gbs"]),
                           "algorithmic_flops_per_launch": fl, "algorithmic_bytes_per_launch": nb,
                           "avg_launch_ms": ab["avg_ms"], "peak_source": tc_src}
    del ws, grads, d_st
    # the whole stack's backward (whale_fusion_backward: its forward on the recompute path, then every
    # layer's backward, last layer first), timed over two calls after one warm-up call
    if w.n_layers > 1:
        raw = raw_weights
        sgrads = [{k: torch.empty(tuple(v.shape), dtype=torch.float32, device=dev) for k, v in lwl.items()
                   if v is not None and k != "w_kabs"} for lwl in raw]
        sws = torch.empty(Wb.whale_backward_workspace_size(cfg, p.hint), dtype=torch.uint8, device=dev)
        s_st = torch.empty(p.states.shape, dtype=p.states.dtype, device=dev)

        def scall():
            Wb.whale_fusion_backward(cfg, p.tokens, p.states, p.offsets_t, raw, d_out, d_tok, s_st, sgrads, p.hint,
                                     sws, stream=stream)
        scall()
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(2):
            scall()
        e1.record(stream)
        torch.cuda.synchronize()
        out["stack"] = {"entry_point": ("whale_fusion_backward (all layers; the forward once, each layer's "
                                        "activations kept for its backward)"),
                        "ms": e0.elapsed_time(e1) / 2, "layers": w.n_layers, "calls": 2}
        del sgrads, sws, s_st
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="hist15k_d512", choices=list(I.WORKLOADS))
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--ref-budget", type=float, default=15.0, help="oracle seconds of the cpu_baseline sample")
    ap.add_argument("--ref-total", type=float, default=90.0,
                    help="oracle seconds of the whole --impl reference run, split across its steps")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--kernel-case", choices=["kv", "attn", "ffn", "fusion", "absorbed", "backward"], default=None,
                    help="profiling aid: run only one step entry point on one layer of the workload")
    ap.add_argument("--batch", type=int, default=None, help="override the workload's batch (kernel cases)")
    ap.add_argument("--shared-kv", action="store_true", help="variant: K = V (one W_K), the pages' shared key/value")
    ap.add_argument("--tied-gate", action="store_true", help="variant: W_gate = W_up, the pages' shared-gate SwiGLU")
    ap.add_argument("--fold-per-call", action="store_true",
                    help="fold the RMSNorm gains into the weights inside every forward instead of once at load")
    ap.add_argument("--no-backward", action="store_true", help="skip the one-layer backward measurement")
    ap.add_argument("--no-graph", action="store_true", help="skip the CUDA-graph replay measurement")
    ap.add_argument("--materialized-kv", action="store_true",
                    help="project K|V and attend over them even where the absorbed attention applies")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.impl == "reference":
        return run_reference(args)
    if args.kernel_case:
        return run_kernel_case(args)

    import torch
    rank, world, local = dist_setup(args.gpus)
    from wukong_hstu_cross_b200 import build
    if rank == 0:
        build.build()
    barrier(world)
    from wukong_hstu_cross_b200 import harness as Hn
    from wukong_hstu_cross_b200 import whale as Wb

    from wukong_hstu_cross_b200 import dist as D
    w = D.shard_workload(I.WORKLOADS[args.workload], rank, world)   # this rank's own examples
    p = Hn.build_problem(w, device="cuda", shared_kv=args.shared_kv, tied_gate=args.tied_gate,
                         materialized_kv=args.materialized_kv)
    absorbed = Hn.absorbed_applies(w, args.materialized_kv)
    raw_weights = p.weights
    if not args.fold_per_call:
        Hn.prepare_weights(p)   # gains folded into the weights once, as at model load
    stream = torch.cuda.current_stream()
    total_L = p.total_L

    # ---------------- device-resident timed region: the whole stack per step ----------------
    # A deployment replays a captured CUDA graph of the forward (launches, their programmatic
    # dependencies and arguments recorded once, the same kernels); that replay is the timed step.
    # The same step launched call by call is timed beside it (`stream_launch`); --no-graph makes the
    # call-by-call launches the timed step.
    for _ in range(args.warmup):
        Hn.run_forward(p, stream)
    torch.cuda.synchronize()

    def timed(step_fn, steps, sample_clocks):
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        clk = ClockSampler(local) if sample_clocks else None
        if clk:
            clk.__enter__()
        try:
            barrier(world)
            torch.cuda.synchronize()
            ev0.record(stream)
            for _ in range(steps):
                step_fn()
            ev1.record(stream)
            torch.cuda.synchronize()
            barrier(world)
        finally:
            if clk:
                clk.__exit__(None, None, None)
        return max_over_ranks(ev0.elapsed_time(ev1) / steps, world), (clk.summary() if clk else None)

    stream_launch = None
    if args.no_graph:
        ms, clocks = timed(lambda: Hn.run_forward(p, stream), args.steps, True)
        launch = "call by call (programmatic dependent launches on one stream)"
    else:
        side = torch.cuda.Stream()
        with torch.cuda.stream(side):
            Hn.run_forward(p, side)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            Hn.run_forward(p, side)
        torch.cuda.synchronize()
        for _ in range(args.warmup):
            g.replay()
        torch.cuda.synchronize()
        ms, clocks = timed(g.replay, args.steps, True)
        s_ms, _ = timed(lambda: Hn.run_forward(p, stream), args.steps, False)
        stream_launch = {"ms_per_step": s_ms, "value": world * w.batch / (s_ms / 1e3), "steps": args.steps,
                         "what": "the same step launched call by call (whale_fusion_forward per step)"}
        launch = "captured CUDA graph of whale_fusion_forward, replayed once per step"
        del g
    value = world * w.batch / (ms / 1e3)

    # ---------------- every kernel of one step, live: the library's per-kernel events -------------
    # (one extra step after the timed region; the events serialise launches, so each kernel's time
    # is its own, and their sum is a little above the step time measured above)
    Wb.whale_profile_begin(4096)
    Hn.run_forward(p, stream)
    recs = Wb.whale_profile_end()
    kern = {}
    for name, kms in recs:
        e = kern.setdefault(kernel_name(name), [0, 0.0])
        e[0] += 1
        e[1] += kms
    kern_total = sum(v[1] for v in kern.values()) or 1.0
    kernels = {n: {"launches": c, "avg_ms": tt / c, "share": tt / kern_total}
               for n, (c, tt) in sorted(kern.items(), key=lambda x: -x[1][1])}

    # ---------------- per-kernel timing of the heavy steps (same stream, CUDA events) ------
    work = step_work(w, total_L, args.shared_kv, args.tied_gate, absorbed)
    Hn_ws = p.workspace
    kv = torch.empty(total_L, (1 if args.shared_kv else 2) * w.d, dtype=torch.bfloat16, device="cuda")
    q = torch.empty(w.batch * w.n_tokens, w.d, dtype=torch.bfloat16, device="cuda")
    a = torch.empty_like(q)
    reps = max(args.steps, 3)

    def timed_per_layer(fn, n):
        for l in range(min(2, w.n_layers)):
            fn(l)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        cnt = 0
        for _ in range(n):
            for l in range(w.n_layers):
                fn(l)
                cnt += 1
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / cnt

    def kv_step(l):
        Wb.whale_project_kv(p.cfg, total_L, p.states[l], raw_weights[l]["g_kv"], raw_weights[l]["w_kv"], kv, Hn_ws,
                            stream=stream)

    def attn_step(l):
        Wb.whale_cross_attention(p.cfg, q, kv, p.offsets_t, a, p.hint, Hn_ws, stream=stream)

    def absorbed_step(l):  # the forward's own S2 + S3 call sequence, prepared weights as loaded
        Wb.whale_attend_states(p.cfg, q, p.states[l], p.offsets_t, p.weights[l], a, p.hint, Hn_ws, stream=stream)

    raw_cfg = Hn.config_of(w)
    Wb.whale_project_queries(raw_cfg, q.shape[0], p.tokens, raw_weights[0]["g_q"], raw_weights[0]["w_q"], q, Hn_ws,
                             stream=stream)
    peaks, peak_src = load_peaks()
    layer_ms = ms / w.n_layers
    t_kv = t_attn = t_abs = None
    if absorbed:
        torch.cuda.synchronize()
        t_abs = timed_per_layer(absorbed_step, reps)
        abs_traffic = None
        passa_traffic_known = w.d == 512 and not args.shared_kv
        if passa_traffic_known and ABS_TRAFFIC_BYTES_PER_ROW_D512 is not None:
            abs_traffic = ABS_TRAFFIC_BYTES_PER_ROW_D512 * total_L
        call = {"entry_point": "whale_attend_states (qa GEMM, pass A, pass B, merge, W_V GEMM, unit starts)",
                **roofline_of(work["attention_absorbed"]["flops"], work["attention_absorbed"]["bytes"], t_abs,
                              tensor_peak(peaks, clocks)[0], peaks["hbm_gbs"]), "avg_call_ms": t_abs,
                "algorithmic_flops": work["attention_absorbed"]["flops"],
                "algorithmic_bytes": work["attention_absorbed"]["bytes"], "traffic": abs_traffic,
                "traffic_source": "ncu dram bytes of the six kernels of one call at the full batch, per row"}
        pa = next((v for k, v in kernels.items() if k.split("<")[0] == "abs_scores_kernel"), None)
        tc_peak, tc_src = tensor_peak(peaks, clocks)
        if pa:
            # the dominant kernel, pass A: S = qa H^T of N*h queries against every history row
            # (2 (N h) d FLOP per row) with the softmax, reading the states once (2 d bytes per row);
            # its ncu DRAM bytes per row scaled by rows
            fa = 2.0 * w.n_tokens * w.n_heads * total_L * w.d
            ba = 2.0 * total_L * w.d
            ta = pa["avg_ms"]
            a_traffic = (ABS_PASSA_BYTES_PER_ROW_D512 * total_L
                         if passa_traffic_known and ABS_PASSA_BYTES_PER_ROW_D512 is not None else None)
            roof = {"kernel": "abs_scores_kernel (absorbed pass A: scores on tcgen05 2-SM, online softmax, weights)",
                    **roofline_of(fa, ba, ta, tc_peak, peaks["hbm_gbs"]), "traffic": a_traffic,
                    "traffic_source": "ncu dram bytes of one launch at the full batch, per row",
                    "algorithmic_flops_per_launch": fa, "algorithmic_bytes_per_launch": ba,
                    "avg_launch_ms": ta, "timing": "library per-kernel events on the bench stream",
                    "peak_source": f"{peak_src}: {tc_src}; HBM copy {peaks['hbm_gbs']} GB/s", "call": call}
        else:
            roof = {"kernel": "whale_attend_states (the absorbed S2 + S3 call)",
                    **roofline_of(work["attention_absorbed"]["flops"], work["attention_absorbed"]["bytes"], t_abs,
                                  tc_peak, peaks["hbm_gbs"]), "traffic": abs_traffic,
                    "algorithmic_flops_per_launch": work["attention_absorbed"]["flops"], "avg_launch_ms": t_abs,
                    "peak_source": f"{peak_src}: {tc_src}", "call": call}
    else:
        kv_step(0)
        torch.cuda.synchronize()
        t_kv = timed_per_layer(kv_step, reps)
        t_attn = timed_per_layer(attn_step, reps)
        share_kv, share_attn = t_kv / layer_ms, t_attn / layer_ms
        kv_traffic = None
        if w.d == 512 and not args.shared_kv:
            kv_traffic = KV_TRAFFIC_BYTES_PER_ROW_D512 * total_L
    if absorbed:
        pass
    elif share_kv >= share_attn:
        tc_peak, tc_src = tensor_peak(peaks, clocks)
        roof = {"kernel": "K|V projection GEMM (tcgen05, RMSNorm row factor fused)",
                **roofline_of(work["kv_proj"]["flops"], work["kv_proj"]["bytes"], t_kv, tc_peak, peaks["hbm_gbs"]),
                "traffic": kv_traffic, "traffic_source": "ncu dram bytes of one launch on 109605 rows, scaled by rows",
                "algorithmic_flops_per_launch": work["kv_proj"]["flops"],
                "algorithmic_bytes_per_launch": work["kv_proj"]["bytes"], "avg_launch_ms": t_kv,
                "peak_source": f"{peak_src}: {tc_src}; HBM copy {peaks['hbm_gbs']} GB/s"}
    elif w.n_tokens >= 128:
        # many queries per history (the serving shape): the query-tiled tensor-core attention is
        # bound by its softmax exponentials. Peak = MUFU ex2 throughput: 16 per clock per SM x SMs x
        # the maximum SM clock (nominal unit counts; sm_max_mhz is the measured maximum clock).
        n_exp = float(w.n_heads) * w.n_tokens * total_L   # every query of an example against its rows
        exp_peak = 16.0 * 148 * peaks.get("sm_max_mhz", 1965.0) * 1e6
        exps = n_exp / (t_attn * 1e-3)
        roof = {"kernel": "query-tiled attention (tcgen05 S and P V, softmax on MUFU + FMA polynomial)",
                "bound": "alu", "achieved": exps / 1e12, "peak": exp_peak / 1e12, "unit": "Texp/s",
                "frac": exps / exp_peak, "traffic": None, "algorithmic_per_launch": n_exp, "avg_launch_ms": t_attn,
                "peak_source": "16 ex2/clk/SM x 148 SMs x max SM clock (nominal unit counts)",
                "tensor_tflops": work["attention"]["flops"] / (t_attn * 1e-3) / 1e12}
    else:
        tc_peak, tc_src = tensor_peak(peaks, clocks)
        roof = {"kernel": "split-L cross-attention + combine",
                **roofline_of(work["attention"]["flops"], work["attention"]["bytes"], t_attn, tc_peak,
                              peaks["hbm_gbs"]), "traffic": None,
                "algorithmic_flops_per_launch": work["attention"]["flops"],
                "algorithmic_bytes_per_launch": work["attention"]["bytes"], "avg_launch_ms": t_attn,
                "peak_source": f"{peak_src}: HBM copy {peaks['hbm_gbs']} GB/s; {tc_src}"}
    # roofline of the whole step: sum over kernels of max(flops / TC peak, bytes / HBM peak)
    t_star = 0.0
    tc_step = tensor_peak(peaks, clocks)[0]
    for k, v in work.items():
        t_star += max(v["flops"] / (tc_step * 1e12), v["bytes"] / (peaks["hbm_gbs"] * 1e9))
    t_star *= w.n_layers * 1e3

    # ---------------- backward pass of one layer (the training path), device-resident ----------------
    bwd = None
    if not args.no_backward:
        bwd = time_backward(p, raw_weights, w, total_L, peaks, clocks, stream, reps=max(3, min(args.steps, 20)))
        if isinstance(bwd, dict) and "stack" in bwd:
            tr = ms + bwd["stack"]["ms"]  # one forward (the timed step) and the stack's backward
            bwd["training_step"] = {"ms": tr, "examples_per_s": world * w.batch / (tr / 1e3),
                                    "what": "forward step + whale_fusion_backward, per rank"}

    # ---------------- end to end: host buffers through the C ABI, copies inside the timed region -----
    e2e = None
    if args.e2e_steps > 0:
        hs = p.states.cpu().pin_memory()
        ht = p.tokens.cpu().pin_memory()
        ho = torch.empty_like(ht).pin_memory()
        hoff = torch.from_numpy(p.offsets).pin_memory()
        hws = torch.empty(Wb.whale_host_workspace_size(p.cfg, p.hint), dtype=torch.uint8, device="cuda")
        del p.workspace
        Wb.whale_fusion_forward_host(p.cfg, ht, hs, hoff, p.weights, ho, p.hint, hws, stream=stream)
        torch.cuda.synchronize()
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.e2e_steps):
            Wb.whale_fusion_forward_host(p.cfg, ht, hs, hoff, p.weights, ho, p.hint, hws, stream=stream)
        e1.record(stream)
        torch.cuda.synchronize()
        e_ms = max_over_ranks(e0.elapsed_time(e1) / args.e2e_steps, world)
        h2d = hs.numel() * hs.element_size() + ht.numel() * ht.element_size() + hoff.numel() * 4
        d2h = ho.numel() * ho.element_size()
        e2e = {"value": world * w.batch / (e_ms / 1e3), "unit": "examples/s", "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(d2h), "ms_per_step": e_ms}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = oracle_sample(w, budget_s=args.ref_budget)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "examples/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1) states and tokens, Xavier weights)",
            "config": workload_config(w, total_L, int(p.lengths.max()), world, args),
            "roofline": roof,
            "step_roofline": {"t_star_ms": t_star, "frac": t_star / ms, "per_layer_ms": layer_ms,
                              "path": "absorbed" if absorbed else "materialized K|V",
                              "kv_proj_ms": t_kv, "attention_ms": t_attn, "absorbed_attention_ms": t_abs,
                              "peaks": f"{peak_src}: {peaks['hbm_gbs']} GB/s, {tc_step} TFLOP/s"},
            "kernels": kernels,
            "launch": launch,
            "stream_launch": stream_launch,
            "backward": bwd,
            "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": (len(recs) or launches_per_step(w, args.fold_per_call, absorbed)) * args.steps,
            "clocks": clocks,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
