"""Failure detection on the device, tested without a fault: every wait in the library's kernels is
bounded, and one that runs out records WHALE_DEVERR_TIMEOUT and lets its kernel return. Here the
self-test kernel (whale_test_bounded_waits) waits on an mbarrier that no thread arrives on and on a
flag that no thread sets, each for 1 ms; the host then sees the timeout through
whale_get_device_error, promptly, and the next forward on the same context still meets the parity
bound (the GPU stayed healthy)."""
import time

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


def test_bounded_waits_time_out_report_and_leave_the_context_usable():
    torch.cuda.synchronize()
    assert W.whale_get_device_error() == 0            # nothing recorded before
    for limit_ns in (1_000_000, 20_000):
        t0 = time.perf_counter()
        W.whale_test_bounded_waits(limit_ns)
        code = W.whale_get_device_error()             # synchronises the stream, reads and clears
        dt = time.perf_counter() - t0
        assert code == W.WHALE_DEVERR_TIMEOUT, code
        assert dt < 0.5, dt                           # the kernel gave up after ~limit_ns
        assert W.whale_get_device_error() == 0        # cleared by the read
    # the context is still usable: a small forward on it meets the parity bound
    w = I.WORKLOADS["stack_d128"].replace(batch=3, n_layers=1, lengths=("uniform", 1, 300))
    p = Hn.build_problem(w, gains="random")
    out = Hn.run_forward(p).float().cpu().numpy()
    for b in range(w.batch):
        ref = O.fusion_stack_example(I.tokens_of_example(w, b), Hn.states_of_example_host(p, b), p.host_weights,
                                     w.n_heads, w.eps)
        assert_parity(out[b], ref, "bf16", what=f"example {b}")
    assert W.whale_get_device_error() == 0
