"""The allocation-free attention entry point (whale_cross_attention_noalloc).

Some callers cannot allocate device memory or pass a workspace — for example code inside a host
framework that owns all device memory through its own allocator, or a serving loop that must not
call cudaMalloc. For them the library keeps the attention partials in one fixed device array.
This file checks, through the C ABI, that two calls in a row give the same result as the
workspace entry point (within the parity tolerance) on both attention kernels and in fp32 mode,
and that a shape whose partials do not fit the fixed array is rejected before any GPU work. It is
collected last on purpose, and passes both alone in a fresh process and after the other tests."""
import numpy as np
import pytest
import torch

from tests.gpu_util import BF16_TOL, bf16_randn
from wukong_hstu_cross_b200 import inputs as I

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from wukong_hstu_cross_b200 import build
    build.build()
    from wukong_hstu_cross_b200 import whale as W


def _bf16(a):
    return torch.from_numpy(I.bf16_bits(a).view(np.int16)).view(torch.bfloat16).cuda()


CASES = [
    (32, 512, 8, [5, 3000, 1, 777, 6000], "bf16"),      # split-L kernel, partials in the fixed array
    (16, 128, 4, [0, 64, 2500, 129], "bf16"),
    # 4 x 16384 queries: the query-tiled kernel, no partials (the split-L plan would need ~77 MB)
    (16384, 256, 8, [2000, 1, 0, 777], "bf16"),
    (8, 64, 2, [0, 1, 130, 256], "fp32"),               # fp32 mode: no scratch at all
]


@pytest.mark.parametrize("N,d,h,lengths,dtype", CASES)
def test_noalloc_matches_workspace_entry_point_on_two_calls(N, d, h, lengths, dtype):
    rng = np.random.default_rng(2024 + d + N)
    L = np.array(lengths, dtype=np.int64)
    off = I.offsets_of(L)
    B, total = len(L), int(off[-1])
    if dtype == "bf16":
        q = _bf16(bf16_randn(rng, B * N, d))
        kv = _bf16(bf16_randn(rng, total, 2 * d))
        tdt, tol = torch.bfloat16, BF16_TOL
    else:
        q = torch.from_numpy(rng.standard_normal((B * N, d)).astype(np.float32)).cuda()
        kv = torch.from_numpy(rng.standard_normal((total, 2 * d)).astype(np.float32)).cuda()
        tdt, tol = torch.float32, 1e-5
    offs = torch.from_numpy(off).cuda()
    cfg = W.make_config(1, d, h, N, 4 * d, 2 * d, W.WHALE_BF16 if dtype == "bf16" else W.WHALE_FP32)
    hint = W.make_hint(B, int(L.max()), total)
    ws = torch.empty(max(W.whale_workspace_size(cfg, hint), 256), dtype=torch.uint8, device="cuda")
    ref = torch.empty(B * N, d, dtype=tdt, device="cuda")
    W.whale_cross_attention(cfg, q, kv, offs, ref, hint, ws)
    torch.cuda.synchronize()
    r = ref.float()
    for _ in range(2):
        a = torch.full((B * N, d), float("nan"), dtype=tdt, device="cuda")
        W.whale_cross_attention_noalloc(cfg, q, kv, offs, a, hint)
        torch.cuda.synchronize()
        err = (a.float() - r).abs()
        assert torch.isfinite(a.float()).all()
        assert bool((err <= tol * (1 + r.abs())).all()), float(err.max())


def test_noalloc_rejects_shapes_beyond_the_fixed_scratch():
    # 2048 examples x 64 queries x 8 heads of split-L partials exceed 32 MiB: rejected before any GPU
    # work. The buffers are real device tensors of the right sizes (offsets all zero: every history
    # empty), so even a call that went ahead would only read valid memory.
    B, N, d, total = 2048, 64, 512, 2048 * 100
    cfg = W.make_config(1, d, 8, N, 4 * d, 2 * d, W.WHALE_BF16)
    hint = W.make_hint(B, 100, total)
    q = torch.zeros(B * N, d, dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros(total, 2 * d, dtype=torch.bfloat16, device="cuda")
    offs = torch.zeros(B + 1, dtype=torch.int32, device="cuda")
    a = torch.zeros(B * N, d, dtype=torch.bfloat16, device="cuda")
    assert W.whale_cross_attention_noalloc(cfg, q, kv, offs, a, hint, raw=True) == 4
    torch.cuda.synchronize()
