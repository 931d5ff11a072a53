"""The allocation-free attention entry point (whale_cross_attention_noalloc).

Some callers cannot allocate device memory or pass a workspace — for example code inside a host
framework that owns all device memory through its own allocator, or a serving loop that must not
call cudaMalloc. For them the library keeps the attention partials in one fixed device array.
This file checks, through the C ABI, that two calls in a row give the same result as the
workspace entry point (within the parity tolerance), and that a shape whose partials do not fit
the fixed array is rejected before any GPU work. It is collected last on purpose, and passes
both alone in a fresh process and after the other tests."""
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


@pytest.mark.parametrize("N,d,h,lengths", [(32, 512, 8, [5, 3000, 1, 777, 6000]), (16, 128, 4, [0, 64, 2500, 129])])
def test_noalloc_matches_workspace_entry_point_on_two_calls(N, d, h, lengths):
    rng = np.random.default_rng(2024 + d)
    L = np.array(lengths, dtype=np.int64)
    off = I.offsets_of(L)
    B, total = len(L), int(off[-1])
    q = _bf16(bf16_randn(rng, B * N, d))
    kv = _bf16(bf16_randn(rng, total, 2 * d))
    offs = torch.from_numpy(off).cuda()
    cfg = W.make_config(1, d, h, N, 4 * d, 2 * d, W.WHALE_BF16)
    hint = W.make_hint(B, int(L.max()), total)
    ws = torch.empty(W.whale_workspace_size(cfg, hint), dtype=torch.uint8, device="cuda")
    ref = torch.empty(B * N, d, dtype=torch.bfloat16, device="cuda")
    W.whale_cross_attention(cfg, q, kv, offs, ref, hint, ws)
    torch.cuda.synchronize()
    r = ref.float()
    for _ in range(2):
        a = torch.full((B * N, d), float("nan"), dtype=torch.bfloat16, device="cuda")
        W.whale_cross_attention_noalloc(cfg, q, kv, offs, a, hint)
        torch.cuda.synchronize()
        err = (a.float() - r).abs()
        assert torch.isfinite(a.float()).all()
        assert bool((err <= BF16_TOL * (1 + r.abs())).all()), float(err.max())


def test_noalloc_rejects_shapes_beyond_the_fixed_scratch():
    # 2048 examples x 64 queries x 8 heads of partials exceed 32 MiB: rejected, no GPU work.
    cfg = W.make_config(1, 512, 8, 64, 2048, 1024, W.WHALE_BF16)
    hint = W.make_hint(2048, 100, 2048 * 100)
    fake = 1 << 20
    assert W.whale_cross_attention_noalloc(cfg, fake, fake, fake, fake, hint, raw=True) == 4
