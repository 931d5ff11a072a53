"""Shared helpers of the GPU parity tests (comparison against the fp64 oracle)."""
import numpy as np

from wukong_hstu_cross_b200 import inputs as I

BF16_TOL = 2e-2   # max |gpu - oracle| <= 2e-2 * (1 + |oracle|) in bf16 mode
FP32_TOL = 1e-4   # max |gpu - oracle| <= 1e-4 in fp32 mode


def to_np(t) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def assert_parity(gpu, ref, dtype: str, rms_rel: float | None = None, what: str = ""):
    g = to_np(gpu) if not isinstance(gpu, np.ndarray) else gpu.astype(np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert g.shape == ref.shape, (g.shape, ref.shape)
    assert np.all(np.isfinite(g)), f"{what}: non-finite GPU output"
    err = np.abs(g - ref)
    if dtype == "bf16":
        bound = BF16_TOL * (1.0 + np.abs(ref))
    else:
        bound = np.full_like(ref, FP32_TOL)
    excess = err - bound
    if excess.size and excess.max() > 0:
        i = np.unravel_index(np.argmax(excess), excess.shape)
        raise AssertionError(f"{what}: |gpu-oracle| {err[i]:.3e} > bound {bound[i]:.3e} at {i} "
                             f"(gpu {g[i]:.6f}, oracle {ref[i]:.6f}); {int((excess > 0).sum())} elements out")
    if rms_rel is not None and ref.size:
        rel = np.sqrt(np.mean(err ** 2)) / max(np.sqrt(np.mean(ref ** 2)), 1e-30)
        assert rel <= rms_rel, f"{what}: relative RMS error {rel:.3e} > {rms_rel}"


def bf16_randn(rng, *shape, scale=1.0) -> np.ndarray:
    return I.bf16_round((rng.standard_normal(shape) * scale).astype(np.float32))
