"""The C ABI from plain C: a C99 program that includes include/whale_fusion.h, links
libwhale_fusion.so and calls the entry points that return before any CUDA call (status strings,
workspace sizes, host-side argument checks). It also prints the header's struct sizes and field
offsets, which must equal the ctypes layouts of the Python binding (the binding passes these structs
by pointer, so a mismatch would shift every field after it). No GPU is needed."""
import ctypes
import os
import shutil
import subprocess

import pytest

from wukong_hstu_cross_b200 import build

build.build()
from wukong_hstu_cross_b200 import whale as W  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "wukong_hstu_cross_b200")

PROGRAM = r"""
#include <stddef.h>
#include <stdio.h>
#include "whale_fusion.h"

#define FIELD(T, f) printf(#T "." #f " %zu\n", offsetof(T, f))

int main(void) {
  printf("sizeof whale_config %zu\n", sizeof(whale_config));
  printf("sizeof whale_layer_weights %zu\n", sizeof(whale_layer_weights));
  printf("sizeof whale_layer_grads %zu\n", sizeof(whale_layer_grads));
  printf("sizeof whale_shape_hint %zu\n", sizeof(whale_shape_hint));
  printf("sizeof whale_kernel_time %zu\n", sizeof(whale_kernel_time));
  FIELD(whale_config, dtype);
  FIELD(whale_config, flags);
  FIELD(whale_config, eps);
  FIELD(whale_layer_weights, w_down);
  FIELD(whale_layer_weights, w_kabs);
  FIELD(whale_layer_grads, w_down);
  FIELD(whale_shape_hint, total_L);
  FIELD(whale_kernel_time, ms);
  for (int s = 0; s <= 5; ++s) printf("status %d %s\n", s, whale_status_string((whale_status)s));

  /* the 2-layer d = 128 stack of 16 tokens, 4 heads */
  whale_config cfg = {2, 128, 4, 16, 512, 256, WHALE_BF16, 0u, 1e-6f};
  whale_shape_hint hint = {8, 3000, 8 * 3000};
  size_t ws = whale_workspace_size(&cfg, &hint);
  printf("workspace %zu\n", ws);
  whale_config bad = cfg;
  bad.n_heads = 3; /* d % n_heads != 0 */
  printf("workspace_bad %zu\n", whale_workspace_size(&bad, &hint));
  printf("backward_workspace %zu\n", whale_backward_workspace_size(&cfg, &hint));

  /* host-side checks: each call returns before any CUDA call */
  whale_layer_weights lw[2] = {{0}};
  void* fake_ws = (void*)(size_t)(1u << 20); /* aligned, never dereferenced: the checks fail first */
  printf("no_workspace %d\n", (int)whale_fusion_forward(&cfg, NULL, NULL, NULL, lw, NULL, &hint, NULL, ws, NULL));
  printf("null_tokens %d\n", (int)whale_fusion_forward(&cfg, NULL, NULL, NULL, lw, NULL, &hint, fake_ws, ws, NULL));
  printf("null_config %d\n", (int)whale_fusion_forward(NULL, NULL, NULL, NULL, lw, NULL, &hint, fake_ws, ws, NULL));
  printf("wait_limit %d\n", (int)whale_test_bounded_waits(999ull, NULL));
  return 0;
}
"""


def _compile_and_run(tmp_path):
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "consumer.c"
    exe = tmp_path / "consumer"
    src.write_text(PROGRAM)
    subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"), str(src),
                    "-L", PKG, "-lwhale_fusion", f"-Wl,-rpath,{PKG}", "-o", str(exe)], check=True,
                   capture_output=True, text=True)
    res = subprocess.run([str(exe)], check=True, capture_output=True, text=True, timeout=120)
    out = {}
    for line in res.stdout.splitlines():
        if line.startswith("status "):
            _, code, text = line.split(" ", 2)
            out[f"status {code}"] = text
        else:
            key, _, val = line.rpartition(" ")
            out[key] = val
    return out


def test_header_compiles_as_c_and_matches_the_binding(tmp_path):
    out = _compile_and_run(tmp_path)
    sizes = {"whale_config": W.whale_config, "whale_layer_weights": W.whale_layer_weights,
             "whale_layer_grads": W.whale_layer_grads, "whale_shape_hint": W.whale_shape_hint,
             "whale_kernel_time": W.whale_kernel_time}
    for name, cls in sizes.items():
        assert int(out[f"sizeof {name}"]) == ctypes.sizeof(cls), name
    for key in ("whale_config.dtype", "whale_config.flags", "whale_config.eps", "whale_layer_weights.w_down",
                "whale_layer_weights.w_kabs", "whale_layer_grads.w_down", "whale_shape_hint.total_L",
                "whale_kernel_time.ms"):
        struct, field = key.split(".")
        assert int(out[key]) == getattr(sizes[struct], field).offset, key
    # the same results through C as through the binding
    cfg = W.make_config(2, 128, 4, 16, 512, 256, W.WHALE_BF16, 0, 1e-6)
    hint = W.make_hint(8, 3000, 8 * 3000)
    assert int(out["workspace"]) == W.whale_workspace_size(cfg, hint) > 0
    assert int(out["backward_workspace"]) == W.whale_backward_workspace_size(cfg, hint) > 0
    assert int(out["workspace_bad"]) == 0
    assert int(out["no_workspace"]) == 4      # WHALE_ERR_WORKSPACE
    assert int(out["null_tokens"]) == 1 and int(out["null_config"]) == 1 and int(out["wait_limit"]) == 1


def test_status_strings_through_c(tmp_path):
    out = _compile_and_run(tmp_path)
    for s in range(6):
        assert out[f"status {s}"] == W.whale_status_string(s), s
