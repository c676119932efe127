"""C-ABI library checks that need no GPU: it loads, exports every entry point that include/dg.h
declares, sizes scratch sensibly, and rejects bad arguments on the host before any launch."""
import ctypes
import math
import os
import re
import subprocess

import pytest

import synth
from block_discrete_diffusion_dg_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    from block_discrete_diffusion_dg_b200 import build
    build.build()


def _header_functions():
    with open(os.path.join(ROOT, "include", "dg.h")) as fh:
        src = fh.read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(dg_[a-z_0-9]+)\s*\(", src)))


def test_header_functions_are_exported():
    names = _header_functions()
    assert "dg_canvas_step" in names and "dg_eb_select" in names and len(names) >= 12
    out = subprocess.run(["nm", "-D", "--defined-only", B.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\s[TW]\s+(dg_\w+)", out))
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    L = B.lib()
    for n in names:
        assert hasattr(L, n)
    assert set(B.exported_symbols()) <= set(names)


def test_workspace_size_scales_and_rejects():
    cfg = B.make_config(synth.get_config("layer"))
    a = B.dg_workspace_size(cfg, 1, 256, 4352)
    b = B.dg_workspace_size(cfg, 2, 256, 4352)
    assert a > 0 and b > a and a % 256 == 0
    bad = B.make_config(synth.get_config("layer"))
    bad.head_dim = 96
    assert B.dg_workspace_size(bad, 1, 256, 4352) == 0
    bad = B.make_config(synth.get_config("layer"))
    bad.act_dtype, bad.w_dtype = B.DG_F32, B.DG_E4M3
    assert B.dg_workspace_size(bad, 1, 256, 4352) == 0
    assert B.dg_workspace_size(cfg, 0, 256, 4352) == 0


def test_host_side_argument_rejection_launches_nothing():
    L = B.lib()
    n0 = L.dg_launch_count()
    cfg = B.make_config(synth.get_config("tiny"))
    # batch 0, canvas > 1024, negative gamma, NaN gamma, null state: all rejected before launch
    assert L.dg_eb_select(0, 16, None, None, 1.0, 16, None, None, None, None, None, None, 0, None, None) \
        == B.DG_ERR_INVALID_ARG
    assert L.dg_eb_select(1, 2048, 8, 8, 1.0, 16, 8, 8, None, 8, 8, 8, 0, None, None) == B.DG_ERR_INVALID_ARG
    assert L.dg_eb_select(1, 16, 8, 8, -1.0, 16, 8, 8, None, 8, 8, 8, 0, None, None) == B.DG_ERR_INVALID_ARG
    assert L.dg_eb_select(1, 16, 8, 8, math.nan, 16, 8, 8, None, 8, 8, 8, 0, None, None) == B.DG_ERR_INVALID_ARG
    assert L.dg_eb_select(1, 16, 8, 8, 1.0, 16, None, 8, None, 8, 8, 8, 0, None, None) == B.DG_ERR_INVALID_ARG
    # workspace too small / misaligned
    assert L.dg_moe_route(ctypes.byref(cfg), 16, 8, 8, None, 8, 8, 8, 8, 8, 256, 16, None, None) \
        == B.DG_ERR_WORKSPACE
    assert L.dg_moe_route(ctypes.byref(cfg), 16, 8, 8, None, 8, 8, 8, 8, 8, 257, 1 << 30, None, None) \
        == B.DG_ERR_INVALID_ARG
    # model with a null layer pointer
    assert L.dg_canvas_step(ctypes.byref(cfg), None, 1, 8, 8, 8, 8, 8, 16, 0.1, 8, 8, 8, 64, None,
                            None, None, None, None, 256, 1 << 30, None, None) == B.DG_ERR_INVALID_ARG
    assert L.dg_launch_count() == n0


def test_new_config_fields_and_entry_points_reject_on_the_host():
    """NVFP4 LM head, shared experts and dg_generate: invalid configurations and arguments are
    refused before any launch (no GPU needed)."""
    L = B.lib()
    n0 = L.dg_launch_count()
    # NVFP4 needs bf16 activations and d_model a multiple of 256 (at most 4096)
    ok = B.make_config(synth.reduced("layer_nvfp4"))
    assert B.dg_workspace_size(ok, 1, 64, 256) > 0
    bad = B.make_config(synth.reduced("layer_nvfp4"))
    bad.d_model = 320
    assert B.dg_workspace_size(bad, 1, 64, 256) == 0
    bad = B.make_config(synth.get_config("layer_nvfp4"))
    bad.d_model = 8192
    assert B.dg_workspace_size(bad, 1, 64, 256) == 0
    bad = B.make_config(synth.get_config("tiny"))
    bad.emb_dtype = B.DG_NVFP4
    assert B.dg_workspace_size(bad, 1, 16, 64) == 0
    # the bf16 LM-head entry point refuses an NVFP4 config; the NVFP4 one a bf16 config and a
    # non-positive tensor scale
    assert L.dg_logits_entropy(ctypes.byref(ok), 4, None, 8, None, 8, 8, 8, None, 256, 1 << 30,
                               None, None) == B.DG_ERR_INVALID_ARG
    bf = B.make_config(synth.reduced("layer"))
    assert L.dg_logits_entropy_nvfp4(ctypes.byref(bf), 4, None, 8, None, 16, 16, 1.0, 8, 8, None,
                                     256, 1 << 30, None, None) == B.DG_ERR_INVALID_ARG
    assert L.dg_logits_entropy_nvfp4(ctypes.byref(ok), 4, None, 8, None, 16, 16, 0.0, 8, 8, None,
                                     256, 1 << 30, None, None) == B.DG_ERR_INVALID_ARG
    # shared experts: n_shared >= 0, E + S <= 256, k + S <= 32; the scratch grows with them
    sh = B.make_config(synth.reduced("layer", n_shared=1))
    base = B.make_config(synth.reduced("layer"))
    assert B.dg_workspace_size(sh, 1, 64, 256) > B.dg_workspace_size(base, 1, 64, 256)
    for field, val in (("n_shared", -1), ("n_shared", 241)):
        bad = B.make_config(synth.reduced("layer"))
        setattr(bad, field, val)
        assert B.dg_workspace_size(bad, 1, 64, 256) == 0
    bad = B.make_config(synth.reduced("layer"))
    bad.top_k, bad.n_shared = 16, 17
    assert B.dg_workspace_size(bad, 1, 64, 256) == 0
    # dg_generate: no model, zero max_steps, negative gamma, append without a cache (a model
    # struct of placeholder pointers passes the null checks; nothing is dereferenced on the host)
    cfg = B.make_config(synth.get_config("tiny"))
    lw = (B.DgLayerWeights * 1)(B.DgLayerWeights(8, None, 8, None, 8, 8, None, 8, None))
    model = B.DgModel(ctypes.cast(lw, ctypes.POINTER(B.DgLayerWeights)), 8, None, 1.0)
    # tokens, masked, n_masked, done, step, max_steps, gamma, sampler, k, v, cache_len,
    # cache_cap, append, ws, ws_bytes, dev_status, stream
    args = [8, 8, 8, 8, 8, 16, 0.1, None, 8, 8, 8, 64, 0, 256, 1 << 30, None, None]
    assert L.dg_generate(ctypes.byref(cfg), None, 1, *args) == B.DG_ERR_INVALID_ARG
    bad_smp = B.make_sampler(math.nan)
    for i, v in ((5, 0), (6, -1.0), (6, math.nan), (7, ctypes.byref(bad_smp))):
        a2 = list(args)
        a2[i] = v
        assert L.dg_generate(ctypes.byref(cfg), ctypes.byref(model), 1, *a2) == B.DG_ERR_INVALID_ARG
    a2 = list(args)
    a2[11], a2[12] = 0, 1          # append with no cache
    assert L.dg_generate(ctypes.byref(cfg), ctypes.byref(model), 1, *a2) == B.DG_ERR_INVALID_ARG
    a2 = list(args)
    a2[13] = 257                   # misaligned scratch
    assert L.dg_generate(ctypes.byref(cfg), ctypes.byref(model), 1, *a2) == B.DG_ERR_INVALID_ARG
    assert L.dg_launch_count() == n0


def test_sampler_entry_points_reject_on_the_host():
    """dg_noise_canvas, dg_canvas_step_sampler and dg_ar_step refuse bad arguments before any
    launch: empty or oversized canvases, a missing or non-finite sampler, missing outputs."""
    L = B.lib()
    n0 = L.dg_launch_count()
    assert L.dg_noise_canvas(0, 16, 512, 1, 8, 8, 8, 8, 8, None) == B.DG_ERR_INVALID_ARG
    assert L.dg_noise_canvas(1, 2048, 512, 1, 8, 8, 8, 8, 8, None) == B.DG_ERR_INVALID_ARG
    assert L.dg_noise_canvas(1, 16, 512, 1, None, 8, 8, 8, 8, None) == B.DG_ERR_INVALID_ARG
    cfg = B.make_config(synth.get_config("tiny"))
    lw = (B.DgLayerWeights * 1)(B.DgLayerWeights(8, None, 8, None, 8, 8, None, 8, None))
    model = B.DgModel(ctypes.cast(lw, ctypes.POINTER(B.DgLayerWeights)), 8, None, 1.0)
    good, nan_smp = B.make_sampler(1.0, 0.5, 3), B.make_sampler(1.0, math.inf, 3)
    # tokens, masked, n_masked, done, step, max_steps, gamma, sampler, k, v, cache_len, cap,
    # entropy, argmax, logits, forced, ws, ws_bytes, dev_status, stream
    args = [8, 8, 8, 8, 8, 16, 0.1, ctypes.byref(good), 8, 8, 8, 64, None, None, None, None, 257,
            1 << 30, None, None]
    assert L.dg_canvas_step_sampler(ctypes.byref(cfg), ctypes.byref(model), 1, *args) \
        == B.DG_ERR_INVALID_ARG                     # misaligned scratch
    for i, v in ((7, None), (7, ctypes.byref(nan_smp))):
        a2 = list(args)
        a2[i], a2[16] = v, 256
        assert L.dg_canvas_step_sampler(ctypes.byref(cfg), ctypes.byref(model), 1, *a2) \
            == B.DG_ERR_INVALID_ARG
    # tokens, n_tokens, k, v, cache_len, cap, sampler, next, entropy, logits, forced, ws, ws_bytes,
    # dev_status, stream
    ar = [8, 1, 8, 8, 8, 64, None, 8, None, None, None, 256, 1 << 30, None, None]
    for i, v in ((7, None), (1, 0), (6, ctypes.byref(nan_smp))):
        a2 = list(ar)
        a2[i] = v
        assert L.dg_ar_step(ctypes.byref(cfg), ctypes.byref(model), 1, *a2) == B.DG_ERR_INVALID_ARG
    a2 = list(ar)
    a2[1] = 65                      # more tokens than the cache holds
    assert L.dg_ar_step(ctypes.byref(cfg), ctypes.byref(model), 1, *a2) == B.DG_ERR_CAPACITY
    assert L.dg_launch_count() == n0


def test_binding_refuses_host_tensors():
    import torch
    with pytest.raises(ValueError):
        B._p(torch.zeros(4))


def test_header_is_plain_c_and_the_library_links_from_c(tmp_path):
    """include/dg.h compiles as strict C99 and a C program linked against libdg.so calls it: the
    boundary needs no C++ or Python.  Without a GPU the calls only exercise the host-side checks."""
    src = tmp_path / "use_dg.c"
    src.write_text(r'''
#include <stdio.h>
#include "dg.h"
int main(void) {
  dg_config c = {0};                                       /* all zero: not a valid model */
  const size_t ws = dg_workspace_size(&c, 1, 256, 0);
  const int rc = dg_eb_select(0, 0, NULL, NULL, 0.0, 0, NULL, NULL, NULL, NULL, NULL, NULL, 0,
                              NULL, NULL);
  const int rs = dg_logits_entropy_static(NULL, 1, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL);
  printf("%zu %d %d\n", ws, rc, rs);
  return (ws == 0 && rc == DG_ERR_INVALID_ARG && rs == DG_ERR_INVALID_ARG) ? 0 : 1;
}
''')
    exe = tmp_path / "use_dg"
    pkg = os.path.dirname(B.LIB_PATH)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                    "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
                    B.LIB_PATH, "-Wl,-rpath," + pkg], check=True, capture_output=True, text=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, (r.stdout, r.stderr)
