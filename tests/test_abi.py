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
    assert L.dg_eb_select(0, 16, None, None, 1.0, 16, None, None, None, None, None, None, None, None) \
        == B.DG_ERR_INVALID_ARG
    assert L.dg_eb_select(1, 2048, 8, 8, 1.0, 16, 8, 8, None, 8, 8, 8, None, None) == B.DG_ERR_INVALID_ARG
    assert L.dg_eb_select(1, 16, 8, 8, -1.0, 16, 8, 8, None, 8, 8, 8, None, None) == B.DG_ERR_INVALID_ARG
    assert L.dg_eb_select(1, 16, 8, 8, math.nan, 16, 8, 8, None, 8, 8, 8, None, None) == B.DG_ERR_INVALID_ARG
    assert L.dg_eb_select(1, 16, 8, 8, 1.0, 16, None, 8, None, 8, 8, 8, None, None) == B.DG_ERR_INVALID_ARG
    # workspace too small / misaligned
    assert L.dg_moe_route(ctypes.byref(cfg), 16, 8, 8, None, 8, 8, 8, 8, 8, 256, 16, None, None) \
        == B.DG_ERR_WORKSPACE
    assert L.dg_moe_route(ctypes.byref(cfg), 16, 8, 8, None, 8, 8, 8, 8, 8, 257, 1 << 30, None, None) \
        == B.DG_ERR_INVALID_ARG
    # model with a null layer pointer
    assert L.dg_canvas_step(ctypes.byref(cfg), None, 1, 8, 8, 8, 8, 8, 16, 0.1, 8, 8, 8, 64, None,
                            None, None, None, None, 256, 1 << 30, None, None) == B.DG_ERR_INVALID_ARG
    assert L.dg_launch_count() == n0


def test_binding_refuses_host_tensors():
    import torch
    with pytest.raises(ValueError):
        B._p(torch.zeros(4))
