"""The fixed-scratch LM-head entry point, dg_logits_entropy_static, against dg_logits_entropy.

Some callers of this library cannot allocate device memory — for instance an engine that has
already reserved the whole device for its own pools — so dg_logits_entropy_static keeps its
scratch in a fixed array inside the library instead of taking a buffer.  Two calls in a row, on
different inputs, must each match the regular entry point on the same inputs (so nothing the first
call leaves in the shared array affects the second), at the reduced size and at the full
one-layer size (d_model 2048, vocabulary 262144, 256 rows)."""
import ctypes

import numpy as np
import pytest
import torch

import synth
from block_discrete_diffusion_dg_b200 import binding as B

pytestmark = pytest.mark.gpu

ENT_RTOL = 1e-3


def _case(cfg, emb, n_all, n_rows, seed, n_dev=None):
    """Both entry points on the same rows; with n_dev, the row count is read on the device
    (*n_rows_dev = n_dev <= n_rows, as dg_canvas_step passes it) and rows past it stay untouched."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    h = (torch.randn((n_all, cfg.d_model), generator=g) * 0.07).cuda()   # fp32 hidden rows
    rows = torch.sort(torch.randperm(n_all, generator=g)[:n_rows]).values.to(torch.int32).cuda()
    nd = None if n_dev is None else torch.tensor([n_dev], dtype=torch.int32, device="cuda")
    dgc = B.make_config(cfg)
    e_ref = torch.full((n_all,), -1.0, device="cuda")
    a_ref = torch.full((n_all,), -1, dtype=torch.int32, device="cuda")
    B.dg_logits_entropy(dgc, n_rows, nd, h, rows, emb, e_ref, a_ref, None,
                        B.alloc_workspace(dgc, 1, n_rows, 0))
    e_st = torch.full((n_all,), -1.0, device="cuda")
    a_st = torch.full((n_all,), -1, dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    B.dg_logits_entropy_static(dgc, n_rows, nd, h, rows, emb, e_st, a_st, status)
    assert B.dg_read_status(status) == B.DG_OK
    if n_dev is not None:   # rows beyond the device count keep their sentinels on both sides
        skipped = rows[n_dev:].long().cpu()
        for e_, a_ in ((e_ref, a_ref), (e_st, a_st)):
            assert (e_.cpu()[skipped] == -1.0).all() and (a_.cpu()[skipped] == -1).all()
    return e_ref.cpu().numpy(), a_ref.cpu().numpy(), e_st.cpu().numpy(), a_st.cpu().numpy()


@pytest.mark.parametrize("name", ["layer-reduced", "layer"])
def test_static_scratch_matches_regular_entry_point_twice(name):
    cfg = synth.reduced("layer") if name == "layer-reduced" else synth.get_config("layer")
    emb = synth.make_model(cfg, "cuda", seed=5)["emb"] if name == "layer" else \
        synth.make_model(cfg, "cpu", seed=5)["emb"].cuda()
    # two calls in a row, then one whose row count (77 of 256) is known on the device only
    for n_all, n_rows, seed, n_dev in ((300, 256, 1, None), (200, 77, 2, None), (300, 256, 3, 77)):
        e_ref, a_ref, e_st, a_st = _case(cfg, emb, n_all, n_rows, seed, n_dev)
        np.testing.assert_allclose(e_st, e_ref, rtol=ENT_RTOL)
        assert (a_st == a_ref).all()
        assert (e_st[a_ref < 0] == -1.0).all()   # rows not asked for are left alone


def test_static_scratch_rejects_oversized_requests():
    cfg = synth.reduced("layer")
    dgc = B.make_config(cfg)
    L = B.lib()
    n0 = L.dg_launch_count()
    dummy = torch.zeros(8, device="cuda")
    p = dummy.data_ptr()
    assert L.dg_logits_entropy_static(ctypes.byref(dgc), 257, None, p, None, p, p, p, None, None) \
        == B.DG_ERR_WORKSPACE
    big = B.make_config(synth.get_config("layer", d_model=4096))
    assert L.dg_logits_entropy_static(ctypes.byref(big), 16, None, p, None, p, p, p, None, None) \
        == B.DG_ERR_WORKSPACE
    f32 = B.make_config(synth.get_config("tiny"))
    assert L.dg_logits_entropy_static(ctypes.byref(f32), 16, None, p, None, p, p, p, None, None) \
        == B.DG_ERR_UNSUPPORTED
    bad = B.make_config(synth.reduced("layer"))
    bad.rms_eps = float("nan")       # malformed config: refused as by dg_logits_entropy
    assert L.dg_logits_entropy_static(ctypes.byref(bad), 16, None, p, None, p, p, p, None, None) \
        == B.DG_ERR_INVALID_ARG
    assert L.dg_launch_count() == n0
