"""The bounded device-side wait of the tensor-core kernels, made to expire on purpose.

The wait primitive of every tcgen05 kernel gives up after a cycle limit, records DG_ERR_TIMEOUT in
the caller's status word, frees the kernel's tensor memory and returns.  dg_debug_wait_probe runs
that primitive alone, holding tensor memory, on an mbarrier phase that nothing completes (no copy
or MMA is ever issued, so expiry leaves nothing in flight).  The test makes the wait run out with
a short limit, reads DG_ERR_TIMEOUT, then checks that the context is still usable: a probe whose
phase does complete reports DG_OK, and a tensor-core LM-head call right after matches the
oracle."""
import numpy as np
import pytest
import torch

import synth
from oracle import dg_oracle as O
from block_discrete_diffusion_dg_b200 import binding as B
from harness import oracle_model

pytestmark = pytest.mark.gpu


def test_bounded_wait_expires_then_the_device_keeps_working():
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    for limit in (1, 200000):                        # ~0 and ~100 us at 2 GHz
        B.dg_clear_status(st)
        B.dg_debug_wait_probe(limit, False, st)
        assert B.dg_read_status(st) == B.DG_ERR_TIMEOUT
    B.dg_clear_status(st)
    B.dg_debug_wait_probe(200000, True, st)           # the phase completes: no timeout
    assert B.dg_read_status(st) == B.DG_OK
    # first error wins: a later timeout does not overwrite an earlier code
    st.fill_(B.DG_ERR_NUMERIC)
    B.dg_debug_wait_probe(1, False, st)
    assert B.dg_read_status(st) == B.DG_ERR_NUMERIC
    # the context is usable: a tensor-core LM head right after matches the oracle
    c = synth.reduced("layer")
    model = synth.make_model(c, "cpu", seed=3)
    g = torch.Generator().manual_seed(4)
    h = torch.randn((40, c.d_model), generator=g) * 0.07
    dgc = B.make_config(c)
    ent = torch.zeros(40, device="cuda")
    am = torch.zeros(40, dtype=torch.int32, device="cuda")
    st.zero_()
    B.dg_logits_entropy(dgc, 40, None, h.cuda(), None, model["emb"].cuda(), ent, am, None,
                        B.alloc_workspace(dgc, 1, 40, 0), st)
    assert B.dg_read_status(st) == B.DG_OK
    H, oam, margin, _ = O.lm_head_rows(c, oracle_model(c, model), h.double().numpy())
    np.testing.assert_allclose(ent.cpu().numpy(), H, rtol=1e-3)
    safe = margin > 4e-2
    assert (am.cpu().numpy()[safe] == oam[safe]).all()


def test_wait_probe_rejects_bad_limits():
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    n0 = B.dg_launch_count()
    for limit in (0, -5, 4000000001):
        with pytest.raises(B.DgError):
            B.dg_debug_wait_probe(limit, False, st)
    assert B.dg_launch_count() == n0
