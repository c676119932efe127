"""GPU parity on the tiny fp32 workload (d_model 64, 8 experts top-2, vocab 512, canvas 16,
prompt 32, gamma 0.1, 16 steps, 2 canvases with a KV append).  Tolerances: logits max-abs 1e-4,
entropies 1e-3 relative; token ids and EB selections bit-exact."""
import math

import numpy as np
import pytest
import torch

import synth
from oracle import dg_oracle as O
from block_discrete_diffusion_dg_b200 import binding as B
from harness import Workload, np_state, torch_state, decode_cache

pytestmark = pytest.mark.gpu

LOGIT_TOL = 1e-4
ENT_RTOL = 1e-3


@pytest.fixture(scope="module")
def wl():
    return Workload(synth.get_config("tiny"), gen_device="cpu")


def _oracle_step(wl, model, st_np):
    cfg = wl.cfg
    kc = decode_cache(cfg, wl.kv["k"])
    vc = decode_cache(cfg, wl.kv["v"])
    cl = synth.to_numpy(wl.kv["cache_len"])
    return O.canvas_step(cfg, model, st_np, kc, vc, cl, cfg.gamma, cfg.max_steps, keep_logits=True)


def test_tiny_step_lockstep(wl):
    cfg = wl.cfg
    model = wl.oracle()
    st_np = np_state(wl.state)
    for s in range(cfg.canvas):
        new_np, info = _oracle_step(wl, model, st_np)
        inf = info[0]
        rows = inf["rows"]
        g_st, ent, am, lg = wl.step(torch_state(st_np), logits=True)
        wl.check_status()
        ent, am, lg = ent.cpu().numpy()[0], am.cpu().numpy()[0], lg.cpu().numpy()
        # logits of every masked row
        diff = np.abs(lg[rows] - inf["logits"]).max()
        assert diff <= LOGIT_TOL, (s, diff)
        # fused argmax == argmax of the GPU's own logits (first index of the max)
        assert (am[rows] == np.argmax(lg[rows], axis=1)).all()
        # tokens equal the oracle's where the oracle's top-2 margin exceeds 2 x tol
        safe = inf["margin"] > 2 * LOGIT_TOL
        assert (am[rows][safe] == inf["argmax"][safe]).all()
        np.testing.assert_allclose(ent[rows], inf["H"], rtol=ENT_RTOL)
        # EB selection bit-exact on the oracle's fp32 entropies
        e_in = torch.zeros((1, cfg.canvas), dtype=torch.float32)
        e_in[0, rows] = torch.from_numpy(inf["H"])
        a_in = torch.zeros((1, cfg.canvas), dtype=torch.int32)
        a_in[0, rows] = torch.from_numpy(inf["argmax"])
        st2 = torch_state(st_np)
        sel = torch.zeros((1, cfg.canvas), dtype=torch.uint8, device="cuda")
        B.dg_eb_select(1, cfg.canvas, e_in.cuda(), a_in.cuda(), cfg.gamma, cfg.max_steps,
                       st2["tokens"], st2["masked"], sel, st2["n_masked"], st2["done"], st2["step"])
        for k in ("tokens", "masked", "n_masked", "done", "step"):
            assert (st2[k].cpu().numpy() == new_np[k]).all(), k
        assert (sel.cpu().numpy()[0].astype(bool) == inf["selected"]).all()
        # the fused step commits the same positions (the oracle's two lowest entropies are apart)
        h_sorted = np.sort(inf["H"])
        if len(h_sorted) < 2 or h_sorted[1] - h_sorted[0] > 1e-5:
            for k in ("masked", "n_masked", "done", "step"):
                assert (g_st[k].cpu().numpy() == new_np[k]).all(), k
        st_np = new_np
        if st_np["done"][0]:
            break
    assert st_np["done"][0] == 1 and st_np["step"][0] == cfg.canvas


def test_tiny_generate_and_append(wl):
    """Two canvases block-autoregressively with the append between them; GPU loop vs oracle."""
    cfg = wl.cfg
    kv0 = {k: v.clone() for k, v in wl.kv.items()}
    model = wl.oracle()
    kc = decode_cache(cfg, kv0["k"])
    vc = decode_cache(cfg, kv0["v"])
    cl = synth.to_numpy(kv0["cache_len"])
    o_tok, o_steps, o_len = O.generate(cfg, model, kc, vc, cl, cfg.n_canvases, cfg.gamma,
                                       cfg.max_steps)
    k_dev, v_dev, len_dev = kv0["k"], kv0["v"], kv0["cache_len"]
    ws = B.alloc_workspace(wl.dgcfg, cfg.batch, cfg.canvas, wl.cap)
    st_ = wl.status
    for c in range(cfg.n_canvases):
        st = torch_state(np_state(synth.make_canvas_state(cfg, "all_mask")))
        steps = 0
        while True:
            B.dg_canvas_step(wl.dgcfg, wl.dgmodel, 1, st["tokens"], st["masked"], st["n_masked"],
                             st["done"], st["step"], cfg.max_steps, cfg.gamma, k_dev, v_dev,
                             len_dev, wl.cap, None, None, None, ws, st_)
            steps += 1
            if int(st["done"].item()):
                break
            assert steps <= cfg.max_steps
        assert steps == o_steps[0, c]
        assert (st["tokens"].cpu().numpy()[0] == o_tok[0, c]).all()
        B.dg_kv_append(wl.dgcfg, wl.dgmodel, 1, st["tokens"], cfg.canvas, k_dev, v_dev, len_dev,
                       wl.cap, ws, st_)
    torch.cuda.synchronize()
    wl.check_status()
    assert int(len_dev.item()) == o_len[0]
    np.testing.assert_allclose(k_dev.cpu().numpy(), kc, atol=1e-5)
    np.testing.assert_allclose(v_dev.cpu().numpy(), vc, atol=1e-5)


def test_tiny_device_generate_matches_oracle(wl):
    """dg_generate (the step loop as one graph with a device-side while condition, then the
    append) over two canvases against the oracle's generation: tokens, step counts, cache."""
    cfg = wl.cfg
    kv0 = {k: v.clone() for k, v in wl.kv.items()}
    model = wl.oracle()
    kc = decode_cache(cfg, kv0["k"])
    vc = decode_cache(cfg, kv0["v"])
    cl = synth.to_numpy(kv0["cache_len"])
    o_tok, o_steps, o_len = O.generate(cfg, model, kc, vc, cl, cfg.n_canvases, cfg.gamma,
                                       cfg.max_steps)
    k_dev, v_dev, len_dev = kv0["k"], kv0["v"], kv0["cache_len"]
    ws = B.alloc_workspace(wl.dgcfg, cfg.batch, cfg.canvas, wl.cap)
    st = torch_state(np_state(synth.make_canvas_state(cfg, "all_mask")))
    for c in range(cfg.n_canvases):
        fresh = torch_state(np_state(synth.make_canvas_state(cfg, "all_mask")))
        for k in st:          # the same state buffers every canvas: the second call reuses the graph
            st[k].copy_(fresh[k])
        B.dg_generate(wl.dgcfg, wl.dgmodel, 1, st["tokens"], st["masked"], st["n_masked"],
                      st["done"], st["step"], cfg.max_steps, cfg.gamma, k_dev, v_dev, len_dev,
                      wl.cap, 1, ws, wl.status)
        torch.cuda.synchronize()
        wl.check_status()
        assert int(st["done"].item()) == 1
        assert int(st["step"].item()) == o_steps[0, c]
        assert (st["tokens"].cpu().numpy()[0] == o_tok[0, c]).all()
    assert int(len_dev.item()) == o_len[0]
    np.testing.assert_allclose(k_dev.cpu().numpy(), kc, atol=1e-5)
    np.testing.assert_allclose(v_dev.cpu().numpy(), vc, atol=1e-5)


def _eb_case(C, rng, gamma, force, nan=False):
    H = rng.choice(np.array([0.0, -0.0, -1e-7, 0.05, 0.1, 0.1, 0.25, 0.3, 1.0, 6.0], np.float32), C)
    H = np.where(rng.uniform(size=C) < 0.5, rng.uniform(0, 2, C).astype(np.float32), H).astype(np.float32)
    masked = (rng.uniform(size=C) < 0.7).astype(np.uint8)
    if nan:
        H[np.nonzero(masked)[0][0]] = np.nan
    am = rng.integers(0, 1000, C).astype(np.int32)
    tokens = np.where(masked != 0, 1000, rng.integers(0, 1000, C)).astype(np.int32)
    return H, am, masked, tokens


@pytest.mark.parametrize("C", [16, 256, 1024, 33])
@pytest.mark.parametrize("gamma", [0.0, 0.1, 0.55, 3.0, math.inf])
def test_eb_select_bit_exact(C, gamma):
    rng = np.random.default_rng(C * 7 + int(min(gamma, 99) * 100))
    Bn = 3
    cases = [_eb_case(C, rng, gamma, False) for _ in range(Bn)]
    H = np.stack([c[0] for c in cases]); am = np.stack([c[1] for c in cases])
    masked = np.stack([c[2] for c in cases]); tokens = np.stack([c[3] for c in cases])
    step = np.array([0, 5, 9], np.int32)         # canvas 2 is at its last allowed step (max 10)
    done = np.array([0, 0, 0], np.int32)
    d = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()  # noqa: E731
    t_tok, t_m, t_sel = d(tokens), d(masked), d(np.zeros_like(masked))
    t_n, t_done, t_step = d(masked.sum(1).astype(np.int32)), d(done), d(step)
    B.dg_eb_select(Bn, C, d(H), d(am), gamma, 10, t_tok, t_m, t_sel, t_n, t_done, t_step)
    torch.cuda.synchronize()
    for b in range(Bn):
        want = O.eb_select(H[b], masked[b], gamma, step[b] >= 9)
        assert (t_sel.cpu().numpy()[b].astype(bool) == want).all(), b
        exp_tok = tokens[b].copy(); exp_tok[want] = am[b][want]
        assert (t_tok.cpu().numpy()[b] == exp_tok).all()
        left = int(masked[b].sum() - want.sum())
        assert t_n.cpu().numpy()[b] == left and t_done.cpu().numpy()[b] == int(left == 0)
        assert t_step.cpu().numpy()[b] == step[b] + 1


def test_eb_select_skips_done_and_flags_nan():
    rng = np.random.default_rng(5)
    C = 64
    H, am, masked, tokens = _eb_case(C, rng, 1.0, False, nan=True)
    d = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()  # noqa: E731
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    t_tok, t_m = d(tokens[None]), d(masked[None])
    t_n = d(np.array([masked.sum()], np.int32))
    t_done, t_step = d(np.array([0], np.int32)), d(np.array([0], np.int32))
    B.dg_eb_select(1, C, d(H[None]), d(am[None]), 1.0, 16, t_tok, t_m, None, t_n, t_done, t_step, st)
    assert B.dg_read_status(st) == B.DG_ERR_NUMERIC
    assert (t_m.cpu().numpy()[0] == masked).all() and int(t_step.item()) == 0
    # a done canvas is left untouched
    H2 = np.abs(np.nan_to_num(H)).astype(np.float32)
    t_done = d(np.array([1], np.int32))
    B.dg_eb_select(1, C, d(H2[None]), d(am[None]), 1.0, 16, t_tok, t_m, None, t_n, t_done, t_step)
    torch.cuda.synchronize()
    assert (t_m.cpu().numpy()[0] == masked).all() and int(t_step.item()) == 0


def test_kv_append_capacity_is_reported(wl):
    cfg = wl.cfg
    k = wl.kv["k"].clone(); v = wl.kv["v"].clone()
    ln = torch.tensor([wl.cap - 4], dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    toks = torch.zeros((1, cfg.canvas), dtype=torch.int32, device="cuda")
    B.dg_kv_append(wl.dgcfg, wl.dgmodel, 1, toks, cfg.canvas, k, v, ln, wl.cap, wl.ws, st)
    assert B.dg_read_status(st) == B.DG_ERR_CAPACITY
    assert int(ln.item()) == wl.cap - 4
    assert torch.equal(k, wl.kv["k"]) and torch.equal(v, wl.kv["v"])
