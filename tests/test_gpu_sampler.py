"""GPU parity of the sampler variants against the oracle: the uniform-noise canvas, the
temperature-annealed Gumbel-max draw (on the CUDA-core LM head of the tiny fp32 workload, the
tensor-core LM heads of the bf16 layer — one CTA per SM up to 128 rows, CTA pairs beyond — and
the NVFP4 LM head), the revisable drafts of a noise canvas, the autoregressive step, and hybrid
decoding (canvases and AR tokens on one cache).

Checks for a drawn token: it is the argmax of the device's own dumped logits times its 1/tau
plus the Gumbel draws that the oracle's generator gives for the same stream (within 1e-4 of the
maximum key: the device's fp32 logarithms against the oracle's fp64 ones); and it equals the
oracle's token wherever the oracle's top-2 key margin exceeds twice the logit bar times 1/tau.
Entropies are those of softmax(z/tau), within the stated relative bar.  EB and the draft revision
are bit-exact on the oracle's entropies and tokens."""
import numpy as np
import pytest
import torch

import synth
from oracle import dg_oracle as O
from block_discrete_diffusion_dg_b200 import binding as B
from harness import Workload, decode_cache, forced_from, np_state, torch_state

pytestmark = pytest.mark.gpu

KEY_TOL = 1e-4


def _state_dev(st_np):
    return torch_state(st_np)


def _device_step(wl, st_np, smp, forced=None):
    cfg = wl.cfg
    st = _state_dev(st_np)
    B_, C = cfg.batch, cfg.canvas
    ent = torch.full((B_, C), float("nan"), device="cuda")
    am = torch.full((B_, C), -1, dtype=torch.int32, device="cuda")
    lg = torch.zeros((B_ * C, cfg.vocab), device="cuda")
    B.dg_canvas_step_sampler(wl.dgcfg, wl.dgmodel, B_, st["tokens"], st["masked"], st["n_masked"],
                             st["done"], st["step"], cfg.max_steps, cfg.gamma, smp, wl.kv["k"],
                             wl.kv["v"], wl.kv["cache_len"], wl.cap, ent, am, lg, wl.ws,
                             wl.status, forced_topk=forced)
    torch.cuda.synchronize()
    wl.check_status()
    return st, ent.cpu().numpy(), am.cpu().numpy(), lg.cpu().numpy()


def _check_draws(cfg, smp_d, st_np, infos, ent, am, lg, logit_tol, ent_rtol):
    """Drawn tokens and entropies of one sampled step against the oracle (see module doc)."""
    n = 0
    for b, inf in enumerate(infos):
        if inf is None:
            continue
        tau = inf["tau"]
        assert tau == O.temperature(int(st_np["step"][b]), cfg.max_steps, smp_d["tau_start"],
                                    smp_d["tau_end"])
        inv = float(O.inv_temperature(tau)) if tau > 0 else 1.0
        for j, i in enumerate(inf["rows"]):
            z = lg[b * cfg.canvas + i].astype(np.float64)
            if tau > 0:
                g = O.gumbel(O.stream_words(smp_d["seed"], O.TAG_DENOISE, b, int(i),
                                            int(st_np["step"][b]), cfg.vocab))
                keys = z * inv + g
            else:
                keys = z
            t = int(am[b, i])
            assert 0 <= t < cfg.vocab
            assert keys[t] >= keys.max() - KEY_TOL, (b, i, keys.max() - keys[t])
            if inf["margin"][j] > 2 * logit_tol * inv + KEY_TOL:
                assert t == inf["argmax"][j], (b, i)
            n += 1
        np.testing.assert_allclose(ent[b, inf["rows"]], inf["H"], rtol=ent_rtol)
    assert n > 0


def _eb_revise_check(cfg, st_np, infos, new_np, revise):
    """EB + commit (+ draft revision) on the oracle's entropies and tokens: bit-exact."""
    e_in = np.zeros((cfg.batch, cfg.canvas), np.float32)
    a_in = np.zeros((cfg.batch, cfg.canvas), np.int32)
    for b, inf in enumerate(infos):
        if inf is not None:
            e_in[b, inf["rows"]] = inf["H"]
            a_in[b, inf["rows"]] = inf["argmax"]
    st2 = torch_state(st_np)
    B.dg_eb_select(cfg.batch, cfg.canvas, torch.from_numpy(e_in).cuda(),
                   torch.from_numpy(a_in).cuda(), cfg.gamma, cfg.max_steps, st2["tokens"],
                   st2["masked"], None, st2["n_masked"], st2["done"], st2["step"], revise=revise)
    for k in ("tokens", "masked", "n_masked", "done", "step"):
        assert (st2[k].cpu().numpy() == new_np[k]).all(), k


def test_noise_canvas_bit_exact():
    for B_, C, V, seed in ((3, 256, 262144, 0x0123456789ABCDEF), (2, 16, 512, 7)):
        st = {"tokens": torch.full((B_, C), -1, dtype=torch.int32, device="cuda"),
              "masked": torch.zeros((B_, C), dtype=torch.uint8, device="cuda"),
              "n_masked": torch.zeros(B_, dtype=torch.int32, device="cuda"),
              "done": torch.ones(B_, dtype=torch.int32, device="cuda"),
              "step": torch.full((B_,), 9, dtype=torch.int32, device="cuda")}
        B.dg_noise_canvas(B_, C, V, seed, st["tokens"], st["masked"], st["n_masked"], st["done"],
                          st["step"])
        ref = O.noise_canvas(seed, B_, C, V)
        for k in ref:
            assert (st[k].cpu().numpy() == ref[k]).all(), k


@pytest.fixture(scope="module")
def tiny():
    return Workload(synth.get_config("tiny"), gen_device="cpu")


@pytest.mark.parametrize("revise", [False, True])
def test_tiny_sampled_lockstep(tiny, revise):
    """The tiny fp32 workload (CUDA-core LM head) through a whole canvas in lockstep: annealed
    temperature 1.2 -> 0.3, from all-MASK (absorbing) or from a noise canvas (revisable drafts)."""
    wl = tiny
    cfg = wl.cfg
    om = wl.oracle()
    smp_d = {"tau_start": 1.2, "tau_end": 0.3, "seed": 0xBEEF, "revise": revise}
    smp = B.make_sampler(1.2, 0.3, 0xBEEF, revise)
    st_np = O.noise_canvas(5, 1, cfg.canvas, cfg.vocab) if revise else np_state(wl.state)
    kc, vc = decode_cache(cfg, wl.kv["k"]), decode_cache(cfg, wl.kv["v"])
    cl = synth.to_numpy(wl.kv["cache_len"])
    for _ in range(cfg.max_steps):
        new_np, infos = O.canvas_step(cfg, om, st_np, kc, vc, cl, cfg.gamma, cfg.max_steps,
                                      keep_logits=True, sampler=smp_d)
        g_st, ent, am, lg = _device_step(wl, st_np, smp)
        rows = infos[0]["rows"]
        assert np.abs(lg[rows] - infos[0]["logits"]).max() <= 1e-4
        _check_draws(cfg, smp_d, st_np, infos, ent, am, lg, 1e-4, 1e-3)
        _eb_revise_check(cfg, st_np, infos, new_np, revise)
        # tiny fp32: the device's own step reproduces the oracle's where no near tie decides it
        # (the two lowest entropies apart, every drawn token's key margin clear of the bar)
        h = np.sort(infos[0]["H"])
        if (len(h) < 2 or h[1] - h[0] > 1e-5) and (infos[0]["margin"] > 1e-3).all():
            for k in ("tokens", "masked", "n_masked", "done", "step"):
                assert (g_st[k].cpu().numpy() == new_np[k]).all(), k
        st_np = new_np
        if st_np["done"][0]:
            break
    assert st_np["done"][0] == 1


@pytest.mark.parametrize("name,kind", [("layer", "all_mask"), ("layer", "half"),
                                       ("layer_nvfp4", "all_mask")])
def test_sampled_step_reduced(name, kind):
    """A sampled step of the reduced bf16 layer on the tensor-core LM heads (all-MASK: more than
    128 rows with batch 3, the CTA-pair kernel; half: the single-CTA kernel; NVFP4 weights), with
    the oracle's expert choices; then the same with revisable drafts from a noise canvas."""
    over = {"router_std": 1.0 / 16.0} if name == "layer_nvfp4" else {}
    cfg = synth.reduced(name, batch=3, **over)
    wl = Workload(cfg, gen_device="cpu")
    om = wl.oracle()
    kc, vc = decode_cache(cfg, wl.kv["k"]), decode_cache(cfg, wl.kv["v"])
    cl = synth.to_numpy(wl.kv["cache_len"])
    for revise in (False, True):
        st_np = O.noise_canvas(3, cfg.batch, cfg.canvas, cfg.vocab) if revise else \
            np_state(synth.make_canvas_state(cfg, kind))
        st_np["step"][:] = [0, 5, 40]                      # three temperatures of the schedule
        smp_d = {"tau_start": 1.0, "tau_end": 0.25, "seed": 77, "revise": revise}
        new_np, infos = O.canvas_step(cfg, om, st_np, kc, vc, cl, cfg.gamma, cfg.max_steps,
                                      keep_logits=True, sampler=smp_d)
        forced = torch.from_numpy(forced_from(cfg, infos).reshape(cfg.n_layers, -1, cfg.top_k)).cuda()
        _, ent, am, lg = _device_step(wl, st_np, B.make_sampler(1.0, 0.25, 77, revise), forced)
        for b, inf in enumerate(infos):
            assert np.abs(lg[b * cfg.canvas + inf["rows"]] - inf["logits"]).max() <= 2e-2
        _check_draws(cfg, smp_d, st_np, infos, ent, am, lg, 2e-2, 1e-3)
        _eb_revise_check(cfg, st_np, infos, new_np, revise)


def test_sampled_step_full_size_both_lm_head_kernels():
    """The full one-layer size: 256 masked rows (CTA pairs) and 128 (one CTA per SM), temperature
    0.7, the oracle's expert choices."""
    cfg = synth.get_config("layer")
    wl = Workload(cfg, gen_device="cuda")
    om = wl.oracle()
    kc, vc = decode_cache(cfg, wl.kv["k"]), decode_cache(cfg, wl.kv["v"])
    cl = synth.to_numpy(wl.kv["cache_len"])
    smp_d = {"tau_start": 0.7, "tau_end": 0.7, "seed": 2024, "revise": False}
    for kind in ("all_mask", "half"):
        st_np = np_state(synth.make_canvas_state(cfg, kind))
        new_np, infos = O.canvas_step(cfg, om, st_np, kc, vc, cl, cfg.gamma, cfg.max_steps,
                                      keep_logits=True, sampler=smp_d)
        forced = torch.from_numpy(forced_from(cfg, infos).reshape(cfg.n_layers, -1, cfg.top_k)).cuda()
        _, ent, am, lg = _device_step(wl, st_np, B.make_sampler(0.7, 0.7, 2024), forced)
        _check_draws(cfg, smp_d, st_np, infos, ent, am, lg, 2e-2, 1e-3)
        _eb_revise_check(cfg, st_np, infos, new_np, False)


@pytest.mark.parametrize("tau", [0.0, 0.8])
def test_tiny_ar_steps_and_hybrid_decoding(tiny, tau):
    """Hybrid decoding on the tiny fp32 workload: a diffusion canvas (sampled at tau) generated to
    completion and appended, then four autoregressive steps (one token each, the last prediction
    fed back), then a two-token AR step, against the oracle: tokens bit-exact, entropies 1e-3
    relative, caches within 1e-5."""
    wl = tiny
    cfg = wl.cfg
    om = wl.oracle()
    k_dev, v_dev, l_dev = wl.kv["k"].clone(), wl.kv["v"].clone(), wl.kv["cache_len"].clone()
    kc, vc = decode_cache(cfg, k_dev), decode_cache(cfg, v_dev)
    cl = synth.to_numpy(l_dev).copy()
    smp_d = {"tau_start": tau, "tau_end": tau, "seed": 31, "revise": False}
    smp = B.make_sampler(tau, tau, 31)
    # 1. a diffusion canvas, the device loop against the oracle's loop
    st_np = np_state(synth.make_canvas_state(cfg, "all_mask"))
    st = torch_state(st_np)
    while not st_np["done"][0]:
        st_np, _ = O.canvas_step(cfg, om, st_np, kc, vc, cl, cfg.gamma, cfg.max_steps,
                                 sampler=smp_d)
        B.dg_canvas_step_sampler(wl.dgcfg, wl.dgmodel, 1, st["tokens"], st["masked"],
                                 st["n_masked"], st["done"], st["step"], cfg.max_steps, cfg.gamma,
                                 smp, k_dev, v_dev, l_dev, wl.cap, None, None, None, wl.ws,
                                 wl.status)
    torch.cuda.synchronize()
    for k in st_np:
        assert (st[k].cpu().numpy() == st_np[k]).all(), k
    cl = O.kv_append(cfg, om, st_np["tokens"], kc, vc, cl)
    B.dg_kv_append(wl.dgcfg, wl.dgmodel, 1, st["tokens"], cfg.canvas, k_dev, v_dev, l_dev, wl.cap,
                   wl.ws, wl.status)
    # 2. autoregressive steps on the same cache, each prediction fed back
    ws_ar = B.alloc_workspace(wl.dgcfg, 1, 2, wl.cap)
    tok = st_np["tokens"][:, -1:].copy()
    for n_new in (1, 1, 1, 1, 2):
        if n_new == 2:
            tok = np.concatenate([tok, np.array([[7]], np.int32)], axis=1)
        nxt_o, H_o, _, cl, z_o = O.ar_step(cfg, om, tok, kc, vc, cl, tau=tau, seed=31)
        nxt = torch.full((1,), -1, dtype=torch.int32, device="cuda")
        ent = torch.zeros(1, device="cuda")
        lg = torch.zeros((1, cfg.vocab), device="cuda")
        B.dg_ar_step(wl.dgcfg, wl.dgmodel, 1, torch.from_numpy(tok).cuda(), tok.shape[1], k_dev,
                     v_dev, l_dev, wl.cap, nxt, ent, lg, ws_ar, wl.status, sampler=smp)
        torch.cuda.synchronize()
        wl.check_status()
        assert np.abs(lg.cpu().numpy() - z_o).max() <= 1e-4
        assert int(nxt.item()) == int(nxt_o[0])
        np.testing.assert_allclose(ent.cpu().numpy(), H_o, rtol=1e-3)
        assert int(l_dev.item()) == int(cl[0])
        tok = nxt_o[:, None].astype(np.int32)
    np.testing.assert_allclose(decode_cache(cfg, k_dev), kc, atol=1e-5)
    np.testing.assert_allclose(decode_cache(cfg, v_dev), vc, atol=1e-5)


def test_ar_step_reduced_bf16_batch():
    """The AR step on the tensor-core path (reduced bf16 layer, batch 2, 3 new tokens per
    sequence, temperature 0.9), with the oracle's expert choices: logits within 2e-2, the drawn
    token checked as in the canvas tests, K/V rows within two bf16 ulps."""
    cfg = synth.reduced("layer", batch=2)
    wl = Workload(cfg, gen_device="cpu")
    om = wl.oracle()
    kc, vc = decode_cache(cfg, wl.kv["k"]), decode_cache(cfg, wl.kv["v"])
    cl = synth.to_numpy(wl.kv["cache_len"]).copy()
    toks = np.array([[11, 4000, 5], [1, 2, 3]], np.int32)
    info = {}
    nxt_o, H_o, margin, cl2, z_o = O.ar_step(cfg, om, toks, kc, vc, cl, tau=0.9, seed=8, info=info)
    forced = np.stack(info["router_idx"]).reshape(cfg.n_layers, -1, cfg.top_k)
    nxt = torch.full((2,), -1, dtype=torch.int32, device="cuda")
    ent = torch.zeros(2, device="cuda")
    lg = torch.zeros((2, cfg.vocab), device="cuda")
    ws = B.alloc_workspace(wl.dgcfg, 2, 3, wl.cap)
    B.dg_ar_step(wl.dgcfg, wl.dgmodel, 2, torch.from_numpy(toks).cuda(), 3, wl.kv["k"], wl.kv["v"],
                 wl.kv["cache_len"], wl.cap, nxt, ent, lg, ws, wl.status,
                 sampler=B.make_sampler(0.9, 0.9, 8),
                 forced_topk=torch.from_numpy(np.ascontiguousarray(forced)).cuda())
    torch.cuda.synchronize()
    wl.check_status()
    lg = lg.cpu().numpy()
    assert np.abs(lg - z_o).max() <= 2e-2
    inv = float(O.inv_temperature(0.9))
    for b in range(2):
        g = O.gumbel(O.stream_words(8, O.TAG_AR, b, int(cl[b]) + 3, 0, cfg.vocab))
        keys = lg[b].astype(np.float64) * inv + g
        t = int(nxt[b].item())
        assert keys[t] >= keys.max() - KEY_TOL
        if margin[b] > 2 * 2e-2 * inv + KEY_TOL:
            assert t == nxt_o[b]
    np.testing.assert_allclose(ent.cpu().numpy(), H_o, rtol=1e-3)
    assert (wl.kv["cache_len"].cpu().numpy() == cl2).all()
    for dev, orc in ((wl.kv["k"], kc), (wl.kv["v"], vc)):
        g = decode_cache(cfg, dev)
        for b in range(2):
            sl = slice(int(cl[b]), int(cl2[b]))
            rows_o = orc[:, b, :, sl]
            rows_g = g[:, b, :, sl]
            assert (np.abs(rows_g - rows_o) <= 2.0 ** -7 * np.abs(rows_o) + 1e-3).all()


def test_device_generate_with_sampler_equals_host_loop():
    """dg_generate with a sampler (noise canvas, revisable drafts, annealed temperature) replays
    the same kernels as the host loop of dg_canvas_step_sampler: identical states and caches."""
    cfg = synth.reduced("layer", batch=2, n_canvases=1, gamma=0.5, max_steps=12)
    wl = Workload(cfg, gen_device="cpu")
    smp = B.make_sampler(1.0, 0.2, 99, True)
    states = []
    for device_loop in (False, True):
        kv = {k: v.clone() for k, v in wl.kv.items()}
        st = {k: v.clone() for k, v in wl.state.items()}
        B.dg_noise_canvas(cfg.batch, cfg.canvas, cfg.vocab, 4, st["tokens"], st["masked"],
                          st["n_masked"], st["done"], st["step"])
        if device_loop:
            B.dg_generate(wl.dgcfg, wl.dgmodel, cfg.batch, st["tokens"], st["masked"],
                          st["n_masked"], st["done"], st["step"], cfg.max_steps, cfg.gamma,
                          kv["k"], kv["v"], kv["cache_len"], wl.cap, 1, wl.ws, wl.status,
                          sampler=smp)
        else:
            n = 0
            while not bool(st["done"].all()):
                B.dg_canvas_step_sampler(wl.dgcfg, wl.dgmodel, cfg.batch, st["tokens"],
                                         st["masked"], st["n_masked"], st["done"], st["step"],
                                         cfg.max_steps, cfg.gamma, smp, kv["k"], kv["v"],
                                         kv["cache_len"], wl.cap, None, None, None, wl.ws,
                                         wl.status)
                n += 1
                assert n <= cfg.max_steps
            B.dg_kv_append(wl.dgcfg, wl.dgmodel, cfg.batch, st["tokens"], cfg.canvas, kv["k"],
                           kv["v"], kv["cache_len"], wl.cap, wl.ws, wl.status)
        torch.cuda.synchronize()
        wl.check_status()
        states.append((st, kv))
    (h, kh), (d, kd) = states
    for k in h:
        assert torch.equal(h[k], d[k]), k
    for k in ("k", "v", "cache_len"):
        assert torch.equal(kh[k], kd[k]), k
    assert bool((d["done"] == 1).all())
