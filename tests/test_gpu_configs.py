"""GPU parity at the full sizes of the long-context, batched-FP8 and 30-layer workloads.

* long context: the one-layer model with 131072 prompt K/V tokens, half-committed canvas; the
  oracle runs the whole step (fp64 attention over 131328 keys).
* batch of 32: 32 canvases x 256 through the one-layer model with e4m3 expert/attention weights
  (one fp32 scale per output channel), 1024 prompt tokens each; the oracle runs eight canvases,
  the first and the last among them (the others are marked done on its side; canvases are
  independent), and every canvas is checked to have taken its one step.
* stacks: a full-width step of a 4-layer stack and of the full 30-layer stack on synthetic prompt
  K/V, and the 30-layer append of a canvas, against the oracle; prefill -> denoise -> append
  against the oracle at full width and 2 layers; and the 30-layer generate loop of the workload
  (prompt 2048 prefilled in 256-token chunks, 4 canvases, at most 32 steps each) checked by its
  invariants.

Bars.  One layer: the stated bf16 bars, logits 2e-2 max-abs and entropies 1e-3 relative, on
every masked row, in a step that takes the oracle's expert choices (forced_topk; the gates are
still the device's own); and in a free-running step on every row without a router near tie
(where a bf16 router input can legitimately pick the other expert), whose count is reported and
held small.  Several layers: two valid evaluations of the method already differ by more than
2e-2 after a few layers (a bf16 rounding flip of one element of q moves every score of its row,
and the flips compound with depth), so the bar there is derived from the oracle alone:
BAR_FACTOR times the spread between the fp64 oracle and the same oracle in fp32 arithmetic on the
same inputs and expert choices, and never below the one-layer bar.  K/V caches after layer 0 are
held the same way (element error relative to its row's RMS).  Argmax is bit-exact against the
device's own logits, EB bit-exact on the oracle's entropies."""
import numpy as np
import pytest
import torch

import synth
from oracle import dg_oracle as O
from block_discrete_diffusion_dg_b200 import binding as B
from harness import (BAR_FACTOR, Workload, decode_cache, forced_from, np_state, oracle_model,
                     rel_to_row_rms, step_spread, torch_state)

pytestmark = pytest.mark.gpu

LOGIT_TOL = 2e-2
ENT_RTOL = 1e-3
ROUTER_TIE = 1e-2
# At most this share of a canvas's rows may be router near ties in the free-running check (the
# forced-routing check covers every row).  With E = 128 router logits ~N(0, s^2), s ~ 1, the gap
# between the 8th and 9th largest is roughly exponential with mean 1 / (E phi(x_8)) ~ 0.06 s, so a
# 1e-2 margin catches ~15-25% of the rows; the cap keeps the free-running comparison substantive.
NEAR_TIE_MAX = 0.3


def _device_forced(cfg, infos):
    """The oracle's expert choices as the device's forced-routing table [n_layers][B C][k]."""
    f = forced_from(cfg, infos).reshape(cfg.n_layers, cfg.batch * cfg.canvas, cfg.top_k)
    return torch.from_numpy(np.ascontiguousarray(f)).cuda()


def _check_step(wl, st_np, canvases=None, derive=False):
    """One device step against the oracle on the canvases listed (default: all): a free-running
    step (one layer only; rows without a router near tie) and a step with the oracle's expert
    choices (every row).  derive: multi-layer bars from the oracle's fp64/fp32 spread."""
    cfg = wl.cfg
    om = getattr(wl, "_om", None) or wl.oracle()
    wl._om = om
    kc, vc = decode_cache(cfg, wl.kv["k"]), decode_cache(cfg, wl.kv["v"])
    cl = synth.to_numpy(wl.kv["cache_len"])
    o_st = {k: np.array(v, copy=True) for k, v in st_np.items()}
    if canvases is not None:
        skip = np.ones(cfg.batch, bool)
        skip[list(canvases)] = False
        o_st["done"][skip] = 1
    new_np, infos = O.canvas_step(cfg, om, o_st, kc, vc, cl, cfg.gamma, cfg.max_steps,
                                  keep_logits=True)
    lbar, ebar = LOGIT_TOL, ENT_RTOL
    if derive:
        dz, dh = step_spread(cfg, om, o_st, kc, vc, cl, infos)
        lbar, ebar = max(LOGIT_TOL, BAR_FACTOR * dz), max(ENT_RTOL, BAR_FACTOR * dh)
        print(f"\n{cfg.n_layers} layers: oracle fp64/fp32 spread logits {dz:.4f} entropy {dh:.2e}"
              f" -> bars {lbar:.4f} / {ebar:.2e}")
    runs = [("forced", _device_forced(cfg, infos))]
    if cfg.n_layers == 1:
        runs.insert(0, ("free", None))
    g_st = None
    for mode, forced in runs:
        g_st, ent, am, lg = wl.step(torch_state(st_np), logits=True, forced=forced)
        wl.check_status()
        ent, am = ent.cpu().numpy(), am.cpu().numpy()
        n_rows, worst = 0, 0.0
        for b, inf in enumerate(infos):
            if inf is None:
                continue
            rows = inf["rows"]
            lgb = lg[b * cfg.canvas:(b + 1) * cfg.canvas].cpu().numpy()[rows]
            assert (am[b, rows] == np.argmax(lgb, axis=1)).all()
            if mode == "free":
                rmarg = np.min(np.stack(inf["router_margin"]), axis=0)[rows]
                ok = rmarg > ROUTER_TIE
                print(f"canvas {b}: {int((~ok).sum())} of {len(rows)} rows are router near ties")
                assert (~ok).sum() <= NEAR_TIE_MAX * len(rows)
            else:
                ok = np.ones(len(rows), bool)
            err = np.abs(lgb[ok] - inf["logits"][ok]).max()
            worst = max(worst, float(err))
            assert err <= lbar, (mode, b, err, lbar)
            np.testing.assert_allclose(ent[b, rows][ok], inf["H"][ok], rtol=ebar)
            safe = ok & (inf["margin"] > 2 * lbar)
            assert (am[b, rows][safe] == inf["argmax"][safe]).all()
            n_rows += len(rows)
        print(f"{mode}: max logit error {worst:.4f} (bar {lbar:.4f}) over {n_rows} rows")
        if canvases is None:
            assert n_rows > 0
    # EB on the oracle's entropies, each canvas alone
    for b, inf in enumerate(infos):
        if inf is None:
            continue
        rows = inf["rows"]
        e_in = np.zeros((1, cfg.canvas), np.float32)
        a_in = np.zeros((1, cfg.canvas), np.int32)
        e_in[0, rows] = inf["H"]
        a_in[0, rows] = inf["argmax"]
        one = {k: torch.from_numpy(np.ascontiguousarray(v[b:b + 1])).cuda() for k, v in st_np.items()}
        B.dg_eb_select(1, cfg.canvas, torch.from_numpy(e_in).cuda(), torch.from_numpy(a_in).cuda(),
                       cfg.gamma, cfg.max_steps, one["tokens"], one["masked"], None,
                       one["n_masked"], one["done"], one["step"])
        for k in ("tokens", "masked", "n_masked", "done", "step"):
            assert (one[k].cpu().numpy()[0] == new_np[k][b]).all(), k
    return g_st


def _append_check(wl, om, toks, ok, ov, ln, n, ws=None):
    """Append `toks` [1, n] on the device (with the oracle's expert choices) and in the oracle
    (fp64, and fp32 with the same choices); every new K/V element of every layer within
    max(2^-7, BAR_FACTOR x the oracle's fp64/fp32 spread), relative to its row's RMS (2^-7: about
    two bf16 ulps of a typical element, the floor for a single rounding flip)."""
    cfg = wl.cfg
    o32k, o32v = ok.copy(), ov.copy()
    info = {}
    ln2 = O.kv_append(cfg, om, toks.cpu().numpy(), ok, ov, ln, info)
    forced_np = np.stack([r for r in info["router_idx"]]) if "router_idx" in info else \
        np.zeros((cfg.n_layers, 1, n, cfg.top_k), np.int32)        # [L][B][n][k]
    with O.accumulation(np.float32):
        O.kv_append(cfg, om, toks.cpu().numpy(), o32k, o32v, ln, None, forced=forced_np)
    forced = torch.from_numpy(np.ascontiguousarray(forced_np.reshape(cfg.n_layers, -1, cfg.top_k))).cuda()
    B.dg_kv_append(wl.dgcfg, wl.dgmodel, 1, toks, n, wl.kv["k"], wl.kv["v"], wl.kv["cache_len"],
                   wl.cap, wl.ws if ws is None else ws, wl.status, forced_topk=forced)
    torch.cuda.synchronize()
    wl.check_status()
    assert int(wl.kv["cache_len"].item()) == ln2[0]
    sl = slice(int(ln[0]), int(ln2[0]))
    for name, dev, o64, o32 in (("k", wl.kv["k"], ok, o32k), ("v", wl.kv["v"], ov, o32v)):
        g = decode_cache(cfg, dev)[:, :, :, sl, :]
        ref = o64[:, :, :, sl, :]
        rel_d = float(rel_to_row_rms(g, ref).max())
        rel_o = float(rel_to_row_rms(o32[:, :, :, sl, :], ref).max())
        bar = max(2.0 ** -7, BAR_FACTOR * rel_o)
        print(f"\n{name}: device {rel_d:.4f} vs oracle spread {rel_o:.4f} -> bar {bar:.4f}")
        assert rel_d <= bar, (name, rel_d, bar)
    return ln2


def test_longctx_step_full_size():
    cfg = synth.get_config("longctx")
    wl = Workload(cfg, gen_device="cuda")
    _check_step(wl, np_state(synth.make_canvas_state(cfg, "half")))


def test_batch32_fp8_step_sampled_canvases():
    cfg = synth.get_config("batch32")
    wl = Workload(cfg, gen_device="cuda")
    st = np_state(synth.make_canvas_state(cfg, "all_mask"))
    g_st = _check_step(wl, st, canvases=(0, 5, 10, 15, 17, 22, 27, 31))
    # every canvas advanced by one step and committed exactly one token (entropies ~ ln V >> gamma)
    assert (g_st["step"].cpu().numpy() == 1).all()
    assert (g_st["n_masked"].cpu().numpy() == cfg.canvas - 1).all()


def test_stack_step_full_width_four_layers():
    cfg = synth.get_config("stack30", n_layers=4, prefill_ids=False, prompt_len=1024)
    wl = Workload(cfg, gen_device="cuda")
    _check_step(wl, np_state(synth.make_canvas_state(cfg, "half")), derive=True)


@pytest.mark.slow
def test_stack30_step_and_append_vs_oracle():
    """The full 30-layer stack at full width: one denoising step of a half-committed canvas over a
    2048-token synthetic prompt cache, then the causal append of a committed canvas, both against
    the oracle with its expert choices handed to the device and bars derived from the oracle's
    fp64/fp32 spread.  The oracle reads the device's weights layer by layer."""
    cfg = synth.get_config("stack30", prefill_ids=False)
    wl = Workload(cfg, gen_device="cuda")
    wl._om = oracle_model(cfg, wl.model, lazy=True)
    _check_step(wl, np_state(synth.make_canvas_state(cfg, "half")), derive=True)
    ok, ov = decode_cache(cfg, wl.kv["k"]), decode_cache(cfg, wl.kv["v"])
    ln = synth.to_numpy(wl.kv["cache_len"]).copy()
    g = torch.Generator(device="cpu").manual_seed(30)
    toks = torch.randint(0, cfg.vocab, (1, cfg.canvas), generator=g, dtype=torch.int32).cuda()
    _append_check(wl, wl._om, toks, ok, ov, ln, cfg.canvas)


def test_stack_prefill_denoise_append_two_layers():
    """Prefill 512 prompt ids in two 256-token chunks, two lockstep denoising steps of a canvas,
    then its append: caches and step outputs against the oracle (full width, 2 layers)."""
    cfg = synth.get_config("stack30", n_layers=2, prompt_len=512, n_canvases=1)
    wl = Workload(cfg, gen_device="cuda")
    om = wl.oracle()
    wl._om = om
    ids = wl.kv["prompt_ids"]
    ok = np.zeros(decode_cache(cfg, wl.kv["k"]).shape)
    ov = np.zeros_like(ok)
    ln = np.zeros(1, np.int32)
    for c0 in range(0, cfg.prompt_len, 256):
        ln = _append_check(wl, om, ids[:, c0:c0 + 256].contiguous(), ok, ov, ln, 256)
    assert int(wl.kv["cache_len"].item()) == ln[0] == cfg.prompt_len
    # two denoising steps from the oracle's state on the oracle-prefilled cache
    wl.kv["k"] = torch.from_numpy(ok).to(torch.bfloat16).cuda()
    wl.kv["v"] = torch.from_numpy(ov).to(torch.bfloat16).cuda()
    wl.kv["cache_len"] = torch.from_numpy(ln).cuda()
    st = np_state(synth.make_canvas_state(cfg, "all_mask"))
    for _ in range(2):
        _check_step(wl, st, derive=True)
        kc, vc = decode_cache(cfg, wl.kv["k"]), decode_cache(cfg, wl.kv["v"])
        st, _ = O.canvas_step(cfg, om, st, kc, vc, ln, cfg.gamma, cfg.max_steps)
    # append a committed canvas
    toks = torch.randint(0, cfg.vocab, (1, cfg.canvas), dtype=torch.int32).cuda()
    ln2 = _append_check(wl, om, toks, ok, ov, ln, cfg.canvas)
    assert ln2[0] == ln[0] + cfg.canvas


def test_prefill_one_call_of_1024_tokens_two_layers():
    """A long prompt prefilled by one dg_kv_append of 1024 tokens (four canvases' worth): causal
    attention over the whole chunk, the expert GEMMs beyond the 256-token split-K path and the
    2048-assignment permutation; caches against the oracle's append of the same ids (full width,
    2 layers, the oracle's expert choices handed to the device as in the other stack tests)."""
    n = 1024
    cfg = synth.get_config("stack30", n_layers=2, prompt_len=n, n_canvases=1)
    wl = Workload(cfg, gen_device="cuda")
    om = wl.oracle()
    ids = wl.kv["prompt_ids"][:, :n].contiguous()
    ws = B.alloc_workspace(wl.dgcfg, 1, n, wl.cap)
    ok = np.zeros(decode_cache(cfg, wl.kv["k"]).shape)
    ov = np.zeros_like(ok)
    ln = _append_check(wl, om, ids, ok, ov, np.zeros(1, np.int32), n, ws=ws)
    assert ln[0] == n


def test_stack30_generate_invariants():
    """The full 30-layer workload: prefill, 4 canvases of at most 32 steps, appends."""
    cfg = synth.get_config("stack30")
    wl = Workload(cfg, gen_device="cuda")
    ids = wl.kv["prompt_ids"]
    k_dev, v_dev, len_dev = wl.kv["k"], wl.kv["v"], wl.kv["cache_len"]
    for c0 in range(0, cfg.prompt_len, 256):
        B.dg_kv_append(wl.dgcfg, wl.dgmodel, 1, ids[:, c0:c0 + 256].contiguous(), 256, k_dev,
                       v_dev, len_dev, wl.cap, wl.ws, wl.status)
    out = []
    for c in range(cfg.n_canvases):
        st = {k: v.cuda() for k, v in synth.make_canvas_state(cfg, "all_mask").items()}
        steps = 0
        while not int(st["done"].item()):
            B.dg_canvas_step(wl.dgcfg, wl.dgmodel, 1, st["tokens"], st["masked"], st["n_masked"],
                             st["done"], st["step"], cfg.max_steps, cfg.gamma, k_dev, v_dev,
                             len_dev, wl.cap, None, None, None, wl.ws, wl.status)
            steps += 1
            assert steps <= cfg.max_steps
        # the canvas always finishes within the step cap (the last allowed step commits the rest)
        assert int(st["step"].item()) == steps <= cfg.max_steps and int(st["n_masked"].item()) == 0
        toks = st["tokens"].cpu().numpy()
        assert (toks >= 0).all() and (toks < cfg.vocab).all()
        out.append(toks)
        B.dg_kv_append(wl.dgcfg, wl.dgmodel, 1, st["tokens"], cfg.canvas, k_dev, v_dev, len_dev,
                       wl.cap, wl.ws, wl.status)
    torch.cuda.synchronize()
    wl.check_status()
    assert int(len_dev.item()) == cfg.prompt_len + cfg.n_canvases * cfg.canvas == wl.cap
    assert torch.isfinite(k_dev.float()).all() and torch.isfinite(v_dev.float()).all()
    # a second canvas step from the same state reproduces the first bit for bit
    st0 = {k: v.cuda() for k, v in synth.make_canvas_state(cfg, "half").items()}
    ents = []
    for _ in range(2):
        st = {k: v.clone() for k, v in st0.items()}
        ent = torch.zeros((1, cfg.canvas), device="cuda")
        B.dg_canvas_step(wl.dgcfg, wl.dgmodel, 1, st["tokens"], st["masked"], st["n_masked"],
                         st["done"], st["step"], cfg.max_steps, cfg.gamma, k_dev, v_dev, len_dev,
                         wl.cap, ent, None, None, wl.ws, wl.status)
        ents.append(ent.cpu())
    assert torch.equal(ents[0], ents[1])
