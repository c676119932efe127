"""CPU pins of the oracle's sampler variants (the noise canvas with revisable drafts, the
temperature-annealed Gumbel-max draw, the autoregressive step), each against something other than
itself: the generator's published known-answer vectors, the Gumbel law's moments, the softmax
frequencies the Gumbel-max rule must reproduce, closed forms, and invariants of the decoding loop.
These run without a GPU."""
import math
import os

import numpy as np
import pytest

import synth
from oracle import dg_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _kat():
    rows = []
    for line in open(os.path.join(GOLDEN, "philox4x32_10_kat.txt")):
        if line.strip() and not line.startswith("#"):
            rows.append([int(x, 16) for x in line.split()])
    return rows


@pytest.mark.parametrize("row", _kat())
def test_philox_known_answer_vectors(row):
    c0, c1, c2, c3, k0, k1 = row[:6]
    out = O.philox4x32_10(c0, c1, c2, c3, k0, k1)
    assert [int(w) for w in out] == row[6:]


def test_philox_vectorised_equals_scalar_calls_and_stream_word_order():
    rng = np.random.default_rng(3)
    c = rng.integers(0, 2 ** 32, size=(4, 17), dtype=np.uint64)
    vec = O.philox4x32_10(c[0], c[1], c[2], c[3], 0x12345678, 0x9ABCDEF0)
    for j in range(17):
        one = O.philox4x32_10(int(c[0, j]), int(c[1, j]), int(c[2, j]), int(c[3, j]),
                              0x12345678, 0x9ABCDEF0)
        assert [int(vec[w][j]) for w in range(4)] == [int(x) for x in one]
    # stream word v is word v & 3 of counter (v >> 2, a1, a2, (tag << 24) | b), key = the seed
    seed = 0x0123456789ABCDEF
    w = O.stream_words(seed, O.TAG_DENOISE, 5, 7, 9, 11)
    for v in range(11):
        ref = O.philox4x32_10(v >> 2, 7, 9, (O.TAG_DENOISE << 24) | 5, seed & 0xFFFFFFFF, seed >> 32)
        assert int(w[v]) == int(ref[v & 3])


def test_uniform_is_exact_and_open_and_gumbel_moments():
    u = O.uniform_open(np.array([0, 511, 512, 2 ** 32 - 1], dtype=np.uint64))
    np.testing.assert_array_equal(u, [2.0 ** -24, 2.0 ** -24, 3 * 2.0 ** -24, 1 - 2.0 ** -24])
    assert (u.astype(np.float32).astype(np.float64) == u).all()        # exact in fp32
    g = O.gumbel(O.stream_words(1, O.TAG_DENOISE, 0, 0, 0, 1 << 20))
    # standard Gumbel: mean = Euler-Mascheroni constant, variance = pi^2 / 6
    assert abs(g.mean() - 0.5772156649015329) < 5e-3
    assert abs(g.var() / (math.pi ** 2 / 6) - 1) < 0.02


def test_gumbel_max_draw_follows_softmax_at_temperature():
    """Frequencies of sample_row's token over 20000 independent streams match softmax(z / tau)
    within 4 standard errors."""
    z = np.array([1.0, 0.2, -0.5, 2.0, 0.0])
    tau = 0.7
    n = 20000
    counts = np.zeros(5)
    for a1 in range(n):
        g = O.gumbel(O.stream_words(99, O.TAG_DENOISE, 0, a1, 3, 5))
        counts[O.sample_row(z, tau, g)[1]] += 1
    p = np.exp(z / tau - (z / tau).max())
    p /= p.sum()
    assert (np.abs(counts / n - p) <= 4 * np.sqrt(p * (1 - p) / n)).all()


def test_temperature_schedule_endpoints_and_greedy():
    assert O.temperature(0, 12, 1.5, 0.5) == 1.5
    assert O.temperature(11, 12, 1.5, 0.5) == 0.5
    assert O.temperature(40, 12, 1.5, 0.5) == 0.5            # past the budget: tau_end
    assert O.temperature(3, 1, 0.8, 0.1) == 0.8                # one-step budget
    taus = [O.temperature(s, 48, 1.0, 0.2) for s in range(48)]
    assert all(a > b for a, b in zip(taus, taus[1:]))          # strictly annealed
    # a larger budget anneals more mildly: a smaller drop per step
    assert O.temperature(1, 192, 1.0, 0.2) > O.temperature(1, 48, 1.0, 0.2)
    z = np.array([0.3, 2.0, 2.0, -1.0])
    H, tok, _ = O.sample_row(z, 0.0, None)                     # greedy: first argmax, tau = 1
    p = np.exp(z - z.max()); p /= p.sum()
    assert tok == 1 and abs(H + (p * np.log(p)).sum()) < 1e-12


def test_entropy_at_temperature_closed_forms():
    # two logits (a, 0) at temperature tau: H = ln(1 + e^x) - x e^x / (1 + e^x), x = a / tau
    for a, tau in ((1.0, 0.5), (3.0, 2.0), (-2.0, 0.25)):
        g = np.zeros(2)
        H, _, _ = O.sample_row(np.array([a, 0.0]), tau, g)
        x = a * float(O.inv_temperature(tau))
        want = math.log1p(math.exp(x)) - x * math.exp(x) / (1 + math.exp(x))
        assert abs(H - want) < 1e-12
    # a very hot distribution is uniform: H -> ln V
    H, _, _ = O.sample_row(np.array([0.1, -0.3, 0.7, 0.2]), 1e9, np.zeros(4))
    assert abs(H - math.log(4)) < 1e-9


def test_noise_canvas_uniform_deterministic_and_per_canvas():
    V, C = 16, 4096
    a = O.noise_canvas(7, 2, C, V)
    b = O.noise_canvas(7, 2, C, V)
    np.testing.assert_array_equal(a["tokens"], b["tokens"])
    t = a["tokens"]
    assert t.min() >= 0 and t.max() < V
    assert not (t[0] == t[1]).all()                          # canvases draw their own streams
    counts = np.bincount(t[0], minlength=V)
    chi2 = ((counts - C / V) ** 2 / (C / V)).sum()
    assert chi2 < 45.0                                       # 15 dof: p ~ 1e-4
    assert (a["masked"] == 1).all() and (a["n_masked"] == C).all()
    # token = (w0 * V) >> 32 of the stream's first word
    w0 = O.philox4x32_10(3, 0, 0, (O.TAG_NOISE << 24) | 1, 7, 0)[0]
    assert t[1, 3] == (int(w0) * V) >> 32


@pytest.fixture(scope="module")
def tiny():
    cfg = synth.get_config("tiny")
    m = synth.make_model(cfg, "cpu")
    arr = {"emb": synth.to_numpy(m["emb"]),
           "layers": [{k: synth.to_numpy(v) for k, v in lay.items()} for lay in m["layers"]]}
    kv = synth.make_prompt_kv(cfg, "cpu")
    kc = synth.to_numpy(kv["k"]).astype(np.float64)
    vc = synth.to_numpy(kv["v"]).astype(np.float64)
    return cfg, O.OracleModel(cfg, arr), kc, vc, synth.to_numpy(kv["cache_len"])


def test_greedy_sampler_equals_the_plain_step(tiny):
    cfg, om, kc, vc, cl = tiny
    st = {k: synth.to_numpy(v) for k, v in synth.make_canvas_state(cfg, "all_mask").items()}
    a, ia = O.canvas_step(cfg, om, st, kc, vc, cl, cfg.gamma, cfg.max_steps)
    b, ib = O.canvas_step(cfg, om, st, kc, vc, cl, cfg.gamma, cfg.max_steps,
                          sampler={"tau_start": 0.0, "tau_end": 0.0, "seed": 5, "revise": False})
    for k in a:
        np.testing.assert_array_equal(a[k], b[k])
    np.testing.assert_array_equal(ia[0]["H"], ib[0]["H"])


def test_noise_canvas_revisable_drafts_loop(tiny):
    """The noise canvas with revisable drafts at temperature 1 -> 0.5: one final commit per step
    (entropies ~ ln V >> gamma), the other non-final positions hold the step's draws, final
    positions never change, the canvas finishes within the step cap, and the run is a function of
    the seed."""
    cfg, om, kc, vc, cl = tiny
    smp = {"tau_start": 1.0, "tau_end": 0.5, "seed": 11, "revise": True}

    def run(seed):
        st = O.noise_canvas(seed, 1, cfg.canvas, cfg.vocab)
        final = {}
        hist = []
        while not st["done"][0]:
            new, info = O.canvas_step(cfg, om, st, kc, vc, cl, 0.0, cfg.max_steps,
                                      sampler=dict(smp, seed=seed))
            inf = info[0]
            assert inf["selected"].sum() == 1 or int(st["step"][0]) == cfg.max_steps - 1
            for i, t in final.items():                    # final positions never change
                assert new["tokens"][0, i] == t
            rows = inf["rows"]
            np.testing.assert_array_equal(new["tokens"][0, rows], inf["argmax"])
            assert abs(inf["tau"] - O.temperature(int(st["step"][0]), cfg.max_steps, 1.0, 0.5)) == 0
            for i in np.nonzero(inf["selected"])[0]:
                final[int(i)] = int(new["tokens"][0, i])
            hist.append(new["tokens"].copy())
            st = new
        assert int(st["step"][0]) <= cfg.max_steps and int(st["n_masked"][0]) == 0
        return np.stack(hist)

    h1, h2, h3 = run(11), run(11), run(12)
    np.testing.assert_array_equal(h1, h2)
    assert not np.array_equal(h1[-1], h3[-1])


def test_ar_step_one_token_at_a_time_equals_one_append(tiny):
    """Autoregressive mode: feeding a sequence token by token gives the same cache as one
    append of the whole sequence (causal attention sees only earlier tokens), and the last step's
    logits equal the LM head on the last row of a single full-depth encode of the sequence;
    greedy picks their argmax."""
    cfg, om, kc0, vc0, cl0 = tiny
    toks = np.array([[3, 200, 17, 511, 0, 42]], dtype=np.int32)
    ka, va = kc0.copy(), vc0.copy()
    la = np.array(cl0, copy=True)
    for j in range(toks.shape[1]):
        nxt, H, _, la, z = O.ar_step(cfg, om, toks[:, j:j + 1], ka, va, la)
    kb, vb = kc0.copy(), vc0.copy()
    last = []
    lb = O.kv_append(cfg, om, toks, kb, vb, cl0, None, None, last)
    np.testing.assert_array_equal(la, lb)
    np.testing.assert_allclose(ka, kb, rtol=0, atol=1e-12)
    np.testing.assert_allclose(va, vb, rtol=0, atol=1e-12)
    Hb, amb, _, zb = O.lm_head_rows(cfg, om, np.stack(last), keep_logits=True)
    np.testing.assert_allclose(z, zb, rtol=0, atol=1e-11)
    assert nxt[0] == amb[0] == int(np.argmax(z[0]))
    # the plain append (no LM head) writes the same cache as the AR mode
    kc2, vc2 = kc0.copy(), vc0.copy()
    O.kv_append(cfg, om, toks, kc2, vc2, cl0)
    np.testing.assert_array_equal(kc2, kb)


def test_ar_step_sampling_uses_the_position_stream(tiny):
    cfg, om, kc, vc, cl = tiny
    toks = np.array([[5]], dtype=np.int32)
    nxt, H, _, _, z = O.ar_step(cfg, om, toks, kc.copy(), vc.copy(), cl, tau=0.8, seed=21)
    p = int(cl[0]) + 1
    g = O.gumbel(O.stream_words(21, O.TAG_AR, 0, p, 0, cfg.vocab))
    zs = z[0] * float(O.inv_temperature(0.8))
    assert nxt[0] == int(np.argmax(zs + g))
    pz = np.exp(zs - zs.max()); pz /= pz.sum()
    assert abs(H[0] + (pz * np.log(pz)).sum()) < 1e-5
