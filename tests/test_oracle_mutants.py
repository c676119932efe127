"""Mutation checks of the oracle's pins (CPU only).

Each case plants one plausible mistake in a single oracle function: a dropped term, a wrong sign,
index or constant, a transposed operand, a tie broken the other way. The mistake lives only for
the duration of the case, patched into the oracle module on the CPU. The case then runs the pins
that cover that function, and at least one of them must fail. A planted mistake that every pin
accepts would be a blind spot in the pins.

Only mistakes against what the pages or the mathematics fix are planted. Readings that are free
choices (e.g. how a noise token is drawn from a uniform word) are held by the bit-exact device
parity tests instead.
"""
import math

import numpy as np
import pytest

import synth
from oracle import dg_oracle as O
import test_oracle_pins as P
import test_oracle_sampler as S


def _tiny():
    """The tiny workload in the form test_oracle_pins' fixture gives it."""
    cfg = synth.get_config("tiny")
    m = synth.make_model(cfg, "cpu")
    arr = {"emb": synth.to_numpy(m["emb"]),
           "layers": [{k: synth.to_numpy(v) for k, v in lay.items()} for lay in m["layers"]]}
    return cfg, O.OracleModel(cfg, arr), synth.make_prompt_kv(cfg, "cpu")


# ----------------------------------------------------------------- number formats

def m_round_bf16_truncates(orig):
    def f(x):
        x = np.asarray(x, dtype=np.float64)
        _, e = np.frexp(x)
        q = np.ldexp(1.0, np.maximum(e, -125) - 8)
        return np.where(np.isfinite(x), np.trunc(x / q) * q, x)
    return f


def m_round_bf16_ties_away(orig):
    def f(x):
        x = np.asarray(x, dtype=np.float64)
        _, e = np.frexp(x)
        q = np.ldexp(1.0, np.maximum(e, -125) - 8)
        return np.where(np.isfinite(x), np.sign(x) * np.floor(np.abs(x) / q + 0.5) * q, x)
    return f


def m_e4m3_bias_8(orig):
    return lambda codes: orig(codes) * 0.5          # exponent bias 8 halves every finite value


def m_e4m3_scale_on_columns(orig):
    def f(arr, kind, scale=None):
        if kind != "e4m3":
            return orig(arr, kind, scale)
        v = O.e4m3_to_f64(arr)
        return v * np.resize(np.asarray(scale, dtype=np.float64), v.shape[-1])
    return f


def m_e2m1_subnormal_unhalved(orig):
    def f(codes):
        c = np.asarray(codes, dtype=np.uint8).astype(np.int64) & 0xF
        v = orig(codes)
        return np.where(((c >> 1) & 3) == 0, 2.0 * v, v)
    return f


def m_nvfp4_nibbles_swapped(orig):
    def f(codes, scales, tensor_scale, rows):
        c = np.asarray(codes, dtype=np.uint8)
        return orig(((c & 0xF) << 4 | (c >> 4)).astype(np.uint8), scales, tensor_scale, rows)
    return f


def m_nvfp4_scale_blocks_reversed(orig):
    return lambda codes, scales, ts, rows: orig(codes, np.ascontiguousarray(scales[..., ::-1]),
                                                ts, rows)


# ----------------------------------------------------------------- layer pieces

def m_rmsnorm_mean_abs(orig):
    def f(x, eps):
        x = np.asarray(x, dtype=np.float64)
        return x / (np.mean(np.abs(x), axis=-1, keepdims=True) + eps)
    return f


def m_rmsnorm_eps_outside_sqrt(orig):
    def f(x, eps):
        x = np.asarray(x, dtype=np.float64)
        return x / (np.sqrt(np.mean(x * x, axis=-1, keepdims=True)) + eps)
    return f


def m_gelu_coefficient(orig):
    return lambda x: 0.5 * x * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (x + 0.0447 * x ** 3)))


def m_gelu_sigmoid_form(orig):
    return lambda x: x / (1.0 + np.exp(-1.702 * x))


def m_rope_rotates_backwards(orig):
    return lambda x, pos, theta: orig(x, -np.asarray(pos, dtype=np.float64), theta)


def m_rope_half_frequency_exponent(orig):
    return lambda x, pos, theta: orig(x, pos, math.sqrt(theta))   # theta^(-i/hd), not -2i/hd


def m_attention_unscaled(orig):
    def f(q, kc, vc, kn, vn, causal):
        q = np.asarray(q, dtype=np.float64)
        return orig(q * math.sqrt(q.shape[-1]), kc, vc, kn, vn, causal)
    return f


def m_attention_causal_masks_diagonal(orig):
    def f(q, kc, vc, kn, vn, causal):
        if not causal:
            return orig(q, kc, vc, kn, vn, causal)
        T, Hq, hd = q.shape
        Hkv = kc.shape[0]
        out = np.empty((T, Hq, hd))
        for i in range(T):                    # query i sees the cache and canvas keys j < i only
            if i == 0:
                out[i] = orig(q[:1], kc, vc, kn[:0], vn[:0], False)[0]
            else:
                kc2 = np.concatenate([kc, np.asarray(kn[:i]).transpose(1, 0, 2)], axis=1)
                vc2 = np.concatenate([vc, np.asarray(vn[:i]).transpose(1, 0, 2)], axis=1)
                out[i] = orig(q[i:i + 1], kc2, vc2, np.zeros((0, Hkv, hd)),
                              np.zeros((0, Hkv, hd)), False)[0]
        return out
    return f


def m_attention_gqa_modulo(orig):
    def f(q, kc, vc, kn, vn, causal):
        T, Hq, hd = q.shape
        Hkv = kc.shape[0]
        rep = Hq // Hkv
        # query head h reads kv head h % Hkv instead of h // rep
        pi = np.array([(h % Hkv) * rep + h // Hkv for h in range(Hq)])
        q2 = np.empty((T, Hq, hd))
        q2[:, pi] = q
        return orig(q2, kc, vc, kn, vn, causal)[:, pi]
    return f


# ----------------------------------------------------------------- router, experts, entropy

def _softmax_rows(z):
    p = np.exp(z - z.max(axis=1, keepdims=True))
    return p / p.sum(axis=1, keepdims=True)


def m_router_not_renormalised(orig):
    def f(y, w_r, top_k, forced=None):
        idx, _, z = orig(y, w_r, top_k, forced)
        return idx, np.take_along_axis(_softmax_rows(z), idx.astype(np.int64), axis=1), z
    return f


def m_router_ties_to_higher_index(orig):
    def f(y, w_r, top_k, forced=None):
        if forced is not None:
            return orig(y, w_r, top_k, forced)
        z = np.asarray(y, dtype=np.float64) @ np.asarray(w_r, dtype=np.float64).T
        p = _softmax_rows(z)
        E = p.shape[1]
        idx = (E - 1 - np.argsort(-p[:, ::-1], axis=1, kind="stable"))[:, :top_k]
        gp = np.take_along_axis(p, idx, axis=1)
        return idx.astype(np.int32), gp / gp.sum(axis=1, keepdims=True), z
    return f


def m_moe_gate_up_swapped(orig):
    def f(y, idx, gates, expert_w, residual, act):
        def swapped(e):
            w_gu, w_d = expert_w(e)
            F = w_d.shape[1]
            return np.concatenate([w_gu[F:], w_gu[:F]]), w_d
        return orig(y, idx, gates, swapped, residual, act)
    return f


def m_moe_gates_ignored(orig):
    return lambda y, idx, gates, ew, res, act: orig(y, idx, np.ones_like(gates), ew, res, act)


def m_moe_residual_dropped(orig):
    return lambda y, idx, gates, ew, res, act: orig(y, idx, gates, ew, np.zeros_like(res), act)


def m_entropy_in_bits(orig):
    def f(z):
        H, am, margin = orig(z)
        return H / math.log(2.0), am, margin
    return f


def m_argmax_ties_to_last(orig):
    def f(z):
        H, _, margin = orig(z)
        z = np.asarray(z)
        am = (z.shape[1] - 1 - np.argmax(z[:, ::-1], axis=1)).astype(np.int32)
        return H, am, margin
    return f


# ----------------------------------------------------------------- EB sampler

def _eb_variant(include_kth: bool, ties_to_higher: bool):
    """eb_select with one of two planted mistakes: the bound applied to the sum that includes the
    k-th entropy, or equal entropies ordered by the higher position first."""
    def f(H, masked, gamma, force_all):
        H = np.asarray(H, dtype=np.float32)
        cand = np.nonzero(np.asarray(masked) != 0)[0]
        sel = np.zeros(len(masked), dtype=bool)
        if len(cand) == 0:
            return sel
        if not np.all(np.isfinite(H[cand])):
            raise FloatingPointError("non-finite entropy")
        hv = np.maximum(H[cand].astype(np.float64), 0.0)
        sign = -1 if ties_to_higher else 1
        order = sorted(range(len(cand)), key=lambda i: (hv[i], sign * int(cand[i])))
        if force_all:
            sel[cand] = True
            return sel
        qg = O.eb_quantize_bound(gamma)
        k, prefix = 1, 0
        for j in range(1, len(order)):
            prefix += O.eb_quantize(np.float32(hv[order[j - 1]]))
            extra = O.eb_quantize(np.float32(hv[order[j]])) if include_kth else 0
            if prefix + extra <= qg:
                k = j + 1
            else:
                break
        sel[cand[[order[i] for i in range(k)]]] = True
        return sel
    return f


def m_eb_includes_kth(orig):
    return _eb_variant(True, False)


def m_eb_ties_to_higher_position(orig):
    return _eb_variant(False, True)


def m_eb_quantize_floor(orig):
    return lambda h: int(np.floor(np.float64(h) * 2.0 ** O.EB_FRAC_BITS))


# ----------------------------------------------------------------- sampler variants

def m_uniform_24_bits(orig):
    return lambda words: ((np.asarray(words, dtype=np.uint64) >> np.uint64(8)).astype(np.float64)
                          + 0.5) * 2.0 ** -24


def m_temperature_over_n(orig):
    def f(step, max_steps, tau_start, tau_end):
        frac = min(int(step), max_steps - 1) / max(max_steps, 1)
        return tau_start + (tau_end - tau_start) * frac
    return f


def m_gumbel_subtracted(orig):
    return lambda z, tau, g: orig(z, tau, None if g is None else -np.asarray(g))


def m_gumbel_sign(orig):
    return lambda words: np.log(-np.log(O.uniform_open(words)))


def m_sample_row_multiplies_by_tau(orig):
    return lambda z, tau, g: orig(z, 1.0 / tau if tau > 0.0 else tau, g)


# ----------------------------------------------------------------- the step and the append

def m_append_sees_later_tokens(orig):
    return lambda cfg, model, l, x, q, k, v, kc, vc, causal, *a, **kw: orig(
        cfg, model, l, x, q, k, v, kc, vc, False, *a, **kw)


def m_append_positions_from_zero(orig):
    def f(cfg, model, l, x, pos):
        p = np.asarray(pos)
        return orig(cfg, model, l, x, p - p[0])
    return f


def m_step_cap_one_late(orig):
    return lambda cfg, model, state, kc, vc, cl, gamma, max_steps, *a, **kw: orig(
        cfg, model, state, kc, vc, cl, gamma, max_steps + 1, *a, **kw)


def m_commit_indexes_argmax_by_position(orig):
    # the committed token read from the argmax list at the canvas position, not at the row index
    def f(cfg, model, state, kc, vc, cl, gamma, max_steps, *a, **kw):
        new, infos = orig(cfg, model, state, kc, vc, cl, gamma, max_steps, *a, **kw)
        for b, info in enumerate(infos):
            if info and "selected" in info:
                pos = np.nonzero(info["selected"])[0]
                am = info["argmax"]
                new["tokens"][b, pos] = am[np.minimum(pos, len(am) - 1)]
        return new, infos
    return f


# ----------------------------------------------------------------- the cases

_TINY = []


def _tiny_once():
    if not _TINY:
        _TINY.append(_tiny())
    return _TINY[0]


def _eb_golden_pins():
    return [(P.test_eb_hand_worked, (c,)) for c in P._golden_eb()]


def _kat_pins():
    return [(S.test_philox_known_answer_vectors, (r,)) for r in S._kat()]


ROUND = [(P.test_round_bf16_matches_torch_conversion, ()),
         (P.test_round_bf16_halfway_ties_to_even, ())]
E4M3 = [(P.test_e4m3_decode_all_codes_vs_torch, ()),
        (P.test_e4m3_channel_scale_lands_on_output_rows_hand_built, ()),
        (P.test_e4m3_decode_recovers_the_fp32_draw_within_one_step, ())]
NVFP4 = [(P.test_e2m1_decode_all_codes_vs_ml_dtypes, ()),
         (P.test_nvfp4_rows_hand_built_layout, ()),
         (P.test_nvfp4_rows_random_vs_library_decoders, ())]
ATTN = [(P.test_attention_brute_force, (False,)), (P.test_attention_brute_force, (True,)),
        (P.test_attention_vs_torch_sdpa_gqa, ()), (P.test_attention_special_cases, ())]
ROUTER = [(P.test_router_uniform_ties_and_brute_force, ()),
          (P.test_router_forced_choice_renormalises_this_routers_probabilities, ())]
MOE = [(P.test_moe_k_equals_E_uniform_gates_is_dense_mean, ()),
       (P.test_moe_single_expert_is_plain_gated_ffn, ()),
       (P.test_shared_expert_adds_a_plain_gated_ffn, ())]
ENTROPY = [(P.test_entropy_closed_forms, ()), (P.test_entropy_random_rows_vs_scipy, ())]
EB = [(P.test_eb_bound_zero_commits_lowest_single, ()),
      (P.test_eb_brute_force_prefix_enumeration, ())]
SAMPLER = [(S.test_temperature_schedule_endpoints_and_greedy, ()),
           (S.test_entropy_at_temperature_closed_forms, ()),
           (S.test_uniform_is_exact_and_open_and_gumbel_moments, ())]

# (case, oracle attribute, replacement factory, the pins that cover it)
MUTANTS = [
    ("bf16 rounding truncates", "round_bf16", m_round_bf16_truncates, ROUND),
    ("bf16 ties away from zero", "round_bf16", m_round_bf16_ties_away, ROUND),
    ("e4m3 exponent bias 8", "e4m3_to_f64", m_e4m3_bias_8, E4M3),
    ("e4m3 scale along columns", "decode_weight", m_e4m3_scale_on_columns, E4M3),
    ("e2m1 subnormal not halved", "e2m1_to_f64", m_e2m1_subnormal_unhalved, NVFP4),
    ("nvfp4 nibble order swapped", "nvfp4_rows", m_nvfp4_nibbles_swapped, NVFP4),
    ("nvfp4 block scales reversed", "nvfp4_rows", m_nvfp4_scale_blocks_reversed, NVFP4),
    ("rmsnorm by mean |x|", "rmsnorm", m_rmsnorm_mean_abs,
     [(P.test_rmsnorm_unit_rms_scale_invariance_and_torch, ())]),
    ("rmsnorm eps outside the root", "rmsnorm", m_rmsnorm_eps_outside_sqrt,
     [(P.test_rmsnorm_unit_rms_scale_invariance_and_torch, ())]),
    ("gelu cubic coefficient", "gelu_tanh", m_gelu_coefficient,
     [(P.test_gelu_tanh_vs_torch_and_limits, ())]),
    ("gelu sigmoid form", "gelu_tanh", m_gelu_sigmoid_form,
     [(P.test_gelu_tanh_vs_torch_and_limits, ())]),
    ("rope rotates backwards", "rope", m_rope_rotates_backwards,
     [(P.test_rope_matches_complex_rotation_and_relative_position, ())]),
    ("rope frequency exponent halved", "rope", m_rope_half_frequency_exponent,
     [(P.test_rope_matches_complex_rotation_and_relative_position, ())]),
    ("attention without 1/sqrt(hd)", "attention", m_attention_unscaled, ATTN),
    ("causal mask hides the diagonal", "attention", m_attention_causal_masks_diagonal, ATTN),
    ("GQA head h reads kv h % Hkv", "attention", m_attention_gqa_modulo, ATTN),
    ("router gates not renormalised", "router_topk", m_router_not_renormalised, ROUTER),
    ("router ties to the higher expert", "router_topk", m_router_ties_to_higher_index, ROUTER),
    ("expert gate and up swapped", "moe_ffn", m_moe_gate_up_swapped, MOE),
    ("expert gates ignored", "moe_ffn", m_moe_gates_ignored, MOE),
    ("expert residual dropped", "moe_ffn", m_moe_residual_dropped, MOE),
    ("entropy in bits", "entropy_argmax", m_entropy_in_bits, ENTROPY),
    ("argmax ties to the last index", "entropy_argmax", m_argmax_ties_to_last,
     ENTROPY + [(P.test_tiny_zero_lm_head_gives_ln_v_and_index_order, (_tiny_once,))]),
    ("EB bound includes the k-th entropy", "eb_select", m_eb_includes_kth,
     EB + [("golden", None)]),
    ("EB ties to the higher position", "eb_select", m_eb_ties_to_higher_position,
     EB + [("golden", None)]),
    ("EB entropies floored", "eb_quantize", m_eb_quantize_floor,
     [(P.test_eb_fixed_point_quantisers_exact_rational, ())]),
    ("Philox key increment W0 off by one", "PHILOX_W0", lambda v: v - 1, [("kat", None)]),
    ("Philox multipliers swapped", "PHILOX_M0", lambda v: O.PHILOX_M1, [("kat", None)]),
    ("uniform from 24 bits", "uniform_open", m_uniform_24_bits, SAMPLER),
    ("temperature over N, not N - 1", "temperature", m_temperature_over_n, SAMPLER),
    ("logits times tau", "sample_row", m_sample_row_multiplies_by_tau,
     SAMPLER + [(S.test_gumbel_max_draw_follows_softmax_at_temperature, ())]),
    ("Gumbel noise subtracted", "sample_row", m_gumbel_subtracted,
     [(S.test_gumbel_max_draw_follows_softmax_at_temperature, ())]),
    ("Gumbel transform sign flipped", "gumbel", m_gumbel_sign, SAMPLER),
    ("append attends to later tokens", "layer_rest", m_append_sees_later_tokens,
     [(P.test_append_is_a_causal_encoder_two_layers, ())]),
    ("positions ignore the cache length", "layer_qkv", m_append_positions_from_zero,
     [(P.test_tiny_kv_append_single_layer_is_direct_projection, (_tiny_once,))]),
    ("step cap one step late", "canvas_step", m_step_cap_one_late,
     [(P.test_tiny_infinite_bound_and_step_cap, (_tiny_once,))]),
    ("commit reads the argmax at the position", "canvas_step",
     m_commit_indexes_argmax_by_position,
     [(P.test_tiny_commit_writes_each_rows_own_argmax, (_tiny_once,))]),
]


def _expand(pins):
    out = []
    for fn, args in pins:
        if fn == "golden":
            out += _eb_golden_pins()
        elif fn == "kat":
            out += _kat_pins()
        else:
            out.append((fn, args))
    return out


def _fails(fn, args) -> bool:
    args = tuple(a() if callable(a) and a is _tiny_once else a for a in args)
    try:
        fn(*args)
    except (Exception, pytest.fail.Exception):
        return True
    return False


@pytest.mark.parametrize("case", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_a_planted_mistake_fails_a_pin(case, monkeypatch):
    name, attr, make, pins = case
    monkeypatch.setattr(O, attr, make(getattr(O, attr)))
    caught = [fn.__name__ for fn, args in _expand(pins) if _fails(fn, args)]
    assert caught, f"no pin caught the planted mistake: {name}"


def test_the_unmutated_oracle_passes_the_same_pins():
    """The pins the cases run all pass on the oracle as it is, so every failure above comes from
    the planted mistake."""
    seen = set()
    for _, _, _, pins in MUTANTS:
        for fn, args in _expand(pins):
            key = (fn.__name__, repr(args))
            if key in seen:
                continue
            seen.add(key)
            assert not _fails(fn, args), fn.__name__
