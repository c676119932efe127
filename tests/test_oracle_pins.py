"""CPU pins of the oracle: each function is checked against something other
than itself — a library routine for a special case, a closed form, an
invariant, brute force on tiny inputs, or hand-worked values
(tests/golden/).  These run without a GPU."""
import itertools
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import dg_oracle as O
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(1234)


# ----------------------------------------------------------------- number formats

def test_round_bf16_matches_torch_conversion():
    x32 = np.concatenate([
        rng.standard_normal(20000).astype(np.float32),
        (rng.standard_normal(2000) * 1e-39).astype(np.float32),   # subnormals
        np.clip(rng.standard_normal(2000) * 3e38, -3.39e38, 3.39e38).astype(np.float32),  # near overflow
        np.array([0.0, -0.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 3.3895313892515355e38], np.float32),
    ])
    ref = torch.from_numpy(x32).to(torch.bfloat16).to(torch.float64).numpy()
    got = O.round_bf16(x32.astype(np.float64))
    np.testing.assert_array_equal(got, ref)


def test_round_bf16_halfway_ties_to_even():
    assert O.round_bf16(np.array(1.0 + 2 ** -8)) == 1.0            # tie -> even (1.0)
    assert O.round_bf16(np.array(1.0 + 3 * 2 ** -8)) == 1.0 + 2 ** -6
    assert O.round_bf16(np.array(1.0 + 2 ** -8 + 2 ** -30)) == 1.0 + 2 ** -7


def test_bf16_bits_roundtrip():
    vals = np.array([0x3F80, 0xBF80, 0x0001, 0x7F7F, 0x4049], dtype=np.uint16)
    got = O.bf16_bits_to_f64(vals)
    ref = torch.from_numpy(vals.view(np.int16)).view(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(got, ref)
    assert got[0] == 1.0 and got[1] == -1.0 and got[2] == 2.0 ** -133


def test_e4m3_decode_all_codes_vs_torch():
    codes = np.arange(256, dtype=np.uint8)
    got = O.e4m3_to_f64(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan) and nan.sum() == 2
    np.testing.assert_array_equal(got[~nan], ref[~nan])
    # OCP FP8 spec values worked by hand
    assert got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9 and got[0x08] == 2.0 ** -6
    assert got[0x38] == 1.0 and got[0xB8] == -1.0


def test_e4m3_channel_scale_lands_on_output_rows_hand_built():
    """decode_weight's per-channel scale multiplies each OUTPUT channel (row of a [out][in]
    matrix; for a stacked [E][out][in] expert tensor, scale [E][out]).  Hand-worked values: OCP
    E4M3 codes 0x38 = 1.0, 0x40 = 2.0, 0x30 = 0.5, 0xB8 = -1.0 (sign bit), 0x01 = 2^-9 (the
    smallest subnormal), with a non-square 2 x 3 matrix so a column-wise scale cannot broadcast."""
    codes = np.array([[0x38, 0x40, 0x30], [0xB8, 0x01, 0x40]], np.uint8)
    scale = np.array([2.0, 0.25], np.float32)
    want = np.array([[2.0, 4.0, 1.0], [-0.25, 0.25 * 2.0 ** -9, 0.5]])
    np.testing.assert_array_equal(O.decode_weight(codes, "e4m3", scale), want)
    stacked = np.stack([codes, codes[::-1]])                      # [E=2][out=2][in=3]
    sc = np.array([[2.0, 0.25], [8.0, 1.0]], np.float32)          # [E][out]
    got = O.decode_weight(stacked, "e4m3", sc)
    np.testing.assert_array_equal(got[0], want)
    np.testing.assert_array_equal(got[1], np.array([[-8.0, 8.0 * 2.0 ** -9, 16.0],
                                                    [1.0, 2.0, 0.5]]))


def test_e4m3_decode_recovers_the_fp32_draw_within_one_step():
    """The stored e4m3 weights of the batched workload, decoded by the oracle, reproduce the fp32
    values they were drawn from within half an e4m3 step: |w - w32| <= 2^-4 |w32| for normals
    (3 mantissa bits) plus half the subnormal quantum 2^-10 * scale.  Rows differ in magnitude by
    up to 10^3 and the matrix is not square, so a scale applied along the wrong axis fails."""
    g = torch.Generator().manual_seed(7)
    w32 = torch.randn((6, 40), generator=g) * torch.tensor([1e-3, 1.0, 0.02, 5.0, 0.3, 2e-2])[:, None]
    codes, scale = synth._store_weight(w32, "e4m3")
    dec = O.decode_weight(synth.to_numpy(codes), "e4m3", synth.to_numpy(scale))
    w = w32.double().numpy()
    sc = synth.to_numpy(scale).astype(np.float64)[:, None]
    assert (np.abs(dec - w) <= 2.0 ** -4 * np.abs(w) + 2.0 ** -10 * sc + 1e-12).all()
    # each row's largest magnitude maps to the largest finite code (448 * scale)
    np.testing.assert_allclose(np.abs(dec).max(axis=1), 448.0 * sc[:, 0], rtol=1e-6)


def test_e2m1_decode_all_codes_vs_ml_dtypes():
    ml_dtypes = pytest.importorskip("ml_dtypes")
    codes = np.arange(16, dtype=np.uint8)
    got = O.e2m1_to_f64(codes)
    ref = codes.view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    np.testing.assert_array_equal(got, ref)
    # OCP MX FP4 E2M1 values worked by hand: 0b0111 = 6, 0b0001 = 0.5 (subnormal), 0b1010 = -1
    assert got[0x7] == 6.0 and got[0x1] == 0.5 and got[0xA] == -1.0 and got[0x8] == 0.0
    # only the low nibble is a code
    assert np.array_equal(O.e2m1_to_f64(codes | 0xF0), got)


def test_round_f16_matches_struct_half_and_ties():
    """Against Python's IEEE binary16 packing of a double (struct 'e'), which rounds once; torch
    converts float64 through binary32 and can round twice near halfway points."""
    import struct
    x = rng.standard_normal(20000) * np.exp2(rng.integers(-20, 12, 20000))
    ref = np.array([struct.unpack("e", struct.pack("e", float(v)))[0] for v in x])
    np.testing.assert_array_equal(O.round_f16(x), ref)
    # halfway between 1 and 1 + 2**-10 rounds to the even 1; 65520 (halfway past the largest
    # finite 65504) overflows to inf; 2**-25 (half the smallest subnormal) rounds to 0
    assert O.round_f16(np.array([1 + 2.0 ** -11]))[0] == 1.0
    assert np.isinf(O.round_f16(np.array([65520.0]))[0])
    assert O.round_f16(np.array([2.0 ** -25]))[0] == 0.0


def test_nvfp4_rows_hand_built_layout():
    """Four nonzero elements placed by hand: nibble order, k-block and 16-element scale block."""
    d, R = 128, 3
    codes = np.zeros((d // 64, R, 32), np.uint8)
    scales = np.full((d // 64, R, 4), 0x38, np.uint8)      # 1.0 everywhere
    codes[1, 2, 5] = 0x4A     # row 2, elements 64+10 (low nibble 0xA = -1), 64+11 (0x4 = 2)
    scales[1, 2, 0] = 0x40    # row 2, elements 64..79: scale 2
    codes[0, 0, 31] = 0x17    # row 0, elements 62 (0x7 = 6), 63 (0x1 = 0.5)
    scales[0, 0, 3] = 0x30    # row 0, elements 48..63: scale 0.5
    got = O.nvfp4_rows(codes, scales, 0.25, np.arange(R))
    want = np.zeros((R, d))
    want[2, 74], want[2, 75] = -1.0 * 2.0 * 0.25, 2.0 * 2.0 * 0.25
    want[0, 62], want[0, 63] = 6.0 * 0.5 * 0.25, 0.5 * 0.5 * 0.25
    np.testing.assert_array_equal(got, want)
    # row selection and order
    np.testing.assert_array_equal(O.nvfp4_rows(codes, scales, 0.25, np.array([2, 0])),
                                  want[[2, 0]])


def test_nvfp4_rows_random_vs_library_decoders():
    ml_dtypes = pytest.importorskip("ml_dtypes")
    g = np.random.default_rng(7)
    d, R = 256, 5
    codes = g.integers(0, 256, (d // 64, R, 32), dtype=np.uint8)
    scales = g.integers(0, 0x7F, (d // 64, R, 4), dtype=np.uint8)   # every finite positive E4M3
    got = O.nvfp4_rows(codes, scales, 0.37, np.arange(R))
    nib = np.stack([codes & 0xF, codes >> 4], axis=-1).reshape(d // 64, R, 64)
    el = nib.astype(np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    sc = torch.from_numpy(scales.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    want = (el * np.repeat(sc, 16, axis=-1) * 0.37).transpose(1, 0, 2).reshape(R, d)
    np.testing.assert_array_equal(got, want)


def test_nvfp4_model_matches_bf16_model_with_the_same_values():
    """With a power-of-two tensor scale every NVFP4 element is exactly a bf16 value, so the
    oracle's NVFP4 embedding / LM head must reproduce the bf16 model holding those values."""
    c16 = synth.reduced("layer", vocab=300, d_model=256)
    c4 = synth.reduced("layer", vocab=300, d_model=256, emb="nvfp4")
    gen = torch.Generator()
    gen.manual_seed(3)
    codes, scales, _ = synth.make_nvfp4_emb(gen, c4.vocab + 1, c4.d_model, 0.02, "cpu")
    codes, scales = codes.numpy(), scales.numpy()
    assert codes.shape == (4, 512, 32) and scales.shape == (4, 512, 4)
    assert not codes[:, 301:].any() and not scales[:, 301:].any()
    ts = 2.0 ** -7
    dense = O.nvfp4_rows(codes, scales, ts, np.arange(c4.vocab + 1))
    assert np.array_equal(O.round_bf16(dense), dense)
    bits = torch.from_numpy(dense.astype(np.float32)).to(torch.bfloat16).view(torch.int16)
    m16 = O.OracleModel(c16, {"emb": bits.numpy().view(np.uint16), "layers": []})
    m4 = O.OracleModel(c4, {"emb": codes, "emb_scale": scales, "emb_scale_global": ts,
                            "layers": []})
    ids = np.array([0, 7, 299, 300])
    np.testing.assert_array_equal(m4.emb_rows(ids), m16.emb_rows(ids))
    for (v0, w16), (v1, w4) in zip(m16.lm_head_chunks(128), m4.lm_head_chunks(128)):
        assert v0 == v1
        np.testing.assert_array_equal(w4, w16)
    # the NVFP4 LM head stores its normalised rows in fp16 (the bf16 one in bf16)
    x = rng.standard_normal((6, c4.d_model))
    f = O.round_f16(O.rmsnorm(x, c4.rms_eps))
    H, am, _, z = O.lm_head_rows(c4, m4, x, keep_logits=True)
    np.testing.assert_array_equal(z, f @ dense[:c4.vocab].T)
    H2, am2, _ = O.entropy_argmax(z)
    np.testing.assert_array_equal(H, H2)
    np.testing.assert_array_equal(am, am2)


# ----------------------------------------------------------------- layer pieces

def test_rmsnorm_unit_rms_scale_invariance_and_torch():
    x = rng.standard_normal((7, 96))
    y = O.rmsnorm(x, 0.0)
    np.testing.assert_allclose(np.sqrt((y * y).mean(-1)), 1.0, rtol=1e-14)
    np.testing.assert_allclose(O.rmsnorm(5.0 * x, 0.0), y, rtol=1e-13)
    ref = torch.nn.functional.rms_norm(torch.from_numpy(x), (96,), eps=1e-6).numpy()
    np.testing.assert_allclose(O.rmsnorm(x, 1e-6), ref, rtol=1e-12)


def test_gelu_tanh_vs_torch_and_limits():
    x = np.linspace(-8, 8, 1001)
    ref = torch.nn.functional.gelu(torch.from_numpy(x), approximate="tanh").numpy()
    np.testing.assert_allclose(O.gelu_tanh(x), ref, rtol=1e-12, atol=1e-15)
    assert O.gelu_tanh(np.array(0.0)) == 0.0
    assert abs(O.gelu_tanh(np.array(30.0)) - 30.0) < 1e-12


def test_rope_matches_complex_rotation_and_relative_position():
    T, H, hd, theta = 5, 3, 16, 10000.0
    x = rng.standard_normal((T, H, hd))
    pos = np.array([0, 1, 7, 4096, 131071])
    got = O.rope(x, pos, theta)
    half = hd // 2
    zc = x[..., :half] + 1j * x[..., half:]
    freqs = np.array([theta ** (-(2 * i) / hd) for i in range(half)])
    rot = zc * np.exp(1j * pos[:, None, None] * freqs[None, None, :])
    np.testing.assert_allclose(got[..., :half], rot.real, atol=1e-12)
    np.testing.assert_allclose(got[..., half:], rot.imag, atol=1e-12)
    np.testing.assert_allclose(np.linalg.norm(got, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-12)
    q, k = rng.standard_normal((1, 1, hd)), rng.standard_normal((1, 1, hd))
    d1 = (O.rope(q, np.array([10]), theta) * O.rope(k, np.array([3]), theta)).sum()
    d2 = (O.rope(q, np.array([107]), theta) * O.rope(k, np.array([100]), theta)).sum()
    assert abs(d1 - d2) < 1e-10


def _brute_attention(q, kc, vc, kn, vn, causal):
    T, Hq, hd = q.shape
    Hkv, P, _ = kc.shape
    out = np.zeros_like(q)
    for i in range(T):
        for h in range(Hq):
            g = h // (Hq // Hkv)
            keys, vals = [], []
            for j in range(P):
                keys.append(kc[g, j]); vals.append(vc[g, j])
            for j in range(T):
                if causal and j > i:
                    continue
                keys.append(kn[j, g]); vals.append(vn[j, g])
            s = [sum(q[i, h, d] * kk[d] for d in range(hd)) / math.sqrt(hd) for kk in keys]
            m = max(s)
            w = [math.exp(v - m) for v in s]
            tot = sum(w)
            for d in range(hd):
                out[i, h, d] = sum(w[n] * vals[n][d] for n in range(len(w))) / tot
    return out


@pytest.mark.parametrize("causal", [False, True])
def test_attention_brute_force(causal):
    T, Hq, Hkv, hd, P = 4, 4, 2, 8, 3
    q = rng.standard_normal((T, Hq, hd))
    kc, vc = rng.standard_normal((Hkv, P, hd)), rng.standard_normal((Hkv, P, hd))
    kn, vn = rng.standard_normal((T, Hkv, hd)), rng.standard_normal((T, Hkv, hd))
    got = O.attention(q, kc, vc, kn, vn, causal)
    np.testing.assert_allclose(got, _brute_attention(q, kc, vc, kn, vn, causal), atol=1e-12)


def test_attention_vs_torch_sdpa_gqa():
    T, Hq, Hkv, hd, P = 6, 4, 2, 16, 9
    q = rng.standard_normal((T, Hq, hd))
    kc, vc = rng.standard_normal((Hkv, P, hd)), rng.standard_normal((Hkv, P, hd))
    kn, vn = rng.standard_normal((T, Hkv, hd)), rng.standard_normal((T, Hkv, hd))
    K = np.concatenate([kc, kn.transpose(1, 0, 2)], axis=1)
    V = np.concatenate([vc, vn.transpose(1, 0, 2)], axis=1)
    Kr = np.repeat(K, Hq // Hkv, axis=0)
    Vr = np.repeat(V, Hq // Hkv, axis=0)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q.transpose(1, 0, 2)), torch.from_numpy(Kr), torch.from_numpy(Vr)).numpy()
    np.testing.assert_allclose(O.attention(q, kc, vc, kn, vn, False), ref.transpose(1, 0, 2), atol=1e-12)


def test_attention_special_cases():
    hd = 8
    q = rng.standard_normal((1, 1, hd))
    v = rng.standard_normal((1, 1, hd))
    k = rng.standard_normal((1, 1, hd))
    empty = np.zeros((1, 0, hd))
    # single key returns its value
    np.testing.assert_allclose(O.attention(q, empty, empty, k, v, False)[0, 0], v[0, 0], atol=1e-14)
    # all-equal keys return the mean of the values
    kc = np.repeat(k[0][:, None, :], 5, axis=1)          # [1, 5, hd]
    vc = rng.standard_normal((1, 5, hd))
    got = O.attention(q, kc, vc, k, v, False)[0, 0]
    np.testing.assert_allclose(got, np.concatenate([vc[0], v[0]]).mean(0), atol=1e-13)
    # duplicating every key/value leaves the output unchanged
    q2 = rng.standard_normal((3, 2, hd))
    kc2, vc2 = rng.standard_normal((1, 4, hd)), rng.standard_normal((1, 4, hd))
    kn2, vn2 = rng.standard_normal((3, 1, hd)), rng.standard_normal((3, 1, hd))
    a = O.attention(q2, kc2, vc2, kn2, vn2, False)
    b = O.attention(q2, np.concatenate([kc2, kc2, kn2.transpose(1, 0, 2)], 1),
                    np.concatenate([vc2, vc2, vn2.transpose(1, 0, 2)], 1), kn2, vn2, False)
    np.testing.assert_allclose(a, b, atol=1e-13)


def test_router_uniform_ties_and_brute_force():
    T, d, E = 5, 12, 8
    y = rng.standard_normal((T, d))
    idx, g, z = O.router_topk(y, np.zeros((E, d)), E)
    np.testing.assert_allclose(g, 1.0 / E)
    assert (idx == np.arange(E)).all()                    # all tied: lower index first
    idx, g, z = O.router_topk(y, np.zeros((E, d)), 3)
    assert (idx == np.arange(3)).all()
    w = rng.standard_normal((E, d))
    idx, g, z = O.router_topk(y, w, 3)
    np.testing.assert_allclose(g.sum(1), 1.0, rtol=1e-14)
    for t in range(T):
        logits = [float(np.dot(y[t], w[e])) for e in range(E)]
        best = sorted(range(E), key=lambda e: (-logits[e], e))[:3]
        assert list(idx[t]) == best
        ex = [math.exp(logits[e]) for e in best]
        np.testing.assert_allclose(g[t], np.array(ex) / sum(ex), rtol=1e-12)


def _experts(E, F, d):
    return [(rng.standard_normal((2 * F, d)) * 0.3, rng.standard_normal((d, F)) * 0.3) for _ in range(E)]


def test_router_forced_choice_renormalises_this_routers_probabilities():
    """Forced expert choices: the given experts, gated by this router's softmax renormalised over
    them (brute force per token); forcing the router's own choice changes nothing."""
    y = rng.standard_normal((5, 12))
    w = rng.standard_normal((9, 12)) * 0.3
    idx, gates, z = O.router_topk(y, w, 3)
    idx2, gates2, _ = O.router_topk(y, w, 3, forced=idx)
    np.testing.assert_array_equal(idx2, idx)
    np.testing.assert_array_equal(gates2, gates)
    forced = np.array([[8, 0, 4]] * 5)
    idx3, gates3, _ = O.router_topk(y, w, 3, forced=forced)
    np.testing.assert_array_equal(idx3, forced)
    for t in range(5):
        p = np.exp(z[t] - z[t].max())
        p /= p.sum()
        np.testing.assert_allclose(gates3[t], p[[8, 0, 4]] / p[[8, 0, 4]].sum(), rtol=1e-12)


def test_fp32_arithmetic_variant_tracks_fp64_and_restores_it(tiny):
    """The fp32-arithmetic run of the oracle (used only to derive tolerances) differs from the
    fp64 run by fp32 rounding on the fp32 workload, and leaving the context restores fp64 bit
    for bit."""
    cfg, om, kv = tiny
    kc = synth.to_numpy(kv["k"]).astype(np.float64)
    vc = synth.to_numpy(kv["v"]).astype(np.float64)
    cl = synth.to_numpy(kv["cache_len"])
    st = {k: synth.to_numpy(v) for k, v in synth.make_canvas_state(cfg, "all_mask").items()}
    _, a = O.canvas_step(cfg, om, st, kc, vc, cl, cfg.gamma, cfg.max_steps, keep_logits=True)
    with O.accumulation(np.float32):
        assert O.acc_dtype() is np.float32
        _, b = O.canvas_step(cfg, om, st, kc, vc, cl, cfg.gamma, cfg.max_steps, keep_logits=True)
    assert O.acc_dtype() is np.float64
    _, c = O.canvas_step(cfg, om, st, kc, vc, cl, cfg.gamma, cfg.max_steps, keep_logits=True)
    d = np.abs(b[0]["logits"] - a[0]["logits"]).max()
    assert 0 < d < 1e-5
    np.testing.assert_array_equal(c[0]["logits"], a[0]["logits"])


def test_moe_k_equals_E_uniform_gates_is_dense_mean():
    T, d, F, E = 6, 10, 7, 4
    y = rng.standard_normal((T, d))
    res = rng.standard_normal((T, d))
    ws = _experts(E, F, d)
    idx, g, _ = O.router_topk(y, np.zeros((E, d)), E)
    got = O.moe_ffn(y, idx, g, lambda e: ws[e], res, "f32")
    dense = np.zeros((T, d))
    for wgu, wd in ws:
        u = y @ wgu.T
        dense += (O.gelu_tanh(u[:, :F]) * u[:, F:]) @ wd.T
    np.testing.assert_allclose(got, res + dense / E, atol=1e-12)


def test_moe_single_expert_is_plain_gated_ffn():
    T, d, F = 5, 9, 6
    y = rng.standard_normal((T, d))
    res = rng.standard_normal((T, d))
    wgu, wd = _experts(1, F, d)[0]
    idx, g, _ = O.router_topk(y, rng.standard_normal((1, d)), 1)
    got = O.moe_ffn(y, idx, g, lambda e: (wgu, wd), res, "f32")
    for t in range(T):
        gate = [sum(y[t, c] * wgu[f, c] for c in range(d)) for f in range(F)]
        up = [sum(y[t, c] * wgu[F + f, c] for c in range(d)) for f in range(F)]
        act = [0.5 * gv * (1 + math.tanh(math.sqrt(2 / math.pi) * (gv + 0.044715 * gv ** 3))) * uv
               for gv, uv in zip(gate, up)]
        for c in range(d):
            want = res[t, c] + sum(act[f] * wd[c, f] for f in range(F))
            assert abs(got[t, c] - want) < 1e-12


def test_shared_expert_adds_a_plain_gated_ffn():
    """Routed experts with zero weights plus one shared expert: the MoE output is the residual
    plus the shared expert's gated FFN with gate 1, whatever the router chose (torch computes
    the FFN: gelu with the tanh approximation, float64 matmuls)."""
    T, d, F, E, k = 7, 16, 12, 4, 2
    y = rng.standard_normal((T, d))
    res = rng.standard_normal((T, d))
    w_gu = rng.standard_normal((2 * F, d)) * 0.3
    w_d = rng.standard_normal((d, F)) * 0.3
    zero = (np.zeros((2 * F, d)), np.zeros((d, F)))
    idx = rng.integers(0, E, (T, k)).astype(np.int32)
    gates = rng.uniform(0.1, 1.0, (T, k))
    idx2, gates2 = O.with_shared_experts(idx, gates, E, 1)
    assert idx2.shape == (T, k + 1) and (idx2[:, k] == E).all() and (gates2[:, k] == 1.0).all()
    assert np.array_equal(idx2[:, :k], idx) and np.array_equal(gates2[:, :k], gates)
    out = O.moe_ffn(y, idx2, gates2, lambda e: (w_gu, w_d) if e == E else zero, res, "f32")
    yt = torch.from_numpy(y)
    u = yt @ torch.from_numpy(w_gu).T
    a = torch.nn.functional.gelu(u[:, :F], approximate="tanh") * u[:, F:]
    want = torch.from_numpy(res) + a @ torch.from_numpy(w_d).T
    np.testing.assert_allclose(out, want.numpy(), rtol=1e-12, atol=1e-12)
    # no shared experts: unchanged routing
    i0, g0 = O.with_shared_experts(idx, gates, E, 0)
    assert i0 is idx and g0 is gates


def test_moe_token_permutation_equivariance():
    T, d, F, E = 8, 10, 6, 5
    y = rng.standard_normal((T, d))
    res = rng.standard_normal((T, d))
    ws = _experts(E, F, d)
    wr = rng.standard_normal((E, d))
    idx, g, _ = O.router_topk(y, wr, 2)
    a = O.moe_ffn(y, idx, g, lambda e: ws[e], res, "f32")
    p = rng.permutation(T)
    idx2, g2, _ = O.router_topk(y[p], wr, 2)
    b = O.moe_ffn(y[p], idx2, g2, lambda e: ws[e], res[p], "f32")
    np.testing.assert_allclose(b, a[p], atol=1e-13)


def test_entropy_closed_forms():
    V = 512
    H, am, _ = O.entropy_argmax(np.zeros((1, V)))
    assert abs(H[0] - math.log(V)) < 1e-12 and am[0] == 0
    z = np.zeros((1, V)); z[0, 17] = 100.0
    H, am, _ = O.entropy_argmax(z)
    eps = math.exp(-100.0)
    p1 = 1.0 / (1.0 + (V - 1) * eps)
    pr = eps * p1
    want = -(p1 * math.log(p1) + (V - 1) * pr * math.log(pr))
    assert abs(H[0] - want) < 1e-40 + 1e-9 * want and am[0] == 17
    z = np.full((1, V), -200.0); z[0, 300] = 50.0; z[0, 42] = 50.0
    H, am, margin = O.entropy_argmax(z)
    assert abs(H[0] - math.log(2.0)) < 1e-12 and am[0] == 42 and margin[0] == 0.0


def test_entropy_random_rows_vs_scipy():
    from scipy.stats import entropy as sp_entropy
    from scipy.special import softmax
    z = rng.standard_normal((4, 3000)) * 3.0
    H, am, margin = O.entropy_argmax(z)
    for r in range(4):
        assert abs(H[r] - sp_entropy(softmax(z[r]))) < 1e-10
        assert am[r] == int(np.argmax(z[r]))
        s = np.sort(z[r])
        assert margin[r] == s[-1] - s[-2]


# ----------------------------------------------------------------- EB sampler

def _golden_eb():
    cases = []
    with open(os.path.join(GOLDEN, "eb_cases.txt")) as fh:
        for line in fh:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            g, h, m, sel = [p.strip() for p in line.split("|")]
            cases.append((float(g), np.array([float(v) for v in h.split(",")], np.float32),
                          np.array([int(v) for v in m.split(",")], np.uint8),
                          [int(v) for v in sel.split(",")] if sel else []))
    return cases



def test_eb_fixed_point_quantisers_exact_rational():
    """Q(H) = nearest integer to H 2^32 (ties to even) and Q(gamma) = floor(gamma 2^32), checked
    with exact rational arithmetic on the binary values (fractions.Fraction)."""
    from fractions import Fraction
    g = np.random.default_rng(11)
    hs = np.concatenate([g.uniform(0, 20, 500), [0.0, 2.0 ** -33, 3 * 2.0 ** -33, 12.5,
                                                 np.float32(0.1), np.float32(math.log(262144))]])
    for h in hs.astype(np.float32):
        exact = Fraction(float(h)) * 2 ** 32
        fl = exact.numerator // exact.denominator
        rem = exact - fl
        want = fl + (1 if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1) else 0)
        assert O.eb_quantize(float(h)) == want
    # ties: 2^-33 is exactly half a unit (rounds to even 0), 3 * 2^-33 is 1.5 units (rounds to 2)
    assert O.eb_quantize(2.0 ** -33) == 0 and O.eb_quantize(3 * 2.0 ** -33) == 2
    for gm in list(g.uniform(0, 50, 200)) + [0.0, 1.0, 0.1, 1e-12]:
        exact = Fraction(float(gm)) * 2 ** 32
        assert O.eb_quantize_bound(gm) == exact.numerator // exact.denominator
    assert O.eb_quantize_bound(math.inf) == np.iinfo(np.int64).max


def test_router_margin_brute_force():
    g = np.random.default_rng(12)
    z = g.standard_normal((40, 9))
    for k in (1, 3, 8):
        m = O.router_margin(z, k)
        for t in range(z.shape[0]):
            srt = sorted(z[t], reverse=True)
            assert m[t] == srt[k - 1] - srt[k]
    assert np.isinf(O.router_margin(z, 9)).all()

@pytest.mark.parametrize("case", _golden_eb())
def test_eb_hand_worked(case):
    gamma, H, masked, want = case
    sel = O.eb_select(H, masked, gamma, False)
    assert sorted(np.nonzero(sel)[0].tolist()) == want


def test_eb_bound_zero_commits_lowest_single():
    for _ in range(50):
        n = 32
        H = rng.uniform(0.01, 12.0, n).astype(np.float32)
        masked = (rng.uniform(size=n) < 0.7).astype(np.uint8)
        if masked.sum() == 0:
            continue
        sel = O.eb_select(H, masked, 0.0, False)
        cand = np.nonzero(masked)[0]
        best = cand[np.lexsort((cand, H[cand]))[0]]
        assert sel.sum() == 1 and sel[best]


def test_eb_infinite_bound_and_force_commit_all():
    H = rng.uniform(0, 12, 40).astype(np.float32)
    masked = (rng.uniform(size=40) < 0.5).astype(np.uint8)
    assert (O.eb_select(H, masked, math.inf, False) == (masked != 0)).all()
    assert (O.eb_select(H, masked, 0.0, True) == (masked != 0)).all()


def test_eb_brute_force_prefix_enumeration():
    for _ in range(200):
        n = int(rng.integers(1, 7))
        H = rng.choice(np.array([0.0, 0.25, 0.5, 0.75, 1.0, 1.5], np.float32), n)
        masked = (rng.uniform(size=n) < 0.8).astype(np.uint8)
        gamma = float(rng.choice([0.0, 0.3, 0.5, 1.0, 2.0]))
        cand = [i for i in range(n) if masked[i]]
        if not cand:
            continue
        order = sorted(cand, key=lambda i: (float(H[i]), i))
        best = 1
        for k in range(1, len(order) + 1):          # every prefix of the sorted candidates
            chosen = [float(H[i]) for i in order[:k]]
            if sum(chosen) - max(chosen) <= gamma:
                best = max(best, k)
        sel = O.eb_select(H, masked, gamma, False)
        assert sorted(np.nonzero(sel)[0].tolist()) == sorted(order[:best])


def test_eb_permutation_invariance():
    n = 64
    H = rng.choice(np.array([0.1, 0.2, 0.3, 5.0], np.float32), n)   # many ties
    masked = np.ones(n, np.uint8)
    sel = O.eb_select(H, masked, 0.65, False)
    p = rng.permutation(n)
    sel_p = O.eb_select(H[p], masked[p], 0.65, False)
    # the committed multiset of entropies is the same; only tie-broken identities may move
    assert sorted(H[sel].tolist()) == sorted(H[p][sel_p].tolist())


def test_eb_rejects_non_finite():
    with pytest.raises(FloatingPointError):
        O.eb_select(np.array([0.1, np.nan], np.float32), np.array([1, 1], np.uint8), 1.0, False)


# ----------------------------------------------------------------- whole-step invariants (tiny workload)

@pytest.fixture(scope="module")
def tiny():
    cfg = synth.get_config("tiny")
    m = synth.make_model(cfg, "cpu")
    arr = {"emb": synth.to_numpy(m["emb"]),
           "layers": [{k: synth.to_numpy(v) for k, v in lay.items()} for lay in m["layers"]]}
    kv = synth.make_prompt_kv(cfg, "cpu")
    return cfg, O.OracleModel(cfg, arr), kv


def _state(cfg):
    st = synth.make_canvas_state(cfg, "all_mask")
    return {k: synth.to_numpy(v) for k, v in st.items()}


def test_tiny_generate_one_commit_per_step(tiny):
    cfg, model, kv = tiny
    kc = synth.to_numpy(kv["k"]).astype(np.float64)
    vc = synth.to_numpy(kv["v"]).astype(np.float64)
    cl = synth.to_numpy(kv["cache_len"])
    st = _state(cfg)
    seen = 0
    for s in range(cfg.canvas):
        st2, info = O.canvas_step(cfg, model, st, kc, vc, cl, cfg.gamma, cfg.max_steps)
        H = info[0]["H"]
        # random-init logits are nearly uniform: entropy ~ ln V >> gamma -> exactly one commit
        assert np.all(H > 0.9 * math.log(cfg.vocab))
        assert st["n_masked"][0] - st2["n_masked"][0] == 1
        lowest = info[0]["rows"][np.lexsort((info[0]["rows"], H))[0]]
        assert st2["masked"][0, lowest] == 0 and st2["tokens"][0, lowest] != cfg.mask_id
        st = st2
        seen += 1
        if st["done"][0]:
            break
    assert seen == cfg.canvas and st["done"][0] == 1 and st["step"][0] == cfg.canvas
    assert (st["tokens"][0] < cfg.vocab).all()


def test_tiny_zero_lm_head_gives_ln_v_and_index_order(tiny):
    cfg, model, kv = tiny
    arr = dict(model.a)
    emb = arr["emb"].copy()
    emb[:cfg.vocab] = 0.0                                  # every logit 0: uniform softmax
    m0 = O.OracleModel(cfg, dict(arr, emb=emb))
    kc = synth.to_numpy(kv["k"]).astype(np.float64)
    vc = synth.to_numpy(kv["v"]).astype(np.float64)
    st = _state(cfg)
    st2, info = O.canvas_step(cfg, m0, st, kc, vc, synth.to_numpy(kv["cache_len"]), 0.0, 16)
    np.testing.assert_allclose(info[0]["H"], math.log(cfg.vocab), rtol=1e-6)
    assert (info[0]["argmax"] == 0).all()
    assert st2["masked"][0, 0] == 0 and st2["masked"][0, 1:].all() and st2["tokens"][0, 0] == 0


def test_tiny_infinite_bound_and_step_cap(tiny):
    cfg, model, kv = tiny
    kc = synth.to_numpy(kv["k"]).astype(np.float64)
    vc = synth.to_numpy(kv["v"]).astype(np.float64)
    cl = synth.to_numpy(kv["cache_len"])
    st2, _ = O.canvas_step(cfg, model, _state(cfg), kc, vc, cl, math.inf, 16)
    assert st2["done"][0] == 1 and st2["n_masked"][0] == 0
    st = _state(cfg)
    st["step"][:] = 15
    st2, _ = O.canvas_step(cfg, model, st, kc, vc, cl, 0.0, 16)   # last allowed step
    assert st2["done"][0] == 1


def test_tiny_kv_append_single_layer_is_direct_projection(tiny):
    cfg, model, kv = tiny
    kc = synth.to_numpy(kv["k"]).astype(np.float64)
    vc = synth.to_numpy(kv["v"]).astype(np.float64)
    cl = synth.to_numpy(kv["cache_len"])
    toks = rng.integers(0, cfg.vocab, (1, cfg.canvas)).astype(np.int32)
    new_len = O.kv_append(cfg, model, toks, kc, vc, cl)
    assert new_len[0] == cl[0] + cfg.canvas
    # one layer: the appended K/V are the projections of the normed embeddings, rotated
    x = model.emb_rows(toks[0])
    a = O.rmsnorm(x, cfg.rms_eps)
    w = model.w(0, "w_qkv")
    Hq, Hkv, hd = cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim
    kraw = (a @ w[Hq * hd:(Hq + Hkv) * hd].T).reshape(cfg.canvas, Hkv, hd)
    vraw = (a @ w[(Hq + Hkv) * hd:].T).reshape(cfg.canvas, Hkv, hd)
    pos = cl[0] + np.arange(cfg.canvas)
    np.testing.assert_allclose(kc[0, 0, :, cl[0]:new_len[0]],
                               O.rope(kraw, pos, cfg.rope_theta).transpose(1, 0, 2), atol=1e-12)
    np.testing.assert_allclose(vc[0, 0, :, cl[0]:new_len[0]], vraw.transpose(1, 0, 2), atol=1e-12)
    # rows outside the appended range are untouched
    assert (kc[0, 0, :, new_len[0]:] == 0).all()


def test_tiny_full_generate_two_canvases(tiny):
    cfg, model, kv = tiny
    kc = synth.to_numpy(kv["k"]).astype(np.float64)
    vc = synth.to_numpy(kv["v"]).astype(np.float64)
    cl = synth.to_numpy(kv["cache_len"])
    toks, steps, new_len = O.generate(cfg, model, kc, vc, cl, cfg.n_canvases, cfg.gamma, cfg.max_steps)
    assert (steps == cfg.canvas).all()            # one commit per step at gamma 0.1
    assert new_len[0] == cfg.prompt_len + cfg.n_canvases * cfg.canvas
    assert (toks < cfg.vocab).all()


def test_tiny_layer_residual_wiring(tiny):
    """Zero output projection and zero expert down-projections: the layer is the
    identity on its residual stream; zero output projection alone: the layer no
    longer depends on the prompt cache."""
    cfg, model, kv = tiny
    lay = dict(model.a["layers"][0])
    lay_zero = dict(lay, w_o=np.zeros_like(lay["w_o"]), w_down=np.zeros_like(lay["w_down"]))
    m0 = O.OracleModel(cfg, dict(model.a, layers=[lay_zero]))
    kc = synth.to_numpy(kv["k"]).astype(np.float64)[:, 0]
    vc = synth.to_numpy(kv["v"]).astype(np.float64)[:, 0]
    toks = rng.integers(0, cfg.vocab, cfg.canvas).astype(np.int32)
    masked = np.zeros(cfg.canvas, np.uint8)
    x = O.canvas_forward(cfg, m0, toks, masked, kc, vc, cfg.prompt_len)
    np.testing.assert_array_equal(x, model.emb_rows(toks))
    m1 = O.OracleModel(cfg, dict(model.a, layers=[dict(lay, w_o=np.zeros_like(lay["w_o"]))]))
    xa = O.canvas_forward(cfg, m1, toks, masked, kc, vc, cfg.prompt_len)
    xb = O.canvas_forward(cfg, m1, toks, masked, kc * 3.0 + 1.0, vc * -2.0, cfg.prompt_len)
    np.testing.assert_array_equal(xa, xb)
    assert not np.array_equal(xa, model.emb_rows(toks))
    xc = O.canvas_forward(cfg, model, toks, masked, kc * 3.0 + 1.0, vc * -2.0, cfg.prompt_len)
    assert np.abs(xc - O.canvas_forward(cfg, model, toks, masked, kc, vc, cfg.prompt_len)).max() > 1e-6


def test_moe_negative_expert_slot_contributes_nothing():
    T, d, F, E = 6, 8, 5, 4
    y = rng.standard_normal((T, d))
    res = rng.standard_normal((T, d))
    ws = _experts(E, F, d)
    idx, g, _ = O.router_topk(y, rng.standard_normal((E, d)), 2)
    full = O.moe_ffn(y, idx, g, lambda e: ws[e], res, "f32")
    idx1 = idx.copy(); idx1[:, 1] = -1
    part = O.moe_ffn(y, idx1, g, lambda e: ws[e], res, "f32")
    only0 = O.moe_ffn(y, idx[:, :1], g[:, :1], lambda e: ws[e], res, "f32")
    np.testing.assert_allclose(part, only0, atol=1e-13)
    assert not np.allclose(part, full)


def test_append_is_a_causal_encoder_two_layers():
    """The append is a causal encoder ("DiffusionGemma Technical Report", Figure 4, stage 3):
    appending the first n tokens of a sequence writes exactly the K/V rows that appending the
    whole sequence writes for them, in every layer, because no row sees a later token; and a row
    of the second layer does depend on the earlier tokens."""
    cfg = synth.get_config("tiny", n_layers=2)
    m = synth.make_model(cfg, "cpu")
    om = O.OracleModel(cfg, {"emb": synth.to_numpy(m["emb"]),
                             "layers": [{k: synth.to_numpy(v) for k, v in lay.items()}
                                        for lay in m["layers"]]})
    kv = synth.make_prompt_kv(cfg, "cpu")
    kc0 = synth.to_numpy(kv["k"]).astype(np.float64)
    vc0 = synth.to_numpy(kv["v"]).astype(np.float64)
    cl = synth.to_numpy(kv["cache_len"])
    toks = rng.integers(0, cfg.vocab, (1, 12)).astype(np.int32)
    ka, va = kc0.copy(), vc0.copy()
    O.kv_append(cfg, om, toks, ka, va, cl)
    kb, vb = kc0.copy(), vc0.copy()
    O.kv_append(cfg, om, toks[:, :5], kb, vb, cl)
    r0, r1 = int(cl[0]), int(cl[0]) + 5
    np.testing.assert_allclose(kb[..., r0:r1, :], ka[..., r0:r1, :], rtol=0, atol=1e-12)
    np.testing.assert_allclose(vb[..., r0:r1, :], va[..., r0:r1, :], rtol=0, atol=1e-12)
    t2 = toks.copy()
    t2[0, 0] = (t2[0, 0] + 1) % cfg.vocab
    kc2, vc2 = kc0.copy(), vc0.copy()
    O.kv_append(cfg, om, t2, kc2, vc2, cl)
    assert np.abs(kc2[1, ..., r0 + 7, :] - ka[1, ..., r0 + 7, :]).max() > 1e-6


def test_tiny_commit_writes_each_rows_own_argmax(tiny):
    """On a canvas whose open rows are not its first positions, every position the step commits
    receives the argmax of its own row's logits (computed here from the returned logits), and the
    final positions keep their tokens.  The open positions carry distinct draft tokens (the
    revisable-draft canvas, greedy), so their rows, and their argmaxes, differ."""
    cfg, model, kv = tiny
    kc = synth.to_numpy(kv["k"]).astype(np.float64)
    vc = synth.to_numpy(kv["v"]).astype(np.float64)
    cl = synth.to_numpy(kv["cache_len"])
    st = _state(cfg)
    g = np.random.default_rng(5)
    st["tokens"][0] = g.integers(0, cfg.vocab, cfg.canvas)
    done_pos = g.permutation(cfg.canvas)[: cfg.canvas // 2]
    st["masked"][0, done_pos] = 0
    st["n_masked"][0] = int(st["masked"][0].sum())
    greedy_drafts = {"tau_start": 0.0, "tau_end": 0.0, "seed": 0, "revise": True}
    st2, info = O.canvas_step(cfg, model, st, kc, vc, cl, 1e9, cfg.max_steps, keep_logits=True,
                              sampler=greedy_drafts)
    rows = info[0]["rows"]
    assert (rows == np.nonzero(st["masked"][0])[0]).all()
    own = np.argmax(info[0]["logits"], axis=1)
    assert len(set(own.tolist())) > 1                       # the check below can tell rows apart
    assert st2["masked"][0].sum() == 0                       # an unbounded gamma commits them all
    np.testing.assert_array_equal(st2["tokens"][0, rows], own)
    np.testing.assert_array_equal(st2["tokens"][0, done_pos], st["tokens"][0, done_pos])
