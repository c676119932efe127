"""Plain, slow, fp64 CPU oracle for one denoising step of block-wise discrete diffusion.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference arm of ``bench.py`` may import or run this module.
It shares no code with the CUDA library and imports nothing from it; the only
thing both sides take from a common place is the seeded synthetic inputs
(``synth``), which carry none of the method's arithmetic.

What it computes (the method as the pages describe it):

* "DiffusionGemma Technical Report" (metalmedia.ai), Figure 4: a prompt is
  encoded causally into a KV cache; a canvas is refined by a decoder with
  bidirectional attention across the canvas and cross-attention to the cache;
  the finished canvas goes back through the causal encoder and is appended.
* Same page, explanatory visual, "Inference: block-wise diffusion decoding",
  and "What they did": an entropy-bounded sampler with adaptive stopping
  finishes a 256-token block in a number of steps.
* Model card "diffusiongemma" (axforge.ai), "Mixture-of-Experts (MoE)
  Efficiency": 8 active experts of 128; Table 1 of the report: vocabulary 262k.
* The entropy-bounded (EB) rule itself is not printed on the pages; the oracle
  follows the published EB sampler (Ben-Hamu et al., 2025, "Accelerated
  Sampling from Masked Diffusion Models via Entropy Bounded Unmasking"):
  commit masked positions in ascending entropy while the sum of the chosen
  entropies minus their maximum stays within the bound gamma.

Precision: every product and sum runs in fp64.  The pages fix no storage
precision for intermediates; the reading taken is that the tensors that feed a
bf16 matrix product or the attention are stored in the workload's activation type
(the normalised rows a, y and f, the attention inputs and output q, k, v, o, and
the expert activation a), while the residual stream (embedding, h, layer
outputs) and the expert outputs Y are kept in fp32.  Where the activation type
is bf16 the oracle rounds the fp64 value to the nearest bf16 at exactly those
tensors and leaves the others unrounded, so the oracle/GPU gap is
accumulation-order error, not storage error.  fp32 workloads are not rounded.

Weights are decoded exactly from their storage: bf16, FP8 E4M3 times a per-channel scale, or
(for the tied embedding / LM head of the NVFP4 workload) NVFP4, FP4 E2M1 codes times an E4M3
scale per 16 elements times one tensor scale; the model card names an NVFP4 build of the
checkpoint but the pages do not define the format, so the oracle follows NVIDIA's published
definition of it (see nvfp4_rows).
"""
from __future__ import annotations

import contextlib
import math
from typing import Dict, List, Optional

import numpy as np

INT64_MAX = np.iinfo(np.int64).max
EB_FRAC_BITS = 32  # fixed-point fraction bits of the EB entropy sums

# Arithmetic type of every product, sum, norm and softmax below: fp64.  The tests derive their
# floating-point tolerances from a second run of this same code with fp32 arithmetic (the
# `accumulation` context), i.e. from the spread between two valid evaluations of the method that
# differ only in accumulation precision and order; nothing else ever changes it.
_ACC = [np.float64]


def acc_dtype():
    return _ACC[0]


@contextlib.contextmanager
def accumulation(dtype):
    """Run the oracle with `dtype` (np.float64 or np.float32) as its arithmetic type.  Storage
    rounding (bf16 / fp16 at the tensors the reading names) is unchanged."""
    prev = _ACC[0]
    _ACC[0] = np.dtype(dtype).type
    try:
        yield
    finally:
        _ACC[0] = prev


def _a(x) -> np.ndarray:
    """x in the arithmetic type."""
    return np.asarray(x, dtype=_ACC[0])


# --------------------------------------------------------------------------- number formats

def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> value: the top half of an IEEE binary32."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round fp64 values to the nearest bf16 value (ties to even), returned as fp64.

    bf16 keeps 8 significant bits and binary32's exponent range: a normal value
    m * 2**e with m in [0.5, 1) becomes rint(m * 2**8) * 2**(e - 8); values
    below the smallest normal share the subnormal quantum 2**-133; values that
    round past the largest finite bf16 become +-inf.
    """
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)
    e = np.maximum(e, -125)                     # subnormal range: fixed quantum 2**-133
    q = np.ldexp(1.0, (e - 8))
    r = np.rint(x / q) * q
    bf16_max = (2.0 - 2.0 ** -7) * 2.0 ** 127
    r = np.where(np.abs(r) > bf16_max, np.copysign(np.inf, x), r)
    return np.where(np.isfinite(x), r, x)


def round_f16(x: np.ndarray) -> np.ndarray:
    """Round fp64 values to the nearest IEEE binary16 value (ties to even), returned as fp64.

    Values that round past the largest finite binary16 (65504) become +-inf."""
    with np.errstate(over="ignore"):
        return np.asarray(x, dtype=np.float64).astype(np.float16).astype(np.float64)


def e4m3_to_f64(codes: np.ndarray) -> np.ndarray:
    """Decode OCP FP8 E4M3 codes: 1 sign, 4 exponent (bias 7), 3 mantissa bits.

    Exponent field 0 is subnormal (m/8 * 2**-6); S.1111.111 is NaN; there is no
    infinity, so the largest finite magnitude is 1.75 * 2**8 = 448.
    """
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    ex = (c >> 3) & 0xF
    man = c & 0x7
    val = np.where(ex == 0, man / 8.0 * 2.0 ** -6, (1.0 + man / 8.0) * np.exp2(ex - 7.0))
    val = np.where((ex == 0xF) & (man == 0x7), np.nan, val)
    return sign * val


def e2m1_to_f64(codes: np.ndarray) -> np.ndarray:
    """Decode FP4 E2M1 codes (the low 4 bits): 1 sign, 2 exponent (bias 1), 1 mantissa bit.

    Exponent field 0 is subnormal (m/2); otherwise (1 + m/2) * 2**(e - 1).  No infinities or
    NaNs, so the magnitudes are 0, 0.5, 1, 1.5, 2, 3, 4 and 6.
    """
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64) & 0xF
    sign = np.where(c & 0x8, -1.0, 1.0)
    ex = (c >> 1) & 0x3
    man = c & 0x1
    val = np.where(ex == 0, man / 2.0, (1.0 + man / 2.0) * np.exp2(ex - 1.0))
    return sign * val


def nvfp4_rows(codes: np.ndarray, scales: np.ndarray, tensor_scale: float,
               rows: np.ndarray) -> np.ndarray:
    """Decode rows of an NVFP4 matrix stored in k-blocks of 64 elements.

    NVFP4 (NVIDIA's 4-bit floating-point format; the model card names an NVFP4 build of the
    checkpoint): element = e2m1(code) * e4m3(block scale) * tensor_scale, one E4M3 scale per 16
    consecutive elements of a row.  Storage: codes [K/64][R][32] bytes, element kb*64 + 2i of
    row r in the low nibble of codes[kb, r, i] and element kb*64 + 2i + 1 in its high nibble;
    scales [K/64][R][4], scales[kb, r, j] for elements kb*64 + 16j .. kb*64 + 16j + 15.
    Returns fp64 [len(rows)][K].
    """
    rows = np.asarray(rows)
    nk = codes.shape[0]
    c = codes[:, rows, :]                                   # [nk][n][32]
    lo = e2m1_to_f64(c & 0xF)
    hi = e2m1_to_f64(c >> 4)
    vals = np.empty(c.shape[:2] + (64,))
    vals[..., 0::2] = lo
    vals[..., 1::2] = hi
    sc = e4m3_to_f64(scales[:, rows, :])                    # [nk][n][4]
    vals = vals * np.repeat(sc, 16, axis=-1) * float(tensor_scale)
    return vals.transpose(1, 0, 2).reshape(len(rows), nk * 64)


def decode_weight(arr: np.ndarray, kind: str, scale: Optional[np.ndarray] = None) -> np.ndarray:
    """Stored weight -> fp64 value.  e4m3 rows are multiplied by their channel scale."""
    if kind == "f32":
        return np.asarray(arr, dtype=np.float64)
    if kind == "bf16":
        return bf16_bits_to_f64(arr)
    if kind == "e4m3":
        return e4m3_to_f64(arr) * np.asarray(scale, dtype=np.float64)[..., None]
    raise ValueError(kind)


def decode_act(arr: np.ndarray, kind: str) -> np.ndarray:
    return bf16_bits_to_f64(arr) if kind == "bf16" else np.asarray(arr, dtype=np.float64)


def storage_round(x: np.ndarray, act: str) -> np.ndarray:
    return round_bf16(x) if act == "bf16" else np.asarray(x, dtype=np.float64)


# --------------------------------------------------------------------------- layer pieces

def rmsnorm(x: np.ndarray, eps: float) -> np.ndarray:
    """x / sqrt(mean(x^2) + eps) over the last axis, unit gain."""
    x = _a(x)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + _ACC[0](eps))


def gelu_tanh(x: np.ndarray) -> np.ndarray:
    """0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3)))."""
    return 0.5 * x * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (x + 0.044715 * x ** 3)))


def rope(x: np.ndarray, pos: np.ndarray, theta: float) -> np.ndarray:
    """Rotate-half rotary embedding on the last axis.

    Pairs (i, i + hd/2) rotate by angle pos * theta**(-2i/hd).  ``x`` is
    [T, ..., hd] and ``pos`` is [T] (absolute positions).
    """
    hd = x.shape[-1]
    half = hd // 2
    inv = theta ** (-2.0 * np.arange(half, dtype=np.float64) / hd)
    ang = np.asarray(pos, dtype=np.float64)[:, None] * inv[None, :]
    shape = (x.shape[0],) + (1,) * (x.ndim - 2) + (half,)
    c = _a(np.cos(ang).reshape(shape))
    s = _a(np.sin(ang).reshape(shape))
    x = _a(x)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def attention(q: np.ndarray, k_cache: np.ndarray, v_cache: np.ndarray,
              k_new: np.ndarray, v_new: np.ndarray, causal: bool) -> np.ndarray:
    """softmax(q K^T / sqrt(hd)) V for one canvas, GQA.

    q [T, Hq, hd]; k_cache, v_cache [Hkv, P, hd] (the prompt/context rows);
    k_new, v_new [T, Hkv, hd] (the canvas's own keys).  Query head h uses kv
    head h // (Hq / Hkv).  Keys are the cache rows followed by the canvas rows.
    ``causal`` False: every query sees every key (the decoder's bidirectional
    canvas attention).  True: query i sees the whole cache and canvas keys
    j <= i (the causal encoder used for the append).
    Returns o [T, Hq, hd].
    """
    T, Hq, hd = q.shape
    Hkv, P = k_cache.shape[0], k_cache.shape[1]
    rep = Hq // Hkv
    q, k_cache, v_cache, k_new, v_new = (_a(t) for t in (q, k_cache, v_cache, k_new, v_new))
    out = np.empty((T, Hq, hd))
    mask = None
    if causal:
        mask = np.zeros((T, P + T), dtype=bool)
        mask[:, P:] = np.triu(np.ones((T, T), dtype=bool), k=1)
    for h in range(Hq):
        g = h // rep
        K = np.concatenate([k_cache[g], k_new[:, g]], axis=0)
        V = np.concatenate([v_cache[g], v_new[:, g]], axis=0)
        s = q[:, h] @ K.T / _ACC[0](math.sqrt(hd))
        if mask is not None:
            s = np.where(mask, -np.inf, s)
        s = s - s.max(axis=1, keepdims=True)
        p = np.exp(s)
        p /= p.sum(axis=1, keepdims=True)
        out[:, h] = p @ V
    return out


def router_topk(y: np.ndarray, w_r: np.ndarray, top_k: int, forced: Optional[np.ndarray] = None):
    """Router: logits z = y W_r^T, p = softmax(z) over all experts, the top_k
    largest p (lower expert index first among equals), renormalised to sum 1.

    ``forced`` (int [T, k], optional) replaces the top-k choice by the given experts, whose gates
    are still this router's p renormalised over them: it lets one evaluation reproduce another's
    expert choices, which bf16 rounding can legitimately flip at near ties.
    Returns (idx [T, k] int32, gates [T, k], z [T, E]).
    """
    z = _a(y) @ _a(w_r).T
    p = np.exp(z - z.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    idx = np.argsort(-p, axis=1, kind="stable")[:, :top_k] if forced is None \
        else np.asarray(forced, dtype=np.int64)
    gp = np.take_along_axis(p, idx, axis=1)
    return idx.astype(np.int32), gp / gp.sum(axis=1, keepdims=True), z


def with_shared_experts(idx: np.ndarray, gates: np.ndarray, n_experts: int, n_shared: int):
    """Append the always-on shared experts to every token's routed slots.

    The model card lists the MoE as 8 active experts of 128 "+1 shared": a shared expert takes
    every token regardless of the router.  Reading taken: shared expert s is stored as expert
    n_experts + s, enters with gate 1 (it is not router-weighted), and its slot follows the
    routed ones (slot order k, k + 1, ...).
    """
    if n_shared <= 0:
        return idx, gates
    T = idx.shape[0]
    ids = np.broadcast_to(np.arange(n_experts, n_experts + n_shared, dtype=np.int32), (T, n_shared))
    return (np.concatenate([idx, ids], axis=1),
            np.concatenate([gates, np.ones((T, n_shared))], axis=1))


def router_margin(z: np.ndarray, top_k: int) -> np.ndarray:
    """Per token: gap between the k-th and (k+1)-th largest router logit (inf if k = E)."""
    E = z.shape[1]
    if top_k >= E:
        return np.full(z.shape[0], np.inf)
    s = -np.sort(-z, axis=1)
    return s[:, top_k - 1] - s[:, top_k]


def moe_ffn(y: np.ndarray, idx: np.ndarray, gates: np.ndarray, expert_w, residual: np.ndarray,
            act: str) -> np.ndarray:
    """Sparse expert FFN plus residual.

    For token t and slot j with expert e = idx[t, j]:
      [g; u] = y_t W_gu,e^T  (the first d_ff outputs are the gate, the next d_ff the up)
      a      = gelu_tanh(g) * u                 (stored in the activation type: rounded)
      Y      = a W_d,e^T                        (fp32 on the device: unrounded)
    out_t = residual_t + sum_j gates[t, j] Y_{t,j}          (residual stream: unrounded)
    ``expert_w(e)`` returns (W_gu,e [2F, d], W_d,e [d, F]) as fp64.  A slot whose expert id is
    negative has no expert and contributes nothing.
    """
    T, k = idx.shape
    acc = np.array(residual, dtype=_ACC[0], copy=True)
    y = _a(y)
    for e in np.unique(idx):
        if e < 0:
            continue
        rows, slots = np.nonzero(idx == e)
        w_gu, w_d = (_a(w) for w in expert_w(int(e)))
        F = w_d.shape[1]
        u = y[rows] @ w_gu.T
        a = _a(storage_round(gelu_tanh(u[:, :F]) * u[:, F:], act))
        Y = a @ w_d.T
        acc[rows] += gates[rows, slots][:, None] * Y
    return acc


def entropy_argmax(z: np.ndarray):
    """Per row of logits z [R, V]: softmax entropy (natural log), greedy argmax
    (lowest index among equal maxima) and the top-1 minus top-2 margin."""
    z = _a(z)
    m = z.max(axis=1, keepdims=True)
    e = np.exp(z - m)
    p = e / e.sum(axis=1, keepdims=True)
    with np.errstate(divide="ignore", invalid="ignore"):
        plogp = np.where(p > 0, p * np.log(p), 0.0)
    H = -plogp.sum(axis=1)
    am = np.argmax(z, axis=1).astype(np.int32)
    if z.shape[1] > 1:
        part = -np.partition(-z, 1, axis=1)
        margin = part[:, 0] - part[:, 1]
    else:
        margin = np.full(z.shape[0], np.inf)
    return H, am, margin


# --------------------------------------------------------------------------- EB sampler

def eb_quantize(h: float) -> int:
    """Fixed-point entropy: nearest integer to h * 2**32 (ties to even).

    The argument is an fp32 value; its product with 2**32 is exact in fp64.
    """
    return int(np.rint(np.float64(h) * 2.0 ** EB_FRAC_BITS))


def eb_quantize_bound(gamma: float) -> int:
    """Fixed-point bound: floor(gamma * 2**32); +inf maps to the largest int64."""
    if math.isinf(gamma):
        return int(INT64_MAX)
    v = math.floor(gamma * 2.0 ** EB_FRAC_BITS)
    return int(min(v, INT64_MAX))


def eb_select(H: np.ndarray, masked: np.ndarray, gamma: float, force_all: bool) -> np.ndarray:
    """Positions of one canvas that the EB sampler commits this step.

    Candidates are the masked positions.  They are ordered by entropy, ascending,
    lower position first among equal entropies (negative rounding residue and
    -0 count as 0).  With sorted entropies H_(1) <= H_(2) <= ..., the sampler
    commits the first k, for the largest k >= 1 such that
        sum_{i<=k} H_(i) - max_{i<=k} H_(i) = sum_{i<k} H_(i) <= gamma,
    the sums taken in 32-fraction-bit fixed point.  ``force_all`` (the last
    allowed step) commits every masked position.  Returns a bool array.
    """
    H = np.asarray(H, dtype=np.float32)
    cand = np.nonzero(np.asarray(masked) != 0)[0]
    sel = np.zeros(len(masked), dtype=bool)
    if len(cand) == 0:
        return sel
    if not np.all(np.isfinite(H[cand])):
        raise FloatingPointError("non-finite entropy at a masked position")
    if not (gamma >= 0.0):
        raise ValueError("the entropy bound must be >= 0")
    hv = np.maximum(H[cand].astype(np.float64), 0.0)
    order = sorted(range(len(cand)), key=lambda i: (hv[i], int(cand[i])))
    if force_all:
        sel[cand] = True
        return sel
    qg = eb_quantize_bound(gamma)
    k = 1
    prefix = 0
    for j in range(1, len(order)):
        prefix += eb_quantize(np.float32(hv[order[j - 1]]))
        if prefix <= qg:
            k = j + 1
        else:
            break
    sel[cand[[order[i] for i in range(k)]]] = True
    return sel


# --------------------------------------------------------------------------- sampler variants
#
# The pages describe a canvas that starts from random noise and is refined over the steps
# ("DiffusionGemma Technical Report": explanatory visual "Inference: block-wise diffusion decoding",
# "What they did", Figure 3 with uniform noise at t = 1.0), a model that corrects its own mistakes
# while denoising, before the output is final (ainewsonline.de article), a sampler whose
# temperature is annealed over the step budget N (report, Figure 9: a larger N anneals more
# mildly; Figure 10: tau_t = 1 when annealing is off), and weights that still run in standard
# autoregressive mode, leaving room for hybrid diffusion-AR decoding (report, "What they did"
# and "Limits and open work").  None of them is given as a formula; the readings taken are:
#
# * temperature: linear in the step index, tau_s = tau_start + (tau_end - tau_start) s / (N - 1)
#   (fp64), N = max_steps.  tau > 0: the token is drawn from softmax(z / tau) and the entropy the
#   EB rule ranks is that distribution's.  tau <= 0: greedy argmax with the entropy at tau = 1
#   (the method without sampling).
# * drawing from softmax(z / tau): the Gumbel-max rule, argmax_v (z_v / tau + G_v) with G_v
#   standard Gumbel, G = -ln(-ln U).  The fp32 value 1 / tau multiplies the logits.
# * randomness: one counter-based generator, Philox4x32-10 (Salmon, Moraes, Dror and Shaw,
#   "Parallel random numbers: as easy as 1, 2, 3", SC 2011), keyed by the 64-bit seed (low word
#   first).  The counter names the draw: (v >> 2, a1, a2, (tag << 24) | b) for vocabulary entry v
#   (word v & 3 of the output) of stream (tag, b, a1, a2).  U = ((w >> 9) + 1/2) 2^-23, exact in
#   fp32 and strictly inside (0, 1).
# * uniform-noise canvas: position i of canvas b holds (w0 * V) >> 32 for the first output word
#   w0 of counter (i, 0, 0, (TAG_NOISE << 24) | b); every position starts not final.
# * revisable drafts (noise canvas): a position that is not final is embedded by its current
#   draft token (not MASK); each step the EB rule makes the lowest-entropy prefix final as
#   before, and every other non-final position takes the step's prediction as its new draft.
#   Final positions never change.
# * autoregressive mode: the same weights as the causal encoder; the new tokens of a sequence
#   are appended to its cache as by the append, the LAST layer runs in full as well, and the
#   final RMSNorm + LM head of the last new row predict the next token (the standard next-token
#   reading of a causal decoder).  Hybrid decoding is a sequence that alternates canvases and
#   autoregressive tokens on one cache.

PHILOX_M0, PHILOX_M1 = 0xD2511F53, 0xCD9E8D57   # round multipliers
PHILOX_W0, PHILOX_W1 = 0x9E3779B9, 0xBB67AE85   # key increments (Weyl sequence)
_M32 = 0xFFFFFFFF
TAG_DENOISE, TAG_NOISE, TAG_AR = 1, 2, 3          # counter word 3 = (tag << 24) | canvas


def philox4x32_10(c0, c1, c2, c3, k0: int, k1: int):
    """Philox4x32 with 10 rounds on 32-bit counter words (numpy arrays or ints, broadcast) and
    the 2-word key.  A round maps (c0, c1, c2, c3) with key (k0, k1) to
        (hi(M1 c2) ^ c1 ^ k0, lo(M1 c2), hi(M0 c0) ^ c3 ^ k1, lo(M0 c0)),
    hi / lo the upper / lower 32 bits of the 64-bit product; the key grows by (W0, W1) before
    every round after the first.  Returns the four output words as uint64 arrays (< 2^32)."""
    c = [np.asarray(x, dtype=np.uint64) & np.uint64(_M32) for x in (c0, c1, c2, c3)]
    c = np.broadcast_arrays(*c)
    c = [np.array(x, dtype=np.uint64) for x in c]
    ka, kb = int(k0) & _M32, int(k1) & _M32
    m0, m1, m32 = np.uint64(PHILOX_M0), np.uint64(PHILOX_M1), np.uint64(_M32)
    for r in range(10):
        if r:
            ka, kb = (ka + PHILOX_W0) & _M32, (kb + PHILOX_W1) & _M32
        p0 = c[0] * m0            # < 2^64: exact in uint64
        p1 = c[2] * m1
        c = [(p1 >> np.uint64(32)) ^ c[1] ^ np.uint64(ka), p1 & m32,
             (p0 >> np.uint64(32)) ^ c[3] ^ np.uint64(kb), p0 & m32]
    return c


def seed_key(seed: int):
    """The generator's key: the 64-bit seed as (low word, high word)."""
    seed = int(seed) & 0xFFFFFFFFFFFFFFFF
    return seed & _M32, seed >> 32


def stream_words(seed: int, tag: int, b: int, a1: int, a2: int, n: int) -> np.ndarray:
    """The 32-bit words w_0 .. w_{n-1} of stream (tag, b, a1, a2): w_v is word v & 3 of the
    generator at counter (v >> 2, a1, a2, (tag << 24) | b)."""
    v = np.arange(n, dtype=np.uint64)
    k0, k1 = seed_key(seed)
    words = philox4x32_10(v >> np.uint64(2), a1, a2, (int(tag) << 24) | int(b), k0, k1)
    return np.choose((v & np.uint64(3)).astype(np.int64), words)


def uniform_open(words: np.ndarray) -> np.ndarray:
    """U = ((w >> 9) + 1/2) 2^-23 in (0, 1), fp64 (exact)."""
    return ((np.asarray(words, dtype=np.uint64) >> np.uint64(9)).astype(np.float64) + 0.5) \
        * 2.0 ** -23


def gumbel(words: np.ndarray) -> np.ndarray:
    """Standard Gumbel draws G = -ln(-ln U) (fp64)."""
    return -np.log(-np.log(uniform_open(words)))


def temperature(step: int, max_steps: int, tau_start: float, tau_end: float) -> float:
    """tau_s, linear from tau_start at step 0 to tau_end at step max_steps - 1 (fp64)."""
    frac = min(int(step), max_steps - 1) / max(max_steps - 1, 1)
    return tau_start + (tau_end - tau_start) * frac


def inv_temperature(tau: float) -> np.float32:
    """The fp32 multiplier 1 / tau applied to the logits."""
    return np.float32(1.0 / tau)


def sample_row(z: np.ndarray, tau: float, g: Optional[np.ndarray]):
    """One row of logits z [V] at temperature tau with Gumbel draws g [V].
    Returns (entropy, token, key margin): tau <= 0 is greedy (entropy at tau = 1, margin the
    top-1 minus top-2 logit); otherwise the entropy of softmax(z / tau), the token
    argmax(z / tau + g) (first index among equal keys) and the margin between its two largest
    keys."""
    z = np.asarray(z, dtype=np.float64)[None, :]
    if not tau > 0.0:
        H, am, margin = entropy_argmax(z)
        return float(H[0]), int(am[0]), float(margin[0])
    zs = z * float(inv_temperature(tau))
    H, _, _ = entropy_argmax(zs)
    keys = zs[0] + g
    tok = int(np.argmax(keys))
    part = -np.partition(-keys, 1)
    return float(H[0]), tok, float(part[0] - part[1])


def noise_canvas(seed: int, batch: int, canvas: int, vocab: int) -> dict:
    """Uniform-noise canvases: tokens [B, C] with every position not final."""
    toks = np.zeros((batch, canvas), dtype=np.int32)
    k0, k1 = seed_key(seed)
    i = np.arange(canvas, dtype=np.uint64)
    for b in range(batch):
        w0 = philox4x32_10(i, 0, 0, (TAG_NOISE << 24) | b, k0, k1)[0]
        toks[b] = ((w0 * np.uint64(vocab)) >> np.uint64(32)).astype(np.int32)
    return {"tokens": toks, "masked": np.ones((batch, canvas), dtype=np.uint8),
            "n_masked": np.full(batch, canvas, dtype=np.int32),
            "done": np.zeros(batch, dtype=np.int32), "step": np.zeros(batch, dtype=np.int32)}


# --------------------------------------------------------------------------- the model

class OracleModel:
    """Decoded view of a synthetic model (the numpy arrays from ``synth.to_numpy``).

    Weights are decoded to fp64 on use so that large workloads fit in host RAM.
    """

    def __init__(self, cfg, arrays: dict):
        self.cfg = cfg
        self.a = arrays

    def _nvfp4(self) -> bool:
        return getattr(self.cfg, "emb", "") == "nvfp4"

    def emb_rows(self, ids: np.ndarray) -> np.ndarray:
        if self._nvfp4():
            return nvfp4_rows(self.a["emb"], self.a["emb_scale"], self.a["emb_scale_global"], ids)
        kind = "f32" if self.cfg.act == "f32" else "bf16"
        return decode_weight(self.a["emb"][ids], kind)

    def lm_head_chunks(self, chunk: int = 16384):
        kind = "f32" if self.cfg.act == "f32" else "bf16"
        V = self.cfg.vocab
        for v0 in range(0, V, chunk):
            v1 = min(V, v0 + chunk)
            if self._nvfp4():
                yield v0, nvfp4_rows(self.a["emb"], self.a["emb_scale"],
                                     self.a["emb_scale_global"], np.arange(v0, v1))
            else:
                yield v0, decode_weight(self.a["emb"][v0:v1], kind)

    def layer(self, l: int) -> dict:
        return self.a["layers"][l]

    def w(self, l: int, name: str) -> np.ndarray:
        lay = self.layer(l)
        sname = {"w_qkv": "s_qkv", "w_o": "s_o"}.get(name)
        kind = self.cfg.w
        if name == "w_router":
            kind = "f32" if self.cfg.w == "f32" else "bf16"
            return decode_weight(lay[name], kind)
        return decode_weight(lay[name], kind, None if sname is None else lay.get(sname))

    def expert(self, l: int, e: int):
        lay = self.layer(l)
        s_gu = None if lay.get("s_gate_up") is None else lay["s_gate_up"][e]
        s_d = None if lay.get("s_down") is None else lay["s_down"][e]
        return (decode_weight(lay["w_gate_up"][e], self.cfg.w, s_gu),
                decode_weight(lay["w_down"][e], self.cfg.w, s_d))


def layer_qkv(cfg, model: OracleModel, l: int, x: np.ndarray, pos: np.ndarray):
    """Pre-norm and projection: a = RMSNorm(x); q, k, v = a W^T; RoPE on q and k."""
    act = cfg.act
    T = x.shape[0]
    Hq, Hkv, hd = cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim
    a = storage_round(rmsnorm(x, cfg.rms_eps), act)
    qkv = _a(a) @ _a(model.w(l, "w_qkv")).T
    q = qkv[:, :Hq * hd].reshape(T, Hq, hd)
    k = qkv[:, Hq * hd:(Hq + Hkv) * hd].reshape(T, Hkv, hd)
    v = qkv[:, (Hq + Hkv) * hd:].reshape(T, Hkv, hd)
    q = storage_round(rope(q, pos, cfg.rope_theta), act)
    k = storage_round(rope(k, pos, cfg.rope_theta), act)
    v = storage_round(v, act)
    return q, k, v


def layer_rest(cfg, model: OracleModel, l: int, x, q, k, v, kc, vc, causal: bool, info=None,
               forced=None):
    """Attention, output projection with residual, and the MoE FFN with residual.

    x and the returned layer output are the residual stream (unrounded).  ``forced``: optional
    expert choices [T, k] for this layer (see router_topk)."""
    act = cfg.act
    T = x.shape[0]
    o = storage_round(attention(q, kc, vc, k, v, causal), act).reshape(T, -1)
    h = _a(x) + _a(o) @ _a(model.w(l, "w_o")).T
    y = storage_round(rmsnorm(h, cfg.rms_eps), act)
    idx, gates, z = router_topk(y, model.w(l, "w_router"), cfg.top_k, forced)
    if info is not None:
        info.setdefault("router_margin", []).append(router_margin(z, cfg.top_k))
        info.setdefault("router_idx", []).append(idx)
    idx, gates = with_shared_experts(idx, gates, cfg.n_experts, getattr(cfg, "n_shared", 0))
    return moe_ffn(y, idx, gates, lambda e: model.expert(l, e), h, act)


def lm_head_rows(cfg, model: OracleModel, x_rows: np.ndarray, keep_logits: bool = False):
    """Final RMSNorm of the given rows, logits over [0, V), entropy and argmax.

    The normalised rows are stored in the activation type, except in front of an NVFP4 LM head:
    its dequantised weights (e2m1 times an E4M3 scale, exact in fp16) meet the rows in an fp16
    product, so the rows are stored in fp16 (the reading taken for the NVFP4 workload)."""
    if getattr(cfg, "emb", "") == "nvfp4":
        f = round_f16(rmsnorm(x_rows, cfg.rms_eps))
    else:
        f = storage_round(rmsnorm(x_rows, cfg.rms_eps), cfg.act)
    R = f.shape[0]
    z = np.empty((R, cfg.vocab))
    for v0, w in model.lm_head_chunks():
        z[:, v0:v0 + w.shape[0]] = _a(f) @ _a(w).T
    H, am, margin = entropy_argmax(z)
    return H, am, margin, (z if keep_logits else None)


def canvas_forward(cfg, model: OracleModel, tokens: np.ndarray, masked: np.ndarray,
                   kcache: np.ndarray, vcache: np.ndarray, cache_len: int, info=None,
                   forced=None, drafts: bool = False):
    """Decoder pass over one canvas.  Returns the final residual stream [C, d].

    kcache, vcache: [L, Hkv, cap, hd] for this canvas (decoded values).  ``forced``: optional
    expert choices [L, C, k] (see router_topk).  ``drafts``: positions that are not final are
    embedded by their draft token (the noise canvas) instead of MASK.
    """
    C = tokens.shape[0]
    ids = tokens if drafts else np.where(masked != 0, cfg.mask_id, tokens)
    x = model.emb_rows(ids)
    pos = cache_len + np.arange(C)
    for l in range(cfg.n_layers):
        q, k, v = layer_qkv(cfg, model, l, x, pos)
        x = layer_rest(cfg, model, l, x, q, k, v, kcache[l, :, :cache_len],
                       vcache[l, :, :cache_len], False, info,
                       None if forced is None else forced[l])
    return x


def canvas_step(cfg, model: OracleModel, state: dict, kcache: np.ndarray, vcache: np.ndarray,
                cache_len: np.ndarray, gamma: float, max_steps: int, keep_logits: bool = False,
                forced=None, sampler: Optional[dict] = None):
    """One denoising step for every canvas of the batch that is not done.

    state: tokens int32 [B, C], masked uint8 [B, C], n_masked int32 [B],
    done int32 [B], step int32 [B] (numpy; not modified).  kcache/vcache:
    decoded [L, B, Hkv, cap, hd].
    For each live canvas: decoder pass; for every masked position the entropy
    (stored as fp32) and greedy argmax of its logits; EB selection (all masked
    positions at step index max_steps - 1); commit selected positions to their
    argmax; step += 1; done = no masked position left.
    ``forced`` (optional, [L, B, C, k]): every layer's expert choices (see router_topk).
    ``sampler`` (optional): {"tau_start", "tau_end", "seed", "revise"} — the temperature-annealed
    Gumbel-max draw of each masked position's token (tau_s of the canvas's step), the EB rule on
    the entropies at tau_s, and with "revise" the noise-canvas drafts (see the sampler-variant
    readings above).  Without it: greedy argmax, entropy at tau = 1, absorbing MASK positions.
    Returns (new_state, info) where info[b] holds H, argmax (the chosen tokens), margin, rows,
    selected, tau, router margins and (optionally) logits.
    """
    new = {k: np.array(v, copy=True) for k, v in state.items()}
    infos: List[Optional[Dict]] = []
    B = state["tokens"].shape[0]
    for b in range(B):
        if state["done"][b]:
            infos.append(None)
            continue
        masked = state["masked"][b]
        rows = np.nonzero(masked)[0]
        info: Dict = {"rows": rows}
        if len(rows) > 0:
            revise = bool(sampler and sampler.get("revise"))
            x = canvas_forward(cfg, model, state["tokens"][b], masked, kcache[:, b], vcache[:, b],
                               int(cache_len[b]), info,
                               None if forced is None else forced[:, b], drafts=revise)
            H, am, margin, z = lm_head_rows(cfg, model, x[rows], keep_logits or sampler is not None)
            if sampler is not None:
                tau = temperature(int(state["step"][b]), max_steps, sampler["tau_start"],
                                  sampler["tau_end"])
                info["tau"] = tau
                for j, i in enumerate(rows):
                    g = None if not tau > 0.0 else gumbel(stream_words(
                        sampler["seed"], TAG_DENOISE, b, int(i), int(state["step"][b]), cfg.vocab))
                    H[j], am[j], margin[j] = sample_row(z[j], tau, g)
                if not keep_logits:
                    z = None
            Hf = H.astype(np.float32)
            full_H = np.zeros(cfg.canvas, dtype=np.float32)
            full_H[rows] = Hf
            force = state["step"][b] >= max_steps - 1
            sel = eb_select(full_H, masked, gamma, force)
            if sampler is not None and sampler.get("revise"):   # drafts take the predictions
                new["tokens"][b, rows] = am
            new["tokens"][b, sel] = am[np.searchsorted(rows, np.nonzero(sel)[0])]
            new["masked"][b, sel] = 0
            info.update(H=Hf, argmax=am, margin=margin, logits=z, selected=sel)
        new["n_masked"][b] = int(new["masked"][b].sum())
        new["step"][b] = state["step"][b] + 1
        new["done"][b] = int(new["n_masked"][b] == 0)
        infos.append(info)
    return new, infos


def kv_append(cfg, model: OracleModel, tokens: np.ndarray, kcache: np.ndarray, vcache: np.ndarray,
              cache_len: np.ndarray, info=None, forced=None, last_rows: Optional[list] = None):
    """Causal encoder pass over finished tokens; their K/V go to the cache.

    tokens int32 [B, n]; kcache/vcache decoded [L, B, Hkv, cap, hd], updated in
    place (rows [len, len+n) of every layer, values as stored).  The encoder
    shares the decoder's weights; its attention sees the whole cache and the
    new tokens causally.  Returns the new cache_len.  With ``info`` (a dict) given, the expert
    choices of each routed layer are collected in info["router_idx"][l] as [B, n, k].
    ``forced`` (optional, [L, B, n, k]): every layer's expert choices (see router_topk).
    ``last_rows`` (a list, optional): the last layer also runs its attention and expert FFN,
    and the final residual row of each sequence's last new token is appended to the list (the
    autoregressive mode's LM-head input).
    """
    B, n = tokens.shape
    new_len = np.array(cache_len, copy=True)
    for b in range(B):
        L0 = int(cache_len[b])
        x = model.emb_rows(tokens[b])
        pos = L0 + np.arange(n)
        for l in range(cfg.n_layers):
            q, k, v = layer_qkv(cfg, model, l, x, pos)
            kc, vc = kcache[l, b, :, :L0], vcache[l, b, :, :L0]
            if l + 1 < cfg.n_layers or last_rows is not None:
                li = {} if info is not None else None
                x = layer_rest(cfg, model, l, x, q, k, v, kc, vc, True, li,
                               None if forced is None else forced[l, b])
                if info is not None:
                    ri = info.setdefault("router_idx", [np.zeros((B, n, cfg.top_k), np.int32)
                                                        for _ in range(cfg.n_layers)])
                    ri[l][b] = li["router_idx"][0]
            kcache[l, b, :, L0:L0 + n] = k.transpose(1, 0, 2)
            vcache[l, b, :, L0:L0 + n] = v.transpose(1, 0, 2)
        new_len[b] = L0 + n
        if last_rows is not None:
            last_rows.append(x[n - 1])
    return new_len


def ar_step(cfg, model: OracleModel, tokens: np.ndarray, kcache: np.ndarray, vcache: np.ndarray,
            cache_len: np.ndarray, tau: float = 0.0, seed: int = 0, info=None, forced=None):
    """Autoregressive mode: append tokens [B, n] (the causal encoder; K/V into the cache, updated
    in place), run the last layer in full, and predict each sequence's next token from the final
    RMSNorm + LM head of its last new row.  tau > 0 draws it from softmax(z / tau) with the
    Gumbel stream (TAG_AR, b, p, 0), p = the position of the predicted token (cache_len + n).
    Returns (next tokens int32 [B], entropies fp32 [B], key margins [B], new cache_len, logits
    [B, V])."""
    B, n = tokens.shape
    last: list = []
    new_len = kv_append(cfg, model, tokens, kcache, vcache, cache_len, info, forced, last)
    H, am, margin, z = lm_head_rows(cfg, model, np.stack(last), keep_logits=True)
    for b in range(B):
        g = None
        if tau > 0.0:
            g = gumbel(stream_words(seed, TAG_AR, b, int(cache_len[b]) + n, 0, cfg.vocab))
        H[b], am[b], margin[b] = sample_row(z[b], tau, g)
    return am.astype(np.int32), H.astype(np.float32), margin, new_len, z


def generate(cfg, model: OracleModel, kcache, vcache, cache_len, n_canvases: int, gamma: float,
             max_steps: int):
    """Block-autoregressive loop: denoise a canvas from all-MASK until done, append it.

    Returns (tokens [B, n_canvases, C], steps per canvas [B, n_canvases], cache_len).
    """
    B, C = cfg.batch, cfg.canvas
    out = np.zeros((B, n_canvases, C), dtype=np.int32)
    steps = np.zeros((B, n_canvases), dtype=np.int32)
    for c in range(n_canvases):
        st = {"tokens": np.full((B, C), cfg.mask_id, dtype=np.int32),
              "masked": np.ones((B, C), dtype=np.uint8),
              "n_masked": np.full(B, C, dtype=np.int32),
              "done": np.zeros(B, dtype=np.int32), "step": np.zeros(B, dtype=np.int32)}
        while not st["done"].all():
            st, _ = canvas_step(cfg, model, st, kcache, vcache, cache_len, gamma, max_steps)
        out[:, c] = st["tokens"]
        steps[:, c] = st["step"]
        cache_len = kv_append(cfg, model, st["tokens"], kcache, vcache, cache_len)
    return out, steps, cache_len
