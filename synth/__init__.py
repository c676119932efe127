"""Seeded synthetic inputs for the canvas-step library, its tests and its benchmark.

This module is shared by the CUDA path's callers and by the oracle, so it holds
no arithmetic of the method: only the workload shapes and the draws of random
weights, prompt K/V and canvas states.  Everything is drawn from one
``torch.Generator`` per call, in a fixed order, so that a (config, seed,
device) triple always gives the same tensors.

Workloads (DiffusionGemma Technical Report, Figure 11 / Figure 12 shapes; the
model card "diffusiongemma", Mixture-of-Experts bullet, 8 of 128 experts):

* ``tiny``      fp32, d_model 64, 2 q / 1 kv heads of 32, 8 experts top-2,
                 expert FFN 128, vocab 512, canvas 16, prompt 32, gamma 0.1,
                 at most 16 steps, 2 canvases with a KV append between them.
* ``layer``     one bf16 decoder layer, d_model 2048, 16 q / 8 kv heads of 128,
                 128 experts top-8, expert FFN 768, vocab 262144, canvas 256,
                 prompt K/V 4096 tokens ~N(0,1), gamma 1.0.
* ``stack30``   30 of those layers, prompt 2048 ids prefilled through the
                 append path, 4 canvases of at most 32 steps.
* ``longctx``   the one layer with 131072 prompt K/V tokens, half committed.
* ``batch32``   32 canvases of 256 through the one layer, FP8 e4m3 expert and
                 attention weights with one fp32 scale per output channel,
                 1024 prompt tokens each, router logits ~N(0,1).
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import numpy as np
import torch

__all__ = ["Cfg", "WORKLOADS", "get_config", "make_model", "make_prompt_kv",
           "make_canvas_state", "to_numpy", "reduced"]


@dataclasses.dataclass(frozen=True)
class Cfg:
    name: str
    d_model: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    n_experts: int
    top_k: int
    d_ff: int
    vocab: int
    canvas: int
    n_layers: int
    act: str                 # "f32" or "bf16": storage type of activations and K/V
    w: str                   # "f32", "bf16" or "e4m3": storage type of layer weights
    batch: int
    prompt_len: int
    gamma: float
    max_steps: int
    n_canvases: int
    seed: int
    weight_std: float = 0.02
    router_std: float = 0.02
    rope_theta: float = 10000.0
    rms_eps: float = 1e-6
    state: str = "all_mask"  # initial canvas state: "all_mask" or "half"
    prefill_ids: bool = False  # prompt given as token ids (prefilled by the append path)
    emb: str = ""            # tied embedding / LM head storage: "" = the activation type, or "nvfp4"
    n_shared: int = 0        # always-on shared experts, stored after the routed ones

    @property
    def mask_id(self) -> int:
        return self.vocab

    @property
    def qkv_rows(self) -> int:
        return (self.n_q_heads + 2 * self.n_kv_heads) * self.head_dim

    @property
    def cache_cap(self) -> int:
        return self.prompt_len + self.n_canvases * self.canvas


WORKLOADS: Dict[str, Cfg] = {
    "tiny": Cfg("tiny", 64, 2, 1, 32, 8, 2, 128, 512, 16, 1, "f32", "f32", 1, 32,
                0.1, 16, 2, 0),
    "layer": Cfg("layer", 2048, 16, 8, 128, 128, 8, 768, 262144, 256, 1, "bf16", "bf16",
                 1, 4096, 1.0, 256, 1, 1),
    "stack30": Cfg("stack30", 2048, 16, 8, 128, 128, 8, 768, 262144, 256, 30, "bf16",
                   "bf16", 1, 2048, 1.0, 32, 4, 2, prefill_ids=True),
    "longctx": Cfg("longctx", 2048, 16, 8, 128, 128, 8, 768, 262144, 256, 1, "bf16",
                   "bf16", 1, 131072, 1.0, 256, 1, 3, state="half"),
    "batch32": Cfg("batch32", 2048, 16, 8, 128, 128, 8, 768, 262144, 256, 1, "bf16",
                   "e4m3", 32, 1024, 1.0, 256, 1, 4,
                   router_std=1.0 / float(np.sqrt(2048.0))),
    # the layer workload with the tied embedding / LM head stored in NVFP4
    "layer_nvfp4": Cfg("layer_nvfp4", 2048, 16, 8, 128, 128, 8, 768, 262144, 256, 1, "bf16",
                       "bf16", 1, 4096, 1.0, 256, 1, 5, emb="nvfp4"),
}

# NVFP4 storage of the embedding (see make_nvfp4_emb): k-blocks of 64 elements, 16-element
# scale blocks, rows padded to a multiple of NVFP4_ROW_PAD
NVFP4_KB = 64
NVFP4_BLOCK = 16
NVFP4_ROW_PAD = 256


def get_config(name: str, **overrides) -> Cfg:
    return dataclasses.replace(WORKLOADS[name], **overrides)


def reduced(name: str, **overrides) -> Cfg:
    """A shape-reduced copy of a workload for fast parity runs.

    Keeps head_dim, head counts, top_k and the storage types (so the same kernel
    code paths run) but shrinks the dims the oracle pays for.
    """
    base = WORKLOADS[name]
    small = dict(d_model=256, n_experts=16, d_ff=128, vocab=4096, canvas=64,
                 prompt_len=192, name=base.name + "-reduced")
    small.update(overrides)
    return dataclasses.replace(base, **small)


def _dtype(kind: str) -> torch.dtype:
    return {"f32": torch.float32, "bf16": torch.bfloat16}[kind]


def _normal(g, shape, std, device):
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std


def _store_weight(w32: torch.Tensor, kind: str):
    """Cast a drawn fp32 weight [rows, cols] to its storage type.

    For e4m3 the per-row (output channel) scale maps the row's largest magnitude
    to 448, the largest finite e4m3 value; torch performs the rounding.
    """
    if kind == "e4m3":
        amax = w32.abs().amax(dim=-1, keepdim=True).clamp_min(1e-30)
        scale = amax / 448.0
        codes = (w32 / scale).to(torch.float8_e4m3fn).view(torch.uint8)
        return codes, scale.squeeze(-1).contiguous()
    return w32.to(_dtype(kind)), None


def nvfp4_rows_padded(n_rows: int) -> int:
    return (n_rows + NVFP4_ROW_PAD - 1) // NVFP4_ROW_PAD * NVFP4_ROW_PAD


def make_nvfp4_emb(g, n_rows: int, d: int, std: float, device):
    """Draw an embedding [n_rows, d] directly in NVFP4 storage (no rounding of drawn values).

    Returns (codes, scales, tensor_scale):
      codes  uint8 [d/64][Rp][32]: k-block kb, row r; byte i holds element kb*64 + 2i in its low
             nibble and element kb*64 + 2i + 1 in its high nibble (FP4 E2M1 codes);
      scales uint8 [d/64][Rp][4]: the FP8 E4M3 scale of elements kb*64 + 16j .. + 15 of row r;
      tensor_scale: one fp32 value; element = e2m1(code) * e4m3(scale) * tensor_scale.
    Rp = n_rows rounded up to 256; rows [n_rows, Rp) are zero.  Codes are uniform over all 16
    values and scales uniform over the E4M3 codes 0x30..0x3F (0.5 .. 1.875), whose RMS products
    are 3.391; the tensor scale brings the element RMS to std.
    """
    Rp = nvfp4_rows_padded(n_rows)
    nk = d // NVFP4_KB
    codes = torch.randint(0, 256, (nk, Rp, NVFP4_KB // 2), generator=g, device=device,
                          dtype=torch.int32).to(torch.uint8)
    scales = torch.randint(0x30, 0x40, (nk, Rp, NVFP4_KB // NVFP4_BLOCK), generator=g,
                           device=device, dtype=torch.int32).to(torch.uint8)
    codes[:, n_rows:] = 0
    scales[:, n_rows:] = 0
    return codes.contiguous(), scales.contiguous(), float(std / 3.391)


def make_model(cfg: Cfg, device="cpu", seed: Optional[int] = None) -> dict:
    """Draw the tied embedding / LM head and every layer's weights.

    Order of draws: embedding [V+1, d]; then per layer: W_qkv, W_o, W_router,
    W_gate_up (expert by expert), W_down (expert by expert).
    Row ``vocab`` of the embedding is the MASK token's row.
    """
    seed = cfg.seed if seed is None else seed
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    d, std = cfg.d_model, cfg.weight_std
    emb_kind = "f32" if cfg.act == "f32" else "bf16"
    if cfg.emb == "nvfp4":
        codes, scales, ts = make_nvfp4_emb(g, cfg.vocab + 1, d, std, device)
        model = {"emb": codes, "emb_scale": scales, "emb_scale_global": ts, "layers": []}
    else:
        model = {"emb": _normal(g, (cfg.vocab + 1, d), std, device).to(_dtype(emb_kind)),
                 "layers": []}
    for _ in range(cfg.n_layers):
        lay = {}
        lay["w_qkv"], lay["s_qkv"] = _store_weight(_normal(g, (cfg.qkv_rows, d), std, device), cfg.w)
        lay["w_o"], lay["s_o"] = _store_weight(
            _normal(g, (d, cfg.n_q_heads * cfg.head_dim), std, device), cfg.w)
        rkind = "f32" if cfg.w == "f32" else "bf16"
        lay["w_router"], _ = _store_weight(_normal(g, (cfg.n_experts, d), cfg.router_std, device), rkind)
        gus, gss, dws, dss = [], [], [], []
        n_all = cfg.n_experts + cfg.n_shared   # shared experts are drawn after the routed ones
        for _e in range(n_all):
            w, s = _store_weight(_normal(g, (2 * cfg.d_ff, d), std, device), cfg.w)
            gus.append(w)
            gss.append(s)
        for _e in range(n_all):
            w, s = _store_weight(_normal(g, (d, cfg.d_ff), std, device), cfg.w)
            dws.append(w)
            dss.append(s)
        lay["w_gate_up"] = torch.stack(gus)
        lay["w_down"] = torch.stack(dws)
        lay["s_gate_up"] = torch.stack(gss) if cfg.w == "e4m3" else None
        lay["s_down"] = torch.stack(dss) if cfg.w == "e4m3" else None
        model["layers"].append(lay)
    return model


def make_prompt_kv(cfg: Cfg, device="cpu", seed: Optional[int] = None, cap: Optional[int] = None):
    """Prompt K/V caches [L][B][H_kv][cap][head_dim] with rows [0, P) ~ N(0,1).

    The synthetic prompt keys are taken as already position-rotated.  For a
    workload whose prompt is given as ids (``prefill_ids``) the caches start
    empty and the ids are returned instead, to be prefilled by the append path.
    """
    seed = (cfg.seed if seed is None else seed) + 1000003
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    cap = cfg.cache_cap if cap is None else cap
    shape = (cfg.n_layers, cfg.batch, cfg.n_kv_heads, cap, cfg.head_dim)
    dt = _dtype(cfg.act)
    k = torch.zeros(shape, dtype=dt, device=device)
    v = torch.zeros(shape, dtype=dt, device=device)
    out = {"k": k, "v": v}
    if cfg.prefill_ids:
        out["prompt_ids"] = torch.randint(0, cfg.vocab, (cfg.batch, cfg.prompt_len),
                                          generator=g, device=device, dtype=torch.int64).to(torch.int32)
        out["cache_len"] = torch.zeros(cfg.batch, dtype=torch.int32, device=device)
        return out
    P = cfg.prompt_len
    for l in range(cfg.n_layers):
        k[l, :, :, :P] = _normal(g, (cfg.batch, cfg.n_kv_heads, P, cfg.head_dim), 1.0, device).to(dt)
        v[l, :, :, :P] = _normal(g, (cfg.batch, cfg.n_kv_heads, P, cfg.head_dim), 1.0, device).to(dt)
    out["cache_len"] = torch.full((cfg.batch,), P, dtype=torch.int32, device=device)
    return out


def make_canvas_state(cfg: Cfg, kind: Optional[str] = None, device="cpu", seed: Optional[int] = None):
    """Canvas state of ``cfg.batch`` canvases.

    ``all_mask``: every position holds MASK (id = vocab).
    ``half``: a seeded permutation of the positions; its first half is already
    committed to ids drawn uniformly from [0, vocab).
    """
    kind = cfg.state if kind is None else kind
    seed = (cfg.seed if seed is None else seed) + 2000003
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    B, C = cfg.batch, cfg.canvas
    tokens = torch.full((B, C), cfg.mask_id, dtype=torch.int32)
    masked = torch.ones((B, C), dtype=torch.uint8)
    if kind == "half":
        for b in range(B):
            perm = torch.randperm(C, generator=g)
            ids = torch.randint(0, cfg.vocab, (C // 2,), generator=g, dtype=torch.int64)
            tokens[b, perm[:C // 2]] = ids.to(torch.int32)
            masked[b, perm[:C // 2]] = 0
    elif kind != "all_mask":
        raise ValueError(kind)
    st = {"tokens": tokens, "masked": masked,
          "n_masked": masked.sum(dim=1).to(torch.int32),
          "done": torch.zeros(B, dtype=torch.int32),
          "step": torch.zeros(B, dtype=torch.int32)}
    return {k: v.to(device) for k, v in st.items()}


def to_numpy(t: Optional[torch.Tensor]):
    """Host copy as numpy: bf16 as uint16 bit patterns, e4m3 codes as uint8."""
    if t is None:
        return None
    t = t.detach().to("cpu")
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16).copy()
    return t.numpy().copy()
