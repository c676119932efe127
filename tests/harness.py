"""Helpers shared by the GPU parity tests: put a synthetic workload on the device, build the
oracle's view of the same numbers, and run the library through its C ABI."""
from __future__ import annotations

import numpy as np
import torch

import synth
from oracle import dg_oracle as O
from block_discrete_diffusion_dg_b200 import binding as B


# Factor between the spread of two oracle evaluations (fp64 and fp32 arithmetic, same storage
# rounding, same expert choices) and the bar a device result is held to.  The device is one more
# fp32 evaluation with its own summation order: it and the fp32 oracle can each sit up to the
# spread S away from the fp64 result, on either side, so a bar of 2 S covers it.  Fixed before any
# device result was compared with it.
BAR_FACTOR = 2.0


class _LazyTensor:
    """A device tensor that the oracle reads piecewise: x[i] copies one slice to the host, and
    np.asarray(x) the whole tensor (so a deep stack's weights never all sit in host memory)."""

    def __init__(self, t):
        self.t = t

    def __getitem__(self, i):
        return synth.to_numpy(self.t[i])

    def __array__(self, dtype=None, copy=None):
        a = synth.to_numpy(self.t)
        return a if dtype is None else a.astype(dtype)


class _LazyLayer(dict):
    def __init__(self, lay):
        super().__init__({k: (None if v is None else _LazyTensor(v)) for k, v in lay.items()})


def oracle_model(cfg, model, lazy: bool = False) -> O.OracleModel:
    """The oracle's view of a device model.  lazy: layer weights are copied to the host slice by
    slice when the oracle reads them (for stacks too large to hold decoded in host memory)."""
    if lazy:
        layers = [_LazyLayer(lay) for lay in model["layers"]]
    else:
        layers = [{k: synth.to_numpy(v) for k, v in lay.items()} for lay in model["layers"]]
    arr = {"emb": synth.to_numpy(model["emb"]), "layers": layers}
    if "emb_scale" in model:
        arr["emb_scale"] = synth.to_numpy(model["emb_scale"])
        arr["emb_scale_global"] = float(model["emb_scale_global"])
    return O.OracleModel(cfg, arr)


def decode_cache(cfg, t: torch.Tensor) -> np.ndarray:
    return O.decode_act(synth.to_numpy(t), cfg.act)


def to_device(obj, device="cuda"):
    if isinstance(obj, torch.Tensor):
        return obj.to(device)
    if isinstance(obj, dict):
        return {k: to_device(v, device) for k, v in obj.items()}
    if isinstance(obj, list):
        return [to_device(v, device) for v in obj]
    return obj


class Workload:
    """Device-resident workload: model, caches, canvas state, dg_config and scratch."""

    def __init__(self, cfg, gen_device="cuda", state_kind=None, cap=None):
        self.cfg = cfg
        model = synth.make_model(cfg, gen_device)
        kv = synth.make_prompt_kv(cfg, gen_device, cap=cap)
        self.model = to_device(model)
        self.kv = to_device(kv)
        self.cap = self.kv["k"].shape[3]
        self.state = to_device(synth.make_canvas_state(cfg, state_kind))
        self.dgcfg = B.make_config(cfg)
        self.dgmodel = B.Model(self.model)
        self.ws = B.alloc_workspace(self.dgcfg, cfg.batch, cfg.canvas, self.cap)
        self.status = torch.zeros(1, dtype=torch.int32, device="cuda")

    def oracle(self) -> O.OracleModel:
        return oracle_model(self.cfg, self.model)

    def step(self, state=None, gamma=None, max_steps=None, logits=False, forced=None):
        """One dg_canvas_step on a copy of `state`; returns (new_state, entropy, argmax, logits)."""
        cfg = self.cfg
        st = {k: v.clone() for k, v in (state or self.state).items()}
        B_, C = cfg.batch, cfg.canvas
        ent = torch.full((B_, C), float("nan"), dtype=torch.float32, device="cuda")
        am = torch.full((B_, C), -1, dtype=torch.int32, device="cuda")
        lg = torch.zeros((B_ * C, cfg.vocab), dtype=torch.float32, device="cuda") if logits else None
        B.dg_canvas_step(self.dgcfg, self.dgmodel, B_, st["tokens"], st["masked"], st["n_masked"],
                         st["done"], st["step"], cfg.max_steps if max_steps is None else max_steps,
                         cfg.gamma if gamma is None else gamma, self.kv["k"], self.kv["v"],
                         self.kv["cache_len"], self.cap, ent, am, lg, self.ws, self.status,
                         forced_topk=forced)
        torch.cuda.synchronize()
        return st, ent, am, lg

    def check_status(self):
        rc = B.dg_read_status(self.status)
        assert rc == B.DG_OK, B.STATUS_NAMES.get(rc, rc)


def forced_from(cfg, infos) -> np.ndarray:
    """The oracle's expert choices of one step, [L][B][C][k] (zeros for skipped canvases)."""
    f = np.zeros((cfg.n_layers, cfg.batch, cfg.canvas, cfg.top_k), np.int32)
    for b, inf in enumerate(infos):
        if inf is None or "router_idx" not in inf:
            continue
        for l, idx in enumerate(inf["router_idx"]):
            f[l, b] = idx
    return f


def step_spread(cfg, om, st, kc, vc, cl, infos):
    """Spread of the step's logits and entropies between the fp64 oracle (infos) and the same
    oracle in fp32 arithmetic on the same inputs and expert choices: (max |dz|, max |dH| / H)."""
    with O.accumulation(np.float32):
        _, inf32 = O.canvas_step(cfg, om, st, kc, vc, cl, cfg.gamma, cfg.max_steps,
                                 keep_logits=True, forced=forced_from(cfg, infos))
    dz, dh = 0.0, 0.0
    for a, b in zip(infos, inf32):
        if a is None or len(a["rows"]) == 0:
            continue
        dz = max(dz, float(np.abs(b["logits"] - a["logits"]).max()))
        dh = max(dh, float((np.abs(b["H"].astype(np.float64) - a["H"]) / a["H"]).max()))
    return dz, dh


def rel_to_row_rms(g, o):
    """|g - o| relative to the RMS of o's row (last axis)."""
    scale = np.sqrt(np.mean(o * o, axis=-1, keepdims=True)) + 1e-30
    return np.abs(g - o) / scale


def np_state(st):
    return {k: synth.to_numpy(v) for k, v in st.items()}


def torch_state(st, device="cuda"):
    return {k: torch.from_numpy(np.ascontiguousarray(v)).to(device) for k, v in st.items()}
