"""Helpers shared by the GPU parity tests: put a synthetic workload on the device, build the
oracle's view of the same numbers, and run the library through its C ABI."""
from __future__ import annotations

import numpy as np
import torch

import synth
from oracle import dg_oracle as O
from block_discrete_diffusion_dg_b200 import binding as B


def oracle_model(cfg, model) -> O.OracleModel:
    arr = {"emb": synth.to_numpy(model["emb"]),
           "layers": [{k: synth.to_numpy(v) for k, v in lay.items()} for lay in model["layers"]]}
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


def np_state(st):
    return {k: synth.to_numpy(v) for k, v in st.items()}


def torch_state(st, device="cuda"):
    return {k: torch.from_numpy(np.ascontiguousarray(v)).to(device) for k, v in st.items()}
