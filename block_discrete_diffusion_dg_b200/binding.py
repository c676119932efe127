"""Thin ctypes binding of ``libdg.so`` (the C ABI in include/dg.h).

Argument marshalling only: every step of the computation runs in the library's CUDA kernels.
Functions carry the C names; tensors are passed as torch tensors (device memory) and turned into
raw pointers; a non-zero status raises :class:`DgError`.  There is no fallback: if the shared
library is missing, :func:`lib` raises.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdg.so")

DG_OK, DG_ERR_INVALID_ARG, DG_ERR_UNSUPPORTED, DG_ERR_CAPACITY, DG_ERR_CUDA, \
    DG_ERR_NUMERIC, DG_ERR_TIMEOUT, DG_ERR_WORKSPACE = range(8)
DG_F32, DG_BF16, DG_E4M3, DG_NVFP4 = 0, 1, 2, 3
STATUS_NAMES = {0: "DG_OK", 1: "DG_ERR_INVALID_ARG", 2: "DG_ERR_UNSUPPORTED", 3: "DG_ERR_CAPACITY",
                4: "DG_ERR_CUDA", 5: "DG_ERR_NUMERIC", 6: "DG_ERR_TIMEOUT", 7: "DG_ERR_WORKSPACE"}


class DgError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {STATUS_NAMES.get(code, code)}"
                         + (f" ({_lib.dg_last_cuda_error().decode()})" if code == DG_ERR_CUDA and _lib else ""))
        self.code = code


class DgConfig(ctypes.Structure):
    _fields_ = [("d_model", ctypes.c_int32), ("n_q_heads", ctypes.c_int32),
                ("n_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("n_experts", ctypes.c_int32), ("top_k", ctypes.c_int32), ("d_ff", ctypes.c_int32),
                ("vocab", ctypes.c_int32), ("canvas", ctypes.c_int32), ("n_layers", ctypes.c_int32),
                ("rope_theta", ctypes.c_double), ("rms_eps", ctypes.c_double),
                ("act_dtype", ctypes.c_int32), ("w_dtype", ctypes.c_int32),
                ("emb_dtype", ctypes.c_int32), ("n_shared", ctypes.c_int32)]


class DgLayerWeights(ctypes.Structure):
    _fields_ = [("w_qkv", ctypes.c_void_p), ("s_qkv", ctypes.c_void_p),
                ("w_o", ctypes.c_void_p), ("s_o", ctypes.c_void_p),
                ("w_router", ctypes.c_void_p),
                ("w_gate_up", ctypes.c_void_p), ("s_gate_up", ctypes.c_void_p),
                ("w_down", ctypes.c_void_p), ("s_down", ctypes.c_void_p)]


class DgModel(ctypes.Structure):
    _fields_ = [("layers", ctypes.POINTER(DgLayerWeights)), ("emb", ctypes.c_void_p),
                ("emb_scale", ctypes.c_void_p), ("emb_scale_global", ctypes.c_float)]


class DgSampler(ctypes.Structure):
    """dg_sampler: temperature schedule (tau_start at step 0 .. tau_end at the last step of the
    budget; <= 0 greedy), the generator's 64-bit seed, and revisable drafts (noise canvas)."""
    _fields_ = [("tau_start", ctypes.c_double), ("tau_end", ctypes.c_double),
                ("seed", ctypes.c_uint64), ("revise", ctypes.c_int32)]


def make_sampler(tau_start=0.0, tau_end=None, seed=0, revise=False) -> DgSampler:
    return DgSampler(float(tau_start), float(tau_start if tau_end is None else tau_end),
                     int(seed) & 0xFFFFFFFFFFFFFFFF, 1 if revise else 0)


_lib: Optional[ctypes.CDLL] = None
_VP, _I32, _SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
_PCFG, _PMODEL, _PLW = ctypes.POINTER(DgConfig), ctypes.POINTER(DgModel), ctypes.POINTER(DgLayerWeights)
_PSMP = ctypes.POINTER(DgSampler)

_SIGS = {
    "dg_workspace_size": (_SZ, [_PCFG, _I32, _I32, _I32]),
    "dg_read_status": (_I32, [_VP, _VP]),
    "dg_clear_status": (_I32, [_VP, _VP]),
    "dg_last_cuda_error": (ctypes.c_char_p, []),
    "dg_launch_count": (ctypes.c_uint64, []),
    "dg_profile_begin": (_I32, [_I32]),
    "dg_profile_mark": (_I32, [_VP]),
    "dg_profile_end": (_I32, [ctypes.POINTER(ctypes.c_float), _I32, ctypes.POINTER(ctypes.c_int)]),
    "dg_profile_name": (ctypes.c_char_p, [_I32]),
    "dg_canvas_attn": (_I32, [_PCFG, _I32, _I32, _VP, _VP, _VP, _VP, _I32, _VP, _VP, _I32, _VP,
                              _VP, _VP, _SZ, _VP, _VP]),
    "dg_moe_route": (_I32, [_PCFG, _I32, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _SZ, _VP, _VP]),
    "dg_moe_ffn": (_I32, [_PCFG, _I32, _VP, _VP, _VP, _VP, _VP, _VP, _PLW, _VP, _VP, _VP, _SZ, _VP,
                          _VP]),
    "dg_logits_entropy": (_I32, [_PCFG, _I32, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _SZ, _VP, _VP]),
    "dg_logits_entropy_static": (_I32, [_PCFG, _I32, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP]),
    "dg_logits_entropy_nvfp4": (_I32, [_PCFG, _I32, _VP, _VP, _VP, _VP, _VP, ctypes.c_float, _VP,
                                       _VP, _VP, _VP, _SZ, _VP, _VP]),
    "dg_eb_select": (_I32, [_I32, _I32, _VP, _VP, ctypes.c_double, _I32, _VP, _VP, _VP, _VP, _VP,
                            _VP, _I32, _VP, _VP]),
    "dg_kv_append": (_I32, [_PCFG, _PMODEL, _I32, _VP, _I32, _VP, _VP, _VP, _I32, _VP, _VP, _SZ,
                            _VP, _VP]),
    "dg_canvas_step": (_I32, [_PCFG, _PMODEL, _I32, _VP, _VP, _VP, _VP, _VP, _I32, ctypes.c_double,
                              _VP, _VP, _VP, _I32, _VP, _VP, _VP, _VP, _VP, _VP, _SZ, _VP, _VP]),
    "dg_generate": (_I32, [_PCFG, _PMODEL, _I32, _VP, _VP, _VP, _VP, _VP, _I32, ctypes.c_double,
                           _PSMP, _VP, _VP, _VP, _I32, _I32, _VP, _SZ, _VP, _VP]),
    "dg_canvas_step_sampler": (_I32, [_PCFG, _PMODEL, _I32, _VP, _VP, _VP, _VP, _VP, _I32,
                                      ctypes.c_double, _PSMP, _VP, _VP, _VP, _I32, _VP, _VP, _VP,
                                      _VP, _VP, _SZ, _VP, _VP]),
    "dg_debug_wait_probe": (_I32, [ctypes.c_longlong, _I32, _VP, _VP]),
    "dg_noise_canvas": (_I32, [_I32, _I32, _I32, ctypes.c_uint64, _VP, _VP, _VP, _VP, _VP, _VP]),
    "dg_ar_step": (_I32, [_PCFG, _PMODEL, _I32, _VP, _I32, _VP, _VP, _VP, _I32, _PSMP, _VP, _VP,
                          _VP, _VP, _VP, _SZ, _VP, _VP]),
}


def lib() -> ctypes.CDLL:
    """Load libdg.so (build it with ``python -m block_discrete_diffusion_dg_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing; the CUDA library has not been built")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype, f.argtypes = res, args
        _lib = L
    return _lib


def _p(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("the library takes device tensors")
    if not t.is_contiguous():
        raise ValueError("the library takes contiguous tensors")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _check(rc: int, what: str):
    if rc != DG_OK:
        raise DgError(rc, what)


# ----------------------------------------------------------------------------- structures

def make_config(c) -> DgConfig:
    """dg_config from a workload description (``synth.Cfg`` or any object with the fields)."""
    act = DG_F32 if c.act == "f32" else DG_BF16
    emb = DG_NVFP4 if getattr(c, "emb", "") == "nvfp4" else act
    return DgConfig(c.d_model, c.n_q_heads, c.n_kv_heads, c.head_dim, c.n_experts, c.top_k, c.d_ff,
                    c.vocab, c.canvas, c.n_layers, float(c.rope_theta), float(c.rms_eps), act,
                    {"f32": DG_F32, "bf16": DG_BF16, "e4m3": DG_E4M3}[c.w], emb,
                    int(getattr(c, "n_shared", 0)))


def make_layer(lay: dict) -> DgLayerWeights:
    g = lambda k: _p(lay.get(k)) if lay.get(k) is not None else None  # noqa: E731
    return DgLayerWeights(g("w_qkv"), g("s_qkv"), g("w_o"), g("s_o"), g("w_router"),
                          g("w_gate_up"), g("s_gate_up"), g("w_down"), g("s_down"))


class Model:
    """Host-side dg_model over device weight tensors (keeps the ctypes arrays alive)."""

    def __init__(self, model: dict):
        self.tensors = model
        n = len(model["layers"])
        self.layer_array = (DgLayerWeights * n)(*[make_layer(l) for l in model["layers"]])
        sc = model.get("emb_scale")
        self.struct = DgModel(ctypes.cast(self.layer_array, ctypes.POINTER(DgLayerWeights)),
                              _p(model["emb"]), _p(sc) if sc is not None else None,
                              float(model.get("emb_scale_global", 1.0)))

    def layer(self, l: int) -> DgLayerWeights:
        return self.layer_array[l]


# ----------------------------------------------------------------------------- entry points

def dg_workspace_size(cfg: DgConfig, batch: int, n_tokens: int, cache_cap: int) -> int:
    return lib().dg_workspace_size(ctypes.byref(cfg), batch, n_tokens, cache_cap)


def alloc_workspace(cfg: DgConfig, batch: int, n_tokens: int, cache_cap: int, device="cuda"):
    n = dg_workspace_size(cfg, batch, n_tokens, cache_cap)
    if n == 0:
        raise DgError(DG_ERR_INVALID_ARG, "dg_workspace_size")
    return torch.empty(n + 256, dtype=torch.uint8, device=device)


def _ws(ws: torch.Tensor):
    base = ws.data_ptr()
    aligned = (base + 255) & ~255
    return aligned, ws.numel() - (aligned - base)


def dg_read_status(dev_status: torch.Tensor, stream=None) -> int:
    return lib().dg_read_status(_p(dev_status), _stream(stream))


def dg_clear_status(dev_status: torch.Tensor, stream=None):
    _check(lib().dg_clear_status(_p(dev_status), _stream(stream)), "dg_clear_status")


def dg_launch_count() -> int:
    return int(lib().dg_launch_count())


def dg_profile_begin(max_records: int):
    _check(lib().dg_profile_begin(max_records), "dg_profile_begin")


def dg_profile_mark(stream=None):
    _check(lib().dg_profile_mark(_stream(stream)), "dg_profile_mark")


def dg_profile_end(max_out: int = 1 << 16):
    """Returns [(kernel name, ms)] for each recorded launch (the time to the next record)."""
    buf = (ctypes.c_float * max_out)()
    n = ctypes.c_int(0)
    _check(lib().dg_profile_end(buf, max_out, ctypes.byref(n)), "dg_profile_end")
    return [(lib().dg_profile_name(i).decode(), float(buf[i])) for i in range(n.value)]


def dg_canvas_attn(cfg, batch, n_tokens, q, k_cache, v_cache, cache_len, cache_cap, k_new, v_new,
                   causal, done, out, ws, dev_status=None, stream=None):
    w, wb = _ws(ws)
    _check(lib().dg_canvas_attn(ctypes.byref(cfg), batch, n_tokens, _p(q), _p(k_cache), _p(v_cache),
                                _p(cache_len), cache_cap, _p(k_new), _p(v_new), int(causal),
                                _p(done), _p(out), w, wb, _p(dev_status), _stream(stream)),
           "dg_canvas_attn")


def dg_moe_route(cfg, n_tokens, y, w_router, token_live, topk_idx, topk_w, expert_off, perm,
                 inv_perm, ws, dev_status=None, stream=None):
    w, wb = _ws(ws)
    _check(lib().dg_moe_route(ctypes.byref(cfg), n_tokens, _p(y), _p(w_router), _p(token_live),
                              _p(topk_idx), _p(topk_w), _p(expert_off), _p(perm), _p(inv_perm),
                              w, wb, _p(dev_status), _stream(stream)), "dg_moe_route")


def dg_moe_ffn(cfg, n_tokens, y, topk_idx, topk_w, expert_off, perm, inv_perm, layer, residual,
               out, ws, dev_status=None, stream=None):
    w, wb = _ws(ws)
    _check(lib().dg_moe_ffn(ctypes.byref(cfg), n_tokens, _p(y), _p(topk_idx), _p(topk_w),
                            _p(expert_off), _p(perm), _p(inv_perm), ctypes.byref(layer),
                            _p(residual), _p(out), w, wb, _p(dev_status), _stream(stream)),
           "dg_moe_ffn")


def dg_logits_entropy(cfg, n_rows, n_rows_dev, h, row_idx, w_lm, entropy, argmax, logits_dbg, ws,
                      dev_status=None, stream=None):
    w, wb = _ws(ws)
    _check(lib().dg_logits_entropy(ctypes.byref(cfg), n_rows, _p(n_rows_dev), _p(h), _p(row_idx),
                                   _p(w_lm), _p(entropy), _p(argmax), _p(logits_dbg), w, wb,
                                   _p(dev_status), _stream(stream)), "dg_logits_entropy")


def dg_logits_entropy_static(cfg, n_rows, n_rows_dev, h, row_idx, w_lm, entropy, argmax,
                             dev_status=None, stream=None):
    """dg_logits_entropy without a scratch argument (its scratch is a fixed array in the library)."""
    _check(lib().dg_logits_entropy_static(ctypes.byref(cfg), n_rows, _p(n_rows_dev), _p(h),
                                          _p(row_idx), _p(w_lm), _p(entropy), _p(argmax),
                                          _p(dev_status), _stream(stream)),
           "dg_logits_entropy_static")


def dg_logits_entropy_nvfp4(cfg, n_rows, n_rows_dev, h, row_idx, w_codes, w_scale, w_scale_global,
                            entropy, argmax, logits_dbg, ws, dev_status=None, stream=None):
    """dg_logits_entropy with the LM head in NVFP4: uint8 codes [d/64][Vp][32], uint8 E4M3
    scales [d/64][Vp][4] and the fp32 tensor scale (cfg.emb_dtype must be DG_NVFP4)."""
    w, wb = _ws(ws)
    _check(lib().dg_logits_entropy_nvfp4(ctypes.byref(cfg), n_rows, _p(n_rows_dev), _p(h),
                                         _p(row_idx), _p(w_codes), _p(w_scale),
                                         float(w_scale_global), _p(entropy), _p(argmax),
                                         _p(logits_dbg), w, wb, _p(dev_status), _stream(stream)),
           "dg_logits_entropy_nvfp4")


def dg_eb_select(batch, canvas, entropy, argmax, gamma, max_steps, tokens, masked, selected,
                 n_masked, done, step, dev_status=None, stream=None, revise=False):
    _check(lib().dg_eb_select(batch, canvas, _p(entropy), _p(argmax), float(gamma), max_steps,
                              _p(tokens), _p(masked), _p(selected), _p(n_masked), _p(done), _p(step),
                              1 if revise else 0, _p(dev_status), _stream(stream)), "dg_eb_select")


def dg_kv_append(cfg, model: Model, batch, tokens, n_tokens, k_cache, v_cache, cache_len, cache_cap,
                 ws, dev_status=None, stream=None, forced_topk=None):
    w, wb = _ws(ws)
    _check(lib().dg_kv_append(ctypes.byref(cfg), ctypes.byref(model.struct), batch, _p(tokens),
                              n_tokens, _p(k_cache), _p(v_cache), _p(cache_len), cache_cap,
                              _p(forced_topk), w, wb, _p(dev_status), _stream(stream)),
           "dg_kv_append")


def dg_canvas_step(cfg, model: Model, batch, tokens, masked, n_masked, done, step, max_steps, gamma,
                   k_cache, v_cache, cache_len, cache_cap, entropy_out, argmax_out, logits_dbg, ws,
                   dev_status=None, stream=None, expert_load=None, forced_topk=None):
    w, wb = _ws(ws)
    _check(lib().dg_canvas_step(ctypes.byref(cfg), ctypes.byref(model.struct), batch, _p(tokens),
                                _p(masked), _p(n_masked), _p(done), _p(step), max_steps,
                                float(gamma), _p(k_cache), _p(v_cache), _p(cache_len), cache_cap,
                                _p(entropy_out), _p(argmax_out), _p(logits_dbg), _p(expert_load),
                                _p(forced_topk), w, wb, _p(dev_status), _stream(stream)),
           "dg_canvas_step")


def dg_generate(cfg, model: Model, batch, tokens, masked, n_masked, done, step, max_steps, gamma,
                k_cache, v_cache, cache_len, cache_cap, append, ws, dev_status=None, stream=None,
                sampler: Optional[DgSampler] = None):
    """The step loop on the device until every canvas is done (one CUDA graph with a
    conditional while node, cached per argument set), then the append if `append`."""
    w, wb = _ws(ws)
    _check(lib().dg_generate(ctypes.byref(cfg), ctypes.byref(model.struct), batch, _p(tokens),
                             _p(masked), _p(n_masked), _p(done), _p(step), max_steps, float(gamma),
                             None if sampler is None else ctypes.byref(sampler),
                             _p(k_cache), _p(v_cache), _p(cache_len), cache_cap, int(append), w, wb,
                             _p(dev_status), _stream(stream)),
           "dg_generate")


def dg_canvas_step_sampler(cfg, model: Model, batch, tokens, masked, n_masked, done, step,
                           max_steps, gamma, sampler: DgSampler, k_cache, v_cache, cache_len,
                           cache_cap, entropy_out, argmax_out, logits_dbg, ws, dev_status=None,
                           stream=None, forced_topk=None):
    """dg_canvas_step with a sampler variant (temperature-annealed draws, revisable drafts)."""
    w, wb = _ws(ws)
    _check(lib().dg_canvas_step_sampler(ctypes.byref(cfg), ctypes.byref(model.struct), batch,
                                        _p(tokens), _p(masked), _p(n_masked), _p(done), _p(step),
                                        max_steps, float(gamma), ctypes.byref(sampler),
                                        _p(k_cache), _p(v_cache), _p(cache_len), cache_cap,
                                        _p(entropy_out), _p(argmax_out), _p(logits_dbg),
                                        _p(forced_topk), w, wb, _p(dev_status), _stream(stream)),
           "dg_canvas_step_sampler")


def dg_noise_canvas(batch, canvas, vocab, seed, tokens, masked, n_masked, done, step, stream=None):
    """Uniform-noise canvases (every position a revisable draft)."""
    _check(lib().dg_noise_canvas(batch, canvas, vocab, int(seed) & 0xFFFFFFFFFFFFFFFF, _p(tokens),
                                 _p(masked), _p(n_masked), _p(done), _p(step), _stream(stream)),
           "dg_noise_canvas")


def dg_ar_step(cfg, model: Model, batch, tokens, n_tokens, k_cache, v_cache, cache_len, cache_cap,
               next_token, entropy, logits_dbg, ws, dev_status=None, stream=None,
               sampler: Optional[DgSampler] = None, forced_topk=None):
    """Autoregressive mode: append the tokens, predict each sequence's next token."""
    w, wb = _ws(ws)
    _check(lib().dg_ar_step(ctypes.byref(cfg), ctypes.byref(model.struct), batch, _p(tokens),
                            n_tokens, _p(k_cache), _p(v_cache), _p(cache_len), cache_cap,
                            None if sampler is None else ctypes.byref(sampler), _p(next_token),
                            _p(entropy), _p(logits_dbg), _p(forced_topk), w, wb, _p(dev_status),
                            _stream(stream)),
           "dg_ar_step")


def dg_debug_wait_probe(limit_cycles, arrive, dev_status, stream=None):
    """Run the bounded device wait alone (see dg.h); expiry records DG_ERR_TIMEOUT."""
    _check(lib().dg_debug_wait_probe(int(limit_cycles), 1 if arrive else 0, _p(dev_status),
                                     _stream(stream)), "dg_debug_wait_probe")


def exported_symbols() -> Sequence[str]:
    return list(_SIGS)
