#!/usr/bin/env python
"""Benchmark of one denoising step of the canvas-step library.

Workload (default): one bf16 decoder layer, d_model 2048, 16 q / 8 kv heads of 128, 128 experts
top-8 with expert FFN 768, vocabulary 262144, canvas 256, prompt K/V 4096 tokens ~N(0,1),
weights N(0, 0.02), seed 1, EB gamma 1.0.  Timed steps alternate between the all-MASK canvas
(step 0) and a canvas with a random half already committed, each restored before its step.

A step streams ~2.3 GB of weights (inputs larger than L2, so no flush is needed).

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl dg|reference]
Multi-GPU (torchrun): replicas — every rank runs the same single-GPU step on its own GPU; there
is no collective on the data path; the timed region is bracketed by barriers and the slowest
rank's time is reported.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

METRIC = "canvas denoise steps/s and output tok/s at batch 1; % of step roofline"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# nominal B200 figures (the ~8 TB/s HBM3e of the DGX part and the dense bf16 tensor peak), for a
# second roofline fraction beside the one against the measured peaks
NOMINAL = {"hbm_gbs": 8000.0, "bf16_tflops": 2250.0}
# the other workloads measured in the same process as the headline one (single GPU only)
EXTRA_WORKLOADS = ("longctx", "batch32", "layer_nvfp4", "stack30")


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


# ------------------------------------------------------------------------------ accounting

def step_bytes(cfg, experts_touched: float) -> dict:
    """Algorithmic HBM bytes of one step: every weight byte the step must read once (for the
    experts: the experts the step routes tokens to, summed over layers), the prompt K/V, and the
    canvas rows (activations are small and are not counted)."""
    L = cfg.n_layers
    wb = 1 if cfg.w == "e4m3" else (4 if cfg.w == "f32" else 2)
    ab = 4 if cfg.act == "f32" else 2
    d, hd = cfg.d_model, cfg.head_dim
    qkv = L * cfg.qkv_rows * d * wb
    wo = L * d * cfg.n_q_heads * hd * wb
    router = L * cfg.n_experts * d * (4 if cfg.w == "f32" else 2)
    expert = (2 * cfg.d_ff * d + d * cfg.d_ff) * wb
    # the tied embedding / LM head: NVFP4 is half a byte per element plus one E4M3 scale per 16
    eb = 9.0 / 16.0 if getattr(cfg, "emb", "") == "nvfp4" else ab
    lm = cfg.vocab * d * eb
    kv = L * cfg.batch * cfg.prompt_len * cfg.n_kv_heads * hd * 2 * ab
    emb_rows = cfg.batch * cfg.canvas * d * eb
    return {"qkv": qkv, "o": wo, "router": router, "experts": experts_touched * expert,
            "expert_gate_up": experts_touched * 2 * cfg.d_ff * d * wb,
            "expert_down": experts_touched * d * cfg.d_ff * wb, "lm_head": lm, "kv": kv,
            "emb_rows": emb_rows,
            "total": qkv + wo + router + experts_touched * expert + lm + kv + emb_rows}


def step_flops(cfg, masked_rows: float) -> dict:
    T = cfg.batch * cfg.canvas
    L = cfg.n_layers
    d, hd = cfg.d_model, cfg.head_dim
    qkv = L * 2 * T * d * cfg.qkv_rows
    o = L * 2 * T * cfg.n_q_heads * hd * d
    attn = L * 4 * cfg.batch * cfg.n_q_heads * cfg.canvas * (cfg.prompt_len + cfg.canvas) * hd
    router = L * 2 * T * d * cfg.n_experts
    moe = L * 2 * T * cfg.top_k * (2 * cfg.d_ff * d + d * cfg.d_ff)
    lm = 2 * masked_rows * d * cfg.vocab
    return {"lm_head": float(lm), "attention": float(attn), "experts": float(moe),
            "total": float(qkv + o + attn + router + moe + lm)}


STATES = {"layer": ("all_mask", "half"), "longctx": ("half",), "batch32": ("all_mask",),
          "tiny": ("all_mask",), "layer_nvfp4": ("all_mask", "half")}


# ------------------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi samples during the timed region (clocks, power, throttle reasons)."""

    FIELDS = ("uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str | None):
        self.uuid = uuid
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for ln in self.lines:
            p = [x.strip() for x in ln.split(",")]
            if len(p) < 9:
                continue
            if self.uuid and self.uuid not in p[0]:
                continue
            rows.append(p)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        pw = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        return {"sm_mhz": float(np.median(sm)) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows), "power_w_max": max(pw) if pw else None}


# ------------------------------------------------------------------------------ oracle sample

def oracle_step_time(cfg, om, state_np, kc, vc, cache_len) -> float:
    """Host seconds of one step of the oracle as it stands (``canvas_step``, fp64 numpy).

    With one canvas (every headline workload) this is the whole step, timed as it runs.  With a
    batch of canvases only the first runs (the others are marked done, so the oracle skips them)
    and the time is multiplied by the batch: the canvases are independent and cost the same.
    """
    from oracle import dg_oracle as O
    st = {k: np.array(v, copy=True) for k, v in state_np.items()}
    st["done"][1:] = 1
    t0 = time.perf_counter()
    O.canvas_step(cfg, om, st, kc, vc, cache_len, cfg.gamma, cfg.max_steps)
    return (time.perf_counter() - t0) * cfg.batch


def oracle_sample_desc(cfg, steps: int) -> str:
    one = (f"{steps} whole oracle canvas step(s), the all-MASK and half-committed canvas states "
           f"alternating, timed as they ran")
    if cfg.batch > 1:
        one += f"; one canvas of the {cfg.batch} runs and its time is multiplied by {cfg.batch}"
    return one


def headline_config(cfg, world: int) -> dict:
    """The ``config`` object of a canvas-step line; both arms print the same one."""
    return {"workload": workload_desc(cfg), "batch": cfg.batch, "canvas": cfg.canvas,
            "prompt_kv": cfg.prompt_len, "parallelism": f"replicas x{world}",
            "l2": "inputs larger than L2 (>2 GB of weights per step); no flush"}


def cpu_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        n = [i.get("num_threads", 0) for i in info if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def host_model(cfg, model):
    import synth
    from oracle import dg_oracle as O
    arr = {"emb": synth.to_numpy(model["emb"]),
           "layers": [{k: synth.to_numpy(v) for k, v in l.items()} for l in model["layers"]]}
    if "emb_scale" in model:
        arr["emb_scale"] = synth.to_numpy(model["emb_scale"])
        arr["emb_scale_global"] = float(model["emb_scale_global"])
    return O.OracleModel(cfg, arr)


# ------------------------------------------------------------------------------ main

def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and args.impl == "dg":
        import torch.distributed as dist
        from datetime import timedelta
        backend = "nccl" if torch.cuda.is_available() and args.impl == "dg" else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world: int) -> None:
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """Max of a per-rank float over all ranks (a device tensor under NCCL, a host one under gloo)."""
    if world <= 1:
        return x
    import torch.distributed as dist
    dev = torch.device("cuda", torch.cuda.current_device()) if dist.get_backend() == "nccl" \
        else torch.device("cpu")
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_rate(units_per_rank: float, ms_local: float, world: int) -> tuple:
    """Whole-job rate of `world` replicas that each processed `units_per_rank` units: all ranks'
    units / the slowest rank's device time.  Returns (units per second, max ms)."""
    ms = max_over_ranks(ms_local, world)
    return world * units_per_rank / (ms / 1e3), ms


def run_reference(args, world, rank):
    """The oracle as the reference arm: timed on the host cores, rank 0 only."""
    import synth
    if rank != 0:
        return
    cfg = synth.get_config(args.workload)
    model = synth.make_model(cfg, "cpu")
    kv = synth.make_prompt_kv(cfg, "cpu")
    om = host_model(cfg, model)
    from oracle import dg_oracle as O
    kc = O.decode_act(synth.to_numpy(kv["k"]), cfg.act)
    vc = O.decode_act(synth.to_numpy(kv["v"]), cfg.act)
    cl = synth.to_numpy(kv["cache_len"])
    states = [{k: synth.to_numpy(v) for k, v in synth.make_canvas_state(cfg, s).items()}
              for s in ("all_mask", "half")]
    for i in range(args.warmup):
        oracle_step_time(cfg, om, states[i % 2], kc, vc, cl)
    times = [oracle_step_time(cfg, om, states[i % 2], kc, vc, cl) for i in range(args.steps)]
    t = float(np.sum(times))
    v = args.steps / t
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "steps/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded random-init weights, N(0,1) prompt K/V)",
            "config": headline_config(cfg, world),
            "cpu_baseline": {"kind": "oracle", "value": v, "unit": "steps/s", "cores": cpu_threads(),
                             "sample": oracle_sample_desc(cfg, args.steps)},
            "e2e": {"value": v, "unit": "steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def workload_desc(cfg) -> str:
    states = " / ".join(STATES.get(cfg.name, ("all_mask",)))
    lm = ", embedding / LM head NVFP4" if getattr(cfg, "emb", "") == "nvfp4" else ""
    return (f"{cfg.name}: {cfg.n_layers} decoder layer(s) {cfg.act}/{cfg.w}{lm}, d_model {cfg.d_model}, "
            f"{cfg.n_q_heads}q/{cfg.n_kv_heads}kv x {cfg.head_dim}, {cfg.n_experts} experts top-"
            f"{cfg.top_k} ff {cfg.d_ff}, vocab {cfg.vocab}, canvas {cfg.canvas}, prompt KV "
            f"{cfg.prompt_len}, gamma {cfg.gamma}, batch {cfg.batch}; canvas states: {states}")


def run_extras(args, world, rank, local) -> dict:
    """The other workloads, one after another in this process (each freed before the next):
    steps/s, ms per step, the step roofline and the dominant kernel's roofline, clocks."""
    out = {}
    sub = argparse.Namespace(**vars(args))
    sub.steps = args.extra_steps
    for name in EXTRA_WORKLOADS:
        torch.cuda.empty_cache()
        try:
            if name == "stack30":
                sub.workload = name
                r = run_generate(sub, world, rank, full=False)
            else:
                r = run_dg(sub, world, rank, local, workload=name, full=False)
            out[name] = r
        except Exception as e:  # a workload that cannot run here is reported, not fatal
            out[name] = {"error": f"{type(e).__name__}: {e}"}
        torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return out


def run_generate(args, world, rank, full=True):
    """Block-autoregressive generation of the 30-layer workload: the prompt (2048 ids) is
    prefilled through the append in 256-token chunks (not timed), then n_canvases canvases are
    denoised from all-MASK until done and appended.  Timed both ways: dg_generate (the step loop
    on the device, one graph per canvas; the reported value) and the host loop that reads each
    step's done flag (in `loops`).  Timed: the denoising steps and the appends (the pages' TPS
    excludes prefill)."""
    import synth
    from block_discrete_diffusion_dg_b200 import binding as B
    B.lib()
    cfg = synth.get_config(args.workload)
    dev = torch.device("cuda", torch.cuda.current_device())
    model = synth.make_model(cfg, dev)
    kv = synth.make_prompt_kv(cfg, dev)
    cap = kv["k"].shape[3]
    dgcfg, dgm = B.make_config(cfg), B.Model(model)
    ws = B.alloc_workspace(dgcfg, cfg.batch, cfg.canvas, cap)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    ids = kv["prompt_ids"]
    for c0 in range(0, cfg.prompt_len, 256):
        B.dg_kv_append(dgcfg, dgm, cfg.batch, ids[:, c0:c0 + 256].contiguous(), 256, kv["k"],
                       kv["v"], kv["cache_len"], cap, ws, status)
    k0, v0, l0 = kv["k"].clone(), kv["v"].clone(), kv["cache_len"].clone()
    stream = torch.cuda.current_stream()

    init = {k: v.to(dev) for k, v in synth.make_canvas_state(cfg, "all_mask").items()}
    st = {k: v.clone() for k, v in init.items()}
    # the experts a representative step routes tokens to (the first step of the first canvas,
    # all MASK, cache = the prefilled prompt): the byte count of the step roofline
    load = torch.zeros((cfg.n_layers, cfg.n_experts + cfg.n_shared), dtype=torch.int32, device=dev)
    B.dg_canvas_step(dgcfg, dgm, cfg.batch, st["tokens"], st["masked"], st["n_masked"], st["done"],
                     st["step"], cfg.max_steps, cfg.gamma, kv["k"], kv["v"], kv["cache_len"], cap,
                     None, None, None, ws, status, stream, expert_load=load)
    touched = float((load > 0).sum().item())
    for k in st:
        st[k].copy_(init[k])

    def generate_host():
        # the host reads each step's done flag
        kv["k"].copy_(k0); kv["v"].copy_(v0); kv["cache_len"].copy_(l0)
        steps = 0
        for _ in range(cfg.n_canvases):
            for k in st:
                st[k].copy_(init[k])
            while True:
                B.dg_canvas_step(dgcfg, dgm, cfg.batch, st["tokens"], st["masked"], st["n_masked"],
                                 st["done"], st["step"], cfg.max_steps, cfg.gamma, kv["k"], kv["v"],
                                 kv["cache_len"], cap, None, None, None, ws, status, stream)
                steps += 1
                if int(st["done"].item()):
                    break
            B.dg_kv_append(dgcfg, dgm, cfg.batch, st["tokens"], cfg.canvas, kv["k"], kv["v"],
                           kv["cache_len"], cap, ws, status, stream)
        return steps

    def generate_device():
        # dg_generate: the step loop runs on the device (one graph per canvas, no host read
        # between steps), then the append; the step counters are read once at the end
        kv["k"].copy_(k0); kv["v"].copy_(v0); kv["cache_len"].copy_(l0)
        counts = []
        for _ in range(cfg.n_canvases):
            for k in st:
                st[k].copy_(init[k])
            B.dg_generate(dgcfg, dgm, cfg.batch, st["tokens"], st["masked"], st["n_masked"],
                          st["done"], st["step"], cfg.max_steps, cfg.gamma, kv["k"], kv["v"],
                          kv["cache_len"], cap, 1, ws, status, stream)
            counts.append(st["step"].max())
        return int(torch.stack(counts).sum().item())

    modes = [("device", generate_device), ("host", generate_host)] if full else \
        [("device", generate_device)]
    try:
        generate_device()
        torch.cuda.synchronize()
    except Exception as e:  # no conditional graph nodes here: time the host loop only
        print(f"device loop unavailable ({e}); timing the host loop", file=sys.stderr)
        modes = [("host", generate_host)]
    for _ in range(args.warmup):
        for _m, fn in modes:
            fn()
    torch.cuda.synchronize()
    uuid = None
    try:
        uuid = str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    clocks = ClockSampler(uuid)
    barrier(world)
    clocks.start()
    time.sleep(0.3)
    timed = {}
    for name, fn in modes:
        n0 = B.dg_launch_count()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        steps = fn()
        e1.record(stream)
        torch.cuda.synchronize()
        timed[name] = (steps, e0.elapsed_time(e1), B.dg_launch_count() - n0)
    barrier(world)
    clk = clocks.stop()
    steps, ms_total, launches = timed[modes[0][0]]
    if B.dg_read_status(status) != B.DG_OK:
        raise RuntimeError("device status set during generation")
    rate, ms = replica_rate(steps, ms_total, world)
    loops = {name: {"steps": v[0], "ms_per_step": round(v[1] / v[0], 4)} for name, v in timed.items()}
    toks = cfg.n_canvases * cfg.canvas * cfg.batch
    peaks, peak_src = load_peaks()
    step_roof = step_roofline(step_bytes(cfg, touched), step_flops(cfg, cfg.batch * cfg.canvas),
                              ms / steps, peaks, peak_src)
    step_roof["experts_touched"] = touched
    step_roof["note"] = ("bytes and FLOPs of the first all-MASK step over the prefilled prompt "
                         "(its routed experts, all 30 layers, the LM head over 256 rows) against "
                         "the loop's mean time per step, which also carries the appends")
    line = {"metric": METRIC, "value": round(rate, 3), "unit": "steps/s",
            "n_gpus": world, "steps": steps, "warmup": args.warmup,
            "ms_per_step": round(ms / steps, 4), "clocks": clk,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded random-init weights, random prompt ids)",
            "config": {"workload": workload_desc(cfg) + f"; generate {cfg.n_canvases} canvases, "
                       f"at most {cfg.max_steps} steps each, prefill not timed",
                       "batch": cfg.batch, "mode": "generate",
                       "loop": modes[0][0] + (" (dg_generate: device-resident step loop)"
                                              if modes[0][0] == "device" else
                                              " (host reads done after each step)")},
            "loops": loops,
            "output_tok_s": round(world * toks / (ms / 1e3), 2),
            "gpu_launches": int(launches) if modes[0][0] == "host" else
            (int(timed["host"][2] + steps) if "host" in timed else None),
            "gpu_launches_note": ("counted launches of the host loop" if modes[0][0] == "host" else
                                  "the device loop replays, per step, the kernels the host loop "
                                  "launches for the same steps (counted there), plus one "
                                  "condition kernel per step"),
            "step_roofline": step_roof,
            "impl": "dg", "peaks": f"{peak_src}: {peaks['hbm_gbs']} GB/s"}
    if not full:   # launches are counted on the host loop, which this short form skips
        line.pop("gpu_launches_note", None)
    return line


def ncu_traffic(kernel: str, workload: str):
    """DRAM bytes (read + write) per launch of `kernel` on `workload` from one ncu capture, as
    recorded in profiles/ncu_traffic.json together with the SHA-256 (first 16 hex digits) of the
    kernel's source file at the time of the capture.  None when there is no record or the source
    has changed since (the counters then describe another build)."""
    import hashlib
    try:
        rec = json.load(open(os.path.join(ROOT, "profiles", "ncu_traffic.json")))
    except (OSError, ValueError):
        return None
    r = rec.get(kernel, {}).get(workload)
    if not r:
        return None
    src = os.path.join(ROOT, "block_discrete_diffusion_dg_b200", "csrc", r["source_file"])
    try:
        sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    except OSError:
        return None
    if sha != r["source_sha16"]:
        return None
    return {"bytes": int(r["bytes_per_launch"]), "source": "profiles/ncu_traffic.json",
            "captured": r.get("command", "")}


def run_dg(args, world, rank, local, workload=None, full=True):
    """One workload's step, replayed from CUDA graphs; returns the JSON line (a dict).  full: also
    the end-to-end leg through the C ABI with host buffers and the CPU baseline."""
    import synth
    from block_discrete_diffusion_dg_b200 import binding as B
    B.lib()
    cfg = synth.get_config(workload or args.workload)
    dev = torch.device("cuda", torch.cuda.current_device())
    model = synth.make_model(cfg, dev)
    kv = synth.make_prompt_kv(cfg, dev)
    cap = kv["k"].shape[3]
    dgcfg, dgm = B.make_config(cfg), B.Model(model)
    ws = B.alloc_workspace(dgcfg, cfg.batch, cfg.canvas, cap)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    states = STATES.get(cfg.name, ("all_mask",))
    init = [{k: v.to(dev) for k, v in synth.make_canvas_state(cfg, s_).items()} for s_ in states]
    ns = len(init)
    st = {k: v.clone() for k, v in init[0].items()}
    load = torch.zeros((cfg.n_layers, cfg.n_experts + cfg.n_shared), dtype=torch.int32,
                       device=dev)

    def one_step(i, stream=None, expert_load=None):
        src = init[i % ns]
        for k in st:
            st[k].copy_(src[k], non_blocking=True)
        B.dg_canvas_step(dgcfg, dgm, cfg.batch, st["tokens"], st["masked"], st["n_masked"],
                         st["done"], st["step"], cfg.max_steps, cfg.gamma, kv["k"], kv["v"],
                         kv["cache_len"], cap, None, None, None, ws, status, stream,
                         expert_load=expert_load)

    for i in range(args.warmup):
        one_step(i)
    torch.cuda.synchronize()
    rc = B.dg_read_status(status)
    if rc != B.DG_OK:
        raise RuntimeError(f"device status {B.STATUS_NAMES.get(rc, rc)} during warm-up")

    # per state: tokens committed by one step, experts the step routes to, kernels it launches
    committed, touched, masked_rows, per_step_launches = [], [], [], 0
    for i in range(ns):
        n0 = B.dg_launch_count()
        one_step(i, expert_load=load)
        torch.cuda.synchronize()
        per_step_launches = B.dg_launch_count() - n0
        committed.append(int(init[i]["n_masked"].sum() - st["n_masked"].sum()))
        touched.append(float((load > 0).sum().item()))      # (layer, expert) pairs with tokens
        masked_rows.append(float(init[i]["n_masked"].sum().item()))

    # ---- timed region: K steps replayed from CUDA graphs (one graph per canvas state) ----
    graphs = []
    if not args.no_graph:
        try:
            for i in range(ns):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g):
                    one_step(i)
                graphs.append(g)
            for g in graphs:
                g.replay()
            torch.cuda.synchronize()
        except Exception as e:  # capture not possible: time the direct launches instead
            print(f"graph capture failed ({e}); timing direct launches", file=sys.stderr)
            graphs = []
    stream = torch.cuda.current_stream()
    uuid = None
    try:
        uuid = str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    clocks = ClockSampler(uuid)
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for i in range(args.steps):
        if graphs:
            graphs[i % ns].replay()
        else:
            one_step(i)
    ev1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    steps_s, ms = replica_rate(args.steps, ev0.elapsed_time(ev1), world)
    rc = B.dg_read_status(status)
    if rc != B.DG_OK:
        raise RuntimeError(f"device status {B.STATUS_NAMES.get(rc, rc)} in the timed region")
    ms_step = ms / args.steps
    launches = per_step_launches * args.steps

    # ---- profile pass: the same steps with a CUDA event before every kernel, captured into one
    # graph (external event-record nodes) and replayed, so launch gaps are not counted ----
    kp = max(4, min(args.steps, 20))
    n_rec = kp * 64 + 16
    torch.cuda.synchronize()
    B.dg_profile_begin(n_rec)
    prof_mode = "graph"
    try:
        gp = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gp):
            cs = torch.cuda.current_stream()
            for i in range(kp):
                one_step(i)
                B.dg_profile_mark(cs)
        gp.replay()
        torch.cuda.synchronize()
        prof = B.dg_profile_end(n_rec)
        del gp
    except Exception as e:
        print(f"profile graph failed ({e}); profiling direct launches", file=sys.stderr)
        prof_mode = "direct"
        B.dg_profile_begin(n_rec)
        for i in range(kp):
            one_step(i, stream)
            B.dg_profile_mark(stream)
        B.dg_profile_mark(stream)
        prof = B.dg_profile_end(n_rec)
    per = {}
    for name, t in prof:
        if name == "(mark)":
            continue
        # the LM head is one step run by one of two kernels (CTA pairs beyond 128 rows, single
        # CTAs below; the other returns at once): count the pair as one launch of "lm_head_tc"
        pair = name == "lm_head_tc2"
        a = per.setdefault("lm_head_tc" if pair else name, [0.0, 0])
        a[0] += t
        a[1] += 0 if pair else 1
    tot = sum(v[0] for v in per.values())
    breakdown = {k: {"ms_total": round(v[0], 4), "launches": v[1],
                     "ms_per_launch": round(v[0] / v[1], 5), "share": round(v[0] / tot, 4)}
                 for k, v in sorted(per.items(), key=lambda kv_: -kv_[1][0])}
    peaks, peak_src = load_peaks()
    t_avg = float(np.mean(touched))
    m_avg = float(np.mean(masked_rows))
    sb = step_bytes(cfg, t_avg)
    sf = step_flops(cfg, m_avg)
    dom = next(iter(breakdown))
    ab = 4 if cfg.act == "f32" else 2
    lm_bytes = sb["lm_head"] + m_avg * cfg.d_model * ab
    dur = breakdown[dom]["ms_per_launch"] / 1e3
    roof = None
    if dom == "attn_tc":  # long contexts: the attention is a tensor-bound contraction
        ach = sf["attention"] / cfg.n_layers / dur / 1e12
        tr = ncu_traffic(dom, cfg.name)
        roof = {"kernel": dom, "bound": "tensor", "achieved": round(ach, 1),
                "peak": peaks["bf16_tflops_sustained"], "unit": "TFLOP/s",
                "frac": round(ach / peaks["bf16_tflops_sustained"], 4),
                "traffic": tr["bytes"] if tr else None,
                "algorithmic_flops_per_launch": sf["attention"] / cfg.n_layers,
                "peak_source": f"{peak_src} (cuBLAS bf16, sustained, of measured)",
                "traffic_source": tr["source"] if tr else
                "none: no ncu capture of this kernel source on this workload"}
    elif dom in ("lm_head_tc", "lm_head_q4") and \
            sf["lm_head"] / (peaks["bf16_tflops_sustained"] * 1e12) > \
            lm_bytes / (peaks["hbm_gbs"] * 1e9):
        ach = sf["lm_head"] / dur / 1e12     # the batched LM head is a tensor-bound contraction
        roof = {"kernel": dom, "bound": "tensor", "achieved": round(ach, 1),
                "peak": peaks["bf16_tflops_sustained"], "unit": "TFLOP/s",
                "frac": round(ach / peaks["bf16_tflops_sustained"], 4),
                "traffic": None, "algorithmic_flops_per_launch": sf["lm_head"],
                "peak_source": f"{peak_src} (cuBLAS bf16, sustained, of measured)"}
    else:
        dom_bytes = {"lm_head_tc": lm_bytes, "lm_head_q4": lm_bytes,
                     "moe_gate_up_tc": sb["expert_gate_up"],
                     "moe_down_tc": sb["expert_down"]}.get(dom)
        if dom_bytes:
            ach = dom_bytes / dur / 1e9
            peak = peaks["hbm_gbs"]
            tr = ncu_traffic(dom, cfg.name)
            roof = {"kernel": dom, "bound": "hbm", "achieved": round(ach, 1), "peak": peak,
                    "unit": "GB/s", "frac": round(ach / peak, 4),
                    "traffic": tr["bytes"] if tr else None,
                    "algorithmic_bytes_per_launch": int(dom_bytes),
                    "peak_source": f"{peak_src} (burst copy, of measured)",
                    "traffic_source": tr["source"] if tr else
                    "none: no ncu capture of this kernel source on this workload"}
    if roof:
        roof["timing"] = f"CUDA events before each launch, {kp}-step profile pass ({prof_mode})"
    step_roof = step_roofline(sb, sf, ms_step, peaks, peak_src)
    step_roof["experts_touched_per_state"] = touched
    if not full:
        return {"metric": METRIC, "value": round(steps_s, 3), "unit": "steps/s",
                "ms_per_step": round(ms_step, 4), "output_tok_s": round(steps_s * float(np.mean(committed)), 2),
                "config": {"workload": workload_desc(cfg), "batch": cfg.batch,
                           "cuda_graph": bool(graphs), "steps": args.steps},
                "step_roofline": step_roof, "roofline": roof, "clocks": clk,
                "gpu_launches": int(launches), "launches_per_step": int(per_step_launches),
                "kernels_top": dict(list(breakdown.items())[:8])}

    # ---- end to end through the C ABI with host buffers ----
    pin = [{k: v.cpu().pin_memory() for k, v in s_.items()} for s_ in init]
    out_h = {k: torch.empty_like(pin[0][k]).pin_memory() for k in ("tokens", "masked", "done")}
    h2d = sum(t.numel() * t.element_size() for t in pin[0].values())
    d2h = sum(t.numel() * t.element_size() for t in out_h.values())
    e_steps = max(4, args.steps // 2)
    barrier(world)
    torch.cuda.synchronize()
    x0, x1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    x0.record(stream)
    for i in range(e_steps):
        src = pin[i % ns]
        for k in st:
            st[k].copy_(src[k], non_blocking=True)
        B.dg_canvas_step(dgcfg, dgm, cfg.batch, st["tokens"], st["masked"], st["n_masked"],
                         st["done"], st["step"], cfg.max_steps, cfg.gamma, kv["k"], kv["v"],
                         kv["cache_len"], cap, None, None, None, ws, status, stream)
        for k in out_h:
            out_h[k].copy_(st[k], non_blocking=True)
        stream.synchronize()       # the caller reads the committed tokens and the done flag
    x1.record(stream)
    torch.cuda.synchronize()
    e_rate, _ = replica_rate(e_steps, x0.elapsed_time(x1), world)
    e2e = {"value": round(e_rate, 3), "unit": "steps/s", "h2d_bytes_per_step": h2d,
           "d2h_bytes_per_step": d2h,
           "note": "direct calls (no graph), host state copied in from pinned memory and the "
                   "result read back every step; CUDA events around the loop"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        om = host_model(cfg, model)
        from oracle import dg_oracle as O
        kc = O.decode_act(synth.to_numpy(kv["k"]), cfg.act)
        vc = O.decode_act(synth.to_numpy(kv["v"]), cfg.act)
        cl = synth.to_numpy(kv["cache_len"])
        ts = [oracle_step_time(cfg, om, {k: synth.to_numpy(v) for k, v in init[i].items()},
                               kc, vc, cl) for i in range(ns)]
        cpu = {"value": ns / float(np.sum(ts)), "unit": "steps/s", "cores": cpu_threads(),
               "kind": "oracle", "sample": oracle_sample_desc(cfg, ns)}

    tok_s = steps_s * float(np.mean(committed))     # tokens committed over all canvases
    line = {"metric": METRIC, "value": round(steps_s, 3), "unit": "steps/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded random-init weights, N(0,1) prompt K/V)",
            "config": headline_config(cfg, world), "cuda_graph": bool(graphs),
            "output_tok_s": round(tok_s, 2), "tokens_committed_per_step": committed,
            "step_roofline": step_roof, "roofline": roof, "kernels": breakdown,
            "gpu_launches": int(launches), "launches_per_step": int(per_step_launches),
            "e2e": e2e, "cpu_baseline": cpu, "clocks": clk, "impl": "dg"}
    return line


def step_roofline(sb: dict, sf: dict, ms_step: float, peaks: dict, peak_src: str) -> dict:
    """max(bytes / HBM peak, FLOPs / tensor peak) for one step against its measured time, with
    the measured peaks (the fraction the target is judged on) and, beside it, the nominal ones."""
    t_bytes = sb["total"] / (peaks["hbm_gbs"] * 1e9)
    t_flops = sf["total"] / (peaks["bf16_tflops_sustained"] * 1e12)
    n_bytes = sb["total"] / (NOMINAL["hbm_gbs"] * 1e9)
    n_flops = sf["total"] / (NOMINAL["bf16_tflops"] * 1e12)
    return {"bound": "hbm" if t_bytes >= t_flops else "tensor",
            "roofline_us": round(1e6 * max(t_bytes, t_flops), 1),
            "measured_us": round(1e3 * ms_step, 1),
            "frac": round(1e6 * max(t_bytes, t_flops) / (1e3 * ms_step), 4),
            "frac_nominal": round(1e6 * max(n_bytes, n_flops) / (1e3 * ms_step), 4),
            "algorithmic_bytes": int(sb["total"]),
            "algorithmic_flops": sf["total"],
            "peaks": f"{peak_src}: {peaks['hbm_gbs']} GB/s, "
                     f"{peaks['bf16_tflops_sustained']} TF/s sustained (frac, of measured); "
                     f"nominal {NOMINAL['hbm_gbs']} GB/s, {NOMINAL['bf16_tflops']} TF/s "
                     f"(frac_nominal)"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="dg", choices=["dg", "reference"])
    ap.add_argument("--workload", default="layer")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="time direct launches")
    ap.add_argument("--no-extra", action="store_true",
                    help="measure the headline workload only (no 'workloads' object)")
    ap.add_argument("--extra-steps", type=int, default=20,
                    help="timed steps of each extra workload")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    world, rank, local = dist_setup(args)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            if args.workload == "stack30":
                line = run_generate(args, world, rank)
            else:
                line = run_dg(args, world, rank, local)
            if world == 1 and args.workload == "layer" and not args.no_extra:
                line["workloads"] = run_extras(args, world, rank, local)
            if rank == 0:
                print(json.dumps(line), flush=True)
    finally:
        if world > 1 and args.impl == "dg":
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
