"""The benchmark's multi-rank host logic on CPU: world-size-2 gloo process groups.

Every workload is independent per canvas, so several GPUs run replicas with no collective on the
data path.  What crosses ranks is only the timing: a barrier around the timed region, the max of
the per-rank device times, and the whole-job rate (all ranks' units / the slowest rank's time).
These tests run that logic in two gloo ranks, and run the benchmark's reference arm under
torchrun with two ranks (rank 0 alone prints its line; rank 1 exits 0 without work)."""
import json
import os
import socket
import subprocess
import time
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, ms_by_rank, units, out):
    import torch.distributed as dist
    from datetime import timedelta
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        import bench
        bench.barrier(world)
        m = bench.max_over_ranks(ms_by_rank[rank], world)
        rate, ms = bench.replica_rate(units, ms_by_rank[rank], world)
        out.put((rank, m, rate, ms))
    finally:
        dist.destroy_process_group()


def test_replica_rate_is_all_units_over_slowest_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    world, port = 2, _free_port()
    ms_by_rank = [12.5, 20.0]          # rank 1 is the slow one
    units = 40                         # steps each rank ran
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, ms_by_rank, units, q))
             for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, m, rate, ms in res:
        assert m == 20.0 and ms == 20.0
        assert rate == pytest.approx(world * units / 0.020)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.0, 1) == 3.0
    rate, ms = bench.replica_rate(10, 5.0, 1)
    assert ms == 5.0 and rate == pytest.approx(2000.0)


def test_reference_arm_under_torchrun_two_ranks(tmp_path):
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
           "--gpus", "2", "--steps", "2", "--warmup", "3"]
    env = dict(os.environ, OMP_NUM_THREADS="1")
    t0 = time.perf_counter()
    r = subprocess.run(cmd, cwd=str(tmp_path), env=env, capture_output=True, text=True,
                       timeout=300)
    wall = time.perf_counter() - t0
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1                   # rank 0 only
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["steps"] == 2
    assert d["value"] > 0 and d["e2e"]["h2d_bytes_per_step"] == 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    # whole oracle steps, timed as they ran: the timed steps fit inside the run's wall clock, and
    # the line carries the same config object as the CUDA arm's
    import bench
    import synth
    assert d["ms_per_step"] * d["steps"] / 1e3 < wall
    assert "whole oracle canvas step" in d["cpu_baseline"]["sample"]
    assert d["config"] == bench.headline_config(synth.get_config("tiny"), 2)


def test_step_byte_accounting_by_weight_format():
    """The step roofline's bytes: the LM head is V d bytes x 2 in bf16 and V d x 9/16 in NVFP4
    (half a byte per code plus one E4M3 scale per 16); experts count only those touched, shared
    experts included through the routing counts."""
    import bench
    import synth
    lay = synth.get_config("layer")
    q4 = synth.get_config("layer_nvfp4")
    a, b = bench.step_bytes(lay, 28.0), bench.step_bytes(q4, 28.0)
    V, d = lay.vocab, lay.d_model
    assert a["lm_head"] == V * d * 2 and b["lm_head"] == V * d * 9 / 16
    assert a["experts"] == b["experts"] == 28.0 * 3 * lay.d_ff * d * 2
    assert a["total"] - b["total"] == (V * d * 2 - V * d * 9 / 16) + lay.canvas * d * (2 - 9 / 16)
    f = bench.step_flops(lay, 256.0)
    assert f["lm_head"] == 2 * 256 * d * V


def test_traffic_records_match_their_kernel_sources():
    """Every DRAM-traffic record under profiles/ names the kernel source it was captured from;
    the benchmark reports it only while that source is unchanged, and drops it otherwise."""
    import hashlib
    import bench
    rec = json.load(open(os.path.join(ROOT, "profiles", "ncu_traffic.json")))
    assert rec
    for kernel, by_wl in rec.items():
        for wl, r in by_wl.items():
            assert r["bytes_per_launch"] >= r["algorithmic_bytes_per_launch"] > 0
            assert "--clock-control none" in r["command"]
            src = os.path.join(ROOT, "block_discrete_diffusion_dg_b200", "csrc", r["source_file"])
            sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
            got = bench.ncu_traffic(kernel, wl)
            if sha == r["source_sha16"]:
                assert got and got["bytes"] == r["bytes_per_launch"]
            else:
                assert got is None
    assert bench.ncu_traffic("no_such_kernel", "layer") is None


def test_step_roofline_bound_and_fractions():
    """The step roofline is max(bytes / HBM peak, FLOPs / tensor peak) against the measured step
    time, reported as a fraction of the measured peaks and, beside it, of the nominal ones."""
    import bench
    peaks = {"hbm_gbs": 6000.0, "bf16_tflops_sustained": 1500.0}
    # 3 GB at 6 TB/s = 500 us; 300 GFLOP at 1.5 PF/s = 200 us: HBM-bound, 500 us of 1000 us
    r = bench.step_roofline({"total": 3e9}, {"total": 3e11}, 1.0, peaks, "measured")
    assert r["bound"] == "hbm" and r["roofline_us"] == pytest.approx(500.0)
    assert r["frac"] == pytest.approx(0.5)
    assert r["frac_nominal"] == pytest.approx(3e9 / (bench.NOMINAL["hbm_gbs"] * 1e9) / 1e-3,
                                              rel=1e-3)
    # 1.2 PFLOP-s of work: tensor-bound (800 us) over a 1 GB stream (167 us)
    r = bench.step_roofline({"total": 1e9}, {"total": 1.2e12}, 1.0, peaks, "measured")
    assert r["bound"] == "tensor" and r["roofline_us"] == pytest.approx(800.0)
    assert r["frac"] == pytest.approx(0.8)
