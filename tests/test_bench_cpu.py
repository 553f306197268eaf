"""bench.py's host side without a GPU: the reference arm (the CPU oracle on a bounded sample
of the workload) prints one JSON line with the contract's keys, and the step-roofline
arithmetic follows its stated formula."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def test_reference_arm_prints_one_contract_line():
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
                          "--steps", "1", "--warmup", "0"], capture_output=True, text=True, env=env, cwd=ROOT,
                         timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "tokens/s"
    for key in ("metric", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling", "vs_baseline",
                "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
    assert d["config"]["workload"] == "tiny"


def test_step_roofline_formula():
    """T_roof = T_prelude + sum over loops of max(F_s / P, B_s / BW), with F_s and B_s as the
    docstring of bench.step_roofline and the measurement section state them."""
    import bench
    from synth import MODELS
    m = MODELS["qwen3-8b"]
    peaks = {"hbm_gbs": 1000.0, "bf16_tflops_sustained": 1000.0}
    B, P, N = 2, 100, 10
    p = m.hidden * m.n_q_heads * m.head_dim * 2 + 2 * m.hidden * m.n_kv_heads * m.head_dim + 3 * m.hidden * m.inter
    assert p == 192_937_984  # 192.9 M parameters per 8B layer
    CD = m.n_core + m.n_coda
    kvl = 2 * 2 * m.n_kv_heads * (P + N) * m.head_dim
    f_pre = 2.0 * B * N * m.n_prelude * p + 4.0 * B * N * (P + N) * m.n_q_heads * m.head_dim * m.n_prelude
    b_pre = 2.0 * p * m.n_prelude + B * m.n_prelude * kvl
    rows, R = 20, 7
    f1 = 2.0 * rows * CD * p + 2.0 * R * m.vocab * m.hidden + 4.0 * rows * (P + N) * m.n_q_heads * m.head_dim * CD
    b1 = 2.0 * p * CD + 2.0 * m.vocab * m.hidden + 2 * CD * kvl
    want = max(f_pre / 1e15, b_pre / 1e12) + max(f1 / 1e15, b1 / 1e12)
    t, F, Bt = bench.step_roofline(m, B, P, N, [rows, 0], [R, 0], peaks)
    assert t == pytest.approx(want, rel=1e-12)
    assert F == pytest.approx(f_pre + f1, rel=1e-12) and Bt == pytest.approx(b_pre + b1, rel=1e-12)


def _free_port():
    import socket
    with socket.socket() as so:
        so.bind(("127.0.0.1", 0))
        return so.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), LOCAL_RANK=str(rank),
                      WORLD_SIZE=str(world), CUDA_VISIBLE_DEVICES="", ALODLM_PG_TIMEOUT_S="60")
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    w, r, _ = bench.dist_setup(world)
    bench.barrier(w)
    # rank r "timed" 1 + r ms and processed 10 * (r + 1) units
    mx = bench.all_max(1.0 + r, w)
    sm = bench.all_sum(10.0 * (r + 1), w)
    q.put((r, w, dist.get_backend(), mx, sm))
    dist.destroy_process_group()


def test_two_rank_collectives_on_gloo():
    """The N > 1 host path of bench.py on CPU: gloo group, barrier, max-over-ranks time and
    summed units (value = units of all ranks / slowest rank's time)."""
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    for r, (rank, world, backend, mx, sm) in enumerate(got):
        assert (rank, world, backend) == (r, 2, "gloo")
        assert mx == 2.0 and sm == 30.0


def test_reference_arm_under_two_ranks():
    """torchrun with 2 ranks on CPU: rank 0 alone runs the oracle and prints the line, rank 1
    exits 0 without work."""
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="", ALODLM_PG_TIMEOUT_S="120")
    out = subprocess.run([sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
                          "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
                          os.path.join(ROOT, "bench.py"), "--gpus", "2", "--impl", "reference", "--workload",
                          "tiny", "--steps", "1", "--warmup", "0"], capture_output=True, text=True, env=env,
                         cwd=ROOT, timeout=600)
    assert out.returncode == 0, out.stderr[-3000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1 and json.loads(lines[0])["impl"] == "reference"


def test_gpu_arm_line_from_a_measurement():
    """The GPU arm's JSON line, assembled from a synthetic measurement (no GPU): whole-job
    throughput over the time, the roofline of whichever linear-layer class takes longer (the
    many-row class against the sustained bf16 peak, the few-row class against HBM), both
    classes under gemm_rooflines, traffic only for a recorded source hash, the step roofline."""
    import argparse
    import bench
    from synth import WORKLOADS
    wl = WORKLOADS["qwen3-8b-bs32"]
    args = argparse.Namespace(tau=0.6, lam=0.5, rule=0, steps=10, warmup=3, workload="qwen3-8b-bs32",
                              no_extras=True)
    peaks = {"hbm_gbs": 6000.0, "bf16_tflops_sustained": 1400.0, "bf16_tflops": 1600.0}
    classes = {
        "gemm": {"ms": 70.0, "launches": 586, "bytes": 586 * 150e6, "flops": 7.0e13},
        "gemm_tile": {"ms": 6.0, "launches": 182, "bytes": 182 * 85e6, "flops": 1.0e12},
        "attention": {"ms": 16.0, "launches": 200, "bytes": 1e9, "flops": 1e12},
    }
    r = {"ms": 1050.0, "e2e_ms": 1070.0, "commits": 1635, "classes": classes, "tensor_bound": True,
         "t_roof": 0.0655, "F": 9.0e13, "B": 1.1e11, "loops": [3] * 32, "active_rows": [2048, 0],
         "readout_rows": [2048, 0], "launches_per_step": 1500, "h2d": 8192, "d2h": 1000, "clocks": None}
    line = bench.assemble_line(args, wl, 1, r, peaks, "test", 1.0)
    assert abs(line["ms_per_step"] - 105.0) < 1e-9
    assert abs(line["value"] - 1635 * 10 / 1.05) < 1e-6
    roof = line["roofline"]
    assert roof["kernel_class"] == "gemm" and roof["bound"] == "tensor" and roof["unit"] == "TFLOP/s"
    assert abs(roof["achieved"] - 7.0e13 / 0.070 / 1e12) < 1e-6 and abs(roof["frac"] - roof["achieved"] / 1400.0) < 1e-12
    tile = line["gemm_rooflines"]["gemm_tile"]
    assert tile["bound"] == "hbm" and abs(tile["achieved"] - 182 * 85e6 / 0.006 / 1e9) < 1e-6
    recorded = bench.GEMM_TRAFFIC.get("qwen3-8b-bs32")
    if recorded and recorded["source"] == bench.gemm_source_hash():
        assert roof["traffic"] == recorded["gemm"]
    else:
        assert roof["traffic"] is None
    assert abs(line["step_roofline"]["frac"] - 65.5 / 105.0) < 1e-9
    assert line["dominant_kernel_class"] == "gemm" and line["gpu_launches"] == 15000
    assert line["e2e"]["h2d_bytes_per_step"] == 8192
    # few rows: the per-tile class dominates and is held against HBM
    classes["gemm"]["ms"] = 1.0
    line = bench.assemble_line(args, wl, 1, r, peaks, "test", 1.0)
    assert line["roofline"]["kernel_class"] == "gemm_tile" and line["roofline"]["bound"] == "hbm"
