"""Benchmark: committed tokens/s per ALoDLM denoising step on Qwen3-8B-shaped synthetic models.

One "step" is one call of alodlm_denoise_step over one batch: Prelude over the block, the
looped Core/Coda with the fused readout and commit/merge, until every sequence halts.
The prefix KV cache is built once (prefill, untimed).  Weights are seeded random bf16 and
inputs are seeded random prefix ids with an all-[MASK] block (no datasets or trained
weights exist here; they stand in for the paper's GSM8K decoding).

    python bench.py [--gpus N --steps K --warmup W] [--workload qwen3-8b-bs32] [--impl reference]

Prints one JSON line (rank 0).  Multi-GPU (torchrun): every rank runs its own replica on its
own batch (sequences are independent; no collective on the data path), value = all ranks'
committed tokens / max-over-ranks time ("scaling": "weak").
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from synth import MODELS, WORKLOADS, make_weights, make_prefix_ids, make_block_ids, make_exit_depths  # noqa: E402

METRIC = "committed tokens/s per denoise step (8B-shape bf16, bs 1/32); % of roofline"
FALLBACK_PEAKS = dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm_gbs=float(d["hbm_gbs"]), bf16_tflops=float(d["bf16_tflops"]),
                    bf16_tflops_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"]))), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------------------------
# distributed plumbing
# ------------------------------------------------------------------------------------

def dist_setup(n_gpus):
    """One process per GPU (torchrun's RANK / LOCAL_RANK / WORLD_SIZE).  The process group is
    NCCL on GPUs; without a GPU (the CPU reference arm, the multi-process host tests) gloo.
    A short timeout makes ranks that wait for a missing peer end with an error."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        timeout = datetime.timedelta(seconds=float(os.environ.get("ALODLM_PG_TIMEOUT_S", "600")))
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=timeout, device_id=torch.device("cuda", local))
        else:
            dist.init_process_group("gloo", timeout=timeout)
    elif torch.cuda.is_available():  # the reference arm (the CPU oracle) also runs without a GPU
        torch.cuda.set_device(0)
    return world, rank, local


def _coll_device():
    import torch.distributed as dist
    return "cuda" if dist.get_backend() == "nccl" else "cpu"


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def all_max(x, world):
    """Maximum over ranks (the job's time is its slowest rank's)."""
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=_coll_device())
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def all_sum(x, world):
    """Sum over ranks (the units every rank processed)."""
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=_coll_device())
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


# ------------------------------------------------------------------------------------
# clocks during the timed region
# ------------------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append(dict(sm=float(parts[1]), smax=float(parts[2]), power=float(parts[3]),
                                 hw=parts[5], hwt=parts[6], swt=parts[7], swp=parts[8]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        reasons = set()
        for r in rows:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"), ("swt", "sw_thermal_slowdown"),
                              ("swp", "sw_power_cap")):
                if r[key].lower().startswith("active"):
                    reasons.add(name)
        loaded = [r["sm"] for r in rows if r["power"] > 200.0] or [r["sm"] for r in rows]
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(r["smax"] for r in rows),
                "reasons": sorted(reasons), "samples": len(rows)}


# ------------------------------------------------------------------------------------
# algorithmic work of a step (roofline)
# ------------------------------------------------------------------------------------

def layer_params(m):
    return (m.hidden * m.n_q_heads * m.head_dim * 2 + 2 * m.hidden * m.n_kv_heads * m.head_dim
            + 3 * m.hidden * m.inter)


def step_roofline(m, B, P, N, active_rows, readout_rows, peaks):
    """T_roof = T_prelude + sum over loops of max(F_s / P_peak, Bytes_s / BW)."""
    p = layer_params(m)
    H, V = m.hidden, m.vocab
    CD = m.n_core + m.n_coda
    kv_bytes_per_layer_seq = 2 * 2 * m.n_kv_heads * (P + N) * m.head_dim
    BW = peaks["hbm_gbs"] * 1e9
    PK = peaks["bf16_tflops_sustained"] * 1e12
    rows0 = B * N
    f_pre = 2.0 * rows0 * m.n_prelude * p + 4.0 * rows0 * (P + N) * m.n_q_heads * m.head_dim * m.n_prelude
    b_pre = 2.0 * p * m.n_prelude + B * m.n_prelude * kv_bytes_per_layer_seq
    t = max(f_pre / PK, b_pre / BW)
    total_f, total_b = f_pre, b_pre
    for rows, R in zip(active_rows, readout_rows):
        if rows <= 0:
            continue
        n_seq = rows // N
        f = 2.0 * rows * CD * p + 2.0 * R * V * H + 4.0 * rows * (P + N) * m.n_q_heads * m.head_dim * CD
        by = 2.0 * p * CD + 2.0 * V * H + n_seq * CD * kv_bytes_per_layer_seq
        t += max(f / PK, by / BW)
        total_f += f
        total_b += by
    return t, total_f, total_b


# DRAM traffic per launch of each linear-layer kernel class, from an ncu capture
# (dram__bytes_read.sum + dram__bytes_write.sum over every GEMM launch of one step), keyed by
# workload and by a hash of the GEMM kernel source it was taken on: a changed kernel reports
# null until captured again.  {workload: {"source": hash, "gemm": bytes, "gemm_tile": bytes}}
GEMM_TRAFFIC = {
    # profiles/gemm_traffic_qwen3-8b-bs32.md, profiles/step_launches_qwen3-8b-bs1.md
    "qwen3-8b-bs32": {"source": "967b1f20f09d80f8", "gemm": 86.858e9 / 586, "gemm_tile": 15.243e9 / 182},
    "qwen3-8b-bs1": {"source": "967b1f20f09d80f8", "gemm_tile": 34.253e9 / 352},
}


def gemm_source_hash():
    import hashlib
    h = hashlib.sha256()
    for f in ("gemm_tc.cuh", "common.cuh"):
        with open(os.path.join(ROOT, "adaptively_looped_masked_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def gemm_traffic_per_launch(workload, kernel_class):
    rec = GEMM_TRAFFIC.get(workload)
    if rec is None or rec["source"] != gemm_source_hash():
        return None
    return rec.get(kernel_class)


# ------------------------------------------------------------------------------------
# CPU baseline: the oracle on a bounded sample
# ------------------------------------------------------------------------------------

# Loop profile of each workload's step (tau 0.6, lambda 0.5, the paper's rule) as the GPU arm
# measured it: loops run per sequence and tokens committed per step.  The reference arm runs
# without the GPU arm's results and scales its per-layer timing by this profile.
GPU_LOOP_PROFILE = {
    "qwen3-8b-bs32": dict(loops=[3, 3, 2, 3, 2, 5, 4, 3, 3, 4, 3, 6, 3, 2, 3, 2, 2, 3, 2, 7, 4, 4, 2, 5, 5, 3, 3,
                                 3, 2, 5, 3, 4], commits=1635),
}


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        nt = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        if nt:
            return int(nt[0])
    except Exception:
        pass
    return len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()


def cpu_sample(m, wl, loops_per_seq, commits_per_step, w_dev, budget_s=20.0):
    """Time the oracle (as it stands) on one sequence: one Core layer over the block against a
    prefix-sized KV context and one readout of the block; scale to a whole step of the
    workload using the given loop profile (an extrapolation: no whole step is run)."""
    from oracle import Oracle
    from synth import weights_to_numpy
    from tests.helpers import oracle_cfg
    li = m.n_prelude  # first Core layer
    wh = weights_to_numpy(w_dev, layers=[li])
    o = Oracle(oracle_cfg(m, wl.k_max), {**wh, "layers": {li: wh["layers"][li]}}, precision="fp64")
    rng = np.random.default_rng(0)
    P, N = wl.prefix, wl.block
    kvshape = (P, m.n_kv_heads, m.head_dim)
    o.kv = [{("core", 0, 1): (rng.standard_normal(kvshape) * 0.5, rng.standard_normal(kvshape) * 0.5)}]
    o.prefix_len = P
    h = rng.standard_normal((N, m.hidden)) * 0.02
    lw = o.layer_weights(li)
    t0 = time.perf_counter()
    n_layer = 0
    while True:
        o.block_layer(0, ("core", 0, 1), lw, h)
        n_layer += 1
        if time.perf_counter() - t0 > budget_s / 2 or n_layer >= 3:
            break
    t_layer = (time.perf_counter() - t0) / n_layer
    o._global("lm_head")
    t1 = time.perf_counter()
    o.readout(h)
    t_read = time.perf_counter() - t1
    CD = m.n_core + m.n_coda
    per_seq = [m.n_prelude * t_layer + L * (CD * t_layer + t_read) for L in loops_per_seq]
    t_step = float(sum(per_seq))
    return dict(value=commits_per_step / t_step, unit="tokens/s", cores=blas_threads(), kind="oracle",
                extrapolated=True,
                sample=(f"oracle float64, one sequence: one Core layer over the {N}-row block against a "
                        f"{P}-position KV context ({t_layer:.2f} s) and one {m.vocab}-vocab readout of the block "
                        f"({t_read:.2f} s), scaled to the step's {sum(loops_per_seq)} sequence-loops "
                        f"(P_l + loops x (C + D) layers + loops readouts per sequence): {t_step:.1f} s per step"),
                seconds_per_step=t_step)


def time_oracle_step(o, block, tau, lam, k_max, rule, threads=None):
    """Wall time of one whole oracle denoise_step (prefix KV already in the oracle), with the BLAS
    pool limited to `threads` (None: as configured).  Returns (seconds, committed, threads used)."""
    from threadpoolctl import threadpool_limits
    if threads is None:
        t0 = time.perf_counter()
        out = o.denoise_step(block, tau, lam, k_max, rule)
        dt = time.perf_counter() - t0
        used = blas_threads()
    else:
        with threadpool_limits(limits=threads, user_api="blas"):
            t0 = time.perf_counter()
            out = o.denoise_step(block, tau, lam, k_max, rule)
            dt = time.perf_counter() - t0
            used = threads
    return dt, int((out["exit_depth"] > 0).sum()), used


def kv_from_handle(handle, m, k_max, b, P):
    """Sequence b's prefix KV cache read from a library handle, in the oracle's layout."""
    keys = [(("prelude", l), l) for l in range(m.n_prelude)]
    keys += [(("core", c, d), m.n_prelude + (d - 1) * m.n_core + c) for d in range(1, k_max + 1)
             for c in range(m.n_core)]
    keys += [(("coda", j), m.n_prelude + k_max * m.n_core + j) for j in range(m.n_coda)]
    out = {}
    for key, slot in keys:
        kk = handle.kv_slot(0, slot, b, P).double().cpu().numpy().transpose(1, 0, 2)
        vv = handle.kv_slot(1, slot, b, P).double().cpu().numpy().transpose(1, 0, 2)
        out[key] = (kk, vv)
    return out


def cpu_measured_steps(tau, lam, rule, handle_17=None, w_17=None, one_core_budget_s=40.0):
    """Whole oracle denoise_steps (float64, as it stands) timed on the host cores, all cores
    and one core: the tiny config (the oracle's own prefill, untimed) and, when a 1.7B handle
    is given, one 1.7B bs 1 sequence whose prefix KV is read from that handle (the oracle's
    prefill at this size alone would take minutes)."""
    from oracle import Oracle
    from synth import weights_to_numpy
    from tests.helpers import oracle_cfg
    res = []
    wl = WORKLOADS["tiny"]
    m = MODELS["tiny"]
    o = Oracle(oracle_cfg(m, wl.k_max), weights_to_numpy(make_weights(m, seed=0)), precision="fp64")
    o.prefill(make_prefix_ids(m, wl.batch, wl.prefix))
    blk = make_block_ids(m, wl.batch, wl.block)
    time_oracle_step(o, blk, tau, lam, wl.k_max, rule, None)  # untimed: the oracle's per-layer weight cache fills
    for threads in (None, 1):
        dt, c, used = time_oracle_step(o, blk, tau, lam, wl.k_max, rule, threads)
        res.append(dict(workload="tiny", cores=used, seconds=dt, committed=c, value=c / dt, unit="tokens/s"))
    if handle_17 is not None:
        wl = WORKLOADS["qwen3-1.7b-bs1"]
        m = MODELS[wl.model]
        o = Oracle(oracle_cfg(m, wl.k_max), weights_to_numpy(w_17), precision="fp64")
        o.kv = [kv_from_handle(handle_17, m, wl.k_max, 0, wl.prefix)]
        o.prefix_len = wl.prefix
        blk = make_block_ids(m, 1, wl.block)
        dt, c, used = time_oracle_step(o, blk, tau, lam, wl.k_max, rule, None)
        res.append(dict(workload=wl.name, cores=used, seconds=dt, committed=c, value=c / dt, unit="tokens/s",
                        prefix_kv="read from the library's arena"))
        if dt * used <= one_core_budget_s * 4:
            dt, c, used = time_oracle_step(o, blk, tau, lam, wl.k_max, rule, 1)
            res.append(dict(workload=wl.name, cores=used, seconds=dt, committed=c, value=c / dt, unit="tokens/s",
                            prefix_kv="read from the library's arena"))
    return res


# ------------------------------------------------------------------------------------
# our arm
# ------------------------------------------------------------------------------------

def measure_step(handle, m, wl, block_np, tau, lam, rule, steps, warmup, world, local, peaks, stream,
                 classes=True, e2e=True, clocks=True):
    """Time `steps` denoising steps of the handle (inputs resident, CUDA events on the handle's
    stream, barrier + synchronize on both sides), then optionally the per-kernel-class device
    times and the end-to-end figure through the public API with host buffers."""
    block = torch.tensor(block_np, device="cuda")
    out = handle.alloc_outputs(wl.batch, wl.block, wl.k_max)
    res = {}
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            handle.denoise_step(block, tau, lam, wl.k_max, rule, out=out)
        handle.sync()
        commits = int((out["exit_depth"] > 0).sum().item())
        res.update(commits=commits, loops=out["loops_run"].cpu().tolist(),
                   active_rows=out["active_rows"].cpu().tolist(), readout_rows=out["readout_rows"].cpu().tolist())
        clk = ClockSampler(local) if clocks else None
        if clk:
            clk.start()
        barrier(world)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            handle.denoise_step(block, tau, lam, wl.k_max, rule, out=out)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        res["clocks"] = clk.stop() if clk else None
        handle.sync()
        res["ms"] = e0.elapsed_time(e1)
        res["launches_per_step"] = handle.step_stats()["launches"]
        assert int((out["exit_depth"] > 0).sum().item()) == commits, "every timed step commits the same tokens"

        if classes:
            handle.set_timing(True)
            prof_steps = max(1, min(steps, 5))
            cls = {}
            for _ in range(prof_steps):
                handle.denoise_step(block, tau, lam, wl.k_max, rule, out=out)
                for k_, v in handle.step_stats()["classes"].items():
                    c = cls.setdefault(k_, dict(ms=0.0, launches=0, bytes=0.0, flops=0.0))
                    for f in c:
                        c[f] += v[f]
            handle.set_timing(False)
            res["classes"] = {k_: {f: v / prof_steps for f, v in c.items()} for k_, c in cls.items()}

        if e2e:
            ids_host = torch.tensor(block_np).pin_memory()
            host_out = {k_: torch.empty(v.shape, dtype=v.dtype).pin_memory() for k_, v in out.items()}
            dev_ids = torch.empty_like(block)
            res["h2d"] = ids_host.numel() * 4
            res["d2h"] = sum(v.numel() * v.element_size() for v in host_out.values())
            barrier(world)
            torch.cuda.synchronize()
            f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            f0.record(stream)
            for _ in range(steps):
                dev_ids.copy_(ids_host, non_blocking=True)
                handle.denoise_step(dev_ids, tau, lam, wl.k_max, rule, out=out)
                for k_, v in out.items():
                    host_out[k_].copy_(v, non_blocking=True)
            f1.record(stream)
            torch.cuda.synchronize()
            barrier(world)
            res["e2e_ms"] = f0.elapsed_time(f1)
    t_roof, F, Bt = step_roofline(m, wl.batch, wl.prefix, wl.block, res["active_rows"], res["readout_rows"], peaks)
    res["t_roof"], res["F"], res["B"] = t_roof, F, Bt
    res["tensor_bound"] = (F / (peaks["bf16_tflops_sustained"] * 1e12)) > (Bt / (peaks["hbm_gbs"] * 1e9))
    return res


def step_summary(name, wl, r, steps, world):
    """The secondary-workload record: the same figures as the headline, one workload."""
    ms_step = r["ms"] / steps
    d = {"workload": name, "value": r["commits"] / (ms_step / 1e3), "unit": "tokens/s", "ms_per_step": ms_step,
         "committed_per_step": r["commits"], "loops_run": r["loops"], "active_rows": r["active_rows"],
         "readout_rows": r["readout_rows"],
         "step_roofline": {"t_roof_ms": r["t_roof"] * 1e3, "frac": r["t_roof"] * 1e3 / ms_step,
                           "bound": "tensor" if r["tensor_bound"] else "hbm"},
         "config": {"model": wl.model, "batch": wl.batch, "prefix": wl.prefix, "block": wl.block, "k_max": wl.k_max,
                    "mixed_exit_depths": wl.mixed_exit_depths},
         "clocks": r.get("clocks"), "gpu_launches_per_step": r["launches_per_step"]}
    if "e2e_ms" in r:
        d["e2e"] = {"value": r["commits"] * steps / (r["e2e_ms"] / 1e3), "unit": "tokens/s",
                    "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"]}
    if "classes" in r:
        tot = max(sum(v["ms"] for v in r["classes"].values()), 1e-9)
        d["kernel_time_share"] = {k_: round(v["ms"] / tot, 4) for k_, v in r["classes"].items()}
    return d


def make_handle(alo, m, wl, w, stream, rank):
    handle = alo.Handle(m, w, k_max=wl.k_max, max_batch=wl.batch, max_prefix=wl.prefix, max_block=wl.block,
                        stream=stream)
    prefix = torch.tensor(make_prefix_ids(m, wl.batch, wl.prefix, seed=1 + rank), device="cuda")
    exit_depth = None
    if wl.mixed_exit_depths:
        exit_depth = torch.tensor(make_exit_depths(wl.batch, wl.prefix, wl.k_max, seed=2 + rank), device="cuda")
    t0 = time.time()
    handle.prefill(prefix, exit_depth)
    handle.sync()
    return handle, time.time() - t0


def assemble_line(args, wl, world, r, peaks, peaks_src, prefill_s):
    """The bench line of the GPU arm from one rank's measurement `r` (measure_step's dict): the
    whole-job throughput over the max-over-ranks time, the roofline of the dominant
    linear-layer kernel class and of each class, the step roofline, e2e and clocks."""
    tau, lam, rule = args.tau, args.lam, args.rule
    max_ms = all_max(r["ms"], world)
    max_e2e = all_max(r["e2e_ms"], world)
    total_commits = all_sum(float(r["commits"]) * args.steps, world)
    value = total_commits / (max_ms / 1e3)
    e2e_value = total_commits / (max_e2e / 1e3)
    ms_step = max_ms / args.steps

    # roofline of the dominant linear-layer kernel class: "gemm" (CTA-pair and persistent
    # kernels, many rows: tensor-bound, against the sustained bf16 peak) or "gemm_tile" (per-tile
    # split-K kernel, few rows: weight streaming, against HBM bandwidth)
    cls = r["classes"]
    dom = max(cls, key=lambda k_: cls[k_]["ms"])
    tensor_bound = r["tensor_bound"]

    def class_roofline(name):
        g = cls[name]
        if name == "gemm":
            achieved = g["flops"] / (g["ms"] / 1e3) / 1e12
            peak = peaks["bf16_tflops_sustained"]
            ro = dict(bound="tensor", achieved=achieved, peak=peak, unit="TFLOP/s", frac=achieved / peak)
        else:
            achieved = g["bytes"] / (g["ms"] / 1e3) / 1e9
            peak = peaks["hbm_gbs"]
            ro = dict(bound="hbm", achieved=achieved, peak=peak, unit="GB/s", frac=achieved / peak)
        ro["traffic"] = gemm_traffic_per_launch(args.workload, name)
        ro.update(kernel={"gemm": "gemm_pair_kernel / gemm_persist_kernel (tcgen05 linear layers, many rows)",
                          "gemm_tile": "gemm_tc_kernel (tcgen05 linear layers, few rows, split-K in a cluster)"}[name],
                  kernel_class=name, peak_source=peaks_src, launches_per_step=g["launches"], ms_per_step=g["ms"],
                  algorithmic_per_launch=(g["flops"] if name == "gemm" else g["bytes"]) / g["launches"],
                  algorithmic_unit="flop" if name == "gemm" else "byte",
                  algorithmic_bytes_per_launch=g["bytes"] / g["launches"])
        return ro

    gemm_names = [k_ for k_ in ("gemm", "gemm_tile") if k_ in cls and cls[k_]["launches"] > 0]
    gdom = max(gemm_names, key=lambda k_: cls[k_]["ms"])
    roof = class_roofline(gdom)
    gemm_rooflines = {k_: class_roofline(k_) for k_ in gemm_names}
    kernel_share = {k_: round(v["ms"] / max(sum(c["ms"] for c in cls.values()), 1e-9), 4) for k_, v in cls.items()}

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded random bf16 weights, random prefix ids, "
                                                      "all-[MASK] block)",
        "config": {"workload": args.workload, "model": wl.model, "batch_per_gpu": wl.batch, "prefix": wl.prefix,
                   "block": wl.block, "k_max": wl.k_max, "tau_H": tau, "lambda": lam,
                   "rule": ["paper", "per_token"][rule], "parallelism": f"replicas x{world}",
                   "l2": "inputs larger than L2 (weights 16 GB + KV arena)"},
        "roofline": roof,
        "gemm_rooflines": gemm_rooflines,
        "step_roofline": {"t_roof_ms": r["t_roof"] * 1e3, "frac": r["t_roof"] * 1e3 / ms_step,
                          "bound": "tensor" if tensor_bound else "hbm", "flops": r["F"], "bytes": r["B"],
                          "peak_source": peaks_src},
        "committed_per_step": r["commits"], "loops_run": r["loops"], "active_rows": r["active_rows"],
        "readout_rows": r["readout_rows"], "per_sequence_tokens_per_s": value / (wl.batch * world),
        "gpu_launches": r["launches_per_step"] * args.steps, "kernel_time_share": kernel_share,
        "dominant_kernel_class": dom, "prefill_s": prefill_s,
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"]},
        "clocks": r["clocks"],
    }

    return line


def run_ours(args, world, rank, local):
    import adaptively_looped_masked_b200 as alo
    wl = WORKLOADS[args.workload]
    m = MODELS[wl.model]
    peaks, peaks_src = load_peaks()
    stream = torch.cuda.Stream()
    w = make_weights(m, seed=0, device="cuda")
    handle, prefill_s = make_handle(alo, m, wl, w, stream, rank)
    torch.cuda.empty_cache()
    block_np = make_block_ids(m, wl.batch, wl.block)
    tau, lam, rule = args.tau, args.lam, args.rule
    r = measure_step(handle, m, wl, block_np, tau, lam, rule, args.steps, args.warmup, world, local, peaks, stream)

    line = assemble_line(args, wl, world, r, peaks, peaks_src, prefill_s)

    if world == 1 and not args.no_extras:
        # the pages' sweep: tau x lambda on the same workload, active-row fraction per loop
        # (an extra that fails is recorded in the line; the headline above stands)
        sweep = []
        try:
            for t_ in wl.taus:
                for l_ in wl.lambdas:
                    rs = measure_step(handle, m, wl, block_np, t_, l_, rule, 5, 3, world, local, peaks, stream,
                                      classes=False, e2e=False, clocks=False)
                    ms_s = rs["ms"] / 5
                    BN = wl.batch * wl.block
                    sweep.append({"tau_H": t_, "lambda": l_, "value": rs["commits"] / (ms_s / 1e3),
                                  "ms_per_step": ms_s, "committed_per_step": rs["commits"],
                                  "mean_loops": float(np.mean(rs["loops"])),
                                  "active_row_fraction": [round(x / BN, 4) for x in rs["active_rows"]],
                                  "readout_row_fraction": [round(x / BN, 4) for x in rs["readout_rows"]],
                                  "step_roofline_frac": rs["t_roof"] * 1e3 / ms_s})
        except Exception as exc:  # noqa: BLE001
            sweep.append({"error": f"{type(exc).__name__}: {exc}"[:300]})
        line["sweep"] = sweep
    handle.close()
    del handle
    torch.cuda.empty_cache()

    handle_17 = w_17 = None
    if world == 1 and not args.no_extras:
        # the other single-GPU configurations, each measured the same way
        secondary = {}
        for name in [n for n in ("qwen3-8b-bs1", "qwen3-1.7b-bs1", "qwen3-8b-long") if n != args.workload]:
            wl2 = WORKLOADS[name]
            m2 = MODELS[wl2.model]
            h2 = None
            try:
                w2 = w if wl2.model == wl.model else make_weights(m2, seed=0, device="cuda")
                h2, p2 = make_handle(alo, m2, wl2, w2, stream, rank)
                r2 = measure_step(h2, m2, wl2, make_block_ids(m2, wl2.batch, wl2.block), tau,
                                  wl2.lambdas[-1] if wl2.mixed_exit_depths else lam, rule, args.steps, args.warmup,
                                  world, local, peaks, stream)
                secondary[name] = step_summary(name, wl2, r2, args.steps, world)
                secondary[name]["prefill_s"] = p2
            except Exception as exc:  # noqa: BLE001
                secondary[name] = {"error": f"{type(exc).__name__}: {exc}"[:300]}
            if h2 is not None and name == "qwen3-1.7b-bs1" and rank == 0 and not args.no_cpu_baseline \
                    and "error" not in secondary[name]:
                handle_17, w_17 = h2, w2
            elif h2 is not None:
                h2.close()
            torch.cuda.empty_cache()
        line["secondary"] = secondary

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = cpu_sample(m, wl, r["loops"], r["commits"], w)
        line["cpu_baseline"] = {k_: cb[k_] for k_ in ("value", "unit", "cores", "kind", "sample", "extrapolated")}
        line["cpu_baseline"]["measured_steps"] = cpu_measured_steps(tau, lam, rule, handle_17, w_17)
    if handle_17 is not None:
        handle_17.close()
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_decode(args, world, rank, local):
    """Block decoding (alodlm_decode_block): denoising steps over the workload's block until no
    [MASK] is left.  value = masks decoded per second over whole decodes; the roofline sums
    the step roofline of every step taken."""
    import adaptively_looped_masked_b200 as alo
    wl = WORKLOADS[args.workload]
    m = MODELS[wl.model]
    peaks, peaks_src = load_peaks()
    stream = torch.cuda.Stream()
    w = make_weights(m, seed=0, device="cuda")
    handle = alo.Handle(m, w, k_max=wl.k_max, max_batch=wl.batch, max_prefix=wl.prefix, max_block=wl.block,
                        stream=stream)
    del w
    torch.cuda.empty_cache()
    prefix = torch.tensor(make_prefix_ids(m, wl.batch, wl.prefix, seed=1 + rank), device="cuda")
    exit_depth = None
    if wl.mixed_exit_depths:
        exit_depth = torch.tensor(make_exit_depths(wl.batch, wl.prefix, wl.k_max, seed=2 + rank), device="cuda")
    handle.prefill(prefix, exit_depth)
    handle.sync()
    block_np = make_block_ids(m, wl.batch, wl.block)
    block = torch.tensor(block_np, device="cuda")
    masks = int((block_np == m.mask_id).sum())
    tau, lam, rule = args.tau, args.lam, args.rule
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            dec = handle.decode_block(block, tau, lam, wl.k_max, rule)
        handle.sync()
        steps = dec["steps"]
        rows = dec["rows"].cpu().numpy()
        left = int((dec["tokens"] == m.mask_id).sum().item())
        clocks = ClockSampler(local)
        clocks.start()
        barrier(world)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            dec = handle.decode_block(block, tau, lam, wl.k_max, rule)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        clk = clocks.stop()
        handle.sync()
        ms = e0.elapsed_time(e1)
        assert dec["steps"] == steps, "decoding is deterministic"
        # end to end: block ids from pinned host memory in, final tokens back out, every call
        ids_host = torch.tensor(block_np).pin_memory()
        tok_host = torch.empty(block_np.shape, dtype=torch.int32).pin_memory()
        dev_ids = torch.empty_like(block)
        torch.cuda.synchronize()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for _ in range(args.steps):
            dev_ids.copy_(ids_host, non_blocking=True)
            dec = handle.decode_block(dev_ids, tau, lam, wl.k_max, rule)
            tok_host.copy_(dec["tokens"], non_blocking=True)
        f1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = f0.elapsed_time(f1)
    launches_last_step = handle.step_stats()["launches"]
    max_ms = all_max(ms, world)
    decoded = all_sum(float(masks - left) * args.steps, world)
    value = decoded / (max_ms / 1e3)
    t_roof = 0.0
    for t in range(steps):
        tr, _, _ = step_roofline(m, wl.batch, wl.prefix, wl.block, rows[t, 0].tolist(), rows[t, 1].tolist(), peaks)
        t_roof += tr
    ms_call = max_ms / args.steps
    line = {
        "metric": "decoded tokens/s (block denoised until no [MASK]; 8B-shape bf16)", "value": value,
        "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_call,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded random bf16 weights, random prefix ids, all-[MASK] block)",
        "config": {"workload": args.workload, "model": wl.model, "batch_per_gpu": wl.batch, "prefix": wl.prefix,
                   "block": wl.block, "k_max": wl.k_max, "tau_H": tau, "lambda": lam,
                   "rule": ["paper", "per_token"][rule], "parallelism": f"replicas x{world}", "mode": "decode_block"},
        "denoising_steps_per_block": steps, "masks_left": left,
        "step_roofline": {"t_roof_ms": t_roof * 1e3, "frac": t_roof * 1e3 / ms_call, "peak_source": peaks_src},
        "e2e": {"value": decoded / (all_max(e2e_ms, world) / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": block_np.size * 4, "d2h_bytes_per_step": block_np.size * 4},
        "gpu_launches": launches_last_step * steps * args.steps, "clocks": clk,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    handle.close()


# ------------------------------------------------------------------------------------
# reference arm: the CPU oracle, as it stands, on bounded samples of the same workload
# ------------------------------------------------------------------------------------

def run_reference(args, world, rank):
    """The oracle, as it stands, on the host cores: each step times one Core layer and one
    readout of one sequence and scales them to the workload's step by the loop profile the GPU
    arm measured for it (GPU_LOOP_PROFILE), so the line is an extrapolation and says so."""
    if rank != 0:
        return
    wl = WORKLOADS[args.workload]
    m = MODELS[wl.model]
    # only the timed Core layer and the heads are generated
    w = make_weights(m, seed=0, device="cuda" if torch.cuda.is_available() else "cpu", only_layers=[m.n_prelude])
    prof = GPU_LOOP_PROFILE.get(args.workload)
    if prof is not None:
        loops, commits = prof["loops"], prof["commits"]
        how = "loop profile of the GPU arm's measured step (loops per sequence, tokens committed)"
    else:
        loops, commits = [2] * wl.batch, wl.batch * wl.block
        how = "no GPU loop profile recorded for this workload: 2 loops per sequence, whole block committed"
    vals = []
    t_all = time.perf_counter()
    for i in range(args.warmup + args.steps):
        cb = cpu_sample(m, wl, loops, commits, w, budget_s=4.0)
        if i >= args.warmup:
            vals.append(cb)
    elapsed = time.perf_counter() - t_all
    value = statistics.median(v["value"] for v in vals)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": statistics.median(v["seconds_per_step"] for v in vals) * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "extrapolated": True,
            "config": {"workload": args.workload, "model": wl.model, "batch_per_gpu": wl.batch, "prefix": wl.prefix,
                       "block": wl.block, "k_max": wl.k_max, "tau_H": args.tau, "lambda": args.lam,
                       "rule": ["paper", "per_token"][args.rule]},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": vals[0]["cores"], "kind": "oracle",
                             "extrapolated": True, "sample": vals[0]["sample"] + "; scaled with the " + how},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "wall_s": elapsed}
    print(json.dumps(line), flush=True)


def run_kernel_gemm(args):
    """Micro-benchmark of the tcgen05 GEMM alone (alodlm_gemm_bf16): C[M,N] = A[M,K] W[N,K]^T.

    Like the step's linear layers, every launch reads its weight cold from HBM: the launches
    rotate over enough weight copies (about 400 MB) that none is still in L2 when it comes back.
    """
    import adaptively_looped_masked_b200 as alo
    M, N, K = (int(x) for x in args.shape.split(","))
    torch.cuda.set_device(0)
    g = torch.Generator(device="cuda").manual_seed(0)
    A = torch.randn((M, K), device="cuda", generator=g).to(torch.bfloat16)
    n_w = max(2, int(400e6 // (2 * N * K)) + 1)
    Ws = [torch.randn((N, K), device="cuda", generator=g).to(torch.bfloat16) for _ in range(n_w)]
    C = torch.empty((M, N), dtype=torch.float32, device="cuda")
    ws = torch.zeros(64, dtype=torch.float32, device="cuda")  # the status word
    peaks, src = load_peaks()
    stream = torch.cuda.current_stream()
    for i in range(args.warmup):
        alo.gemm_bf16(A, Ws[i % n_w], out=C, workspace=ws)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(args.steps):
        alo.gemm_bf16(A, Ws[i % n_w], out=C, workspace=ws)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    by = 2.0 * N * K + 2.0 * M * K + 4.0 * M * N
    fl = 2.0 * M * N * K
    print(json.dumps({"kernel": "gemm_bf16", "M": M, "N": N, "K": K, "ms": ms, "GB/s": by / ms / 1e6,
                      "TFLOP/s": fl / ms / 1e9, "hbm_frac": by / ms / 1e6 / peaks["hbm_gbs"],
                      "tensor_frac": fl / ms / 1e9 / peaks["bf16_tflops"], "peak_source": src,
                      "weights": f"{n_w} rotating copies (cold in L2)"}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="qwen3-8b-bs32", choices=sorted(WORKLOADS))
    ap.add_argument("--tau", type=float, default=0.6)
    ap.add_argument("--lam", type=float, default=0.5)
    ap.add_argument("--rule", type=int, default=0, choices=[0, 1])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="headline workload only: no tau x lambda sweep and no secondary workloads")
    ap.add_argument("--decode", action="store_true",
                    help="time block decoding (steps until no [MASK]) instead of one step")
    ap.add_argument("--kernel", default=None, choices=["gemm"],
                    help="micro-benchmark one kernel instead of the step")
    ap.add_argument("--shape", default="32,24576,4096", help="M,N,K for --kernel gemm")
    args = ap.parse_args()
    if args.kernel == "gemm":
        run_kernel_gemm(args)
        return
    world, rank, local = dist_setup(args.gpus)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        elif args.decode:
            run_decode(args, world, rank, local)
        else:
            run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
