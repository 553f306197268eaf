"""Writes tests/golden/oracle_spread.json: how far a correct bf16 implementation of the step
lands from the exact (float64) step, measured on the oracle alone.

For each configuration the oracle runs the same step three times from the same seeded weights
and ids: in its bf16 precision (every matrix operand rounded to bfloat16 where the CUDA kernels
round it) with float64 accumulation, the same with float32 accumulation (as the tensor cores
accumulate), and in float64 throughout.  Commits are disabled (tau below every entropy,
lambda above 1, the paper's rule) so that every loop 1..K runs on every position.  Per loop s
it records, over both bf16 runs, the largest deviation from the float64 run of:
  state    per-row ||d|| / ||ref|| of h^(s-1), h~^(s) and r^(s)
  logits   per-row ||d|| / ||ref|| of the LM-head logits
  entropy  |dH| (nats)
  halt     |d lambda| and |d a|
  gap      the change of the top-two logit gap (at the float64 run's top two ids)
The GPU tests take their end-to-end tolerances from this table (twice the spread at loop s,
never below the fixed readout-stage values), so no tolerance depends on the GPU's own error.
The batch and block match the tests that use each row (the spread is a maximum over
positions); the Qwen3 shapes use a shorter prefix than their workloads (the spread grows
with the number of layer applications, not with the prefix length) and host-generated
weights of the same scales.

    python tests/golden/make_oracle_spread.py [tiny mid attn-probe qwen3-1.7b qwen3-8b]
"""
import json
import os
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from oracle import Oracle  # noqa: E402
from synth import MODELS, make_block_ids, make_prefix_ids, make_weights, weights_to_numpy  # noqa: E402
from tests.helpers import oracle_cfg  # noqa: E402

OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_spread.json")

# model -> (batch, prefix, block, K): K covers the deepest loop any workload of the model runs
CALIB = {"tiny": (1, 48, 16, 4), "mid": (3, 75, 20, 5), "attn-probe": (12, 160, 72, 3),
         "qwen3-1.7b": (1, 256, 32, 8), "qwen3-8b": (2, 128, 64, 12)}


def host_weights(m):
    """The seeded weights as float32 numpy arrays, drawn one layer at a time (the 8B shape's
    full torch draw and its float32 copy would not both fit in host memory)."""
    w = weights_to_numpy(make_weights(m, seed=0, only_layers=[]), layers=[])
    w["layers"] = []
    for li in range(m.n_layers):
        lw = make_weights(m, seed=0, only_layers=[li], with_globals=False)["layers"][li]
        w["layers"].append({k: v.to(torch.float32).numpy() for k, v in lw.items()})
    return w


def rel(a, b):
    return np.linalg.norm(a - b, axis=-1) / np.maximum(np.linalg.norm(b, axis=-1), 1e-30)


def spread(name):
    B, P, N, K = CALIB[name]
    m = MODELS[name]
    w = host_weights(m)
    pre, blk = make_prefix_ids(m, B, P), make_block_ids(m, B, N)
    runs = {}
    for tag, prec, dt in (("bf16", "bf16", np.float64), ("bf16_f32acc", "bf16", np.float32),
                          ("fp64", "fp64", np.float64)):
        t0 = time.time()
        o = Oracle(oracle_cfg(m, K), w, precision=prec, dtype=dt)
        o.prefill(pre)
        runs[tag] = o.denoise_step(blk, -1.0, 2.0, K, 0)
        del o
        print(f"{name} {tag}: {time.time() - t0:.0f} s", flush=True)
    ref = runs["fp64"]
    W = w["lm_head"].astype(np.float64)
    per = []
    for s in range(K):
        row = dict(loop=s + 1, state=0.0, logits=0.0, entropy=0.0, halt=0.0, gap=0.0)
        for tag in ("bf16", "bf16_f32acc"):
            a = runs[tag]
            for b in range(B):
                row["state"] = max(row["state"], max(float(rel(np.asarray(a[k][b][s], np.float64),
                                                                  ref[k][b][s]).max())
                                                      for k in ("h_in", "h_tilde", "r")))
                za = np.asarray(a["r"][b][s], np.float64) @ W.T
                zb = ref["r"][b][s] @ W.T
                top = np.argsort(zb, axis=1)[:, -2:]
                ga = np.take_along_axis(za, top, 1)
                gb = np.take_along_axis(zb, top, 1)
                row["logits"] = max(row["logits"], float(rel(za, zb).max()))
                row["gap"] = max(row["gap"], float(np.abs((ga[:, 1] - ga[:, 0]) - (gb[:, 1] - gb[:, 0])).max()))
            row["entropy"] = max(row["entropy"], float(np.nanmax(np.abs(a["entropy"][:, s] - ref["entropy"][:, s]))))
            row["halt"] = max(row["halt"], float(np.nanmax(np.abs(a["halt"][:, s] - ref["halt"][:, s]))),
                              float(np.nanmax(np.abs(a["cum_halt"][:, s] - ref["cum_halt"][:, s]))))
        per.append(row)
        print(name, per[-1], flush=True)
    return dict(batch=B, prefix=P, block=N, k_max=K, layers_per_loop=m.n_core + m.n_coda, n_prelude=m.n_prelude,
                per_loop=per)


if __name__ == "__main__":
    names = sys.argv[1:] or list(CALIB)
    for n in names:
        row = spread(n)
        table = json.load(open(OUT)) if os.path.exists(OUT) else {}  # merge with rows written meanwhile
        table[n] = row
        with open(OUT, "w") as f:
            json.dump(table, f, indent=1)
