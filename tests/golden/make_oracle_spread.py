"""Writes tests/golden/oracle_spread.json: how far a correct bf16 implementation of the step
lands from the exact (float64) step, measured on the oracle alone.

For each configuration the oracle runs the same step twice from the same seeded weights and
ids: once in its bf16 precision (every matrix operand rounded to bfloat16 where the CUDA
kernels round it, float64 accumulation) and once in float64 throughout.  Commits are disabled
(tau below every entropy, lambda above 1, the paper's rule) so that every loop 1..K runs on
every position.  Per loop s it records the largest deviation between the two runs of:
  state    per-row ||d|| / ||ref|| of h^(s-1), h~^(s) and r^(s)
  logits   per-row ||d|| / ||ref|| of the LM-head logits
  entropy  |dH| (nats)
  halt     |d lambda| and |d a|
  gap      the change of the top-two logit gap (at the float64 run's top two ids)
The GPU tests take their end-to-end tolerances from this table (twice the spread at loop s,
never below the fixed readout-stage values), so no tolerance depends on the GPU's own error.
The Qwen3 shapes use a shorter prefix than their workloads (the spread grows with the number
of layer applications, not with the prefix length) and host-generated weights of the same
scales.

    python tests/golden/make_oracle_spread.py [tiny mid qwen3-1.7b qwen3-8b]
"""
import json
import os
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from oracle import Oracle  # noqa: E402
from synth import MODELS, make_block_ids, make_prefix_ids, make_weights, weights_to_numpy  # noqa: E402
from tests.helpers import oracle_cfg  # noqa: E402

OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_spread.json")

# model -> (prefix, block, K): K covers the deepest loop any workload of the model runs
CALIB = {"tiny": (48, 16, 4), "mid": (75, 20, 5), "qwen3-1.7b": (256, 32, 8), "qwen3-8b": (128, 32, 12)}


def rel(a, b):
    return np.linalg.norm(a - b, axis=-1) / np.maximum(np.linalg.norm(b, axis=-1), 1e-30)


def spread(name):
    P, N, K = CALIB[name]
    m = MODELS[name]
    w = weights_to_numpy(make_weights(m, seed=0))
    pre, blk = make_prefix_ids(m, 1, P), make_block_ids(m, 1, N)
    runs = {}
    for prec in ("bf16", "fp64"):
        t0 = time.time()
        o = Oracle(oracle_cfg(m, K), w, precision=prec, dtype=np.float64)
        o.prefill(pre)
        runs[prec] = o.denoise_step(blk, -1.0, 2.0, K, 0)
        print(f"{name} {prec}: {time.time() - t0:.0f} s", flush=True)
    a, b = runs["bf16"], runs["fp64"]
    W = w["lm_head"].astype(np.float64)
    per = []
    for s in range(K):
        st = max(float(rel(a[k][0][s], b[k][0][s]).max()) for k in ("h_in", "h_tilde", "r"))
        za, zb = a["r"][0][s] @ W.T, b["r"][0][s] @ W.T
        top = np.argsort(zb, axis=1)[:, -2:]
        ga = np.take_along_axis(za, top, 1)
        gb = np.take_along_axis(zb, top, 1)
        per.append(dict(loop=s + 1, state=st, logits=float(rel(za, zb).max()),
                        entropy=float(np.nanmax(np.abs(a["entropy"][0, s] - b["entropy"][0, s]))),
                        halt=float(max(np.nanmax(np.abs(a["halt"][0, s] - b["halt"][0, s])),
                                       np.nanmax(np.abs(a["cum_halt"][0, s] - b["cum_halt"][0, s])))),
                        gap=float(np.abs((ga[:, 1] - ga[:, 0]) - (gb[:, 1] - gb[:, 0])).max())))
        print(name, per[-1], flush=True)
    return dict(prefix=P, block=N, k_max=K, layers_per_loop=m.n_core + m.n_coda, n_prelude=m.n_prelude,
                per_loop=per)


if __name__ == "__main__":
    names = sys.argv[1:] or list(CALIB)
    table = json.load(open(OUT)) if os.path.exists(OUT) else {}
    for n in names:
        table[n] = spread(n)
        with open(OUT, "w") as f:
            json.dump(table, f, indent=1)
