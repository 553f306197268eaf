"""Helpers of the GPU tests: build a library handle and an oracle from the same seeded
inputs, and compare a step's outputs with the oracle's.

Every tolerance and band below is fixed before the GPU runs.

Readout stage, on the GPU's own readout states r^(s), i.e. the same inputs on both sides:
  ENTROPY_TOL  |dH| <= 1e-2 nats
  GATE_TOL     |d lambda| <= 1e-3
  BAND         the argmax must match unless the top-two logit gap is below 1e-3

End to end, the float64 oracle running the whole step from the same ids and weights, at loop
s (e2e_tolerances): per-row relative deviation of the states h^(s-1), h~^(s), r^(s) and of
the logits, |dH|, |d lambda| and |d a|, and the top-two logit gap below which either token
is a correct argmax.  Each is three times the spread between the oracle in its bf16
precision (float64 or float32 accumulation, whichever lies further) and the oracle in
float64 at that loop (tests/golden/oracle_spread.json, written by make_oracle_spread.py from
the oracle alone), and never below the fixed values 2e-2 (states, logits), 1e-2 nats, 1e-3
(halts, argmax gap).  The factor covers the kernels' own rounding that no oracle variant
models (approximate exp2, softmax probabilities rounded against a running maximum, the
order of additions).  The entropy, halt and argmax values are also
the bands within which a decision may go either way: outside them every decision (commit,
exit depth, token, halt, forced pick) must be the oracle's own.

Why a per-loop table: with bf16 activations the rounding of every matrix operand adds an
independent error at every layer application, so two correct implementations drift apart as
the loop deepens -- at the Qwen3-1.7B shape the bf16 oracle lies 3.6e-2 (state) and 0.56
nats from the float64 oracle after 8 loops of 20 layers; at the tiny config 7e-3 and 0.05.
"""
import json
import os

import numpy as np
import torch

from oracle import Oracle
from synth import MODELS, WORKLOADS, make_weights, weights_to_numpy, make_prefix_ids, make_block_ids
from tests.helpers import oracle_cfg

ENTROPY_TOL = 1e-2
GATE_TOL = 1e-3
BAND = 1e-3
STATE_REL_TOL = 2e-2
SPREAD_FACTOR = 3.0
SPREAD_FILE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "oracle_spread.json")
_SPREAD_MODEL = {"tiny_fullcore": "tiny"}


def e2e_tolerances(model: str, K: int) -> dict:
    """Per-loop end-to-end tolerances, lists indexed by s - 1 (s = 1..K): state, logits,
    entropy, halt, argmax.  A deeper loop is never held tighter than a shallower one."""
    with open(SPREAD_FILE) as f:
        rows = json.load(f)[_SPREAD_MODEL.get(model, model)]["per_loop"]
    floor = dict(state=STATE_REL_TOL, logits=STATE_REL_TOL, entropy=ENTROPY_TOL, halt=GATE_TOL, gap=BAND)
    run = {k: 0.0 for k in floor}
    out = {k: [] for k in floor}
    for s in range(1, K + 1):
        r = rows[min(s, len(rows)) - 1]
        for k in floor:
            run[k] = max(run[k], r[k])
            out[k].append(max(floor[k], SPREAD_FACTOR * run[k]))
    out["argmax"] = out.pop("gap")
    return out


def e2e_bands(model: str, K: int) -> dict:
    t = e2e_tolerances(model, K)
    return dict(entropy=t["entropy"], halt=t["halt"], argmax=t["argmax"])


class Case:
    """One model + workload: device weights, a library handle, and host copies for the oracle."""

    def __init__(self, model: str, batch: int, prefix: int, block: int, k_max: int, debug=True, seed=0,
                 stream=None, weights=None):
        import adaptively_looped_masked_b200 as alo
        self.m = MODELS[model]
        self.batch, self.prefix, self.block, self.k_max = batch, prefix, block, k_max
        big = self.m.hidden >= 1024
        if weights is not None:
            self.w_dev = weights
        else:
            self.w_dev = make_weights(self.m, seed=seed, device="cuda" if big else "cpu")
            if not big:
                self.w_dev = _to_cuda(self.w_dev)
        self.stream = stream if stream is not None else torch.cuda.Stream()
        self.handle = alo.Handle(self.m, self.w_dev, k_max=k_max, max_batch=batch, max_prefix=prefix,
                                 max_block=block, debug_dump=debug, stream=self.stream)
        self.prefix_ids = make_prefix_ids(self.m, batch, prefix)
        self.block_ids = make_block_ids(self.m, batch, block)
        self._w_host = None

    @property
    def w_host(self):
        if self._w_host is None:
            self._w_host = weights_to_numpy(self.w_dev)
        return self._w_host

    def oracle(self, precision="bf16", dtype=np.float64):
        return Oracle(oracle_cfg(self.m, self.k_max), self.w_host, precision=precision, dtype=dtype)

    def prefill(self, exit_depth=None):
        ids = torch.tensor(self.prefix_ids, device="cuda")
        e = None if exit_depth is None else torch.tensor(exit_depth, device="cuda")
        self.handle.prefill(ids, e)
        self.handle.sync()

    def step(self, tau, lam, k_max=None, rule=0, block_ids=None):
        k = self.k_max if k_max is None else k_max
        blk = torch.tensor(self.block_ids if block_ids is None else block_ids, device="cuda")
        out = self.handle.denoise_step(blk, tau, lam, k, rule)
        self.handle.sync()
        return {kk: v.cpu().numpy() for kk, v in out.items()}

    def kv_from_gpu(self, b: int, dtype=np.float32) -> dict:
        """Sequence b's depth-aware KV cache as the oracle stores it, read from the library's
        arena: {("prelude", l) | ("core", c, d) | ("coda", j): (K, V)}, each [P, nkv, hd]."""
        m, K, P = self.m, self.k_max, self.prefix
        keys = [(("prelude", l), l) for l in range(m.n_prelude)]
        keys += [(("core", c, d), m.n_prelude + (d - 1) * m.n_core + c)
                 for d in range(1, K + 1) for c in range(m.n_core)]
        keys += [(("coda", j), m.n_prelude + K * m.n_core + j) for j in range(m.n_coda)]
        out = {}
        for key, slot in keys:
            kk = self.handle.kv_slot(0, slot, b, P).float().cpu().numpy().transpose(1, 0, 2)
            vv = self.handle.kv_slot(1, slot, b, P).float().cpu().numpy().transpose(1, 0, 2)
            out[key] = (kk.astype(dtype), vv.astype(dtype))
        return out


def _to_cuda(w):
    out = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in w.items() if k != "layers"}
    out["layers"] = [{k: v.cuda() for k, v in lw.items()} for lw in w["layers"]]
    return out


def follow_of(gpu: dict, seqs=None) -> dict:
    sel = slice(None) if seqs is None else np.asarray(seqs)
    return dict(tokens=gpu["tokens"][sel], exit_depth=gpu["exit_depth"][sel], loops_run=gpu["loops_run"][sel])


def compare_decisions(gpu: dict, ref: dict, rows=True):
    """Tokens, exit depths, loops and the NaN pattern of the traces match exactly (and the
    per-loop row counters, for a whole batch)."""
    np.testing.assert_array_equal(gpu["loops_run"], ref["loops_run"])
    np.testing.assert_array_equal(gpu["exit_depth"], ref["exit_depth"])
    np.testing.assert_array_equal(gpu["tokens"], ref["tokens"])
    np.testing.assert_array_equal(np.isnan(gpu["entropy"]), np.isnan(ref["entropy"]))
    if rows:
        np.testing.assert_array_equal(gpu["active_rows"], ref["active_rows"])
        np.testing.assert_array_equal(gpu["readout_rows"], ref["readout_rows"])


def row_rel_err(a: np.ndarray, ref: np.ndarray) -> np.ndarray:
    return np.linalg.norm(a - ref, axis=-1) / np.maximum(np.linalg.norm(ref, axis=-1), 1e-30)


def readout_stage_check(case, gpu: dict, r_by_loop: dict, seqs=None, rows_per_loop=None, rng=None, ob=None,
                        sample_key=None):
    """Readout parity on the GPU's own readout states r^(s): the oracle's LM head + entropy +
    argmax + ExitGate in the kernels' precision.  Returns token_at(b, s, i) for the replay and
    the max deviations.  rows_per_loop (optional) samples that many rows per (b, s).  With
    sample_key the token is the oracle's Gumbel-max draw on the same logits."""
    from oracle.alodlm_oracle import gumbel_scores
    ob = ob if ob is not None else case.oracle("bf16")
    toks, max_dH, max_dl, n_ties = {}, 0.0, 0.0, 0
    B, K, N = gpu["entropy"].shape
    for b in (range(B) if seqs is None else seqs):
        for s in range(1, int(gpu["loops_run"][b]) + 1):
            idx = np.nonzero(~np.isnan(gpu["entropy"][b, s - 1]))[0]
            if len(idx) == 0:
                continue
            if rows_per_loop is not None and len(idx) > rows_per_loop:
                idx = np.sort(rng.choice(idx, size=rows_per_loop, replace=False))
            H, y, lam, z = ob.readout(r_by_loop[s][b][idx].astype(ob.dt))
            if sample_key is not None:  # the token is the draw: argmax of z + g
                z = np.stack([gumbel_scores(z[t], sample_key, b * N + int(i), s) for t, i in enumerate(idx)])
                y = np.argmax(z, axis=-1)
            dH = np.abs(H - gpu["entropy"][b, s - 1, idx])
            dl = np.abs(lam - gpu["halt"][b, s - 1, idx])
            max_dH, max_dl = max(max_dH, float(dH.max())), max(max_dl, float(dl.max()))
            top2 = np.sort(z, axis=-1)[:, -2:]
            for t, i in enumerate(idx):
                tok = int(y[t])
                committed_here = gpu["exit_depth"][b, i] == s
                if top2[t, 1] - top2[t, 0] < BAND:  # near tie: either id is a correct argmax
                    n_ties += 1
                    if committed_here and z[t, gpu["tokens"][b, i]] >= top2[t, 1] - BAND:
                        tok = int(gpu["tokens"][b, i])
                elif committed_here:
                    assert gpu["tokens"][b, i] == tok, ("argmax", b, s, int(i))
                toks[(b, s, int(i))] = tok
    assert max_dH <= ENTROPY_TOL, f"readout entropy |d| {max_dH}"
    assert max_dl <= GATE_TOL, f"exit gate |d| {max_dl}"

    def token_at(b, s, i):
        return toks.get((b, s, i), int(gpu["tokens"][b, i]))
    return token_at, dict(readout_dH=max_dH, readout_dlam=max_dl, argmax_ties=n_ties)


def step_parity(case, gpu: dict, tau: float, lam: float, K: int, rule: int, block_ids: np.ndarray,
                states=True, oracle=None, seqs=None, rows_per_loop=None, ob=None, sample_key=None) -> dict:
    """The three parity checks of one step (see tests/test_gpu_parity.py).

    oracle: a float64 (or float32) oracle whose prefix KV is ready -- prefilled by the oracle
    itself, or read from the library's arena; default: a float64 oracle prefilled here.
    seqs: the sequences to check end to end (default all; the oracle then holds only these).
    sample_key: (seed, step) of a sampled step (tokens drawn by Gumbel-max)."""
    from oracle.alodlm_oracle import replay_decisions
    B = block_ids.shape[0]
    seq_list = list(range(B)) if seqs is None else [int(b) for b in seqs]
    rng = np.random.default_rng(0)
    r_by_loop = {s: case.handle.debug_state(2, s).cpu().numpy() for s in range(1, int(gpu["loops_run"].max()) + 1)}
    # (1) readout stage on the GPU's own r
    token_at, stats = readout_stage_check(case, gpu, r_by_loop, seqs=seq_list, rows_per_loop=rows_per_loop,
                                          rng=rng, ob=ob, sample_key=sample_key)
    # (2) every decision re-taken from the GPU's traces by the oracle's rules: exact
    rep = replay_decisions(block_ids, case.m.mask_id, gpu["entropy"], gpu["cum_halt"], token_at, tau, lam, K, rule)
    assert not rep["ambiguous"], rep["ambiguous"]
    np.testing.assert_array_equal(gpu["exit_depth"], rep["exit_depth"])
    np.testing.assert_array_equal(gpu["tokens"], rep["tokens"])
    np.testing.assert_array_equal(gpu["loops_run"], rep["loops_run"])
    # (3) end to end: the oracle takes its own decisions except inside the fixed bands
    of = oracle
    if of is None:
        of = case.oracle("fp64")
        of.prefill(case.prefix_ids)
    sel = np.asarray(seq_list)
    assert seqs is None or sample_key is None, "a sampled draw depends on the sequence's index in the batch"
    tol = e2e_tolerances(case.m.name, K)
    ref = of.denoise_step(block_ids[sel], tau, lam, K, rule, follow=follow_of(gpu, sel),
                          band=dict(entropy=tol["entropy"], halt=tol["halt"], argmax=tol["argmax"]),
                          sample_key=sample_key)
    sub = {k: gpu[k][sel] for k in ("tokens", "exit_depth", "loops_run", "entropy", "halt", "cum_halt")}
    sub["active_rows"], sub["readout_rows"] = gpu["active_rows"], gpu["readout_rows"]
    compare_decisions(sub, ref, rows=seqs is None)
    W = of._global("lm_head")
    worst = dict(state=0.0, logits=0.0, entropy=0.0, halt=0.0)
    keys = ((2, "r"),) if not states else ((0, "h_in"), (1, "h_tilde"), (2, "r"))
    dbg = {(which, s): (r_by_loop[s] if which == 2 else case.handle.debug_state(which, s).cpu().numpy())
           for which, _ in keys for s in range(1, int(gpu["loops_run"][sel].max()) + 1)}
    for j, b in enumerate(seq_list):
        for s in range(1, int(gpu["loops_run"][b]) + 1):
            for which, key in keys:
                rel = row_rel_err(dbg[(which, s)][b], ref[key][j][s - 1])
                worst["state"] = max(worst["state"], float(rel.max()))
                assert rel.max() <= tol["state"][s - 1], (key, b, s, rel.max(), tol["state"][s - 1])
            idx = np.nonzero(~np.isnan(gpu["entropy"][b, s - 1]))[0]
            if len(idx) == 0:
                continue
            r_ref = ref["r"][j][s - 1][idx]
            z_ref = r_ref @ W.T
            dz = (dbg[(2, s)][b][idx].astype(z_ref.dtype) - r_ref) @ W.T
            lrel = np.linalg.norm(dz, axis=-1) / np.linalg.norm(z_ref, axis=-1)
            worst["logits"] = max(worst["logits"], float(lrel.max()))
            assert lrel.max() <= tol["logits"][s - 1], ("logits", b, s, lrel.max(), tol["logits"][s - 1])
            dH = np.abs(gpu["entropy"][b, s - 1, idx] - ref["entropy"][j, s - 1, idx])
            worst["entropy"] = max(worst["entropy"], float(dH.max()))
            assert dH.max() <= tol["entropy"][s - 1], ("entropy", b, s, float(dH.max()), tol["entropy"][s - 1])
            for key in ("halt", "cum_halt"):
                da = np.abs(gpu[key][b, s - 1, idx] - ref[key][j, s - 1, idx])
                worst["halt"] = max(worst["halt"], float(da.max()))
                assert da.max() <= tol["halt"][s - 1], (key, b, s, float(da.max()), tol["halt"][s - 1])
    differing = [f for f in ref["followed"] if f.get("own") != f.get("taken")]
    stats.update({f"e2e_{k}": v for k, v in worst.items()})
    stats["e2e_followed"] = len(ref["followed"])
    stats["e2e_followed_differing"] = len(differing)
    stats["e2e_differing_margins"] = sorted((f["kind"], round(abs(f["margin"]), 4)) for f in differing)[:8]
    return stats
