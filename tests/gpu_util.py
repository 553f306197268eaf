"""Helpers of the GPU tests: build a library handle and an oracle from the same seeded
inputs, and compare a step's outputs with the oracle's."""
import numpy as np
import torch

from oracle import Oracle
from synth import MODELS, WORKLOADS, make_weights, weights_to_numpy, make_prefix_ids, make_block_ids
from tests.helpers import oracle_cfg

ENTROPY_TOL = 1e-2      # nats
STATE_REL_TOL = 2e-2    # per-row ||d||/||ref|| of hidden / readout states
GATE_TOL = 1e-2         # lambda and cumulative halt (absolute)
BAND = 1e-3             # near-threshold band within which a decision is followed


class Case:
    """One model + workload: device weights, a library handle, and host copies for the oracle."""

    def __init__(self, model: str, batch: int, prefix: int, block: int, k_max: int, debug=True, seed=0,
                 stream=None):
        import adaptively_looped_masked_b200 as alo
        self.m = MODELS[model]
        self.batch, self.prefix, self.block, self.k_max = batch, prefix, block, k_max
        big = self.m.hidden >= 1024
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


def _to_cuda(w):
    out = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in w.items() if k != "layers"}
    out["layers"] = [{k: v.cuda() for k, v in lw.items()} for lw in w["layers"]]
    return out


def follow_of(gpu: dict) -> dict:
    return dict(tokens=gpu["tokens"], exit_depth=gpu["exit_depth"], loops_run=gpu["loops_run"])




def compare_decisions(gpu: dict, ref: dict):
    """Tokens, exit depths, loops, row counters and the NaN pattern of the traces match exactly."""
    np.testing.assert_array_equal(gpu["loops_run"], ref["loops_run"])
    np.testing.assert_array_equal(gpu["exit_depth"], ref["exit_depth"])
    np.testing.assert_array_equal(gpu["tokens"], ref["tokens"])
    np.testing.assert_array_equal(np.isnan(gpu["entropy"]), np.isnan(ref["entropy"]))
    np.testing.assert_array_equal(gpu["active_rows"], ref["active_rows"])
    np.testing.assert_array_equal(gpu["readout_rows"], ref["readout_rows"])


def row_rel_err(a: np.ndarray, ref: np.ndarray) -> np.ndarray:
    return np.linalg.norm(a - ref, axis=-1) / np.maximum(np.linalg.norm(ref, axis=-1), 1e-30)


def readout_stage_check(case, gpu: dict, r_by_loop: dict):
    """Readout parity on the GPU's own readout states r^(s): the oracle's LM head + entropy +
    argmax + ExitGate in the kernels' precision.  Returns token_at(b, s, i) for the replay and
    the max deviations."""
    ob = case.oracle("bf16")
    toks, max_dH, max_dl, n_ties = {}, 0.0, 0.0, 0
    B, K, N = gpu["entropy"].shape
    for b in range(B):
        for s in range(1, int(gpu["loops_run"][b]) + 1):
            idx = np.nonzero(~np.isnan(gpu["entropy"][b, s - 1]))[0]
            if len(idx) == 0:
                continue
            H, y, lam, z = ob.readout(r_by_loop[s][b][idx])
            dH = np.abs(H - gpu["entropy"][b, s - 1, idx])
            dl = np.abs(lam - gpu["halt"][b, s - 1, idx])
            max_dH, max_dl = max(max_dH, float(dH.max())), max(max_dl, float(dl.max()))
            top2 = np.sort(z, axis=-1)[:, -2:]
            for t, i in enumerate(idx):
                tok = int(y[t])
                if top2[t, 1] - top2[t, 0] < BAND:  # near tie: either id is a correct argmax
                    n_ties += 1
                    if gpu["exit_depth"][b, i] == s and z[t, gpu["tokens"][b, i]] >= top2[t, 1] - BAND:
                        tok = int(gpu["tokens"][b, i])
                toks[(b, s, int(i))] = tok
    assert max_dH <= ENTROPY_TOL, f"readout entropy |d| {max_dH}"
    assert max_dl <= GATE_TOL, f"exit gate |d| {max_dl}"
    return (lambda b, s, i: toks[(b, s, i)]), dict(readout_dH=max_dH, readout_dlam=max_dl, argmax_ties=n_ties)


def step_parity(case, gpu: dict, tau: float, lam: float, K: int, rule: int, block_ids: np.ndarray,
                states=True) -> dict:
    """The three parity checks of one step (see tests/test_gpu_parity.py)."""
    from oracle.alodlm_oracle import replay_decisions
    B = block_ids.shape[0]
    r_by_loop = {s: case.handle.debug_state(2, s).cpu().numpy() for s in range(1, int(gpu["loops_run"].max()) + 1)}
    # (1) readout stage on the GPU's own r
    token_at, stats = readout_stage_check(case, gpu, r_by_loop)
    # (2) every decision re-taken from the GPU's traces by the oracle's rules: exact
    rep = replay_decisions(block_ids, case.m.mask_id, gpu["entropy"], gpu["cum_halt"], token_at, tau, lam, K, rule)
    assert not rep["ambiguous"], rep["ambiguous"]
    np.testing.assert_array_equal(gpu["exit_depth"], rep["exit_depth"])
    np.testing.assert_array_equal(gpu["tokens"], rep["tokens"])
    np.testing.assert_array_equal(gpu["loops_run"], rep["loops_run"])
    # (3) end to end against the float64 oracle taking the GPU's decisions
    of = case.oracle("fp64")
    of.prefill(case.prefix_ids)
    ref = of.denoise_step(block_ids, tau, lam, K, rule, follow=follow_of(gpu), band=np.inf)
    compare_decisions(gpu, ref)
    W = of._global("lm_head")
    worst = dict(state=0.0, logits=0.0, entropy=0.0, entropy_excess=0.0)
    for b in range(B):
        for s in range(1, int(gpu["loops_run"][b]) + 1):
            r_gpu, r_ref = r_by_loop[s][b], ref["r"][b][s - 1]
            keys = ((2, "r"),) if not states else ((0, "h_in"), (1, "h_tilde"), (2, "r"))
            for which, key in keys:
                st = r_gpu if which == 2 else case.handle.debug_state(which, s)[b].cpu().numpy()
                rel = row_rel_err(st, ref[key][b][s - 1])
                worst["state"] = max(worst["state"], float(rel.max()))
                assert rel.max() <= STATE_REL_TOL, (key, b, s, rel.max())
            idx = np.nonzero(~np.isnan(gpu["entropy"][b, s - 1]))[0]
            if len(idx) == 0:
                continue
            z_ref = r_ref[idx] @ W.T
            dz = (r_gpu[idx].astype(np.float64) - r_ref[idx]) @ W.T
            lrel = np.linalg.norm(dz, axis=-1) / np.linalg.norm(z_ref, axis=-1)
            worst["logits"] = max(worst["logits"], float(lrel.max()))
            assert lrel.max() <= STATE_REL_TOL, ("logits", b, s, lrel.max())
            # entropy: |dH| <= 1e-2 + 1.5 * sum_v |dH/dz_v| * max_v |dz_v| (first-order bound
            # from the logit deviation; dH/dz_v = -p_v (log p_v + H))
            logp = z_ref - z_ref.max(-1, keepdims=True)
            logp = logp - np.log(np.exp(logp).sum(-1, keepdims=True))
            p = np.exp(logp)
            Hr = -(p * logp).sum(-1)
            L1 = (p * np.abs(logp + Hr[:, None])).sum(-1)
            dzc = dz - dz.mean(-1, keepdims=True)
            bound = ENTROPY_TOL + 1.5 * L1 * np.abs(dzc).max(-1)
            dH = np.abs(gpu["entropy"][b, s - 1, idx] - ref["entropy"][b, s - 1, idx])
            worst["entropy"] = max(worst["entropy"], float(dH.max()))
            worst["entropy_excess"] = max(worst["entropy_excess"], float((dH - bound).max()))
            assert (dH <= bound).all(), ("entropy", b, s, dH.max(), bound.min())
    disagree = [f for f in ref["followed"] if f["kind"] in ("commit", "halt") and f.get("own") != f.get("taken")]
    stats.update(worst)
    stats["e2e_decisions_differing"] = len(disagree)
    stats["e2e_margins"] = sorted(abs(f["margin"]) for f in disagree)[:5]
    return stats
