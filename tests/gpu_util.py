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
        self.handle = alo.Handle(self.m, self.w_dev, k_max=k_max, max_batch=batch, max_prefix=prefix,
                                 max_block=block, debug_dump=debug, stream=stream)
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
    """Tokens, exit depths, loops and the NaN pattern of the traces must match exactly."""
    np.testing.assert_array_equal(gpu["loops_run"], ref["loops_run"])
    np.testing.assert_array_equal(gpu["exit_depth"], ref["exit_depth"])
    np.testing.assert_array_equal(gpu["tokens"], ref["tokens"])
    np.testing.assert_array_equal(np.isnan(gpu["entropy"]), np.isnan(ref["entropy"]))
    np.testing.assert_array_equal(gpu["active_rows"], ref["active_rows"])
    np.testing.assert_array_equal(gpu["readout_rows"], ref["readout_rows"])


def compare_values(gpu: dict, ref: dict):
    ok = ~np.isnan(ref["entropy"])
    dH = np.abs(gpu["entropy"][ok] - ref["entropy"][ok])
    assert dH.max(initial=0.0) <= ENTROPY_TOL, f"entropy max |d| {dH.max()}"
    for key in ("halt", "cum_halt"):
        d = np.abs(gpu[key][ok] - ref[key][ok])
        assert d.max(initial=0.0) <= GATE_TOL, f"{key} max |d| {d.max()}"
    return float(dH.max(initial=0.0))


def row_rel_err(a: np.ndarray, ref: np.ndarray) -> np.ndarray:
    return np.linalg.norm(a - ref, axis=-1) / np.maximum(np.linalg.norm(ref, axis=-1), 1e-30)
