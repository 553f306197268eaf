"""GPU parity of block decoding (denoising steps until no [MASK] is left, digest "Method
steps", Algorithm 1 (5)).

* The library's alodlm_decode_block equals the same steps taken one by one through the public
  alodlm_denoise_step with the tokens fed back from the host: bit-exact tokens, commit steps
  and depths, loops and row counts.
* Every one of those steps passes the step parity checks against the oracle (readout stage,
  decisions re-taken from the traces, float64 end to end).
* The oracle's decode_block, taking the GPU's decision only where its deciding value lies
  within the fixed end-to-end bands (its own decision everywhere else), composes the same
  steps: same step count, commit steps, depths, tokens and per-sequence step counts.
"""
import numpy as np
import pytest
import torch

from oracle.alodlm_oracle import decode_block
from synth import MODELS, WORKLOADS
from tests.gpu_util import e2e_bands, Case, follow_of, step_parity

pytestmark = pytest.mark.gpu


def _np(d):
    return {k: (v.cpu().numpy() if torch.is_tensor(v) else v) for k, v in d.items()}


# (mid, -1, 0.5) is the pages' conservative quality mode (digest "Results", Table 1): no entropy
# passes tau, so under the paper's rule every step commits exactly its lowest-entropy position
@pytest.mark.parametrize("name,tau,lam", [("tiny", 0.6, 0.5), ("tiny", 0.1, 0.9), ("mid", 0.6, 0.5),
                                          ("mid", -1.0, 0.5)])
@pytest.mark.parametrize("rule", [0, 1])
def test_decode_block_stepwise_and_oracle(name, tau, lam, rule):
    wl = WORKLOADS[name]
    m = MODELS[wl.model]
    K, N = wl.k_max, wl.block
    case = Case(wl.model, wl.batch, wl.prefix, N, K, debug=True)
    case.prefill()
    block = case.block_ids.copy()
    if wl.batch > 1:
        block[1] = np.arange(N) % (m.vocab - 1)  # a sequence with nothing to decode
    dec = _np(case.handle.decode_block(torch.tensor(block, device="cuda"), tau, lam, K, rule))
    case.handle.sync()

    # the same steps through the public step entry point, tokens fed back on the host
    ids, steps = block.copy(), []
    while (ids == m.mask_id).any() and len(steps) < N:
        gpu = case.step(tau, lam, rule=rule, block_ids=ids)
        step_parity(case, gpu, tau, lam, K, rule, ids, states=False)
        steps.append((ids, gpu))
        ids = gpu["tokens"]
    T = len(steps)
    assert dec["steps"] == T and not (ids == m.mask_id).any()
    if tau < 0 and rule == 0:  # quality mode: one commit per sequence per step while it has masks
        for _, g in steps:
            assert ((g["exit_depth"] > 0).sum(axis=1) <= 1).all()
    np.testing.assert_array_equal(dec["tokens"], ids)
    cs = np.zeros_like(block)
    cd = np.zeros_like(block)
    runs = np.zeros(block.shape[0], np.int64)
    for t, (ids_in, g) in enumerate(steps, start=1):
        new = g["exit_depth"] > 0
        cs[new] = t
        cd[new] = g["exit_depth"][new]
        runs[(ids_in == m.mask_id).any(axis=1)] = t
        np.testing.assert_array_equal(dec["loops"][t - 1], g["loops_run"])
        np.testing.assert_array_equal(dec["rows"][t - 1, 0], g["active_rows"])
        np.testing.assert_array_equal(dec["rows"][t - 1, 1], g["readout_rows"])
    assert (dec["loops"][T:] == 0).all()
    np.testing.assert_array_equal(dec["commit_step"], cs)
    np.testing.assert_array_equal(dec["commit_depth"], cd)
    np.testing.assert_array_equal(dec["steps_run"], runs)

    # the oracle composes the same steps, taking the GPU's decisions only inside the fixed bands
    of = case.oracle("fp64")
    of.prefill(case.prefix_ids)
    ref = decode_block(of, block, tau, lam, K, rule, follow_steps=[follow_of(g) for _, g in steps], band=e2e_bands(m.name, K))
    assert ref["steps"] == T
    for key in ("tokens", "commit_step", "commit_depth", "steps_run"):
        np.testing.assert_array_equal(ref[key], dec[key])
    np.testing.assert_array_equal(ref["loops"], dec["loops"][:T])
    case.handle.close()


def test_decode_block_step_bound_and_empty_block():
    wl = WORKLOADS["tiny"]
    m = MODELS[wl.model]
    case = Case(wl.model, wl.batch, wl.prefix, wl.block, wl.k_max, debug=False)
    case.prefill()
    # nothing below tau and no halting: one forced commit per step; a bound of 3 steps
    dec = _np(case.handle.decode_block(torch.tensor(case.block_ids, device="cuda"), -1.0, 2.0, wl.k_max, 0,
                                       max_steps=3))
    case.handle.sync()
    assert dec["steps"] == 3 and (dec["tokens"] == m.mask_id).sum() == wl.block - 3
    assert sorted(dec["commit_step"][dec["commit_step"] > 0].tolist()) == [1, 2, 3]
    assert (dec["commit_depth"][dec["commit_step"] > 0] == wl.k_max).all()
    # a block without masks takes no step and comes back unchanged
    full = (np.arange(wl.block) % (m.vocab - 1)).astype(np.int32)[None, :]
    dec = _np(case.handle.decode_block(torch.tensor(full, device="cuda"), 0.6, 0.5, wl.k_max, 0))
    case.handle.sync()
    assert dec["steps"] == 0 and (dec["tokens"] == full).all() and (dec["commit_step"] == 0).all()
    assert (dec["steps_run"] == 0).all() and (dec["loops"] == 0).all()
    case.handle.close()
