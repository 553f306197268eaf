"""GPU parity of sampled commits (alodlm_denoise_step_sampled / alodlm_decode_block_sampled;
digest "Method steps", Algorithm 1 (3): each committed position samples y_i ~ p_i^(s)).

The draw is Gumbel-max with Philox4x64-10 noise under key (seed, step), fused into the LM-head
readout on the GPU and written out plainly in the oracle (gumbel_scores).

* Readout stage: on the GPU's own readout states, every committed token is the oracle's draw
  (argmax of z + g over the same logits) unless the top-two score gap is below 1e-3.
* Decisions re-taken from the GPU's traces, and the float64 oracle end to end taking its own
  draws, exactly as for greedy steps (tests/gpu_util.py).
* The draw depends on the seed and the step index, repeats bit for bit, and at high-entropy
  positions differs from the argmax.
* Block decoding with sampling matches the oracle's decode_block with the same seed.
"""
import numpy as np
import pytest
import torch

from oracle.alodlm_oracle import decode_block
from synth import MODELS, WORKLOADS
from tests.gpu_util import e2e_bands, Case, follow_of, step_parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mid():
    c = Case("mid", 3, 75, 20, 5)
    c.prefill()
    return c


def _sampled(case, tau, lam, rule, key, K=None):
    k = case.k_max if K is None else K
    out = case.handle.denoise_step(torch.tensor(case.block_ids, device="cuda"), tau, lam, k, rule, sample=key)
    case.handle.sync()
    return {kk: v.cpu().numpy() for kk, v in out.items()}


@pytest.mark.parametrize("tau,lam", [(0.6, 0.5), (0.9, 0.1), (1e9, 0.5)])
@pytest.mark.parametrize("rule", [0, 1])
def test_sampled_step_matches_oracle(mid, tau, lam, rule):
    key = (1234, 7)
    gpu = _sampled(mid, tau, lam, rule, key)
    print("sampled", tau, lam, rule, step_parity(mid, gpu, tau, lam, mid.k_max, rule, mid.block_ids, sample_key=key))


def test_sampled_step_tiny():
    case = Case("tiny", 1, 48, 16, 4)
    case.prefill()
    key = (99, 1)
    gpu = _sampled(case, 0.9, 0.5, 0, key)
    print("sampled tiny", step_parity(case, gpu, 0.9, 0.5, 4, 0, case.block_ids, sample_key=key))
    case.handle.close()


def test_draw_depends_on_seed_and_step_and_repeats(mid):
    # tau above every entropy: every position commits at loop 1, so the draw is over full distributions
    greedy = mid.step(1e9, 0.5, rule=0)
    a = _sampled(mid, 1e9, 0.5, 0, (5, 1))
    a2 = _sampled(mid, 1e9, 0.5, 0, (5, 1))
    b = _sampled(mid, 1e9, 0.5, 0, (6, 1))
    c = _sampled(mid, 1e9, 0.5, 0, (5, 2))
    np.testing.assert_array_equal(a["tokens"], a2["tokens"])
    assert (a["tokens"] != b["tokens"]).any() and (a["tokens"] != c["tokens"]).any()
    # the draws differ from the argmax only where the distribution is spread out
    H = greedy["entropy"][:, 0, :]
    diff = a["tokens"] != greedy["tokens"]
    assert diff.any()
    assert H[diff].mean() > H[~diff].mean()


@pytest.mark.parametrize("rule", [0, 1])
def test_sampled_decode_matches_oracle(mid, rule):
    wl = WORKLOADS["mid"]
    K, N = wl.k_max, wl.block
    seed, tau, lam = 31, 0.6, 0.5
    dec = mid.handle.decode_block(torch.tensor(mid.block_ids, device="cuda"), tau, lam, K, rule, sample_seed=seed)
    mid.handle.sync()
    got = {k: (v.cpu().numpy() if torch.is_tensor(v) else v) for k, v in dec.items()}
    T = got["steps"]
    follow, ids = [], mid.block_ids.copy()
    for t in range(T):
        step_tok = np.where(got["commit_step"] == t + 1, got["tokens"], ids)
        step_ex = np.where(got["commit_step"] == t + 1, got["commit_depth"], 0)
        follow.append(dict(tokens=step_tok, exit_depth=step_ex, loops_run=got["loops"][t]))
        ids = step_tok
    of = mid.oracle("fp64")
    of.prefill(mid.prefix_ids)
    ref = decode_block(of, mid.block_ids, tau, lam, K, rule, follow_steps=follow, band=e2e_bands("mid", K),
                       sample_seed=seed)
    assert ref["steps"] == T
    for key in ("tokens", "commit_step", "commit_depth", "steps_run"):
        np.testing.assert_array_equal(ref[key], got[key], err_msg=key)
