"""GPU parity of appending a decoded block to the cached prefix (alodlm_append; digest "Method
steps", Algorithm 1 (5) and "Technical novelty": committed tokens join the sequence, every
position is served at its own loop depth).

* The arena after prefill(P0) + append(N), with mixed exit depths on both parts, matches the
  oracle's prefill + append slot by slot (every slot, every position); for appended positions
  with e_j < d the Core slot d holds a bit-exact copy of their depth-e_j K/V.
* prefill(P0) + append(N) gives the arena of one prefill of the P0 + N positions (up to the
  order of floating-point additions, which depends on how rows are grouped into tiles).
* A denoising step after the append passes the step parity checks against an oracle that
  prefilled and appended the same way.
* Two blocks decoded in a stream -- decode, append the decoded block at its commit depths,
  decode the next block -- match the oracle doing the same (decisions outside the fixed bands
  must be the oracle's own).
"""
import numpy as np
import pytest
import torch

from oracle.alodlm_oracle import decode_block
from synth import MODELS, WORKLOADS, make_block_ids, make_exit_depths
from tests.gpu_util import e2e_bands, STATE_REL_TOL, Case, follow_of, row_rel_err, step_parity

pytestmark = pytest.mark.gpu


def _slots(m, K):
    out = [(("prelude", l), l) for l in range(m.n_prelude)]
    out += [(("core", c, d), m.n_prelude + (d - 1) * m.n_core + c) for d in range(1, K + 1) for c in range(m.n_core)]
    out += [(("coda", j), m.n_prelude + K * m.n_core + j) for j in range(m.n_coda)]
    return out


def _prefill_append(case, P0, e):
    ids = torch.tensor(case.prefix_ids, device="cuda")
    et = torch.tensor(e, device="cuda")
    case.handle.prefill(ids[:, :P0].contiguous(), et[:, :P0].contiguous())
    case.handle.append(ids[:, P0:].contiguous(), et[:, P0:].contiguous())
    case.handle.sync()


def _append_shape(name):
    """(model, batch, P0, N, k_max): the tiny and mid workloads, and "attn-probe": the Qwen3-8B
    attention geometry (32 q / 8 kv heads, head_dim 128) on 300 + 37 positions.  Its causal rows
    run on the tensor-core attention: 32 positions per 128-row query tile, three key tiles (the
    last ragged), rows compacted to the positions that reach depths 2 and 3, and an append that
    starts at position 300, inside a query tile's span of positions."""
    if name == "attn-probe":
        return "attn-probe", 2, 300, 37, 3
    wl = WORKLOADS[name]
    return wl.model, wl.batch, wl.prefix, wl.block, wl.k_max


@pytest.mark.parametrize("name", ["tiny", "mid", "attn-probe"])
def test_append_matches_oracle_and_one_long_prefill(name):
    model, B, P0, N, K = _append_shape(name)
    m = MODELS[model]
    case = Case(model, B, P0 + N, N, K, debug=True)
    e = make_exit_depths(B, P0 + N, K, seed=5)
    _prefill_append(case, P0, e)
    o = case.oracle("bf16")
    o.prefill(case.prefix_ids[:, :P0], e[:, :P0])
    o.append(case.prefix_ids[:, P0:], e[:, P0:])
    assert o.prefix_len == P0 + N
    slots = _slots(m, K)
    got = {}
    for b in range(B):
        for key, slot in slots:
            for which in (0, 1):
                g = case.handle.kv_slot(which, slot, b, P0 + N).float().cpu().numpy()  # [nkv, P, hd]
                got[(b, slot, which)] = g
                rel = row_rel_err(g, o.kv[b][key][which].transpose(1, 0, 2))
                assert rel.max() < STATE_REL_TOL, (b, key, which, rel.max())
        # write-time fallback of the appended positions is a bit-exact copy
        for c in range(m.n_core):
            for d in range(2, K + 1):
                kd = case.handle.kv_slot(0, m.n_prelude + (d - 1) * m.n_core + c, b, P0 + N).cpu()
                for dd in range(1, d):
                    sel = np.zeros(P0 + N, bool)
                    sel[P0:] = e[b, P0:] == dd
                    if sel.any():
                        ke = case.handle.kv_slot(0, m.n_prelude + (dd - 1) * m.n_core + c, b, P0 + N).cpu()
                        assert torch.equal(kd[:, torch.tensor(sel)], ke[:, torch.tensor(sel)])
    # the same arena from one prefill of all P0 + N positions
    case.handle.prefill(torch.tensor(case.prefix_ids, device="cuda"), torch.tensor(e, device="cuda"))
    case.handle.sync()
    worst = 0.0
    for b in range(B):
        for key, slot in slots:
            for which in (0, 1):
                g = case.handle.kv_slot(which, slot, b, P0 + N).float().cpu().numpy()
                worst = max(worst, float(row_rel_err(got[(b, slot, which)], g).max()))
    assert worst < 1e-2, worst
    print(f"{name}: append vs one long prefill, max row rel {worst:.2e}")
    case.handle.close()


@pytest.mark.parametrize("rule", [0, 1])
def test_step_after_append(rule):
    wl = WORKLOADS["mid"]
    m, K, B = MODELS[wl.model], wl.k_max, wl.batch
    P0, N = wl.prefix, wl.block
    case = Case(wl.model, B, P0 + N, N, K, debug=True)
    e = make_exit_depths(B, P0 + N, K, seed=6)
    _prefill_append(case, P0, e)
    gpu = case.step(0.6, 0.5, rule=rule)
    of = case.oracle("fp64")
    of.prefill(case.prefix_ids[:, :P0], e[:, :P0])
    of.append(case.prefix_ids[:, P0:], e[:, P0:])
    print("step after append", rule, step_parity(case, gpu, 0.6, 0.5, K, rule, case.block_ids, oracle=of))
    case.handle.close()


def test_two_blocks_decoded_in_a_stream():
    wl = WORKLOADS["mid"]
    m, K, B = MODELS[wl.model], wl.k_max, wl.batch
    P0, N = wl.prefix, wl.block
    tau, lam, rule = 0.6, 0.5, 0
    case = Case(wl.model, B, P0 + N, N, K, debug=False)
    case.handle.prefill(torch.tensor(case.prefix_ids[:, :P0], device="cuda"))
    of = case.oracle("fp64")
    of.prefill(case.prefix_ids[:, :P0])
    block = make_block_ids(m, B, N)
    for blk_i in range(2):
        dec = case.handle.decode_block(torch.tensor(block, device="cuda"), tau, lam, K, rule)
        case.handle.sync()
        got = {k: (v.cpu().numpy() if torch.is_tensor(v) else v) for k, v in dec.items()}
        # the oracle decodes the same block, following the GPU only inside the fixed bands
        T = got["steps"]
        follow = []
        ids = block.copy()
        for t in range(T):
            # per-step decisions of the GPU, rebuilt from its commit steps and depths
            step_tok = np.where(got["commit_step"] == t + 1, got["tokens"], ids)
            step_ex = np.where(got["commit_step"] == t + 1, got["commit_depth"], 0)
            follow.append(dict(tokens=step_tok, exit_depth=step_ex, loops_run=got["loops"][t]))
            ids = step_tok
        ref = decode_block(of, block, tau, lam, K, rule, follow_steps=follow, band=e2e_bands(m.name, K))
        assert ref["steps"] == T
        for key in ("tokens", "commit_step", "commit_depth", "steps_run"):
            np.testing.assert_array_equal(ref[key], got[key], err_msg=f"block {blk_i} {key}")
        if blk_i == 1:
            break
        # append the decoded block at its commit depths (never-committed / given ids at k_max)
        depth = np.where(got["commit_depth"] > 0, got["commit_depth"], K).astype(np.int32)
        case.handle.append(torch.tensor(got["tokens"], device="cuda"), torch.tensor(depth, device="cuda"))
        case.handle.sync()
        of.append(got["tokens"], depth)
    case.handle.close()
