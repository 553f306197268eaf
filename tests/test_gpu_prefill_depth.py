"""GPU parity of depth-on-demand prefill (digest "Limitations", first weakness: build the cache
only as deep as needed, fill deeper depths when a deep loop first needs them).

* Prefix positions whose exit depths stop short of k_max: only those depths are built, each
  position runs the Core only up to its own exit depth (rows compacted per depth), the slots of
  every depth read back equal to the oracle's (deeper depths served by the deepest built one,
  which is what the fallback rule gives), and a step looping past the built depth matches the
  oracle's step.
* An append whose positions loop deeper than every cached one first extends the cached
  positions to that depth; the arena then equals the oracle's prefill + append.
* An exit depth outside 1..k_max is refused, and the handle stays usable.
"""
import numpy as np
import pytest
import torch

from synth import MODELS, WORKLOADS
from tests.gpu_util import STATE_REL_TOL, Case, row_rel_err, step_parity

pytestmark = pytest.mark.gpu


def _slots(m, K):
    out = [(("prelude", l), l) for l in range(m.n_prelude)]
    out += [(("core", c, d), m.n_prelude + (d - 1) * m.n_core + c) for d in range(1, K + 1) for c in range(m.n_core)]
    out += [(("coda", j), m.n_prelude + K * m.n_core + j) for j in range(m.n_coda)]
    return out


def _check_arena(case, o, n_pos):
    m, K = case.m, case.k_max
    for b in range(case.batch):
        for key, slot in _slots(m, K):
            for which in (0, 1):
                g = case.handle.kv_slot(which, slot, b, n_pos).float().cpu().numpy()
                rel = row_rel_err(g, o.kv[b][key][which].transpose(1, 0, 2))
                assert rel.max() < STATE_REL_TOL, (b, key, which, rel.max())


@pytest.mark.parametrize("rule", [0, 1])
def test_shallow_exit_depths_build_only_what_is_needed(rule):
    wl = WORKLOADS["mid"]
    K = wl.k_max  # 5
    case = Case(wl.model, wl.batch, wl.prefix, wl.block, K, debug=True)
    rng = np.random.default_rng(11)
    e = rng.integers(1, 3, size=(wl.batch, wl.prefix)).astype(np.int32)  # depths 1..2 only
    case.prefill(e)
    o = case.oracle("bf16")
    o.prefill(case.prefix_ids, e)
    _check_arena(case, o, wl.prefix)
    # a step that loops past depth 2 (commits off until the forced one: every loop runs)
    gpu = case.step(-1.0, 2.0, rule=rule)
    assert (gpu["loops_run"] == K).all()
    of = case.oracle("fp64")
    of.prefill(case.prefix_ids, e)
    print("shallow prefix", rule, step_parity(case, gpu, -1.0, 2.0, K, rule, case.block_ids, oracle=of))
    case.handle.close()


def test_append_deeper_than_the_prefix_extends_it():
    wl = WORKLOADS["mid"]
    K, B = wl.k_max, wl.batch
    P0, N = wl.prefix, wl.block
    case = Case(wl.model, B, P0 + N, N, K, debug=False)
    rng = np.random.default_rng(12)
    e0 = rng.integers(1, 3, size=(B, P0)).astype(np.int32)       # prefix: depths 1..2
    e1 = rng.integers(1, K + 1, size=(B, N)).astype(np.int32)    # appended: up to K
    ids = torch.tensor(case.prefix_ids, device="cuda")
    case.handle.prefill(ids[:, :P0].contiguous(), torch.tensor(e0, device="cuda"))
    case.handle.append(ids[:, P0:].contiguous(), torch.tensor(e1, device="cuda"))
    case.handle.sync()
    o = case.oracle("bf16")
    o.prefill(case.prefix_ids[:, :P0], e0)
    o.append(case.prefix_ids[:, P0:], e1)
    _check_arena(case, o, P0 + N)
    case.handle.close()


def test_exit_depth_out_of_range_is_refused():
    import adaptively_looped_masked_b200 as alo
    wl = WORKLOADS["tiny"]
    case = Case(wl.model, 1, wl.prefix, wl.block, wl.k_max, debug=False)
    e = np.full((1, wl.prefix), wl.k_max + 1, np.int32)
    with pytest.raises(alo.AlodlmError) as err:
        case.prefill(e)
    assert err.value.code == -4
    case.prefill()  # the handle stays usable
    case.handle.close()
