"""GPU parity at the Qwen3 shapes and batch sizes the benchmark times, against decisions the
oracle computes itself.

* 1.7B bs 1 and 8B bs 1: the oracle builds the prefix KV cache itself (prefill) and runs the
  whole step; every decision is asserted against the oracle's own except inside the fixed
  end-to-end bands, and states, logits, entropies and halts are held to the fixed tolerances
  (tests/gpu_util.py).  The oracle runs in float32 without bf16 rounding (its "fp64"
  precision at dtype float32) to finish in minutes.
* 8B bs 32 and 8B long context (mixed exit depths 1..12): a seeded subset of two sequences.
  The oracle's step runs from the library's KV cache of those sequences (read from its arena),
  with the same checks; the prefill is checked layer-locally: Prelude layer 0 K/V of sampled
  prefix positions straight from their embeddings, and, with mixed exit depths, every Core
  slot d holds a bit-exact copy of the depth-e_j KV for positions with e_j < d.
* On every case, invariants that hold at any size: exit depths within the loops run, at
  least one commit per sequence under the paper's rule, traces defined exactly on the
  unresolved rows of each loop.
"""
import gc

import numpy as np
import pytest
import torch

from oracle import Oracle
from synth import MODELS, WORKLOADS, make_exit_depths, make_weights, weights_to_numpy
from tests.gpu_util import STATE_REL_TOL, Case, e2e_tolerances, row_rel_err, step_parity
from tests.helpers import oracle_cfg

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

_MODEL = {}


@pytest.fixture(scope="module", autouse=True)
def _release_models():
    yield
    _MODEL.clear()
    gc.collect()
    torch.cuda.empty_cache()


def _weights(model):
    """Device weights (seeded) and their float32 host copy, shared by the tests of one model."""
    if model not in _MODEL:
        _MODEL.clear()
        gc.collect()
        w_dev = make_weights(MODELS[model], seed=0, device="cuda")
        _MODEL[model] = (w_dev, weights_to_numpy(w_dev))
    return _MODEL[model]


def _free(case):
    case.handle.close()
    del case
    gc.collect()
    torch.cuda.empty_cache()


def _invariants(case, gpu):
    ex = gpu["exit_depth"]
    B = ex.shape[0]
    assert (ex >= 0).all() and (ex <= gpu["loops_run"][:, None]).all()
    assert ((ex > 0).sum(1) >= 1).all()
    assert ((gpu["tokens"] >= 0) & (gpu["tokens"] < case.m.vocab)).all()
    for b in range(B):
        L = int(gpu["loops_run"][b])
        assert np.isnan(gpu["entropy"][b, L:]).all()
        for s in range(1, L + 1):  # loop s reads out exactly the positions not committed before s
            unresolved = (ex[b] == 0) | (ex[b] >= s)
            np.testing.assert_array_equal(~np.isnan(gpu["entropy"][b, s - 1]), unresolved)


def _run(name):
    wl = WORKLOADS[name]
    w_dev, w_host = _weights(wl.model)
    case = Case(wl.model, wl.batch, wl.prefix, wl.block, wl.k_max, debug=True, weights=w_dev)
    case._w_host = w_host
    e = make_exit_depths(wl.batch, wl.prefix, wl.k_max, seed=2) if wl.mixed_exit_depths else None
    case.prefill(e)
    tau, lam, rule = wl.taus[len(wl.taus) // 2], wl.lambdas[-1], 0
    gpu = case.step(tau, lam, rule=rule)
    _invariants(case, gpu)
    return wl, case, e, (tau, lam, rule), gpu


@pytest.mark.parametrize("name", ["qwen3-1.7b-bs1", "qwen3-8b-bs1"])
def test_fullsize_end_to_end_with_oracle_prefill(name):
    wl, case, e, (tau, lam, rule), gpu = _run(name)
    of = Oracle(oracle_cfg(case.m, wl.k_max), case.w_host, precision="fp64", dtype=np.float32)
    of.prefill(case.prefix_ids, e)
    ob = Oracle(oracle_cfg(case.m, wl.k_max), case.w_host, precision="bf16", dtype=np.float32)
    stats = step_parity(case, gpu, tau, lam, wl.k_max, rule, case.block_ids, oracle=of, ob=ob)
    # the prefix KV cache against the oracle's own, on the first and the deepest slots.  A slot
    # of Core depth d holds projections of the prefix states after the Prelude and d Core
    # passes, which carry the bf16 drift of that depth: each is held to the state tolerance of
    # loop d (the Prelude's to loop 1's, the Coda's to loop K's; R20)
    m, K = case.m, wl.k_max
    state_tol = e2e_tolerances(wl.model, K)["state"]
    slots = [(("prelude", 0), 0, 1), (("core", 0, 1), m.n_prelude, 1),
             (("core", m.n_core - 1, K), m.n_prelude + K * m.n_core - 1, K),
             (("coda", m.n_coda - 1), m.n_prelude + K * m.n_core + m.n_coda - 1, K)]
    worst_kv = 0.0
    for key, slot, depth in slots:
        for which in (0, 1):
            got = case.handle.kv_slot(which, slot, 0, wl.prefix).float().cpu().numpy()  # [nkv, P, hd]
            ref = of.kv[0][key][which].transpose(1, 0, 2)
            rel = row_rel_err(got, ref)
            worst_kv = max(worst_kv, float(rel.max()))
            assert rel.max() <= state_tol[depth - 1], (key, which, rel.max(), state_tol[depth - 1])
    print(f"{name}: loops {gpu['loops_run'].tolist()} commits {int((gpu['exit_depth'] > 0).sum())} "
          f"kv rel {worst_kv:.2e} {stats}")
    _free(case)


@pytest.mark.parametrize("name", ["qwen3-8b-bs32", "qwen3-8b-long"])
def test_fullsize_sequence_subset_from_library_kv(name):
    wl, case, e, (tau, lam, rule), gpu = _run(name)
    m, P = case.m, wl.prefix
    seqs = sorted(np.random.default_rng(7).choice(wl.batch, size=2, replace=False).tolist())
    of = Oracle(oracle_cfg(m, wl.k_max), case.w_host, precision="fp64", dtype=np.float32)
    of.kv = [case.kv_from_gpu(b) for b in seqs]
    of.prefix_len = P
    ob = Oracle(oracle_cfg(m, wl.k_max), case.w_host, precision="bf16", dtype=np.float32)
    stats = step_parity(case, gpu, tau, lam, wl.k_max, rule, case.block_ids, oracle=of, seqs=seqs, ob=ob)
    of.kv = None
    gc.collect()

    # prefill, layer-locally: Prelude layer 0 K/V from the embeddings of sampled positions
    rng = np.random.default_rng(0)
    b = seqs[0]
    o0 = Oracle(oracle_cfg(m, wl.k_max), case.w_host, precision="bf16", dtype=np.float64)
    pos = np.sort(rng.choice(P, size=16, replace=False))
    emb = case.w_host["embed"][case.prefix_ids[b][pos]].astype(np.float64)
    _, k0, v0 = o0.qkv(o0.layer_weights(0), emb, pos)
    gk = case.handle.kv_slot(0, 0, b, P).float().cpu().numpy()[:, pos].transpose(1, 0, 2)
    gv = case.handle.kv_slot(1, 0, b, P).float().cpu().numpy()[:, pos].transpose(1, 0, 2)
    assert row_rel_err(gk, k0).max() < STATE_REL_TOL and row_rel_err(gv, v0).max() < STATE_REL_TOL

    # mixed exit depths: write-time fallback copies are exact
    if e is not None:
        for c in (0, m.n_core - 1):
            for d in (2, wl.k_max):
                kd = case.handle.kv_slot(0, m.n_prelude + (d - 1) * m.n_core + c, b, P).cpu()
                for dd in range(1, d):
                    sel = torch.tensor(e[b] == dd)
                    if sel.any():
                        ke = case.handle.kv_slot(0, m.n_prelude + (dd - 1) * m.n_core + c, b, P).cpu()
                        assert torch.equal(kd[:, sel], ke[:, sel])
    print(f"{name} seqs {seqs}: loops {gpu['loops_run'][seqs].tolist()} {stats}")
    _free(case)
