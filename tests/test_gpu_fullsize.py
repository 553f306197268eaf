"""GPU parity at the Qwen3 shapes and batch sizes the benchmark times (1.7B bs 1, 8B bs 1,
8B bs 32, 8B long context with mixed exit depths), on outputs the oracle can compute one by
one and on properties that hold at any size:

* readout stage: sampled readout rows r^(s) (the GPU's own) through the oracle's LM head,
  entropy, argmax and ExitGate in the kernels' precision;
* decisions: the whole step re-taken from the GPU's traces by the oracle's rules (tokens of
  unsampled rows are the GPU's argmax, checked on the sampled rows above);
* one layer: the first Core layer of loop s recomputed by the oracle from the GPU's input to
  it (loop input h^(s-1)) and the GPU's prefix KV of that slot, for one sequence;
* prefill: Prelude layer 0 K/V of sampled prefix positions straight from their embeddings;
  with mixed exit depths, every Core slot d holds a bit-exact copy of the depth-e_j KV for
  positions with e_j < d;
* invariants: exit depths within the loops run, at least one commit per sequence (PAPER),
  traces defined exactly on the unresolved rows.
"""
import gc

import numpy as np
import pytest
import torch

from oracle import Oracle
from oracle.alodlm_oracle import replay_decisions
from synth import MODELS, WORKLOADS, make_exit_depths, weights_to_numpy
from tests.gpu_util import BAND, ENTROPY_TOL, GATE_TOL, STATE_REL_TOL, Case, row_rel_err
from tests.helpers import oracle_cfg

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

CASES = ["qwen3-1.7b-bs1", "qwen3-8b-bs1", "qwen3-8b-bs32", "qwen3-8b-long"]


def _free(case):
    case.handle.close()
    del case
    gc.collect()
    torch.cuda.empty_cache()


@pytest.mark.parametrize("name", CASES)
def test_fullsize_step(name):
    wl = WORKLOADS[name]
    m = MODELS[wl.model]
    tau, lam, rule = wl.taus[len(wl.taus) // 2], wl.lambdas[-1], 0
    case = Case(wl.model, wl.batch, wl.prefix, wl.block, wl.k_max, debug=True)
    e = make_exit_depths(wl.batch, wl.prefix, wl.k_max, seed=2) if wl.mixed_exit_depths else None
    case.prefill(e)
    gpu = case.step(tau, lam, rule=rule)
    B, K, N = gpu["entropy"].shape
    rng = np.random.default_rng(0)

    # ---- invariants ----
    ex = gpu["exit_depth"]
    assert (ex >= 0).all() and (ex <= gpu["loops_run"][:, None]).all()
    assert ((ex > 0).sum(1) >= 1).all()
    assert ((gpu["tokens"] >= 0) & (gpu["tokens"] < m.vocab)).all()
    for b in range(B):
        L = int(gpu["loops_run"][b])
        assert np.isnan(gpu["entropy"][b, L:]).all()
        # loop s reads out exactly the positions not committed before s
        for s in range(1, L + 1):
            unresolved = (ex[b] == 0) | (ex[b] >= s)
            np.testing.assert_array_equal(~np.isnan(gpu["entropy"][b, s - 1]), unresolved)

    # ---- readout stage on sampled rows ----
    w_host = {k: case.w_dev[k] for k in ("embed", "lm_head", "final_norm", "exit_w", "exit_b")}
    w_host["layers"] = []
    glob = weights_to_numpy({**w_host, "layers": []}, layers=[])
    glob["layers"] = {}
    ob = Oracle(oracle_cfg(m, wl.k_max), glob, precision="bf16", dtype=np.float32)
    samples = [(int(b), 1) for b in rng.choice(B, size=min(B, 3), replace=False)]
    samples += [(b, int(gpu["loops_run"][b])) for b, _ in samples if gpu["loops_run"][b] > 1]
    toks = {}
    max_dH = 0.0
    for b, s in samples:
        r = case.handle.debug_state(2, s)[b].cpu().numpy()
        idx = np.nonzero(~np.isnan(gpu["entropy"][b, s - 1]))[0]
        idx = idx[rng.choice(len(idx), size=min(len(idx), 8), replace=False)]
        H, y, lmb, z = ob.readout(r[idx].astype(np.float64))
        dH = np.abs(H - gpu["entropy"][b, s - 1, idx])
        max_dH = max(max_dH, float(dH.max()))
        assert dH.max() <= ENTROPY_TOL, (b, s, dH.max())
        assert np.abs(lmb - gpu["halt"][b, s - 1, idx]).max() <= GATE_TOL
        top2 = np.sort(z, axis=-1)[:, -2:]
        for t, i in enumerate(idx):
            if ex[b, i] == s and top2[t, 1] - top2[t, 0] >= BAND:
                assert gpu["tokens"][b, i] == y[t], (b, s, i)
            toks[(b, s, int(i))] = int(y[t])

    # ---- decisions re-taken from the traces ----
    token_at = lambda b, s, i: toks.get((b, s, i), int(gpu["tokens"][b, i]))  # noqa: E731
    rep = replay_decisions(case.block_ids, m.mask_id, gpu["entropy"], gpu["cum_halt"], token_at, tau, lam, K, rule)
    np.testing.assert_array_equal(rep["exit_depth"], ex)
    np.testing.assert_array_equal(rep["loops_run"], gpu["loops_run"])

    # ---- one Core layer of loop s recomputed from the GPU's input to it ----
    b = samples[0][0]
    s = int(gpu["loops_run"][b])
    li = m.n_prelude
    lw_np = weights_to_numpy({**w_host, "layers": case.w_dev["layers"]}, layers=[li])["layers"][li]
    o1 = Oracle(oracle_cfg(m, wl.k_max), {**glob, "layers": {li: lw_np}}, precision="fp64", dtype=np.float64)
    slot = m.n_prelude + (s - 1) * m.n_core
    P = wl.prefix
    kp = case.handle.kv_slot(0, slot, b, P).float().cpu().numpy().transpose(1, 0, 2)
    vp = case.handle.kv_slot(1, slot, b, P).float().cpu().numpy().transpose(1, 0, 2)
    o1.kv = [None] * B
    o1.kv[b] = {("core", 0, s): (kp.astype(np.float64), vp.astype(np.float64))}
    o1.prefix_len = P
    h_in = case.handle.debug_state(0, s)[b].cpu().numpy().astype(np.float64)
    ref = o1.block_layer(b, ("core", 0, s), o1.layer_weights(li), h_in)
    got = case.handle.debug_state(3, s)[b].cpu().numpy()
    rel = row_rel_err(got, ref)
    assert rel.max() <= STATE_REL_TOL, rel.max()

    # ---- prefill: Prelude layer 0 K/V from the embeddings of sampled positions ----
    if m.n_prelude:
        lw0 = weights_to_numpy({**w_host, "layers": case.w_dev["layers"]}, layers=[0])["layers"][0]
        o0 = Oracle(oracle_cfg(m, wl.k_max), {**glob, "layers": {0: lw0}}, precision="bf16", dtype=np.float64)
        pos = np.sort(rng.choice(P, size=min(P, 16), replace=False))
        emb = case.w_dev["embed"][torch.tensor(case.prefix_ids[b][pos], device="cuda").long()].float().cpu().numpy()
        _, k0, v0 = o0.qkv(o0.layer_weights(0), emb.astype(np.float64), pos)
        gk = case.handle.kv_slot(0, 0, b, P).float().cpu().numpy()[:, pos].transpose(1, 0, 2)
        gv = case.handle.kv_slot(1, 0, b, P).float().cpu().numpy()[:, pos].transpose(1, 0, 2)
        assert row_rel_err(gk, k0).max() < 2e-2 and row_rel_err(gv, v0).max() < 2e-2

    # ---- mixed exit depths: write-time fallback copies are exact ----
    if e is not None:
        for c in (0, m.n_core - 1):
            for d in (2, wl.k_max):
                kd = case.handle.kv_slot(0, m.n_prelude + (d - 1) * m.n_core + c, b, P).cpu()
                for dd in range(1, d):
                    sel = torch.tensor(e[b] == dd)
                    if sel.any():
                        ke = case.handle.kv_slot(0, m.n_prelude + (dd - 1) * m.n_core + c, b, P).cpu()
                        assert torch.equal(kd[:, sel], ke[:, sel])
    print(f"{name}: loops {gpu['loops_run'].tolist()[:8]} commits {int((ex > 0).sum())} "
          f"readout |dH| {max_dH:.2e} core-layer rel {rel.max():.2e}")
    _free(case)
