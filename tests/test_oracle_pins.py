"""Pins of the CPU oracle against what the pages and the mathematics fix.

Every check here compares the oracle with something other than itself: closed forms,
textbook definitions written as brute-force loops, library routines (scipy) for special
cases, structural reductions of the looped model, and counts the pages print.  The
``test_planted_*`` tests plant a plausible mistake in the oracle (on the CPU) and show
that one of the pins catches it.
"""
import math

import numpy as np
import pytest
import scipy.special
import scipy.stats
import torch

import oracle.alodlm_oracle as om
from oracle import Oracle, RULE_PAPER, RULE_PER_TOKEN
from synth import MODELS, make_weights, weights_to_numpy, make_prefix_ids, make_block_ids, make_exit_depths
from tests.helpers import oracle_cfg, small_shape

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def build(shape, k_max, seed=0):
    w = weights_to_numpy(make_weights(shape, seed=seed))
    return Oracle(oracle_cfg(shape, k_max), w), w


# ------------------------------------------------------------------------------------
# brute-force references (textbook definitions, written as loops)
# ------------------------------------------------------------------------------------

def bf_matmul(A, B):
    n, k = A.shape
    k2, m = B.shape
    assert k == k2
    C = np.zeros((n, m))
    for i in range(n):
        for j in range(m):
            acc = 0.0
            for t in range(k):
                acc += A[i, t] * B[t, j]
            C[i, j] = acc
    return C


def bf_rmsnorm(x, g, eps):
    out = np.zeros_like(x)
    for i in range(x.shape[0]):
        ms = sum(v * v for v in x[i]) / x.shape[1]
        out[i] = [x[i, j] / math.sqrt(ms + eps) * g[j] for j in range(x.shape[1])]
    return out


def bf_rope(x, positions, base):
    """Rotate-half RoPE as a complex rotation of the pairs (x_j, x_{j+hd/2})."""
    T, nh, hd = x.shape
    half = hd // 2
    out = np.zeros_like(x)
    for t in range(T):
        for h in range(nh):
            for j in range(half):
                theta = positions[t] * base ** (-2.0 * j / hd)
                zc = complex(x[t, h, j], x[t, h, j + half]) * complex(math.cos(theta), math.sin(theta))
                out[t, h, j] = zc.real
                out[t, h, j + half] = zc.imag
    return out


def bf_attention(q, k, v, visible):
    """Grouped-query attention: KV heads repeated G times in order, then per-head softmax."""
    Tq, nq, hd = q.shape
    G = nq // k.shape[1]
    k_rep = np.repeat(k, G, axis=1)
    v_rep = np.repeat(v, G, axis=1)
    out = np.zeros_like(q)
    for h in range(nq):
        for i in range(Tq):
            scores = [sum(q[i, h, d] * k_rep[j, h, d] for d in range(hd)) / math.sqrt(hd)
                      if visible[i, j] else None for j in range(k.shape[0])]
            mx = max(s for s in scores if s is not None)
            ws = [math.exp(s - mx) if s is not None else 0.0 for s in scores]
            tot = sum(ws)
            for d in range(hd):
                out[i, h, d] = sum(ws[j] * v_rep[j, h, d] for j in range(k.shape[0])) / tot
    return out


def scipy_readout(r, W, exit_w, exit_b):
    z = r @ W.T
    logp = z - scipy.special.logsumexp(z, axis=-1, keepdims=True)
    H = scipy.special.entr(np.exp(logp)).sum(-1)
    return H, np.argmax(z, -1), scipy.special.expit(r @ exit_w + exit_b)


# ------------------------------------------------------------------------------------
# checks (functions, so the planted-mistake tests can call them)
# ------------------------------------------------------------------------------------

def check_primitives(seed=0):
    rng = np.random.default_rng(seed)
    A, B = rng.normal(size=(5, 7)), rng.normal(size=(7, 3))
    np.testing.assert_allclose(A @ B, bf_matmul(A, B), rtol=1e-12, atol=1e-12)
    x, g = rng.normal(size=(4, 9)), rng.normal(size=9)
    np.testing.assert_allclose(om.rmsnorm(x, g, 1e-6), bf_rmsnorm(x, g, 1e-6), rtol=1e-12)
    q = rng.normal(size=(5, 4, 8))
    pos = np.array([0, 1, 7, 100, 5000])
    cos, sin = om.rope_cos_sin(pos, 8, 1e6, np.float64)
    np.testing.assert_allclose(om.apply_rope(q, cos, sin), bf_rope(q, pos, 1e6), rtol=1e-10, atol=1e-12)
    k, v = rng.normal(size=(6, 2, 8)), rng.normal(size=(6, 2, 8))
    vis = rng.random((5, 6)) < 0.7
    vis[:, 0] = True
    np.testing.assert_allclose(om.attention(q, k, v, vis, False), bf_attention(q, k, v, vis),
                               rtol=1e-10, atol=1e-12)
    xs = rng.normal(size=20)
    np.testing.assert_allclose(om.silu(xs), xs * scipy.special.expit(xs), rtol=1e-12)


def check_entropy_closed_forms():
    H, V = 16, 50
    o, _ = build(small_shape(hidden=H, vocab=V), 2)
    rng = np.random.default_rng(1)
    r = rng.normal(size=(3, H))
    # uniform distribution: LM head of zeros -> H = log V, argmax = 0 (lowest index)
    o.W = dict(o.W, lm_head=np.zeros((V, H)))
    o._layer_cache.clear()
    Hs, y, _, _ = o.readout(r)
    np.testing.assert_allclose(Hs, math.log(V), rtol=1e-12)
    assert (y == 0).all()
    # one-hot: a single huge logit -> H = 0 (to e^-big), argmax at that id
    W = np.zeros((V, H))
    W[7] = 400.0 * r[0] / np.dot(r[0], r[0])
    o.W = dict(o.W, lm_head=W)
    o._layer_cache.clear()
    Hs, y, _, _ = o.readout(r[:1])
    assert abs(Hs[0]) < 1e-100 and y[0] == 7
    # two-point distribution (1/4, 3/4) plus zero-probability rest: H = log 4 - 3/4 log 3
    W = np.zeros((V, H))
    u = r[1] / np.dot(r[1], r[1])
    W[:] = -800.0 * u
    W[3] = 0.0 * u
    W[9] = math.log(3.0) * u
    o.W = dict(o.W, lm_head=W)
    o._layer_cache.clear()
    Hs, y, _, _ = o.readout(r[1:2])
    np.testing.assert_allclose(Hs[0], math.log(4) - 0.75 * math.log(3), rtol=1e-12)
    assert y[0] == 9
    # exit gate: lambda = sigmoid(w . r + b)
    o.W = dict(o.W, exit_w=np.eye(H)[2] * 3.0, exit_b=-0.5)
    o._layer_cache.clear()
    _, _, lam, _ = o.readout(r)
    np.testing.assert_allclose(lam, 1.0 / (1.0 + np.exp(-(3.0 * r[:, 2] - 0.5))), rtol=1e-12)


def unrolled_forward(o: Oracle, prefix, block, n_core_reps, with_coda):
    """A plain non-shared transformer over [prefix; block]: Prelude, the Core written out
    n_core_reps times, then (optionally) the Coda and final norm.  Prefix rows are causal,
    block rows see every position.  Returns the block rows' final states."""
    c = o.cfg
    P, N = len(prefix), len(block)
    ids = np.concatenate([prefix, block])
    pos = np.arange(P + N)
    vis = np.zeros((P + N, P + N), dtype=bool)
    vis[:P, :P] = np.tril(np.ones((P, P), dtype=bool))
    vis[P:, :] = True
    layers = list(range(c["n_prelude"]))
    layers += [c["n_prelude"] + j for _ in range(n_core_reps) for j in range(c["n_core"])]
    if with_coda:
        layers += [c["n_prelude"] + c["n_core"] + j for j in range(c["n_coda"])]
    h = o._global("embed")[ids]
    for li in layers:
        lw = o.layer_weights(li)
        q, k, v = o.qkv(lw, h, pos)
        h = o.finish_layer(lw, h, q, k, v, vis)
    if with_coda:
        h = om.rmsnorm(h, o._global("final_norm"), c["rms_eps"])
    return h[P:]


def check_unrolled(shape, K, P=7, N=5):
    """Commits disabled (tau < 0, halting threshold > 1): loop s's Core output equals the
    unrolled stack Prelude + s x Core over [prefix; block]; the last readout equals
    Prelude + K x Core + Coda (the looped-transformer definition, Prerequisites section)."""
    o, _ = build(shape, K)
    prefix = make_prefix_ids(shape, 1, P, seed=5)[0]
    block = make_block_ids(shape, 1, N)[0]
    o.prefill(prefix[None])
    out = o.denoise_step(block[None], tau=-1.0, lam=2.0, k_max=K, rule=RULE_PAPER)
    assert out["loops_run"][0] == K
    for s in range(1, K + 1):
        ref = unrolled_forward(o, prefix, block, s, with_coda=False)
        np.testing.assert_allclose(out["h_tilde"][0][s - 1], ref, rtol=1e-9, atol=1e-12)
    ref = unrolled_forward(o, prefix, block, K, with_coda=True)
    np.testing.assert_allclose(out["r"][0][K - 1], ref, rtol=1e-9, atol=1e-12)
    return o, out


def bf_prefill_states(o: Oracle, prefix, e):
    """Depth-aware prefill position by position: state of position j entering Core layer c at
    depth d, where every key k <= j is read at depth min(d, e_k) (Technical novelty section:
    matching depth, deepest available as fallback).  Memoised recursion."""
    c = o.cfg
    P = len(prefix)
    pos = np.arange(P)
    # Prelude: plain causal stack
    h = o._global("embed")[prefix]
    vis = np.tril(np.ones((P, P), dtype=bool))
    for l in range(c["n_prelude"]):
        lw = o.layer_weights(l)
        q, k, v = o.qkv(lw, h, pos)
        h = o.finish_layer(lw, h, q, k, v, vis)
    prelude_out = h
    memo_in, memo_kv = {}, {}

    def state_in(li, d, j):
        key = (li, d, j)
        if key not in memo_in:
            if li == 0:
                memo_in[key] = prelude_out[j] if d == 1 else state_out(c["n_core"] - 1, d - 1, j)
            else:
                memo_in[key] = state_out(li - 1, d, j)
        return memo_in[key]

    def kv(li, d, j):
        key = (li, d, j)
        if key not in memo_kv:
            lw = o.layer_weights(o.core_layer_index(li))
            q, k, v = o.qkv(lw, state_in(li, d, j)[None], np.array([j]))
            memo_kv[key] = (q[0], k[0], v[0])
        return memo_kv[key]

    memo_out = {}

    def state_out(li, d, j):
        key = (li, d, j)
        if key not in memo_out:
            assert d <= e[j]
            lw = o.layer_weights(o.core_layer_index(li))
            q = kv(li, d, j)[0]
            ks = np.stack([kv(li, min(d, e[t]), t)[1] for t in range(j + 1)])
            vs = np.stack([kv(li, min(d, e[t]), t)[2] for t in range(j + 1)])
            memo_out[key] = o.finish_layer(lw, state_in(li, d, j)[None], q[None], ks, vs,
                                           np.ones((1, j + 1), dtype=bool))[0]
        return memo_out[key]

    return kv, state_out


def check_fallback(shape, K=3, P=6, seed=7):
    o, _ = build(shape, K)
    prefix = make_prefix_ids(shape, 1, P, seed=seed)[0]
    e = make_exit_depths(1, P, K, seed=seed)[0]
    e[0] = K  # at least one position at full depth
    kvc = o.prefill(prefix[None], e[None])[0]
    kv, state_out = bf_prefill_states(o, prefix, e)
    for li in range(shape.n_core):
        for d in range(1, K + 1):
            Kd, Vd = kvc[("core", li, d)]
            for j in range(P):
                kk, vv = kv(li, min(d, e[j]), j)[1:]
                np.testing.assert_allclose(Kd[j], kk, rtol=1e-9, atol=1e-12)
                np.testing.assert_allclose(Vd[j], vv, rtol=1e-9, atol=1e-12)
    # the Coda reads each position's exit-depth state: check its first-layer K
    if shape.n_coda:
        lw = o.layer_weights(o.coda_layer_index(0))
        h_exit = np.stack([state_out(shape.n_core - 1, e[j], j) for j in range(P)])
        _, kref, _ = o.qkv(lw, h_exit, np.arange(P))
        np.testing.assert_allclose(kvc[("coda", 0)][0], kref, rtol=1e-9, atol=1e-12)


# ------------------------------------------------------------------------------------
# pins
# ------------------------------------------------------------------------------------

def test_primitives_against_brute_force():
    check_primitives()


def test_entropy_and_gate_closed_forms():
    check_entropy_closed_forms()


def test_bf16_rounding_is_round_to_nearest_even():
    x = np.array([1.0, 1.0 + 2**-8, 1.0 + 3 * 2**-9, 1.0 + 2**-9, -2.5, 1e-3, 65504.0])
    got = om.round_bf16(x)
    ref = torch.tensor(x, dtype=torch.float32).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(got, ref)


@pytest.mark.parametrize("shape", [small_shape(), small_shape(n_prelude=0, n_coda=0, name="fullcore"),
                                   small_shape(n_q_heads=6, n_kv_heads=2, n_prelude=2, n_core=1, n_coda=2)])
@pytest.mark.parametrize("K", [1, 3])
def test_commit_disabled_step_equals_unrolled_stack(shape, K):
    check_unrolled(shape, K)


def test_k1_is_a_plain_masked_dlm_step():
    """K = 1: one pass of Prelude + Core + Coda; PAPER commits {H <= tau} (or the lowest
    entropy alone), PER_TOKEN commits every masked position with its argmax."""
    shape = small_shape()
    o, w = build(shape, 1)
    prefix = make_prefix_ids(shape, 1, 9, seed=11)[0]
    block = make_block_ids(shape, 1, 6)[0]
    o.prefill(prefix[None])
    r = unrolled_forward(o, prefix, block, 1, with_coda=True)
    H, y, lam = scipy_readout(r, o._global("lm_head"), o._global("exit_w"), w["exit_b"])
    for tau in (float(np.median(H)), -1.0):
        out = o.denoise_step(block[None], tau=tau, lam=0.5, k_max=1, rule=RULE_PAPER)
        np.testing.assert_allclose(out["entropy"][0, 0], H, rtol=1e-9)
        np.testing.assert_allclose(out["halt"][0, 0], lam, rtol=1e-9)
        want = H <= tau
        if not want.any():
            want = np.zeros_like(want)
            want[np.argmin(H)] = True
        np.testing.assert_array_equal(out["exit_depth"][0] == 1, want)
        np.testing.assert_array_equal(out["tokens"][0][want], y[want])
        assert (out["tokens"][0][~want] == shape.mask_id).all()
    out = o.denoise_step(block[None], tau=-1.0, lam=2.0, k_max=1, rule=RULE_PER_TOKEN)
    np.testing.assert_array_equal(out["tokens"][0], y)
    assert (out["exit_depth"][0] == 1).all()


@pytest.mark.parametrize("shape", [small_shape(), small_shape(n_prelude=0, n_coda=0, name="fullcore")])
def test_depth_fallback_against_positionwise_recursion(shape):
    check_fallback(shape)


def test_fallback_special_cases():
    """All e_j = K equals the default prefill; all e_j = 1 equals a K = 1 model's prefill
    with every deeper Core slot holding the depth-1 KV."""
    shape = small_shape()
    K, P = 3, 8
    prefix = make_prefix_ids(shape, 2, P, seed=13)
    o, w = build(shape, K)
    a = o.prefill(prefix)
    b = o.prefill(prefix, np.full((2, P), K))
    for s in range(2):
        for key in a[s]:
            np.testing.assert_array_equal(a[s][key][0], b[s][key][0])
    one = o.prefill(prefix, np.ones((2, P), dtype=int))
    o1 = Oracle(oracle_cfg(shape, 1), w)
    ref = o1.prefill(prefix)
    for s in range(2):
        for key, (kk, vv) in one[s].items():
            rkey = ("core", key[1], 1) if key[0] == "core" else key
            np.testing.assert_allclose(kk, ref[s][rkey][0], rtol=1e-12, atol=1e-14)
            np.testing.assert_allclose(vv, ref[s][rkey][1], rtol=1e-12, atol=1e-14)


def _golden(name):
    import json
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", name)
    return json.load(open(path))


def test_counts_printed_by_the_pages():
    """8B at K = 4 (tests/golden/page_counts.json): L + (K-1) m = 84 KV buffers (Limitations
    section), 10 + 4 x (16 + 10) = 114 layer executions without early exit and 4 x 36 = 144 if
    every layer looped (Technical novelty section)."""
    g = _golden("page_counts.json")
    shape = small_shape(hidden=16, n_q_heads=2, n_kv_heads=1, head_dim=8, inter=16, vocab=20,
                        n_prelude=10, n_core=16, n_coda=10)
    o, _ = build(shape, 4)
    assert o.n_kv_slots() == g["kv_buffers_8b_k4"]["value"]
    o.prefill(make_prefix_ids(shape, 1, 3)[None][0])
    kv = o.kv[0]
    assert len(kv) == g["kv_buffers_8b_k4"]["value"]
    out = o.denoise_step(make_block_ids(shape, 1, 2), tau=-1.0, lam=2.0, k_max=4)
    assert o.layer_execs == g["layer_executions_8b_k4"]["value"]
    assert out["loops_run"][0] == 4
    full = small_shape(hidden=16, n_q_heads=2, n_kv_heads=1, head_dim=8, inter=16, vocab=20,
                       n_prelude=0, n_core=36, n_coda=0)
    of, _ = build(full, 4)
    of.prefill(make_prefix_ids(full, 1, 3)[None][0])
    of.denoise_step(make_block_ids(full, 1, 2), tau=-1.0, lam=2.0, k_max=4)
    assert of.layer_execs == g["layer_executions_full_stack_k4"]["value"]


def test_cumulative_halting_closed_form_and_invariants():
    shape = MODELS["tiny"]
    o, _ = build(shape, 4)
    o.prefill(make_prefix_ids(shape, 1, 48))
    block = make_block_ids(shape, 1, 16, n_given=3)
    out = o.denoise_step(block, tau=-1.0, lam=2.0, k_max=4, rule=RULE_PAPER)
    lam, a = out["halt"][0], out["cum_halt"][0]
    U = block[0] == shape.mask_id
    for s in range(4):
        np.testing.assert_allclose(a[s, U], 1.0 - np.prod(1.0 - lam[: s + 1, U], axis=0), rtol=1e-12)
    assert np.all(np.diff(a[:, U], axis=0) >= 0) and np.all((a[:, U] >= 0) & (a[:, U] < 1))
    assert np.isnan(lam[:, ~U]).all()
    # given (non-mask) ids are kept and never committed
    np.testing.assert_array_equal(out["tokens"][0][~U], block[0][~U])
    assert (out["exit_depth"][0][~U] == 0).all()


@pytest.mark.parametrize("tau", [0.1, 0.6, 0.9])
@pytest.mark.parametrize("lam", [0.1, 0.9])
@pytest.mark.parametrize("rule", [RULE_PAPER, RULE_PER_TOKEN])
def test_step_invariants_tiny(tau, lam, rule):
    shape = MODELS["tiny"]
    o, _ = build(shape, 4)
    o.prefill(make_prefix_ids(shape, 1, 48))
    block = make_block_ids(shape, 1, 16)
    out = o.denoise_step(block, tau=tau, lam=lam, k_max=4, rule=rule)
    ex = out["exit_depth"][0]
    L = out["loops_run"][0]
    assert ex.max() <= L <= 4
    committed = ex > 0
    assert (out["tokens"][0][~committed] == shape.mask_id).all()
    if rule == RULE_PER_TOKEN:
        assert committed.all()
    else:
        assert committed.sum() >= 1
    any_passed = False
    for s in range(L):
        H, a = out["entropy"][0, s], out["cum_halt"][0, s]
        inU = ~np.isnan(H)
        passed = inU & (H <= tau)
        any_passed |= passed.any()
        done_here = ex == s + 1
        if rule == RULE_PAPER:
            if s == L - 1 and not any_passed:
                want = np.zeros_like(done_here)
                want[np.nanargmin(H)] = True
            else:
                want = passed
        else:
            want = inU & (passed | (a >= lam) | (s == 3))
        np.testing.assert_array_equal(done_here, want)


def test_rule_edge_cases():
    shape = MODELS["tiny"]
    o, _ = build(shape, 4)
    o.prefill(make_prefix_ids(shape, 1, 48))
    block = make_block_ids(shape, 1, 16)
    # tau = +inf: everything commits at loop 1
    out = o.denoise_step(block, tau=1e9, lam=0.5, k_max=4, rule=RULE_PAPER)
    assert (out["exit_depth"][0] == 1).all() and out["loops_run"][0] == 1
    # halting threshold 0 (PAPER): the loop stops after one pass
    out = o.denoise_step(block, tau=-1.0, lam=0.0, k_max=4, rule=RULE_PAPER)
    assert out["loops_run"][0] == 1 and (out["exit_depth"][0] > 0).sum() == 1
    # nothing passes tau (PAPER): exactly the lowest-entropy position of the last loop commits
    out = o.denoise_step(block, tau=-1.0, lam=2.0, k_max=4, rule=RULE_PAPER)
    ex = out["exit_depth"][0]
    assert out["loops_run"][0] == 4 and (ex > 0).sum() == 1
    assert np.argmax(ex) == np.nanargmin(out["entropy"][0, 3])
    # PER_TOKEN with threshold 0: a >= 0 always -> all commit at loop 1
    out = o.denoise_step(block, tau=-1.0, lam=0.0, k_max=4, rule=RULE_PER_TOKEN)
    assert (out["exit_depth"][0] == 1).all()


def test_merge_follows_eq3():
    """Eq. 3: entering loop s+1, a committed row holds Emb(y), any other row h~^(s)."""
    shape = MODELS["tiny"]
    o, w = build(shape, 4)
    o.prefill(make_prefix_ids(shape, 1, 48))
    block = make_block_ids(shape, 1, 16, n_given=2)
    H_all = o.denoise_step(block, tau=-1.0, lam=2.0, k_max=4)["entropy"][0]
    tau = float(np.nanquantile(H_all[0], 0.3))
    out = o.denoise_step(block, tau=tau, lam=2.0, k_max=4)
    ex = out["exit_depth"][0]
    assert out["loops_run"][0] >= 2 and ((ex >= 1) & (ex < out["loops_run"][0])).any()
    emb = np.asarray(w["embed"], dtype=np.float64)
    for s in range(1, out["loops_run"][0]):
        com = (ex >= 1) & (ex <= s)
        np.testing.assert_array_equal(out["h_in"][0][s][com], emb[out["tokens"][0][com]])
        np.testing.assert_array_equal(out["h_in"][0][s][~com], out["h_tilde"][0][s - 1][~com])


def test_follow_mode_takes_the_other_decision():
    shape = MODELS["tiny"]
    o, _ = build(shape, 4)
    o.prefill(make_prefix_ids(shape, 1, 48))
    block = make_block_ids(shape, 1, 16)
    base = o.denoise_step(block, tau=0.6, lam=0.5, k_max=4)
    flipped = dict(tokens=base["tokens"].copy(), exit_depth=base["exit_depth"].copy(),
                   loops_run=base["loops_run"].copy())
    out = o.denoise_step(block, tau=0.6, lam=0.5, k_max=4, follow=flipped, band=np.inf)
    np.testing.assert_array_equal(out["tokens"], base["tokens"])
    np.testing.assert_array_equal(out["exit_depth"], base["exit_depth"])
    assert len(out["followed"]) > 0


def test_bf16_precision_is_close_to_fp64():
    shape = MODELS["tiny"]
    w = weights_to_numpy(make_weights(shape))
    ofp = Oracle(oracle_cfg(shape, 4), w)
    obf = Oracle(oracle_cfg(shape, 4), w, precision="bf16")
    prefix = make_prefix_ids(shape, 1, 48)
    block = make_block_ids(shape, 1, 16)
    for o in (ofp, obf):
        o.prefill(prefix)
    a = ofp.denoise_step(block, tau=-1.0, lam=2.0, k_max=4)
    b = obf.denoise_step(block, tau=-1.0, lam=2.0, k_max=4)
    ra, rb = a["r"][0], b["r"][0]
    rel = np.linalg.norm(ra - rb, axis=-1) / np.linalg.norm(ra, axis=-1)
    assert rel.max() < 2e-2
    assert np.nanmax(np.abs(a["entropy"] - b["entropy"])) < 5e-2


# ------------------------------------------------------------------------------------
# planted mistakes: each must make a pin fail
# ------------------------------------------------------------------------------------

def test_planted_rope_sign(monkeypatch):
    good = om.apply_rope

    def bad(x, cos, sin):
        return good(x, cos, -sin)
    monkeypatch.setattr(om, "apply_rope", bad)
    with pytest.raises(AssertionError):
        check_primitives()


def test_planted_gqa_mapping(monkeypatch):
    def bad_attention(q, k, v, visible, bf16):
        Tq, nq, hd = q.shape
        nkv = k.shape[1]
        out = np.zeros_like(q)
        for h in range(nq):
            kh = h % nkv
            s = (q[:, h] @ k[:, kh].T) / math.sqrt(hd)
            s = np.where(visible, s, -np.inf)
            p = np.exp(s - s.max(-1, keepdims=True))
            out[:, h] = (p @ v[:, kh]) / p.sum(-1, keepdims=True)
        return out
    monkeypatch.setattr(om, "attention", bad_attention)
    with pytest.raises(AssertionError):
        check_primitives()


def test_planted_entropy_term(monkeypatch):
    good = om.Oracle.readout

    def bad(self, r):
        H, y, lam, z = good(self, r)
        return H + 0.0 * H - 1e-3 * np.log(z.shape[-1]), y, lam, z
    monkeypatch.setattr(om.Oracle, "readout", bad)
    with pytest.raises(AssertionError):
        check_entropy_closed_forms()


def test_planted_core_depth_off_by_one(monkeypatch):
    good = om.Oracle.block_layer

    def bad(self, b, key, lw, h):
        if key[0] == "core" and key[2] > 1:
            key = ("core", key[1], key[2] - 1)
        return good(self, b, key, lw, h)
    monkeypatch.setattr(om.Oracle, "block_layer", bad)
    with pytest.raises(AssertionError):
        check_unrolled(small_shape(), 3)


def test_planted_fallback_to_shallowest(monkeypatch):
    good = om.Oracle.prefill

    def bad(self, prefix_ids, exit_depth=None):
        kv = good(self, prefix_ids, exit_depth)
        K = self.cfg["k_max"]
        for b in range(len(kv)):
            for j in range(self.cfg["n_core"]):
                for d in range(2, K + 1):
                    kv[b][("core", j, d)] = tuple(x.copy() for x in kv[b][("core", j, 1)])
        return kv
    monkeypatch.setattr(om.Oracle, "prefill", bad)
    with pytest.raises(AssertionError):
        check_fallback(small_shape())


def test_planted_merge_keeps_latent(monkeypatch):
    def bad(self, committed, tok, h_tilde):
        return h_tilde
    monkeypatch.setattr(om.Oracle, "merge", bad)
    with pytest.raises(AssertionError):
        test_merge_follows_eq3()


@pytest.mark.parametrize("rule", [RULE_PAPER, RULE_PER_TOKEN])
def test_replay_of_own_traces_reproduces_decisions(rule):
    """The decision rules re-taken from a run's traces give that run's decisions."""
    shape = MODELS["mid"]
    o, _ = build(shape, 5)
    o.prefill(make_prefix_ids(shape, 3, 30))
    block = make_block_ids(shape, 3, 12, n_given=2)
    for tau, lam in ((0.1, 0.1), (0.6, 0.9), (0.9, 0.5), (-1.0, 2.0)):
        out = o.denoise_step(block, tau, lam, 5, rule)
        rep = om.replay_decisions(block, shape.mask_id, out["entropy"], out["cum_halt"],
                                  lambda b, s, i: int(out["tokens"][b, i]), tau, lam, 5, rule)
        np.testing.assert_array_equal(rep["exit_depth"], out["exit_depth"])
        np.testing.assert_array_equal(rep["tokens"], out["tokens"])
        np.testing.assert_array_equal(rep["loops_run"], out["loops_run"])


# ------------------------------------------------------------------------------------
# decoding a block until no [MASK] is left (Algorithm 1 step (5))
# ------------------------------------------------------------------------------------

def _decoder(n_given=0, B=1, N=12, K=3):
    shape = small_shape()
    o, _ = build(shape, K)
    o.prefill(make_prefix_ids(shape, B, 10))
    return o, shape, make_block_ids(shape, B, N, n_given=n_given)


def test_decode_per_token_finishes_in_one_step():
    """PER_TOKEN commits all of U at s = K: one step decodes the whole block."""
    o, shape, block = _decoder()
    out = om.decode_block(o, block, tau=-1.0, lam=2.0, k_max=3, rule=RULE_PER_TOKEN)
    assert out["steps"] == 1 and (out["tokens"] != shape.mask_id).all()
    assert (out["commit_step"] == 1).all() and (out["commit_depth"] == 3).all()


def test_decode_forced_commits_take_one_position_per_step():
    """PAPER with nothing below tau and no halting: each step commits exactly the forced
    position (lowest entropy of loop K), so a block of N masks takes N steps, each at depth K."""
    o, shape, block = _decoder(N=6)
    out = om.decode_block(o, block, tau=-1.0, lam=2.0, k_max=3, rule=RULE_PAPER)
    assert out["steps"] == 6 and (out["tokens"] != shape.mask_id).all()
    assert sorted(out["commit_step"][0].tolist()) == [1, 2, 3, 4, 5, 6]
    assert (out["commit_depth"] == 3).all() and (out["loops"] == 3).all()
    # the position committed at step t is the lowest-entropy one of that step's last loop
    for t, st in enumerate(out["per_step"], start=1):
        H = st["entropy"][0, 2]
        assert out["commit_step"][0, np.nanargmin(H)] == t


def test_decode_all_below_tau_is_one_loop():
    o, shape, block = _decoder()
    out = om.decode_block(o, block, tau=1e9, lam=0.5, k_max=3, rule=RULE_PAPER)
    assert out["steps"] == 1 and (out["commit_depth"] == 1).all() and (out["loops"] == 1).all()


def test_decode_keeps_given_ids_and_skips_finished_sequences():
    """Given ids are never in U; a sequence without masks counts no step and is unchanged."""
    o, shape, block = _decoder(n_given=4, B=2, N=8)
    block[1] = np.arange(8) % (shape.vocab - 1)  # sequence 1: nothing to decode
    out = om.decode_block(o, block, tau=-1.0, lam=2.0, k_max=3, rule=RULE_PAPER)
    given = block != shape.mask_id
    np.testing.assert_array_equal(out["tokens"][given], block[given])
    assert (out["commit_step"][given] == 0).all()
    assert out["steps_run"][1] == 0 and out["steps_run"][0] == 4 == out["steps"]
    assert (out["tokens"] != shape.mask_id).all()


def test_decode_step_bound():
    o, shape, block = _decoder(N=6)
    out = om.decode_block(o, block, tau=-1.0, lam=2.0, k_max=3, rule=RULE_PAPER, max_steps=2)
    assert out["steps"] == 2 and (out["tokens"] == shape.mask_id).sum() == 4
    assert ((out["commit_step"] > 0) == (out["tokens"] != shape.mask_id)).all()


# ------------------------------------------------------------------------------------
# appending a decoded block to the prefix
# ------------------------------------------------------------------------------------

@pytest.mark.parametrize("shape", [small_shape(), small_shape(n_prelude=0, n_coda=0, name="fullcore")])
def test_append_equals_prefill_of_the_longer_prefix(shape):
    """Prefix attention is causal, so extending a cached prefix by N positions must give the
    KV (every slot, every depth, fallback included) of one prefill over the longer sequence."""
    K = 3
    ids = make_prefix_ids(shape, 2, 14)
    e = make_exit_depths(2, 14, K, seed=5)
    o1, _ = build(shape, K)
    o1.prefill(ids[:, :9], e[:, :9])
    o1.append(ids[:, 9:], e[:, 9:])
    o2, _ = build(shape, K)
    o2.prefill(ids, e)
    assert o1.prefix_len == o2.prefix_len == 14
    for b in range(2):
        assert set(o1.kv[b]) == set(o2.kv[b])
        for key in o2.kv[b]:
            for a1, a2 in zip(o1.kv[b][key], o2.kv[b][key]):
                np.testing.assert_allclose(a1, a2, rtol=1e-11, atol=1e-12)


def test_step_after_append_equals_step_after_full_prefill():
    shape = small_shape()
    K = 3
    ids = make_prefix_ids(shape, 1, 12)
    block = make_block_ids(shape, 1, 6)
    o1, _ = build(shape, K)
    o1.prefill(ids[:, :7])
    o1.append(ids[:, 7:])
    o2, _ = build(shape, K)
    o2.prefill(ids)
    r1 = o1.denoise_step(block, tau=0.6, lam=0.5, k_max=K)
    r2 = o2.denoise_step(block, tau=0.6, lam=0.5, k_max=K)
    np.testing.assert_array_equal(r1["exit_depth"], r2["exit_depth"])
    np.testing.assert_allclose(r1["entropy"], r2["entropy"], rtol=1e-10, equal_nan=True)


# ------------------------------------------------------------------------------------
# sampled commits: Philox4x64-10 and the Gumbel-max draw
# ------------------------------------------------------------------------------------

def test_philox_matches_numpy_bit_generator():
    """numpy's Philox bit generator is Philox4x64-10; it increments its counter before each
    block, so its n-th block of four is the function at counter n + 1."""
    for key in ((1, 2), (0, 0), (0xFFFFFFFFFFFFFFFF, 0x0123456789ABCDEF)):
        bg = np.random.Philox(key=np.array(key, dtype=np.uint64), counter=np.zeros(4, dtype=np.uint64))
        ref = bg.random_raw(4 * 6)
        ctr = np.zeros((6, 4), dtype=np.uint64)
        ctr[:, 0] = np.arange(1, 7, dtype=np.uint64)
        np.testing.assert_array_equal(om.philox4x64(ctr, key).reshape(-1), ref)
    # the higher counter words and a carry into them
    bg = np.random.Philox(key=np.array((7, 9), dtype=np.uint64),
                          counter=np.array((0xFFFFFFFFFFFFFFFF, 3, 5, 0), dtype=np.uint64))
    got = om.philox4x64(np.array([[0, 4, 5, 0]], dtype=np.uint64), (7, 9)).reshape(-1)
    np.testing.assert_array_equal(got, bg.random_raw(4))


def test_gumbel_max_draws_follow_softmax():
    """Gumbel-max: P(argmax_v z_v + g_v = w) = softmax(z)_w.  20000 draws (one per counter
    position) of a 5-entry distribution pass a chi-square test at the 1e-6 level."""
    z = np.array([1.0, 0.2, -0.5, 2.0, 0.0])
    p = np.exp(z - z.max())
    p /= p.sum()
    n = 20000
    counts = np.zeros(5)
    for pos in range(n):
        counts[om.gumbel_argmax(z, (11, 3), pos, 1)] += 1
    chi2 = (((counts - n * p) ** 2) / (n * p)).sum()
    assert chi2 < scipy.stats.chi2.isf(1e-6, df=4), chi2
    # a logit far above the rest is always drawn
    z2 = np.array([0.0, 60.0, 1.0, -3.0])
    assert all(om.gumbel_argmax(z2, (5, 5), pos, 2) == 1 for pos in range(200))


def test_sampled_step_commits_the_same_positions_at_loop_one():
    """Sampling changes which token a committed position gets, not its entropy: at loop 1 the
    entropies and the committed positions equal the greedy step's, and each committed token
    is the Gumbel-max draw of its logits."""
    shape = MODELS["tiny"]
    o, _ = build(shape, 4)
    o.prefill(make_prefix_ids(shape, 1, 48))
    block = make_block_ids(shape, 1, 16)
    g = o.denoise_step(block, tau=0.6, lam=0.9, k_max=4)
    rows = [(0, 1, i) for i in range(16)]
    sm = o.denoise_step(block, tau=0.6, lam=0.9, k_max=4, sample_key=(42, 1), logit_rows=rows)
    np.testing.assert_allclose(sm["entropy"][0, 0], g["entropy"][0, 0], equal_nan=True)
    first = g["exit_depth"][0] == 1
    np.testing.assert_array_equal(sm["exit_depth"][0] == 1, first)
    for i in np.nonzero(first)[0]:
        assert sm["tokens"][0, i] == om.gumbel_argmax(sm["logits"][(0, 1, int(i))], (42, 1), int(i), 1)


# ------------------------------------------------------------------------------------
# the halting criterion on hand-built traces ([digest] "Method steps", Algorithm 1 (3)-(4))
# ------------------------------------------------------------------------------------

def _scripted_step(H, lam_loop, tau, q, K, rule, monkeypatch):
    """Run the oracle's denoise_step with every layer replaced by "row i -> basis vector e_i"
    and the readout by a script: at loop s, position i has entropy H[s-1][i], gate output
    lam_loop[s-1][i] and argmax token 10 + i.  Only the decision logic of the step is left."""
    shape = small_shape()
    o, _ = build(shape, K)
    N = len(H[0])
    o.kv = [{}]
    o.prefix_len = 0
    state = {"s": 0}

    def layer(self, b, key, lw, h):
        if key[0] == "core":
            state["s"] = key[2]
        out = np.zeros_like(h)
        out[np.arange(N), np.arange(N)] = 1.0
        return out

    def readout(self, r):
        pos = np.argmax(r, axis=1)
        s = state["s"]
        z = np.zeros((len(pos), shape.vocab))
        z[np.arange(len(pos)), 10 + pos] = 5.0
        return (np.array([H[s - 1][i] for i in pos], float), 10 + pos,
                np.array([lam_loop[s - 1][i] for i in pos], float), z)

    monkeypatch.setattr(om.Oracle, "block_layer", layer)
    monkeypatch.setattr(om.Oracle, "readout", readout)
    block = np.full((1, N), shape.mask_id, dtype=np.int32)
    return o.denoise_step(block, tau, q, K, rule)


# PAPER, K 4, tau 0.5, q 0.5.  Loop 1 commits position 0 (H 0.1); its a (0.95) must leave the
# mean.  Mean over U after the commits: 0.4, 0.46, 0.568 -> the loop stops at s = 3.  Taken before
# the commits are removed, loop 1's mean is (0.95 + 3 x 0.4) / 4 = 0.5375 -> stop at 1; over all
# masked positions (committed ones kept at their last a), loop 2's is (0.95 + 3 x 0.46) / 4 =
# 0.5825 -> stop at 2.
HALT_H = [[0.1, 5, 5, 5], [9, 5, 5, 5], [9, 5, 5, 5], [9, 5, 5, 5]]
HALT_LAM = [[0.95, 0.4, 0.4, 0.4], [0, 0.1, 0.1, 0.1], [0, 0.2, 0.2, 0.2], [0, 0.5, 0.5, 0.5]]


def check_halting_mean(monkeypatch):
    out = _scripted_step(HALT_H, HALT_LAM, 0.5, 0.5, 4, RULE_PAPER, monkeypatch)
    assert out["loops_run"][0] == 3, out["loops_run"]
    np.testing.assert_array_equal(out["exit_depth"][0], [1, 0, 0, 0])
    np.testing.assert_array_equal(out["tokens"][0][:1], [10])
    np.testing.assert_allclose(out["cum_halt"][0, 2, 1:], 1 - 0.6 * 0.9 * 0.8, rtol=1e-12)
    # the same decisions re-taken from the traces
    rep = om.replay_decisions(np.full((1, 4), small_shape().mask_id), small_shape().mask_id, out["entropy"],
                              out["cum_halt"], lambda b, s, i: 10 + i, 0.5, 0.5, 4, RULE_PAPER)
    assert rep["loops_run"][0] == 3
    np.testing.assert_array_equal(rep["exit_depth"][0], [1, 0, 0, 0])


def test_halting_mean_is_over_u_after_this_loops_commits(monkeypatch):
    check_halting_mean(monkeypatch)


def test_planted_halting_mean_before_commits_are_removed(monkeypatch):
    monkeypatch.setattr(om, "halting_mean", _plant_population("before"))
    with pytest.raises(AssertionError):
        check_halting_mean(monkeypatch)


def test_planted_halting_mean_over_all_masked_positions(monkeypatch):
    monkeypatch.setattr(om, "halting_mean", _plant_population("all"))
    with pytest.raises(AssertionError):
        check_halting_mean(monkeypatch)


def _plant_population(kind):
    """A halting mean over the wrong population, recovered from the oracle's own state: the
    loop's a holds a value for every position the loop read out (U before the commits) and
    keeps the last value of positions committed earlier (all masked positions)."""
    import inspect

    def bad(a, unresolved):
        frame = inspect.currentframe().f_back
        loc = frame.f_locals
        if kind == "before":
            pop = unresolved.copy()
            pop[loc["idx"]] = True          # this loop's readout rows, commits included
        else:
            pop = loc["block_ids"][loc["b"]] == loc["mask_id"]  # every masked position
        return float(np.mean(a[pop])) if pop.any() else 0.0
    return bad


# PER_TOKEN, K 3, tau 0.5, lambda 0.5, no entropy passes tau.  a after loop 1: 0.6 (commits),
# 0.3, 0.1, 0.1; after loop 2: 0.51 (commits), 0.19, 0.55 (commits); loop 3 = K commits the rest.
# A test on the loop's own lambda instead of the cumulative a would commit position 1 at loop 3.
TOK_H = [[5, 5, 5, 5]] * 3
TOK_LAM = [[0.6, 0.3, 0.1, 0.1], [0, 0.3, 0.1, 0.5], [0, 0, 0.1, 0]]


def test_per_token_rule_on_cumulative_halt_at_k3(monkeypatch):
    out = _scripted_step(TOK_H, TOK_LAM, 0.5, 0.5, 3, RULE_PER_TOKEN, monkeypatch)
    np.testing.assert_array_equal(out["exit_depth"][0], [1, 2, 3, 2])
    np.testing.assert_array_equal(out["tokens"][0], [10, 11, 12, 13])
    assert out["loops_run"][0] == 3
    np.testing.assert_allclose(out["cum_halt"][0, 1, [1, 2, 3]], [0.51, 0.19, 0.55], rtol=1e-12)
    rep = om.replay_decisions(np.full((1, 4), small_shape().mask_id), small_shape().mask_id, out["entropy"],
                              out["cum_halt"], lambda b, s, i: 10 + i, 0.5, 0.5, 3, RULE_PER_TOKEN)
    np.testing.assert_array_equal(rep["exit_depth"][0], [1, 2, 3, 2])
