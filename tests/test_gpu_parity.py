"""GPU parity: the CUDA library (through the C ABI) against the CPU oracle on the same
seeded inputs.  Three checks per step (tests/gpu_util.py, ``step_parity``):

1. readout stage: the oracle's LM head, entropy, argmax and ExitGate applied to the GPU's
   own readout states r^(s) (kernel precision, r rounded to bf16 as the kernel does) match
   the GPU's traces: entropy within 1e-2 nats, lambda within 1e-3, argmax exact except
   where the top-two logit gap is below 1e-3;
2. decisions: every commit, exit depth, token and halt is re-taken from the GPU's traces by
   the oracle's rules (float32 thresholds) and must match bit-exactly;
3. end to end: the float64 oracle runs the whole step from the same ids and weights and
   takes its own decisions; only where a deciding value lies inside a fixed band around its
   threshold (per loop, three times the oracle's own bf16-vs-float64 spread, written by
   tests/golden/make_oracle_spread.py from the oracle alone, never below 1e-2 nats and 1e-3)
   does it take the GPU's decision.  Tokens, exit depths, loops and row counts must then be
   equal, and states, logits, entropies and halts lie within that loop's fixed tolerance.
   The followed decisions whose own choice differed are counted and printed with margins.
"""
import numpy as np
import pytest
import torch

from synth import WORKLOADS, make_exit_depths, make_block_ids
from tests.gpu_util import Case, row_rel_err, step_parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tiny():
    c = Case("tiny", 1, 48, 16, 4)
    c.prefill()
    return c


@pytest.fixture(scope="module")
def mid():
    c = Case("mid", 3, 75, 20, 5)
    c.prefill()
    return c


def _gemm_ref(A, W):
    return (A.double() @ W.double().T).float()


@pytest.mark.parametrize("M,N,K", [(1, 128, 64), (16, 200, 256), (32, 384, 880), (33, 1376, 256), (100, 512, 320),
                                   (128, 256, 4096), (300, 640, 768), (2048, 512, 1024), (20, 6144, 4096),
                                   (512, 4096, 1024), (2048, 6144, 4096), (1000, 3000, 880),
                                   (832, 6144, 4096), (1536, 4096, 4096), (32, 4096, 2112),
                                   (1000, 6016, 880), (300, 19072, 256), (2048, 24576, 4096),
                                   (64, 4096, 12288), (48, 24576, 4096)])
def test_gemm_tcgen05_against_fp64(M, N, K):
    """The shapes cover every GEMM path: split-K clusters of 2-8 CTAs (few rows; 64-row tiles with
    their three-stage ring split and unsplit), the persistent
    kernel with 128- and 256-wide tiles, and the CTA-pair kernel (256 x 256 tiles; ragged
    edges in M, N and K, and an odd number of 128-row weight tiles, whose last pair half reads
    past the matrix).  K = 2112 (33 k-tiles) cannot be cut into 8 equal non-empty ranges: the
    plan must fall back to 4.  The workspace holds only the status word."""
    import adaptively_looped_masked_b200 as alo
    g = torch.Generator(device="cuda").manual_seed(M * 7 + N)
    A = torch.randn((M, K), device="cuda", generator=g).to(torch.bfloat16)
    W = torch.randn((N, K), device="cuda", generator=g).to(torch.bfloat16)
    ws = torch.zeros(64, dtype=torch.float32, device="cuda")
    C = alo.gemm_bf16(A, W, workspace=ws)
    torch.cuda.synchronize()
    assert int(ws[:1].view(torch.int32).item()) == 0
    ref = _gemm_ref(A, W)
    err = (C - ref).abs().max().item() / ref.abs().max().item()
    assert err < 1e-5, (M, N, K, err)


def _check_prefill_kv(case, oracle, b_list, slots):
    """KV arena slots against the oracle's cache (bf16 values, rows of hd)."""
    m = case.m
    for b in b_list:
        for key, slot in slots:
            for which in (0, 1):
                gpu = case.handle.kv_slot(which, slot, b, case.prefix).float().cpu().numpy()  # [nkv, P, hd]
                ref = oracle.kv[b][key][which].transpose(1, 0, 2)
                rel = row_rel_err(gpu, ref)
                assert rel.max() < 2e-2, (b, key, which, rel.max())


def _slots(case):
    m, K = case.m, case.k_max
    out = [(("prelude", l), l) for l in range(m.n_prelude)]
    out += [(("core", c, d), m.n_prelude + (d - 1) * m.n_core + c) for d in range(1, K + 1) for c in range(m.n_core)]
    out += [(("coda", j), m.n_prelude + K * m.n_core + j) for j in range(m.n_coda)]
    return out


@pytest.mark.parametrize("name", ["tiny", "mid"])
def test_prefill_kv_matches_oracle(name, tiny, mid):
    case = tiny if name == "tiny" else mid
    o = case.oracle("bf16")
    o.prefill(case.prefix_ids)
    _check_prefill_kv(case, o, range(case.batch), _slots(case))


def test_prefill_mixed_exit_depths_fallback():
    case = Case("mid", 2, 75, 20, 5)
    e = make_exit_depths(2, 75, 5, seed=2)
    case.prefill(e)
    o = case.oracle("bf16")
    o.prefill(case.prefix_ids, e)
    _check_prefill_kv(case, o, range(2), _slots(case))
    # write-time fallback: positions with e_j < d hold exactly their depth-e_j KV
    m = case.m
    for b in range(2):
        for c in range(m.n_core):
            for d in range(2, 6):
                kd = case.handle.kv_slot(0, m.n_prelude + (d - 1) * m.n_core + c, b, 75).cpu()
                for dd in range(1, d):
                    sel = torch.tensor(e[b] == dd)
                    ke = case.handle.kv_slot(0, m.n_prelude + (dd - 1) * m.n_core + c, b, 75).cpu()
                    assert torch.equal(kd[:, sel], ke[:, sel])


def _step_parity(case, tau, lam, rule, block_ids=None, k_max=None):
    K = case.k_max if k_max is None else k_max
    blk = case.block_ids if block_ids is None else block_ids
    gpu = case.step(tau, lam, k_max=K, rule=rule, block_ids=blk)
    return step_parity(case, gpu, tau, lam, K, rule, blk)


@pytest.mark.parametrize("tau", [0.1, 0.6, 0.9])
@pytest.mark.parametrize("lam", [0.1, 0.9])
@pytest.mark.parametrize("rule", [0, 1])
def test_step_parity_tiny(tiny, tau, lam, rule):
    print("tiny", tau, lam, rule, _step_parity(tiny, tau, lam, rule))


@pytest.mark.parametrize("tau", [0.1, 0.6, 0.9])
@pytest.mark.parametrize("lam", [0.1, 0.9])
@pytest.mark.parametrize("rule", [0, 1])
def test_step_parity_mid(mid, tau, lam, rule):
    print("mid", tau, lam, rule, _step_parity(mid, tau, lam, rule))


def test_step_edge_cases(mid):
    # k_max below the arena's depth, given (non-mask) ids in the block, a block shorter than max_block
    blk = make_block_ids(mid.m, 3, 20, n_given=4, seed=9)
    _step_parity(mid, 0.6, 0.9, 0, block_ids=blk, k_max=3)
    _step_parity(mid, 0.6, 0.5, 1, block_ids=blk[:, :11].copy(), k_max=2)
    # commits disabled (PAPER): all loops run, one forced commit per sequence
    _step_parity(mid, -1.0, 2.0, 0)
    # everything commits at loop 1
    _step_parity(mid, 1e9, 0.5, 0)
    # a block without any [MASK]: nothing to read out, every sequence stops after loop 1
    full = make_block_ids(mid.m, 3, 20, n_given=20, seed=4)
    gpu = mid.step(0.6, 0.5, rule=0, block_ids=full)
    np.testing.assert_array_equal(gpu["tokens"], full)
    assert (gpu["exit_depth"] == 0).all() and (gpu["loops_run"] == 1).all()
    assert np.isnan(gpu["entropy"]).all()


def test_step_is_deterministic(mid):
    a = mid.step(0.6, 0.9, rule=0)
    b = mid.step(0.6, 0.9, rule=0)
    for k in a:
        np.testing.assert_array_equal(np.nan_to_num(a[k], nan=-7.0), np.nan_to_num(b[k], nan=-7.0))
    r1 = mid.handle.debug_state(2, 1).cpu()
    mid.step(0.6, 0.9, rule=0)
    assert torch.equal(r1, mid.handle.debug_state(2, 1).cpu())


def test_graph_replay_matches_direct_launches(mid):
    """Loops recorded as CUDA graphs and replayed give the same bits as direct launches."""
    mid.handle.set_graphs(True)
    a = mid.step(0.6, 0.9, rule=0)
    a2 = mid.step(0.6, 0.9, rule=0)  # replay of the recorded graphs
    r_graph = mid.handle.debug_state(2, 1).cpu()
    mid.handle.set_graphs(False)
    b = mid.step(0.6, 0.9, rule=0)
    r_direct = mid.handle.debug_state(2, 1).cpu()
    mid.handle.set_graphs(True)
    for k in a:
        np.testing.assert_array_equal(np.nan_to_num(a[k], nan=-7.0), np.nan_to_num(b[k], nan=-7.0))
        np.testing.assert_array_equal(np.nan_to_num(a2[k], nan=-7.0), np.nan_to_num(b[k], nan=-7.0))
    assert torch.equal(r_graph, r_direct)


def test_full_core_model_without_prelude_or_coda():
    case = Case("tiny_fullcore", 1, 48, 16, 3)
    case.prefill()
    _step_parity(case, 0.6, 0.5, 0)
    _step_parity(case, 0.6, 0.5, 1)


def test_state_and_argument_errors():
    import adaptively_looped_masked_b200 as alo
    case = Case("tiny", 2, 48, 16, 4, debug=False)
    blk = torch.tensor(case.block_ids, device="cuda")
    with pytest.raises(alo.AlodlmError) as e:
        case.handle.denoise_step(blk, 0.5, 0.5, 4)
    assert e.value.code == -6  # ESTATE: no prefill
    case.prefill()
    with pytest.raises(alo.AlodlmError) as e:
        case.handle.denoise_step(blk[:1], 0.5, 0.5, 4)
    assert e.value.code == -6  # batch differs
    with pytest.raises(alo.AlodlmError) as e:
        case.handle.denoise_step(blk, 0.5, 0.5, 5)
    assert e.value.code == -1  # k_max above the arena's depth
    with pytest.raises(alo.AlodlmError) as e:
        case.handle.denoise_step(torch.zeros((2, 17), dtype=torch.int32, device="cuda"), 0.5, 0.5, 4)
    assert e.value.code == -1  # N above max_block
    bad = blk.clone()
    bad[0, 0] = 10 ** 6  # token id out of range: flagged by the embedding gather, reported as EDEVICE
    with pytest.raises(alo.AlodlmError) as e:
        case.handle.denoise_step(bad, 0.5, 0.5, 4)
        case.handle.sync()
    assert e.value.code == -4
    case.handle.sync()  # the error word was cleared; the handle stays usable
    out = case.step(0.6, 0.9)
    assert (out["exit_depth"] >= 0).all()


def test_expired_wait_reports_timeout_and_the_next_step_is_unchanged(mid):
    """The error path of every bounded device wait, without a GPU fault: a probe kernel waits on
    an mbarrier that nothing arrives on until the library's wait limit expires.  sync() reports
    ALODLM_ETIMEOUT and clears the error word; the next step on
    the same handle is bit-identical to the one before the timeout and matches the oracle."""
    import time
    import adaptively_looped_masked_b200 as alo
    before = mid.step(0.6, 0.5, rule=0)
    t0 = time.time()
    mid.handle.inject_wait_timeout()
    with pytest.raises(alo.AlodlmError) as e:
        mid.handle.sync()
    assert e.value.code == -5  # ALODLM_ETIMEOUT
    assert time.time() - t0 > 1.0  # the wait ran to its limit
    mid.handle.sync()  # cleared: the handle is usable
    after = mid.step(0.6, 0.5, rule=0)
    for k in before:
        np.testing.assert_array_equal(np.nan_to_num(before[k], nan=-7.0), np.nan_to_num(after[k], nan=-7.0))
    print("after an expired wait", _step_parity(mid, 0.6, 0.5, 0))


def test_memory_limit_gives_enomem():
    import adaptively_looped_masked_b200 as alo
    from synth import MODELS
    from tests.gpu_util import _to_cuda
    from synth import make_weights
    m = MODELS["tiny"]
    w = _to_cuda(make_weights(m))
    with pytest.raises(alo.AlodlmError) as e:
        alo.Handle(m, w, k_max=4, max_batch=1, max_prefix=48, max_block=16, mem_limit_bytes=1 << 20)
    assert e.value.code == -2


@pytest.mark.parametrize("rule", [0, 1])
def test_step_parity_two_query_tiles_per_cta(rule):
    """The Qwen3-8B attention geometry (32 q / 8 kv heads, head_dim 128) with 12 sequences and a
    72-position block: 288 packed query rows per (sequence, KV head), so the step attention runs
    two 128-row query tiles per CTA and, for the third tile, one (attention_pq.cuh); loops whose
    looping sequences no longer fill the SMs fall back to one tile per CTA."""
    wl = WORKLOADS["attn-probe-pq"]
    case = Case(wl.model, wl.batch, wl.prefix, wl.block, wl.k_max)
    case.prefill()
    print("two query tiles per CTA", rule, _step_parity(case, 0.6, 0.5, rule))
    case.handle.close()


def test_step_parity_key_split_over_sixteen_ctas():
    """One sequence of the Qwen3-8B attention geometry (32 q / 8 kv heads, head_dim 128, block
    32) against a 1040-position prefix: 9 key tiles, the last ragged, for each of the 8 query
    tiles.  The step attention then splits the keys over a 16-CTA cluster where the device holds
    eight such clusters at once (one key tile per CTA, seven ranks without keys whose empty
    partials the merge skips), else over 8."""
    case = Case("attn-probe", 1, 1040, 32, 2)
    case.prefill()
    print("16-way key split", _step_parity(case, 0.6, 0.5, 0))
    case.handle.close()


def test_head_dim_64_over_several_tiles():
    """The tiny model (head_dim 64: one 64-wide half per head vector) against a 300-position
    prefix, two sequences.  The causal prefill runs 5 query tiles of 2 x 300 packed rows (the
    last ragged) over up to 3 key tiles, checked slot by slot against the oracle's prefill; the
    step's 316 keys (3 tiles, the last ragged) are split over a 4-CTA cluster whose last rank
    gets no keys, checked under both commit rules."""
    case = Case("tiny", 2, 300, 16, 4)
    case.prefill()
    o = case.oracle("bf16")
    o.prefill(case.prefix_ids)
    _check_prefill_kv(case, o, range(2), _slots(case))
    for rule in (0, 1):
        print("head_dim 64, several tiles", rule, _step_parity(case, 0.6, 0.9, rule))
    case.handle.close()
