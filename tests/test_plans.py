"""Host-side checks of how the library cuts its launches into CTAs (no GPU needed).

The library exports its work-partition planners as pure functions (alodlm_plan_gemm,
alodlm_plan_gemm_noalloc, alodlm_plan_attention).  A partition that leaves a k-range or a key
range uncovered, covers one twice, gives a split-K cluster an empty rank, or sizes the
allocation-free GEMM's split partials below what its CTAs write would compute a wrong result
or write out of bounds on the GPU; here every partition of a wide sweep of shapes is checked
against those invariants, with the coverage counted key by key and unit by unit.
"""
import itertools

import numpy as np
import pytest

import adaptively_looped_masked_b200 as alo

KT = 64    # k-tile of the linear-layer kernels
BKV = 128  # key tile of the attention kernels
BQ = 128   # query rows per attention tile
SMS = 148


def _cdiv(a, b):
    return -(-a // b)


@pytest.fixture(scope="module", autouse=True)
def _library():
    alo.lib()


def test_gemm_plans_cover_k_once_with_power_of_two_clusters():
    Ms = (1, 7, 16, 20, 32, 33, 48, 64, 65, 100, 128, 129, 256, 300, 1000, 2048, 4096)
    Ns = (64, 128, 200, 880, 1376, 4096, 6144, 12288, 24576, 151936)
    Ks = (64, 192, 256, 880, 2112, 4096, 12288)
    for M, N, K in itertools.product(Ms, Ns, Ks):
        g = alo.plan_gemm(M, N, K)
        assert g["k_tiles"] == _cdiv(K, KT)
        bn = g["bn"]
        assert bn in (32, 64, 128, 256)
        if M <= 128:
            assert bn == min(b for b in (32, 64, 128) if b >= M), (M, bn)
        s, kps = g["splits"], g["kps"]
        assert s in (1, 2, 4, 8), (M, N, K, s)
        # every rank of the cluster gets a non-empty k-range and the ranges cover all k-tiles
        ranges = [(r * kps, min(g["k_tiles"], (r + 1) * kps)) for r in range(s)]
        assert all(b > a for a, b in ranges), (M, N, K, g)
        cover = np.zeros(g["k_tiles"], dtype=int)
        for a, b in ranges:
            cover[a:b] += 1
        assert (cover == 1).all(), (M, N, K, g)
        if s > 1:
            assert kps >= 4, (M, N, K, g)
            tiles = _cdiv(N, 128) * _cdiv(M, bn)
            per_sm = 2 if bn <= 64 else 1
            assert tiles * s <= SMS * per_sm, (M, N, K, g)  # the split grid is one wave


def test_gemm_plan_falls_back_when_equal_ranges_would_leave_a_rank_empty():
    # 33 k-tiles: 8 ranges of 5 would leave the eighth empty, so the cluster shrinks to 4
    g = alo.plan_gemm(32, 4096, 2112)
    assert (g["splits"], g["kps"], g["k_tiles"]) == (4, 9, 33)


@pytest.mark.parametrize("sms", [1, 7, 132, 148])
def test_noalloc_stream_k_units_and_partials(sms):
    for M, N, K in itertools.product((1, 20, 32, 33, 64), (64, 128, 1376, 4096, 6144, 32768),
                                     (64, 880, 4096, 12288, 32768)):
        p = alo.plan_gemm_noalloc(M, N, K, sms)
        assert p["bn"] == (32 if M <= 32 else 64)
        assert p["n_tiles"] == _cdiv(N, 128) and p["k_tiles"] == _cdiv(K, KT)
        total = p["n_tiles"] * p["k_tiles"]
        grid, upc = p["grid"], p["upc"]
        assert 1 <= grid <= sms
        # CTA c walks units [c * upc, (c + 1) * upc): all covered, none twice, no CTA idle
        owner = np.arange(total) // upc
        assert owner.max() == grid - 1
        assert np.bincount(owner, minlength=grid).min() >= 1
        # partials are kept per (weight tile, segment): the most CTAs any tile is split over
        segs = max(len(np.unique(owner[t * p["k_tiles"]:(t + 1) * p["k_tiles"]])) for t in range(p["n_tiles"]))
        assert p["max_seg"] == segs, (M, N, K, sms, p, segs)


def test_noalloc_limits_fit_its_fixed_scratch_on_a_b200():
    """Every shape within the allocation-free GEMM's documented limits (M <= 64, N <= 32768,
    K <= 32768) fits its fixed array on a 148-SM B200: at most 1024 tile counters and at most
    4 Mi floats of split partials (a weight tile's partials are 128 x bn floats per segment)."""
    Ns = sorted(set([1, 128, 129, 1000, 4096, 6144, 12288, 24576, 32640, 32768] + list(range(128, 32769, 1280))))
    Ks = sorted(set([8, 64, 72, 880, 2112, 4096, 12288, 32760, 32768] + list(range(64, 32769, 2048))))
    for M, N, K in itertools.product((1, 32, 33, 64), Ns, Ks):
        p = alo.plan_gemm_noalloc(M, N, K, SMS)
        assert p["n_tiles"] <= 1024
        assert p["n_tiles"] * p["max_seg"] * 128 * p["bn"] <= 4 << 20, (M, N, K, p)


def _key_cover(kv_len, a):
    s, kps = a["splits"], a["keys_per_split"]
    cover = np.zeros(kv_len, dtype=int)
    for r in range(s):
        start = r * kps
        end = kv_len if (a["last_to_end"] and r == s - 1) else min(kv_len, start + kps)
        if end > start:
            cover[start:end] += 1
        if a["last_to_end"] and r == s - 1:
            assert end - start < kps + BKV  # only a remainder shorter than one tile rides along
    return cover


def test_attention_plans_cover_every_key_once():
    kv_lens = sorted(set([1, 2, 31, 32, 33, 64, 127, 128, 129, 255, 256, 257, 316, 500, 1024, 1040, 1056,
                          1072, 2112, 4000, 8224] + list(range(1, 2000, 37))))
    for RP, nkv, n_seq, causal, sms, pq_ok, c16 in itertools.product(
            (8, 32, 96, 128, 129, 288, 600, 4096), (1, 2, 8), (1, 3, 8, 32), (0, 1), (148, 132, 16, 1),
            (0, 1), (0, 1)):
        for kv_len in kv_lens:
            a = alo.plan_attention(RP, nkv, n_seq, kv_len, causal, sms, pq_ok, c16)
            qtiles = _cdiv(RP, BQ)
            assert a["qtiles"] == qtiles
            s, kps = a["splits"], a["keys_per_split"]
            assert kps > 0 and kps % BKV == 0
            assert s >= 1 and s & (s - 1) == 0 and s <= (16 if c16 else 8)
            if causal:
                assert s == 1 and not a["two_tile"]
            if a["two_tile"]:
                assert pq_ok and not causal and qtiles >= 2 and s == 1
                assert 2 * _cdiv(qtiles, 2) * nkv * n_seq >= sms
            if s > 1:
                assert s * qtiles * nkv * n_seq <= sms  # the split grid is one wave
            else:
                assert not a["last_to_end"]
            cover = _key_cover(kv_len, a)
            assert (cover == 1).all(), (RP, nkv, n_seq, kv_len, causal, sms, pq_ok, c16, a)


def test_attention_plans_of_the_documented_geometries():
    # Qwen3-8B bs 1 step: 8 KV heads x one query tile, 1024 + 32 keys: 8 ranks of one tile,
    # the 32-key remainder on the last (16-CTA clusters do not fit there)
    a = alo.plan_attention(128, 8, 1, 1056, 0, SMS, 1, 0)
    assert (a["splits"], a["keys_per_split"], a["last_to_end"], a["two_tile"]) == (8, 128, 1, 0)
    # the same geometry over 1040 + 32 keys where 16-CTA clusters fit: 9 ranks hold one tile each
    a = alo.plan_attention(128, 8, 1, 1072, 0, SMS, 1, 1)
    assert (a["splits"], a["keys_per_split"], a["last_to_end"]) == (16, 128, 0)
    # the tiny model over 300 + 16 keys, two sequences: a 4-CTA cluster whose last rank is empty
    a = alo.plan_attention(32, 2, 2, 316, 0, SMS, 0, 0)
    assert (a["splits"], a["keys_per_split"], a["last_to_end"]) == (4, 128, 0)
    # 12 sequences with 288 packed rows: three query tiles, two per CTA
    a = alo.plan_attention(288, 8, 12, 232, 0, SMS, 1, 0)
    assert (a["qtiles"], a["two_tile"], a["splits"]) == (3, 1, 1)
    # causal prefill rows: one split, every key tile in one range
    a = alo.plan_attention(4 * 1024, 8, 1, 1024, 1, SMS, 1, 1)
    assert (a["qtiles"], a["splits"], a["keys_per_split"]) == (32, 1, 1024)


def test_plans_reject_bad_arguments():
    with pytest.raises(alo.AlodlmError):
        alo.plan_gemm(0, 128, 64)
    with pytest.raises(alo.AlodlmError):
        alo.plan_gemm_noalloc(65, 128, 64, SMS)
    with pytest.raises(alo.AlodlmError):
        alo.plan_attention(128, 8, 1, 0, 0, SMS, 1, 0)
