"""Pins for the CPU oracle: each check ties the oracle to something other than
itself -- hand-derived fixtures, closed forms, brute force on tiny inputs,
library routines (numpy, torch CPU fp64 SDPA), and invariants -- chosen so
that a dropped term, a wrong sign or index, or a transposed operand fails.

These tests need no GPU.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from block_sparse_long_sparda_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def bits(x):
    """float array -> bf16 bits (values in these tests are bf16-exact)."""
    b = W.f32_to_bf16_bits(np.asarray(x, np.float32))
    assert np.array_equal(W.bf16_bits_to_f32(b), np.asarray(x, np.float32)), "not bf16-exact"
    return b


def closed_form(expr: str) -> float:
    return eval(expr, {"__builtins__": {}}, {"exp": math.exp, "log": math.log, "sqrt": math.sqrt})


# --------------------------------------------------------------------------
# bf16 rounding used by the oracle's compressed-key output
# --------------------------------------------------------------------------

def test_bf16_round_to_nearest_even_pins():
    r = oracle.double_to_bf16
    assert r(1.0) == 0x3F80
    assert r(1.0 + 2.0 ** -7) == 0x3F81            # representable
    assert r(1.0 + 2.0 ** -8) == 0x3F80            # halfway -> even (…0)
    assert r(1.0 + 3 * 2.0 ** -8) == 0x3F82        # halfway -> even (…10)
    assert r(1.0 + 2.0 ** -8 + 2.0 ** -30) == 0x3F81   # just above halfway
    assert r(-(1.0 + 2.0 ** -8)) == 0xBF80
    # one rounding, not two: via binary32 this would first become 1+2^-8 and then 1.0
    assert r(1.0 + 2.0 ** -8 + 2.0 ** -40) == 0x3F81
    assert r(0.0) == 0x0000 and r(-0.0) == 0x8000
    assert oracle.bf16_to_double(0x3F82) == 1.015625


def test_bf16_rounding_matches_torch_on_float32_values():
    rng = np.random.default_rng(7)
    x = (rng.standard_normal(4000) * np.exp(rng.uniform(-20, 20, 4000))).astype(np.float32)
    ours = np.array([oracle.double_to_bf16(float(v)) for v in x], np.uint16)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


# --------------------------------------------------------------------------
# o1 compressed keys
# --------------------------------------------------------------------------

def test_compress_matches_numpy_mean_with_ragged_tail():
    rng = np.random.default_rng(1)
    B, G, T, d, blk = 2, 3, 200, 8, 64                 # 200 = 3*64 + 8: a short last block
    K = W.normal_bf16(rng, (B, G, T, d))
    kc, kcb = oracle.compress_keys(K, blk)
    Kf = W.bf16_bits_to_f32(K).astype(np.float64)
    NB = 4
    assert kc.shape == (B, G, NB, d)
    for j in range(NB):
        ref = Kf[:, :, j * blk:min(T, (j + 1) * blk), :].mean(axis=2)
        np.testing.assert_allclose(kc[:, :, j, :], ref, rtol=0, atol=1e-13)
    # the bf16 output is the fp64 mean rounded once
    for v, bb in zip(kc.reshape(-1)[:500], kcb.reshape(-1)[:500]):
        assert oracle.double_to_bf16(float(v)) == int(bb)


def test_compress_constant_block_is_exact():
    rng = np.random.default_rng(2)
    B, G, T, d, blk = 1, 2, 256, 16, 64
    rows = W.normal_bf16(rng, (B, G, T // blk, d))
    K = np.repeat(rows, blk, axis=2)                    # every row of block j equals rows[j]
    kc, kcb = oracle.compress_keys(K, blk)
    assert np.array_equal(kcb, rows)
    assert np.array_equal(kc, W.bf16_bits_to_f32(rows).astype(np.float64))


def test_compress_linear_ramp_closed_form():
    # K[t] = t (exact in bf16 for t < 256): block j mean = j*blk + (blk-1)/2
    blk, T = 16, 128
    K = np.broadcast_to(np.arange(T, dtype=np.float32)[None, None, :, None], (1, 1, T, 4))
    kc, _ = oracle.compress_keys(bits(K), blk)
    for j in range(T // blk):
        assert np.all(kc[0, 0, j] == j * blk + (blk - 1) / 2)


# --------------------------------------------------------------------------
# o2 selection
# --------------------------------------------------------------------------

def _select_tiny(F_list, kc_rows, k, n_init, n_local, pos, blk, nf=1):
    d = len(kc_rows[0])
    kc = bits(np.asarray(kc_rows, np.float32)).reshape(1, 1, len(kc_rows), d)
    F = bits(np.asarray(F_list, np.float32)).reshape(1, 1, 1, nf, d)
    idx, kth, kth1 = oracle.select(F, kc, k, n_init, n_local, pos, blk)
    return idx[0, 0, 0].tolist(), kth[0, 0, 0], kth1[0, 0, 0]


def test_select_golden_tiny():
    g = load("select_tiny.json")
    for case in g["cases"]:
        got, _, _ = _select_tiny(g["F"], g["kc"], case["k"], g["n_init"], g["n_local"], g["pos"], g["blk"])
        assert got == case["expect"], case


def test_select_golden_positions():
    g = load("select_positions.json")
    kc = [[0.0] * g["d"]] * g["NB"]
    for case in g["cases"]:
        got, _, _ = _select_tiny([0.0] * g["d"], kc, g["k"], g["n_init"], g["n_local"], case["pos"], g["blk"])
        assert got == case["expect"], case


def test_select_golden_multihead_vs_forecast():
    g = load("select_multihead.json")
    got, _, _ = _select_tiny(g["baseline_heads"], g["kc"], g["k"], g["n_init"], g["n_local"], g["pos"],
                             g["blk"], nf=len(g["baseline_heads"]))
    assert got == g["baseline_expect"]
    got, _, _ = _select_tiny([g["forecast"]], g["kc"], g["k"], g["n_init"], g["n_local"], g["pos"], g["blk"])
    assert got == g["forecast_expect"]


def _brute_force_set(scores, k, n_init, n_local, pos, blk, S):
    """Rank counting (no sort): candidate j is taken iff fewer than k candidates
    beat it, where i beats j if s_i > s_j, or s_i == s_j and i < j."""
    c = pos // blk
    window = set(range(max(0, c - n_local + 1), c + 1))
    init = set(j for j in range(n_init) if j <= c) - window
    cands = [j for j in range(c + 1) if j not in window and j not in init and j >= n_init]
    taken = []
    for j in cands:
        beaters = sum(1 for i in cands if scores[i] > scores[j] or (scores[i] == scores[j] and i < j))
        if beaters < k:
            taken.append(j)
    full = sorted(init | window | set(taken))
    return full + [-1] * (S - len(full))


@pytest.mark.parametrize("seed", range(12))
def test_select_brute_force_tiny(seed):
    rng = np.random.default_rng(100 + seed)
    blk, d = 4, 3
    NB = int(rng.integers(1, 16))
    n_init = int(rng.integers(0, 3))
    n_local = int(rng.integers(0, 4))
    k = int(rng.integers(0, 8))
    pos = int(rng.integers(0, NB * blk))
    # small integers so that exact ties are common
    kc = rng.integers(-2, 3, size=(1, 1, NB, d)).astype(np.float32)
    F = rng.integers(-2, 3, size=(1, 1, 1, 1, d)).astype(np.float32)
    idx, _, _ = oracle.select(bits(F), bits(kc), k, n_init, n_local, pos, blk)
    scores = {j: float(np.dot(F[0, 0, 0, 0].astype(np.float64), kc[0, 0, j].astype(np.float64)))
              for j in range(NB)}
    S = k + n_init + n_local
    assert idx[0, 0, 0].tolist() == _brute_force_set(scores, k, n_init, n_local, pos, blk, S)


def test_select_planted_ties_lower_index_wins():
    blk, NB, d = 4, 12, 2
    vals = [0, 5, 1, 5, 5, 2, 5, 0, 3, 0, 0, 0]        # candidates 1..9 at pos 47 (block 11)
    kc = [[v, 0] for v in vals]
    got, kth, kth1 = _select_tiny([[1.0, 0.0]], kc, 3, 1, 2, 47, blk)
    assert got == [0, 1, 3, 4, 10, 11]                 # four blocks score 5: 1,3,4 win, 6 loses
    assert kth == 5.0 and kth1 == 5.0


def test_select_zero_forecast_takes_lowest_candidates():
    rng = np.random.default_rng(3)
    blk, NB, d, k = 64, 40, 128, 7
    kc = W.normal_bf16(rng, (1, 1, NB, d))
    F = np.zeros((1, 1, 1, 1, d), np.uint16)
    idx, _, _ = oracle.select(F, kc, k, 1, 2, NB * blk - 1, blk)
    assert idx[0, 0, 0].tolist() == [0] + list(range(1, 1 + k)) + [NB - 2, NB - 1]


def test_select_k_covering_all_candidates_gives_every_causal_block():
    rng = np.random.default_rng(4)
    blk, NB, d = 64, 20, 128
    kc = W.normal_bf16(rng, (2, 3, NB, d))
    F = W.normal_bf16(rng, (2, 1, 3, 1, d))
    pos = 13 * blk + 5                                   # own block 13
    for k in (11, 12, 30):                               # 11 candidates: [1, 12)
        idx, _, _ = oracle.select(F, kc, k, 1, 2, pos, blk)
        expect = list(range(14)) + [-1] * (k + 3 - 14)
        assert all(idx[b, 0, g].tolist() == expect for b in range(2) for g in range(3))


def test_select_invariants_and_score_order():
    rng = np.random.default_rng(5)
    blk, NB, d, k = 64, 300, 128, 32
    kc = W.normal_bf16(rng, (2, 4, NB, d))
    F = W.normal_bf16(rng, (2, 1, 4, 1, d))
    pos = NB * blk - 1
    idx, kth, kth1 = oracle.select(F, kc, k, 1, 2, pos, blk)
    kcf = W.bf16_bits_to_f32(kc).astype(np.float64)
    Ff = W.bf16_bits_to_f32(F).astype(np.float64)
    for b in range(2):
        for g in range(4):
            s = idx[b, 0, g]
            assert len(s) == k + 3 and np.all(np.diff(s) > 0)
            assert s[0] == 0 and s[-2] == NB - 2 and s[-1] == NB - 1
            scores = kcf[b, g] @ Ff[b, 0, g, 0]
            top = set(s[1:-2].tolist())
            inside = min(scores[j] for j in top)
            outside = max(scores[j] for j in range(1, NB - 2) if j not in top)
            assert inside >= outside
            assert kth[b, 0, g] == pytest.approx(inside, abs=1e-9)
            assert kth1[b, 0, g] == pytest.approx(outside, abs=1e-9)


def test_baseline_with_one_head_is_the_forecast_selector():
    rng = np.random.default_rng(6)
    blk, NB, d, k = 64, 100, 128, 16
    kc = W.normal_bf16(rng, (1, 2, NB, d))
    F = W.normal_bf16(rng, (1, 1, 2, 1, d))
    a, _, _ = oracle.select(F, kc, k, 1, 2, NB * blk - 1, blk)
    # baseline with r identical heads: scores are r times the single-head ones
    Fr = np.repeat(F, 4, axis=3)
    b, _, _ = oracle.select(Fr, kc, k, 1, 2, NB * blk - 1, blk)
    assert np.array_equal(a, b)


def test_baseline_sums_heads_not_averages_one():
    # two heads whose sum points one way while each alone points elsewhere
    g = load("select_multihead.json")
    got, kth, _ = _select_tiny(g["baseline_heads"], g["kc"], 1, 1, 2, 31, 4, nf=2)
    assert got == [0, 3, 6, 7] and kth == 3.0


def test_planted_hot_blocks_recall():
    w = W.scaled(W.WORKLOADS["decode_b4_t32k_planted"], B=1, G=8, Hq=32)
    x = W.decode_inputs(w)
    _, kcb = oracle.compress_keys(x["K"], w.blk)
    idx, _, _ = oracle.select(x["F"].reshape(w.B, 1, w.G, 1, w.d), kcb, w.k, w.n_init, w.n_local,
                              w.T - 1, w.blk)
    recalls = []
    for g in range(w.G):
        hot = set(x["hot"][0, g].tolist())
        recalls.append(len(hot & set(idx[0, 0, g].tolist())) / len(hot))
    assert np.mean(recalls) >= 0.95 and min(recalls) >= 0.8, recalls


# --------------------------------------------------------------------------
# o3 gather
# --------------------------------------------------------------------------

def test_gather_is_fancy_indexing_and_skips_resident():
    rng = np.random.default_rng(8)
    B, G, NB, blk, d = 2, 3, 10, 4, 8
    host = rng.integers(0, 65535, size=(B, G, NB, 2, blk, d), dtype=np.uint16)
    pos = NB * blk - 1
    idx = np.array([[[0, 2, 5, 8, 9], [0, 1, 3, 8, 9], [0, 4, -1, 8, 9]]] * B, np.int32)
    full = oracle.gather_blocks(host, idx, pos, 1, 2, skip_resident=False)
    for b in range(B):
        for g in range(G):
            for s in range(5):
                j = idx[b, g, s]
                if j >= 0:
                    assert np.array_equal(full[b, g, s], host[b, g, j])
                else:
                    assert not full[b, g, s].any()
    part = oracle.gather_blocks(host, idx, pos, 1, 2, skip_resident=True)
    assert not part[:, :, 0].any() and not part[:, :, 3:].any()      # init + local untouched
    assert np.array_equal(part[:, :, 1:2], full[:, :, 1:2])


# --------------------------------------------------------------------------
# o4 / o5 attention
# --------------------------------------------------------------------------

def test_attention_golden_tiny():
    g = load("attention_tiny.json")
    Q = bits(np.asarray(g["q"], np.float32)).reshape(1, 1, 1, 2)
    K = bits(np.asarray(g["K"], np.float32)).reshape(1, 1, 4, 2)
    V = bits(np.asarray(g["V"], np.float32)).reshape(1, 1, 4, 2)
    for case in g["cases"]:
        idx = np.array(case["set"], np.int32).reshape(1, 1, 1, -1)
        O = oracle.sparse_attention(Q, K, V, idx, q_start=case["pos"], T=g["T"], blk=g["blk"],
                                    scale=g["scale"])
        expect = [closed_form(e) for e in case["expect"]]
        np.testing.assert_allclose(O[0, 0, 0], expect, rtol=1e-14, atol=1e-14)


def _sdpa_fp64(Q, K, V, q_start, mask_fn, scale):
    """torch CPU fp64 scaled_dot_product_attention with an explicit mask."""
    B, nq, Hq, d = Q.shape
    G, T = K.shape[1], K.shape[2]
    r = Hq // G
    q = torch.from_numpy(W.bf16_bits_to_f32(Q).astype(np.float64)).permute(0, 2, 1, 3)
    k = torch.from_numpy(W.bf16_bits_to_f32(K).astype(np.float64)).repeat_interleave(r, dim=1)
    v = torch.from_numpy(W.bf16_bits_to_f32(V).astype(np.float64)).repeat_interleave(r, dim=1)
    mask = torch.zeros(B, Hq, nq, T, dtype=torch.bool)
    for b in range(B):
        for h in range(Hq):
            for i in range(nq):
                mask[b, h, i] = torch.from_numpy(mask_fn(b, h // r, i, q_start + i))
    out = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=mask, scale=scale)
    return out.permute(0, 2, 1, 3).numpy()


def test_dense_causal_matches_torch_sdpa_fp64():
    rng = np.random.default_rng(9)
    B, nq, Hq, G, T, d = 2, 5, 4, 2, 150, 16
    Q = W.normal_bf16(rng, (B, nq, Hq, d))
    K = W.normal_bf16(rng, (B, G, T, d))
    V = W.normal_bf16(rng, (B, G, T, d))
    q_start = T - nq
    ours = oracle.dense_causal_attention(Q, K, V, q_start)
    ref = _sdpa_fp64(Q, K, V, q_start, lambda b, g, i, p: np.arange(T) <= p, 1 / math.sqrt(d))
    np.testing.assert_allclose(ours, ref, rtol=1e-12, atol=1e-12)


def test_sparse_with_every_block_is_dense_causal():
    rng = np.random.default_rng(10)
    B, nq, Hq, G, T, d, blk = 1, 6, 8, 2, 300, 32, 64
    Q = W.normal_bf16(rng, (B, nq, Hq, d))
    K = W.normal_bf16(rng, (B, G, T, d))
    V = W.normal_bf16(rng, (B, G, T, d))
    q_start = T - nq
    NB = (T + blk - 1) // blk
    idx = np.broadcast_to(np.arange(NB, dtype=np.int32), (B, nq, G, NB)).copy()
    sparse = oracle.sparse_attention(Q, K, V, idx, q_start, T, blk)
    dense = oracle.dense_causal_attention(Q, K, V, q_start)
    np.testing.assert_allclose(sparse, dense, rtol=1e-12, atol=1e-13)


def test_sparse_matches_block_masked_sdpa_fp64():
    rng = np.random.default_rng(11)
    B, nq, Hq, G, T, d, blk, S = 2, 7, 4, 2, 640, 16, 64, 4
    Q = W.normal_bf16(rng, (B, nq, Hq, d))
    K = W.normal_bf16(rng, (B, G, T, d))
    V = W.normal_bf16(rng, (B, G, T, d))
    q_start = 600
    idx = np.empty((B, nq, G, S), np.int32)
    for b, i, g in itertools.product(range(B), range(nq), range(G)):
        c = (q_start + i) // blk
        idx[b, i, g] = np.sort(rng.choice(c + 1, size=S, replace=False))
    ours = oracle.sparse_attention(Q, K, V, idx, q_start, T, blk)

    def mask(b, g, i, p):
        t = np.arange(T)
        return np.isin(t // blk, idx[b, i, g]) & (t <= p)

    ref = _sdpa_fp64(Q, K, V, q_start, mask, 1 / math.sqrt(d))
    np.testing.assert_allclose(ours, ref, rtol=1e-12, atol=1e-12)


def test_single_block_of_identical_keys_gives_mean_of_values():
    rng = np.random.default_rng(12)
    B, Hq, G, T, d, blk = 1, 2, 1, 256, 8, 64
    Q = W.normal_bf16(rng, (B, 1, Hq, d))
    K = W.normal_bf16(rng, (B, G, T, d))
    K[:, :, 128:192, :] = K[:, :, 128:129, :]           # block 2: 64 identical keys
    V = W.normal_bf16(rng, (B, G, T, d))
    idx = np.array([2], np.int32).reshape(1, 1, 1, 1)
    O = oracle.sparse_attention(Q, K, V, idx, T - 1, T, blk)
    ref = W.bf16_bits_to_f32(V[0, 0, 128:192]).astype(np.float64).mean(axis=0)
    np.testing.assert_allclose(O[0, 0, 0], ref, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(O[0, 0, 1], ref, rtol=1e-13, atol=1e-14)


def test_sparse_ignores_order_padding_and_repeats():
    rng = np.random.default_rng(13)
    B, Hq, G, T, d, blk = 1, 4, 2, 512, 16, 64
    Q = W.normal_bf16(rng, (B, 1, Hq, d))
    K = W.normal_bf16(rng, (B, G, T, d))
    V = W.normal_bf16(rng, (B, G, T, d))
    a = np.array([0, 3, 5, 7], np.int32).reshape(1, 1, 1, 4).repeat(G, axis=2)
    b = np.array([7, -1, 5, 0, 3, 3], np.int32).reshape(1, 1, 1, 6).repeat(G, axis=2)
    Oa = oracle.sparse_attention(Q, K, V, a, T - 1, T, blk)
    Ob = oracle.sparse_attention(Q, K, V, b, T - 1, T, blk)
    np.testing.assert_allclose(Oa, Ob, rtol=1e-13, atol=1e-14)


def test_sparse_interleaved_layout_matches_plain_layout():
    rng = np.random.default_rng(14)
    B, Hq, G, NB, d, blk = 2, 4, 2, 6, 16, 64
    T = NB * blk
    Q = W.normal_bf16(rng, (B, 1, Hq, d))
    K = W.normal_bf16(rng, (B, G, T, d))
    V = W.normal_bf16(rng, (B, G, T, d))
    KV = np.stack([K.reshape(B, G, NB, blk, d), V.reshape(B, G, NB, blk, d)], axis=3)
    idx = np.array([0, 2, 4, 5], np.int32).reshape(1, 1, 1, 4).repeat(B, 0).repeat(G, 2)
    plain = oracle.sparse_attention(Q, K, V, idx, T - 1, T, blk)
    inter = oracle.sparse_attention(Q, KV.reshape(-1), KV.reshape(-1)[blk * d:], idx, T - 1, T, blk,
                                    bg_stride=NB * 2 * blk * d, blk_stride=2 * blk * d, G=G)
    np.testing.assert_allclose(plain, inter, rtol=0, atol=0)


# --------------------------------------------------------------------------
# device slot cache across decode steps (the fetch-only-what-is-new policy)
# --------------------------------------------------------------------------

def test_cache_plan_hand_derived_steps():
    """Five steps of one (b, g) with C = 4 slots, S = 3 entries, NB = 16,
    worked by hand from the policy's definition: hits keep their slot; each
    miss, in list order, takes the clock hand's next slot that holds none of
    the step's blocks."""
    NB = 16
    blk = np.full((1, 1, 4), -1, np.int32)
    hd = np.zeros((1, 1), np.int32)
    steps = [
        # idx            phys          fetch      block_of after      hand
        ([5, 7, 9],      [0, 1, 2],    [1, 1, 1], [5, 7, 9, -1],      3),   # cold start
        ([5, 9, 11],     [0, 2, 3],    [0, 0, 1], [5, 7, 9, 11],      0),   # two hits, hand wraps
        ([2, 5, 12],     [1, 0, 2],    [1, 0, 1], [5, 2, 12, 11],     3),   # hand skips the hit slot 0
        ([-1, 11, 2],    [-1, 3, 1],   [0, 0, 0], [5, 2, 12, 11],     3),   # padding, all hits
        ([20, 3, 4],     [-1, 3, 0],   [0, 1, 1], [4, 2, 12, 3],      1),   # out of range id skipped
    ]
    for ids, ph_want, fe_want, blk_want, hand_want in steps:
        idx = np.array(ids, np.int32).reshape(1, 1, 3)
        phys, fetch, blk, hd = oracle.cache_plan(idx, blk, hd, NB)
        assert phys.reshape(-1).tolist() == ph_want, (ids, phys)
        assert fetch.reshape(-1).tolist() == fe_want, (ids, fetch)
        assert blk.reshape(-1).tolist() == blk_want, (ids, blk)
        assert int(hd[0, 0]) == hand_want


def test_cache_plan_needs_as_many_slots_as_entries():
    with pytest.raises(ValueError):
        oracle.cache_plan(np.zeros((1, 1, 5), np.int32), np.full((1, 1, 4), -1, np.int32),
                          np.zeros((1, 1), np.int32), 16)


def test_cache_plan_invariants_over_drifting_sets():
    """Over many steps of slowly changing sets: every valid entry ends up
    held at its slot, exactly the blocks not held before are fetched, no slot
    holds two blocks, and a block that stays selected never moves."""
    rng = np.random.default_rng(5)
    B, G, S, C, NB = 2, 3, 10, 16, 64
    blk = np.full((B, G, C), -1, np.int32)
    hd = np.zeros((B, G), np.int32)
    cur = np.stack([np.stack([rng.choice(NB, S, replace=False) for _ in range(G)]) for _ in range(B)])
    total_fetch = 0
    for step in range(60):
        # replace a couple of each row's blocks by new ones
        for b in range(B):
            for g in range(G):
                for s in rng.choice(S, 2, replace=False):
                    fresh = [x for x in range(NB) if x not in cur[b, g]]
                    cur[b, g, s] = rng.choice(fresh)
        idx = np.sort(cur, axis=2).astype(np.int32)
        before = blk.copy()
        phys, fetch, blk, hd = oracle.cache_plan(idx, blk, hd, NB)
        for b in range(B):
            for g in range(G):
                held_before = {int(x): c for c, x in enumerate(before[b, g]) if x >= 0}
                row_slots = phys[b, g]
                assert len(set(row_slots.tolist())) == S
                for s in range(S):
                    j = int(idx[b, g, s])
                    assert blk[b, g, row_slots[s]] == j
                    assert fetch[b, g, s] == (0 if j in held_before else 1)
                    if j in held_before:
                        assert row_slots[s] == held_before[j]
                held = blk[b, g][blk[b, g] >= 0]
                assert len(set(held.tolist())) == len(held)
        total_fetch += int(fetch.sum())
        if step > 0:
            assert fetch.sum() <= 2 * B * G  # only the replaced blocks can be new
    assert total_fetch > 0


def test_gather_cached_copies_only_fetched_entries():
    rng = np.random.default_rng(6)
    B, G, NB, S, C, blk, d = 1, 2, 12, 3, 5, 4, 8
    host = rng.integers(0, 65535, (B, G, NB, 2, blk, d), dtype=np.uint16)
    cache = np.zeros((B, G, C, 2, blk, d), np.uint16)
    idx = np.array([[[1, 4, 7], [0, 2, 9]]], np.int32)
    phys = np.array([[[3, 0, 1], [2, 4, 0]]], np.int32)
    fetch = np.array([[[1, 0, 1], [0, 1, 1]]], np.int32)
    out = oracle.gather_cached(host, idx, phys, fetch, cache)
    for g in range(G):
        for s in range(S):
            c = phys[0, g, s]
            if fetch[0, g, s]:
                assert np.array_equal(out[0, g, c], host[0, g, idx[0, g, s]])
    assert not out[0, 0, 0].any() and not out[0, 0, 2].any() and not out[0, 0, 4].any()
    assert not out[0, 1, 1].any() and not out[0, 1, 3].any()


# --------------------------------------------------------------------------
# the window grid of the real models (32-token windows, stride 16) with
# max-pooled block scores
# --------------------------------------------------------------------------

def test_window_counts():
    assert [oracle.window_count(T) for T in (0, 31, 32, 47, 48, 64, 4096)] == [0, 0, 1, 1, 2, 3, 255]


def test_compress_windows_linear_ramp_closed_form():
    """Keys equal to their position (exact in bf16 below 256): window w
    averages positions 16w .. 16w+31, so its mean is 16w + 15.5."""
    T, d = 200, 4
    K = np.empty((1, 1, T, d), np.uint16)
    for t in range(T):
        K[0, 0, t, :] = oracle.double_to_bf16(float(t))
    kw, kwb = oracle.compress_windows(K)
    NW = (T - 32) // 16 + 1
    assert kw.shape == (1, 1, NW, d)
    for w in range(NW):
        assert np.all(kw[0, 0, w] == 16 * w + 15.5)
        assert np.all(kwb[0, 0, w] == oracle.double_to_bf16(16 * w + 15.5))


def _window_keys(values, d=8):
    """kw [1][1][NW][d] whose first coordinate is values[w], the rest zero."""
    kw = np.zeros((1, 1, len(values), d), np.uint16)
    for w, v in enumerate(values):
        kw[0, 0, w, 0] = oracle.double_to_bf16(float(v))
    return kw


def test_select_windows_max_inside_block_not_crossing_windows():
    """F = e_0, so a window's score is its first coordinate.  Block j holds
    windows 4j, 4j+1, 4j+2 (4j+3 straddles blocks j and j+1 and belongs to
    neither).  Block 5 has one high window, block 3 three medium ones, block 6
    only a huge straddling window: the top-2 are {5, 3}, not 6."""
    T = 64 * 12
    NW = oracle.window_count(T)
    vals = [0.0] * NW
    vals[4 * 5 + 1] = 100.0
    for w in (12, 13, 14):
        vals[w] = 10.0
    vals[4 * 6 + 3] = 1000.0          # the window starting at 64*6 + 48
    kw = _window_keys(vals)
    F = np.zeros((1, 1, 1, 1, 8), np.uint16)
    F[..., 0] = oracle.double_to_bf16(1.0)
    idx, kth, kth1 = oracle.select_windows(F, kw, T, k=2, n_init=1, n_local=2, q_start=T - 1)
    assert idx.reshape(-1).tolist() == [0, 3, 5, 10, 11]
    assert kth[0, 0, 0] == 10.0


def test_select_windows_takes_the_max_not_the_mean():
    """Block 2's windows score (9, 0, 0), block 4's (6, 6, 6): with k = 1 the
    max picks block 2 (a mean would pick block 4)."""
    T = 64 * 10
    vals = [0.0] * oracle.window_count(T)
    vals[8] = 9.0
    vals[16] = vals[17] = vals[18] = 6.0
    F = np.zeros((1, 1, 1, 1, 8), np.uint16)
    F[..., 0] = oracle.double_to_bf16(1.0)
    idx, _, _ = oracle.select_windows(F, _window_keys(vals), T, k=1, n_init=1, n_local=2,
                                      q_start=T - 1)
    assert idx.reshape(-1).tolist() == [0, 2, 8, 9]


def test_select_windows_equals_block_selection_when_windows_agree():
    """If the three windows inside every block hold the same key v_j, the
    window selection is the block selection with Kc[j] = v_j."""
    rng = np.random.default_rng(7)
    B, G, nq, d, NB = 2, 3, 2, 16, 40
    T = NB * 64
    NW = oracle.window_count(T)
    kc = rng.integers(0, 65535, (B, G, NB, d), dtype=np.uint16)
    kc = np.where((kc & 0x7F80) == 0x7F80, 0, kc).astype(np.uint16)   # finite values only
    kw = rng.integers(0, 65535, (B, G, NW, d), dtype=np.uint16)
    kw = np.where((kw & 0x7F80) == 0x7F80, 0, kw).astype(np.uint16)
    for j in range(NB):
        for w in (4 * j, 4 * j + 1, 4 * j + 2):
            if w < NW:
                kw[:, :, w] = kc[:, :, j]
    F = W.normal_bf16(rng, (B, nq, G, 1, d))
    a = oracle.select_windows(F, kw, T, k=7, n_init=1, n_local=2, q_start=T - nq)
    b = oracle.select(F, kc, 7, 1, 2, T - nq)
    assert np.array_equal(a[0], b[0])


# --------------------------------------------------------------------------
# the original selector's per-head softmax form ("Training: distilling the
# selector you already have", Eq. 6): S = sum_h softmax(Q_h . Kc^T / tau)
# --------------------------------------------------------------------------

def _two_head_keys(a, b, d=8):
    """Rows r = a[r] e_0 + b[r] e_1; head A queries e_0, head B e_1, so head
    A scores a and head B scores b."""
    R = len(a)
    kc = np.zeros((1, 1, R, d), np.float32)
    kc[0, 0, :, 0] = a
    kc[0, 0, :, 1] = b
    Q = np.zeros((1, 1, 2, d), np.float32)
    Q[0, 0, 0, 0] = 1.0
    Q[0, 0, 1, 1] = 1.0
    return bits(Q), bits(kc)


def test_head_softmax_closed_form_differs_from_summed_scores():
    """Blocks 0..4, init {0}, local {4}, candidates {1, 2, 3}, k = 1, tau = 1.
    Head A scores (0, 10, 9.875, 0, 0): blocks 1 and 2 split its mass.
    Head B scores (0, 0, 0, 3, 0): block 3 keeps most of it.  Each softmax
    runs over all five rows the query sees (the initial and local rows
    included), so Z_A = e^10 + e^9.875 + 3 and Z_B = e^3 + 4, and
      w1 = e^10/Z_A + 1/Z_B = 0.5727,  w2 = e^9.875/Z_A + 1/Z_B = 0.5103,
      w3 = 1/Z_A + e^3/Z_B = 0.8339:
    the per-head softmax keeps block 3, where summed scores (10, 9.875, 3)
    keep block 1."""
    Q, kc = _two_head_keys([0, 10, 9.875, 0, 0], [0, 0, 0, 3, 0])
    T = 64 * 5
    idx, kth, kth1, wb = oracle.select_head_softmax(Q, kc, T, k=1, n_init=1, n_local=1,
                                                    q_start=T - 1, tau=1.0)
    assert idx.reshape(-1).tolist() == [0, 3, 4]
    ZA = "(exp(10) + exp(9.875) + 3)"
    ZB = "(exp(3) + 4)"
    want = [closed_form("1/%s + 1/%s" % (ZA, ZB)),
            closed_form("exp(10)/%s + 1/%s" % (ZA, ZB)),
            closed_form("exp(9.875)/%s + 1/%s" % (ZA, ZB)),
            closed_form("1/%s + exp(3)/%s" % (ZA, ZB)),
            closed_form("1/%s + 1/%s" % (ZA, ZB))]
    np.testing.assert_allclose(wb[0, 0], want, rtol=1e-12)
    assert abs(want[3] - 0.8339) < 1e-4 and abs(want[1] - 0.5727) < 1e-4
    assert kth[0, 0] == wb[0, 0, 3] and kth1[0, 0] == wb[0, 0, 1]
    # summed raw scores rank block 1 first
    F = Q.reshape(1, 1, 1, 2, 8)
    ref, _, _ = oracle.select(F, kc, 1, 1, 1, T - 1)
    assert ref.reshape(-1).tolist() == [0, 1, 4]


def test_head_softmax_mass_is_one_per_head():
    """On the block grid every seen row is a block: the weights of blocks
    0..c sum to the number of heads, and blocks past c weigh -inf."""
    rng = np.random.default_rng(21)
    B, G, nf, d, NB = 2, 3, 4, 32, 30
    T = NB * 64
    kc = W.normal_bf16(rng, (B, G, NB, d))
    Q = W.normal_bf16(rng, (B, G, nf, d))
    q = T - 64 * 5 - 7                       # block c = NB - 6
    _, _, _, wb = oracle.select_head_softmax(Q, kc, T, 4, 1, 2, q, tau=math.sqrt(d))
    c = q // 64
    np.testing.assert_allclose(wb[..., :c + 1].sum(-1), nf, rtol=1e-12)
    assert np.all(wb[..., c + 1:] == -np.inf)
    assert np.all(wb[..., :c + 1] > 0) and np.all(wb[..., :c + 1] < nf)


def test_head_softmax_shift_and_temperature_invariance():
    """A component u shared by every key row shifts head h's scores by
    Q_h . u, a different constant per head, which no softmax sees; scaling the
    queries and tau by 2 together changes nothing either.  Integer entries keep
    every product exact in fp64, so the weights agree to the last bit."""
    rng = np.random.default_rng(22)
    B, G, nf, d, NB = 2, 2, 4, 16, 40
    T = NB * 64
    kc = rng.integers(-3, 4, (B, G, NB, d)).astype(np.float32)
    Q = rng.integers(-3, 4, (B, G, nf, d)).astype(np.float32)
    u = rng.integers(-4, 5, (B, G, 1, d)).astype(np.float32)
    base = oracle.select_head_softmax(bits(Q), bits(kc), T, 6, 1, 2, T - 1, tau=4.0)
    shifted = oracle.select_head_softmax(bits(Q), bits(kc + u), T, 6, 1, 2, T - 1, tau=4.0)
    scaled = oracle.select_head_softmax(bits(2 * Q), bits(kc), T, 6, 1, 2, T - 1, tau=8.0)
    for other in (shifted, scaled):
        assert np.array_equal(base[0], other[0])
        np.testing.assert_allclose(base[3], other[3], rtol=1e-13)
    # tau divides: with tau -> tau / 2 the weights do change
    sharper = oracle.select_head_softmax(bits(Q), bits(kc), T, 6, 1, 2, T - 1, tau=2.0)
    assert not np.allclose(base[3], sharper[3])


def test_head_softmax_head_order_does_not_matter():
    rng = np.random.default_rng(23)
    B, G, nf, d, NB = 1, 2, 4, 32, 50
    T = NB * 64
    kc = W.normal_bf16(rng, (B, G, NB, d))
    Q = W.normal_bf16(rng, (B, G, nf, d))
    a = oracle.select_head_softmax(Q, kc, T, 8, 1, 2, T - 1, tau=math.sqrt(d))
    b = oracle.select_head_softmax(np.ascontiguousarray(Q[:, :, ::-1]), kc, T, 8, 1, 2, T - 1,
                                   tau=math.sqrt(d))
    assert np.array_equal(a[0], b[0])
    np.testing.assert_allclose(a[3], b[3], rtol=1e-12)


@pytest.mark.parametrize("windows", [False, True])
def test_head_softmax_one_head_ranks_as_raw_scores(windows):
    """With one head the weight is an increasing function of the (pooled)
    score, so the set is the raw-score selector's."""
    rng = np.random.default_rng(24)
    B, G, d, NB = 2, 3, 64, 45
    T = NB * 64 - 9
    NR = oracle.window_count(T) if windows else NB
    kc = W.normal_bf16(rng, (B, G, NR, d))
    Q = W.normal_bf16(rng, (B, G, 1, d))
    got = oracle.select_head_softmax(Q, kc, T, 9, 1, 3, T - 1, tau=8.0, windows=windows)[0]
    F = Q.reshape(B, 1, G, 1, d)
    if windows:
        ref = oracle.select_windows(F, kc, T, 9, 1, 3, T - 1)[0]
    else:
        ref = oracle.select(F, kc, 9, 1, 3, T - 1)[0]
    assert np.array_equal(got, ref.reshape(B, G, -1))


@pytest.mark.parametrize("windows", [False, True])
def test_head_softmax_normalises_over_rows_outside_the_candidates(windows):
    """Head A puts a score of 60 on a row that is not a candidate -- the
    initial block (block grid) or a window straddling two blocks (window
    grid, in the normalisation but inside no block) -- so its softmax leaves
    every candidate below e^-50 and head B alone decides: the set is head B's
    raw-score top-k.  Head A's scores on the candidates run opposite to head
    B's, so a softmax over the candidates only would pick other blocks."""
    NB, d = 24, 8
    T = NB * 64
    NR = oracle.window_count(T) if windows else NB
    perm = np.random.default_rng(25).permutation(NR).astype(np.float32)
    b = perm / 4.0                          # distinct, bf16-exact
    a = 10.0 - b / 2.0                      # opposite order
    if windows:
        a[4 * 0 + 3] = 60.0                 # window 3 straddles blocks 0 and 1
    else:
        a[0] = 60.0                         # the initial block
    Q, kc = _two_head_keys(a.tolist(), b.tolist(), d)
    k = 5
    got = oracle.select_head_softmax(Q, kc, T, k, 1, 2, T - 1, tau=1.0, windows=windows)[0]
    Fb = Q[:, :, 1:2].reshape(1, 1, 1, 1, d)
    if windows:
        ref = oracle.select_windows(Fb, kc, T, k, 1, 2, T - 1)[0]
    else:
        ref = oracle.select(Fb, kc, k, 1, 2, T - 1)[0]
    assert np.array_equal(got.reshape(-1), ref.reshape(-1))
    Fa = Q[:, :, 0:1].reshape(1, 1, 1, 1, d)
    other = (oracle.select_windows(Fa, kc, T, k, 1, 2, T - 1) if windows
             else oracle.select(Fa, kc, k, 1, 2, T - 1))[0]
    assert not np.array_equal(got.reshape(-1), other.reshape(-1))
