"""Pins for the oracle's indexer (score, Top-K, block maxima, pool, Reindex) and attention.

Sources: "DeepSeek V4.1 Flash 拆解" (austincafe.tech), section 一 -- Full mode computes its own
indexer and emits a Top-K; the first decoder layer's Top-512 is followed by a pool of 2048 blocks
x 8 positions that later layers score (Reindex, with their own indexer query); Reuse layers run
sparse attention directly over reused indices; the SWA KV is FP8.

Pins: closed forms (one-hot queries, plain dot products), brute-force sorting with Python's
``sorted`` on tiny inputs, the hand-worked example in golden/topk_example.txt, the invariant that
the pool contains the Top-K, the reduction of attention to dense softmax attention (torch
``scaled_dot_product_attention`` / ``logsumexp`` in float64) when every entry is selected, and the
softmax sum and constant-value properties.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bits(t):
    return t.to(torch.bfloat16).contiguous().view(torch.int16).numpy().view(np.uint16)


# ------------------------------------------------------------------------------------------ score

def test_score_one_hot_closed_form():
    """iq_h = a_h * e_{i_h}: the score is sum_h w_h * max(0, a_h * k[i_h])."""
    iq = torch.zeros(4, 64)
    cols, a = [3, 17, 40, 63], [2.0, -1.0, 0.5, 4.0]
    for h in range(4):
        iq[h, cols[h]] = a[h]
    w = np.array([1.0, 2.0, 3.0, 0.25], np.float32)
    k = torch.zeros(5, 64)
    k[0, [3, 17, 40, 63]] = torch.tensor([1.0, 1.0, 1.0, 1.0])
    k[1, [3, 17, 40, 63]] = torch.tensor([-1.0, -3.0, 2.0, 0.0])
    k[2, 5] = 7.0  # touches no query column -> 0
    k[3, [3, 17, 40, 63]] = torch.tensor([-1.0, 1.0, -1.0, -1.0])  # every dot <= 0 -> 0
    k[4, [3, 63]] = torch.tensor([0.5, 2.0])
    got = oracle.index_scores(bits(iq), w, bits(k))
    want = [1 * 2 + 3 * 0.5 + 0.25 * 4,
            2 * 3 + 3 * 1.0,
            0.0,
            0.0,
            1 * 1 + 0.25 * 8]
    assert list(got) == want


def test_score_reduces_to_plain_dot_product():
    """w = e_h and a positive query/key pair (ReLU inactive): the score is q_h . k (numpy dot)."""
    rng = np.random.default_rng(0)
    for h in range(4):
        iq = torch.from_numpy(rng.uniform(0.1, 1, (4, 64)).astype(np.float32))
        k = torch.from_numpy(rng.uniform(0.1, 1, (8, 64)).astype(np.float32))
        w = np.zeros(4, np.float32)
        w[h] = 1.0
        got = oracle.index_scores(bits(iq), w, bits(k))
        qf = iq.to(torch.bfloat16).double().numpy()[h]
        kf = k.to(torch.bfloat16).double().numpy()
        assert np.allclose(got, kf @ qf, rtol=1e-15, atol=0)


def test_score_positive_homogeneity_and_sign():
    torch.manual_seed(1)
    iq, k = torch.randn(4, 64), torch.randn(6, 64)
    w = np.array([0.7, 1.1, 0.9, 1.3], np.float32)
    s1 = oracle.index_scores(bits(iq), w, bits(k))
    s2 = oracle.index_scores(bits(iq), w, bits(2 * k.to(torch.bfloat16).float()))
    assert np.array_equal(2 * s1, s2)  # scaling by 2 is exact
    sn = oracle.index_scores(bits(iq), w, bits(-k.to(torch.bfloat16).float()))
    # ReLU(d) + ReLU(-d) = |d|: the two halves add up to sum_h w_h |q_h . k|
    dots = k.to(torch.bfloat16).double().numpy() @ iq.to(torch.bfloat16).double().numpy().T
    assert np.allclose(s1 + sn, np.abs(dots) @ w.astype(np.float64), rtol=1e-14)


# ------------------------------------------------------------------------------------------ top-K

def brute_topk(score, k, index=None):
    n = len(score)
    index = list(range(n)) if index is None else list(index)
    order = sorted(range(n), key=lambda i: (-score[i], index[i]))
    sel = sorted(index[i] for i in order[:k])
    return sel + [-1] * (k - len(sel))


@pytest.mark.parametrize("seed", range(6))
def test_topk_matches_bruteforce_with_ties(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 300))
    score = rng.integers(-3, 4, n).astype(np.float64)  # heavy ties
    score[rng.random(n) < 0.1] = -0.0
    for k in (1, 5, 64, 400):
        assert list(oracle.topk(score, k)) == brute_topk(list(score), k)
    idx = rng.permutation(10 * n)[:n]
    assert list(oracle.topk(score, 7, idx)) == brute_topk(list(score), 7, idx)


def test_topk_negative_zero_equals_zero():
    score = np.array([0.0, -0.0, 0.0, -0.0])
    assert list(oracle.topk(score, 2)) == [0, 1]
    score = np.array([-0.0, 0.0])
    assert list(oracle.topk(score, 1)) == [0]


def _keys_for_scores(scores):
    """Keys/queries whose indexer score equals the given non-negative integers exactly."""
    iq = torch.zeros(4, 64)
    iq[0, 0] = 1.0
    w = np.array([1.0, 0.0, 0.0, 0.0], np.float32)
    k = torch.zeros(len(scores), 64)
    k[:, 0] = torch.tensor(scores, dtype=torch.float32)
    return bits(iq), w, bits(k)


def test_full_index_hand_worked_example():
    spec = {}
    for line in open(os.path.join(GOLDEN, "topk_example.txt")):
        if line.startswith("#") or ":" not in line:
            continue
        key, val = line.split(":")
        spec[key.strip()] = [float(v) for v in val.split()]
    scores, K, P = spec["scores"], int(spec["K"][0]), int(spec["P"][0])
    iq, w, k = _keys_for_scores(scores)
    r = oracle.index_full(iq[None], w[None], k[None], [len(scores)], K, P)
    assert list(r["topk"][0]) == [int(v) for v in spec["topk"]]
    assert list(r["blockmax"][0]) == spec["blockmax"]
    assert list(r["pool"][0]) == [int(v) for v in spec["pool"]]


@pytest.mark.parametrize("seed", range(5))
def test_full_index_matches_bruteforce(seed):
    rng = np.random.default_rng(10 + seed)
    N = int(rng.integers(1, 90))
    K, P = int(rng.integers(1, 20)), int(rng.integers(1, 8))
    scores = rng.integers(0, 6, N).tolist()
    iq, w, k = _keys_for_scores(scores)
    r = oracle.index_full(iq[None], w[None], k[None], [N], K, P)
    assert list(r["topk"][0]) == brute_topk(scores, K)
    nb = (N + 7) // 8
    bmax = [max(scores[8 * j:min(8 * j + 8, N)]) for j in range(nb)]
    assert list(r["blockmax"][0]) == bmax
    blocks = [b for b in brute_topk(bmax, P) if b >= 0]
    pool = []
    for b in blocks:
        pool += [p if p < N else -1 for p in range(8 * b, 8 * b + 8)]
    pool += [-1] * (8 * P - len(pool))
    assert list(r["pool"][0]) == pool


@pytest.mark.parametrize("seed", range(4))
def test_pool_contains_topk_and_reindex_same_query_returns_topk(seed):
    """With P >= K the pool holds every Top-K position; a Reindex layer given the Full layer's
    own query and weights therefore returns exactly the Full Top-K."""
    torch.manual_seed(20 + seed)
    N, K, P = 3000 + 37 * seed, 32, 40
    iq = torch.randn(4, 64)
    w = (torch.rand(4) + 0.5).numpy().astype(np.float32)
    k = torch.randn(N, 64)
    if seed % 2:
        k = torch.round(k * 2) / 2  # many exact score ties
    r = oracle.index_full(bits(iq)[None], w[None], bits(k)[None], [N], K, P)
    topk, pool = r["topk"][0], r["pool"][0]
    assert set(topk[topk >= 0]) <= set(pool[pool >= 0])
    rr = oracle.index_reindex(bits(iq)[None], w[None], bits(k)[None], pool[None], K)
    assert np.array_equal(rr["topk"][0], topk)


def test_index_short_sequences_pad_with_minus_one():
    iq, w, k = _keys_for_scores([3, 1, 2])
    r = oracle.index_full(iq[None], w[None], k[None], [3], 5, 4)
    assert list(r["topk"][0]) == [0, 1, 2, -1, -1]
    assert list(r["pool"][0]) == [0, 1, 2] + [-1] * 29
    r0 = oracle.index_full(iq[None], w[None], k[None], [0], 2, 1)
    assert list(r0["topk"][0]) == [-1, -1] and list(r0["pool"][0]) == [-1] * 8


def test_reindex_skips_empty_slots_and_breaks_ties_by_position():
    iq, w, k = _keys_for_scores([5, 5, 1, 5, 0, 7])
    pool = np.array([[5, -1, 3, 0, -1, 1, 2]], np.int64)
    rr = oracle.index_reindex(iq[None], w[None], k[None], pool, 3)
    assert list(rr["topk"][0]) == [0, 1, 5]  # 7@5, then the 5s at positions 0, 1 (3 loses)
    rr = oracle.index_reindex(iq[None], w[None], k[None], pool, 9)
    assert list(rr["topk"][0]) == [0, 1, 2, 3, 5, -1, -1, -1, -1]


# ------------------------------------------------------------------------------------------ attend

def _cache(n, seed, W=0):
    torch.manual_seed(seed)
    x = torch.randn(n, 512)
    codes, scales = oracle.mxfp4_quantize(bits(x))
    swa = swsc = None
    if W:
        e, sc = oracle.swa_quantize(bits(torch.randn(W, 512)))
        swa, swsc = e, sc
    return codes, scales, swa, swsc


@pytest.mark.parametrize("W", [0, 5])
def test_attend_equals_dense_softmax_attention_when_all_entries_selected(W):
    n = 37
    codes, scales, swa, swsc = _cache(n, 30, W)
    torch.manual_seed(31)
    q = torch.randn(16, 512) / math.sqrt(512)
    scale = 0.75
    idx = np.arange(n, dtype=np.int64)
    out, lse = oracle.attend_seq(bits(q), scale, codes, scales, idx, swa, swsc, W)
    v = oracle.mxfp4_dequantize(codes, scales)
    if W:
        vs = oracle.e4m3_decode(swa.ravel()).reshape(W, 512) * swsc[:, None].astype(np.float64)
        v = np.concatenate([v, vs])
    V = torch.from_numpy(v)[None]
    Q = q.to(torch.bfloat16).double()[None]
    ref = torch.nn.functional.scaled_dot_product_attention(Q, V, V, scale=scale)[0].numpy()
    ref_lse = torch.logsumexp(scale * Q[0] @ V[0].T, dim=-1).numpy()
    assert np.allclose(out, ref, rtol=0, atol=1e-6 * np.abs(ref).max())
    assert np.allclose(lse, ref_lse, rtol=1e-6, atol=1e-6)


def test_attend_weights_sum_to_one_and_skip_padding():
    codes, scales, swa, swsc = _cache(50, 32, 7)
    torch.manual_seed(33)
    q = torch.randn(16, 512)
    idx = np.array([4, -1, 9, 11, -1, 49], np.int64)
    out, lse, wts = oracle.attend_seq(bits(q), 0.05, codes, scales, idx, swa, swsc, 7,
                                      want_weights=True)
    assert wts.shape == (16, 4 + 7)
    assert np.all(np.abs(wts.sum(1) - 1.0) <= 1e-12)
    # weights reproduce the output
    v = oracle.mxfp4_dequantize(codes[[4, 9, 11, 49]], scales[[4, 9, 11, 49]])
    vs = oracle.e4m3_decode(swa.ravel()).reshape(7, 512) * swsc[:, None].astype(np.float64)
    assert np.allclose(out, wts @ np.concatenate([v, vs]), rtol=1e-6, atol=1e-7)


def test_attend_constant_value_returns_that_value():
    x = torch.randn(1, 512)
    codes, scales = oracle.mxfp4_quantize(bits(x))
    codes = np.repeat(codes, 20, 0)
    scales = np.repeat(scales, 20, 0)
    idx = np.array([0, 3, 7, 19, -1], np.int64)
    q = torch.randn(16, 512)
    out, lse = oracle.attend_seq(bits(q), 0.1, codes, scales, idx, None, None, 0)
    v = oracle.mxfp4_dequantize(codes[:1], scales[:1])[0]
    assert np.allclose(out, np.broadcast_to(v, out.shape), rtol=1e-6, atol=0)
    # four equal logits: lse = z + log 4
    z = 0.1 * (q.to(torch.bfloat16).double().numpy() @ v)
    assert np.allclose(lse, z + math.log(4), rtol=1e-6, atol=1e-6)


def test_attend_empty_set():
    codes, scales, _, _ = _cache(4, 34)
    q = torch.randn(16, 512)
    out, lse = oracle.attend_seq(bits(q), 1.0, codes, scales, np.full(3, -1, np.int64), None,
                                 None, 0)
    assert not out.any() and np.all(np.isneginf(lse))


def test_attend_duplicate_index_counts_twice():
    codes, scales, _, _ = _cache(6, 35)
    q = torch.randn(16, 512) * 0.05
    o1, l1 = oracle.attend_seq(bits(q), 1.0, codes, scales, np.array([2, 2, 5], np.int64), None,
                               None, 0)
    v = oracle.mxfp4_dequantize(codes[[2, 2, 5]], scales[[2, 2, 5]])
    V = torch.from_numpy(v)[None]
    Q = q.to(torch.bfloat16).double()[None]
    ref = torch.nn.functional.scaled_dot_product_attention(Q, V, V, scale=1.0)[0].numpy()
    assert np.allclose(o1, ref, atol=1e-6 * np.abs(ref).max(), rtol=0)
