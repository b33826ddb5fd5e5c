"""GPU sparse attention on the tensor-core (tcgen05) path against the oracle.

From 64 queries up `csa2_attend` runs the persistent tcgen05 kernel (`csrc/attend_tc.cu`): tiles
of 128 items, S^T = V q^T and O^T = V^T P^T accumulated in tensor memory, one CTA per SM looping
over (query, split) units. These cases drive its paths: splits with partial outputs and the merge
kernel, CTAs that take several units, ragged index and SWA tiles, several SWA tiles, no SWA, empty
queries, invalid indices, unknown sequences and clamped windows of the multi-query form, query
magnitudes that move the softmax reference maxima between tiles (the lazy rescaling of O), CTAs
whose first tile is an index tile (issued by the dequantisation warps) or an SWA tile (issued by
the gather warps), and lse requested or not on both the single-unit and the split path.

Method: "DeepSeek V4.1 Flash 拆解" (austincafe.tech), section 一 -- a Reuse layer runs sparse
attention directly over reused indices; the main KV is MXFP4, the SWA KV FP8, both in one
softmax. Tolerance as in test_gpu_attend.py: max|d| <= 1e-3 * max|ref| + 1e-4 per call, lse
within 1e-4 + 1e-5|lse|.
"""
import math

import numpy as np
import pytest
import torch

import sparse_attention_decode_kv_b200 as csa2
from _helpers import check_attention
from test_gpu_attend import build_cache, oracle_attend, run_attend

pytestmark = pytest.mark.gpu


def sorted_indices(rng, B, K, N, pad):
    idx = np.full((B, K), -1, np.int32)
    for b in range(B):
        take = max(0, min(K, N[b]) - pad[b])
        idx[b, :take] = np.sort(rng.choice(N[b], take, replace=False))
    return idx


# (B, n_cap, K, W), 148 SMs:
#   64 x (512 + 128): 5 tiles, 2 splits per query (2 + 3 tiles), partials merged
#   64 x (300 + 200): ragged last index tile, two SWA tiles (128 + 72 rows), 2 splits
#   96 x 130, no SWA: two index tiles, the second with 2 items
#   80 x (40 + 256): one short index tile, two full SWA tiles
#   200 x (256 + 64): one unit per query, 200 units on 148 CTAs (some CTAs take two)
#   64 x (40 + 256): three tiles in two splits, so every second CTA starts on an SWA tile (its
#   first tile then comes from the gather warps, not the dequantisation warps)
@pytest.mark.parametrize("B,n_cap,K,W", [(64, 1024, 512, 128), (64, 2048, 300, 200),
                                         (96, 512, 130, 0), (80, 256, 40, 256),
                                         (200, 512, 256, 64), (64, 512, 40, 256)])
def test_tc_attend_matches_oracle(gpu, B, n_cap, K, W):
    dev = gpu
    rng = np.random.default_rng(B * 7 + K)
    N = [n_cap - 8 * (b % 5) for b in range(B)]
    swa_len = [max(0, W - 3 * (b % 7)) if W else 0 for b in range(B)]
    if W:
        swa_len[5] = 0
    heavy = torch.where(torch.rand(B, n_cap, 1, generator=torch.Generator().manual_seed(B)) < 0.01,
                        8.0, 1.0)
    cache, codes, scales, swa, swsc = build_cache(B, n_cap, N, W, swa_len, seed=K + W, dev=dev,
                                                  scale_rows=heavy)
    idx = sorted_indices(rng, B, K, N, [(b % 4) * 7 for b in range(B)])
    idx[1, 3] = idx[1, 2]  # a duplicate counts twice
    idx_t = torch.from_numpy(idx)
    q = (torch.randn(B, 16, 512, generator=torch.Generator().manual_seed(K)) /
         math.sqrt(512)).to(torch.bfloat16)
    out, lse, err = run_attend(csa2.MODE_REUSE, q, 1.0, cache, N, idx_t, swa_len, dev)
    assert err == 0
    ref_out, ref_lse = oracle_attend(q, 1.0, codes, scales, idx_t, swa, swsc, swa_len)
    check_attention(out, lse, ref_out, ref_lse)


def test_tc_partials_without_lse(gpu):
    """Split partials merged into out with lse not requested."""
    dev = gpu
    B, n_cap, K, W = 64, 1024, 512, 128
    assert csa2.attend_workspace_bytes(B, K, W) > 0  # partials go through the workspace
    N = [n_cap] * B
    swa_len = [W] * B
    cache, codes, scales, swa, swsc = build_cache(B, n_cap, N, W, swa_len, seed=21, dev=dev)
    rng = np.random.default_rng(21)
    idx = torch.from_numpy(sorted_indices(rng, B, K, N, [0] * B))
    q = (torch.randn(B, 16, 512, generator=torch.Generator().manual_seed(22)) * 0.05).to(torch.bfloat16)
    out, lse, err = run_attend(csa2.MODE_FULL, q, 1.0, cache, N, idx, swa_len, dev, with_lse=False)
    assert err == 0 and lse is None
    ref_out, _ = oracle_attend(q, 1.0, codes, scales, idx, swa, swsc, swa_len)
    check_attention(out, None, ref_out, None)


def test_tc_single_split_without_lse(gpu):
    """One unit per query (no partials) with lse not requested: the epilogue writes out only."""
    dev = gpu
    B, n_cap, K, W = 96, 1024, 384, 128
    assert csa2.attend_workspace_bytes(B, K, W) >= 0
    N = [n_cap - 16 * (b % 3) for b in range(B)]
    swa_len = [W - (b % 5) for b in range(B)]
    cache, codes, scales, swa, swsc = build_cache(B, n_cap, N, W, swa_len, seed=23, dev=dev)
    rng = np.random.default_rng(23)
    idx = torch.from_numpy(sorted_indices(rng, B, K, N, [(b % 3) * 5 for b in range(B)]))
    q = (torch.randn(B, 16, 512, generator=torch.Generator().manual_seed(24)) /
         math.sqrt(512)).to(torch.bfloat16)
    out, lse, err = run_attend(csa2.MODE_REUSE, q, 1.0, cache, N, idx, swa_len, dev, with_lse=False)
    assert err == 0 and lse is None
    ref_out, _ = oracle_attend(q, 1.0, codes, scales, idx, swa, swsc, swa_len)
    check_attention(out, None, ref_out, None)


def test_tc_empty_queries_and_invalid_indices(gpu):
    """A query with nothing to attend to gives zeros and lse = -inf; indices outside [0, N) other
    than -1 are skipped and flagged."""
    dev = gpu
    B, n_cap, K, W = 64, 512, 128, 64
    N = [n_cap] * B
    N[2] = 100
    swa_len = [W] * B
    swa_len[0] = 0
    cache, codes, scales, swa, swsc = build_cache(B, n_cap, N, W, swa_len, seed=31, dev=dev)
    rng = np.random.default_rng(31)
    idx = sorted_indices(rng, B, K, N, [0] * B)
    idx[0, :] = -1            # query 0: no index, no SWA row
    idx[2, 7] = 300           # >= N[2]: skipped, flagged
    idx[3, 9] = -5            # negative, not -1: skipped, flagged
    q = (torch.randn(B, 16, 512, generator=torch.Generator().manual_seed(32)) * 0.05).to(torch.bfloat16)
    out, lse, err = run_attend(csa2.MODE_REUSE, q, 1.0, cache, N, torch.from_numpy(idx), swa_len, dev)
    assert err & csa2.DEVERR_INDEX_RANGE
    assert not out[0].any() and np.all(np.isneginf(lse[0]))
    ref_idx = idx.copy()
    ref_idx[2, 7] = -1
    ref_idx[3, 9] = -1
    ref_out, ref_lse = oracle_attend(q, 1.0, codes, scales, torch.from_numpy(ref_idx), swa, swsc,
                                     swa_len)
    check_attention(out, lse, ref_out, ref_lse)


@pytest.mark.parametrize("qmag", [1e-30, 30.0, 1e30])
def test_tc_query_magnitudes(gpu, qmag):
    """Tiny and huge queries. At qmag = 30 the logits span hundreds of units across tiles, so the
    reference maxima move between tiles and O is rescaled in tensor memory."""
    dev = gpu
    B, n_cap, K, W = 64, 1024, 512, 128
    cache, codes, scales, swa, swsc = build_cache(B, n_cap, [n_cap] * B, W, [W] * B, seed=41, dev=dev)
    rng = np.random.default_rng(41)
    idx = torch.from_numpy(sorted_indices(rng, B, K, [n_cap] * B, [0] * B))
    q = (torch.randn(B, 16, 512, generator=torch.Generator().manual_seed(42)) * qmag).to(torch.bfloat16)
    scale = 1.0 / (qmag * 512) if qmag > 1e3 else 1.0
    out, lse, err = run_attend(csa2.MODE_REUSE, q, scale, cache, [n_cap] * B, idx, [W] * B, dev)
    assert err == 0
    ref_out, ref_lse = oracle_attend(q, scale, codes, scales, idx, swa, swsc, [W] * B)
    check_attention(out, lse, ref_out, ref_lse)


def test_tc_rising_logits_rescale(gpu):
    """Later tiles hold rows scaled up by 64, so each query's maximum logit rises tile after tile
    by far more than the rescaling gap."""
    dev = gpu
    B, n_cap, K, W = 64, 1024, 512, 0
    ramp = torch.ones(B, n_cap, 1)
    ramp[:, n_cap // 2:] = 64.0
    cache, codes, scales, swa, swsc = build_cache(B, n_cap, [n_cap] * B, W, [0] * B, seed=51, dev=dev,
                                                  scale_rows=ramp)
    idx = torch.from_numpy(np.stack([np.arange(0, n_cap, 2, dtype=np.int32)] * B))  # sorted: low rows first
    q = (torch.randn(B, 16, 512, generator=torch.Generator().manual_seed(52)) * 0.2).to(torch.bfloat16)
    out, lse, err = run_attend(csa2.MODE_REUSE, q, 1.0, cache, [n_cap] * B, idx, [0] * B, dev)
    assert err == 0
    ref_out, ref_lse = oracle_attend(q, 1.0, codes, scales, idx, swa, swsc, [0] * B)
    check_attention(out, lse, ref_out, ref_lse)


def test_tc_reuse_equals_full_bit_for_bit(gpu):
    dev = gpu
    B, n_cap, K, W = 96, 1024, 512, 128
    swa_len = [W - (b % 9) for b in range(B)]
    cache, *_ = build_cache(B, n_cap, [n_cap] * B, W, swa_len, seed=61, dev=dev)
    rng = np.random.default_rng(61)
    idx = torch.from_numpy(sorted_indices(rng, B, K, [n_cap] * B, [0] * B))
    q = (torch.randn(B, 16, 512, generator=torch.Generator().manual_seed(62)) /
         math.sqrt(512)).to(torch.bfloat16)
    outs = [run_attend(m, q, 1.0, cache, [n_cap] * B, idx, swa_len, dev)
            for m in (csa2.MODE_FULL, csa2.MODE_REUSE, csa2.MODE_REUSE)]
    for o, l, _ in outs[1:]:
        assert np.array_equal(o, outs[0][0]) and np.array_equal(l, outs[0][1])


def test_tc_queries_bad_sequences_and_clamped_windows(gpu):
    """csa2_attend_queries with 80 queries (the tcgen05 kernel): queries naming no sequence give
    zeros and lse = -inf and are flagged; windows running past the SWA buffer are clamped and
    flagged. Two SWA tiles per query (W = 200) start at arbitrary rows, so the tiled window loads
    begin at odd offsets and run past the buffer's end."""
    from test_gpu_attend_queries import _oracle_query, _run_queries, _swa_buffer
    dev = gpu
    B, n_cap, K, W, S = 3, 1024, 100, 200, 256
    N = [1024, 900, 1000]
    cache, codes, scales, _, _ = build_cache(B, n_cap, N, 0, [0] * B, seed=71, dev=dev)
    swa, swsc = _swa_buffer(B, S, seed=72)
    Q = 80
    rng = np.random.default_rng(73)
    qseq = [[0, 1, 2, -1, 5][i % 5] for i in range(Q)]
    idx = np.full((Q, K), -1, np.int32)
    for i in range(Q):
        nb = N[qseq[i]] if 0 <= qseq[i] < B else 1024
        take = K - (i % 3) * 11
        idx[i, :take] = np.sort(rng.choice(nb, take, replace=False))
    lo = [(37 * i) % S for i in range(Q)]
    ln = [[200, 0, 131, 64, 199][i % 5] for i in range(Q)]
    q = (torch.randn(Q, 16, 512, generator=torch.Generator().manual_seed(74)) /
         math.sqrt(512)).to(torch.bfloat16)
    out, lse, err = _run_queries(q, cache, N, qseq, idx, swa, swsc, lo, ln, W, dev)
    assert err & csa2.DEVERR_INDEX_RANGE and err & csa2.DEVERR_NLEN
    for i in range(Q):
        b = qseq[i]
        if not 0 <= b < B:
            assert np.all(out[i] == 0) and np.all(np.isneginf(lse[i]))
            continue
        l = min(ln[i], S - lo[i])
        ro, rl = _oracle_query(q[i], codes, scales, b, idx[i], swa, swsc, lo[i], l)
        check_attention(out[i], lse[i], ro, rl)
