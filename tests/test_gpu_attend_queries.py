"""GPU multi-query sparse attention (csa2_attend_queries) against the oracle.

Method: "DeepSeek V4.1 Flash 拆解" (austincafe.tech), section 一 (a Reuse layer runs sparse
attention over its indices, the main KV in MXFP4 and the SWA KV in FP8) and section 二 (the
Reuse layer's prefill flow): in prefill every prompt token is a query with its own selected
entries and its own sliding window. Each query is compared with the oracle's attention of that
one query; the decode call is the case of one query per sequence, and the two must agree bit for
bit there.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import sparse_attention_decode_kv_b200 as csa2
from _helpers import bits, check_attention
from test_gpu_attend import build_cache, run_attend

pytestmark = pytest.mark.gpu


def _swa_buffer(B, S, seed):
    """FP8 SWA rows of every position, from the oracle's SWA codec (an input here)."""
    g = torch.Generator().manual_seed(seed)
    xs = (torch.randn(B, S, 512, generator=g) * 2.0).to(torch.bfloat16)
    e, sc = oracle.swa_quantize(bits(xs).reshape(-1, 512))
    return e.reshape(B, S, 512), sc.reshape(B, S)


def _run_queries(q, cache, N, qseq, idx, swa, swsc, swa_lo, swa_len, W, dev, lse=True):
    Q, K = idx.shape
    out = torch.empty(Q, 16, 512, dtype=torch.float32, device=dev)
    lse_t = torch.empty(Q, 16, dtype=torch.float32, device=dev) if lse else None
    ws = csa2.workspace(csa2.attend_workspace_bytes(Q, K, W), device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    t = lambda a: torch.as_tensor(np.asarray(a), dtype=torch.int32).to(dev)
    csa2.attend_queries(q.to(dev), 1.0, cache.codes, cache.scales, t(N), t(qseq), t(idx),
                        None if swa is None else torch.from_numpy(swa).to(dev),
                        None if swsc is None else torch.from_numpy(swsc).to(dev),
                        None if swa is None else t(swa_lo), None if swa is None else t(swa_len),
                        W, out, lse_t, ws, err)
    torch.cuda.synchronize()
    return out.cpu().numpy(), None if lse_t is None else lse_t.cpu().numpy(), int(err.item())


def _oracle_query(q, codes, scales, b, idx, swa, swsc, lo, ln):
    return oracle.attend_seq(bits(q), 1.0, codes[b], scales[b], np.asarray(idx, np.int64),
                             swa[b, lo:lo + ln] if ln else None, swsc[b, lo:lo + ln] if ln else None,
                             ln)


@pytest.mark.parametrize("T,K,W", [(40, 128, 32), (9, 512, 128), (70, 64, 0)])
def test_prefill_queries_match_the_oracle(gpu, T, K, W):
    """T prompt tokens per sequence, each attending to its own causal selection and window."""
    B, n_cap = 2, 4096
    N = [4096, 3000]
    cache, codes, scales, _, _ = build_cache(B, n_cap, N, 0, [0, 0], seed=T + K, dev=gpu)
    S = n_cap
    swa, swsc = _swa_buffer(B, S, seed=T) if W else (None, None)
    rng = np.random.default_rng(T * 7 + K)
    qseq, lo, ln, idx = [], [], [], []
    for b in range(B):
        for t in range(T):
            p = N[b] - T + t                       # position of this prompt token
            qseq.append(b)
            start = max(0, p - W + 1)
            lo.append(start)
            ln.append(p - start + 1 if W else 0)
            take = min(K, p) - (t % 4) * 3
            row = np.full(K, -1, np.int32)
            row[:take] = np.sort(rng.choice(p, take, replace=False))
            idx.append(row)
    idx = np.stack(idx)
    Q = len(qseq)
    g = torch.Generator().manual_seed(T + 11)
    q = (torch.randn(Q, 16, 512, generator=g) / math.sqrt(512)).to(torch.bfloat16)
    out, lse, err = _run_queries(q, cache, N, qseq, idx, swa, swsc, lo, ln, W, gpu)
    assert err == 0
    for i in range(Q):
        ro, rl = _oracle_query(q[i], codes, scales, qseq[i], idx[i], swa, swsc, lo[i], ln[i])
        check_attention(out[i], lse[i], ro, rl)


def test_one_query_per_sequence_equals_the_decode_call(gpu):
    B, n_cap, K, W = 4, 2048, 256, 64
    N = [2048, 2000, 1500, 900]
    swa_len = [64, 64, 30, 0]
    cache, codes, scales, swa, swsc = build_cache(B, n_cap, N, W, swa_len, seed=5, dev=gpu)
    rng = np.random.default_rng(5)
    idx = np.stack([np.sort(rng.choice(N[b], K, replace=False)) for b in range(B)]).astype(np.int32)
    g = torch.Generator().manual_seed(6)
    q = (torch.randn(B, 16, 512, generator=g) / math.sqrt(512)).to(torch.bfloat16)
    out_d, lse_d, err_d = run_attend(csa2.MODE_REUSE, q, 1.0, cache, N, torch.from_numpy(idx),
                                     swa_len, gpu)
    out_q, lse_q, err_q = _run_queries(q, cache, N, list(range(B)), idx, swa, swsc, [0] * B,
                                       swa_len, W, gpu)
    assert err_d == 0 and err_q == 0
    assert np.array_equal(out_d, out_q) and np.array_equal(lse_d, lse_q)


def test_bad_sequences_and_windows_are_flagged(gpu):
    B, n_cap, K, W = 2, 1024, 32, 16
    N = [1024, 1024]
    cache, codes, scales, _, _ = build_cache(B, n_cap, N, 0, [0, 0], seed=8, dev=gpu)
    S = 64
    swa, swsc = _swa_buffer(B, S, seed=8)
    rng = np.random.default_rng(8)
    idx = np.stack([np.sort(rng.choice(1024, K, replace=False)) for _ in range(4)]).astype(np.int32)
    qseq = [0, 5, 1, -1]                    # queries 1 and 3 name no sequence
    lo, ln = [10, 0, 60, 0], [16, 16, 16, 4]  # query 2's window runs past row 63: clamped to 4
    g = torch.Generator().manual_seed(9)
    q = (torch.randn(4, 16, 512, generator=g) / math.sqrt(512)).to(torch.bfloat16)
    out, lse, err = _run_queries(q, cache, N, qseq, idx, swa, swsc, lo, ln, W, gpu)
    assert err & csa2.DEVERR_INDEX_RANGE and err & csa2.DEVERR_NLEN
    for i in (1, 3):                        # empty: zero output, lse -inf
        assert np.all(out[i] == 0) and np.all(np.isneginf(lse[i]))
    ro, rl = _oracle_query(q[0], codes, scales, 0, idx[0], swa, swsc, 10, 16)
    check_attention(out[0], lse[0], ro, rl)
    ro, rl = _oracle_query(q[2], codes, scales, 1, idx[2], swa, swsc, 60, 4)
    check_attention(out[2], lse[2], ro, rl)


def test_more_queries_than_one_grid_dimension_row(gpu):
    """70,000 queries: more than the 65,535 blocks a grid's y or z dimension can hold."""
    B, n_cap, K = 1, 1024, 64
    N = [1024]
    cache, codes, scales, _, _ = build_cache(B, n_cap, N, 0, [0], seed=12, dev=gpu)
    Q = 70000
    rng = np.random.default_rng(12)
    base = np.stack([np.sort(rng.choice(1024, K, replace=False)) for _ in range(16)]).astype(np.int32)
    idx = base[np.arange(Q) % 16]
    g = torch.Generator().manual_seed(13)
    q = (torch.randn(16, 16, 512, generator=g) / math.sqrt(512)).to(torch.bfloat16)
    qq = q[torch.arange(Q) % 16]
    out, lse, err = _run_queries(qq, cache, N, [0] * Q, idx, None, None, None, None, 0, gpu)
    assert err == 0
    for i in (0, 1, 65534, 65535, 65536, Q - 1):
        ro, rl = _oracle_query(q[i % 16], codes, scales, 0, idx[i], None, None, 0, 0)
        check_attention(out[i], lse[i], ro, rl)
