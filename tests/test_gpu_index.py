"""GPU Full-mode and Reindex-mode indexers against the oracle.

Method: "DeepSeek V4.1 Flash 拆解" (austincafe.tech), section 一 -- the Full layer selects a Top-K
and builds a pool of blocks x 8 positions; Reindex layers score only the pool with their own
indexer query. Index sets must equal the oracle's except for boundary swaps that fp32 rounding of
the scores can explain (each logged); the pool is checked exactly against the GPU's own block
selection, and the Reindex layer against the oracle run on the GPU's pool.
"""
import numpy as np
import pytest
import torch

import oracle
import sparse_attention_decode_kv_b200 as csa2
from _helpers import ascending_padded, bits, check_selection

pytestmark = pytest.mark.gpu


def run_full(iq, w, ik, N, K, P, dev):
    B, n_cap = ik.shape[:2]
    ws = csa2.workspace(csa2.index_full_workspace_bytes(B, n_cap, K, P), device=dev)
    topk = torch.empty(B, K, dtype=torch.int32, device=dev)
    pool = torch.empty(B, P * 8, dtype=torch.int32, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    Nt = torch.tensor(N, dtype=torch.int32, device=dev)
    csa2.index_full(iq.to(dev), w.to(dev), ik.to(dev), Nt, K, P, topk, pool, ws, err)
    torch.cuda.synchronize()
    scores = ws[: B * n_cap * 4].view(torch.float32).view(B, n_cap).cpu().numpy()
    return topk.cpu().numpy(), pool.cpu().numpy(), scores, int(err.item())


def run_reindex(iq, w, ik, N, pool, K, dev):
    B, n_cap = ik.shape[:2]
    L = pool.shape[1]
    ws = csa2.workspace(csa2.index_reindex_workspace_bytes(B, L, K), device=dev)
    topk = torch.empty(B, K, dtype=torch.int32, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    csa2.index_reindex(iq.to(dev), w.to(dev), ik.to(dev), torch.tensor(N, dtype=torch.int32, device=dev),
                       torch.as_tensor(pool, dtype=torch.int32).to(dev), K, topk, ws, err)
    torch.cuda.synchronize()
    return topk.cpu().numpy(), int(err.item())


def check_full(iq, w, ik, N, K, P, topk, pool, gpu_scores, log=None):
    """Scores within the fp32 bound, Top-K and block sets within the swap rule, pool exact."""
    B = ik.shape[0]
    iqb, ikb = bits(iq).reshape(B, 4, 64), bits(ik).reshape(B, ik.shape[1], 64)
    wn = w.numpy()
    ref = oracle.index_full(iqb, wn, ikb, N, K, P)
    n_swaps = 0
    for b in range(B):
        n = N[b]
        s, tau = oracle.index_scores(iqb[b], wn[b], ikb[b, :n], with_tol=True)
        if n:
            d = np.abs(gpu_scores[b, :n].astype(np.float64) - s)
            assert np.all(d <= tau), f"seq {b}: score error {d.max():.3e} above the fp32 bound"
        ascending_padded(topk[b], K)
        n_swaps += len(check_selection(topk[b], ref["topk"][b], lambda i: s[i], lambda i: tau[i],
                                       f"full topk b={b}", log))
        nb = (n + 7) // 8
        bm = np.array([s[8 * j:min(8 * j + 8, n)].max() for j in range(nb)])
        bt = np.array([tau[8 * j:min(8 * j + 8, n)].max() for j in range(nb)])
        gblocks = sorted(set(int(p) // 8 for p in pool[b] if p >= 0))
        oblocks = sorted(set(int(p) // 8 for p in ref["pool"][b] if p >= 0))
        n_swaps += len(check_selection(gblocks, oblocks, lambda j: bm[j], lambda j: bt[j],
                                       f"pool blocks b={b}", log))
        expect = []
        for j in gblocks:
            expect += [p if p < n else -1 for p in range(8 * j, 8 * j + 8)]
        expect += [-1] * (8 * P - len(expect))
        assert list(pool[b]) == expect, f"seq {b}: pool is not the expansion of its block set"
    return n_swaps


def make_case(B, n_cap, seed, kind="gauss"):
    g = torch.Generator().manual_seed(seed)
    iq = torch.randn(B, 4, 64, generator=g).to(torch.bfloat16)
    w = (torch.rand(B, 4, generator=g) + 0.5).float()
    if kind == "gauss":
        ik = torch.randn(B, n_cap, 64, generator=g)
    elif kind == "ties":
        ik = torch.round(torch.randn(B, n_cap, 64, generator=g) * 1.5) / 2
        iq = torch.round(iq.float() * 2).to(torch.bfloat16) / 2
    elif kind == "cluster":
        centres = torch.randn(B, 64, 64, generator=g)
        assign = torch.randint(0, 64, (B, n_cap // 8), generator=g)
        ik = torch.stack([centres[b][assign[b]] for b in range(B)]).repeat_interleave(8, 1)
        ik = ik + 0.5 * torch.randn(B, n_cap, 64, generator=g)
    return iq, w, ik.to(torch.bfloat16)


@pytest.mark.parametrize("B,n_cap,N,K,P,kind", [
    (1, 4096, [4096], 64, 64, "gauss"),                      # the tiny Full-layer workload
    (3, 8320, [8320, 37, 5001], 512, 128, "gauss"),          # ragged N: partial tiles, N < K
    (2, 20480, [20480, 19999], 512, 2048, "cluster"),        # top 2048 of 2560 blocks
    (2, 16384, [16384, 12000], 256, 256, "ties"),            # many exact ties
])
def test_full_index_matches_oracle(gpu, B, n_cap, N, K, P, kind):
    iq, w, ik = make_case(B, n_cap, seed=n_cap + K, kind=kind)
    topk, pool, scores, err = run_full(iq, w, ik, N, K, P, gpu)
    assert err == 0
    check_full(iq, w, ik, N, K, P, topk, pool, scores)


def test_full_index_all_equal_scores_takes_lowest_indices(gpu):
    """A zero query makes every score 0: ties go to the lowest positions and blocks, and every
    block is a candidate of the select."""
    B, n_cap, K, P = 2, 40960, 512, 2048
    iq = torch.zeros(B, 4, 64, dtype=torch.bfloat16)
    w = torch.ones(B, 4)
    ik = torch.randn(B, n_cap, 64).to(torch.bfloat16)
    N = [40960, 40000]
    topk, pool, scores, err = run_full(iq, w, ik, N, K, P, gpu)
    assert err == 0
    for b in range(B):
        assert list(topk[b]) == list(range(K))
        assert list(pool[b]) == list(range(8 * P))
        assert np.all(scores[b, :N[b]] == 0) and not np.signbit(scores[b, :N[b]]).any()


def test_full_index_candidates_beyond_shared_memory(gpu):
    """Equal block maxima over 32,768 blocks: every block is a candidate (more than one CTA's
    shared memory holds), so the select reads the chunked candidate regions from global memory."""
    B, n_cap, K, P = 1, 262144, 64, 32
    iq = torch.zeros(B, 4, 64, dtype=torch.bfloat16)
    w = torch.ones(B, 4)
    ik = torch.randn(B, n_cap, 64).to(torch.bfloat16)
    topk, pool, scores, err = run_full(iq, w, ik, [n_cap], K, P, gpu)
    assert err == 0
    assert list(topk[0]) == list(range(K))
    assert list(pool[0]) == list(range(8 * P))


@pytest.mark.parametrize("K,P,kind", [(4096, 2048, "gauss"), (512, 4096, "cluster"),
                                      (4096, 4096, "ties"), (3000, 2100, "gauss")])
def test_full_index_wide_selection(gpu, K, P, kind):
    """max(K, P) above 2,048: the position Top-K runs over more than 16,384 positions (up to the
    32,768 of 4,096 blocks), beyond what the selection keeps in registers, so the scores of the
    wide blocks' positions are staged in shared memory."""
    B, n_cap = 2, 40960
    iq, w, ik = make_case(B, n_cap, seed=K + 3 * P, kind=kind)
    N = [40960, 37003]
    topk, pool, scores, err = run_full(iq, w, ik, N, K, P, gpu)
    assert err == 0
    check_full(iq, w, ik, N, K, P, topk, pool, scores)


def test_full_index_wide_selection_all_equal(gpu):
    """Every score equal and max(K, P) = 4,096: all 32,768 positions of the wide blocks fall in
    the threshold bin, more candidates than the compaction buffer holds, so the select runs over
    the staged keys themselves. Ties go to the lowest positions and blocks."""
    B, n_cap, K, P = 1, 40960, 4096, 4096
    iq = torch.zeros(B, 4, 64, dtype=torch.bfloat16)
    w = torch.ones(B, 4)
    ik = torch.randn(B, n_cap, 64).to(torch.bfloat16)
    topk, pool, scores, err = run_full(iq, w, ik, [n_cap], K, P, gpu)
    assert err == 0
    assert list(topk[0]) == list(range(K))
    assert list(pool[0]) == list(range(8 * P))


@pytest.mark.parametrize("K,P", [(512, 16), (100, 7)])
def test_full_index_pool_smaller_than_topk(gpu, K, P):
    """P < K: the Top-K comes from the top-K blocks while the pool keeps only the top P."""
    B, n_cap = 2, 8192
    iq, w, ik = make_case(B, n_cap, seed=K + P)
    N = [8192, 6001]
    topk, pool, scores, err = run_full(iq, w, ik, N, K, P, gpu)
    assert err == 0
    check_full(iq, w, ik, N, K, P, topk, pool, scores)


def test_full_index_empty_and_tiny_sequences(gpu):
    B, n_cap, K, P = 3, 128, 16, 4
    iq, w, ik = make_case(B, n_cap, seed=11)
    N = [0, 5, 128]
    topk, pool, scores, err = run_full(iq, w, ik, N, K, P, gpu)
    assert err == 0
    assert list(topk[0]) == [-1] * K and list(pool[0]) == [-1] * 32
    assert list(topk[1][:5]) == [0, 1, 2, 3, 4] and list(topk[1][5:]) == [-1] * (K - 5)
    assert list(pool[1]) == [0, 1, 2, 3, 4, -1, -1, -1] + [-1] * 24
    check_full(iq, w, ik, N, K, P, topk, pool, scores)


def test_full_index_flags_bad_lengths(gpu):
    B, n_cap = 1, 256
    iq, w, ik = make_case(B, n_cap, seed=12)
    topk, pool, scores, err = run_full(iq, w, ik, [300], 8, 4, gpu)
    assert err & csa2.DEVERR_NLEN
    check_full(iq, w, ik, [256], 8, 4, topk, pool, scores)  # clamped to n_cap


@pytest.mark.parametrize("kind", ["gauss", "ties"])
def test_reindex_matches_oracle_on_gpu_pool(gpu, kind):
    B, n_cap, K, P = 3, 16384, 512, 256
    iq, w, ik = make_case(B, n_cap, seed=21, kind=kind)
    N = [16384, 9000, 600]
    _, pool, _, _ = run_full(iq, w, ik, N, K, P, gpu)
    g = torch.Generator().manual_seed(22)
    iq2 = (0.7 * iq.float() + 0.714 * torch.randn(B, 4, 64, generator=g)).to(torch.bfloat16)
    if kind == "ties":
        iq2 = torch.round(iq2.float() * 2).to(torch.bfloat16) / 2
    w2 = (torch.rand(B, 4, generator=g) + 0.5).float()
    topk2, err = run_reindex(iq2, w2, ik, N, pool, K, gpu)
    assert err == 0
    iqb, ikb = bits(iq2).reshape(B, 4, 64), bits(ik).reshape(B, n_cap, 64)
    ref = oracle.index_reindex(iqb, w2.numpy(), ikb, pool.astype(np.int64), K)
    for b in range(B):
        s, tau = oracle.index_scores(iqb[b], w2.numpy()[b], ikb[b, :N[b]], with_tol=True)
        ascending_padded(topk2[b], K)
        check_selection(topk2[b], ref["topk"][b], lambda i: s[i], lambda i: tau[i],
                        f"reindex b={b}")


def test_reindex_unsorted_pool_with_holes_and_bad_entries(gpu):
    B, n_cap, K = 1, 1024, 20
    iq, w, ik = make_case(B, n_cap, seed=31)
    rng = np.random.default_rng(31)
    pool = rng.permutation(1000)[:300].astype(np.int32)[None]
    pool[0, ::7] = -1
    pool[0, 3] = 1000   # >= N: skipped and flagged
    topk2, err = run_reindex(iq, w, ik, [1000], pool, K, gpu)
    assert err & csa2.DEVERR_INDEX_RANGE
    clean = pool.astype(np.int64).copy()
    clean[0, 3] = -1
    iqb, ikb = bits(iq).reshape(B, 4, 64), bits(ik).reshape(B, n_cap, 64)
    ref = oracle.index_reindex(iqb, w.numpy(), ikb, clean, K)
    s, tau = oracle.index_scores(iqb[0], w.numpy()[0], ikb[0, :1000], with_tol=True)
    check_selection(topk2[0], ref["topk"][0], lambda i: s[i], lambda i: tau[i], "reindex holes")


def test_reindex_with_full_query_recovers_full_topk(gpu):
    """Invariant: the pool holds the Full Top-K, so rescoring the pool with the Full layer's own
    query returns the same set (up to fp32 boundary swaps)."""
    B, n_cap, K, P = 2, 32768, 512, 2048
    iq, w, ik = make_case(B, n_cap, seed=41)
    N = [32768, 30000]
    topk, pool, _, _ = run_full(iq, w, ik, N, K, P, gpu)
    topk2, _ = run_reindex(iq, w, ik, N, pool, K, gpu)
    iqb, ikb = bits(iq).reshape(B, 4, 64), bits(ik).reshape(B, n_cap, 64)
    for b in range(B):
        assert set(topk[b][topk[b] >= 0]) <= set(pool[b][pool[b] >= 0])
        s, tau = oracle.index_scores(iqb[b], w.numpy()[b], ikb[b, :N[b]], with_tol=True)
        check_selection(topk2[b], topk[b], lambda i: s[i], lambda i: tau[i], f"RI==F b={b}")


def _reindex_vs_oracle(iq, w, ik, N, pool, K, gpu, what):
    B, n_cap = ik.shape[:2]
    topk2, err = run_reindex(iq, w, ik, N, pool, K, gpu)
    iqb, ikb = bits(iq).reshape(B, 4, 64), bits(ik).reshape(B, n_cap, 64)
    ref = oracle.index_reindex(iqb, w.numpy(), ikb, np.asarray(pool, np.int64), K)
    for b in range(B):
        s, tau = oracle.index_scores(iqb[b], w.numpy()[b], ikb[b, :N[b]], with_tol=True)
        ascending_padded(topk2[b], K)
        check_selection(topk2[b], ref["topk"][b], lambda i: s[i], lambda i: tau[i], f"{what} b={b}")
    return topk2, err


def test_reindex_top_k_concentrated_in_one_stretch_of_the_pool(gpu):
    """Every Top-K slot lies among the first 600 slots of a 16,384-slot pool."""
    B, n_cap, K = 2, 16384, 512
    iq, w, ik = make_case(B, n_cap, seed=51)
    u = (w[:, :, None] * iq.float()).sum(1)
    u = u / u.norm(dim=1, keepdim=True)
    ik = ik.float()
    ik[:, :600] += 6.0 * u[:, None, :]          # slots 0..599 outscore the rest
    ik = ik.to(torch.bfloat16)
    pool = np.tile(np.arange(n_cap, dtype=np.int32), (B, 1))
    _reindex_vs_oracle(iq, w, ik, [n_cap, n_cap], pool, K, gpu, "one-tile top")


@pytest.mark.parametrize("L,K,kind", [(32768, 512, "gauss"), (32768, 4096, "cluster"),
                                      (700, 512, "gauss"), (5000, 512, "ties")])
def test_reindex_pool_sizes(gpu, L, K, kind):
    B, n_cap = 2, 32768
    iq, w, ik = make_case(B, n_cap, seed=L + K, kind=kind)
    rng = np.random.default_rng(L)
    pool = np.stack([np.sort(rng.choice(n_cap, L, replace=False)) for _ in range(B)]).astype(np.int32)
    pool[:, 5::11] = -1
    _reindex_vs_oracle(iq, w, ik, [n_cap, n_cap], pool, K, gpu, f"L={L} K={K}")
