"""The allocation-free Reindex entry point (csa2_index_reindex_noalloc) gives the same Top-K as
csa2_index_reindex with a caller workspace, on two calls in a row.

It exists for callers that may not allocate device memory where they run the decode step; its
scratch is a fixed array inside the library. This file is collected last so that a run stopping
at the first failure has run every other test before it, and it works both alone in a fresh
process (the first call sets up the array's address) and after the other tests.
"""
import numpy as np
import pytest
import torch

import sparse_attention_decode_kv_b200 as csa2

pytestmark = pytest.mark.gpu

MAX_SLOTS = 262144  # CSA2_NOALLOC_REINDEX_MAX_SLOTS


def _case(seed, B, n_cap, K, P, dev):
    g = torch.Generator().manual_seed(seed)
    iq = torch.randn(B, 4, 64, generator=g).to(torch.bfloat16).to(dev)
    w = (torch.rand(B, 4, generator=g) + 0.5).to(dev)
    ik = torch.randn(B, n_cap, 64, generator=g).to(torch.bfloat16).to(dev)
    N = torch.tensor([n_cap - 7 * b for b in range(B)], dtype=torch.int32, device=dev)
    topk = torch.empty(B, K, dtype=torch.int32, device=dev)
    pool = torch.empty(B, 8 * P, dtype=torch.int32, device=dev)
    ws = csa2.workspace(csa2.index_full_workspace_bytes(B, n_cap, K, P), dev)
    csa2.index_full(iq, w, ik, N, K, P, topk, pool, ws)
    iq2 = torch.randn(B, 4, 64, generator=g).to(torch.bfloat16).to(dev)
    w2 = (torch.rand(B, 4, generator=g) + 0.5).to(dev)
    return iq2, w2, ik, N, pool


def _reference(iq, w, ik, N, pool, K, dev):
    B, L = pool.shape
    out = torch.empty(B, K, dtype=torch.int32, device=dev)
    ws = csa2.workspace(csa2.index_reindex_workspace_bytes(B, L, K), dev)
    csa2.index_reindex(iq, w, ik, N, pool, K, out, ws)
    return out


def test_noalloc_reindex_matches_workspace_reindex_twice_in_a_row(gpu):
    dev = gpu
    K = 512
    cases = [_case(1, 4, 16384, K, 2048, dev), _case(2, 3, 8192, K, 512, dev)]
    refs = [_reference(*c, K, dev) for c in cases]
    outs = []
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    for iq, w, ik, N, pool in cases:  # two different calls back to back on the shared array
        out = torch.full((pool.shape[0], K), -7, dtype=torch.int32, device=dev)
        csa2.index_reindex_noalloc(iq, w, ik, N, pool, K, out, err)
        outs.append(out)
    torch.cuda.synchronize()
    assert err.item() == 0
    for out, ref in zip(outs, refs):
        # same kernels and the same arithmetic: the index sets agree exactly
        assert np.array_equal(out.cpu().numpy(), ref.cpu().numpy())


@pytest.mark.parametrize("B,n_cap,P", [(16, 16384, 2048), (8, 32768, 4096)])
def test_noalloc_reindex_fills_its_whole_array(gpu, B, n_cap, P):
    """B * L exactly the array's size: the last slot is written and read. The second case has
    pools of 32,768 slots, above what the selection keeps in registers, so it reads its keys back
    from the array on every pass."""
    dev = gpu
    K = 512
    assert B * 8 * P == MAX_SLOTS
    case = _case(3 + B, B, n_cap, K, P, dev)
    ref = _reference(*case, K, dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    outs = []
    for _ in range(2):
        out = torch.full((B, K), -7, dtype=torch.int32, device=dev)
        csa2.index_reindex_noalloc(*case, K, out, err)
        outs.append(out)
    torch.cuda.synchronize()
    assert err.item() == 0
    for out in outs:
        assert np.array_equal(out.cpu().numpy(), ref.cpu().numpy())


def test_noalloc_reindex_rejects_more_slots_than_its_array(gpu):
    dev = gpu
    B, L, K = 17, 16384, 64  # 278,528 slots > 262,144
    assert B * L > MAX_SLOTS
    iq = torch.zeros(B, 4, 64, dtype=torch.bfloat16, device=dev)
    w = torch.ones(B, 4, device=dev)
    ik = torch.zeros(B, 64, 64, dtype=torch.bfloat16, device=dev)
    N = torch.full((B,), 64, dtype=torch.int32, device=dev)
    pool = torch.full((B, L), -1, dtype=torch.int32, device=dev)
    out = torch.empty(B, K, dtype=torch.int32, device=dev)
    with pytest.raises(csa2.Csa2Error) as e:
        csa2.index_reindex_noalloc(iq, w, ik, N, pool, K, out)
    assert e.value.status == -2  # CSA2_ERR_UNSUPPORTED
