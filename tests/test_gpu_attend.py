"""GPU sparse attention against the oracle.

Method: "DeepSeek V4.1 Flash 拆解" (austincafe.tech), section 一 -- a Reuse layer runs sparse
attention directly over reused indices; the main KV is MXFP4, the SWA KV FP8, both in one
softmax. Outputs must satisfy max|d| <= 1e-3 * max|ref| + 1e-4 per call; lse within 1e-4 + 1e-5|lse|.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import sparse_attention_decode_kv_b200 as csa2
from _helpers import bits, check_attention

pytestmark = pytest.mark.gpu


def build_cache(B, n_cap, N, W, swa_len, seed, dev, scale_rows=None):
    """Fill a device cache through the GPU append (its bytes are checked bit-exact elsewhere) and
    the host mirror through the oracle's own append of the same bf16 rows."""
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(B, n_cap, 512, generator=g)
    if scale_rows is not None:
        x = x * scale_rows
    x = x.to(torch.bfloat16)
    cache = csa2.Cache(B, n_cap, W, device=dev)
    pos = torch.zeros(B, dtype=torch.int32, device=dev)
    # main KV: all n_cap rows
    csa2.append_quant(x.to(dev), None, pos, cache.codes, cache.scales, None)
    codes = np.zeros((B, n_cap, 256), np.uint8)
    scales = np.zeros((B, n_cap, 32), np.uint8)
    oracle.append(bits(x), None, np.zeros(B, np.int32), n_cap, codes, scales, None)
    # SWA ring: W tokens per sequence in slots 0..W-1; swa_len[b] says how many are valid
    swa = np.zeros((B, W, 512), np.uint8)
    swsc = np.zeros((B, W), np.float32)
    if W:
        xs = (torch.randn(B, W, 512, generator=g) * 2.0).to(torch.bfloat16)
        tmp_codes = torch.zeros(B, ((W + 7) // 8) * 8, 256, dtype=torch.uint8, device=dev)
        tmp_scales = torch.zeros(B, ((W + 7) // 8) * 8, 32, dtype=torch.uint8, device=dev)
        csa2.append_quant(xs.to(dev), None, pos, tmp_codes, tmp_scales, None, cache.swa,
                          cache.swa_scale)
        e, sc = oracle.swa_quantize(bits(xs).reshape(-1, 512))
        swa[:] = e.reshape(B, W, 512)
        swsc[:] = sc.reshape(B, W)
    torch.cuda.synchronize()
    assert np.array_equal(cache.codes.cpu().numpy(), codes)
    if W:
        assert np.array_equal(cache.swa.cpu().numpy(), swa)
    return cache, codes, scales, swa, swsc


def run_attend(mode, q, scale, cache, N, idx, swa_len, dev, with_lse=True):
    B, K = idx.shape
    out = torch.empty(B, 16, 512, dtype=torch.float32, device=dev)
    lse = torch.empty(B, 16, dtype=torch.float32, device=dev) if with_lse else None
    ws = csa2.workspace(csa2.attend_workspace_bytes(B, K, cache.W), device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    W = cache.W
    csa2.attend(mode, q.to(dev), scale, cache.codes, cache.scales,
                torch.tensor(N, dtype=torch.int32, device=dev), idx.to(dev),
                cache.swa if W else None, cache.swa_scale if W else None,
                torch.tensor(swa_len, dtype=torch.int32, device=dev) if W else None, out, lse, ws,
                err)
    torch.cuda.synchronize()
    return out.cpu().numpy(), None if lse is None else lse.cpu().numpy(), int(err.item())


def oracle_attend(q, scale, codes, scales, idx, swa, swsc, swa_len):
    return oracle.attend(bits(q).reshape(q.shape[0], 16, 512), scale, codes, scales,
                         idx.numpy().astype(np.int64), swa if swa.shape[1] else None,
                         swsc if swa.shape[1] else None, swa_len)


# splits per sequence: 4 and 10 (merged inside a thread-block cluster), 1 (no merge), 66 (more
# than a cluster holds: partials through the workspace and the merge kernel)
@pytest.mark.parametrize("B,n_cap,K,W", [(3, 1024, 100, 70), (2, 4096, 512, 128), (5, 512, 64, 0),
                                         (8, 4096, 512, 128), (2, 8192, 4096, 128)])
def test_attend_matches_oracle(gpu, B, n_cap, K, W):
    dev = gpu
    rng = np.random.default_rng(B * 1000 + K)
    N = [n_cap - 3 * b for b in range(B)]
    swa_len = [W - 2 * b if W else 0 for b in range(B)]
    swa_len[-1] = 0 if W else 0
    heavy = torch.where(torch.rand(B, n_cap, 1, generator=torch.Generator().manual_seed(9)) < 0.01,
                        8.0, 1.0)
    cache, codes, scales, swa, swsc = build_cache(B, n_cap, N, W, swa_len, seed=K, dev=dev,
                                                  scale_rows=heavy)
    idx = np.full((B, K), -1, np.int32)
    for b in range(B):
        take = min(K, N[b]) - (b % 3) * 5  # some -1 padding
        idx[b, :take] = np.sort(rng.choice(N[b], take, replace=False))
    if B > 1:
        idx[1, 3] = idx[1, 2]  # a duplicate counts twice
    idx_t = torch.from_numpy(idx)
    g = torch.Generator().manual_seed(K + 1)
    q = (torch.randn(B, 16, 512, generator=g) / math.sqrt(512)).to(torch.bfloat16)
    out, lse, err = run_attend(csa2.MODE_REUSE, q, 1.0, cache, N, idx_t, swa_len, dev)
    assert err == 0
    ref_out, ref_lse = oracle_attend(q, 1.0, codes, scales, idx_t, swa, swsc, swa_len)
    check_attention(out, lse, ref_out, ref_lse)


def test_attend_one_cta_per_sequence_path(gpu):
    """Large B: one CTA covers all tiles of a sequence (no split, no merge)."""
    dev = gpu
    B, n_cap, K, W = 300, 256, 96, 40
    assert csa2.attend_workspace_bytes(B, K, W) == 0
    N = [n_cap] * B
    swa_len = [W] * B
    cache, codes, scales, swa, swsc = build_cache(B, n_cap, N, W, swa_len, seed=3, dev=dev)
    rng = np.random.default_rng(3)
    idx = np.stack([np.sort(rng.choice(n_cap, K, replace=False)) for _ in range(B)]).astype(np.int32)
    q = (torch.randn(B, 16, 512, generator=torch.Generator().manual_seed(4)) * 0.05).to(torch.bfloat16)
    out, lse, err = run_attend(csa2.MODE_REUSE, q, 1.0, cache, N, torch.from_numpy(idx), swa_len, dev)
    ref_out, ref_lse = oracle_attend(q, 1.0, codes, scales, torch.from_numpy(idx), swa, swsc, swa_len)
    check_attention(out, lse, ref_out, ref_lse)


def test_reuse_equals_full_bit_for_bit(gpu):
    dev = gpu
    B, n_cap, K, W = 2, 1024, 512, 128
    cache, *_ = build_cache(B, n_cap, [n_cap] * B, W, [W, 17], seed=5, dev=dev)
    rng = np.random.default_rng(5)
    idx = torch.from_numpy(np.stack([np.sort(rng.choice(n_cap, K, replace=False))
                                     for _ in range(B)]).astype(np.int32))
    q = (torch.randn(B, 16, 512) / math.sqrt(512)).to(torch.bfloat16)
    outs = [run_attend(m, q, 1.0, cache, [n_cap] * B, idx, [W, 17], dev)
            for m in (csa2.MODE_FULL, csa2.MODE_REINDEX, csa2.MODE_REUSE)]
    for o, l, _ in outs[1:]:
        assert np.array_equal(o, outs[0][0]) and np.array_equal(l, outs[0][1])


def test_constant_value_and_empty_set(gpu):
    dev = gpu
    B, n_cap, K = 2, 64, 16
    x = torch.randn(1, 512).to(torch.bfloat16).expand(B, n_cap, 512).contiguous()
    cache = csa2.Cache(B, n_cap, 0, device=dev)
    csa2.append_quant(x.to(dev), None, torch.zeros(B, dtype=torch.int32, device=dev),
                      cache.codes, cache.scales, None)
    idx = torch.full((B, K), -1, dtype=torch.int32)
    idx[0, :10] = torch.arange(10, dtype=torch.int32) * 3
    q = torch.randn(B, 16, 512).to(torch.bfloat16)
    out, lse, err = run_attend(csa2.MODE_REUSE, q, 0.3, cache, [n_cap] * B, idx, [0] * B, dev)
    c, s = oracle.mxfp4_quantize(bits(x[0, :1]))
    v = oracle.mxfp4_dequantize(c, s)[0]
    assert np.allclose(out[0], np.broadcast_to(v, (16, 512)), rtol=2e-3, atol=1e-6)
    assert not out[1].any() and np.all(np.isneginf(lse[1]))


def test_invalid_indices_are_skipped_and_flagged(gpu):
    dev = gpu
    B, n_cap, K, W = 1, 256, 32, 0
    cache, codes, scales, swa, swsc = build_cache(B, n_cap, [200], W, [0], seed=6, dev=dev)
    idx = torch.arange(K, dtype=torch.int32)[None] * 6  # all below N = 200
    idx[0, 5] = 250       # >= N: skipped, flagged
    idx[0, 6] = -7        # negative but not -1: skipped, flagged
    q = torch.randn(B, 16, 512).to(torch.bfloat16) * 0.05
    out, lse, err = run_attend(csa2.MODE_REUSE, q, 1.0, cache, [200], idx, [0], dev)
    assert err & csa2.DEVERR_INDEX_RANGE
    ref_idx = idx.clone()
    ref_idx[0, 5] = -1
    ref_idx[0, 6] = -1
    ref_out, ref_lse = oracle_attend(q, 1.0, codes, scales, ref_idx, swa, swsc, [0])
    check_attention(out, lse, ref_out, ref_lse)


@pytest.mark.parametrize("qmag", [1e-30, 1e-3, 30.0, 1e30])
def test_query_magnitudes(gpu, qmag):
    """q is rescaled per head by a power of two into fp16's range: tiny and huge queries."""
    dev = gpu
    B, n_cap, K, W = 1, 512, 128, 64
    cache, codes, scales, swa, swsc = build_cache(B, n_cap, [n_cap], W, [W], seed=7, dev=dev)
    idx = torch.arange(0, 4 * K, 4, dtype=torch.int32)[None]
    q = (torch.randn(B, 16, 512) * qmag).to(torch.bfloat16)
    scale = 1.0 / (qmag * 512) if qmag > 1 else 1.0
    out, lse, err = run_attend(csa2.MODE_REUSE, q, scale, cache, [n_cap], idx, [W], dev)
    ref_out, ref_lse = oracle_attend(q, scale, codes, scales, idx, swa, swsc, [W])
    check_attention(out, lse, ref_out, ref_lse)


def test_reuse_right_after_the_index_call_that_wrote_its_indices(gpu):
    """A Reuse-mode call straight after the Reindex call that wrote its indices (on the same
    stream) must wait for them: the library gathers early only after its own attention calls.
    Its output equals the Full-mode call's on the same indices, bit for bit."""
    dev = gpu
    B, n_cap, K, W = 4, 8192, 512, 128
    cache, codes, scales, swa, swsc = build_cache(B, n_cap, [n_cap] * B, W, [W] * B, seed=11, dev=dev)
    g = torch.Generator().manual_seed(11)
    ik = torch.randn(B, n_cap, 64, generator=g).to(torch.bfloat16).to(dev)
    iq = torch.randn(B, 4, 64, generator=g).to(torch.bfloat16).to(dev)
    w = (torch.rand(B, 4, generator=g) + 0.5).to(dev)
    Nt = torch.full((B,), n_cap, dtype=torch.int32, device=dev)
    pool = torch.arange(n_cap, dtype=torch.int32, device=dev)[None].repeat(B, 1)
    q = (torch.randn(B, 16, 512, generator=g) / math.sqrt(512)).to(torch.bfloat16).to(dev)
    swa_len = torch.full((B,), W, dtype=torch.int32, device=dev)
    outs = []
    for mode in (csa2.MODE_REUSE, csa2.MODE_FULL):
        topk = torch.full((B, K), -1, dtype=torch.int32, device=dev)
        ws_re = csa2.workspace(csa2.index_reindex_workspace_bytes(B, n_cap, K), dev)
        ws_at = csa2.workspace(csa2.attend_workspace_bytes(B, K, W), dev)
        out = torch.empty(B, 16, 512, device=dev)
        lse = torch.empty(B, 16, device=dev)
        err = torch.zeros(1, dtype=torch.int32, device=dev)
        csa2.index_reindex(iq, w, ik, Nt, pool, K, topk, ws_re, err)
        csa2.attend(mode, q, 1.0, cache.codes, cache.scales, Nt, topk, cache.swa, cache.swa_scale,
                    swa_len, out, lse, ws_at, err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        outs.append((out.cpu().numpy(), lse.cpu().numpy(), topk.cpu().numpy()))
    assert np.array_equal(outs[0][2], outs[1][2])
    assert np.array_equal(outs[0][0], outs[1][0]) and np.array_equal(outs[0][1], outs[1][1])
    ref_out, ref_lse = oracle_attend(q.cpu(), 1.0, codes, scales, torch.from_numpy(outs[0][2]),
                                     swa, swsc, [W] * B)
    check_attention(outs[0][0], outs[0][1], ref_out, ref_lse)
