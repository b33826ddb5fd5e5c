"""The append and Reuse-attention sweep workloads at their full sizes against the oracle.

Method: "DeepSeek V4.1 Flash 拆解" (austincafe.tech), section 一. New entries are quantised to
MXFP4 on append (E2M1 codes, one E4M3 scale per 16 channels). A Reuse layer attends over reused
indices and the FP8 SWA rows in one softmax.

The workloads:
- append: 1,048,576 new bf16 entries, N(0,1) with 0.1 % of the elements × 20.
- Reuse attention: batch 1, 8, 64 and 256 over N = 131,072 cached entries, Top-512 indices
  drawn uniformly without replacement, a 128-row SWA window.

Every input comes from the workloads' seeded generators. The oracle quantises the rows it needs
itself.

Checks:
- MXFP4 bytes of sampled appended rows: bit for bit.
- Attention of sampled sequences: within the output tolerance, on each batch size's own launch
  shape (10, 10 and 4 splits with the merge, one CTA per sequence at 256).
"""
import numpy as np
import pytest
import torch

import oracle
import sparse_attention_decode_kv_b200 as csa2
import workloads
from _helpers import bits, check_attention

pytestmark = pytest.mark.gpu


def test_append_1m_sampled_rows(gpu):
    wl = workloads.APPEND_1M
    x = workloads.append_rows(wl, gpu)                     # [1, 1,048,576, 512] bf16
    n = wl.n
    codes = torch.full((1, n, 256), 0xAB, dtype=torch.uint8, device=gpu)
    scales = torch.full((1, n, 32), 0xAB, dtype=torch.uint8, device=gpu)
    err = torch.zeros(1, dtype=torch.int32, device=gpu)
    csa2.append_quant(x, None, torch.zeros(1, dtype=torch.int32, device=gpu), codes, scales, None,
                      dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    rng = np.random.default_rng(11)
    rows = np.unique(np.concatenate([rng.choice(n, 16384, replace=False), [0, 1, n - 2, n - 1]]))
    sel = torch.as_tensor(rows, device=gpu)
    oc, osc = oracle.mxfp4_quantize(bits(x[0, sel]))
    assert np.array_equal(codes[0, sel].cpu().numpy(), oc)
    assert np.array_equal(scales[0, sel].cpu().numpy(), osc)
    # the sample holds rows with outliers (x20): their scales are the large ones
    assert (np.abs((x[0, sel].float()).cpu().numpy()).max(1) > 8).sum() > 1000


def _fill(wl, cache, dev):
    for b0 in range(0, wl.B, 16):
        b1 = min(wl.B, b0 + 16)
        for c in range(workloads.n_chunks(wl)):
            x = torch.stack([workloads.reuse_kv_chunk(wl, b, c, dev) for b in range(b0, b1)])
            pos = torch.full((b1 - b0,), c * workloads.CHUNK, dtype=torch.int32, device=dev)
            csa2.append_quant(x, None, pos, cache.codes[b0:b1], cache.scales[b0:b1], None,
                              cache.swa[b0:b1], cache.swa_scale[b0:b1])
            del x


def _rows(wl, b, pos, dev):
    pos = np.asarray(pos, np.int64)
    out = np.zeros((len(pos), 512), np.uint16)
    for c in np.unique(pos // workloads.CHUNK):
        m = pos // workloads.CHUNK == c
        x = workloads.reuse_kv_chunk(wl, b, int(c), dev)
        out[m] = bits(x[torch.as_tensor(pos[m] - c * workloads.CHUNK, device=dev)])
    return out


@pytest.mark.parametrize("wl", workloads.REUSE_SWEEP, ids=lambda w: w.name)
def test_reuse_attend_sweep(gpu, wl):
    B, N, K, W = wl.B, wl.N, wl.K, wl.W
    cache = csa2.Cache(B, N, W, device=gpu)
    _fill(wl, cache, gpu)
    idx = workloads.reuse_indices(wl, gpu)
    q = workloads.reuse_queries(wl, gpu)
    out = torch.full((B, 16, 512), float("nan"), device=gpu)
    lse = torch.full((B, 16), float("nan"), device=gpu)
    ws = csa2.workspace(csa2.attend_workspace_bytes(B, K, W), device=gpu)
    err = torch.zeros(1, dtype=torch.int32, device=gpu)
    scale = 1.0  # q carries the 1/sqrt(512)
    csa2.attend(csa2.MODE_REUSE, q, scale, cache.codes, cache.scales,
                torch.full((B,), N, dtype=torch.int32, device=gpu), idx, cache.swa, cache.swa_scale,
                torch.full((B,), W, dtype=torch.int32, device=gpu), out, lse, ws, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    idx_h = idx.cpu().numpy()
    wpos = list(range(N - W, N))
    for b in sorted({0, B // 2, B - 1}):
        need = idx_h[b].astype(np.int64)
        codes, scales = oracle.mxfp4_quantize(_rows(wl, b, need, gpu))
        e, sc = oracle.swa_quantize(_rows(wl, b, wpos, gpu))
        ring = np.zeros((W, 512), np.uint8)
        rsc = np.zeros(W, np.float32)
        for i, p in enumerate(wpos):
            ring[p % W], rsc[p % W] = e[i], sc[i]
        ro, rl = oracle.attend_seq(bits(q[b]), scale, codes, scales, np.arange(K), ring, rsc, W)
        check_attention(out[b].cpu().numpy(), lse[b].cpu().numpy(), ro, rl)
