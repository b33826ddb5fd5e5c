"""GPU quantize-on-append against the oracle: MXFP4 codes and scales, FP8 SWA bytes and scales,
and the indexer-key copy must match bit for bit.

Format source: "DeepSeek V4.1 Flash 拆解" (austincafe.tech), section 一, FP4 KV Cache paragraph
(E2M1 values, one E4M3 scale per 16 channels; SWA KV in FP8).
"""
import numpy as np
import pytest
import torch

import oracle
import sparse_attention_decode_kv_b200 as csa2
from _helpers import bits

pytestmark = pytest.mark.gpu


def gpu_append(x, ik=None, pos=None, n_cap=None, W=0, pos_list=None, gpu_dev="cuda"):
    """Append x [B,n,512] (bf16, host or device) into fresh device caches; returns host arrays."""
    x = x.to(gpu_dev)
    B, n = x.shape[:2]
    n_cap = n_cap or ((n + 7) // 8) * 8
    pos_t = torch.tensor(pos_list if pos_list is not None else [0] * B, dtype=torch.int32,
                         device=gpu_dev)
    codes = torch.zeros(B, n_cap, 256, dtype=torch.uint8, device=gpu_dev)
    scales = torch.zeros(B, n_cap, 32, dtype=torch.uint8, device=gpu_dev)
    ikc = torch.zeros(B, n_cap, 64, dtype=torch.bfloat16, device=gpu_dev) if ik is not None else None
    swa = torch.zeros(B, W, 512, dtype=torch.uint8, device=gpu_dev) if W else None
    swsc = torch.zeros(B, W, dtype=torch.float32, device=gpu_dev) if W else None
    err = torch.zeros(1, dtype=torch.int32, device=gpu_dev)
    csa2.append_quant(x, None if ik is None else ik.to(gpu_dev), pos_t, codes, scales, ikc, swa,
                      swsc, err)
    torch.cuda.synchronize()
    return dict(codes=codes.cpu().numpy(), scales=scales.cpu().numpy(),
                ik=None if ikc is None else bits(ikc),
                swa=None if swa is None else swa.cpu().numpy(),
                swa_scale=None if swsc is None else swsc.cpu().numpy(), err=int(err.item()))


def rows_from_groups(groups):
    """list of 16-value bf16 bit arrays -> [n, 512] rows (zero padded)."""
    ng = len(groups)
    flat = np.zeros(((ng + 31) // 32) * 32 * 16, np.uint16)
    for i, g in enumerate(groups):
        flat[16 * i:16 * i + 16] = g
    return flat.reshape(-1, 512)


def to_bf16_tensor(u16):
    return torch.from_numpy(np.ascontiguousarray(u16).view(np.int16)).view(torch.bfloat16)


def test_scale_byte_for_every_bf16_amax(gpu):
    """Each group holds one bf16 magnitude (all 32,640 positive finite values) and zeros: the
    scale byte is E4M3-RNE(fp32 amax/6) for every possible amax."""
    v = (np.arange(1, 0x7F80, dtype=np.uint32)).astype(np.uint16)  # +0 excluded, below +inf
    groups = []
    for i, b in enumerate(v):
        g = np.zeros(16, np.uint16)
        g[i % 16] = b | (0x8000 if i % 3 == 0 else 0)  # also negative amax carriers
        groups.append(g)
    rows = rows_from_groups(groups)
    x = to_bf16_tensor(rows)[None]
    r = gpu_append(x, gpu_dev=gpu)
    oc, os_ = oracle.mxfp4_quantize(rows)
    n = len(rows)
    assert np.array_equal(r["scales"][0][:n], os_)
    assert np.array_equal(r["codes"][0][:n], oc)


def test_codes_for_every_bf16_value_at_unit_scale(gpu):
    """Groups anchored by 6.0 have scale 1.0: every bf16 value of magnitude <= 6 is coded."""
    allv = (np.arange(65536, dtype=np.uint32) << 16).view(np.float32)
    keep = np.isfinite(allv) & (np.abs(allv) <= 6.0)
    vb = (np.arange(65536, dtype=np.uint32)[keep]).astype(np.uint16)
    six = np.uint16(0x40C0)  # 6.0 in bf16
    groups = []
    for i in range(0, len(vb), 15):
        g = np.zeros(16, np.uint16)
        g[0] = six
        g[1:1 + len(vb[i:i + 15])] = vb[i:i + 15]
        groups.append(g)
    rows = rows_from_groups(groups)
    r = gpu_append(to_bf16_tensor(rows)[None], gpu_dev=gpu)
    oc, os_ = oracle.mxfp4_quantize(rows)
    assert np.all(os_.reshape(-1)[:len(groups)] == 0x38)
    n = len(rows)
    assert np.array_equal(r["scales"][0][:n], os_)
    assert np.array_equal(r["codes"][0][:n], oc)


def test_codes_at_every_scale_with_exact_ties(gpu):
    """For every non-zero E4M3 scale s that amax = 6s selects, place the E2M1 midpoints t*s and
    their bf16 neighbours in the group: round-half-even must hold at every scale."""
    e4 = oracle.e4m3_decode(np.arange(1, 127, dtype=np.uint8))
    ties = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0]
    groups = []
    for s in e4:
        amax = np.float32(6.0 * s)
        if not np.isfinite(amax) or amax > 3e38:
            continue
        for sign in (1.0, -1.0):
            vals = [amax] + [sign * t * s for t in ties]
            vals = np.array(vals, np.float32)
            tb = torch.from_numpy(vals).to(torch.bfloat16)
            if not torch.equal(tb.float(), torch.from_numpy(vals)):
                continue  # not representable in bf16 (subnormal corner)
            u = bits(tb)
            g = np.zeros(16, np.uint16)
            g[:len(u)] = u
            groups.append(g)
            # neighbours: one bf16 ulp above / below each tie
            nb = u.copy()
            nb[1:] = nb[1:] + 1
            g2 = np.zeros(16, np.uint16)
            g2[:len(nb)] = nb
            groups.append(g2)
    assert len(groups) > 300
    rows = rows_from_groups(groups)
    r = gpu_append(to_bf16_tensor(rows)[None], gpu_dev=gpu)
    oc, os_ = oracle.mxfp4_quantize(rows)
    n = len(rows)
    assert np.array_equal(r["scales"][0][:n], os_)
    assert np.array_equal(r["codes"][0][:n], oc)


@pytest.mark.parametrize("seed", [0, 1])
def test_random_entries_ring_and_key_copy(gpu, seed):
    """Random entries over a wide dynamic range (subnormal to saturated scales), ragged append
    positions, a ring shorter than the append (only the last W tokens survive)."""
    torch.manual_seed(seed)
    B, n, n_cap, W = 3, 300, 512, 64
    x = torch.randn(B, n, 512) * torch.exp(torch.randn(B, n, 1) * 4.0)
    x[0, 5] = 0.0
    x[1, 7, :16] = -0.0
    x[2, 9] *= 1e25
    x = x.to(torch.bfloat16)
    ik = torch.randn(B, n, 64).to(torch.bfloat16)
    pos = [0, 100, 212]
    r = gpu_append(x, ik, n_cap=n_cap, W=W, pos_list=pos, gpu_dev=gpu)
    assert r["err"] == 0
    codes = np.zeros((B, n_cap, 256), np.uint8)
    scales = np.zeros((B, n_cap, 32), np.uint8)
    ikc = np.zeros((B, n_cap, 64), np.uint16)
    swa = np.zeros((B, W, 512), np.uint8)
    swsc = np.zeros((B, W), np.float32)
    oracle.append(bits(x).reshape(B, n, 512), bits(ik).reshape(B, n, 64), np.array(pos, np.int32),
                  n_cap, codes, scales, ikc, swa, swsc, W)
    assert np.array_equal(r["codes"], codes)
    assert np.array_equal(r["scales"], scales)
    assert np.array_equal(r["ik"], ikc)
    assert np.array_equal(r["swa"], swa)
    assert np.array_equal(r["swa_scale"].view(np.uint32), swsc.view(np.uint32))


def test_swa_fp8_every_bf16_value(gpu):
    """SWA tokens built from all finite bf16 values (one magnitude anchor per token)."""
    allb = np.arange(65536, dtype=np.uint32)
    f = (allb << 16).view(np.float32)
    vb = allb[np.isfinite(f)].astype(np.uint16)
    n = (len(vb) + 511) // 512
    rows = np.zeros(n * 512, np.uint16)
    rows[:len(vb)] = vb
    rows = rows.reshape(n, 512)
    x = to_bf16_tensor(rows)[None]
    W = n
    r = gpu_append(x, W=W, gpu_dev=gpu)
    e, sc = oracle.swa_quantize(rows)
    assert np.array_equal(r["swa"][0], e)
    assert np.array_equal(r["swa_scale"][0].view(np.uint32), sc.view(np.uint32))


def test_out_of_range_rows_are_skipped_and_flagged(gpu):
    x = torch.randn(2, 4, 512).to(torch.bfloat16)
    r = gpu_append(x, n_cap=16, pos_list=[14, 0], gpu_dev=gpu)
    assert r["err"] & csa2.DEVERR_POS_RANGE
    oc, os_ = oracle.mxfp4_quantize(bits(x[0, :2]))
    assert np.array_equal(r["codes"][0, 14:16], oc)  # rows 14, 15 written; 16, 17 skipped
    assert np.array_equal(r["scales"][0, 14:16], os_)
    oc1, _ = oracle.mxfp4_quantize(bits(x[1]))
    assert np.array_equal(r["codes"][1, :4], oc1)
