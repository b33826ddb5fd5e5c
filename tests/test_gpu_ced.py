"""GPU CED KV projection with the MXFP4 epilogue (csa2_ced_project_quant) against the oracle.

Method: "DeepSeek V4.1 Flash 拆解" (austincafe.tech), section 一, CED paragraph: the decoder
layers' global KV is projected from the middle layer's hidden state, C_l = H_{L/2} W^KV_l, and
stored as MXFP4 (E2M1 codes, one E4M3 scale per 16 channels).

Two kinds of checks. With integer-valued inputs every partial sum is exact in fp32 whatever the
accumulation order, so the GPU's codes and scales must equal the oracle's quantisation of the
exact product bit for bit. With Gaussian inputs the GPU's fp32 accumulation may differ from the
exact sum by at most tau = d * 2^-23 * sum|h w| per element (a deliberate over-bound of fp32
summation in any order); every GPU code and scale must then be the quantisation of some value
within tau of the exact one, and almost all must equal the oracle's exactly.
"""
import numpy as np
import pytest
import torch

import oracle
import sparse_attention_decode_kv_b200 as csa2
from _helpers import bits

pytestmark = pytest.mark.gpu

SENTINEL = 0xAB


def _run(h, w, pos, n_cap, dev, err=None):
    B, n, d = h.shape
    codes = torch.full((B, n_cap, 256), SENTINEL, dtype=torch.uint8, device=dev)
    scales = torch.full((B, n_cap, 32), SENTINEL, dtype=torch.uint8, device=dev)
    if err is None:
        err = torch.zeros(1, dtype=torch.int32, device=dev)
    csa2.ced_project_quant(h.to(dev), w.to(dev), torch.tensor(pos, dtype=torch.int32, device=dev),
                           codes, scales, err)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), scales.cpu().numpy(), int(err.item())


def _oracle(h, w):
    B, n, d = h.shape
    c, a = oracle.ced_project(bits(h).reshape(B * n, d), bits(w))
    return c.reshape(B, n, 512), a.reshape(B, n, 512)


def _rows(x, pos, n):
    """Cache rows pos[b] .. pos[b] + n - 1 of every sequence."""
    return np.stack([x[b, pos[b]:pos[b] + n] for b in range(len(pos))])


def _nibbles(codes):
    lo, hi = codes & 0xF, codes >> 4
    return np.stack([lo, hi], -1).reshape(codes.shape[:-1] + (512,))


@pytest.mark.parametrize("B,n,d", [(2, 200, 256), (1, 128, 64), (3, 77, 4160), (1, 513, 1024),
                                   (4, 5000, 128), (2, 9500, 64), (2, 150, 4160)])
def test_integer_inputs_bit_exact(gpu, B, n, d):
    """Ragged token tiles, one d-slice (64), a d that wraps the stage ring (4160 = 65 slices).
    Calls of fewer than 256 token rows run on single CTAs; (3, 77, 4160) and (1, 128, 64) take
    that path. The others run on CTA pairs; (2, 150, 4160) wraps the pairs' 6-stage ring. With
    158 and 150 pair tiles over 74 clusters, each cluster reuses both TMEM accumulators and the
    last wave is partial."""
    rng = np.random.default_rng(B * 7 + n + d)
    h = torch.from_numpy(rng.integers(-3, 4, (B, n, d)).astype(np.float32)).to(torch.bfloat16)
    w = torch.from_numpy(rng.integers(-2, 3, (512, d)).astype(np.float32) / 4).to(torch.bfloat16)
    h[0, 0] = 0.0                                      # an all-zero row: zero scales and codes
    pos = [5 + 37 * b for b in range(B)]
    n_cap = max(pos) + n + 8
    n_cap += (-n_cap) % 8
    codes, scales, err = _run(h, w, pos, n_cap, gpu)
    assert err == 0
    c, _ = _oracle(h, w)
    assert np.all(np.abs(c) < 2.0 ** 23)               # every partial sum is exact in fp32
    oc, osc = oracle.mxfp4_quantize_f32(c.astype(np.float32))
    assert np.array_equal(_rows(scales, pos, n), osc)
    assert np.array_equal(_rows(codes, pos, n), oc)
    # rows outside pos[b] .. pos[b] + n - 1 are untouched
    mask = np.ones(codes.shape[:2], bool)
    for b, p in enumerate(pos):
        mask[b, p:p + n] = False
    assert np.all(codes[mask] == SENTINEL) and np.all(scales[mask] == SENTINEL)


def _e4m3_interval(lo, hi):
    return oracle.e4m3_encode(np.float32(lo)), oracle.e4m3_encode(np.float32(hi))


def test_gaussian_inputs_within_fp32_rounding(gpu):
    B, n, d = 2, 300, 1024
    g = torch.Generator().manual_seed(3)
    h = torch.randn(B, n, d, generator=g).to(torch.bfloat16)
    w = (torch.randn(512, d, generator=g) / 32).to(torch.bfloat16)
    pos = [0, 1000]
    codes, scales, err = _run(h, w, pos, 1304, gpu)
    assert err == 0
    c, a = _oracle(h, w)
    tau = d * 2.0 ** -23 * a
    gc = _nibbles(_rows(codes, pos, n)).reshape(-1, 32, 16)
    gs = _rows(scales, pos, n).reshape(-1, 32)
    cx = c.reshape(-1, 32, 16)
    tx = tau.reshape(-1, 32, 16)
    # scales: E4M3 RNE of (amax / 6) is monotone in amax
    amax = np.abs(cx).max(-1)
    tmax = tx.max(-1)
    s_lo = oracle.e4m3_encode((np.maximum(amax - tmax, 0) / 6).astype(np.float32))
    s_hi = oracle.e4m3_encode(((amax + tmax) / 6).astype(np.float32))
    assert np.all((gs >= s_lo) & (gs <= s_hi)), "a scale outside the fp32-rounding interval"
    # codes: given the GPU's scale, E2M1 RNE of |x| / s is monotone in |x|; the sign may only
    # differ where 0 lies within tau
    s = oracle.e4m3_decode(gs)[..., None]
    ax = np.abs(cx)
    with np.errstate(divide="ignore", invalid="ignore"):
        q_lo = np.where(s > 0, np.maximum(ax - tx, 0) / s, 0).astype(np.float32)
        q_hi = np.where(s > 0, (ax + tx) / s, 0).astype(np.float32)
    m_lo = oracle.e2m1_encode(q_lo.ravel()).reshape(q_lo.shape)
    m_hi = oracle.e2m1_encode(q_hi.ravel()).reshape(q_hi.shape)
    mag = gc & 7
    assert np.all((mag >= m_lo) & (mag <= m_hi)), "a code outside the fp32-rounding interval"
    sign_ok = ((gc >> 3) == (cx < 0)) | (ax <= tx) | (mag == 0)
    assert np.all(sign_ok), "a code with the wrong sign"
    # and in practice the fp32 sum is far closer than tau: nearly every code is the oracle's
    oc, osc = oracle.mxfp4_quantize_f32(c.astype(np.float32))
    same = _nibbles(oc).reshape(gc.shape) == gc
    assert same.mean() > 0.995, f"only {same.mean():.4f} of the codes equal the oracle's"


def test_rows_outside_the_cache_are_skipped_and_flagged(gpu):
    B, n, d = 2, 40, 128
    rng = np.random.default_rng(9)
    h = torch.from_numpy(rng.integers(-3, 4, (B, n, d)).astype(np.float32)).to(torch.bfloat16)
    w = torch.from_numpy(rng.integers(-2, 3, (512, d)).astype(np.float32)).to(torch.bfloat16)
    n_cap = 64
    pos = [40, -3]                    # rows 64..79 of sequence 0 and -3..-1 of sequence 1 invalid
    codes, scales, err = _run(h, w, pos, n_cap, gpu)
    assert err & csa2.DEVERR_POS_RANGE
    c, _ = _oracle(h, w)
    oc, osc = oracle.mxfp4_quantize_f32(c.astype(np.float32))
    assert np.array_equal(codes[0, 40:64], oc[0, :24]) and np.array_equal(scales[0, 40:64], osc[0, :24])
    assert np.array_equal(codes[1, 0:37], oc[1, 3:40]) and np.array_equal(scales[1, 0:37], osc[1, 3:40])
    assert np.all(codes[0, :40] == SENTINEL) and np.all(codes[1, 37:] == SENTINEL)
