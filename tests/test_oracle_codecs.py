"""Pins for the oracle's format codecs (E2M1, E4M3, MXFP4 groups, FP8 SWA tokens).

Each check compares the oracle with something other than itself: the format tables of the OCP
specifications (golden fixtures), torch's float8_e4m3fn cast (a library routine), exact rational
arithmetic (fractions.Fraction) for the nearest-value-with-ties-to-even rule, and hand-worked
groups. The page "DeepSeek V4.1 Flash 拆解" (austincafe.tech), section 一, fixes the formats: E2M1
codes with one E4M3 scale per 16 channels for the main KV, FP8 for the sliding window.
"""
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def f32(x):
    return np.float32(x)


def bf16_of(values):
    t = torch.tensor(values, dtype=torch.float32).to(torch.bfloat16)
    assert torch.equal(t.float(), torch.tensor(values, dtype=torch.float32)), "not exact in bf16"
    return t.view(torch.int16).numpy().view(np.uint16)


# ------------------------------------------------------------------------------------------ E2M1

def test_e2m1_table_matches_format_definition():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "e2m1_table.txt")) if l[0] != "#"]
    for code_s, val_s in rows:
        code, val = int(code_s, 16), float(val_s)
        got = oracle.e2m1_decode([code])[0]
        assert got == val and np.signbit(got) == np.signbit(val), (code, got, val)


E2M1_MAGS = [Fraction(0), Fraction(1, 2), Fraction(1), Fraction(3, 2), Fraction(2), Fraction(3),
             Fraction(4), Fraction(6)]


def e2m1_bruteforce(r: float) -> int:
    """Nearest magnitude by exact distance; equal distances go to the even code; > 6 -> 6."""
    a = abs(Fraction(float(r)))
    if a > 6:
        mag = 7
    else:
        d = [abs(a - m) for m in E2M1_MAGS]
        best = min(d)
        cands = [i for i, x in enumerate(d) if x == best]
        mag = cands[0] if len(cands) == 1 else [c for c in cands if c % 2 == 0][0]
    return mag | (8 if np.signbit(np.float32(r)) else 0)


def test_e2m1_ties_go_to_even_code():
    ties = {0.25: 0, 0.75: 2, 1.25: 2, 1.75: 4, 2.5: 4, 3.5: 6, 5.0: 6}
    for v, code in ties.items():
        assert oracle.e2m1_encode([v])[0] == code, v
        assert oracle.e2m1_encode([-v])[0] == code | 8, -v


def test_e2m1_saturation_and_sign():
    assert oracle.e2m1_encode([6.0, 6.5, 7.0, 1e30])[0] == 7
    assert list(oracle.e2m1_encode([6.0, 6.5, 7.0, 1e30])) == [7, 7, 7, 7]
    assert list(oracle.e2m1_encode([-0.1, -0.0, 0.0, 0.1])) == [8, 8, 0, 0]


def test_e2m1_encode_matches_exact_nearest_on_dense_sweep():
    rng = np.random.default_rng(0)
    pts = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, 0.5, 1.0, 2.0, 3.0, 4.0]
    vals = []
    for p in pts:  # each grid point and tie point with its fp32 neighbours
        x = np.float32(p)
        vals += [x, np.nextafter(x, np.float32(0)), np.nextafter(x, np.float32(10))]
    vals += list(rng.uniform(-7, 7, 4000).astype(np.float32))
    vals = np.array(vals, np.float32)
    got = oracle.e2m1_encode(vals)
    for v, g in zip(vals, got):
        assert g == e2m1_bruteforce(v), (float(v), g)


# ------------------------------------------------------------------------------------------ E4M3

def test_e4m3_decode_matches_torch_for_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = oracle.e4m3_decode(codes)
    both_nan = np.isnan(ref) & np.isnan(got)
    assert np.all(both_nan | (ref == got))
    assert np.all(np.signbit(ref[~both_nan]) == np.signbit(got[~both_nan]))
    assert oracle.e4m3_decode([0x7E])[0] == 448.0 and oracle.e4m3_decode([0x01])[0] == 2.0 ** -9


def _torch_e4m3(v):
    return torch.from_numpy(np.ascontiguousarray(v, np.float32)).to(torch.float8_e4m3fn) \
        .view(torch.uint8).numpy()


def test_e4m3_encode_matches_torch_on_all_bf16_values():
    bits = np.arange(65536, dtype=np.uint32) << 16
    v = bits.view(np.float32)
    keep = np.isfinite(v) & (np.abs(v) < 464.0)  # torch does not saturate above 464 (gives NaN)
    v = v[keep]
    assert np.array_equal(oracle.e4m3_encode(v), _torch_e4m3(v))


def test_e4m3_encode_matches_torch_on_dense_fp32_sweep():
    rng = np.random.default_rng(1)
    # every exponent that E4M3 can reach (and a little below), random mantissas, both signs
    e = rng.integers(-20, 9, 1 << 20)
    m = rng.uniform(1.0, 2.0, 1 << 20)
    v = (np.ldexp(m, e) * rng.choice([-1.0, 1.0], 1 << 20)).astype(np.float32)
    # exact midpoints between neighbouring E4M3 values and their fp32 neighbours
    grid = np.sort(np.abs(oracle.e4m3_decode(np.arange(127, dtype=np.uint8))))
    mids = ((grid[1:] + grid[:-1]) / 2).astype(np.float32)
    v = np.concatenate([v, mids, np.nextafter(mids, np.float32(0)),
                        np.nextafter(mids, np.float32(1e9)), -mids])
    v = v[np.abs(v) < 464.0]
    assert np.array_equal(oracle.e4m3_encode(v), _torch_e4m3(v))


def test_e4m3_saturates_to_448():
    big = np.array([448.0, 460.0, 464.0, 465.0, 1000.0, 3e38], np.float32)
    assert list(oracle.e4m3_encode(big)) == [0x7E] * 6
    assert list(oracle.e4m3_encode(-big)) == [0xFE] * 6


# ------------------------------------------------------------------------------------------ MXFP4

def _read_groups():
    out = []
    for line in open(os.path.join(GOLDEN, "mxfp4_groups.txt")):
        if line.startswith("#") or not line.strip():
            continue
        name, vals, scale, codes = [p.strip() for p in line.split("|")]
        out.append((name, [float(x) for x in vals.split()], int(scale, 16),
                    [int(c, 16) for c in codes.split()]))
    return out


@pytest.mark.parametrize("grp", _read_groups(), ids=lambda g: g[0])
def test_mxfp4_hand_worked_groups(grp):
    name, vals, scale, codes = grp
    x = np.zeros(512, np.uint16)
    x[:16] = bf16_of(vals)
    c, s = oracle.mxfp4_quantize(x[None])
    assert s[0, 0] == scale, name
    assert list(c[0, :8]) == codes, name


def _e4m3_exact_nearest(q: Fraction) -> int:
    grid = [Fraction(oracle.e4m3_decode([c])[0]) for c in range(127)]
    if q >= 448:
        return 0x7E
    d = [abs(q - g) for g in grid]
    best = min(d)
    cands = [i for i, x in enumerate(d) if x == best]
    return cands[0] if len(cands) == 1 else [c for c in cands if c % 2 == 0][0]


def test_mxfp4_matches_exact_rational_definition():
    """Scale = nearest E4M3 to the exact rational amax/6 and code = nearest E2M1 to the exact
    rational x/scale: the oracle's fp32 quotients give the same bytes on bf16 inputs."""
    rng = np.random.default_rng(2)
    torch.manual_seed(0)
    n = 96
    x = torch.randn(n, 512)
    x[::7] *= 40.0
    x[::11] *= 1e-3
    x[3, 16:32] = torch.tensor([6.375, 3.1875] + [0.5] * 14)  # amax/6 = 1.0625, an E4M3 tie
    xb = x.to(torch.bfloat16)
    bits = xb.view(torch.int16).numpy().view(np.uint16)
    codes, scales = oracle.mxfp4_quantize(bits)
    xf = xb.float().numpy()
    for i in rng.choice(n, 24, replace=False).tolist() + [3]:
        for g in range(32):
            grp = xf[i, 16 * g:16 * g + 16]
            amax = max(abs(Fraction(float(v))) for v in grp)
            sc = _e4m3_exact_nearest(amax / 6)
            assert scales[i, g] == sc, (i, g)
            s = Fraction(oracle.e4m3_decode([sc])[0])
            for j in range(16):
                byte = codes[i, 8 * g + j // 2]
                code = (byte >> 4) if j % 2 else (byte & 15)
                if s == 0:
                    assert code == 0
                    continue
                r = Fraction(float(grp[j])) / s
                assert code == e2m1_bruteforce_fraction(r, np.signbit(grp[j])), (i, g, j)


def e2m1_bruteforce_fraction(r: Fraction, neg: bool) -> int:
    a = abs(r)
    if a > 6:
        mag = 7
    else:
        d = [abs(a - m) for m in E2M1_MAGS]
        best = min(d)
        cands = [i for i, x in enumerate(d) if x == best]
        mag = cands[0] if len(cands) == 1 else [c for c in cands if c % 2 == 0][0]
    return mag | (8 if neg else 0)


def test_mxfp4_round_trip_bound():
    """|x - s*c| <= s * (half the local E2M1 gap), plus the excess over 6*s when the scale
    rounded down."""
    torch.manual_seed(3)
    x = torch.randn(64, 512) * torch.exp(torch.randn(64, 1) * 2)
    xb = x.to(torch.bfloat16)
    bits = xb.view(torch.int16).numpy().view(np.uint16)
    codes, scales = oracle.mxfp4_quantize(bits)
    deq = oracle.mxfp4_dequantize(codes, scales)
    xf = xb.double().numpy()
    s = oracle.e4m3_decode(scales.ravel()).reshape(64, 32).repeat(16, axis=1)
    a = np.abs(xf)
    half_gap = np.where(a < 2 * s, 0.25, np.where(a < 4 * s, 0.5, 1.0)) * s
    excess = np.maximum(a - 6 * s, 0)
    assert np.all(np.abs(xf - deq) <= half_gap + excess + 1e-300)
    assert np.all(np.sign(deq) * np.sign(xf) >= 0)


def test_mxfp4_exhaustive_bf16_at_unit_scale():
    """Groups anchored by a 6.0 have scale 1.0, so every code is the E2M1 RNE of x itself: all
    bf16 values of magnitude up to 8 are checked against the exact nearest-value rule."""
    bits = np.arange(65536, dtype=np.uint32)
    v = (bits << 16).view(np.float32)
    v = v[np.isfinite(v) & (np.abs(v) <= 8.0)]
    vb = torch.from_numpy(v.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    per = 15
    ngrp = (len(vb) + per - 1) // per
    rows = np.zeros((ngrp + 31) // 32 * 32 * 16, np.uint16)
    six = bf16_of([6.0])[0]
    flat = []
    for g in range(ngrp):
        chunk = vb[g * per:(g + 1) * per]
        rows[g * 16] = six
        rows[g * 16 + 1:g * 16 + 1 + len(chunk)] = chunk
        flat.append(chunk)
    codes, scales = oracle.mxfp4_quantize(rows.reshape(-1, 512))
    # every group whose true amax is 6 has scale 1.0 (0x38); groups with |x| > 6 rescale, skip them
    allc = np.empty((codes.shape[0], 512), np.uint8)
    allc[:, 0::2] = codes & 15
    allc[:, 1::2] = codes >> 4
    allc = allc.reshape(-1, 16)
    sc = scales.reshape(-1)
    vf = v
    k = 0
    for g in range(ngrp):
        chunk = vf[g * per:(g + 1) * per]
        if np.max(np.abs(chunk)) <= 6.0:
            assert sc[g] == 0x38
            for j, xv in enumerate(chunk):
                assert allc[g, j + 1] == e2m1_bruteforce(xv), (float(xv), allc[g, j + 1])
                k += 1
    assert k > 30000


# ------------------------------------------------------------------------------------------ FP8 SWA

def test_swa_token_matches_torch_division_and_cast():
    """Scale = fp32 amax/448; element = E4M3 RNE of the fp32 quotient x/scale (torch computes both
    the quotient and the cast independently)."""
    torch.manual_seed(4)
    x = (torch.randn(40, 512) * torch.exp(torch.randn(40, 1) * 3)).to(torch.bfloat16)
    x[5] = 0
    bits = x.view(torch.int16).numpy().view(np.uint16)
    e, sc = oracle.swa_quantize(bits)
    xf = x.float()
    amax = xf.abs().amax(1)
    s_ref = amax / 448.0
    assert np.array_equal(sc, s_ref.numpy())
    q = torch.where(s_ref[:, None] > 0, xf / s_ref[:, None].clamp_min(1e-45), torch.zeros_like(xf))
    ref = q.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ref[5] = 0
    assert np.array_equal(e, ref)


def test_swa_round_trip_bound():
    torch.manual_seed(5)
    x = torch.randn(16, 512).to(torch.bfloat16)
    e, sc = oracle.swa_quantize(x.view(torch.int16).numpy().view(np.uint16))
    deq = oracle.e4m3_decode(e.ravel()).reshape(16, 512) * sc[:, None].astype(np.float64)
    xf = x.double().numpy()
    # relative 2^-4 for normal E4M3 values, absolute s * 2^-10 in the subnormal range
    bound = np.maximum(np.abs(xf) * 2.0 ** -4, sc[:, None] * 2.0 ** -10)
    assert np.all(np.abs(xf - deq) <= bound * (1 + 1e-12))


def test_append_ring_keeps_last_w_tokens():
    torch.manual_seed(6)
    B, n, W, n_cap = 2, 11, 4, 32
    x = torch.randn(B, n, 512).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    ik = torch.randn(B, n, 64).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    pos = np.array([3, 17], np.int32)
    codes = np.zeros((B, n_cap, 256), np.uint8)
    scales = np.zeros((B, n_cap, 32), np.uint8)
    ikc = np.zeros((B, n_cap, 64), np.uint16)
    swa = np.zeros((B, W, 512), np.uint8)
    swsc = np.zeros((B, W), np.float32)
    oracle.append(x, ik, pos, n_cap, codes, scales, ikc, swa, swsc, W)
    for b in range(B):
        c, s = oracle.mxfp4_quantize(x[b])
        assert np.array_equal(codes[b, pos[b]:pos[b] + n], c)
        assert np.array_equal(scales[b, pos[b]:pos[b] + n], s)
        assert np.array_equal(ikc[b, pos[b]:pos[b] + n], ik[b])
        assert not codes[b, :pos[b]].any() and not codes[b, pos[b] + n:].any()
        e, es = oracle.swa_quantize(x[b])
        for i in range(n - W, n):  # only the last W tokens survive, in slot (position mod W)
            slot = (pos[b] + i) % W
            assert np.array_equal(swa[b, slot], e[i]) and swsc[b, slot] == es[i]
    with pytest.raises(ValueError):
        oracle.append(x, ik, np.array([0, 30], np.int32), n_cap, codes, scales, ikc, swa, swsc, W)
