"""Pins of the oracle's SWA bounded replay and of its double -> bf16 rounding.

Method: "DeepSeek-V4.1-Flash: Pushing the Limits of KV Cache Compression" (abstract: SWA Bounded
Replay keeps the persistent KV cache at about 1/8), the Juju Radar note on the report (the
persistent cache rebuilds the local sliding-window state instead of storing it) and "DeepSeek
V4.1 Flash 拆解" (austincafe.tech), section 一 (FP8 SWA KV). Reading: a restore rebuilds ring slot
p mod W from the hidden state of the token at position p, x = bf16_RNE(h w^T), with the same SWA
codec an append of x uses.

The rounding is pinned to torch's float32 -> bfloat16 conversion (one rounding, so equal on
float32-exact inputs) and to hand-worked ties, including one that a double -> float -> bf16 path
would round the wrong way. The replay is pinned to the oracle's append (itself pinned to the OCP
E4M3 table) fed with numpy's own integer matrix product.
"""
import numpy as np
import pytest
import torch

import oracle


def _bf16_of_f32(x):
    t = torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def test_f64_to_bf16_hand_cases():
    cases = {
        1.0: 0x3F80,
        1.0 + 2.0 ** -8: 0x3F80,                   # tie -> even (1.0)
        1.0 + 2.0 ** -8 + 2.0 ** -40: 0x3F81,      # just above the tie; via float32 it would tie
        1.0 + 3 * 2.0 ** -8: 0x3F82,               # tie between 0x3F81 and 0x3F82 -> even
        -2.5: 0xC020,
        257.0: 0x4380,                             # 256 and 258 tie -> 256
        259.0: 0x4382,                             # 258 and 260 tie -> 260 (even significand)
        2.0 ** -130: 0x0008,                       # subnormal, exact
        2.0 ** -134: 0x0000,                       # half the smallest subnormal: tie -> 0
        3 * 2.0 ** -135: 0x0001,                   # above half -> smallest subnormal
        3.4e38: 0x7F80,                            # rounds past the largest finite -> inf
        -0.0: 0x8000,
    }
    got = oracle.f64_to_bf16(np.array(list(cases)))
    assert [int(g) for g in got] == [int(v) for v in cases.values()]


def test_f64_to_bf16_equals_torch_on_float32_values():
    rng = np.random.default_rng(1)
    x = np.concatenate([
        rng.standard_normal(20000).astype(np.float32),
        (rng.standard_normal(2000) * 1e-39).astype(np.float32),   # float32 subnormals
        (rng.standard_normal(2000) * 1e37).astype(np.float32),
        np.array([3.3895e38, -3.3895e38, 1e-45, 0.0], np.float32),
    ])
    assert np.array_equal(oracle.f64_to_bf16(x.astype(np.float64)), _bf16_of_f32(x))


def _ring(B, W, fill=0xAB):
    return np.full((B, W, 512), fill, np.uint8), np.full((B, W), -1.0, np.float32)


def _bits_of_exact(x):
    """bf16 bits of values that bf16 holds exactly (checked)."""
    b = _bf16_of_f32(x.astype(np.float32))
    back = (b.astype(np.uint32) << 16).view(np.float32)
    assert np.array_equal(back.astype(np.float64), x)
    return b


@pytest.mark.parametrize("B,Wr,W,d,N", [(2, 8, 8, 64, [8, 20]), (1, 5, 12, 128, [30]),
                                        (3, 6, 6, 64, [4, 6, 0])])
def test_replay_equals_append_of_the_projected_rows(B, Wr, W, d, N):
    """Integer inputs, |x| <= 128: every projected value is exact in bf16, so the replayed ring must
    equal the ring an append of x = h w^T (numpy's integer product) at the same positions writes."""
    rng = np.random.default_rng(B * 100 + Wr + d)
    hi = rng.integers(-2, 3, (B, Wr, d))
    wi = rng.integers(-1, 2, (512, d))
    x = np.einsum("brk,jk->brj", hi, wi).astype(np.float64)
    assert np.abs(x).max() <= 256
    h_bits = _bits_of_exact(hi.astype(np.float64))
    w_bits = _bits_of_exact(wi.astype(np.float64))
    swa, sc = _ring(B, W)
    oracle.swa_replay(h_bits, w_bits, N, swa, sc)
    # the same rows appended one token at a time at their positions
    swa2, sc2 = _ring(B, W)
    n_cap = max(max(N), 1) + 8
    codes = np.zeros((B, n_cap, 256), np.uint8)
    scales = np.zeros((B, n_cap, 32), np.uint8)
    ikc = np.zeros((B, n_cap, 64), np.uint16)
    xb = _bits_of_exact(x)
    for b in range(B):
        for r in range(Wr):
            p = N[b] - Wr + r
            if p < 0:
                continue
            one = np.zeros((B, 1, 512), np.uint16)
            pos = np.full(B, n_cap - 1, np.int32)
            one[b, 0] = xb[b, r]
            pos[b] = p
            # every sequence appends one row; only sequence b's row is a real token here
            ring_b, ring_s = swa2.copy(), sc2.copy()
            oracle.append(one, None, pos, n_cap, codes, scales, ikc, ring_b, ring_s, W)
            swa2[b], sc2[b] = ring_b[b], ring_s[b]
    assert np.array_equal(swa, swa2)
    assert np.array_equal(sc, sc2)


def test_replay_rounds_the_projection_to_bf16():
    """x = 257 is not a bf16 value: the replayed row is that of 256 (the nearest-even bf16)."""
    d = 64
    h = np.zeros((1, 1, d))
    h[0, 0, :2] = [1.0, 1.0]
    w = np.zeros((512, d))
    w[:, 0] = 256.0
    w[:, 1] = 1.0                                 # every channel: 256 + 1 = 257
    w[7, 1] = -3.0                                # channel 7: 253, exact
    swa, sc = _ring(1, 4)
    oracle.swa_replay(_bits_of_exact(h), _bits_of_exact(w), [3], swa, sc)
    x = np.full(512, 256.0)
    x[7] = 253.0
    e, s = oracle.swa_quantize(_bits_of_exact(x)[None])
    assert np.array_equal(swa[0, 2], e[0]) and sc[0, 2] == s[0]   # position 2 -> slot 2
    assert np.all(swa[0, [0, 1, 3]] == 0xAB) and np.all(sc[0, [0, 1, 3]] == -1.0)


def test_replay_slots_and_short_sequences():
    """Slot p mod W for p = N - Wr .. N - 1; rows with p < 0 are skipped; other slots are kept."""
    B, Wr, W, d = 3, 4, 6, 64
    rng = np.random.default_rng(7)
    h = rng.integers(1, 3, (B, Wr, d)).astype(np.float64)   # every row non-zero
    w = rng.integers(1, 2, (512, d)).astype(np.float64)
    N = [9, 2, 0]
    swa, sc = _ring(B, W)
    oracle.swa_replay(_bits_of_exact(h), _bits_of_exact(w), N, swa, sc)
    written = {0: {5 % 6, 6 % 6, 7 % 6, 8 % 6}, 1: {0, 1}, 2: set()}
    for b in range(B):
        for slot in range(W):
            touched = sc[b, slot] != -1.0
            assert touched == (slot in written[b]), (b, slot)
    # sequence 1 holds tokens 0 and 1: rows r = 2 and 3 of its window
    x = np.einsum("rk,jk->rj", h[1], w)
    e, s = oracle.swa_quantize(_bits_of_exact(x[2:4]))
    assert np.array_equal(swa[1, 0:2], e) and np.array_equal(sc[1, 0:2], s)
