"""Pins of the oracle's CED KV projection and of its MXFP4 quantiser for fp32 rows.

Method: "DeepSeek V4.1 Flash 拆解" (austincafe.tech), section 一, CED paragraph (the decoder's
global KV is projected from the middle layer's hidden state, C_l = H_{L/2} W^KV_l) and the FP4 KV
cache paragraph (E2M1 + one E4M3 scale per 16 channels). The projection is pinned to numpy's own
matrix product; the fp32 quantiser is pinned to the bf16 quantiser (itself pinned to the OCP
tables) on values both can take, and to hand-worked groups where fp32 values sit on or next to an
E2M1 midpoint.
"""
import numpy as np
import pytest

import oracle


def _bf16_bits(x):
    """float32 -> bf16 bits (round to nearest even), as numpy uint16."""
    u = np.asarray(x, np.float32).view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)
    return r


def _bf16_to_f64(b):
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


@pytest.mark.parametrize("M,d", [(1, 64), (5, 128), (17, 320)])
def test_projection_equals_numpy_matmul(M, d):
    rng = np.random.default_rng(M * 1000 + d)
    h = _bf16_bits(rng.standard_normal((M, d)))
    w = _bf16_bits(rng.standard_normal((512, d)) * 0.1)
    c, a = oracle.ced_project(h, w)
    hf, wf = _bf16_to_f64(h), _bf16_to_f64(w)
    ref = hf @ wf.T                       # row m, channel j: sum_k h[m,k] w[j,k]
    assert np.allclose(c, ref, rtol=1e-12, atol=1e-12)
    assert np.allclose(a, np.abs(hf) @ np.abs(wf).T, rtol=1e-12, atol=1e-12)
    # the orientation matters: w is [channel, d], not [d, channel]
    if d != 512:
        assert c.shape == (M, 512)


def test_projection_one_hot_picks_a_weight_column():
    d = 64
    h = np.zeros((3, d), np.uint16)
    for m, k in enumerate([0, 17, 63]):
        h[m, k] = _bf16_bits(np.float32(2.0))
    w = _bf16_bits(np.arange(512 * d, dtype=np.float32).reshape(512, d) % 251 - 125)
    c, _ = oracle.ced_project(h, w)
    wf = _bf16_to_f64(w)
    for m, k in enumerate([0, 17, 63]):
        assert np.array_equal(c[m], 2.0 * wf[:, k])


def test_fp32_quantiser_equals_bf16_quantiser_on_bf16_values():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((64, 512)).astype(np.float32)
    x[::7] *= 40.0
    x[3, :16] = 0.0                        # zero group -> zero scale, zero codes
    x[4, 16:32] = -0.0
    x[5, :16] = 1e-30                      # scale underflows to 0
    xb = _bf16_bits(x)
    xf = (xb.astype(np.uint32) << 16).view(np.float32)
    c1, s1 = oracle.mxfp4_quantize(xb)
    c2, s2 = oracle.mxfp4_quantize_f32(xf)
    assert np.array_equal(s1, s2)
    assert np.array_equal(c1, c2)


def _group(values):
    x = np.zeros(512, np.float32)
    x[:len(values)] = np.asarray(values, np.float32)
    codes, scales = oracle.mxfp4_quantize_f32(x[None])
    nib = [(codes[0, j // 2] >> (4 * (j % 2))) & 0xF for j in range(16)]
    return int(scales[0, 0]), nib


def test_fp32_groups_worked_by_hand():
    # amax 6 -> scale 6 / 6 = 1.0 = E4M3 0x38; every quotient is the value itself
    up = np.nextafter(np.float32(0.25), np.float32(1.0))     # one fp32 ulp above a midpoint
    down = np.nextafter(np.float32(0.75), np.float32(0.0))   # one ulp below a midpoint
    # amax 6.3: 6.3 / 6 = 1.05 rounds to the E4M3 value 1.0 (below the midpoint 1.0625), so 6.3
    # itself lands above 6 and saturates
    sc, nib = _group([6.0, 0.25, up, 0.75, down, 2.5, -2.5, 5.0, 6.3, -0.0, 1.75])
    assert sc == 0x38
    # 6 -> 7 (6.0); 0.25 tie -> 0 (even); just above -> 1 (0.5); 0.75 tie -> 2 (1.0);
    # just below -> 1 (0.5); 2.5 tie -> 4 (2.0); -2.5 -> 0x8|4; 5.0 tie -> 6 (4.0);
    # 6.3 saturates -> 7; -0.0 -> 0x8; 1.75 tie -> 4 (2.0)
    assert nib[:11] == [7, 0, 1, 2, 1, 4, 12, 6, 7, 8, 4]
    # amax 7.5: 7.5 / 6 = 1.25, an E4M3 value; 0.625 / 1.25 = 0.5 -> code 1
    sc, nib = _group([7.5, 0.625, -0.3125])
    assert sc == 0x3A and nib[:3] == [7, 1, 8 | 0]   # 0.3125 / 1.25 = 0.25 tie -> 0, sign kept
