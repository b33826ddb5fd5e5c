"""Pins for the oracle's indexer-score tolerance tau (the bound that gates every Top-K swap).

tau = 2^-16 * sum_h |w_h| * sum_i |q[h,i] * k[i]| must (a) cover what fp32 accumulation of the
score can lose in any summation order, and (b) stay close enough to that loss that a real ranking
error cannot hide under it. Pinned by: hand-worked cases (tests/golden/score_tol.txt, including a
worst-order fp32 sum whose error is known in closed form) and a sweep of fp32 sums in many orders,
emulated with numpy float32 (IEEE round-to-nearest-even), against the oracle's fp64 score.

Score definition: "DeepSeek V4.1 Flash 拆解" (austincafe.tech), section 一, hierarchical sparse
indexer, with the head sum I = sum_h w_h ReLU(q_h . k).
"""
import os
from fractions import Fraction

import numpy as np

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "score_tol.txt")


def _bf16(a):
    """bf16 bit patterns of values that are exactly bf16 (asserted)."""
    f = np.asarray(a, np.float32)
    bits = f.view(np.uint32)
    assert np.all(bits & 0xFFFF == 0), "value is not exactly bf16"
    return (bits >> 16).astype(np.uint16)


def _case(name):
    q = np.zeros((4, 64), np.float32)
    k = np.zeros(64, np.float32)
    if name == "ones":
        q[:], k[:], w = 1.0, 1.0, [1.0, 0.5, 2.0, -1.0]
    elif name == "onehot":
        k[:] = 7.0
        for h, (a, c, kv) in enumerate([(2.0, 0, 1.5), (-3.0, 5, 2.0), (0.5, 63, -4.0),
                                        (1.0, 17, 0.25)]):
            q[h, c] = a
            k[c] = kv
        w = [1.0, 1.25, -0.75, 2.0]
    elif name == "cancel":
        q[:] = np.where(np.arange(64) % 2 == 0, 1.0, -1.0)
        k[:], w = 0.5, [1.0, 1.0, 1.0, 1.0]
    elif name == "adversarial":
        q[0, 0], k[0] = 1.0, 1.0
        q[0, 1:] = 2.0 ** -12
        k[1:] = 2.0 ** -12 * (1 + 2.0 ** -7)
        w = [1.0, 1.0, 1.0, 1.0]
    else:
        raise KeyError(name)
    return q, k, np.asarray(w, np.float32)


def _golden():
    cases = {}
    for line in open(GOLDEN):
        if not line.strip() or line.startswith("#"):
            continue
        tok = line.split()
        cases[tok[0]] = {tok[i]: Fraction(tok[i + 1]) for i in range(1, len(tok), 2)}
    return cases


def test_golden_scores_and_tolerances():
    g = _golden()
    assert set(g) == {"ones", "onehot", "cancel", "adversarial"}
    for name, want in g.items():
        q, k, w = _case(name)
        s, t = oracle.index_scores(_bf16(q), w, _bf16(k)[None, :], with_tol=True)
        assert Fraction(float(s[0])) == want["score"], (name, s[0])
        assert Fraction(float(t[0])) == want["tau"], (name, t[0])


def test_worst_order_fp32_error_is_covered_and_tau_is_not_vacuous():
    g = _golden()["adversarial"]
    q, k, w = _case("adversarial")
    # left-to-right fp32 accumulation of head 0's products (products are exact in fp32)
    prod = (q[0] * k).astype(np.float32)
    acc = np.float32(0.0)
    for p in prod:
        acc = np.float32(acc + p)
    assert Fraction(float(acc)) == g["fp32_sequential"]
    s, t = oracle.index_scores(_bf16(q), w, _bf16(k)[None, :], with_tol=True)
    err = abs(Fraction(float(acc)) - Fraction(float(s[0])))
    assert err == Fraction(8001, 2 ** 31)
    assert Fraction(float(t[0])) >= err, "tau misses an error fp32 really makes"
    assert Fraction(float(t[0])) <= 16 * err, "tau is far looser than a real fp32 error"


def _fp32_scores(q, k, w, order, rng):
    """fp32 scores of rows k [R,64] for q [4,64], w [4] with one summation order per call."""
    R = k.shape[0]
    prod = (k[:, None, :] * q[None, :, :]).astype(np.float32)  # [R,4,64], exact
    if order == "sequential":
        dots = np.add.accumulate(prod, axis=2, dtype=np.float32)[:, :, -1]
    elif order == "reversed":
        dots = np.add.accumulate(prod[:, :, ::-1], axis=2, dtype=np.float32)[:, :, -1]
    elif order == "permuted":
        perm = rng.permutation(64)
        dots = np.add.accumulate(prod[:, :, perm], axis=2, dtype=np.float32)[:, :, -1]
    elif order == "pairwise":
        p = prod
        while p.shape[2] > 1:
            p = (p[:, :, 0::2] + p[:, :, 1::2]).astype(np.float32)
        dots = p[:, :, 0]
    elif order == "blocks16":  # four 16-wide partial sums, then accumulated across blocks
        part = np.add.accumulate(prod.reshape(R, 4, 4, 16), axis=3, dtype=np.float32)[..., -1]
        dots = np.add.accumulate(part, axis=2, dtype=np.float32)[:, :, -1]
    else:
        raise KeyError(order)
    relu = np.maximum(dots, np.float32(0.0))
    terms = (relu * w[None, :]).astype(np.float32)
    hp = rng.permutation(4)
    return np.add.accumulate(terms[:, hp], axis=1, dtype=np.float32)[:, -1]


def test_tau_covers_fp32_scores_in_many_orders():
    rng = np.random.default_rng(20261202)
    worst = 0.0
    for trial in range(12):
        R = 2048
        qf = rng.standard_normal((4, 64)).astype(np.float32)
        kf = rng.standard_normal((R, 64)).astype(np.float32)
        if trial % 3 == 1:  # heavy tails: a few large components
            kf[rng.random((R, 64)) < 0.02] *= 64.0
        if trial % 3 == 2:  # near-cancelling dot products: k almost orthogonal to each head
            kf -= (kf @ qf[0])[:, None] * qf[0][None, :] / float(qf[0] @ qf[0])
        w = rng.uniform(-1.5, 1.5, 4).astype(np.float32)
        # round to bf16 (truncate to a bf16-exact value: any bf16 input will do)
        qb = (qf.view(np.uint32) >> 16).astype(np.uint16)
        kb = (kf.view(np.uint32) >> 16).astype(np.uint16)
        q = (qb.astype(np.uint32) << 16).view(np.float32)
        k = (kb.astype(np.uint32) << 16).view(np.float32)
        s, t = oracle.index_scores(qb, w, kb, with_tol=True)
        for order in ("sequential", "reversed", "permuted", "pairwise", "blocks16"):
            f = _fp32_scores(q, k, w, order, rng).astype(np.float64)
            err = np.abs(f - s)
            assert np.all(err <= t), (trial, order, float((err / t).max()))
            worst = max(worst, float((err / np.where(t > 0, t, 1.0)).max()))
    # random inputs lose far less than the worst order; the bound still sits within 2^12 of them
    assert worst > 2.0 ** -12, worst
