"""Shared test helpers: bf16 bit views, the Top-K boundary-swap rule and tolerances."""
from __future__ import annotations

import numpy as np
import torch

# Attention outputs: max|out - ref| <= ATT_REL * max|ref| + ATT_ABS over one call's output.
ATT_REL, ATT_ABS = 1e-3, 1e-4
# lse: fp32 logits and exp/log in fp32 against an fp64 reference.
LSE_REL, LSE_ABS = 1e-5, 1e-4


def bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor (any device) -> numpy uint16 bit patterns."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def check_attention(out, lse, ref_out, ref_lse):
    out = np.asarray(out, np.float64)
    ref_out = np.asarray(ref_out, np.float64)
    err = np.abs(out - ref_out).max() if out.size else 0.0
    bound = ATT_REL * np.abs(ref_out).max() + ATT_ABS
    assert err <= bound, f"attention max|d| {err:.3e} > {bound:.3e}"
    if lse is not None:
        lse = np.asarray(lse, np.float64)
        ref_lse = np.asarray(ref_lse, np.float64)
        inf = np.isneginf(ref_lse)
        assert np.array_equal(np.isneginf(lse), inf), "lse -inf pattern differs"
        d = np.abs(lse[~inf] - ref_lse[~inf])
        assert np.all(d <= LSE_ABS + LSE_REL * np.abs(ref_lse[~inf])), f"lse max|d| {d.max():.3e}"
    return err


def check_selection(gpu_sel, oracle_sel, score_of, tol_of, what="topk", log=None):
    """Compare a GPU selection with the oracle's.

    gpu_sel / oracle_sel: iterables of selected ids (-1 ignored). score_of / tol_of: callables
    giving the oracle's fp64 score and the fp32 rounding bound of an id. The sets must have the
    same size; a GPU-only id j and an oracle-only id i are a tolerated boundary swap only if
    score(i) - score(j) <= tol(i) + tol(j), i.e. fp32 rounding could have reordered them.
    Returns the list of tolerated swaps (each logged)."""
    g = set(int(v) for v in gpu_sel if v >= 0)
    o = set(int(v) for v in oracle_sel if v >= 0)
    assert len(g) == len(o), f"{what}: GPU selected {len(g)}, oracle {len(o)}"
    g_only, o_only = sorted(g - o), sorted(o - g)
    swaps = []
    for i in o_only:
        for j in g_only:
            gap = score_of(i) - score_of(j)
            bound = tol_of(i) + tol_of(j)
            assert gap <= bound, (f"{what}: GPU chose {j} (score {score_of(j)!r}) over {i} "
                                  f"(score {score_of(i)!r}); gap {gap:.3e} > fp32 bound {bound:.3e}")
    for i, j in zip(o_only, g_only):
        swaps.append((i, j, score_of(i), score_of(j)))
        msg = f"TOPK-SWAP {what}: oracle {i} ({score_of(i)!r}) <-> GPU {j} ({score_of(j)!r})"
        print(msg)
        if log is not None:
            log.append(msg)
    return swaps


def ascending_padded(sel, k):
    """Selections are written ascending with -1 padding at the end."""
    sel = np.asarray(sel)
    n = int((sel >= 0).sum())
    assert np.all(sel[n:] == -1), "padding must be trailing -1"
    assert np.all(np.diff(sel[:n]) > 0), "indices must be strictly ascending"
    assert len(sel) == k
