"""CPU oracle for the CSA2 decode path: thin numpy/ctypes wrapper over oracle.c.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline arm of
``bench.py`` may import this package. It shares no code with ``sparse_attention_decode_kv_b200``
and neither package imports the other.

Array conventions: bf16 data travel as ``numpy.uint16`` bit patterns; MXFP4 codes, E4M3 scales and
SWA bytes as ``numpy.uint8``; indices as ``numpy.int64`` with -1 as padding.

Every function restates a definition from the pages (cited in oracle.c):
"DeepSeek V4.1 Flash 拆解" (austincafe.tech), section 一 -- layer modes, hierarchical sparse
indexer, MXFP4 main KV, FP8 SWA KV.
"""
from __future__ import annotations

import ctypes

import numpy as np

from . import build as _build

D, HQ, HI, DI, S = 512, 16, 4, 64, 8

_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        path = _build.build()
        _lib = ctypes.CDLL(path)
        _declare(_lib)
    return _lib


_P = ctypes.c_void_p


def _declare(L):
    L.oracle_e2m1_decode.restype = ctypes.c_double
    L.oracle_e2m1_decode.argtypes = [ctypes.c_uint8]
    L.oracle_e4m3_decode.restype = ctypes.c_double
    L.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
    L.oracle_e2m1_encode.restype = ctypes.c_uint8
    L.oracle_e2m1_encode.argtypes = [ctypes.c_float]
    L.oracle_e4m3_encode.restype = ctypes.c_uint8
    L.oracle_e4m3_encode.argtypes = [ctypes.c_float]
    L.oracle_e4m3_encode_array.argtypes = [_P, ctypes.c_int64, _P]
    L.oracle_e2m1_encode_array.argtypes = [_P, ctypes.c_int64, _P]
    L.oracle_mxfp4_quantize_entry.argtypes = [_P, _P, _P]
    L.oracle_mxfp4_quantize_f32.argtypes = [_P, _P, _P]
    L.oracle_ced_project.argtypes = [_P, _P, ctypes.c_int64, ctypes.c_int, _P, _P]
    L.oracle_mxfp4_dequantize_entry.argtypes = [_P, _P, _P]
    L.oracle_swa_quantize_token.argtypes = [_P, _P, _P]
    L.oracle_f64_to_bf16.restype = ctypes.c_uint16
    L.oracle_f64_to_bf16.argtypes = [ctypes.c_double]
    L.oracle_swa_replay.argtypes = [_P, _P, ctypes.c_int, ctypes.c_int, ctypes.c_int, _P, _P, _P,
                                    ctypes.c_int]
    L.oracle_append.restype = ctypes.c_int
    L.oracle_append.argtypes = [_P, _P, ctypes.c_int, ctypes.c_int, _P, ctypes.c_int, _P, _P, _P,
                                _P, _P, ctypes.c_int]
    L.oracle_index_score.restype = ctypes.c_double
    L.oracle_index_score.argtypes = [_P, _P, _P]
    L.oracle_index_scores.argtypes = [_P, _P, _P, ctypes.c_int64, _P, _P]
    L.oracle_topk.restype = ctypes.c_int
    L.oracle_topk.argtypes = [_P, _P, ctypes.c_int64, ctypes.c_int, _P]
    L.oracle_index_full_seq.restype = ctypes.c_int
    L.oracle_index_full_seq.argtypes = [_P, _P, _P, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                                        _P, _P, _P, _P]
    L.oracle_index_reindex_seq.restype = ctypes.c_int
    L.oracle_index_reindex_seq.argtypes = [_P, _P, _P, _P, ctypes.c_int64, ctypes.c_int, _P, _P]
    L.oracle_attend_seq.restype = ctypes.c_int
    L.oracle_attend_seq.argtypes = [_P, ctypes.c_float, _P, _P, _P, ctypes.c_int, _P, _P,
                                    ctypes.c_int, _P, _P, _P]


def _ptr(a):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ------------------------------------------------------------------------------------------ codecs

def e2m1_decode(codes) -> np.ndarray:
    L = lib()
    return np.array([L.oracle_e2m1_decode(int(c)) for c in np.ravel(codes)]).reshape(np.shape(codes))


def e4m3_decode(codes) -> np.ndarray:
    L = lib()
    return np.array([L.oracle_e4m3_decode(int(c)) for c in np.ravel(codes)]).reshape(np.shape(codes))


def e4m3_encode(values) -> np.ndarray:
    v = _c(values, np.float32)
    out = np.empty(v.shape, np.uint8)
    lib().oracle_e4m3_encode_array(_ptr(v), v.size, _ptr(out))
    return out


def e2m1_encode(values) -> np.ndarray:
    v = _c(values, np.float32)
    out = np.empty(v.shape, np.uint8)
    lib().oracle_e2m1_encode_array(_ptr(v), v.size, _ptr(out))
    return out


def mxfp4_quantize(x_bf16) -> tuple[np.ndarray, np.ndarray]:
    """[n, 512] bf16 bits -> (codes [n, 256] u8, scales [n, 32] u8)."""
    x = _c(x_bf16, np.uint16).reshape(-1, D)
    n = x.shape[0]
    codes = np.empty((n, D // 2), np.uint8)
    scales = np.empty((n, D // 16), np.uint8)
    L = lib()
    for i in range(n):
        L.oracle_mxfp4_quantize_entry(_ptr(x[i]), _ptr(codes[i]), _ptr(scales[i]))
    return codes, scales


def mxfp4_quantize_f32(x) -> tuple[np.ndarray, np.ndarray]:
    """fp32 rows [..., 512] -> (codes uint8 [..., 256], scales uint8 [..., 32]); the same
    definition as mxfp4_quantize, applied to fp32 values (the CED projection output)."""
    x = _c(x, np.float32)
    rows = x.reshape(-1, 512)
    codes = np.zeros((rows.shape[0], 256), np.uint8)
    scales = np.zeros((rows.shape[0], 32), np.uint8)
    L = lib()
    for r in range(rows.shape[0]):
        L.oracle_mxfp4_quantize_f32(_ptr(rows[r]), _ptr(codes[r]), _ptr(scales[r]))
    return codes.reshape(x.shape[:-1] + (256,)), scales.reshape(x.shape[:-1] + (32,))


def ced_project(h_bits, w_bits):
    """CED KV projection C = h w^T in double [T1 CED paragraph]. h_bits uint16 (bf16 bits)
    [M, d], w_bits uint16 [512, d] -> (C float64 [M, 512], sum |h w| float64 [M, 512])."""
    h = _c(h_bits, np.uint16)
    w = _c(w_bits, np.uint16)
    M, d = h.shape
    assert w.shape == (512, d)
    c = np.zeros((M, 512), np.float64)
    a = np.zeros((M, 512), np.float64)
    lib().oracle_ced_project(_ptr(h), _ptr(w), M, d, _ptr(c), _ptr(a))
    return c, a


def f64_to_bf16(x) -> np.ndarray:
    """float64 values -> bf16 bit patterns (uint16), one rounding to nearest even."""
    xs = np.asarray(x, np.float64)
    L = lib()
    return np.array([L.oracle_f64_to_bf16(float(v)) for v in xs.ravel()], np.uint16).reshape(xs.shape)


def swa_replay(h_bits, w_bits, N, swa, swa_scale):
    """SWA bounded replay [A abstract; Juju Radar note; T1 "最后的结果"]: rebuild ring slots from
    the last Wr tokens' hidden states. h_bits uint16 [B, Wr, d]; w_bits uint16 [512, d]; N [B];
    swa uint8 [B, W, 512] and swa_scale float32 [B, W] are updated in place (other slots kept)."""
    h = _c(h_bits, np.uint16)
    w = _c(w_bits, np.uint16)
    B, Wr, d = h.shape
    assert w.shape == (512, d)
    n = _c(N, np.int32)
    assert swa.dtype == np.uint8 and swa.flags.c_contiguous and swa.shape[0] == B
    assert swa_scale.dtype == np.float32 and swa_scale.flags.c_contiguous
    W = swa.shape[1]
    lib().oracle_swa_replay(_ptr(h), _ptr(w), B, Wr, d, _ptr(n), _ptr(swa), _ptr(swa_scale), W)


def mxfp4_dequantize(codes, scales) -> np.ndarray:
    c = _c(codes, np.uint8).reshape(-1, D // 2)
    s = _c(scales, np.uint8).reshape(-1, D // 16)
    out = np.empty((c.shape[0], D), np.float64)
    L = lib()
    for i in range(c.shape[0]):
        L.oracle_mxfp4_dequantize_entry(_ptr(c[i]), _ptr(s[i]), _ptr(out[i]))
    return out


def swa_quantize(x_bf16) -> tuple[np.ndarray, np.ndarray]:
    """[n, 512] bf16 bits -> (e4m3 [n, 512] u8, scale [n] f32)."""
    x = _c(x_bf16, np.uint16).reshape(-1, D)
    n = x.shape[0]
    e = np.empty((n, D), np.uint8)
    sc = np.empty((n,), np.float32)
    L = lib()
    for i in range(n):
        L.oracle_swa_quantize_token(_ptr(x[i]), _ptr(e[i]), _ptr(sc[i:i + 1]))
    return e, sc


# ------------------------------------------------------------------------------------------ append

def append(x, ik, pos, n_cap, codes, scales, ik_cache, swa=None, swa_scale=None, W=0) -> None:
    """In-place append of x [B, n, 512] (and ik [B, n, 64]) at rows pos[b] .. pos[b]+n-1."""
    x = _c(x, np.uint16)
    B, n = x.shape[0], x.shape[1]
    ik = None if ik is None else _c(ik, np.uint16)
    pos = _c(pos, np.int32)
    for a in (codes, scales, ik_cache, swa, swa_scale):
        assert a is None or a.flags.c_contiguous
    rc = lib().oracle_append(_ptr(x), _ptr(ik), B, n, _ptr(pos), n_cap, _ptr(codes), _ptr(scales),
                             _ptr(ik_cache), _ptr(swa), _ptr(swa_scale), int(W))
    if rc != 0:
        raise ValueError("append row out of range")


# ------------------------------------------------------------------------------------------ index

def index_scores(iq, w, ik_rows, with_tol=False):
    """Scores of key rows ik_rows [n, 64] for one query iq [4, 64], w [4]."""
    iq = _c(iq, np.uint16)
    w = _c(w, np.float32)
    k = _c(ik_rows, np.uint16).reshape(-1, DI)
    s = np.empty(k.shape[0], np.float64)
    t = np.empty(k.shape[0], np.float64) if with_tol else None
    lib().oracle_index_scores(_ptr(iq), _ptr(w), _ptr(k), k.shape[0], _ptr(s), _ptr(t))
    return (s, t) if with_tol else s


def topk(score, k, index=None) -> np.ndarray:
    score = _c(score, np.float64)
    idx = None if index is None else _c(index, np.int64)
    out = np.empty(k, np.int64)
    lib().oracle_topk(_ptr(score), _ptr(idx), score.size, k, _ptr(out))
    return out


def index_full(iq, w, ik_cache, N, K, P):
    """Full-mode indexer over a batch. iq [B,4,64] u16, w [B,4] f32, ik_cache [B,n_cap,64] u16,
    N [B]. Returns dict(topk [B,K] i64, pool [B,8P] i64, score list, blockmax list)."""
    iq = _c(iq, np.uint16)
    w = _c(w, np.float32)
    B = iq.shape[0]
    topk_out = np.empty((B, K), np.int64)
    pool = np.empty((B, P * S), np.int64)
    scores, bmax = [], []
    L = lib()
    for b in range(B):
        n = int(N[b])
        rows = _c(ik_cache[b, :n], np.uint16)
        sc = np.empty(n, np.float64)
        bm = np.empty((n + S - 1) // S, np.float64)
        rc = L.oracle_index_full_seq(_ptr(iq[b]), _ptr(w[b]), _ptr(rows), n, K, P, _ptr(sc),
                                     _ptr(bm), _ptr(topk_out[b]), _ptr(pool[b]))
        if rc != 0:
            raise MemoryError
        scores.append(sc)
        bmax.append(bm)
    return dict(topk=topk_out, pool=pool, score=scores, blockmax=bmax)


def index_reindex(iq, w, ik_cache, pool, K):
    """Reindex-mode indexer: own iq [B,4,64], w [B,4]; scores only pool [B,L] positions."""
    iq = _c(iq, np.uint16)
    w = _c(w, np.float32)
    pool = _c(pool, np.int64)
    B, Lp = pool.shape
    topk_out = np.empty((B, K), np.int64)
    scores = np.empty((B, Lp), np.float64)
    L = lib()
    for b in range(B):
        rows = _c(ik_cache[b], np.uint16)
        rc = L.oracle_index_reindex_seq(_ptr(iq[b]), _ptr(w[b]), _ptr(rows), _ptr(pool[b]), Lp, K,
                                        _ptr(scores[b]), _ptr(topk_out[b]))
        if rc != 0:
            raise MemoryError
    return dict(topk=topk_out, score=scores)


# ------------------------------------------------------------------------------------------ attend

def attend_seq(q, softmax_scale, codes_rows, scales_rows, idx, swa_rows, swa_scale, swa_len,
               want_weights=False):
    """One sequence. q [16,512] u16; codes_rows [n_cap,256]; scales_rows [n_cap,32];
    idx [K] i64 (-1 padding); swa_rows [W,512] u8; swa_scale [W] f32."""
    q = _c(q, np.uint16)
    idx = _c(idx, np.int64)
    codes_rows = _c(codes_rows, np.uint8)
    scales_rows = _c(scales_rows, np.uint8)
    swa_len = int(swa_len)
    if swa_len > 0:
        swa_rows = _c(swa_rows, np.uint8)
        swa_scale = _c(swa_scale, np.float32)
    else:
        swa_rows = np.zeros((1, D), np.uint8)
        swa_scale = np.zeros((1,), np.float32)
    out = np.empty((HQ, D), np.float32)
    lse = np.empty((HQ,), np.float32)
    n_items = int((idx >= 0).sum()) + swa_len
    wts = np.empty((HQ, max(n_items, 1)), np.float64) if want_weights else None
    rc = lib().oracle_attend_seq(_ptr(q), float(softmax_scale), _ptr(codes_rows), _ptr(scales_rows),
                                 _ptr(idx), idx.size, _ptr(swa_rows), _ptr(swa_scale), swa_len,
                                 _ptr(out), _ptr(lse), _ptr(wts))
    if rc < 0:
        raise MemoryError
    if want_weights:
        return out, lse, wts[:, :n_items]
    return out, lse


def attend(q, softmax_scale, codes, scales, idx, swa, swa_scale, swa_len):
    """Batch. q [B,16,512] u16; codes [B,n_cap,256]; scales [B,n_cap,32]; idx [B,K];
    swa [B,W,512] u8 or None; swa_scale [B,W]; swa_len [B]."""
    B = q.shape[0]
    out = np.empty((B, HQ, D), np.float32)
    lse = np.empty((B, HQ), np.float32)
    for b in range(B):
        sl = int(swa_len[b]) if swa_len is not None else 0
        o, l = attend_seq(q[b], softmax_scale, codes[b], scales[b], idx[b],
                          None if sl == 0 else swa[b], None if sl == 0 else swa_scale[b], sl)
        out[b], lse[b] = o, l
    return out, lse


# ------------------------------------------------------------------------------------------ stack

def run_stack(modes, q, iq, w, ik_cache, codes, scales, N, K, P, swa, swa_scale, swa_len,
              softmax_scale=1.0):
    """One decode step of a CSA2 layer stack ("F" Full, "RI" Reindex, "U" Reuse).

    q [L,B,16,512]; iq / w are indexed by the position of each index-producing layer among the
    F/RI layers ([n_idx,B,4,64] / [n_idx,B,4]). A Reindex layer scores the pool of the most recent
    Full layer; a Reuse layer takes the indices of the most recent index-producing layer. All
    layers read the same main KV, indexer-key cache and SWA ring (cross-layer reuse).
    Returns a list of per-layer dicts (topk, pool when Full, out, lse)."""
    layers = []
    cur_topk = cur_pool = None
    j = 0
    for l, m in enumerate(modes):
        rec = {"mode": m}
        if m == "F":
            r = index_full(iq[j], w[j], ik_cache, N, K, P)
            cur_topk, cur_pool = r["topk"], r["pool"]
            rec.update(topk=cur_topk, pool=cur_pool)
            j += 1
        elif m == "RI":
            r = index_reindex(iq[j], w[j], ik_cache, cur_pool, K)
            cur_topk = r["topk"]
            rec.update(topk=cur_topk)
            j += 1
        elif m != "U":
            raise ValueError(m)
        out, lse = attend(q[l], softmax_scale, codes, scales, cur_topk, swa, swa_scale, swa_len)
        rec.update(out=out, lse=lse, idx=cur_topk)
        layers.append(rec)
    return layers


def cores_used() -> int:
    """The oracle is single-threaded."""
    return 1

