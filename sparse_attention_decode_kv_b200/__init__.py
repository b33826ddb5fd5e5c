"""CSA2 sparse-attention decode over an MXFP4 KV cache on B200 (sm_100a).

Thin ctypes binding of ``libcsa2.so`` (built in-tree by ``build.py``; C ABI in
``include/csa2.h``). Every function takes torch CUDA tensors, checks dtype/shape/contiguity,
and passes raw device pointers and the current CUDA stream to the library. All compute runs in
the library's kernels; there is no fallback path. Importing the package does not need a GPU, but
any call fails loudly if ``libcsa2.so`` is missing.

Method ("DeepSeek V4.1 Flash 拆解", austincafe.tech, section 一): Full / Reindex / Reuse CSA2 layer
modes, the hierarchical sparse indexer (Top-512 then 2048 blocks x 8 positions), the MXFP4 main KV
(E2M1 + one E4M3 scale per 16 channels) and the FP8 sliding-window KV.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

D, HQ, HI, DI, S = 512, 16, 4, 64, 8
MODE_FULL, MODE_REINDEX, MODE_REUSE = 0, 1, 2
DEVERR_INDEX_RANGE, DEVERR_POS_RANGE, DEVERR_TIMEOUT, DEVERR_NLEN = 1, 2, 4, 8

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcsa2.so")
_lib: Optional[ctypes.CDLL] = None


class Csa2Error(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn}: {status_string(status)} ({status})")
        self.status = status


def lib() -> ctypes.CDLL:
    """The loaded libcsa2.so; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m sparse_attention_decode_kv_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        L.csa2_append_quant.argtypes = [P, P, I, I, P, I, P, P, P, P, P, I, P, P]
        L.csa2_ced_project_quant.argtypes = [P, P, I, I, I, P, I, P, P, P, P]
        L.csa2_index_full_workspace_bytes.argtypes = [I, I, I, I]
        L.csa2_index_full_workspace_bytes.restype = Z
        L.csa2_index_full.argtypes = [P, P, P, P, I, I, I, I, P, P, P, Z, P, P]
        L.csa2_index_reindex_workspace_bytes.argtypes = [I, I, I]
        L.csa2_index_reindex_workspace_bytes.restype = Z
        L.csa2_index_reindex.argtypes = [P, P, P, P, I, I, P, I, I, P, P, Z, P, P]
        L.csa2_index_reindex_noalloc.argtypes = [P, P, P, P, I, I, P, I, I, P, P, P]
        L.csa2_attend_workspace_bytes.argtypes = [I, I, I]
        L.csa2_attend_workspace_bytes.restype = Z
        L.csa2_attend.argtypes = [I, P, ctypes.c_float, P, P, I, P, P, I, P, P, P, I, I, P, P, P,
                                  Z, P, P]
        L.csa2_attend_queries.argtypes = [P, ctypes.c_float, P, P, I, I, P, P, P, I, P, P, I, P, P,
                                          I, I, P, P, P, Z, P, P]
        L.csa2_cache_restore.argtypes = [P, P, P, I, I, P, I, P, P, P, P]
        L.csa2_cache_persist.argtypes = [P, P, P, I, I, P, I, P, P, P, P]
        L.csa2_swa_replay_workspace_bytes.argtypes = [I, I, I]
        L.csa2_swa_replay_workspace_bytes.restype = Z
        L.csa2_swa_replay.argtypes = [P, P, I, I, I, P, P, P, I, P, Z, P, P]
        L.csa2_status_string.argtypes = [I]
        L.csa2_status_string.restype = ctypes.c_char_p
        L.csa2_launch_count.restype = ctypes.c_uint64
        L.csa2_abi_version.restype = ctypes.c_int
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().csa2_status_string(int(status)).decode()


def launch_count() -> int:
    """Kernels launched by libcsa2.so in this process so far."""
    return int(lib().csa2_launch_count())


def _check(fn: str, status: int) -> None:
    if status != 0:
        raise Csa2Error(fn, status)


def _ptr(t: Optional[torch.Tensor], dtype=None, name="tensor"):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _hptr(t: Optional[torch.Tensor], dtype, name="tensor"):
    """Pointer of a host (CPU) tensor; page-locked memory lets the copies run asynchronously."""
    if t is None:
        return None
    if t.is_cuda:
        raise ValueError(f"{name} must be a host (CPU) tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _host_counts(N, B):
    vals = [int(v) for v in N]
    if len(vals) != B:
        raise ValueError(f"N must hold {B} counts")
    return (ctypes.c_int32 * B)(*vals)


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


# ------------------------------------------------------------------------------------- entry points

def append_quant(x, ik, pos, codes, scales, ik_cache, swa=None, swa_scale=None, dev_err=None,
                 stream=None) -> None:
    """Quantize-on-append. x bf16 [B,n,512]; ik bf16 [B,n,64] or None; pos int32 [B];
    codes uint8 [B,n_cap,256]; scales uint8 [B,n_cap,32]; ik_cache bf16 [B,n_cap,64];
    swa uint8 [B,W,512] / swa_scale f32 [B,W] or None."""
    B, n = x.shape[0], x.shape[1]
    n_cap = codes.shape[1]
    W = 0 if swa is None else swa.shape[1]
    st = lib().csa2_append_quant(
        _ptr(x, torch.bfloat16, "x"), _ptr(ik, torch.bfloat16, "ik"), B, n,
        _ptr(pos, torch.int32, "pos"), n_cap, _ptr(codes, torch.uint8, "codes"),
        _ptr(scales, torch.uint8, "scales"),
        _ptr(ik_cache, torch.bfloat16, "ik_cache") if ik is not None else None,
        _ptr(swa, torch.uint8, "swa"), _ptr(swa_scale, torch.float32, "swa_scale"), W,
        _ptr(dev_err, torch.int32, "dev_err"), _stream(stream))
    _check("csa2_append_quant", st)


def ced_project_quant(h, w, pos, codes, scales, dev_err=None, stream=None) -> None:
    """CED KV projection C = h w^T with the MXFP4 quantisation fused into the GEMM epilogue.
    h bf16 [B,n,d]; w bf16 [512,d]; pos int32 [B]; codes uint8 [B,n_cap,256];
    scales uint8 [B,n_cap,32] (token i of sequence b goes to row pos[b] + i)."""
    B, n, d = h.shape
    if tuple(w.shape) != (D, d):
        raise ValueError(f"w must be [{D}, {d}], got {tuple(w.shape)}")
    n_cap = codes.shape[1]
    st = lib().csa2_ced_project_quant(
        _ptr(h, torch.bfloat16, "h"), _ptr(w, torch.bfloat16, "w"), B, n, d,
        _ptr(pos, torch.int32, "pos"), n_cap, _ptr(codes, torch.uint8, "codes"),
        _ptr(scales, torch.uint8, "scales"), _ptr(dev_err, torch.int32, "dev_err"),
        _stream(stream))
    _check("csa2_ced_project_quant", st)


def cache_restore(host_codes, host_scales, host_ik, N, codes, scales, ik_cache=None,
                  stream=None) -> None:
    """SWA bounded replay, restore side: copy rows 0 .. N[b]-1 of the persisted MXFP4 cache (and
    indexer keys) from host tensors [B, n_host, ...] into the device cache [B, n_cap, ...].
    N is a host sequence of B ints."""
    B, n_host = host_codes.shape[0], host_codes.shape[1]
    n_cap = codes.shape[1]
    n = _host_counts(N, B)
    st = lib().csa2_cache_restore(
        _hptr(host_codes, torch.uint8, "host_codes"), _hptr(host_scales, torch.uint8, "host_scales"),
        _hptr(host_ik, torch.bfloat16, "host_ik"), B, n_host, n, n_cap,
        _ptr(codes, torch.uint8, "codes"), _ptr(scales, torch.uint8, "scales"),
        _ptr(ik_cache, torch.bfloat16, "ik_cache"), _stream(stream))
    _check("csa2_cache_restore", st)


def cache_persist(codes, scales, ik_cache, N, host_codes, host_scales, host_ik=None,
                  stream=None) -> None:
    """The inverse of cache_restore: rows 0 .. N[b]-1 of the device cache to host tensors."""
    B, n_cap = codes.shape[0], codes.shape[1]
    n_host = host_codes.shape[1]
    n = _host_counts(N, B)
    st = lib().csa2_cache_persist(
        _ptr(codes, torch.uint8, "codes"), _ptr(scales, torch.uint8, "scales"),
        _ptr(ik_cache, torch.bfloat16, "ik_cache"), B, n_cap, n, n_host,
        _hptr(host_codes, torch.uint8, "host_codes"), _hptr(host_scales, torch.uint8, "host_scales"),
        _hptr(host_ik, torch.bfloat16, "host_ik"), _stream(stream))
    _check("csa2_cache_persist", st)


def swa_replay_workspace_bytes(B: int, Wr: int, d: int) -> int:
    return int(lib().csa2_swa_replay_workspace_bytes(B, Wr, d))


def swa_replay(h, w, N, swa, swa_scale, ws, dev_err=None, stream=None) -> None:
    """SWA bounded replay: ring slot (N[b] - Wr + r) mod W of sequence b gets the SWA codec of
    bf16_RNE(h[b, r] w^T). h bf16 [B, Wr, d]; w bf16 [512, d]; N int32 [B] (device);
    swa uint8 [B, W, 512]; swa_scale f32 [B, W]; ws of swa_replay_workspace_bytes bytes."""
    B, Wr, d = h.shape
    if tuple(w.shape) != (D, d):
        raise ValueError(f"w must be [{D}, {d}], got {tuple(w.shape)}")
    W = swa.shape[1]
    st = lib().csa2_swa_replay(
        _ptr(h, torch.bfloat16, "h"), _ptr(w, torch.bfloat16, "w"), B, Wr, d,
        _ptr(N, torch.int32, "N"), _ptr(swa, torch.uint8, "swa"),
        _ptr(swa_scale, torch.float32, "swa_scale"), W, _ptr(ws, None, "ws"),
        ws.numel() * ws.element_size(), _ptr(dev_err, torch.int32, "dev_err"), _stream(stream))
    _check("csa2_swa_replay", st)


def index_full_workspace_bytes(B: int, n_cap: int, K: int, P: int) -> int:
    return int(lib().csa2_index_full_workspace_bytes(B, n_cap, K, P))


def index_full(iq, w, ik_cache, N, K, P, topk, pool, ws, dev_err=None, stream=None) -> None:
    """Full-mode indexer. iq bf16 [B,4,64]; w f32 [B,4]; ik_cache bf16 [B,n_cap,64]; N int32 [B];
    topk int32 [B,K] out; pool int32 [B,8P] out; ws uint8 workspace."""
    B, n_cap = ik_cache.shape[0], ik_cache.shape[1]
    st = lib().csa2_index_full(
        _ptr(iq, torch.bfloat16, "iq"), _ptr(w, torch.float32, "w"),
        _ptr(ik_cache, torch.bfloat16, "ik_cache"), _ptr(N, torch.int32, "N"), B, n_cap, K, P,
        _ptr(topk, torch.int32, "topk"), _ptr(pool, torch.int32, "pool"), _ptr(ws, None, "ws"),
        ws.numel() * ws.element_size(), _ptr(dev_err, torch.int32, "dev_err"), _stream(stream))
    _check("csa2_index_full", st)


def index_reindex_workspace_bytes(B: int, L: int, K: int) -> int:
    return int(lib().csa2_index_reindex_workspace_bytes(B, L, K))


def index_reindex(iq, w, ik_cache, N, pool, K, topk, ws, dev_err=None, stream=None) -> None:
    """Reindex-mode indexer over pool int32 [B,L]; topk int32 [B,K] out."""
    B, n_cap = ik_cache.shape[0], ik_cache.shape[1]
    L = pool.shape[1]
    st = lib().csa2_index_reindex(
        _ptr(iq, torch.bfloat16, "iq"), _ptr(w, torch.float32, "w"),
        _ptr(ik_cache, torch.bfloat16, "ik_cache"), _ptr(N, torch.int32, "N"), B, n_cap,
        _ptr(pool, torch.int32, "pool"), L, K, _ptr(topk, torch.int32, "topk"),
        _ptr(ws, None, "ws"), ws.numel() * ws.element_size(), _ptr(dev_err, torch.int32, "dev_err"),
        _stream(stream))
    _check("csa2_index_reindex", st)


def index_reindex_noalloc(iq, w, ik_cache, N, pool, K, topk, dev_err=None, stream=None) -> None:
    """Reindex-mode indexer without a workspace: the library uses its own fixed 2 MiB device
    array (B * L up to 262,144 slots). For callers that cannot allocate device memory; calls that
    overlap on one GPU share that array and must not run concurrently."""
    B, n_cap = ik_cache.shape[0], ik_cache.shape[1]
    L = pool.shape[1]
    st = lib().csa2_index_reindex_noalloc(
        _ptr(iq, torch.bfloat16, "iq"), _ptr(w, torch.float32, "w"),
        _ptr(ik_cache, torch.bfloat16, "ik_cache"), _ptr(N, torch.int32, "N"), B, n_cap,
        _ptr(pool, torch.int32, "pool"), L, K, _ptr(topk, torch.int32, "topk"),
        _ptr(dev_err, torch.int32, "dev_err"), _stream(stream))
    _check("csa2_index_reindex_noalloc", st)


def attend_workspace_bytes(B: int, K: int, W: int) -> int:
    return int(lib().csa2_attend_workspace_bytes(B, K, W))


def attend(mode, q, softmax_scale, codes, scales, N, idx, swa, swa_scale, swa_len, out, lse, ws,
           dev_err=None, stream=None) -> None:
    """Sparse attention. q bf16 [B,16,512]; codes/scales as appended; N int32 [B]; idx int32 [B,K];
    swa uint8 [B,W,512] / swa_scale f32 [B,W] / swa_len int32 [B] (or None); out f32 [B,16,512];
    lse f32 [B,16] or None; ws uint8 workspace (may be empty when none is needed).
    With MODE_REUSE the kernel gathers idx's first rows before it waits for the preceding kernel:
    the library call right before it on the stream must write neither idx nor those cache rows
    (in a decode step it is the previous layer's attend)."""
    B, K = idx.shape
    n_cap = codes.shape[1]
    W = 0 if swa is None else swa.shape[1]
    ws_ptr = _ptr(ws, None, "ws") if ws is not None and ws.numel() > 0 else None
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    st = lib().csa2_attend(
        int(mode), _ptr(q, torch.bfloat16, "q"), float(softmax_scale),
        _ptr(codes, torch.uint8, "codes"), _ptr(scales, torch.uint8, "scales"), n_cap,
        _ptr(N, torch.int32, "N"), _ptr(idx, torch.int32, "idx"), K,
        _ptr(swa, torch.uint8, "swa"), _ptr(swa_scale, torch.float32, "swa_scale"),
        _ptr(swa_len, torch.int32, "swa_len"), W, B, _ptr(out, torch.float32, "out"),
        _ptr(lse, torch.float32, "lse"), ws_ptr, ws_bytes, _ptr(dev_err, torch.int32, "dev_err"),
        _stream(stream))
    _check("csa2_attend", st)


def attend_queries(q, softmax_scale, codes, scales, N, qseq, idx, swa, swa_scale, swa_lo, swa_len,
                   W, out, lse, ws, dev_err=None, stream=None) -> None:
    """Sparse attention of many queries per sequence. q bf16 [Q,16,512]; codes/scales of B
    sequences; N int32 [B]; qseq int32 [Q] (each query's sequence); idx int32 [Q,K];
    swa uint8 [B,S,512] / swa_scale f32 [B,S] / swa_lo, swa_len int32 [Q] (the query's SWA rows,
    swa_len <= W), or all None with W = 0; out f32 [Q,16,512]; lse f32 [Q,16] or None."""
    Q, K = idx.shape
    B, n_cap = codes.shape[0], codes.shape[1]
    S = 0 if swa is None else swa.shape[1]
    ws_ptr = _ptr(ws, None, "ws") if ws is not None and ws.numel() > 0 else None
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    st = lib().csa2_attend_queries(
        _ptr(q, torch.bfloat16, "q"), float(softmax_scale), _ptr(codes, torch.uint8, "codes"),
        _ptr(scales, torch.uint8, "scales"), B, n_cap, _ptr(N, torch.int32, "N"),
        _ptr(qseq, torch.int32, "qseq"), _ptr(idx, torch.int32, "idx"), K,
        _ptr(swa, torch.uint8, "swa"), _ptr(swa_scale, torch.float32, "swa_scale"), S,
        _ptr(swa_lo, torch.int32, "swa_lo"), _ptr(swa_len, torch.int32, "swa_len"), int(W), Q,
        _ptr(out, torch.float32, "out"), _ptr(lse, torch.float32, "lse"), ws_ptr, ws_bytes,
        _ptr(dev_err, torch.int32, "dev_err"), _stream(stream))
    _check("csa2_attend_queries", st)


# ------------------------------------------------------------------------------- buffer helpers

class Cache:
    """Device buffers of one cache group shared by a CSA2 layer stack (cross-layer reuse): the
    MXFP4 main KV, the bf16 indexer keys and the FP8 SWA ring."""

    def __init__(self, B: int, n_cap: int, W: int, device="cuda"):
        if n_cap % S:
            raise ValueError("n_cap must be a multiple of 8")
        self.B, self.n_cap, self.W = B, n_cap, W
        self.codes = torch.zeros(B, n_cap, D // 2, dtype=torch.uint8, device=device)
        self.scales = torch.zeros(B, n_cap, D // 16, dtype=torch.uint8, device=device)
        self.ik = torch.zeros(B, n_cap, DI, dtype=torch.bfloat16, device=device)
        self.swa = torch.zeros(B, max(W, 1), D, dtype=torch.uint8, device=device)[:, :W]
        self.swa_scale = torch.zeros(B, max(W, 1), dtype=torch.float32, device=device)[:, :W]
        self.swa = self.swa.contiguous()
        self.swa_scale = self.swa_scale.contiguous()

    def append(self, x, ik, pos, dev_err=None, stream=None):
        append_quant(x, ik, pos, self.codes, self.scales, self.ik,
                     self.swa if self.W else None, self.swa_scale if self.W else None, dev_err,
                     stream)


def workspace(nbytes: int, device="cuda") -> torch.Tensor:
    return torch.empty(max(int(nbytes), 16), dtype=torch.uint8, device=device)
