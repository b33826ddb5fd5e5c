"""Seeded synthetic inputs for the CSA2 decode path.

Shared by the tests, the smoke check and the benchmark; holds none of the method's arithmetic
(no quantisation, no scoring, no selection, no attention). Every tensor is drawn from a
``torch.Generator`` whose seed is derived from (workload seed, stream tag, sequence, chunk) by
splitmix64, so any chunk of any sequence can be regenerated on its own, on the CPU or on a GPU
(the two devices give different but individually reproducible draws).

Shapes follow the pages' description of the decoder: main KV entries of width 512 (shared K = V),
16 attention heads of width 512, an indexer with 4 heads of width 64, a Top-512 over the entries
and a pool of 2048 blocks x 8 positions, and an FP8 sliding window of recent tokens
("DeepSeek V4.1 Flash 拆解", austincafe.tech, section 一). The pages name no dataset or benchmark,
so the value distributions below are synthetic stand-ins.
"""
from __future__ import annotations

import dataclasses
import math

import torch

D, HQ, HI, DI, S = 512, 16, 4, 64, 8
CHUNK = 65536  # rows per independently seeded chunk

_MASK64 = (1 << 64) - 1
_TAGS = {"kv": 1, "ik": 2, "q": 3, "iq": 4, "w": 5, "plant": 6, "cluster": 7, "idx": 8,
         "heavy": 9, "new": 10, "outlier": 11, "assign": 12}


def _splitmix64(x: int) -> int:
    x = (x + 0x9E3779B97F4A7C15) & _MASK64
    x = ((x ^ (x >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
    x = ((x ^ (x >> 27)) * 0x94D049BB133111EB) & _MASK64
    return x ^ (x >> 31)


def derive_seed(seed: int, tag: str, *parts: int) -> int:
    h = _splitmix64(seed)
    h = _splitmix64(h ^ _TAGS[tag])
    for p in parts:
        h = _splitmix64(h ^ (p & _MASK64))
    return h & 0x7FFFFFFFFFFFFFFF


def gen(device, seed: int, tag: str, *parts: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(derive_seed(seed, tag, *parts))
    return g


@dataclasses.dataclass
class StackWorkload:
    """One CSA2 layer stack decoding a batch of B sequences of N entries each."""
    name: str
    B: int
    N: int
    modes: tuple  # "F" Full, "RI" Reindex, "U" Reuse, in layer order
    K: int = 512
    P: int = 2048
    W: int = 128
    seed: int = 0
    n_planted: int = 0        # per sequence: indexer keys shifted by +3 sigma toward the Full query
    ik_kind: str = "gauss"    # "gauss" N(0,1) or "cluster" (64-cluster Gaussian mixture per block)
    heavy_row_frac: float = 0.0   # fraction of main-KV entries (rows) multiplied by heavy_row_scale
    heavy_row_scale: float = 1.0
    ri_corr: float = 0.7      # correlation of a Reindex layer's indexer query with the Full one's
    softmax_scale: float = 1.0  # q is pre-scaled by 1/sqrt(512) instead

    @property
    def n_idx(self) -> int:
        return sum(m in ("F", "RI") for m in self.modes)

    @property
    def L(self) -> int:
        return len(self.modes)

    @property
    def n_cap(self) -> int:
        return ((self.N + 127) // 128) * 128


# Tiny Full layer (the parity case), the three-layer stack, the 8-layer pattern, the
# million-entry decode over that pattern.
TINY = StackWorkload("tiny-full-B1-N4096", B=1, N=4096, modes=("F",), K=64, P=64, W=64, seed=0,
                     n_planted=32)
STACK3 = StackWorkload("stack3-FRIU-B4-N65536", B=4, N=65536, modes=("F", "RI", "U"), seed=1,
                       n_planted=256)
PATTERN8 = StackWorkload("pattern8-B16-N262144", B=16, N=262144,
                         modes=("F", "RI", "RI", "U", "U", "U", "U", "U"), seed=2,
                         ik_kind="cluster")
MILLION = StackWorkload("decode-1M-pattern8-B8-N1048576", B=8, N=1048576,
                        modes=("F", "RI", "RI", "U", "U", "U", "U", "U"), seed=3,
                        heavy_row_frac=0.01, heavy_row_scale=8.0)


def bf16_bits(t: torch.Tensor):
    """bf16 tensor -> numpy uint16 bit patterns (host)."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view("uint16")


# ------------------------------------------------------------------------------ per-step inputs

def step_inputs(wl: StackWorkload, device="cpu", step: int = 0):
    """Queries of one decode step: q [L,B,16,512] bf16 (N(0,1)/sqrt(512)), iq [n_idx,B,4,64] bf16,
    w [n_idx,B,4] f32 ~ U(0.5,1.5). Reindex queries are 0.7*iq_Full + sqrt(0.51)*z."""
    gq = gen(device, wl.seed, "q", step)
    q = (torch.randn(wl.L, wl.B, HQ, D, generator=gq, device=device) / math.sqrt(D))
    gi = gen(device, wl.seed, "iq", step)
    iq0 = torch.randn(wl.B, HI, DI, generator=gi, device=device)
    iqs = []
    for m in wl.modes:
        if m == "F":
            iqs.append(iq0)
        elif m == "RI":
            z = torch.randn(wl.B, HI, DI, generator=gi, device=device)
            iqs.append(wl.ri_corr * iq0 + math.sqrt(1.0 - wl.ri_corr ** 2) * z)
    gw = gen(device, wl.seed, "w", step)
    w = torch.rand(wl.n_idx, wl.B, HI, generator=gw, device=device) + 0.5
    return dict(q=q.to(torch.bfloat16), iq=torch.stack(iqs).to(torch.bfloat16), w=w.float())


def new_token(wl: StackWorkload, device="cpu", step: int = 0):
    """The decode step's new entry per sequence: x [B,1,512] bf16, ik [B,1,64] bf16."""
    g = gen(device, wl.seed, "new", step)
    x = torch.randn(wl.B, 1, D, generator=g, device=device).to(torch.bfloat16)
    ik = torch.randn(wl.B, 1, DI, generator=g, device=device).to(torch.bfloat16)
    return x, ik


# ------------------------------------------------------------------------------ cache contents

def kv_chunk(wl: StackWorkload, b: int, c: int, device="cpu") -> torch.Tensor:
    """Main-KV rows [c*CHUNK, min((c+1)*CHUNK, N)) of sequence b, bf16 [rows, 512]."""
    r0 = c * CHUNK
    rows = min(CHUNK, wl.N - r0)
    g = gen(device, wl.seed, "kv", b, c)
    x = torch.randn(rows, D, generator=g, device=device)
    if wl.heavy_row_frac > 0:
        gh = gen(device, wl.seed, "heavy", b, c)
        heavy = torch.rand(rows, generator=gh, device=device) < wl.heavy_row_frac
        x[heavy] *= wl.heavy_row_scale
    return x.to(torch.bfloat16)


def planted_positions(wl: StackWorkload, b: int) -> torch.Tensor:
    g = gen("cpu", wl.seed, "plant", b)
    return torch.randperm(wl.N, generator=g)[: wl.n_planted].sort().values


def plant_direction(iq_full_b: torch.Tensor, w_b: torch.Tensor) -> torch.Tensor:
    """Unit vector of sum_h w_h iq_h (float32 [64]); planted keys move 3 sigma along it."""
    v = (w_b.float().view(HI, 1) * iq_full_b.float()).sum(0)
    return v / v.norm().clamp_min(1e-30)


def ik_chunk(wl: StackWorkload, b: int, c: int, device="cpu", plant_dir=None) -> torch.Tensor:
    """Indexer-key rows of chunk c of sequence b, bf16 [rows, 64]."""
    r0 = c * CHUNK
    rows = min(CHUNK, wl.N - r0)
    g = gen(device, wl.seed, "ik", b, c)
    if wl.ik_kind == "gauss":
        k = torch.randn(rows, DI, generator=g, device=device)
    elif wl.ik_kind == "cluster":
        # 64 cluster centres ~ N(0,1) per sequence; each 8-position block draws one centre;
        # key = centre + 0.5 * N(0,1)
        gc = gen(device, wl.seed, "cluster", b)
        centres = torch.randn(64, DI, generator=gc, device=device)
        ga = gen(device, wl.seed, "assign", b, c)
        nblk = (rows + S - 1) // S
        assign = torch.randint(0, 64, (nblk,), generator=ga, device=device)
        k = centres[assign].repeat_interleave(S, 0)[:rows] + \
            0.5 * torch.randn(rows, DI, generator=g, device=device)
    else:
        raise ValueError(wl.ik_kind)
    if wl.n_planted > 0:
        assert plant_dir is not None
        pp = planted_positions(wl, b)
        sel = pp[(pp >= r0) & (pp < r0 + rows)] - r0
        if sel.numel() > 0:
            k[sel.to(k.device)] += 3.0 * plant_dir.to(k.device)
    return k.to(torch.bfloat16)


def n_chunks(wl: StackWorkload) -> int:
    return (wl.N + CHUNK - 1) // CHUNK


def full_cache_rows(wl: StackWorkload, device="cpu", step_q=None):
    """Whole main-KV and indexer-key contents: x [B,N,512] bf16, ik [B,N,64] bf16 (small
    workloads only)."""
    if step_q is None:
        step_q = step_inputs(wl, device)
    xs, iks = [], []
    for b in range(wl.B):
        pdir = plant_direction(step_q["iq"][0, b], step_q["w"][0, b]) if wl.n_planted else None
        xs.append(torch.cat([kv_chunk(wl, b, c, device) for c in range(n_chunks(wl))]))
        iks.append(torch.cat([ik_chunk(wl, b, c, device, pdir) for c in range(n_chunks(wl))]))
    return torch.stack(xs), torch.stack(iks)


# ------------------------------------------------------------------------------ append / attend

@dataclasses.dataclass
class AppendWorkload:
    """Quantize-append of n new bf16 entries (N(0,1) with a fraction of elements x outlier_scale)."""
    name: str
    B: int
    n: int
    outlier_frac: float = 0.001
    outlier_scale: float = 20.0
    seed: int = 4


APPEND_1M = AppendWorkload("append-1M", B=1, n=1048576)


def append_rows(wl: AppendWorkload, device="cpu") -> torch.Tensor:
    g = gen(device, wl.seed, "kv", 0)
    x = torch.randn(wl.B, wl.n, D, generator=g, device=device)
    go = gen(device, wl.seed, "outlier", 0)
    mask = torch.rand(wl.B, wl.n, D, generator=go, device=device) < wl.outlier_frac
    x[mask] *= wl.outlier_scale
    return x.to(torch.bfloat16)


@dataclasses.dataclass
class ReuseAttendWorkload:
    """Reuse-mode attention: K indices drawn uniformly without replacement from N entries."""
    name: str
    B: int
    N: int = 131072
    K: int = 512
    W: int = 128
    seed: int = 4


# The throughput sweep's Reuse-mode attention: batch 1, 8, 64 and 256 over N = 131,072.
REUSE_SWEEP = tuple(ReuseAttendWorkload(f"reuse-attend-B{B}-N131072", B=B) for B in (1, 8, 64, 256))


def reuse_kv_chunk(wl: ReuseAttendWorkload, b: int, c: int, device="cpu") -> torch.Tensor:
    """Main-KV rows [c*CHUNK, min((c+1)*CHUNK, N)) of sequence b, N(0,1) bf16 [rows, 512]."""
    rows = min(CHUNK, wl.N - c * CHUNK)
    g = gen(device, wl.seed, "kv", b, c)
    return torch.randn(rows, D, generator=g, device=device).to(torch.bfloat16)


def reuse_queries(wl: ReuseAttendWorkload, device="cpu") -> torch.Tensor:
    """q [B, 16, 512] bf16, N(0,1)/sqrt(512)."""
    g = gen(device, wl.seed, "q", 0)
    return (torch.randn(wl.B, HQ, D, generator=g, device=device) / math.sqrt(D)).to(torch.bfloat16)


def reuse_indices(wl: ReuseAttendWorkload, device="cpu") -> torch.Tensor:
    out = torch.empty(wl.B, wl.K, dtype=torch.int32)
    for b in range(wl.B):
        g = gen("cpu", wl.seed, "idx", b)
        out[b] = torch.randperm(wl.N, generator=g)[: wl.K].sort().values.to(torch.int32)
    return out.to(device)
