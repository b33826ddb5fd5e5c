"""The oracle baselines that bench.py times on the host threads (CPU only).

bench.py splits the oracle's work over the host threads: ctypes releases the GIL while the C
oracle runs, so the threads really run at once. Two things are checked here:
- the oracle gives the same codes when called from many threads at once as when called from one;
- each mode's `cpu_baseline` reports the contract keys, with the thread count in `cores`.
"""
import concurrent.futures as cf

import numpy as np
import torch

import bench
import oracle


def _rows(seed, n):
    rng = np.random.default_rng(seed)
    # magnitudes over many binades, so that every E4M3 scale and E2M1 code is reached
    return (rng.standard_normal((n, 512)) * np.exp2(rng.integers(-12, 12, (n, 1)))).astype(np.float32)


def test_oracle_codecs_are_the_same_from_concurrent_threads():
    parts = [_rows(s, 64) for s in range(16)]
    seq = [oracle.mxfp4_quantize_f32(p) for p in parts]
    seq_e4 = [oracle.e4m3_encode(p[:, :64].ravel()) for p in parts]
    with cf.ThreadPoolExecutor(max_workers=8) as ex:
        par = list(ex.map(oracle.mxfp4_quantize_f32, parts))
        par_e4 = list(ex.map(lambda p: oracle.e4m3_encode(p[:, :64].ravel()), parts))
    for (c0, s0), (c1, s1) in zip(seq, par):
        assert np.array_equal(c0, c1) and np.array_equal(s0, s1)
    for a, b in zip(seq_e4, par_e4):
        assert np.array_equal(a, b)


def _check_line(cpu, unit):
    assert cpu["kind"] == "oracle" and cpu["unit"] == unit
    assert cpu["value"] > 0 and cpu["cores"] >= 1
    assert isinstance(cpu["sample"], str) and cpu["sample"]


def test_ced_baseline_reports_its_threads():
    h = torch.randn(1, 64, 256).to(torch.bfloat16)
    w = (torch.randn(512, 256) / 16).to(torch.bfloat16)
    cpu = bench.ced_cpu_baseline(h, w, rows=64)
    _check_line(cpu, "TFLOP/s")
    assert cpu["cores"] <= min(bench.host_threads(), 4)  # at least 16 rows per thread


def test_queries_baseline_reports_its_threads():
    rng = np.random.default_rng(0)
    B, n_cap, S, K, Q = 2, 2048, 256, 64, 24
    codes = rng.integers(0, 256, (B, n_cap, 256), dtype=np.uint8)
    scales = rng.integers(40, 60, (B, n_cap, 32), dtype=np.uint8)
    swa = rng.integers(0, 120, (B, S, 512), dtype=np.uint8)
    swsc = rng.random((B, S), dtype=np.float32)
    q = (torch.randn(Q, 16, 512) / 20).to(torch.bfloat16)
    idx = np.stack([np.sort(rng.choice(n_cap, K, replace=False)) for _ in range(Q)]).astype(np.int32)
    qseq = np.array([i % B for i in range(Q)], np.int32)
    lo = np.array([(7 * i) % 128 for i in range(Q)], np.int32)
    ln = np.full(Q, 64, np.int32)
    cpu = bench.queries_cpu_baseline(q, codes, scales, idx, swa, swsc, qseq, lo, ln, n_sample=8)
    _check_line(cpu, "queries/s")
    assert cpu["sample"].startswith(f"{min(Q, max(8, 8 * cpu['cores']))} of {Q} queries")


def test_replay_baseline_reports_its_threads():
    w = (torch.randn(512, 256) / 16).to(torch.bfloat16)
    hc = torch.zeros(3, 256, 256, dtype=torch.uint8)
    hs = torch.zeros(3, 256, 32, dtype=torch.uint8)
    hi = torch.zeros(3, 256, 64, dtype=torch.bfloat16)
    hwin = torch.randn(3, 128, 256).to(torch.bfloat16)
    cpu = bench.replay_cpu_baseline(hc, hs, hi, hwin, w, 200)
    _check_line(cpu, "restores/s")
    assert cpu["cores"] == min(bench.host_threads(), 3)
