#!/usr/bin/env python
"""Benchmark of the CSA2 decode step on B200.

One step = one decode step of an 8-layer CSA2 stack (Full, Reindex, Reindex, Reuse x 5) for a batch
of sequences: quantize-append of the new entry, the Full-mode indexer over every cached entry, two
Reindex-mode indexers over the pool, and sparse attention in every layer. Default workload: B = 8
sequences of N = 1,048,576 entries (the million-entry decode). Metric: decode layer-steps/s (one
layer-step = one layer's decode step for the whole batch) and achieved HBM GB/s over the
algorithmic bytes (indexer keys read + gathered MXFP4 codes and scales + FP8 SWA rows).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]
  python bench.py --ced [--steps K] [--warmup W]
  python bench.py --replay [--replay-n N] [--steps K] [--warmup W]
  python bench.py --queries [--steps K] [--warmup W]
  python bench.py --append [--steps K] [--warmup W]
  python bench.py --sweep [--sweep-batches 1,8,64,256] [--steps K] [--warmup W]

--ced measures the CED KV projection with the MXFP4 epilogue instead (8 x 4,096 new tokens,
hidden size 4,096: a tensor-core-bound GEMM), reported in TFLOP/s against the measured bf16
tensor peak.
--queries measures csa2_attend_queries on a prefill chunk: 8 sequences of 131,072 cached entries,
512 query tokens each (4,096 queries), every query with its own 512 selected entries and its own
causal window of 128 FP8 SWA rows; reported in queries/s and GB/s of gathered bytes.
--replay measures the SWA bounded replay restore of 8 persisted sequences of N tokens (default
1,048,576): the host-to-device reload of their MXFP4 KV and indexer keys from pinned memory
(reported against a plain pinned copy of the same bytes) and the replay of their FP8 SWA rings
from the last 128 tokens' hidden states (d = 4,096; tcgen05 projection, TFLOP/s).

--append measures the MXFP4 quantize-append of 1,048,576 new bf16 entries (N(0,1), 0.1% of the
elements x20) into one cache: GB/s over the bf16 rows read plus the codes and scales written.
--sweep measures Reuse-mode attention over N = 131,072 cached entries at batch 1, 8, 64 and 256
(512 indices per sequence drawn uniformly without replacement, a 128-row SWA window), one JSON
line per batch size: GB/s over the gathered MXFP4 entries and SWA rows, every call timed alone
after an L2 flush.

With --gpus N > 1 run under torchrun: every rank decodes its own batch (data parallel, no
collective on the data path); the step time is the max over ranks.
--impl reference times the CPU oracle (a plain restatement of the same definitions) on whole decode
steps of the same workload (every sequence of the batch, one per host thread), on rank 0 only.
"""
from __future__ import annotations

import argparse
import ctypes
import dataclasses
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "decode layer-steps/s and achieved HBM GB/s (% of 8 TB/s) at 1M ctx, 1 B200"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0

WORKLOADS = {w.name: w for w in (workloads.TINY, workloads.STACK3, workloads.PATTERN8,
                                  workloads.MILLION)}
DEFAULT = workloads.MILLION.name


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default 1000; the reference arm's default is 10)")
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT, choices=sorted(WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--replay", action="store_true",
                    help="measure the SWA bounded replay restore (host reload + ring replay)")
    ap.add_argument("--queries", action="store_true",
                    help="measure multi-query sparse attention (prefill / verification queries)")
    ap.add_argument("--replay-n", type=int, default=1 << 20,
                    help="tokens per restored sequence for --replay (default 1,048,576)")
    ap.add_argument("--ced", action="store_true",
                    help="measure the CED KV projection with the MXFP4 epilogue instead")
    ap.add_argument("--append", action="store_true",
                    help="measure the 1,048,576-entry MXFP4 quantize-append instead")
    ap.add_argument("--sweep", action="store_true",
                    help="measure Reuse-mode attention at the sweep's batch sizes (one line each)")
    ap.add_argument("--sweep-batches", default="1,8,64,256",
                    help="batch sizes of --sweep (default 1,8,64,256)")
    ap.add_argument("--sweep-n", type=int, default=131072,
                    help="cached entries per sequence for --sweep (default 131,072)")
    ap.add_argument("--breakdown", action="store_true",
                    help="also time each library call of the step (eager, synchronised)")
    return ap.parse_args()


def measured_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def measured_tensor_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return 1590.0, "fallback"


def scan_traffic_per_launch(wl):
    """DRAM bytes per scan launch from the committed ncu capture (profiles/index_scan_traffic.json),
    scaled by entries scored; None once the scan kernel's source differs from the captured one."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "index_scan_traffic.json")) as f:
            cap = json.load(f)
        csrc = os.path.join(ROOT, "sparse_attention_decode_kv_b200", "csrc")
        src = open(os.path.join(csrc, "index.cu")).read()
        a = src.index("__global__ void __launch_bounds__(kScanThreads, 1)")
        b = src.index("\n}\n", a) + 3
        region = src[a:b] + open(os.path.join(csrc, "common.cuh")).read()
        if hashlib.sha256(region.encode()).hexdigest() != cap["source_sha256"]:
            return None
        return int(round(cap["dram_bytes_per_entry"] * wl.B * wl.N))
    except Exception:
        return None


def captured_traffic(record: str):
    """DRAM bytes per launch from a committed ncu capture (profiles/<record>), or None once the
    sources the record's hash covers differ from the captured ones."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", record)) as f:
            cap = json.load(f)
        csrc = os.path.join(ROOT, "sparse_attention_decode_kv_b200", "csrc")
        text = "".join(open(os.path.join(csrc, n)).read() for n in cap["hash_files"])
        if hashlib.sha256(text.encode()).hexdigest() != cap["source_sha256"]:
            return None
        return cap
    except Exception:
        return None


def ced_traffic_per_launch(tokens):
    """CED DRAM bytes per launch (profiles/ced_projection_traffic.json), scaled by token rows."""
    cap = captured_traffic("ced_projection_traffic.json")
    return None if cap is None else int(round(cap["dram_bytes_per_token"] * tokens))


def algorithmic_bytes(wl) -> dict:
    """Bytes the step must move (indexer keys + gathered MXFP4 entries + scales + SWA rows)."""
    full = wl.B * wl.N * 128
    reindex = wl.B * min(wl.P * 8, wl.N) * 128
    attend = wl.B * (min(wl.K, wl.N) * 288 + wl.W * 516)
    n_f = sum(m == "F" for m in wl.modes)
    n_ri = sum(m == "RI" for m in wl.modes)
    return dict(full=full, reindex=reindex, attend=attend,
                step=n_f * full + n_ri * reindex + wl.L * attend)


# --------------------------------------------------------------------------------- distributed

def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(world, value: float, dev) -> float:
    """The slowest rank's time (an NCCL all-reduce on the device; gloo uses the host)."""
    if world == 1:
        return value
    import torch.distributed as dist
    if dist.get_backend() == "gloo":
        dev = torch.device("cpu")
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_workload(base, rank: int):
    """Data parallel: every rank decodes its own batch of independent sequences."""
    return dataclasses.replace(base, seed=base.seed + 1000 * rank)


def aggregate_value(world: int, layers: int, steps: int, ms_max: float) -> float:
    """Whole-job layer-steps/s: every rank runs `layers` layer-steps per step."""
    return world * layers * steps / (ms_max / 1e3)


# --------------------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu_index = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu_index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        for line in open(self.path):
            p = [x.strip() for x in line.split(",")]
            if len(p) < 9:
                continue
            try:
                rows.append(dict(sm=float(p[1]), smax=float(p[2]), power=float(p[3]),
                                 active=p[4], hw=p[5], hwt=p[6], swt=p[7], pcap=p[8]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        loaded = [r for r in rows if r["power"] > 200] or rows
        reasons = set()
        for r in loaded:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("pcap", "sw_power_cap")):
                if r[key].lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in loaded),
                "sm_max_mhz": max(r["smax"] for r in rows), "reasons": sorted(reasons),
                "samples": len(rows), "samples_under_load": len(loaded),
                "power_w_max": max(r["power"] for r in rows)}


# --------------------------------------------------------------------------------- our arm

class Stack:
    """Device state and the step of one CSA2 layer stack decoding a batch."""

    def __init__(self, wl, dev):
        import sparse_attention_decode_kv_b200 as csa2
        self.csa2, self.wl, self.dev = csa2, wl, dev
        B, K, P, W = wl.B, wl.K, wl.P, wl.W
        self.n_cap = wl.n_cap
        self.cache = csa2.Cache(B, self.n_cap, W, device=dev)
        self._fill()
        self.N = torch.full((B,), wl.N, dtype=torch.int32, device=dev)
        self.swa_len = torch.full((B,), min(wl.N, W), dtype=torch.int32, device=dev)
        self.pos_new = torch.full((B,), wl.N - 1, dtype=torch.int32, device=dev)
        si = workloads.step_inputs(wl, dev)
        self.q, self.iq, self.w = si["q"].contiguous(), si["iq"].contiguous(), si["w"].contiguous()
        x_new, ik_new = workloads.new_token(wl, dev)
        self.x_new, self.ik_new = x_new.contiguous(), ik_new.contiguous()
        self.topk = torch.empty(wl.n_idx, B, K, dtype=torch.int32, device=dev)
        self.pool = torch.empty(B, P * 8, dtype=torch.int32, device=dev)
        self.out = torch.empty(wl.L, B, 16, 512, dtype=torch.float32, device=dev)
        self.lse = torch.empty(wl.L, B, 16, dtype=torch.float32, device=dev)
        self.ws_full = csa2.workspace(csa2.index_full_workspace_bytes(B, self.n_cap, K, P), dev)
        self.ws_re = csa2.workspace(csa2.index_reindex_workspace_bytes(B, P * 8, K), dev)
        self.ws_att = csa2.workspace(csa2.attend_workspace_bytes(B, K, W), dev)
        self.dev_err = torch.zeros(1, dtype=torch.int32, device=dev)

    def _fill(self):
        wl, dev, csa2 = self.wl, self.dev, self.csa2
        si = workloads.step_inputs(wl, dev)
        pdirs = [workloads.plant_direction(si["iq"][0, b], si["w"][0, b]) if wl.n_planted else None
                 for b in range(wl.B)]
        for c in range(workloads.n_chunks(wl)):
            x = torch.stack([workloads.kv_chunk(wl, b, c, dev) for b in range(wl.B)])
            ik = torch.stack([workloads.ik_chunk(wl, b, c, dev, pdirs[b]) for b in range(wl.B)])
            pos = torch.full((wl.B,), c * workloads.CHUNK, dtype=torch.int32, device=dev)
            self.cache.append(x, ik, pos)
            del x, ik
        torch.cuda.synchronize()

    # pieces of the step
    def append_new(self):
        self.cache.append(self.x_new, self.ik_new, self.pos_new, self.dev_err)

    def index_full(self):
        c = self.csa2
        c.index_full(self.iq[0], self.w[0], self.cache.ik, self.N, self.wl.K, self.wl.P,
                     self.topk[0], self.pool, self.ws_full, self.dev_err)

    def layers(self):
        """Everything after the Full index: Reindex layers and every layer's attention."""
        c, wl, cache = self.csa2, self.wl, self.cache
        j = 0
        cur = None
        for l, m in enumerate(wl.modes):
            if m == "F":
                cur = self.topk[j]
                j += 1
                mode = c.MODE_FULL
            elif m == "RI":
                c.index_reindex(self.iq[j], self.w[j], cache.ik, self.N, self.pool, wl.K,
                                self.topk[j], self.ws_re, self.dev_err)
                cur = self.topk[j]
                j += 1
                mode = c.MODE_REINDEX
            else:
                mode = c.MODE_REUSE
            c.attend(mode, self.q[l], wl.softmax_scale, cache.codes, cache.scales, self.N, cur,
                     cache.swa, cache.swa_scale, self.swa_len, self.out[l], self.lse[l],
                     self.ws_att, self.dev_err)

    def eager_step(self):
        self.append_new()
        self.index_full()
        self.layers()


def run_ours(args, world, rank, local):
    import sparse_attention_decode_kv_b200 as csa2
    from sparse_attention_decode_kv_b200 import build as csa2_build
    if rank == 0:
        csa2_build.build()
    barrier(world)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    base = WORKLOADS[args.workload]
    wl = rank_workload(base, rank)
    st = Stack(wl, dev)
    stream = torch.cuda.current_stream(dev)

    # warm-up (eager), then capture the whole step into one CUDA graph for the headline loop,
    # which records no events inside the step. A second pass times the scan kernel on its own
    # events: the append and the layers after the Full index replay from their own graphs and
    # the Full index is launched eagerly between them, so that its scan gets an event pair.
    launches0 = csa2.launch_count()
    st.eager_step()
    torch.cuda.synchronize()
    per_step_launches = csa2.launch_count() - launches0
    g_step = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_step, stream=torch.cuda.Stream(dev)):
        st.eager_step()
    g_app, g_layers = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_app, stream=torch.cuda.Stream(dev)):
        st.append_new()
    with torch.cuda.graph(g_layers, stream=torch.cuda.Stream(dev)):
        st.layers()
    torch.cuda.synchronize()

    K, W = args.steps, args.warmup
    ev_scan = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(K)]
    L = csa2.lib()

    def step():
        g_step.replay()

    def probed_step(i):
        g_app.replay()
        L.csa2_set_profile_events(1, ctypes.c_void_p(ev_scan[i][0].cuda_event),
                                  ctypes.c_void_p(ev_scan[i][1].cuda_event))
        st.index_full()
        L.csa2_set_profile_events(1, None, None)
        g_layers.replay()

    for e in ev_scan:  # materialise the event handles
        e[0].record(stream)
        e[1].record(stream)
    for _ in range(W):
        step()
    torch.cuda.synchronize()
    barrier(world)

    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        barrier(world)
        torch.cuda.synchronize()
        t0.record(stream)
        for _ in range(K):
            step()
        t1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        # roofline pass: the same steps with the scan bracketed by its own events
        for i in range(K):
            probed_step(i)
        torch.cuda.synchronize()
        barrier(world)
    ms_local = t0.elapsed_time(t1)
    ms = max_over_ranks(world, ms_local, dev)
    scan_ms = statistics.mean(a.elapsed_time(b) for a, b in ev_scan)
    err = int(st.dev_err.item())
    if err:
        raise RuntimeError(f"device error flags {err:#x} during the benchmark")

    ab = algorithmic_bytes(wl)
    ms_step = ms / K
    value = aggregate_value(world, wl.L, K, ms)
    achieved_step_gbs = world * ab["step"] * K / (ms / 1e3) / 1e9
    peak, peak_kind = measured_peak()
    scan_gbs = ab["full"] / (scan_ms / 1e3) / 1e9

    e2e = None if args.no_e2e else run_e2e(st, step, K, W, world, dev)
    parts = breakdown(st) if args.breakdown else None
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl, dev)

    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "layer-steps/s", "n_gpus": world,
        "steps": K, "warmup": W, "ms_per_step": round(ms_step, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16/fp16-in fp32-acc (mxfp4+fp8 cache)",
        "data": "synthetic",
        "config": {"workload": wl.name, "B_per_gpu": wl.B, "N": wl.N, "layers": ",".join(wl.modes),
                   "K": wl.K, "P": wl.P, "W": wl.W, "cuda_graph": "whole step (append, Full index, layers) as one graph",
                   "l2": "inputs larger than L2 (indexer keys %.2f GB per step)" % (ab["full"] / 1e9),
                   "parallelism": f"dp{world} (independent sequences)"},
        "achieved_gbs": round(achieved_step_gbs, 1),
        "pct_of_8TBs": round(100 * achieved_step_gbs / NOMINAL_HBM_GBS / world, 2),
        "pct_of_measured_hbm": round(100 * achieved_step_gbs / peak / world, 2),
        "sequence_layer_steps_per_s": round(value * wl.B, 1),
        "roofline": {"kernel": "index_scan_kernel (Full-mode score scan)", "bound": "hbm",
                     "achieved": round(scan_gbs, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(scan_gbs / peak, 4), "peak_kind": peak_kind,
                     "algorithmic_bytes_per_launch": ab["full"],
                     "launch_ms": round(scan_ms, 4), "traffic": scan_traffic_per_launch(wl),
                     "timing": "CUDA events around every scan launch in a second pass of K steps "
                               "(append and layers from graphs, the Full index eager)",
                     "traffic_source": "profiles/index_scan_traffic.json (ncu, scaled by entries)"},
        "gpu_launches": per_step_launches * K,
        "clocks": clocks.summary(),
    }
    if e2e is not None:
        line["e2e"] = e2e
    if parts is not None:
        line["breakdown_us"] = parts
    if cpu is not None:
        line["cpu_baseline"] = cpu
    if rank == 0:
        print(json.dumps(line), flush=True)


def breakdown(st, steps=20):
    """Median device time (us) of each library call of an eager step, from CUDA events recorded
    around every call on the launching stream (diagnostic; not the headline number)."""
    stream = torch.cuda.current_stream(st.dev)
    L = st.csa2.lib()
    parts = {}

    def pair():
        # torch creates the CUDA event on first record; record once so the handle exists
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        b.record(stream)
        return a, b

    def timed(name, kernel_id, fn):
        a, b = pair()
        L.csa2_set_profile_events(kernel_id, ctypes.c_void_p(a.cuda_event),
                                  ctypes.c_void_p(b.cuda_event))
        fn()
        L.csa2_set_profile_events(kernel_id, None, None)
        parts.setdefault(name, []).append((a, b))

    wl, c, cache = st.wl, st.csa2, st.cache
    samples = {}
    for _ in range(steps):
        parts.clear()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        timed("append", 0, st.append_new)
        ev = [pair(), pair()]
        L.csa2_set_profile_events(1, ctypes.c_void_p(ev[0][0].cuda_event), ctypes.c_void_p(ev[0][1].cuda_event))
        L.csa2_set_profile_events(2, ctypes.c_void_p(ev[1][0].cuda_event), ctypes.c_void_p(ev[1][1].cuda_event))
        st.index_full()
        L.csa2_set_profile_events(1, None, None)
        L.csa2_set_profile_events(2, None, None)
        parts["index_scan"] = [ev[0]]
        parts["index_select"] = [ev[1]]
        j, cur = 0, None
        for l, m in enumerate(wl.modes):
            if m == "F":
                cur, j, mode = st.topk[j], j + 1, c.MODE_FULL
            elif m == "RI":
                jj = j
                timed("reindex", 3, lambda jj=jj: c.index_reindex(
                    st.iq[jj], st.w[jj], cache.ik, st.N, st.pool, wl.K, st.topk[jj], st.ws_re,
                    st.dev_err))
                cur, j, mode = st.topk[j], j + 1, c.MODE_REINDEX
            else:
                mode = c.MODE_REUSE
            timed("attend", 4, lambda l=l, mode=mode, cur=cur: c.attend(
                mode, st.q[l], wl.softmax_scale, cache.codes, cache.scales, st.N, cur, cache.swa,
                cache.swa_scale, st.swa_len, st.out[l], st.lse[l], st.ws_att, st.dev_err))
        a1.record(stream)
        torch.cuda.synchronize()
        for name, evs in parts.items():
            samples.setdefault(name, []).append(sum(x.elapsed_time(y) for x, y in evs) * 1e3)
        samples.setdefault("eager_step", []).append(a0.elapsed_time(a1) * 1e3)
    return {k: round(statistics.median(v), 2) for k, v in samples.items()}


def run_e2e(st, step, K, W, world, dev):
    """Same metric through the public API with host buffers. Every step copies its inputs from
    pinned host memory and reads its outputs back. Like a serving loop, the transfers overlap
    the compute: the inputs of step i+1 go in on one copy stream and the outputs of step i-1
    come back on another while step i runs. There are two device buffer sets, each with its own
    captured graphs. The timed region runs from the first input copy to the last read-back."""
    stream = torch.cuda.current_stream(dev)
    names_in = ("q", "iq", "w", "x_new", "ik_new")
    host_in = {k: getattr(st, k).detach().cpu().pin_memory() for k in names_in}
    sets = [{k: getattr(st, k) for k in names_in + ("out", "lse")},
            {k: torch.empty_like(getattr(st, k)) for k in names_in + ("out", "lse")}]
    host_out = [(torch.empty(st.out.shape, dtype=st.out.dtype).pin_memory(),
                 torch.empty(st.lse.shape, dtype=st.lse.dtype).pin_memory()) for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in host_in.values())
    d2h = host_out[0][0].numel() * 4 + host_out[0][1].numel() * 4

    def use(j):
        for k, t in sets[j].items():
            setattr(st, k, t)

    # graphs of the second buffer set (the caller's graphs read the first)
    for k in names_in:
        sets[1][k].copy_(sets[0][k])
    use(1)
    g_step1 = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_step1, stream=torch.cuda.Stream(dev)):
        st.eager_step()
    use(0)
    torch.cuda.synchronize()

    def step_set(j):
        if j == 0:
            step()
        else:
            g_step1.replay()

    h2d_s, d2h_s = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()
    ev_in, ev_step, ev_d2h = [ev(), ev()], [ev(), ev()], [ev(), ev()]

    def h2d_copy(i):
        j = i & 1
        with torch.cuda.stream(h2d_s):
            if i >= 2:
                h2d_s.wait_event(ev_step[j])  # step i-2 no longer reads this set's inputs
            for k in names_in:
                sets[j][k].copy_(host_in[k], non_blocking=True)
            ev_in[j].record(h2d_s)

    def compute(i):
        j = i & 1
        stream.wait_event(ev_in[j])
        if i >= 2:
            stream.wait_event(ev_d2h[j])  # step i-2's outputs in this set have been read back
        step_set(j)
        ev_step[j].record(stream)

    def d2h_copy(i):
        j = i & 1
        with torch.cuda.stream(d2h_s):
            d2h_s.wait_event(ev_step[j])
            host_out[j][0].copy_(sets[j]["out"], non_blocking=True)
            host_out[j][1].copy_(sets[j]["lse"], non_blocking=True)
            ev_d2h[j].record(d2h_s)

    def run(n, t0=None, t1=None):
        if t0 is not None:
            t0.record(h2d_s)
        h2d_copy(0)
        for i in range(n):
            if i + 1 < n:
                h2d_copy(i + 1)
            compute(i)
            d2h_copy(i)
        if t1 is not None:
            t1.record(d2h_s)

    run(max(W, 2))
    torch.cuda.synchronize()
    barrier(world)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    run(K, t0, t1)
    torch.cuda.synchronize()
    ms = max_over_ranks(world, t0.elapsed_time(t1), dev)

    # the same steps with every copy on the compute stream, one after the other (for contrast)
    def serial_step():
        for k in names_in:
            sets[0][k].copy_(host_in[k], non_blocking=True)
        step()
        host_out[0][0].copy_(sets[0]["out"], non_blocking=True)
        host_out[0][1].copy_(sets[0]["lse"], non_blocking=True)

    torch.cuda.synchronize()
    barrier(world)
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s0.record(stream)
    for _ in range(K):
        serial_step()
    s1.record(stream)
    torch.cuda.synchronize()
    ms_serial = max_over_ranks(world, s0.elapsed_time(s1), dev)
    return {"value": round(world * st.wl.L * K / (ms / 1e3), 2), "unit": "layer-steps/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": round(ms / K, 4),
            "pipelining": "step i+1's inputs in and step i-1's outputs out on two copy streams "
                          "while step i runs (two buffer sets, one step graph each)",
            "serialized": {"value": round(world * st.wl.L * K / (ms_serial / 1e3), 2),
                           "ms_per_step": round(ms_serial / K, 4),
                           "note": "the same copies and steps in order on one stream"}}


# --------------------------------------------------------------------------------- oracle arm

def oracle_sample_inputs(wl, dev, seqs):
    """Host inputs for the oracle on sequences `seqs` of the workload (the same generators as the
    GPU arm; nothing the CUDA kernels produced)."""
    import numpy as np
    si = workloads.step_inputs(wl, dev)
    out = []
    for b in seqs:
        pdir = workloads.plant_direction(si["iq"][0, b], si["w"][0, b]) if wl.n_planted else None
        ik = torch.cat([workloads.ik_chunk(wl, b, c, dev, pdir) for c in range(workloads.n_chunks(wl))])
        out.append(dict(b=b, ik=workloads.bf16_bits(ik), q=workloads.bf16_bits(si["q"][:, b]),
                        iq=workloads.bf16_bits(si["iq"][:, b]), w=si["w"][:, b].cpu().numpy()))
    return out, np


def oracle_rows(wl, b, rows, dev):
    """bf16 main-KV rows `rows` of sequence b, regenerated chunk by chunk."""
    import numpy as np
    rows = np.asarray(rows, np.int64)
    res = np.zeros((len(rows), 512), np.uint16)
    for c in np.unique(rows // workloads.CHUNK):
        m = rows // workloads.CHUNK == c
        x = workloads.kv_chunk(wl, b, int(c), dev)
        res[m] = workloads.bf16_bits(x[torch.as_tensor(rows[m] - c * workloads.CHUNK, device=dev)])
    return res


def host_threads() -> int:
    """Host cores this process may run on."""
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


class OracleDecode:
    """The oracle's decode step (Full index, Reindex layers, every layer's attention) for a set of
    sequences, one sequence per host thread. The oracle itself is plain single-threaded C; ctypes
    releases the GIL while it runs, so the sequences proceed in parallel. Between the index part
    and the attention part the rows the attention needs are regenerated and quantised by the
    oracle into a compact cache; that preparation is not timed and is kept for later steps."""

    def __init__(self, wl, dev, seqs, threads):
        import concurrent.futures as cf
        self.wl, self.dev = wl, dev
        self.inputs, _ = oracle_sample_inputs(wl, dev, seqs)
        self.threads = max(1, min(threads, len(self.inputs)))
        self.pool = cf.ThreadPoolExecutor(max_workers=self.threads)
        self.prep = {}

    def close(self):
        self.pool.shutdown()

    def _index(self, sample):
        import oracle
        wl = self.wl
        ik = sample["ik"][None]
        r = oracle.index_full(sample["iq"][0][None], sample["w"][0][None], ik, [wl.N], wl.K, wl.P)
        per_layer, j, cur = [], 1, r["topk"][0]
        for m in wl.modes:
            if m == "RI":
                cur = oracle.index_reindex(sample["iq"][j][None], sample["w"][j][None], ik,
                                           r["pool"], wl.K)["topk"][0]
                j += 1
            per_layer.append(cur)
        return per_layer

    def _prepare(self, sample, per_layer):
        import numpy as np

        import oracle
        wl, b = self.wl, sample["b"]
        key = tuple(tuple(int(v) for v in tk) for tk in per_layer)
        hit = self.prep.get(b)
        if hit is not None and hit[0] == key:
            return hit[1]
        N, W = wl.N, wl.W
        need = sorted(set(int(v) for tk in per_layer for v in tk if v >= 0))
        codes, scales = oracle.mxfp4_quantize(oracle_rows(wl, b, need, self.dev))
        remap = {p: i for i, p in enumerate(need)}
        swa, swsc = oracle.swa_quantize(oracle_rows(wl, b, list(range(N - min(N, W), N)), self.dev))
        ring = np.zeros((W, 512), np.uint8)
        rsc = np.zeros((W,), np.float32)
        for i, p in enumerate(range(N - min(N, W), N)):  # ring slot of position p is p mod W
            ring[p % W], rsc[p % W] = swa[i], swsc[i]
        idx = [np.array([remap[int(v)] if v >= 0 else -1 for v in tk], np.int64) for tk in per_layer]
        prep = (codes, scales, idx, ring, rsc)
        self.prep[b] = (key, prep)
        return prep

    def _attend(self, sample, prep):
        import oracle
        wl = self.wl
        codes, scales, idx, ring, rsc = prep
        for l in range(wl.L):
            oracle.attend_seq(sample["q"][l], wl.softmax_scale, codes, scales, idx[l], ring, rsc,
                              min(wl.N, wl.W))

    def step(self) -> float:
        """Seconds of oracle compute for one decode step of every sequence in the set."""
        t = time.perf_counter()
        per = list(self.pool.map(self._index, self.inputs))
        t_index = time.perf_counter() - t
        preps = [self._prepare(smp, p) for smp, p in zip(self.inputs, per)]  # not timed
        t = time.perf_counter()
        list(self.pool.map(self._attend, self.inputs, preps))
        return t_index + time.perf_counter() - t


CPU_BASELINE_MIN_CPU_S = 10.0   # thread-seconds of oracle work the sample should reach
CPU_BASELINE_MAX_STEPS = 8


def cpu_baseline(wl, dev):
    """Whole oracle decode steps of the batch, one sequence per host thread, repeated until the
    sample holds about CPU_BASELINE_MIN_CPU_S thread-seconds (at most CPU_BASELINE_MAX_STEPS)."""
    od = OracleDecode(wl, dev, list(range(wl.B)), host_threads())
    secs = []
    try:
        while not secs or (sum(secs) * od.threads < CPU_BASELINE_MIN_CPU_S
                           and len(secs) < CPU_BASELINE_MAX_STEPS):
            secs.append(od.step())
    finally:
        od.close()
    sec = sum(secs)
    return {"value": round(wl.L * len(secs) / sec, 4), "unit": "layer-steps/s", "cores": od.threads,
            "kind": "oracle",
            "sample": (f"{len(secs)} whole decode step(s): all {wl.B} sequences through all {wl.L} "
                       f"layers (Full index over N={wl.N}, {sum(m == 'RI' for m in wl.modes)} Reindex, "
                       f"{wl.L} attentions), one sequence per thread: {sec:.2f} s"),
            "seconds": round(sec, 2)}


REFERENCE_DEFAULT_STEPS = 10


def run_reference(args, world, rank, local):
    """The oracle timed as the reference arm: every step is one whole decode step of the batch
    (all B sequences, one per host thread), so ms_per_step is the wall time of one step."""
    if rank != 0:
        return
    from oracle import build as oracle_build
    oracle_build.build()
    dev = torch.device("cuda", local) if torch.cuda.is_available() else torch.device("cpu")
    wl = WORKLOADS[args.workload]
    steps = args.steps if args.steps is not None else REFERENCE_DEFAULT_STEPS
    od = OracleDecode(wl, dev, list(range(wl.B)), host_threads())
    try:
        for _ in range(args.warmup):
            od.step()
        secs = [od.step() for _ in range(steps)]
    finally:
        od.close()
    per_step = statistics.mean(secs)
    value = wl.L / per_step
    sample = (f"every step: all {wl.B} sequences through all {wl.L} layers, one sequence per "
              f"thread on {od.threads} threads ({per_step:.2f} s per step)")
    line = {"metric": METRIC, "value": round(value, 4), "unit": "layer-steps/s", "n_gpus": world,
            "steps": steps, "warmup": args.warmup,
            "ms_per_step": round(per_step * 1e3, 2), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": wl.name, "B_per_gpu": wl.B, "N": wl.N,
                       "layers": ",".join(wl.modes), "K": wl.K, "P": wl.P, "W": wl.W,
                       "parallelism": f"dp{world} (independent sequences)"},
            "cpu_baseline": {"value": round(value, 4), "unit": "layer-steps/s",
                             "cores": od.threads, "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 4), "unit": "layer-steps/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ CED projection measurement

CED_METRIC = "CED KV projection + MXFP4 epilogue TFLOP/s (bf16 tensor cores), 1 B200"
CED_SHAPE = dict(B=8, n=4096, d=4096)   # 32,768 new tokens, hidden size 4,096


def ced_cpu_baseline(h, w, rows=4096):
    """The oracle's projection and quantisation of a few rows, split over the host threads (ctypes
    releases the GIL while the oracle runs), scaled to TFLOP/s."""
    import concurrent.futures as cf
    import numpy as np
    import oracle
    from oracle import build as oracle_build
    oracle_build.build()
    d = h.shape[-1]
    hb = h.reshape(-1, d)[:rows].contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    wb = w.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    threads = max(1, min(host_threads(), rows // 16, 64))
    parts = np.array_split(hb, threads)

    def one(part):
        c, _ = oracle.ced_project(np.ascontiguousarray(part), wb)
        oracle.mxfp4_quantize_f32(c.astype(np.float32))

    with cf.ThreadPoolExecutor(max_workers=threads) as ex:
        t = time.perf_counter()
        list(ex.map(one, parts))
        sec = time.perf_counter() - t
    value = 2.0 * rows * 512 * d / sec / 1e12
    return {"value": round(value, 6), "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
            "sample": f"{rows} token rows of d = {d} projected and quantised, split over {threads} "
                      f"threads ({sec:.2f} s)",
            "seconds": round(sec, 2)}


def run_ced(args, world, rank, local):
    import sparse_attention_decode_kv_b200 as csa2
    from sparse_attention_decode_kv_b200 import build as csa2_build
    if rank == 0:
        csa2_build.build()
    barrier(world)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    B, n, d = CED_SHAPE["B"], CED_SHAPE["n"], CED_SHAPE["d"]
    g = torch.Generator(device=dev).manual_seed(1000 + rank)
    h = torch.randn(B, n, d, device=dev, generator=g).to(torch.bfloat16)
    w = (torch.randn(512, d, device=dev, generator=g) / d ** 0.5).to(torch.bfloat16)
    codes = torch.empty(B, n, 256, dtype=torch.uint8, device=dev)
    scales = torch.empty(B, n, 32, dtype=torch.uint8, device=dev)
    pos = torch.zeros(B, dtype=torch.int32, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        csa2.ced_project_quant(h, w, pos, codes, scales, err)

    K, W = args.steps, args.warmup
    launches0 = csa2.launch_count()
    step()
    torch.cuda.synchronize()
    per_step_launches = csa2.launch_count() - launches0
    for _ in range(W):
        step()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        barrier(world)
        torch.cuda.synchronize()
        t0.record(stream)
        for _ in range(K):
            step()
        t1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
    ms = max_over_ranks(world, t0.elapsed_time(t1), dev) / K
    if int(err.item()):
        raise RuntimeError(f"device error flags {int(err.item()):#x} during the benchmark")
    flop = 2.0 * B * n * 512 * d
    tflops = flop / (ms / 1e3) / 1e12
    peak, peak_kind = measured_tensor_peak()

    e2e = None
    if not args.no_e2e:
        hh = h.cpu().pin_memory()
        hc = torch.empty(codes.shape, dtype=torch.uint8).pin_memory()
        hs = torch.empty(scales.shape, dtype=torch.uint8).pin_memory()
        ke = max(1, min(K, 20))
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(ke):
            h.copy_(hh, non_blocking=True)
            step()
            hc.copy_(codes, non_blocking=True)
            hs.copy_(scales, non_blocking=True)
        b.record(stream)
        torch.cuda.synchronize()
        e_ms = a.elapsed_time(b) / ke
        e2e = {"value": round(flop / (e_ms / 1e3) / 1e12, 2), "unit": "TFLOP/s",
               "h2d_bytes_per_step": h.numel() * 2,
               "d2h_bytes_per_step": codes.numel() + scales.numel()}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = ced_cpu_baseline(h, w)
    line = {
        "metric": CED_METRIC, "value": round(world * tflops, 2), "unit": "TFLOP/s",
        "n_gpus": world, "steps": K, "warmup": W, "ms_per_step": round(ms, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16-in fp32-acc (mxfp4 out)", "data": "synthetic",
        "config": {"workload": f"ced-projection-B{B}-n{n}-d{d}", "tokens_per_gpu": B * n,
                   "d": d, "channels": 512,
                   "l2": "inputs larger than L2 (h is %.0f MB)" % (h.numel() * 2 / 1e6),
                   "parallelism": f"dp{world} (independent token batches)"},
        "roofline": {"kernel": "ced_pair_kernel (tcgen05 cta_group::2 GEMM + MXFP4 epilogue)",
                     "bound": "tensor", "achieved": round(tflops, 1), "peak": peak,
                     "unit": "TFLOP/s", "frac": round(tflops / peak, 4), "peak_kind": peak_kind,
                     "algorithmic_flop_per_launch": flop, "launch_ms": round(ms, 4),
                     "traffic": ced_traffic_per_launch(B * n),
                     "algorithmic_bytes_per_launch": h.numel() * 2 + w.numel() * 2
                     + codes.numel() + scales.numel()},
        "gpu_launches": per_step_launches * K,
        "clocks": clocks.summary(),
    }
    if e2e is not None:
        line["e2e"] = e2e
    if cpu is not None:
        line["cpu_baseline"] = cpu
    if rank == 0:
        print(json.dumps(line), flush=True)

QUERIES_METRIC = ("multi-query sparse attention (prefill / verification): queries/s and achieved GB/s "
                  "of gathered MXFP4 + FP8 SWA bytes, 1 B200")
QUERIES_SHAPE = dict(B=8, N=131072, T=512, K=512, W=128)


def queries_cpu_baseline(q, codes, scales, idx, swa, swsc, qseq, lo, ln, n_sample=320):
    """The oracle's attention of a sample of the queries, split over the host threads (ctypes
    releases the GIL while the oracle runs), scaled to queries/s."""
    import concurrent.futures as cf
    import numpy as np
    import oracle
    from oracle import build as oracle_build
    oracle_build.build()
    Q = q.shape[0]
    threads = max(1, min(host_threads(), 64))
    n_sample = min(Q, max(n_sample, 8 * threads))
    pick = np.linspace(0, Q - 1, n_sample).astype(np.int64)
    qb = q[pick].contiguous().view(torch.int16).cpu().numpy().view(np.uint16)

    def one(j):
        i = pick[j]
        b, a, n = int(qseq[i]), int(lo[i]), int(ln[i])
        oracle.attend_seq(qb[j], 1.0, codes[b], scales[b], idx[i].astype(np.int64),
                          swa[b, a:a + n], swsc[b, a:a + n], n)

    with cf.ThreadPoolExecutor(max_workers=threads) as ex:
        t0 = time.perf_counter()
        list(ex.map(one, range(n_sample)))
        sec = time.perf_counter() - t0
    return {"value": round(n_sample / sec, 3), "unit": "queries/s", "cores": threads, "kind": "oracle",
            "sample": f"{n_sample} of {Q} queries, evenly spaced, over {threads} threads ({sec:.2f} s)",
            "seconds": round(sec, 2)}


def run_queries(args, world, rank, local):
    import numpy as np
    import sparse_attention_decode_kv_b200 as csa2
    from sparse_attention_decode_kv_b200 import build as csa2_build
    if rank == 0:
        csa2_build.build()
    barrier(world)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    B, N, T, K, W = (QUERIES_SHAPE[k] for k in ("B", "N", "T", "K", "W"))
    Q = B * T
    g = torch.Generator(device=dev).manual_seed(3000 + rank)
    stream = torch.cuda.current_stream(dev)
    # the prefix: N cached entries per sequence, appended in chunks through the library
    cache = csa2.Cache(B, N, 0, device=dev)
    chunk = 16384
    for c0 in range(0, N, chunk):
        x = torch.randn(B, chunk, 512, device=dev, generator=g).to(torch.bfloat16)
        csa2.append_quant(x, None, torch.full((B,), c0, dtype=torch.int32, device=dev),
                          cache.codes, cache.scales, None)
    # FP8 SWA rows of every position (E4M3 magnitudes below 448: bytes 0x00..0x7E per sign)
    mag = torch.randint(0, 0x7F, (B, N, 512), dtype=torch.uint8, device=dev, generator=g)
    sgn = torch.randint(0, 2, (B, N, 512), dtype=torch.uint8, device=dev, generator=g) << 7
    swa = mag | sgn
    del mag, sgn
    swsc = torch.rand(B, N, device=dev, generator=g) * 0.01 + 1e-4
    # query t of sequence b is the prompt token at position p = N - T + t: its selection is K
    # positions below p (sorted), its window the rows max(0, p - W + 1) .. p
    qseq = torch.arange(B, device=dev, dtype=torch.int32).repeat_interleave(T)
    pos = (N - T + torch.arange(T, device=dev)).repeat(B)
    idx = (torch.rand(Q, K, device=dev, generator=g) * pos[:, None]).to(torch.int32).sort(1).values
    lo = (pos - W + 1).clamp(min=0).to(torch.int32)
    ln = (pos - lo + 1).to(torch.int32)
    q = (torch.randn(Q, 16, 512, device=dev, generator=g) / 512 ** 0.5).to(torch.bfloat16)
    out = torch.empty(Q, 16, 512, device=dev)
    lse = torch.empty(Q, 16, device=dev)
    ws = csa2.workspace(csa2.attend_workspace_bytes(Q, K, W), dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    Nt = torch.full((B,), N, dtype=torch.int32, device=dev)
    torch.cuda.synchronize()

    def step():
        csa2.attend_queries(q, 1.0, cache.codes, cache.scales, Nt, qseq, idx, swa, swsc, lo, ln, W,
                            out, lse, ws, err)

    Ks, Wu = args.steps, args.warmup
    launches0 = csa2.launch_count()
    step()
    torch.cuda.synchronize()
    per_step_launches = csa2.launch_count() - launches0
    for _ in range(Wu):
        step()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        barrier(world)
        torch.cuda.synchronize()
        t0.record(stream)
        for _ in range(Ks):
            step()
        t1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
    ms = max_over_ranks(world, t0.elapsed_time(t1), dev) / Ks
    if int(err.item()):
        raise RuntimeError(f"device error flags {int(err.item()):#x} during the benchmark")
    per_query = K * 288 + W * 516
    byts = Q * per_query
    gbs = byts / (ms / 1e3) / 1e9
    peak, peak_kind = measured_peak()
    e2e = None
    if not args.no_e2e:
        q_h = q.cpu().pin_memory()
        idx_h = idx.cpu().pin_memory()
        out_h = torch.empty(out.shape, dtype=torch.float32).pin_memory()
        ke = max(1, min(Ks, 20))
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(ke):
            q.copy_(q_h, non_blocking=True)
            idx.copy_(idx_h, non_blocking=True)
            step()
            out_h.copy_(out, non_blocking=True)
        b.record(stream)
        torch.cuda.synchronize()
        e_ms = a.elapsed_time(b) / ke
        e2e = {"value": round(world * Q / (e_ms / 1e3), 1), "unit": "queries/s",
               "h2d_bytes_per_step": q.numel() * 2 + idx.numel() * 4,
               "d2h_bytes_per_step": out.numel() * 4}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = queries_cpu_baseline(q.cpu(), cache.codes.cpu().numpy(), cache.scales.cpu().numpy(),
                                   idx.cpu().numpy(), swa.cpu().numpy(), swsc.cpu().numpy(),
                                   qseq.cpu().numpy(), lo.cpu().numpy(), ln.cpu().numpy())
    line = {
        "metric": QUERIES_METRIC, "value": round(world * Q / (ms / 1e3), 1), "unit": "queries/s",
        "n_gpus": world, "steps": Ks, "warmup": Wu, "ms_per_step": round(ms, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "fp16-in fp32-acc (mxfp4 + fp8 cache)", "data": "synthetic",
        "config": {"workload": f"prefill-queries-B{B}-N{N}-T{T}-K{K}-W{W}", "queries": Q,
                   "sequences": B, "cached_entries": N, "K": K, "W": W,
                   "l2": "inputs larger than L2 (%.0f MB of MXFP4 cache, %.0f MB of SWA rows)"
                         % (cache.codes.numel() * 1.125 / 1e6, swa.numel() * 1.0078 / 1e6),
                   "parallelism": f"dp{world} (independent sequences)"},
        "achieved_gbs": round(gbs, 1),
        "roofline": {"kernel": "attend_tc_kernel (tcgen05, multi-query)", "bound": "hbm",
                     "achieved": round(gbs, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(gbs / peak, 4), "peak_kind": peak_kind,
                     "algorithmic_bytes_per_launch": byts,
                     "algorithmic_bytes_per_query": per_query,
                     "launch_ms": round(ms, 4),
                     "traffic": (lambda c: None if c is None else c["dram_bytes_per_launch"])(
                         captured_traffic("attend_queries_traffic.json")),
                     "note": "algorithmic bytes count every query's gathered rows; neighbouring "
                             "queries share window rows, which L2 serves"},
        "gpu_launches": per_step_launches * Ks,
        "clocks": clocks.summary(),
    }
    if e2e is not None:
        line["e2e"] = e2e
    if cpu is not None:
        line["cpu_baseline"] = cpu
    if rank == 0:
        print(json.dumps(line), flush=True)


REPLAY_METRIC = ("SWA bounded replay: sequence-batch restores/s (8 prefixes: host->HBM reload of the "
                 "MXFP4 KV + indexer keys, FP8 SWA ring replayed from the last 128 tokens), 1 B200")
REPLAY_SHAPE = dict(B=8, N=1 << 20, W=128, d=4096)


def replay_cpu_baseline(hc, hs, hi, hwin, w, N):
    """The oracle as it stands: the reload as numpy copies of the persisted rows, and the oracle's
    replay of one sequence's window, scaled to the B sequences of one restore."""
    import numpy as np
    import oracle
    from oracle import build as oracle_build
    oracle_build.build()
    import concurrent.futures as cf
    B, W = hwin.shape[0], hwin.shape[1]
    hb = hwin.contiguous().view(torch.int16).numpy().view(np.uint16)
    wb = w.contiguous().view(torch.int16).numpy().view(np.uint16)
    t0 = time.perf_counter()
    for src in (hc, hs, hi.view(torch.int16)):
        np.copy(src.numpy())
    t_copy = time.perf_counter() - t0
    # the windows' replays, one sequence per host thread (ctypes releases the GIL)
    threads = max(1, min(host_threads(), B))

    def one(b):
        swa = np.zeros((1, W, 512), np.uint8)
        sc = np.zeros((1, W), np.float32)
        oracle.swa_replay(np.ascontiguousarray(hb[b:b + 1]), wb, [N], swa, sc)

    with cf.ThreadPoolExecutor(max_workers=threads) as ex:
        t0 = time.perf_counter()
        list(ex.map(one, range(threads)))
        t_rep = time.perf_counter() - t0
    rounds = -(-B // threads)
    sec = t_copy + rounds * t_rep
    return {"value": round(1.0 / sec, 4), "unit": "restores/s", "cores": threads, "kind": "oracle",
            "sample": f"all {B} sequences' rows copied with numpy ({t_copy:.2f} s) + the oracle's "
                      f"replay of {threads} of {B} windows in parallel ({t_rep:.2f} s), "
                      f"scaled to {rounds} round(s)",
            "seconds": round(t_copy + t_rep, 2)}


def run_replay(args, world, rank, local):
    import sparse_attention_decode_kv_b200 as csa2
    from sparse_attention_decode_kv_b200 import build as csa2_build
    if rank == 0:
        csa2_build.build()
    barrier(world)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    B, N, W, d = (REPLAY_SHAPE[k] for k in ("B", "N", "W", "d"))
    N = int(args.replay_n)
    if N < W or N % 8:
        raise SystemExit("--replay-n must be a multiple of 8 and at least the window (128)")
    g = torch.Generator(device=dev).manual_seed(2000 + rank)
    stream = torch.cuda.current_stream(dev)
    # the persisted state: written once from device buffers through csa2_cache_persist
    cache = csa2.Cache(B, N, W, device=dev)
    cache.codes.copy_(torch.randint(0, 256, cache.codes.shape, dtype=torch.uint8, device=dev,
                                    generator=g))
    cache.scales.copy_(torch.randint(0x28, 0x40, cache.scales.shape, dtype=torch.uint8, device=dev,
                                     generator=g))
    cache.ik.copy_(torch.randn(cache.ik.shape, device=dev, generator=g).to(torch.bfloat16))
    hc = torch.empty(cache.codes.shape, dtype=torch.uint8, pin_memory=True)
    hs = torch.empty(cache.scales.shape, dtype=torch.uint8, pin_memory=True)
    hi = torch.empty(cache.ik.shape, dtype=torch.bfloat16, pin_memory=True)
    Ns = [N] * B
    csa2.cache_persist(cache.codes, cache.scales, cache.ik, Ns, hc, hs, hi)
    hwin = torch.randn(B, W, d, device=dev, generator=g).to(torch.bfloat16)
    w = (torch.randn(512, d, device=dev, generator=g) / d ** 0.5).to(torch.bfloat16)
    Nt = torch.full((B,), N, dtype=torch.int32, device=dev)
    ws = csa2.workspace(csa2.swa_replay_workspace_bytes(B, W, d), device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    torch.cuda.synchronize()
    reload_bytes = hc.numel() + hs.numel() + hi.numel() * 2

    def step():
        csa2.cache_restore(hc, hs, hi, Ns, cache.codes, cache.scales, cache.ik)
        csa2.swa_replay(hwin, w, Nt, cache.swa, cache.swa_scale, ws, err)

    K, Wu = args.steps, args.warmup
    launches0 = csa2.launch_count()
    step()
    torch.cuda.synchronize()
    per_step_launches = csa2.launch_count() - launches0
    for _ in range(Wu):
        step()
    torch.cuda.synchronize()
    ev = lambda: torch.cuda.Event(enable_timing=True)
    # per-step events: step start, replay start and replay end (the last two recorded by the
    # library's profile hook around its two replay kernels); the reload is start -> replay start
    evs = [(ev(), ev(), ev()) for _ in range(K)]
    for trio in evs:  # materialise the event handles
        for e in trio:
            e.record(stream)
    L = csa2.lib()
    t0, t1 = ev(), ev()
    with ClockSampler(local) as clocks:
        barrier(world)
        torch.cuda.synchronize()
        t0.record(stream)
        for i in range(K):
            evs[i][0].record(stream)
            L.csa2_set_profile_events(6, ctypes.c_void_p(evs[i][1].cuda_event),
                                      ctypes.c_void_p(evs[i][2].cuda_event))
            step()
        t1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
    L.csa2_set_profile_events(6, None, None)
    copy_ms = [a.elapsed_time(b) for a, b, _ in evs]
    replay_ms = [b.elapsed_time(c) for _, b, c in evs]
    ms = max_over_ranks(world, t0.elapsed_time(t1), dev) / K
    if int(err.item()):
        raise RuntimeError(f"device error flags {int(err.item()):#x} during the benchmark")
    # the host link's own figure: one plain pinned host->device copy of the same bytes
    flat_h = torch.empty(reload_bytes, dtype=torch.uint8, pin_memory=True)
    flat_d = torch.empty(reload_bytes, dtype=torch.uint8, device=dev)
    flat_d.copy_(flat_h, non_blocking=True)
    torch.cuda.synchronize()
    a, b = ev(), ev()
    a.record(stream)
    for _ in range(3):
        flat_d.copy_(flat_h, non_blocking=True)
    b.record(stream)
    torch.cuda.synchronize()
    link_gbs = reload_bytes / (a.elapsed_time(b) / 3 / 1e3) / 1e9
    del flat_h, flat_d
    c_ms = statistics.median(copy_ms)
    r_ms = statistics.median(replay_ms)
    flop = 2.0 * B * W * 512 * d
    peak, peak_kind = measured_tensor_peak()
    e2e = None
    if not args.no_e2e:
        hw_host = hwin.cpu().pin_memory()
        sc_host = torch.empty(cache.swa_scale.shape, dtype=torch.float32).pin_memory()
        ke = max(1, min(K, 5))
        torch.cuda.synchronize()
        a, b = ev(), ev()
        a.record(stream)
        for _ in range(ke):
            hwin.copy_(hw_host, non_blocking=True)
            step()
            sc_host.copy_(cache.swa_scale, non_blocking=True)
        b.record(stream)
        torch.cuda.synchronize()
        e_ms = a.elapsed_time(b) / ke
        e2e = {"value": round(1e3 / e_ms, 3), "unit": "restores/s",
               "h2d_bytes_per_step": reload_bytes + hwin.numel() * 2,
               "d2h_bytes_per_step": cache.swa_scale.numel() * 4}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = replay_cpu_baseline(hc, hs, hi, hwin.cpu(), w.cpu(), N)
    line = {
        "metric": REPLAY_METRIC, "value": round(world * 1e3 / ms, 3), "unit": "restores/s",
        "n_gpus": world, "steps": K, "warmup": Wu, "ms_per_step": round(ms, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "u8 copies + bf16-in fp32-acc (fp8 out)", "data": "synthetic",
        "config": {"workload": f"swa-replay-restore-B{B}-N{N}-W{W}-d{d}", "sequences": B,
                   "tokens_per_sequence": N, "window": W, "d": d,
                   "l2": "inputs larger than L2 (%.2f GB reloaded per step)" % (reload_bytes / 1e9),
                   "parallelism": f"dp{world} (independent sequences)"},
        "reload": {"achieved_gbs": round(reload_bytes / (c_ms / 1e3) / 1e9, 1),
                   "peak_gbs": round(link_gbs, 1),
                   "peak_kind": "measured in this run: one pinned host-to-device copy of the same bytes",
                   "frac": round((reload_bytes / (c_ms / 1e3) / 1e9) / link_gbs, 4),
                   "bytes_per_step": reload_bytes, "ms": round(c_ms, 3)},
        "roofline": {"kernel": "replay_proj_kernel + replay_swa_kernel (tcgen05 split-K GEMM, "
                               "sum / bf16 / FP8 pass)",
                     "bound": "tensor", "achieved": round(flop / (r_ms / 1e3) / 1e12, 1),
                     "peak": peak, "unit": "TFLOP/s",
                     "frac": round(flop / (r_ms / 1e3) / 1e12 / peak, 4), "peak_kind": peak_kind,
                     "algorithmic_flop_per_launch": flop, "launch_ms": round(r_ms, 4),
                     "traffic": (lambda c: None if c is None else c["dram_bytes_per_launch"])(
                         captured_traffic("replay_traffic.json"))},
        "gpu_launches": per_step_launches * K,
        "clocks": clocks.summary(),
    }
    if e2e is not None:
        line["e2e"] = e2e
    if cpu is not None:
        line["cpu_baseline"] = cpu
    if rank == 0:
        print(json.dumps(line), flush=True)


# ------------------------------------------------------------- throughput sweep: append + Reuse

APPEND_METRIC = ("MXFP4 quantize-append GB/s (bf16 rows read + E2M1 codes and E4M3 scales written), "
                 "1,048,576 entries, 1 B200")
SWEEP_METRIC = ("Reuse-mode sparse attention GB/s (gathered MXFP4 entries + FP8 SWA rows), "
                "N={N:,}, 1 B200")
L2_FLUSH_BYTES = 256 << 20  # twice the 126 MB L2


def l2_flush(buf):
    """Evict L2 by reading a buffer twice its size. A read leaves clean lines behind, so the next
    kernel's misses never wait for dirty data to be written back (a write flush would)."""
    torch.amax(buf)


def append_cpu_baseline(x, rows=65536):
    """The oracle's MXFP4 quantisation of `rows` entries, split over the host threads, scaled to
    GB/s of the same algorithmic bytes per entry."""
    import concurrent.futures as cf

    import numpy as np

    import oracle
    from oracle import build as oracle_build
    oracle_build.build()
    xb = x.reshape(-1, 512)[:rows].contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    threads = max(1, min(host_threads(), 64))
    parts = np.array_split(xb, threads)
    with cf.ThreadPoolExecutor(max_workers=threads) as ex:
        t = time.perf_counter()
        list(ex.map(oracle.mxfp4_quantize, parts))
        sec = time.perf_counter() - t
    per_entry = 512 * 2 + 256 + 32
    return {"value": round(rows * per_entry / sec / 1e9, 4), "unit": "GB/s", "cores": threads,
            "kind": "oracle",
            "sample": f"{rows} of {x.shape[0] * x.shape[1]} entries split over {threads} threads "
                      f"({sec:.2f} s)",
            "seconds": round(sec, 2)}


def run_append(args, world, rank, local):
    import sparse_attention_decode_kv_b200 as csa2
    from sparse_attention_decode_kv_b200 import build as csa2_build
    if rank == 0:
        csa2_build.build()
    barrier(world)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    wl = dataclasses.replace(workloads.APPEND_1M, seed=workloads.APPEND_1M.seed + 1000 * rank)
    x = workloads.append_rows(wl, dev)  # [1, 1,048,576, 512] bf16: 1.07 GB, larger than L2
    B, n = wl.B, wl.n
    codes = torch.empty(B, n, 256, dtype=torch.uint8, device=dev)
    scales = torch.empty(B, n, 32, dtype=torch.uint8, device=dev)
    pos = torch.zeros(B, dtype=torch.int32, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    L = csa2.lib()

    def step():
        csa2.append_quant(x, None, pos, codes, scales, None, dev_err=err)

    K, Wu = args.steps, args.warmup
    launches0 = csa2.launch_count()
    step()
    torch.cuda.synchronize()
    per_step_launches = csa2.launch_count() - launches0
    for _ in range(Wu):
        step()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(K)]
    for a, b in ev:
        a.record(stream)
        b.record(stream)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        barrier(world)
        torch.cuda.synchronize()
        t0.record(stream)
        for _ in range(K):
            step()
        t1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        for i in range(K):  # the kernel's own launch times, in a second pass
            L.csa2_set_profile_events(0, ctypes.c_void_p(ev[i][0].cuda_event),
                                      ctypes.c_void_p(ev[i][1].cuda_event))
            step()
            L.csa2_set_profile_events(0, None, None)
        torch.cuda.synchronize()
    if int(err.item()):
        raise RuntimeError(f"device error flags {int(err.item()):#x} during the benchmark")
    ms = max_over_ranks(world, t0.elapsed_time(t1), dev) / K
    launch_ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    per_entry = 512 * 2 + 256 + 32
    byts = B * n * per_entry
    peak, peak_kind = measured_peak()
    gbs = world * byts / (ms / 1e3) / 1e9
    k_gbs = byts / (launch_ms / 1e3) / 1e9
    e2e = None
    if not args.no_e2e:
        # the rows come from pinned host memory every step; the appended cache stays in HBM for
        # the decode step that reads it, and the step's result read back is the error word
        x_h = x.cpu().pin_memory()
        err_h = torch.empty(1, dtype=torch.int32).pin_memory()
        ke = max(1, min(K, 10))
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(ke):
            x.copy_(x_h, non_blocking=True)
            step()
            err_h.copy_(err, non_blocking=True)
        b.record(stream)
        torch.cuda.synchronize()
        e_ms = max_over_ranks(world, a.elapsed_time(b), dev) / ke
        e2e = {"value": round(world * byts / (e_ms / 1e3) / 1e9, 1), "unit": "GB/s",
               "h2d_bytes_per_step": x.numel() * 2, "d2h_bytes_per_step": 4,
               "ms_per_step": round(e_ms, 4),
               "note": "bounded by the host link: the 1.07 GB of bf16 rows cross it every step"}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = append_cpu_baseline(x)
    line = {
        "metric": APPEND_METRIC, "value": round(gbs, 1), "unit": "GB/s", "n_gpus": world,
        "steps": K, "warmup": Wu, "ms_per_step": round(ms, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16 in, e2m1 codes + e4m3 scales out",
        "data": "synthetic",
        "config": {"workload": f"append-1M-B{B}-n{n}", "entries": B * n,
                   "values": "N(0,1), 0.1% of elements x20",
                   "l2": "inputs larger than L2 (%.2f GB of bf16 rows per step)" % (x.numel() * 2 / 1e9),
                   "parallelism": f"dp{world} (independent caches)"},
        "entries_per_s": round(world * B * n / (ms / 1e3), 1),
        "roofline": {"kernel": "append_kernel (MXFP4 quantize-append)", "bound": "hbm",
                     "achieved": round(k_gbs, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(k_gbs / peak, 4), "peak_kind": peak_kind,
                     "algorithmic_bytes_per_launch": byts,
                     "algorithmic_bytes_per_entry": per_entry, "launch_ms": round(launch_ms, 4),
                     "traffic": (lambda c: None if c is None else int(round(c["dram_bytes_per_entry"] * B * n)))(
                         captured_traffic("append_traffic.json")),
                     "timing": "CUDA events around every append launch in a second pass"},
        "gpu_launches": per_step_launches * K,
        "clocks": clocks.summary(),
    }
    if e2e is not None:
        line["e2e"] = e2e
    if cpu is not None:
        line["cpu_baseline"] = cpu
    if rank == 0:
        print(json.dumps(line), flush=True)


def fill_reuse_cache(csa2, wl, cache, dev):
    """Append every sequence's N rows through the library (the ring keeps the last W)."""
    for b0 in range(0, wl.B, 16):
        b1 = min(wl.B, b0 + 16)
        for c in range(workloads.n_chunks(wl)):
            x = torch.stack([workloads.reuse_kv_chunk(wl, b, c, dev) for b in range(b0, b1)])
            pos = torch.full((b1 - b0,), c * workloads.CHUNK, dtype=torch.int32, device=dev)
            csa2.append_quant(x, None, pos, cache.codes[b0:b1], cache.scales[b0:b1], None,
                              cache.swa[b0:b1], cache.swa_scale[b0:b1])
            del x
    torch.cuda.synchronize()


def sweep_cpu_baseline(wl, q, idx, dev, budget_s=4.0):
    """The oracle's attention for sampled sequences (their rows regenerated and quantised by the
    oracle, not timed), one sequence per host thread, repeated to about `budget_s`, scaled to
    GB/s of the same algorithmic bytes."""
    import concurrent.futures as cf

    import numpy as np

    import oracle
    from oracle import build as oracle_build
    oracle_build.build()
    N, K, W = wl.N, wl.K, wl.W
    threads = max(1, min(host_threads(), wl.B, 16))
    seqs = list(range(threads))
    qb = workloads.bf16_bits(q[seqs])
    idx_h = idx[seqs].cpu().numpy()
    wpos = list(range(N - W, N))
    prep = []
    for j, b in enumerate(seqs):
        rows = np.zeros((K, 512), np.uint16)
        need = idx_h[j].astype(np.int64)
        for c in np.unique(need // workloads.CHUNK):
            m = need // workloads.CHUNK == c
            x = workloads.reuse_kv_chunk(wl, b, int(c), dev)
            rows[m] = workloads.bf16_bits(x[torch.as_tensor(need[m] - c * workloads.CHUNK, device=dev)])
        codes, scales = oracle.mxfp4_quantize(rows)
        xw = workloads.reuse_kv_chunk(wl, b, (N - 1) // workloads.CHUNK, dev)
        e, sc = oracle.swa_quantize(workloads.bf16_bits(xw[-W:]))
        ring = np.zeros((W, 512), np.uint8)
        rsc = np.zeros(W, np.float32)
        for i, p in enumerate(wpos):
            ring[p % W], rsc[p % W] = e[i], sc[i]
        prep.append((qb[j], codes, scales, np.arange(K, dtype=np.int64), ring, rsc))

    def one(p):
        oracle.attend_seq(p[0], 1.0, p[1], p[2], p[3], p[4], p[5], W)

    with cf.ThreadPoolExecutor(max_workers=threads) as ex:
        reps, sec = 0, 0.0
        while sec < budget_s:
            t = time.perf_counter()
            list(ex.map(one, prep))
            sec += time.perf_counter() - t
            reps += 1
    per_seq = K * 288 + W * 516
    return {"value": round(reps * threads * per_seq / sec / 1e9, 5), "unit": "GB/s",
            "cores": threads, "kind": "oracle",
            "sample": f"{threads} of {wl.B} sequences, one per thread, {reps} rounds ({sec:.2f} s)",
            "seconds": round(sec, 2)}


def run_sweep(args, world, rank, local):
    import sparse_attention_decode_kv_b200 as csa2
    from sparse_attention_decode_kv_b200 import build as csa2_build
    if rank == 0:
        csa2_build.build()
    barrier(world)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    L = csa2.lib()
    flush = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.int32, device=dev)
    batches = [int(v) for v in args.sweep_batches.split(",")]
    for B in batches:
        base = next((w for w in workloads.REUSE_SWEEP if w.B == B), None)
        if base is None or args.sweep_n != base.N:
            base = workloads.ReuseAttendWorkload(f"reuse-attend-B{B}-N{args.sweep_n}", B=B,
                                                 N=args.sweep_n)
        wl = dataclasses.replace(base, seed=base.seed + 1000 * rank)
        N, K, W = wl.N, wl.K, wl.W
        cache = csa2.Cache(B, N, W, device=dev)
        fill_reuse_cache(csa2, wl, cache, dev)
        idx = workloads.reuse_indices(wl, dev)
        q = workloads.reuse_queries(wl, dev)
        out = torch.empty(B, 16, 512, device=dev)
        lse = torch.empty(B, 16, device=dev)
        ws = csa2.workspace(csa2.attend_workspace_bytes(B, K, W), dev)
        err = torch.zeros(1, dtype=torch.int32, device=dev)
        Nt = torch.full((B,), N, dtype=torch.int32, device=dev)
        swa_len = torch.full((B,), W, dtype=torch.int32, device=dev)

        def call():
            csa2.attend(csa2.MODE_REUSE, q, 1.0, cache.codes, cache.scales, Nt, idx, cache.swa,
                        cache.swa_scale, swa_len, out, lse, ws, err)

        Ks, Wu = args.steps, args.warmup
        launches0 = csa2.launch_count()
        call()
        torch.cuda.synchronize()
        per_call_launches = csa2.launch_count() - launches0
        for _ in range(Wu):
            l2_flush(flush)
            call()
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(Ks)]
        for a, b in ev:
            a.record(stream)
            b.record(stream)
        # every call follows an L2 flush (a 256 MB read); the events bracket the call alone
        with ClockSampler(local) as clocks:
            barrier(world)
            torch.cuda.synchronize()
            for i in range(Ks):
                l2_flush(flush)
                L.csa2_set_profile_events(4, ctypes.c_void_p(ev[i][0].cuda_event),
                                          ctypes.c_void_p(ev[i][1].cuda_event))
                call()
                L.csa2_set_profile_events(4, None, None)
            torch.cuda.synchronize()
            barrier(world)
        if int(err.item()):
            raise RuntimeError(f"device error flags {int(err.item()):#x} during the benchmark")
        call_ms = max_over_ranks(world, statistics.mean(a.elapsed_time(b) for a, b in ev), dev)
        per_seq = K * 288 + W * 516
        byts = B * per_seq
        gbs = world * byts / (call_ms / 1e3) / 1e9
        peak, peak_kind = measured_peak()
        e2e = None
        if not args.no_e2e:
            q_h, idx_h = q.cpu().pin_memory(), idx.cpu().pin_memory()
            out_h = torch.empty(out.shape, dtype=torch.float32).pin_memory()
            lse_h = torch.empty(lse.shape, dtype=torch.float32).pin_memory()
            ee = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(Ks)]
            torch.cuda.synchronize()
            for i in range(Ks):
                l2_flush(flush)
                ee[i][0].record(stream)
                q.copy_(q_h, non_blocking=True)
                idx.copy_(idx_h, non_blocking=True)
                call()
                out_h.copy_(out, non_blocking=True)
                lse_h.copy_(lse, non_blocking=True)
                ee[i][1].record(stream)
            torch.cuda.synchronize()
            e_ms = max_over_ranks(world, statistics.mean(a.elapsed_time(b) for a, b in ee), dev)
            e2e = {"value": round(world * byts / (e_ms / 1e3) / 1e9, 2), "unit": "GB/s",
                   "h2d_bytes_per_step": q.numel() * 2 + idx.numel() * 4,
                   "d2h_bytes_per_step": out.numel() * 4 + lse.numel() * 4,
                   "ms_per_step": round(e_ms, 5)}
        cpu = None
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            cpu = sweep_cpu_baseline(wl, q, idx, dev)
        line = {
            "metric": SWEEP_METRIC.format(N=N), "value": round(gbs, 1), "unit": "GB/s", "n_gpus": world,
            "steps": Ks, "warmup": Wu, "ms_per_step": round(call_ms, 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "fp16-in fp32-acc (mxfp4 + fp8 cache)",
            "data": "synthetic",
            "config": {"workload": wl.name, "B_per_gpu": B, "N": N, "K": K, "W": W,
                       "indices": "512 uniform without replacement per sequence",
                       "l2": "flushed before every call (a 256 MB read outside the events)",
                       "parallelism": f"dp{world} (independent sequences)"},
            "calls_per_s": round(world * 1e3 / call_ms, 1),
            "roofline": {"kernel": ("attend_tc_kernel (tcgen05)" if B >= 64 else
                                    "attend_kernel + attend_merge_kernel (mma.sync)") + ", one csa2_attend call",
                         "bound": "hbm", "achieved": round(byts / (call_ms / 1e3) / 1e9, 1),
                         "peak": peak, "unit": "GB/s",
                         "frac": round(byts / (call_ms / 1e3) / 1e9 / peak, 4),
                         "peak_kind": peak_kind, "algorithmic_bytes_per_launch": byts,
                         "algorithmic_bytes_per_sequence": per_seq,
                         "launch_ms": round(call_ms, 5),
                         "traffic": (lambda c: None if c is None else int(round(c["dram_bytes_per_sequence"] * B)))(
                             captured_traffic("attend_reuse_traffic.json")),
                         "timing": "CUDA events around every call, after an L2 flush"},
            "gpu_launches": per_call_launches * Ks,
            "clocks": clocks.summary(),
        }
        if e2e is not None:
            line["e2e"] = e2e
        if cpu is not None:
            line["cpu_baseline"] = cpu
        if rank == 0:
            print(json.dumps(line), flush=True)
        del cache, ws
        torch.cuda.empty_cache()


def main():
    args = parse()
    if args.steps is None and args.impl == "ours":
        args.steps = 1000
    world, rank, local = dist_setup()
    try:
        if args.ced and args.impl == "ours":
            run_ced(args, world, rank, local)
        elif args.replay and args.impl == "ours":
            run_replay(args, world, rank, local)
        elif args.queries and args.impl == "ours":
            run_queries(args, world, rank, local)
        elif args.append and args.impl == "ours":
            run_append(args, world, rank, local)
        elif args.sweep and args.impl == "ours":
            run_sweep(args, world, rank, local)
        elif args.impl == "reference":
            run_reference(args, world, rank, local)
        else:
            run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
