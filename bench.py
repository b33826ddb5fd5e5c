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

With --gpus N > 1 run under torchrun: every rank decodes its own batch (data parallel, no
collective on the data path); the step time is the max over ranks.
--impl reference times the CPU oracle (a plain restatement of the same definitions) on a bounded
sample of the same workload, on rank 0 only.
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
    ap.add_argument("--steps", type=int, default=1000)
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

    # warm-up (eager), then capture the parts around the Full index into CUDA graphs; the Full
    # index call is launched eagerly each step so that its scan kernel gets its own events
    launches0 = csa2.launch_count()
    st.eager_step()
    torch.cuda.synchronize()
    per_step_launches = csa2.launch_count() - launches0
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

    def step(i=None):
        g_app.replay()
        if i is not None:
            L.csa2_set_profile_events(1, ctypes.c_void_p(ev_scan[i][0].cuda_event),
                                      ctypes.c_void_p(ev_scan[i][1].cuda_event))
        st.index_full()
        if i is not None:
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
        for i in range(K):
            step(i)
        t1.record(stream)
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
        cpu = cpu_baseline(wl, dev, samples=wl.B)

    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "layer-steps/s", "n_gpus": world,
        "steps": K, "warmup": W, "ms_per_step": round(ms_step, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16/fp16-in fp32-acc (mxfp4+fp8 cache)",
        "data": "synthetic",
        "config": {"workload": wl.name, "B_per_gpu": wl.B, "N": wl.N, "layers": ",".join(wl.modes),
                   "K": wl.K, "P": wl.P, "W": wl.W, "cuda_graph": "append+layers; Full index eager",
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
    g_app1, g_layers1 = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_app1, stream=torch.cuda.Stream(dev)):
        st.append_new()
    with torch.cuda.graph(g_layers1, stream=torch.cuda.Stream(dev)):
        st.layers()
    use(0)
    torch.cuda.synchronize()

    def step_set(j):
        if j == 0:
            step()
        else:
            g_app1.replay()
            use(1)
            st.index_full()
            use(0)
            g_layers1.replay()

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
                          "while step i runs (two buffer sets, two graph pairs)",
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


def oracle_one_sequence(wl, sample, dev):
    """Time the oracle on one sequence's full stack step. Returns seconds of oracle compute (data
    preparation between the index and attention parts is not timed)."""
    import numpy as np

    import oracle
    N, K, P, W = wl.N, wl.K, wl.P, wl.W
    ik = sample["ik"][None]
    t_index = 0.0
    topks = []
    t = time.perf_counter()
    r = oracle.index_full(sample["iq"][0][None], sample["w"][0][None], ik, [N], K, P)
    t_index += time.perf_counter() - t
    pool = r["pool"]
    topks.append(r["topk"][0])
    j = 1
    per_layer = []
    for m in wl.modes:
        if m == "F":
            per_layer.append(topks[0])
        elif m == "RI":
            t = time.perf_counter()
            rr = oracle.index_reindex(sample["iq"][j][None], sample["w"][j][None], ik, pool, K)
            t_index += time.perf_counter() - t
            topks.append(rr["topk"][0])
            per_layer.append(rr["topk"][0])
            j += 1
        else:
            per_layer.append(per_layer[-1])
    # untimed: the oracle quantises the rows the attention needs (remapped to a compact cache)
    need = sorted(set(int(v) for tk in per_layer for v in tk if v >= 0))
    rows = oracle_rows(wl, sample["b"], need, dev)
    codes, scales = oracle.mxfp4_quantize(rows)
    remap = {p: i for i, p in enumerate(need)}
    swa_rows = oracle_rows(wl, sample["b"], list(range(N - min(N, W), N)), dev)
    swa, swsc = oracle.swa_quantize(swa_rows)
    # ring slot of position p is p mod W
    ring = np.zeros((W, 512), np.uint8)
    rsc = np.zeros((W,), np.float32)
    for i, p in enumerate(range(N - min(N, W), N)):
        ring[p % W], rsc[p % W] = swa[i], swsc[i]
    t_att = 0.0
    for l, tk in enumerate(per_layer):
        idx = np.array([remap[int(v)] if v >= 0 else -1 for v in tk], np.int64)
        t = time.perf_counter()
        oracle.attend_seq(sample["q"][l], wl.softmax_scale, codes, scales, idx, ring, rsc, min(N, W))
        t_att += time.perf_counter() - t
    return t_index + t_att


def cpu_baseline(wl, dev, samples=1):
    seqs = list(range(min(samples, wl.B)))
    inputs, _ = oracle_sample_inputs(wl, dev, seqs)
    secs = [oracle_one_sequence(wl, s, dev) for s in inputs]
    per_seq = statistics.mean(secs)
    value = wl.L / (per_seq * wl.B)
    return {"value": round(value, 4), "unit": "layer-steps/s", "cores": 1, "kind": "oracle",
            "sample": (f"{len(seqs)} of {wl.B} sequences through all {wl.L} layers "
                       f"(Full index over N={wl.N}, {sum(m == 'RI' for m in wl.modes)} Reindex, "
                       f"{wl.L} attentions), scaled to the batch: {per_seq:.2f} s per sequence"),
            "seconds": round(sum(secs), 2)}


def run_reference(args, world, rank, local):
    if rank != 0:
        return
    from oracle import build as oracle_build
    oracle_build.build()
    dev = torch.device("cuda", local) if torch.cuda.is_available() else torch.device("cpu")
    wl = WORKLOADS[args.workload]
    inputs, _ = oracle_sample_inputs(wl, dev, [0])
    for _ in range(args.warmup):
        oracle_one_sequence(wl, inputs[0], dev)
    secs = [oracle_one_sequence(wl, inputs[0], dev) for _ in range(args.steps)]
    per_seq = statistics.mean(secs)
    value = wl.L / (per_seq * wl.B)
    sample = (f"sequence 0 of {wl.B} through all {wl.L} layers per step, scaled to the batch "
              f"({per_seq:.2f} s per sequence)")
    line = {"metric": METRIC, "value": round(value, 4), "unit": "layer-steps/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(per_seq * wl.B * 1e3, 2), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": wl.name, "B_per_gpu": wl.B, "N": wl.N,
                       "layers": ",".join(wl.modes), "K": wl.K, "P": wl.P, "W": wl.W},
            "cpu_baseline": {"value": round(value, 4), "unit": "layer-steps/s", "cores": 1,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 4), "unit": "layer-steps/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)



# ------------------------------------------------------------------ CED projection measurement

CED_METRIC = "CED KV projection + MXFP4 epilogue TFLOP/s (bf16 tensor cores), 1 B200"
CED_SHAPE = dict(B=8, n=4096, d=4096)   # 32,768 new tokens, hidden size 4,096


def ced_cpu_baseline(h, w, rows=4096):
    """The oracle's projection and quantisation of a few rows, scaled to TFLOP/s."""
    import numpy as np
    import oracle
    from oracle import build as oracle_build
    oracle_build.build()
    d = h.shape[-1]
    hb = h.reshape(-1, d)[:rows].contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    wb = w.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    t = time.perf_counter()
    c, _ = oracle.ced_project(hb, wb)
    oracle.mxfp4_quantize_f32(c.astype(np.float32))
    sec = time.perf_counter() - t
    value = 2.0 * rows * 512 * d / sec / 1e12
    return {"value": round(value, 6), "unit": "TFLOP/s", "cores": 1, "kind": "oracle",
            "sample": f"{rows} token rows of d = {d} projected and quantised ({sec:.2f} s)",
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
    """The oracle's attention of a sample of the queries, scaled to queries/s."""
    import numpy as np
    import oracle
    from oracle import build as oracle_build
    oracle_build.build()
    Q = q.shape[0]
    pick = np.linspace(0, Q - 1, n_sample).astype(np.int64)
    qb = q[pick].contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    t0 = time.perf_counter()
    for j, i in enumerate(pick):
        b, a, n = int(qseq[i]), int(lo[i]), int(ln[i])
        oracle.attend_seq(qb[j], 1.0, codes[b], scales[b], idx[i].astype(np.int64),
                          swa[b, a:a + n], swsc[b, a:a + n], n)
    sec = time.perf_counter() - t0
    return {"value": round(n_sample / sec, 3), "unit": "queries/s", "cores": 1, "kind": "oracle",
            "sample": f"{n_sample} of {Q} queries, evenly spaced ({sec:.2f} s)",
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
        "roofline": {"kernel": "attend_kernel (multi-query)", "bound": "hbm",
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
    B, W = hwin.shape[0], hwin.shape[1]
    hb = hwin[:1].contiguous().view(torch.int16).numpy().view(np.uint16)
    wb = w.contiguous().view(torch.int16).numpy().view(np.uint16)
    t0 = time.perf_counter()
    for src in (hc, hs, hi.view(torch.int16)):
        np.copy(src.numpy())
    t_copy = time.perf_counter() - t0
    swa = np.zeros((1, W, 512), np.uint8)
    sc = np.zeros((1, W), np.float32)
    t0 = time.perf_counter()
    oracle.swa_replay(hb, wb, [N], swa, sc)
    t_rep = time.perf_counter() - t0
    sec = t_copy + B * t_rep
    return {"value": round(1.0 / sec, 4), "unit": "restores/s", "cores": 1, "kind": "oracle",
            "sample": f"all {B} sequences' rows copied with numpy ({t_copy:.2f} s) + the oracle's "
                      f"replay of 1 of {B} windows ({t_rep:.2f} s), scaled to {B}",
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


def main():
    args = parse()
    world, rank, local = dist_setup()
    try:
        if args.ced and args.impl == "ours":
            run_ced(args, world, rank, local)
        elif args.replay and args.impl == "ours":
            run_replay(args, world, rank, local)
        elif args.queries and args.impl == "ours":
            run_queries(args, world, rank, local)
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
