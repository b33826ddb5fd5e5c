"""The whole decode step at each stack workload's full size, launched the way bench.py times it,
checked on sampled sequences against the oracle run on regenerated inputs.

Method: "DeepSeek V4.1 Flash 拆解" (austincafe.tech), section 一. The decode step appends the new
entry (MXFP4 main KV, FP8 SWA ring, indexer key). The Full layer scores every entry, takes the
Top-K and builds the pool of blocks × 8 positions. Reindex layers rescore the pool with their own
query. Every layer attends over its indices and the SWA rows in one softmax; Reuse layers take
the most recent indices.

The workloads:
- tiny Full layer (B 1, N 4,096);
- the 3-layer stack (B 4, N 65,536);
- the 8-layer pattern (B 16, N 262,144);
- the million-entry decode (B 8, N 1,048,576).

Launch pattern, as in bench.py: one eager warm-up step, then the append and the layers captured
as CUDA graphs and replayed around an eager Full-index call. For a sample of sequences the
oracle recomputes everything from the workload's seeded generators, nothing the kernels wrote:
- the cache rows and keys, with row N-1 replaced by the step's new token;
- the Full Top-K and the pool;
- the Reindex selections;
- every layer's attention over its own quantisation of the rows.

Checks:
- Index sets follow the boundary-swap rule.
- The pool is the expansion of the GPU's block set.
- Attention is within the output tolerance.
- A sampled row's MXFP4 bytes are exact.

Where a tolerated swap makes the GPU's set differ from the oracle's, the stage after it is
computed by the oracle on the GPU's set (logged), so a swap never cascades.
"""
import numpy as np
import pytest
import torch

import bench
import oracle
import workloads
from _helpers import ascending_padded, check_attention, check_selection

pytestmark = pytest.mark.gpu

CASES = {
    "tiny": (workloads.TINY, [0]),
    "stack3": (workloads.STACK3, [0, 3]),
    "pattern8": (workloads.PATTERN8, [0, 15]),
    "decode-1M": (workloads.MILLION, [5]),
}


def _run_step_as_bench(wl, dev):
    st = bench.Stack(wl, dev)
    st.eager_step()                        # warm-up step, as bench.py does
    torch.cuda.synchronize()
    g_app, g_layers = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_app, stream=torch.cuda.Stream(dev)):
        st.append_new()
    with torch.cuda.graph(g_layers, stream=torch.cuda.Stream(dev)):
        st.layers()
    torch.cuda.synchronize()
    st.out.fill_(float("nan"))             # the timed step must write every output again
    st.lse.fill_(float("nan"))
    st.topk.fill_(-7)
    st.pool.fill_(-7)
    g_app.replay()
    st.index_full()
    g_layers.replay()
    torch.cuda.synchronize()
    return st


def _oracle_inputs(wl, b, dev):
    """bf16 bits of sequence b after the step: indexer keys [N, 64], the step's queries, and a
    function giving main-KV rows (row N-1 is the step's new token)."""
    si = workloads.step_inputs(wl, dev)
    x_new, ik_new = workloads.new_token(wl, dev)
    pdir = workloads.plant_direction(si["iq"][0, b], si["w"][0, b]) if wl.n_planted else None
    ik = torch.cat([workloads.ik_chunk(wl, b, c, dev, pdir) for c in range(workloads.n_chunks(wl))])
    ik[wl.N - 1] = ik_new[b, 0]
    new_row = workloads.bf16_bits(x_new[b, 0])

    def rows(pos):
        pos = np.asarray(pos, np.int64)
        out = np.zeros((len(pos), 512), np.uint16)
        for c in np.unique(pos // workloads.CHUNK):
            m = pos // workloads.CHUNK == c
            x = workloads.kv_chunk(wl, b, int(c), dev)
            out[m] = workloads.bf16_bits(x[torch.as_tensor(pos[m] - c * workloads.CHUNK, device=dev)])
        out[pos == wl.N - 1] = new_row
        return out

    return dict(ik=workloads.bf16_bits(ik), iq=workloads.bf16_bits(si["iq"][:, b]),
                w=si["w"][:, b].cpu().numpy(), q=workloads.bf16_bits(si["q"][:, b]), rows=rows)


@pytest.mark.parametrize("case", list(CASES))
def test_decode_step_matches_oracle(gpu, case):
    wl, seqs = CASES[case]
    st = _run_step_as_bench(wl, gpu)
    assert int(st.dev_err.item()) == 0
    N, K, P, W = wl.N, wl.K, wl.P, wl.W
    topk_gpu = st.topk.cpu().numpy()
    pool_gpu = st.pool.cpu().numpy()
    out_gpu = st.out.cpu().numpy()
    lse_gpu = st.lse.cpu().numpy()
    for b in seqs:
        inp = _oracle_inputs(wl, b, gpu)
        ik = inp["ik"]
        # ---- Full layer: Top-K positions and the pool
        s, tau = oracle.index_scores(inp["iq"][0], inp["w"][0], ik, with_tol=True)
        ref = oracle.index_full(inp["iq"][0][None], inp["w"][0][None], ik[None], [N], K, P)
        ascending_padded(topk_gpu[0, b], K)
        check_selection(topk_gpu[0, b], ref["topk"][0], lambda i: s[i], lambda i: tau[i],
                        f"{case} full topk b={b}")
        nb = (N + 7) // 8
        bm = s[: nb * 8].reshape(nb, 8).max(1)
        bt = tau[: nb * 8].reshape(nb, 8).max(1)
        gblocks = sorted(set(int(p) // 8 for p in pool_gpu[b] if p >= 0))
        oblocks = sorted(set(int(p) // 8 for p in ref["pool"][0] if p >= 0))
        check_selection(gblocks, oblocks, lambda j: bm[j], lambda j: bt[j], f"{case} pool b={b}")
        expect = []
        for j in gblocks:
            expect += [p if p < N else -1 for p in range(8 * j, 8 * j + 8)]
        expect += [-1] * (8 * P - len(expect))
        assert list(pool_gpu[b]) == expect, "the pool is not the expansion of its block set"
        same_pool = gblocks == oblocks
        if not same_pool:
            print(f"POOL-SWAP {case} b={b}: Reindex layers checked on the GPU's pool")
        pool_for_oracle = (ref["pool"] if same_pool else pool_gpu[b][None]).astype(np.int64)
        # ---- Reindex layers and the indices each layer attends over
        sel = {0: ref["topk"][0]}
        for j in range(1, wl.n_idx):
            rr = oracle.index_reindex(inp["iq"][j][None], inp["w"][j][None], ik[None],
                                      pool_for_oracle, K)
            sj, tj = oracle.index_scores(inp["iq"][j], inp["w"][j], ik, with_tol=True)
            ascending_padded(topk_gpu[j, b], K)
            check_selection(topk_gpu[j, b], rr["topk"][0], lambda i: sj[i], lambda i: tj[i],
                            f"{case} reindex {j} b={b}")
            sel[j] = rr["topk"][0]
        for j in sel:  # a tolerated swap: the attention of that layer uses the GPU's own set
            g = set(int(v) for v in topk_gpu[j, b] if v >= 0)
            if g != set(int(v) for v in sel[j] if v >= 0):
                print(f"TOPK-SWAP {case} b={b} index layer {j}: attention checked on the GPU set")
                sel[j] = topk_gpu[j, b].astype(np.int64)
        # ---- the oracle's own quantisation of the rows the layers read
        need = sorted(set(int(v) for j in sel for v in sel[j] if v >= 0) | {N - 1})
        xr = inp["rows"](need)
        codes, scales = oracle.mxfp4_quantize(xr)
        cg = st.cache.codes[b, torch.as_tensor(need, device=gpu)].cpu().numpy()
        sg = st.cache.scales[b, torch.as_tensor(need, device=gpu)].cpu().numpy()
        assert np.array_equal(cg, codes) and np.array_equal(sg, scales), "MXFP4 rows differ"
        remap = {p: i for i, p in enumerate(need)}
        sl = min(N, W)
        wpos = list(range(N - sl, N))
        e, sc = oracle.swa_quantize(inp["rows"](wpos))
        ring = np.zeros((W, 512), np.uint8)
        rsc = np.zeros(W, np.float32)
        for i, p in enumerate(wpos):
            ring[p % W], rsc[p % W] = e[i], sc[i]
        assert np.array_equal(st.cache.swa[b].cpu().numpy()[:sl], ring[:sl]), "SWA ring differs"
        # ---- every layer's attention
        j = -1
        for l, m in enumerate(wl.modes):
            if m in ("F", "RI"):
                j += 1
            idx = np.array([remap[int(v)] if v >= 0 else -1 for v in sel[j]], np.int64)
            ro, rl = oracle.attend_seq(inp["q"][l], wl.softmax_scale, codes, scales, idx,
                                       ring[:sl], rsc[:sl], sl)
            check_attention(out_gpu[l, b], lse_gpu[l, b], ro, rl)
