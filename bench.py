"""Benchmark of one draft-tree verification step (tree attention + LM-head logits + the
accept/resample walk) on B200, through the library's C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--temperature T]

Default workload: the Vicuna-7B-shaped static EAGLE tree (batch 1, 32 heads, head_dim 128,
bf16, prefix 1024, 45 tree rows, hidden 4096, vocab 32000) at temperature 1.  The batch-1
step does not shard, so N GPUs run N independent replicas ("scaling": "weak"); the value
is all replicas' steps over the slowest rank's device time.  Rank 0 prints one JSON line.

--impl reference times the CPU oracle (fp64, all host cores) on a bounded sample of the
same workload; it is a reported baseline, not a tuned program.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as wl  # noqa: E402

METRIC = "tree-verify steps/s and tree-tokens/s at 1 B200; achieved HBM GB/s as % of peak"
L2_FLUSH_BYTES = 512 << 20
FALLBACK_HBM_GBS = 6650.0
RERANK_CANDIDATES = 256
DRAFT_ROWS, DRAFT_K = 10, 10
STACK_LAYERS = 32  # the stacked-attention workload: one verify pass through every layer


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def _lm_head_traffic(workload: str):
    """DRAM bytes per LM-head launch from the committed ncu capture of this workload, or
    None when there is none or the kernel's sources changed since it was taken."""
    import hashlib
    path = os.path.join(ROOT, "profiles", f"lm_head_tc_{workload}.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    for rel, digest in rec["sources_sha256"].items():
        with open(os.path.join(ROOT, rel), "rb") as src:
            if hashlib.sha256(src.read()).hexdigest() != digest:
                return None
    return int(rec["traffic_bytes_per_launch"])


def step_bytes(w, prefix_lens):
    el = 2 if w.dtype == wl.BF16 else 4
    B, N, Hq, Hkv, D, H, V = (w.batch, w.num_nodes, w.num_q_heads, w.num_kv_heads, w.head_dim,
                              w.hidden, w.vocab)
    kv = int(np.sum(prefix_lens)) * Hkv * D * 2 * el
    wbytes = V * H * el
    lm = wbytes + B * N * H * el + B * N * V * 4
    return dict(kv=kv, w=wbytes, lm_head=lm, roofline_bytes=kv + wbytes)


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """Samples the SM clock and the clock-event reasons through NVML every 20 ms while
    the timed region runs (read-only queries)."""
    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}

    def __init__(self, device_index: int):
        self.idx = device_index
        self.samples = []
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None

    def _sample(self, nv, h):
        sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
        get = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        self.samples.append((sm, int(get(h))))

    def _run(self):
        try:
            import pynvml as nv
            nv.nvmlInit()
            h = nv.nvmlDeviceGetHandleByIndex(self._physical_index())
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
            self._sample(nv, h)
            while not self._stop.wait(0.02):
                self._sample(nv, h)
            self._sample(nv, h)
        except Exception as e:  # clocks are reported as unavailable, never fatal
            self.error = repr(e)

    def _physical_index(self):
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        if vis:
            ids = [v for v in vis.split(",") if v.strip()]
            if self.idx < len(ids) and ids[self.idx].strip().isdigit():
                return int(ids[self.idx])
        return self.idx

    def __enter__(self):
        self._t = threading.Thread(target=self._run, daemon=True)
        self._t.start()
        time.sleep(0.05)
        return self

    def __exit__(self, *exc):
        self._stop.set()
        self._t.join(timeout=5)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0,
                    "error": getattr(self, "error", "no samples")}
        mask = 0
        for _, r in self.samples:
            mask |= r
        reasons = sorted(n for n, bit in self.REASONS.items() if mask & bit)
        return {"sm_mhz": statistics.median(s for s, _ in self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(self.samples)}


# ---------------------------------------------------------------- oracle (CPU baseline)

def oracle_step_sample(w, inp, T, lm_stride=8):
    """One oracle step on a bounded sample: attention for every row, LM-head logits for
    every `lm_stride`-th tree row, and the full accept walk (which computes the logits
    rows it visits).  Returns the extrapolated seconds of one whole step and a label."""
    import oracle
    oracle.build()
    t0 = time.perf_counter()
    oracle.tree_attention(inp["q"], inp["k_prefix"], inp["v_prefix"], inp["prefix_lens"],
                          inp["k_tree"], inp["v_tree"], inp["parents"])
    t1 = time.perf_counter()
    M = w.batch * w.num_nodes
    rows = np.arange(0, M, lm_stride, dtype=np.int32)
    oracle.lm_head(inp["hidden"], inp["w_lm"], rows=rows)
    t2 = time.perf_counter()
    oracle.tree_accept(inp["draft_probs"], inp["tokens"], inp["parents"], T,
                       hidden=inp["hidden"], w_lm=inp["w_lm"])
    t3 = time.perf_counter()
    full = (t1 - t0) + (t2 - t1) * M / len(rows) + (t3 - t2)
    label = (f"attention all {w.batch * w.num_nodes * w.num_q_heads} rows + LM head {len(rows)} of "
             f"{M} rows (scaled x{M / len(rows):.2f}) + full accept walk; fp64 C oracle")
    return full, label, oracle.num_threads()


# ---------------------------------------------------------------- main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="vicuna7b_static", choices=sorted(wl.WORKLOADS))
    ap.add_argument("--temperature", type=float, default=1.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    w = wl.WORKLOADS[args.workload]
    T = args.temperature
    config = {"workload": f"{w.name}: B{w.batch} Hq{w.num_q_heads}/Hkv{w.num_kv_heads} D{w.head_dim} "
                          f"{w.dtype} prefix {w.prefix_len if w.prefix_min is None else f'U[{w.prefix_min},{w.prefix_len}]'} "
                          f"N{w.num_nodes} H{w.hidden} V{w.vocab} T{T:g}",
              "batch": w.batch, "tree_nodes": w.num_nodes, "prefix_len": w.prefix_len,
              "hidden": w.hidden, "vocab": w.vocab, "temperature": T,
              "l2": "flushed before every step: 512 MiB write then 256 MiB read, untimed",
              "parallelism": "replicas" if world > 1 else "single"}

    if args.impl == "reference":
        if rank != 0:
            return
        inp = wl.generate(w, T)
        times = []
        label, cores = "", 1
        for i in range(args.steps + args.warmup):
            t, label, cores = oracle_step_sample(w, inp, T)
            if i >= args.warmup:
                times.append(t)
        sec = float(np.mean(times))
        value = 1.0 / sec
        print(json.dumps({
            "impl": "reference", "metric": METRIC, "value": value, "unit": "verify-steps/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config,
            "tree_tokens_per_s": value * w.batch * w.num_nodes,
            "cpu_baseline": {"value": value, "unit": "verify-steps/s", "cores": cores,
                             "kind": "oracle", "sample": label},
            "e2e": {"value": value, "unit": "verify-steps/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}))
        return

    import torch
    from tree_verify_b200 import binding
    from tree_verify_b200.replicas import max_over_ranks
    from tree_verify_b200.step import StepInputs, VerifyStep, shape_from_workload

    dist = None
    if world > 1:
        import torch.distributed as dist
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    binding.load()

    inp = wl.generate(w, T, seed=None)
    shape = shape_from_workload(w)
    x = StepInputs.from_numpy(inp, w.dtype, device=dev)
    step = VerifyStep(shape, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flush_read = torch.zeros(L2_FLUSH_BYTES // 2, dtype=torch.uint8, device=dev)

    def l2_flush():
        # write more than L2 holds, then read another buffer, so the step starts with an L2
        # of clean, unrelated lines (no dirty write-backs charged to the timed kernels)
        flush.zero_()
        flush_read.max()

    stream = torch.cuda.current_stream(dev)
    nb = step_bytes(w, inp["prefix_lens"])
    # kernels this library launches per step: attention (+ split merge), LM head, walk
    attn_splits = binding.workspace_bytes(shape) > 0
    launches_per_step = 3 + (1 if attn_splits else 0)

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize(dev)

    for i in range(args.warmup):
        l2_flush()
        step.run(x, T, seed=rank, offset=i)
    barrier()
    assert binding.device_error(reset=True) == 0

    # ---- timed region: K whole steps through eagle_verify_step, L2 flushed before each
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    sampler = ClockSampler(local)
    with sampler:
        barrier()
        for i in range(args.steps):
            l2_flush()
            starts[i].record(stream)
            step.run(x, T, seed=rank, offset=i)
            ends[i].record(stream)
        barrier()
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total_ms = float(np.sum(step_ms))

    # ---- the same step replayed from a CUDA graph (one fixed seed/offset per capture),
    # timed the same way: what launch gaps cost the stream-launched step
    # Capture may fail on a rank (it is reported, never required); every rank still takes
    # the same barriers, timing the stream-launched step in its place.
    graph, graph_err = None, None
    try:
        gstream = torch.cuda.Stream(dev)
        gstream.wait_stream(stream)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.stream(gstream):
            step.run(x, T, seed=rank, offset=0)  # warm the capture stream
            gstream.synchronize()
            with torch.cuda.graph(graph, stream=gstream):
                step.run(x, T, seed=rank, offset=0, stream=gstream)
        stream.wait_stream(gstream)
    except Exception as exc:
        graph, graph_err = None, f"{type(exc).__name__}: {exc}"[:200]
    torch.cuda.synchronize(dev)
    gs = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ge = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    barrier()
    for i in range(args.steps):
        l2_flush()
        gs[i].record(stream)
        if graph is not None:
            graph.replay()
        else:
            step.run(x, T, seed=rank, offset=0)
        ge[i].record(stream)
    barrier()
    graph_ms = float(np.mean([s_.elapsed_time(e_) for s_, e_ in zip(gs, ge)]))
    assert binding.device_error(reset=True) == 0
    graph_info = ({"ms_per_step": graph_ms, "value": world / (graph_ms / 1e3),
                   "note": "eagle_verify_step captured once (seed rank, offset 0) and replayed"}
                  if graph_err is None else {"unavailable": graph_err})
    del graph

    # ---- dominant kernel alone (LM head), same conditions, for the roofline
    ls = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    le = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    barrier()
    for i in range(args.steps):
        l2_flush()
        ls[i].record(stream)
        step.lm_head(x)
        le[i].record(stream)
    barrier()
    lm_ms = float(np.mean([s.elapsed_time(e) for s, e in zip(ls, le)]))

    # ---- the post-accept commit of the last step's walk (timed on its own, not part of the
    # step): the root and accepted nodes into a cache with room for them, L2 flushed first
    B, N, Hkv, D, H = w.batch, w.num_nodes, w.num_kv_heads, w.head_dim, w.hidden
    k_cache = torch.zeros((B, Hkv, w.prefix_len + N, D), dtype=x.k_prefix.dtype, device=dev)
    v_cache = torch.zeros_like(k_cache)
    new_lens = torch.empty((B,), dtype=torch.int32, device=dev)
    feat = torch.empty((B, N, H), dtype=x.hidden.dtype, device=dev)
    cs = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ce = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    barrier()
    for i in range(args.steps):
        l2_flush()
        cs[i].record(stream)
        step.commit(x, k_cache, v_cache, new_lens, feat)
        ce[i].record(stream)
    barrier()
    commit_ms = float(np.mean([s.elapsed_time(e) for s, e in zip(cs, ce)]))
    assert binding.device_error(reset=True) == 0
    alen = step.accept_len.cpu().numpy()
    commit_rows = int(np.sum(alen[alen >= 0] + 1))
    el = x.k_prefix.element_size()
    # each committed row: K and V of every kv head and one hidden row, read once, written once
    commit_bytes = commit_rows * (Hkv * D * el * 2 + H * el) * 2

    # ---- EAGLE-2 reranking of an expanded candidate tree down to this workload's N nodes
    # (timed on its own): RERANK_CANDIDATES candidates per sequence, random parents of depth
    # <= 10 and uniform confidences, L2 flushed first
    rr = np.random.default_rng(1234)
    r_par = np.stack([wl.random_parents(rr, RERANK_CANDIDATES, 10) for _ in range(B)])
    r_in = [torch.from_numpy(a).to(dev) for a in
            (r_par.astype(np.int32), rr.integers(0, w.vocab, r_par.shape).astype(np.int32),
             rr.uniform(0.0, 1.0, r_par.shape).astype(np.float32))]
    r_out = [torch.empty((B, N), dtype=torch.int32, device=dev) for _ in range(3)]
    r_masks = torch.empty((B, N), dtype=torch.int64, device=dev)
    r_n = torch.empty((B,), dtype=torch.int32, device=dev)
    rs_ = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    re_ = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    barrier()
    for i in range(args.steps):
        l2_flush()
        rs_[i].record(stream)
        binding.tree_rerank(*r_in, N, *r_out, r_masks, r_n)
        re_[i].record(stream)
    barrier()
    rerank_ms = float(np.mean([s.elapsed_time(e) for s, e in zip(rs_, re_)]))
    assert (r_n.cpu().numpy() == min(N, RERANK_CANDIDATES)).all()

    # ---- children of DRAFT_ROWS draft nodes per sequence (DRAFT_K each) from draft LM-head
    # logits over this vocabulary, at the step's temperature (timed on its own)
    d_logits = torch.from_numpy((rr.standard_normal((B, DRAFT_ROWS, w.vocab)) * 2.0)
                                .astype(np.float32)).to(dev)
    d_tok = torch.empty((B, DRAFT_ROWS, DRAFT_K), dtype=torch.int32, device=dev)
    d_conf = torch.empty((B, DRAFT_ROWS, DRAFT_K), dtype=torch.float32, device=dev)
    d_probs = torch.empty_like(d_logits)
    ds_ = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    de_ = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    barrier()
    for i in range(args.steps):
        l2_flush()
        ds_[i].record(stream)
        binding.draft_select(d_logits, T, DRAFT_K, rank, i, d_tok, d_conf, d_probs)
        de_[i].record(stream)
    barrier()
    draft_ms = float(np.mean([s.elapsed_time(e) for s, e in zip(ds_, de_)]))
    assert binding.device_error(reset=True) == 0
    draft_bytes = B * DRAFT_ROWS * w.vocab * 4 * 2  # logits read, distribution written

    # ---- the same children drawn without replacement, then the row each was drawn from
    # (timed together and the rows alone, each L2-flushed)
    d_rows = torch.empty((B, DRAFT_ROWS, DRAFT_K, w.vocab), dtype=torch.float32, device=dev)
    dd_s = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    dd_m = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    dd_e = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    barrier()
    for i in range(args.steps):
        l2_flush()
        dd_s[i].record(stream)
        binding.draft_select_distinct(d_logits, T, DRAFT_K, rank, i, d_tok, d_conf, d_probs)
        dd_m[i].record(stream)
        binding.draft_child_rows(d_probs, d_tok, d_rows)
        dd_e[i].record(stream)
    barrier()
    distinct_ms = float(np.mean([s.elapsed_time(e) for s, e in zip(dd_s, dd_m)]))
    rows_ms = float(np.mean([s.elapsed_time(e) for s, e in zip(dd_m, dd_e)]))
    assert binding.device_error(reset=True) == 0
    rows_bytes = B * DRAFT_ROWS * w.vocab * 4 * (1 + DRAFT_K)  # distribution read, k rows written

    # ---- stacked layers: the tree attention of every layer of a STACK_LAYERS-layer model,
    # each layer with its own prefix K/V cache, queries and tree K/V (seeded device normals),
    # back to back as in one verify pass; the caches (STACK_LAYERS x the step's) exceed L2
    gen = torch.Generator(device=dev)
    gen.manual_seed(4321 + rank)
    kv_dt = x.k_prefix.dtype
    def _layers(t):
        return torch.randn((STACK_LAYERS,) + tuple(t.shape), generator=gen, device=dev,
                           dtype=torch.float32).to(kv_dt)
    st_q, st_kp, st_vp, st_kt, st_vt = (_layers(t) for t in (x.q, x.k_prefix, x.v_prefix, x.k_tree, x.v_tree))
    st_out = torch.empty_like(st_q)
    def stacked_pass(st=None):
        for l in range(STACK_LAYERS):
            binding.tree_attention(step.shape, st_q[l], st_kp[l], st_vp[l], x.prefix_lens, st_kt[l], st_vt[l],
                                   x.parents, st_out[l], step.workspace, stream if st is None else st)
    stacked_pass()
    torch.cuda.synchronize(dev)
    # launched from the host the pass is bounded by Python's per-call overhead, so it is
    # captured once in a CUDA graph and replayed (the stream-launched time is reported too)
    stacked_graph = None
    try:
        sg_stream = torch.cuda.Stream(dev)
        sg_stream.wait_stream(stream)
        stacked_graph = torch.cuda.CUDAGraph()
        with torch.cuda.stream(sg_stream):
            with torch.cuda.graph(stacked_graph, stream=sg_stream):
                stacked_pass(sg_stream)
        stream.wait_stream(sg_stream)
        torch.cuda.synchronize(dev)
    except Exception:  # the stream-launched pass is still measured
        stacked_graph = None
        torch.cuda.synchronize(dev)
    def timed(fn):
        ss_ = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        se_ = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        barrier()
        for i in range(args.steps):
            l2_flush()
            ss_[i].record(stream)
            fn()
            se_[i].record(stream)
        barrier()
        return float(np.mean([s.elapsed_time(e) for s, e in zip(ss_, se_)]))
    stacked_launch_ms = timed(stacked_pass)
    # the same number of barriers on every rank, graph or not
    stacked_ms = timed(stacked_graph.replay if stacked_graph is not None else stacked_pass)
    assert binding.device_error(reset=True) == 0
    lens_h = x.prefix_lens.cpu().numpy().astype(np.int64)
    stacked_kv = int(STACK_LAYERS * lens_h.sum() * w.num_kv_heads * w.head_dim * 2 * x.k_prefix.element_size())
    stacked_graph_ok = stacked_graph is not None
    del stacked_graph
    del st_q, st_kp, st_vp, st_kt, st_vt, st_out

    # ---- end to end through the public API with host buffers: per-step tree inputs
    # (queries, tree K/V, hidden states, parents, tokens, draft distributions) copied from
    # pinned host memory, the walk's results read back; the prefix K/V cache and W stay
    # resident as model state.
    per_step = ["q", "k_tree", "v_tree", "hidden", "parents", "tokens", "draft_probs", "prefix_lens"]
    host = {n: getattr(x, n).cpu().pin_memory() for n in per_step}
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    out_host = [torch.empty_like(t, device="cpu").pin_memory()
                for t in (step.accepted_nodes, step.accept_len, step.next_token)]
    d2h = sum(t.numel() * t.element_size() for t in out_host)
    es = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ee = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    barrier()
    for i in range(args.steps):
        l2_flush()
        es[i].record(stream)
        for n in per_step:
            getattr(x, n).copy_(host[n], non_blocking=True)
        step.run(x, T, seed=rank, offset=i)
        for dst, src in zip(out_host, (step.accepted_nodes, step.accept_len, step.next_token)):
            dst.copy_(src, non_blocking=True)
        ee[i].record(stream)
    barrier()
    e2e_ms = float(np.sum([s.elapsed_time(e) for s, e in zip(es, ee)]))
    assert binding.device_error(reset=True) == 0

    # ---- max over ranks
    (total_ms, e2e_ms, lm_ms, commit_ms, rerank_ms, draft_ms, distinct_ms, rows_ms, stacked_ms,
     stacked_launch_ms) = max_over_ranks(
        [total_ms, e2e_ms, lm_ms, commit_ms, rerank_ms, draft_ms, distinct_ms, rows_ms, stacked_ms,
         stacked_launch_ms], dist, dev)
    if rank != 0:
        if dist is not None:
            dist.destroy_process_group()
        return

    value = world * args.steps / (total_ms / 1e3)
    ms_per_step = total_ms / args.steps
    peak, peak_kind = _peaks()
    lm_gbs = nb["lm_head"] / (lm_ms / 1e3) / 1e9
    step_gbs = nb["roofline_bytes"] / (ms_per_step / 1e3) / 1e9
    result = {
        "metric": METRIC, "value": value, "unit": "verify-steps/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic", "config": config,
        "tree_tokens_per_s": value * w.batch * w.num_nodes,
        "step_hbm_gbs": step_gbs,
        "step_roofline_frac": step_gbs / peak,
        "step_roofline_note": f"(KV + W bytes) / step time vs {peak_kind} HBM {peak:.0f} GB/s; "
                              f"(KV + W) = {nb['roofline_bytes']} B",
        "step_ms_p10_p50_p90": [float(np.percentile(step_ms, q)) for q in (10, 50, 90)],
        "roofline": {"kernel": "lm_head_tc_kernel", "bound": "hbm", "achieved": lm_gbs,
                     "peak": peak, "unit": "GB/s", "frac": lm_gbs / peak,
                     "traffic": _lm_head_traffic(w.name), "bytes_per_launch": nb["lm_head"],
                     "us_per_launch": lm_ms * 1e3, "peak_kind": peak_kind},
        "commit": {"kernel": "commit_kernel", "us_per_launch": commit_ms * 1e3,
                   "rows": commit_rows, "bytes_per_launch": commit_bytes,
                   "achieved_gbs": commit_bytes / (commit_ms / 1e3) / 1e9,
                   "frac": commit_bytes / (commit_ms / 1e3) / 1e9 / peak, "bound": "latency"},
        "graph": graph_info,
        "draft": {"kernel": "draft_select_kernel", "us_per_launch": draft_ms * 1e3,
                  "rows": B * DRAFT_ROWS, "k": DRAFT_K, "vocab": w.vocab,
                  "bytes_per_launch": draft_bytes,
                  "achieved_gbs": draft_bytes / (draft_ms / 1e3) / 1e9,
                  "frac": draft_bytes / (draft_ms / 1e3) / 1e9 / peak,
                  "bound": "latency" if T == 0.0 else "alu (k Philox draws per entry)"},
        "draft_distinct": {"kernel": "draft_select_kernel (one race) + draft_child_rows_kernel",
                           "select_us": distinct_ms * 1e3, "child_rows_us": rows_ms * 1e3,
                           "child_rows_bytes": rows_bytes,
                           "child_rows_frac": rows_bytes / (rows_ms / 1e3) / 1e9 / peak},
        "stacked_layers": {"workload": f"{w.name}, tree attention of {STACK_LAYERS} layers per pass, "
                                       "own caches per layer",
                           "layers": STACK_LAYERS, "us_per_pass": stacked_ms * 1e3,
                           "us_per_pass_launched": stacked_launch_ms * 1e3,
                           "timing": "CUDA graph replay of the pass" if stacked_graph_ok
                                     else "stream-launched (capture failed)",
                           "us_per_layer": stacked_ms * 1e3 / STACK_LAYERS,
                           "prefix_kv_bytes_per_pass": stacked_kv,
                           "achieved_gbs": stacked_kv / (stacked_ms / 1e3) / 1e9,
                           "frac": stacked_kv / (stacked_ms / 1e3) / 1e9 / peak},
        "rerank": {"kernel": "rerank_kernel", "us_per_launch": rerank_ms * 1e3,
                   "candidates": RERANK_CANDIDATES, "kept": N, "bound": "latency"},
        "e2e": {"value": world * args.steps / (e2e_ms / 1e3), "unit": "verify-steps/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": sampler.summary(),
    }
    if not args.no_cpu_baseline:
        # about 10-30 s of oracle work: repeat the bounded sample, report the mean
        secs, t0 = [], time.perf_counter()
        while not secs or (time.perf_counter() - t0 < 10.0 and len(secs) < 50):
            sec, label, cores = oracle_step_sample(w, inp, T)
            secs.append(sec)
        result["cpu_baseline"] = {"value": 1.0 / float(np.mean(secs)), "unit": "verify-steps/s",
                                  "cores": cores, "kind": "oracle",
                                  "sample": f"{len(secs)} x [{label}]"}
        # the oracle's commit of the same accepted nodes (it copies the whole cache first)
        import oracle
        acc_h = step.accepted_nodes.cpu().numpy()
        hid = inp["hidden"].reshape(B, N, H)
        kc, vc = k_cache.cpu(), v_cache.cpu()
        if kc.dtype == torch.bfloat16:
            kc, vc = kc.view(torch.int16).numpy().view(np.uint16), vc.view(torch.int16).numpy().view(np.uint16)
        else:
            kc, vc = kc.numpy(), vc.numpy()
        t0 = time.perf_counter()
        reps = 0
        while reps < 3 or time.perf_counter() - t0 < 1.0:
            oracle.commit(kc, vc, inp["prefix_lens"], inp["k_tree"], inp["v_tree"], hid,
                          inp["parents"], acc_h, alen)
            reps += 1
        result["commit"]["oracle_us"] = (time.perf_counter() - t0) / reps * 1e6
        t0, reps = time.perf_counter(), 0
        while reps < 3 or time.perf_counter() - t0 < 1.0:
            oracle.tree_rerank(r_par, r_in[1].cpu().numpy(), r_in[2].cpu().numpy(), N)
            reps += 1
        result["rerank"]["oracle_us"] = (time.perf_counter() - t0) / reps * 1e6
        lg_h = d_logits.cpu().numpy()
        t0, reps = time.perf_counter(), 0
        while reps < 1 or time.perf_counter() - t0 < 1.0:
            oracle.draft_select(lg_h, T, DRAFT_K, seed=rank, offset=reps, with_probs=True)
            reps += 1
        result["draft"]["oracle_us"] = (time.perf_counter() - t0) / reps * 1e6
    print(json.dumps(result))
    if dist is not None:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
