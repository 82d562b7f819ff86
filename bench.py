"""Benchmark of the draft-tree verification step (tree attention + LM-head logits + the
accept/resample walk) on B200, through the library's C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME --temperature T] [--extras] [--no-cpu-baseline]

By default every workload and temperature of the five synthetic verify-step shapes is
timed in one run: tiny_chain T1, vicuna7b_static T0/T1, llama70b_dyn T1, batched7b T1,
llama3_8b T0/T1.  The headline (the top-level `value`) is the largest single-GPU shape,
llama3_8b (batch 8, 32/8 heads, head_dim 128, bf16, prefix 8192, 64-node trees, hidden
4096, vocab 128256) at temperature 1; every case, the headline included, is reported under
`per_workload` with its own roofline.  `--workload/--temperature` times one case only.
N GPUs run N independent replicas ("scaling": "weak"): the value is all replicas' steps
over the slowest rank's device time.  Rank 0 prints one JSON line.

--impl reference times the CPU oracle (fp64, all host cores) on a bounded sample of the
headline workload per step; it is a reported baseline, not a tuned program.
"""
from __future__ import annotations

import argparse
import hashlib
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
UNIT = "verify-steps/s"
L2_FLUSH_BYTES = 512 << 20
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
NOMINAL_HBM_GBS = 8000.0  # the HBM roofline the verify-step target is stated against
# the headline first, on a GPU that has not yet run the others
CASES = [("llama3_8b", 1.0), ("llama3_8b", 0.0), ("batched7b", 1.0), ("llama70b_dyn", 1.0),
         ("vicuna7b_static", 1.0), ("vicuna7b_static", 0.0), ("tiny_chain", 1.0)]
HEADLINE = ("llama3_8b", 1.0)
RERANK_CANDIDATES = 256
DRAFT_ROWS, DRAFT_K = 10, 10
STACK_LAYERS = 32  # the stacked-attention workload: one verify pass through every layer


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in FALLBACK}, "measured"
    return dict(FALLBACK), "fallback"


def _kernel_profile(kernel: str, workload: str):
    """The committed ncu capture of `kernel` on `workload` (DRAM bytes per launch, tensor-pipe
    use), or None when there is none or the kernel's sources changed since it was taken."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    for rel, digest in rec["sources_sha256"].items():
        with open(os.path.join(ROOT, rel), "rb") as src:
            if hashlib.sha256(src.read()).hexdigest() != digest:
                return None
    return rec


def _kernel_traffic(kernel: str, workload: str):
    rec = _kernel_profile(kernel, workload)
    return None if rec is None else int(rec["traffic_bytes_per_launch"])


def algorithmic(w, prefix_lens):
    """What one step must move or compute: bytes per stage, and the LM head's flops."""
    el = 2 if w.dtype == wl.BF16 else 4
    B, N, Hq, Hkv, D, H, V = (w.batch, w.num_nodes, w.num_q_heads, w.num_kv_heads, w.head_dim,
                              w.hidden, w.vocab)
    M = B * N
    kv = int(np.sum(prefix_lens)) * Hkv * D * 2 * el
    wbytes = V * H * el
    attn = kv + 2 * M * Hq * D * el + 2 * M * Hkv * D * el  # prefix K/V, Q and O, tree K/V
    lm = wbytes + M * H * el + M * V * 4
    attn_flops = int(np.sum(prefix_lens)) * N * Hq * D * 4  # QK^T and PV over the prefix
    return dict(kv=kv, w=wbytes, roofline_bytes=kv + wbytes, attention=attn, lm_head=lm,
                lm_flops=2 * M * V * H, attn_flops=attn_flops)


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
        self.active = threading.Event()
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
            while not self._stop.wait(0.02):
                if self.active.is_set():
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

def oracle_sample_plan(w):
    """The bounded sample of one step the oracle times: a seeded subset of attention rows,
    a subset of LM-head rows and the walks of the first sequences (whose visited logits rows
    the oracle computes itself), sized to a few GFLOP of fp64 work; the step's time is
    extrapolated stage by stage from the fractions."""
    B, N, Hq, D, H, V = w.batch, w.num_nodes, w.num_q_heads, w.head_dim, w.hidden, w.vocab
    rows_total = B * N * Hq
    per_row = 4.0 * (w.prefix_len + N) * D
    n_attn = int(min(rows_total, max(1, 0.4e9 // per_row)))
    M = B * N
    n_lm = int(min(M, max(1, 1.5e9 // (2.0 * V * H))))
    n_seq = 1 if B > 1 else B
    rng = np.random.default_rng(99)
    flat = np.sort(rng.choice(rows_total, size=n_attn, replace=False))
    attn_rows = np.stack([flat // (N * Hq), (flat // Hq) % N, flat % Hq], 1).astype(np.int32)
    lm_rows = np.sort(rng.choice(M, size=n_lm, replace=False)).astype(np.int32)
    return dict(attn_rows=attn_rows, lm_rows=lm_rows, n_seq=n_seq,
                f_attn=n_attn / rows_total, f_lm=n_lm / M, f_walk=n_seq / B)


def oracle_step_sample(w, inp, T, plan, seed=0, offset=0):
    """Times the oracle on `plan` once.  Returns (measured seconds, extrapolated seconds of
    a whole step, the sample's outputs)."""
    import oracle
    oracle.build()
    t0 = time.perf_counter()
    att = oracle.tree_attention(inp["q"], inp["k_prefix"], inp["v_prefix"], inp["prefix_lens"],
                                inp["k_tree"], inp["v_tree"], inp["parents"], rows=plan["attn_rows"])
    t1 = time.perf_counter()
    lg = oracle.lm_head(inp["hidden"], inp["w_lm"], rows=plan["lm_rows"])
    t2 = time.perf_counter()
    s, N = plan["n_seq"], w.num_nodes
    acc = oracle.tree_accept(inp["draft_probs"][:s], inp["tokens"][:s], inp["parents"][:s], T,
                             seed=seed, offset=offset, hidden=inp["hidden"][:s * N], w_lm=inp["w_lm"])
    t3 = time.perf_counter()
    full = (t1 - t0) / plan["f_attn"] + (t2 - t1) / plan["f_lm"] + (t3 - t2) / plan["f_walk"]
    return t3 - t0, full, dict(attention=att, logits=lg, walk=acc)


def oracle_sample_label(w, plan):
    return (f"{len(plan['attn_rows'])} of {w.batch * w.num_nodes * w.num_q_heads} attention rows, "
            f"{len(plan['lm_rows'])} of {w.batch * w.num_nodes} LM-head rows and the walks of "
            f"{plan['n_seq']} of {w.batch} sequences (visited logits rows computed by the oracle); "
            "the step's time is extrapolated stage by stage from these fractions; fp64 C oracle")


def case_config(w, T, world):
    pl = w.prefix_len if w.prefix_min is None else f"U[{w.prefix_min},{w.prefix_len}]"
    return {"workload": f"{w.name}: B{w.batch} Hq{w.num_q_heads}/Hkv{w.num_kv_heads} D{w.head_dim} "
                        f"{w.dtype} prefix {pl} N{w.num_nodes} H{w.hidden} V{w.vocab} T{T:g}",
            "batch": w.batch, "tree_nodes": w.num_nodes, "prefix_len": w.prefix_len,
            "hidden": w.hidden, "vocab": w.vocab, "temperature": T,
            "l2": "flushed before every timed launch: 512 MiB write then 256 MiB read, untimed",
            "parallelism": "replicas" if world > 1 else "single"}


def reference_arm(args, world, rank):
    """The oracle on the host cores, one bounded sample of the headline workload per step."""
    if rank != 0:
        return
    name, T = (args.workload, args.temperature) if args.workload else HEADLINE
    w = wl.WORKLOADS[name]
    inp = wl.generate(w, T)
    plan = oracle_sample_plan(w)
    import oracle
    meas, full = [], []
    for i in range(args.steps + args.warmup):
        m, f, _ = oracle_step_sample(w, inp, T, plan)
        if i >= args.warmup:
            meas.append(m)
            full.append(f)
    value = 1.0 / float(np.mean(full))
    label = oracle_sample_label(w, plan)
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": float(np.mean(meas)) * 1e3,
        "ms_per_step_note": "measured time of one step's bounded sample; value is the whole-step "
                            "rate extrapolated from it",
        "extrapolated": True, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic", "config": case_config(w, T, world),
        "tree_tokens_per_s": value * w.batch * w.num_nodes,
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": label, "extrapolated": True},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}))


# ---------------------------------------------------------------- GPU arm

class Ctx:
    def __init__(self, torch, dist, dev, rank, world, steps, warmup):
        self.torch, self.dist, self.dev = torch, dist, dev
        self.rank, self.world, self.steps, self.warmup = rank, world, steps, warmup
        self.stream = torch.cuda.current_stream(dev)
        self.flush_w = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
        self.flush_r = torch.zeros(L2_FLUSH_BYTES // 2, dtype=torch.uint8, device=dev)

    def l2_flush(self):
        # write more than L2 holds, then read another buffer, so a launch starts with an L2
        # of clean, unrelated lines (no dirty write-backs charged to the timed kernels)
        self.flush_w.zero_()
        self.flush_r.max()

    def barrier(self):
        if self.dist is not None:
            self.dist.barrier()
        self.torch.cuda.synchronize(self.dev)

    def timed(self, fn, n=None):
        """Per-launch device times (ms) of n calls of fn(i), L2 flushed before each."""
        torch = self.torch
        n = self.steps if n is None else n
        s = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        e = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        self.barrier()
        for i in range(n):
            self.l2_flush()
            s[i].record(self.stream)
            fn(i)
            e[i].record(self.stream)
        self.barrier()
        return [a.elapsed_time(b) for a, b in zip(s, e)]


def run_case(ctx, w, T, peaks, sampler):
    torch = ctx.torch
    from tree_verify_b200 import binding
    from tree_verify_b200.replicas import max_over_ranks
    from tree_verify_b200.step import StepInputs, VerifyStep, shape_from_workload

    inp = wl.generate(w, T)
    shape = shape_from_workload(w)
    x = StepInputs.from_numpy(inp, w.dtype, device=ctx.dev)
    step = VerifyStep(shape, device=ctx.dev)
    for i in range(ctx.warmup):
        ctx.l2_flush()
        step.run(x, T, seed=ctx.rank, offset=i)
    ctx.barrier()
    assert binding.device_error(reset=True) == 0
    sampler.active.set()
    step_ms = ctx.timed(lambda i: step.run(x, T, seed=ctx.rank, offset=i))
    lm_ms = ctx.timed(lambda i: step.lm_head(x))
    attn_ms = ctx.timed(lambda i: step.attention(x))
    step.lm_head(x)
    acc_ms = ctx.timed(lambda i: step.accept(x, T, seed=ctx.rank, offset=i))
    sampler.active.clear()
    assert binding.device_error(reset=True) == 0
    # tokens per target forward (accepted nodes + the extra token) over seeded walks
    taus = []
    for i in range(16):
        step.accept(x, T, seed=ctx.rank, offset=10_000 + i)
        a = step.accept_len.cpu().numpy()
        taus.append(a[a >= 0] + 1)
    tau = float(np.mean(np.concatenate(taus)))
    total_ms, lm_t, attn_t, acc_t = max_over_ranks(
        [float(np.sum(step_ms)), float(np.mean(lm_ms)), float(np.mean(attn_ms)), float(np.mean(acc_ms))],
        ctx.dist, ctx.dev)
    n = ctx.steps
    ms = total_ms / n
    value = ctx.world * n / (total_ms / 1e3)
    alg = algorithmic(w, inp["prefix_lens"])
    # the step repeats back to back for seconds, so its tensor-bound LM head is held to the
    # sustained GEMM figure (the burst one is reported beside it)
    hbm, tflops, tflops_burst = peaks["hbm_gbs"], peaks["bf16_tflops_sustained"], peaks["bf16_tflops"]
    step_gbs = alg["roofline_bytes"] / (ms / 1e3) / 1e9
    t_hbm = alg["roofline_bytes"] / (hbm * 1e9)
    t_tensor = alg["lm_flops"] / (tflops * 1e12) if w.dtype == wl.BF16 else 0.0
    lm_gbs = alg["lm_head"] / (lm_t / 1e3) / 1e9
    lm_tfs = alg["lm_flops"] / (lm_t / 1e3) / 1e12
    lm_tensor_bound = w.dtype == wl.BF16 and alg["lm_flops"] / (tflops * 1e12) > alg["lm_head"] / (hbm * 1e9)
    attn_gbs = alg["attention"] / (attn_t / 1e3) / 1e9
    lm_roof = ({"kernel": "lm_head_tc_persist_kernel" if w.batch * w.num_nodes > 256 else "lm_head_tc_kernel",
                "bound": "tensor", "achieved": lm_tfs, "peak": tflops, "peak_figure": "sustained",
                "unit": "TFLOP/s", "frac": lm_tfs / tflops, "frac_of_burst": lm_tfs / tflops_burst,
                "flops_per_launch": alg["lm_flops"]}
               if lm_tensor_bound else
               {"kernel": "lm_head_tc_kernel" if w.dtype == wl.BF16 else "lm_head_f32_kernel",
                "bound": "hbm", "achieved": lm_gbs, "peak": hbm, "unit": "GB/s", "frac": lm_gbs / hbm,
                "bytes_per_launch": alg["lm_head"]})
    lm_roof["us_per_launch"] = lm_t * 1e3
    lm_prof = _kernel_profile("lm_head_tc", w.name) if w.dtype == wl.BF16 else None
    lm_roof["traffic"] = None if lm_prof is None else int(lm_prof["traffic_bytes_per_launch"])
    if lm_prof is not None and "tensor_pipe_active_pct" in lm_prof:
        lm_roof["tensor_pipe_active_pct"] = lm_prof["tensor_pipe_active_pct"]
    attn_roof = {"kernel": "tree_attn_tc_kernel + tree_attn_combine_kernel" if w.dtype == wl.BF16
                 else "tree_attn_f32_kernel", "bound": "hbm", "achieved": attn_gbs, "peak": hbm,
                 "unit": "GB/s", "frac": attn_gbs / hbm, "bytes_per_launch": alg["attention"],
                 "us_per_launch": attn_t * 1e3,
                 "traffic": _kernel_traffic("tree_attn_tc", w.name) if w.dtype == wl.BF16 else None}
    stages = {"lm_head": lm_t * 1e3, "attention": attn_t * 1e3, "walk": acc_t * 1e3}
    dominant = max(("lm_head", "attention"), key=lambda k: stages[k])
    launches = 3 + (1 if binding.workspace_bytes(shape) > 0 else 0)
    rec = {
        "workload": w.name, "temperature": T, "config": case_config(w, T, ctx.world)["workload"],
        "ms_per_step": ms, "steps_per_s": value, "tree_tokens_per_s": value * w.batch * w.num_nodes,
        "step_ms_p10_p50_p90": [float(np.percentile(step_ms, q)) for q in (10, 50, 90)],
        "kv_plus_w_bytes": alg["roofline_bytes"],
        "step_hbm_gbs": step_gbs,
        "step_frac_of_measured_hbm": step_gbs / hbm,
        "step_frac_of_8tbs": step_gbs / NOMINAL_HBM_GBS,
        "binding_bound": "tensor" if t_tensor > t_hbm else "hbm",
        "binding_roofline_us": max(t_hbm, t_tensor) * 1e6,
        "step_frac_of_binding": max(t_hbm, t_tensor) / (ms / 1e3),
        "stages_us": stages, "dominant_kernel": dominant,
        "lm_head": lm_roof, "attention": attn_roof,
        "tau": tau, "launches_per_step": launches,
    }
    rec["roofline"] = dict(lm_roof if dominant == "lm_head" else attn_roof)
    return rec, (inp, x, step, shape)


def e2e_case(ctx, w, T, state):
    """The headline step end to end through the public API with host buffers: each step's
    tree inputs (queries, tree K/V, hidden states, parents, tokens, draft distributions,
    prefix lengths) packed in one pinned host buffer and copied with one H2D copy into one
    of two device staging buffers on a copy stream, so step i+1's copy overlaps step i; the
    walk's results read back to pinned memory after every step.  The prefix K/V cache and
    W stay resident as model state."""
    torch = ctx.torch
    from tree_verify_b200.replicas import max_over_ranks
    inp, x, step, shape = state
    names = ["q", "k_tree", "v_tree", "hidden", "parents", "tokens", "draft_probs", "prefix_lens"]
    segs, off = [], 0
    for n in names:
        t = getattr(x, n)
        nb = t.numel() * t.element_size()
        segs.append((n, off, nb, t))
        off += (nb + 255) // 256 * 256
    host = torch.empty(off, dtype=torch.uint8).pin_memory()
    for n, o, nb, t in segs:
        host[o:o + nb].copy_(t.reshape(-1).view(torch.uint8).cpu())
    stage = [torch.empty(off, dtype=torch.uint8, device=ctx.dev) for _ in range(2)]

    def views(buf):
        from tree_verify_b200.step import StepInputs
        kw = {n: getattr(x, n) for n in ("k_prefix", "v_prefix", "w_lm")}
        for n, o, nb, t in segs:
            kw[n] = buf[o:o + nb].view(t.dtype).view(t.shape)
        return StepInputs(**kw)

    xs = [views(b) for b in stage]
    res = (step.accepted_nodes, step.accept_len, step.next_token)
    out_host = [torch.empty_like(t, device="cpu").pin_memory() for t in res]
    d2h = sum(t.numel() * t.element_size() for t in out_host)
    copy = torch.cuda.Stream(ctx.dev)
    n = ctx.steps
    copied = [torch.cuda.Event() for _ in range(2)]
    used = [torch.cuda.Event() for _ in range(2)]
    for e in used:
        e.record(ctx.stream)

    def issue_copy(i):
        k = i % 2
        copy.wait_event(used[k])
        with torch.cuda.stream(copy):
            stage[k].copy_(host, non_blocking=True)
        copied[k].record(copy)

    # copy-only rate (one H2D per step), for the record
    c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ctx.barrier()
    c0.record(copy)
    for i in range(n):
        with torch.cuda.stream(copy):
            stage[i % 2].copy_(host, non_blocking=True)
    c1.record(copy)
    ctx.barrier()
    copy_ms = c0.elapsed_time(c1) / n
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ctx.barrier()
    t0.record(ctx.stream)
    copy.wait_stream(ctx.stream)
    issue_copy(0)
    for i in range(n):
        if i + 1 < n:
            issue_copy(i + 1)
        ctx.stream.wait_event(copied[i % 2])
        step.run(xs[i % 2], T, seed=ctx.rank, offset=i)
        used[i % 2].record(ctx.stream)
        for dst, src in zip(out_host, res):
            dst.copy_(src, non_blocking=True)
    t1.record(ctx.stream)
    ctx.barrier()
    e2e_ms, copy_ms = max_over_ranks([t0.elapsed_time(t1), copy_ms], ctx.dist, ctx.dev)
    return {"value": ctx.world * n / (e2e_ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": off,
            "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms / n, "h2d_copy_ms_per_step": copy_ms,
            "h2d_gbs": off / (copy_ms / 1e3) / 1e9, "copies_per_step": 1,
            "note": "one pinned H2D copy per step into one of two staging buffers (copy of step i+1 "
                    "overlaps step i); results read back to pinned memory every step"}


def graph_case(ctx, T, state):
    """The headline step captured once in a CUDA graph and replayed (fixed seed/offset)."""
    torch = ctx.torch
    from tree_verify_b200.replicas import max_over_ranks
    inp, x, step, shape = state
    graph, err = None, None
    try:
        gstream = torch.cuda.Stream(ctx.dev)
        gstream.wait_stream(ctx.stream)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.stream(gstream):
            step.run(x, T, seed=ctx.rank, offset=0)
            gstream.synchronize()
            with torch.cuda.graph(graph, stream=gstream):
                step.run(x, T, seed=ctx.rank, offset=0, stream=gstream)
        ctx.stream.wait_stream(gstream)
    except Exception as exc:  # reported, never required; every rank still takes the barriers
        graph, err = None, f"{type(exc).__name__}: {exc}"[:200]
    torch.cuda.synchronize(ctx.dev)
    ms = ctx.timed(lambda i: graph.replay() if graph is not None else step.run(x, T, seed=ctx.rank, offset=0))
    (g_ms,) = max_over_ranks([float(np.mean(ms))], ctx.dist, ctx.dev)
    del graph
    if err is not None:
        return {"unavailable": err}
    return {"ms_per_step": g_ms, "value": ctx.world / (g_ms / 1e3),
            "note": "eagle_verify_step captured once (seed rank, offset 0) and replayed"}


def extras_case(ctx, w, T, state, peak_hbm):
    """The kernels around the step, each timed on its own (L2 flushed): post-accept commit,
    EAGLE-2 reranking, draft children (with and without replacement) and the tree attention
    of a 32-layer verify pass."""
    torch = ctx.torch
    from tree_verify_b200 import binding
    from tree_verify_b200.replicas import max_over_ranks
    inp, x, step, shape = state
    dev = ctx.dev
    B, N, Hkv, D, H = w.batch, w.num_nodes, w.num_kv_heads, w.head_dim, w.hidden
    step.run(x, T, seed=ctx.rank, offset=0)
    k_cache = torch.zeros((B, Hkv, w.prefix_len + N, D), dtype=x.k_prefix.dtype, device=dev)
    v_cache = torch.zeros_like(k_cache)
    new_lens = torch.empty((B,), dtype=torch.int32, device=dev)
    feat = torch.empty((B, N, H), dtype=x.hidden.dtype, device=dev)
    commit_ms = float(np.mean(ctx.timed(lambda i: step.commit(x, k_cache, v_cache, new_lens, feat))))
    alen = step.accept_len.cpu().numpy()
    commit_rows = int(np.sum(alen[alen >= 0] + 1))
    el = x.k_prefix.element_size()
    commit_bytes = commit_rows * (Hkv * D * el * 2 + H * el) * 2
    rr = np.random.default_rng(1234)
    r_par = np.stack([wl.random_parents(rr, RERANK_CANDIDATES, 10) for _ in range(B)])
    r_in = [torch.from_numpy(a).to(dev) for a in
            (r_par.astype(np.int32), rr.integers(0, w.vocab, r_par.shape).astype(np.int32),
             rr.uniform(0.0, 1.0, r_par.shape).astype(np.float32))]
    r_out = [torch.empty((B, N), dtype=torch.int32, device=dev) for _ in range(3)]
    r_masks = torch.empty((B, N), dtype=torch.int64, device=dev)
    r_n = torch.empty((B,), dtype=torch.int32, device=dev)
    rerank_ms = float(np.mean(ctx.timed(lambda i: binding.tree_rerank(*r_in, N, *r_out, r_masks, r_n))))
    d_logits = torch.from_numpy((rr.standard_normal((B, DRAFT_ROWS, w.vocab)) * 2.0)
                                .astype(np.float32)).to(dev)
    d_tok = torch.empty((B, DRAFT_ROWS, DRAFT_K), dtype=torch.int32, device=dev)
    d_conf = torch.empty((B, DRAFT_ROWS, DRAFT_K), dtype=torch.float32, device=dev)
    d_probs = torch.empty_like(d_logits)
    draft_ms = float(np.mean(ctx.timed(
        lambda i: binding.draft_select(d_logits, T, DRAFT_K, ctx.rank, i, d_tok, d_conf, d_probs))))
    distinct_ms = float(np.mean(ctx.timed(
        lambda i: binding.draft_select_distinct(d_logits, T, DRAFT_K, ctx.rank, i, d_tok, d_conf, d_probs))))
    d_rows = torch.empty((B, DRAFT_ROWS, DRAFT_K, w.vocab), dtype=torch.float32, device=dev)
    rows_ms = float(np.mean(ctx.timed(lambda i: binding.draft_child_rows(d_probs, d_tok, d_rows))))
    rows_bytes = B * DRAFT_ROWS * w.vocab * 4 * (1 + DRAFT_K)
    gen = torch.Generator(device=dev)
    gen.manual_seed(4321 + ctx.rank)
    kv_dt = x.k_prefix.dtype

    def _layers(t):
        return torch.randn((STACK_LAYERS,) + tuple(t.shape), generator=gen, device=dev,
                           dtype=torch.float32).to(kv_dt)
    st_q, st_kp, st_vp, st_kt, st_vt = (_layers(t) for t in (x.q, x.k_prefix, x.v_prefix, x.k_tree, x.v_tree))
    st_out = torch.empty_like(st_q)

    def stacked_pass(st=None):
        for l in range(STACK_LAYERS):
            binding.tree_attention(step.shape, st_q[l], st_kp[l], st_vp[l], x.prefix_lens, st_kt[l], st_vt[l],
                                   x.parents, st_out[l], step.workspace, ctx.stream if st is None else st)
    stacked_pass()
    torch.cuda.synchronize(dev)
    graph = None
    try:
        sg = torch.cuda.Stream(dev)
        sg.wait_stream(ctx.stream)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.stream(sg):
            with torch.cuda.graph(graph, stream=sg):
                stacked_pass(sg)
        ctx.stream.wait_stream(sg)
    except Exception:
        graph = None
    torch.cuda.synchronize(dev)
    stacked_ms = float(np.mean(ctx.timed(lambda i: graph.replay() if graph is not None else stacked_pass(),
                                         n=min(ctx.steps, 50))))
    assert binding.device_error(reset=True) == 0
    lens_h = x.prefix_lens.cpu().numpy().astype(np.int64)
    stacked_kv = int(STACK_LAYERS * lens_h.sum() * w.num_kv_heads * w.head_dim * 2 * el)
    del graph, st_q, st_kp, st_vp, st_kt, st_vt, st_out
    (commit_ms, rerank_ms, draft_ms, distinct_ms, rows_ms, stacked_ms) = max_over_ranks(
        [commit_ms, rerank_ms, draft_ms, distinct_ms, rows_ms, stacked_ms], ctx.dist, dev)
    return {
        "workload": w.name,
        "commit": {"kernel": "commit_kernel", "us_per_launch": commit_ms * 1e3, "rows": commit_rows,
                   "bytes_per_launch": commit_bytes, "bound": "latency"},
        "rerank": {"kernel": "rerank_kernel", "us_per_launch": rerank_ms * 1e3,
                   "candidates": RERANK_CANDIDATES, "kept": N, "bound": "latency"},
        "draft": {"kernel": "draft_select_kernel", "us_per_launch": draft_ms * 1e3, "rows": B * DRAFT_ROWS,
                  "k": DRAFT_K, "vocab": w.vocab},
        "draft_distinct": {"select_us": distinct_ms * 1e3, "child_rows_us": rows_ms * 1e3,
                           "child_rows_bytes": rows_bytes,
                           "child_rows_frac": rows_bytes / (rows_ms / 1e3) / 1e9 / peak_hbm},
        "stacked_layers": {"layers": STACK_LAYERS, "us_per_pass": stacked_ms * 1e3,
                           "prefix_kv_bytes_per_pass": stacked_kv,
                           "frac": stacked_kv / (stacked_ms / 1e3) / 1e9 / peak_hbm},
    }


def cpu_baseline(w, T, state, rank):
    """The oracle, as it stands, on the host cores over bounded samples of the headline
    workload (about 10 s), plus the parity of the GPU step on the same sample: attention and
    logits row errors and the walk decisions compared under the margin rule."""
    import oracle
    inp, x, step, shape = state
    plan = oracle_sample_plan(w)
    meas, full = [], []
    t_start = time.perf_counter()
    outs = None
    while not full or (time.perf_counter() - t_start < 10.0 and len(full) < 50):
        m, f, o = oracle_step_sample(w, inp, T, plan)
        outs = outs or o
        meas.append(m)
        full.append(f)
    # parity on the sample: the GPU step at seed 0, offset 0 (the oracle sample's)
    step.run(x, T, seed=0, offset=0)
    out = step.out.float().cpu().numpy()
    lg = step.logits.cpu().numpy()
    r = plan["attn_rows"]
    a_err = np.abs(out[r[:, 0], r[:, 1], r[:, 2]] - outs["attention"]).max(-1) / \
        np.abs(outs["attention"]).max(-1)
    l_err = np.abs(lg[plan["lm_rows"]] - outs["logits"]).max(-1) / np.abs(outs["logits"]).max(-1)
    s = plan["n_seq"]
    g_len = step.accept_len.cpu().numpy()[:s]
    ref = outs["walk"]
    first = ref["first_near"]
    decided = np.where(first < 0, ref["decisions"], first)
    same_len = [int(g_len[b]) == int(ref["accept_len"][b]) for b in range(s) if first[b] < 0]
    return {"value": 1.0 / float(np.mean(full)), "unit": UNIT, "cores": oracle.num_threads(),
            "kind": "oracle", "extrapolated": True,
            "sample": f"{len(full)} x [{oracle_sample_label(w, plan)}]",
            "measured_s_per_sample": float(np.mean(meas)),
            "parity": {"attention_max_row_err": float(a_err.max()), "logits_max_row_err": float(l_err.max()),
                       "walk_decisions": int(np.sum(ref["decisions"])),
                       "walk_decisions_compared": int(np.sum(decided)),
                       "walk_decisions_excluded_by_margin": int(np.sum(ref["decisions"] - decided)),
                       "walk_lengths_equal": bool(all(same_len)),
                       "sequences": s}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=None, choices=sorted(wl.WORKLOADS))
    ap.add_argument("--temperature", type=float, default=None)
    ap.add_argument("--extras", action="store_true",
                    help="also time commit, rerank, draft children and the stacked-layer pass")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.workload and args.temperature is None:
        args.temperature = wl.WORKLOADS[args.workload].temperatures[-1]

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        reference_arm(args, world, rank)
        return

    import torch
    from tree_verify_b200 import binding

    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    binding.load()
    peaks, peak_kind = _peaks()
    ctx = Ctx(torch, dist, dev, rank, world, args.steps, args.warmup)
    cases = [(args.workload, args.temperature)] if args.workload else CASES
    head = cases[0] if args.workload else HEADLINE
    per, head_rec, head_state, extras, graph_info, e2e = [], None, None, None, None, None
    sampler = ClockSampler(local)
    with sampler:
        for name, T in cases:
            w = wl.WORKLOADS[name]
            rec, state = run_case(ctx, w, T, peaks, sampler)
            per.append(rec)
            if (name, T) == head:
                head_rec = rec
                sampler.active.set()
                graph_info = graph_case(ctx, T, state)
                e2e = e2e_case(ctx, w, T, state)
                sampler.active.clear()
                if args.extras:
                    extras = extras_case(ctx, w, T, state, peaks["hbm_gbs"])
                head_state = state
            else:
                del state
            torch.cuda.empty_cache()
    assert binding.device_error(reset=True) == 0
    if rank != 0:
        if dist is not None:
            dist.destroy_process_group()
        return

    w = wl.WORKLOADS[head[0]]
    T = head[1]
    r = head_rec
    result = {
        "metric": METRIC, "value": r["steps_per_s"], "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": r["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic (seeded normals of the workload recipe; no model weights or datasets)",
        "config": case_config(w, T, world),
        "tree_tokens_per_s": r["tree_tokens_per_s"],
        "step_hbm_gbs": r["step_hbm_gbs"],
        "step_roofline_frac": r["step_frac_of_measured_hbm"],
        "step_roofline_frac_8tbs": r["step_frac_of_8tbs"],
        "step_binding_bound": r["binding_bound"],
        "step_frac_of_binding_roofline": r["step_frac_of_binding"],
        "step_roofline_note": f"(KV + W bytes) / step time against the {peak_kind} HBM "
                              f"{peaks['hbm_gbs']:.0f} GB/s (step_roofline_frac) and against 8 TB/s "
                              f"(step_roofline_frac_8tbs, the stated target); binding roofline = "
                              f"max((KV + W) / HBM, LM-head flops / sustained bf16 "
                              f"{peaks['bf16_tflops_sustained']:.0f} TFLOP/s)",
        "step_ms_p10_p50_p90": r["step_ms_p10_p50_p90"],
        "stages_us": r["stages_us"],
        "tau": r["tau"],
        "roofline": dict(r["roofline"], peak_kind=peak_kind),
        "per_workload": per,
        "graph": graph_info,
        "e2e": e2e,
        "gpu_launches": r["launches_per_step"] * args.steps,
        "clocks": sampler.summary(),
    }
    if extras is not None:
        result["extras"] = extras
    if not args.no_cpu_baseline and world == 1:
        result["cpu_baseline"] = cpu_baseline(w, T, head_state, rank)
    print(json.dumps(result))
    if dist is not None:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
