"""Launch one stage of the verification step a few times on a workload, for an external
profiler (ncu).  It holds only that workload's inputs on the device, so a profiler that
saves and restores device memory between its passes stays quick, and it prints no timing.

    python -m tree_verify_b200.profile_case --workload vicuna7b_static --stage lm_head --launches 3

Stages: attention, lm_head, accept, step (eagle_verify_step), and the kernels around the step:
commit (the root and accepted nodes of one walk into a cache with room for them), rerank
(256 random candidates down to the workload's N nodes) and draft (the children of 10 draft
nodes per sequence, k = 10, from logits over the workload's vocabulary).
"""
from __future__ import annotations

import argparse
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def main() -> None:
    import torch

    import workloads as wl
    from tree_verify_b200 import binding
    from tree_verify_b200.step import StepInputs, VerifyStep, shape_from_workload

    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="vicuna7b_static", choices=sorted(wl.WORKLOADS))
    ap.add_argument("--stage", default="lm_head",
                    choices=["attention", "lm_head", "accept", "step", "commit", "rerank", "draft"])
    ap.add_argument("--temperature", type=float, default=1.0)
    ap.add_argument("--launches", type=int, default=3)
    args = ap.parse_args()

    import numpy as np

    w = wl.WORKLOADS[args.workload]
    dev = torch.device("cuda")
    B, N, T = w.batch, w.num_nodes, args.temperature
    if args.stage == "draft":
        rng = np.random.default_rng(1234)
        d_logits = torch.from_numpy((rng.standard_normal((B, 10, w.vocab)) * 2.0).astype(np.float32)).to(dev)
        d_tok = torch.empty((B, 10, 10), dtype=torch.int32, device=dev)
        d_conf = torch.empty((B, 10, 10), dtype=torch.float32, device=dev)
        d_probs = torch.empty_like(d_logits)
        for i in range(args.launches):
            binding.draft_select(d_logits, T, 10, 0, i, d_tok, d_conf, d_probs)
            torch.cuda.synchronize()
        assert binding.device_error(reset=True) == 0
        print(f"draft x{args.launches} on {w.name}: ok")
        return
    if args.stage == "rerank":
        rng = np.random.default_rng(1234)
        par = np.stack([wl.random_parents(rng, 256, 10) for _ in range(B)]).astype(np.int32)
        r_in = [torch.from_numpy(a).to(dev) for a in
                (par, rng.integers(0, w.vocab, par.shape).astype(np.int32),
                 rng.uniform(0.0, 1.0, par.shape).astype(np.float32))]
        r_out = [torch.empty((B, N), dtype=torch.int32, device=dev) for _ in range(3)]
        r_masks = torch.empty((B, N), dtype=torch.int64, device=dev)
        r_n = torch.empty((B,), dtype=torch.int32, device=dev)
        for i in range(args.launches):
            binding.tree_rerank(*r_in, N, *r_out, r_masks, r_n)
            torch.cuda.synchronize()
        assert binding.device_error(reset=True) == 0
        print(f"rerank x{args.launches} on {w.name}: ok")
        return

    inp = wl.generate(w, args.temperature)
    x = StepInputs.from_numpy(inp, w.dtype)
    step = VerifyStep(shape_from_workload(w))
    step.lm_head(x)  # logits for the accept stage
    torch.cuda.synchronize()
    if args.stage == "commit":
        step.run(x, T, 0, 0)  # the walk whose accepted nodes are committed
        k_cache = torch.zeros((B, w.num_kv_heads, w.prefix_len + N, w.head_dim), dtype=x.k_prefix.dtype,
                              device=dev)
        v_cache = torch.zeros_like(k_cache)
        new_lens = torch.empty((B,), dtype=torch.int32, device=dev)
        feat = torch.empty((B, N, w.hidden), dtype=x.hidden.dtype, device=dev)
        torch.cuda.synchronize()
    for i in range(args.launches):
        if args.stage == "commit":
            step.commit(x, k_cache, v_cache, new_lens, feat)
        elif args.stage == "attention":
            step.attention(x)
        elif args.stage == "lm_head":
            step.lm_head(x)
        elif args.stage == "accept":
            step.accept(x, args.temperature, 0, i)
        else:
            step.run(x, args.temperature, 0, i)
        torch.cuda.synchronize()
    assert binding.device_error(reset=True) == 0
    print(f"{args.stage} x{args.launches} on {w.name}: ok")


if __name__ == "__main__":
    main()
