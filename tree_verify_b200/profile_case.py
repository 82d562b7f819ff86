"""Launch one stage of the verification step a few times on a workload, for an external
profiler (ncu).  It holds only that workload's inputs on the device, so a profiler that
saves and restores device memory between its passes stays quick, and it prints no timing.

    python -m tree_verify_b200.profile_case --workload vicuna7b_static --stage lm_head --launches 3
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
    ap.add_argument("--stage", default="lm_head", choices=["attention", "lm_head", "accept", "step"])
    ap.add_argument("--temperature", type=float, default=1.0)
    ap.add_argument("--launches", type=int, default=3)
    args = ap.parse_args()

    w = wl.WORKLOADS[args.workload]
    inp = wl.generate(w, args.temperature)
    x = StepInputs.from_numpy(inp, w.dtype)
    step = VerifyStep(shape_from_workload(w))
    step.lm_head(x)  # logits for the accept stage
    torch.cuda.synchronize()
    for i in range(args.launches):
        if args.stage == "attention":
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
