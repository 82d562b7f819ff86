"""Full-size verification steps (the five workload shapes) through eagle_verify_step, in
the launch configuration the benchmark times, checked against the oracle on sampled
outputs: attention rows and logits rows it recomputes one by one, and the whole accept
walk, whose visited logits rows the oracle computes itself in fp64 from hidden and W."""
import numpy as np
import pytest
import torch

import workloads as wl
from tests.parity import MARGIN, TOL, compare_accept, row_rel_err

pytestmark = pytest.mark.gpu

CASES = [("tiny_chain", 1.0), ("vicuna7b_static", 0.0), ("vicuna7b_static", 1.0),
         ("llama70b_dyn", 1.0), ("batched7b", 1.0), ("llama3_8b", 0.0), ("llama3_8b", 1.0)]


@pytest.mark.parametrize("name,T", CASES, ids=[f"{n}-T{t:g}" for n, t in CASES])
def test_verify_step_full_size(cuda_lib, orc, name, T):
    from tree_verify_b200.step import StepInputs, VerifyStep, shape_from_workload
    w = wl.WORKLOADS[name]
    inp = wl.generate(w, T)
    shape = shape_from_workload(w)
    x = StepInputs.from_numpy(inp, w.dtype)
    step = VerifyStep(shape)
    seed, offset = 0, 0
    step.run(x, T, seed, offset)
    torch.cuda.synchronize()
    assert cuda_lib.device_error(reset=True) == 0
    B, N = w.batch, w.num_nodes
    rng = np.random.default_rng(5)

    # attention: sampled rows (all rows for the tiny case)
    out = step.out.float().cpu().numpy()
    if B * N * w.num_q_heads <= 4096:
        ref = orc.tree_attention(inp["q"], inp["k_prefix"], inp["v_prefix"], inp["prefix_lens"],
                                 inp["k_tree"], inp["v_tree"], inp["parents"])
        err = row_rel_err(out.reshape(-1, w.head_dim), ref.reshape(-1, w.head_dim))
    else:
        rows = np.stack([rng.integers(0, B, 256), rng.integers(0, N, 256),
                         rng.integers(0, w.num_q_heads, 256)], 1).astype(np.int32)
        rows[0] = [B - 1, N - 1, w.num_q_heads - 1]
        ref = orc.tree_attention(inp["q"], inp["k_prefix"], inp["v_prefix"], inp["prefix_lens"],
                                 inp["k_tree"], inp["v_tree"], inp["parents"], rows=rows)
        err = row_rel_err(out[rows[:, 0], rows[:, 1], rows[:, 2]], ref)
    assert err.max() <= TOL[w.dtype], f"attention max row error {err.max():.3e}"

    # logits: sampled rows
    logits = step.logits.cpu().numpy()
    lrows = np.unique(np.array([0, B * N - 1, int(rng.integers(0, B * N))], np.int32))
    lref = orc.lm_head(inp["hidden"], inp["w_lm"], rows=lrows)
    lerr = row_rel_err(logits[lrows], lref)
    assert lerr.max() <= TOL[w.dtype], f"logits max row error {lerr.max():.3e}"

    # the walk, against the oracle walking on its own fp64 logits
    ref_acc = orc.tree_accept(inp["draft_probs"], inp["tokens"], inp["parents"], T, seed=seed,
                              offset=offset, hidden=inp["hidden"], w_lm=inp["w_lm"], margin=MARGIN)
    got = dict(accepted_nodes=step.accepted_nodes.cpu().numpy(),
               accept_len=step.accept_len.cpu().numpy(), next_token=step.next_token.cpu().numpy())
    st = compare_accept(got, ref_acc, inp["parents"])
    # every decision before a sequence's first near one was compared bit for bit; a sequence
    # whose very first decision is near is the only one allowed to compare none
    for b in range(B):
        if ref_acc["first_near"][b] != 0:
            assert st.per_seq[b] >= 1, (b, st)
    assert st.compared >= 0.75 * st.decisions, st


STEP_CASES = {
    # one sequence, the bench workload's tree (45 nodes) on a shorter prefix
    "vicuna": ("vicuna7b_static", dict(prefix_len=700, vocab=5000, hidden=1024)),
    # two sequences of ragged length, a random tree of 20 nodes
    "ragged": ("batched7b", dict(batch=2, tree_arg=(20, 6), prefix_len=900, prefix_min=1, vocab=5000,
                                 hidden=1024)),
    # head dim 64, four query heads per kv head
    "d64": ("batched7b", dict(batch=2, num_q_heads=8, num_kv_heads=2, head_dim=64, tree_arg=(20, 6),
                              prefix_len=500, prefix_min=40, vocab=3000, hidden=512)),
}


@pytest.mark.parametrize("case", sorted(STEP_CASES))
@pytest.mark.parametrize("T", [0.0, 1.0])
def test_verify_step_two_stream_schedule(cuda_lib, orc, case, T):
    """eagle_verify_step's two-stream schedule (attention and its merge on the library's
    side stream, beside the walk) gives the same logits and walk bits as the stage calls in
    sequence, and attention that matches the oracle and the stand-alone call."""
    from tree_verify_b200.step import StepInputs, VerifyStep, shape_from_workload
    base, kw = STEP_CASES[case]
    w = wl.scaled(wl.WORKLOADS[base], **kw)
    inp = wl.generate(w, T)
    shape = shape_from_workload(w)
    x = StepInputs.from_numpy(inp, w.dtype)
    a, b = VerifyStep(shape), VerifyStep(shape)
    a.run(x, T, 3, 4)
    b.attention(x)
    b.lm_head(x)
    b.accept(x, T, 3, 4)
    torch.cuda.synchronize()
    assert cuda_lib.device_error(reset=True) == 0
    for name in ("logits", "accepted_nodes", "accept_len", "next_token"):
        assert torch.equal(getattr(a, name), getattr(b, name)), name
    ref = orc.tree_attention(inp["q"], inp["k_prefix"], inp["v_prefix"], inp["prefix_lens"],
                             inp["k_tree"], inp["v_tree"], inp["parents"])
    got = a.out.float().cpu().numpy().reshape(-1, w.head_dim)
    err = row_rel_err(got, ref.reshape(-1, w.head_dim))
    assert err.max() <= TOL[w.dtype], f"attention max row error {err.max():.3e}"
    alone = b.out.float().cpu().numpy().reshape(-1, w.head_dim)
    assert row_rel_err(got, alone).max() <= TOL[w.dtype]


def test_verify_step_stages_equal_fused_call(cuda_lib):
    """The three stage entry points in sequence give the same bits as eagle_verify_step
    (three sequences of ragged length)."""
    from tree_verify_b200.step import StepInputs, VerifyStep, shape_from_workload
    w = wl.scaled(wl.WORKLOADS["batched7b"], batch=3, prefix_len=700, prefix_min=100, vocab=5000,
                  hidden=1024)
    inp = wl.generate(w, 1.0)
    x = StepInputs.from_numpy(inp, w.dtype)
    a, b = VerifyStep(shape_from_workload(w)), VerifyStep(shape_from_workload(w))
    a.run(x, 1.0, 11, 12)
    b.attention(x)
    b.lm_head(x)
    b.accept(x, 1.0, 11, 12)
    torch.cuda.synchronize()
    assert cuda_lib.device_error(reset=True) == 0
    for name in ("out", "logits", "accepted_nodes", "accept_len", "next_token"):
        assert torch.equal(getattr(a, name), getattr(b, name)), name


@pytest.mark.parametrize("T", [0.0, 1.0])
def test_verify_step_reads_inputs_written_just_before_on_its_stream(cuda_lib, orc, T):
    """Inputs written on the caller's stream right before eagle_verify_step, behind a kernel
    that spins for about 10 ms, are the ones the step reads, the side stream's attention
    included (it starts after the LM head, so after all earlier work on the caller's
    stream).  The step's buffers hold NaN until the copies land."""
    from tree_verify_b200.step import StepInputs, VerifyStep, shape_from_workload
    base, kw = STEP_CASES["vicuna"]
    w = wl.scaled(wl.WORKLOADS[base], **kw)
    inp = wl.generate(w, T)
    shape = shape_from_workload(w)
    src = StepInputs.from_numpy(inp, w.dtype)
    x = StepInputs.from_numpy(inp, w.dtype)
    names = ("q", "k_prefix", "v_prefix", "k_tree", "v_tree", "hidden", "w_lm", "draft_probs")
    for n in names:
        getattr(x, n).fill_(float("nan"))
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    a, b = VerifyStep(shape), VerifyStep(shape)
    with torch.cuda.stream(s):
        torch.cuda._sleep(20_000_000)
        for n in names:
            getattr(x, n).copy_(getattr(src, n))
    a.run(x, T, 3, 4, stream=s)
    torch.cuda.synchronize()
    b.attention(src)
    b.lm_head(src)
    b.accept(src, T, 3, 4)
    torch.cuda.synchronize()
    assert cuda_lib.device_error(reset=True) == 0
    for name in ("logits", "accepted_nodes", "accept_len", "next_token"):
        assert torch.equal(getattr(a, name), getattr(b, name)), name
    ref = orc.tree_attention(inp["q"], inp["k_prefix"], inp["v_prefix"], inp["prefix_lens"],
                             inp["k_tree"], inp["v_tree"], inp["parents"])
    got = a.out.float().cpu().numpy().reshape(-1, w.head_dim)
    err = row_rel_err(got, ref.reshape(-1, w.head_dim))
    assert err.max() <= TOL[w.dtype], f"attention max row error {err.max():.3e}"
