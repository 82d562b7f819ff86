"""GPU parity of each kernel against the CPU oracle, through the C ABI.

Sizes are small enough for the oracle to finish in seconds but span several tiles and a
ragged tail in every tiled dimension: prefix keys (64-key tiles, varlen, empty prefix,
one split and many splits), query rows (GQA, several 64-row blocks), vocabulary
(128-entry tiles, V not a multiple of 4), hidden size (64-element K blocks) and tree
rows (several 256-row chunks)."""
import ctypes
import json
import os
import subprocess
import zlib

import numpy as np
import pytest
import torch

import workloads as wl
from tests.parity import MARGIN, TOL, compare_accept, row_rel_err

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(autouse=True)
def _no_device_error(cuda_lib):
    yield
    torch.cuda.synchronize()
    assert cuda_lib.device_error(reset=True) == 0


def _mk(rng, shape, dtype):
    x = rng.standard_normal(shape).astype(np.float32)
    return wl.round_to_bf16_bits(x) if dtype == "bf16" else x


def _attn_case(rng, B, N, Hq, Hkv, D, Lmax, lens, dtype, max_depth=5):
    par = np.stack([wl.random_parents(rng, N, max_depth) for _ in range(B)]).astype(np.int32)
    k_prefix = _mk(rng, (B, Hkv, Lmax, D), dtype)
    v_prefix = _mk(rng, (B, Hkv, Lmax, D), dtype)
    for b, L in enumerate(lens):  # poison the padding past L_b
        if dtype == "bf16":
            k_prefix[b, :, L:] = 0x7FC0  # NaN
            v_prefix[b, :, L:] = 0x7FC0
        else:
            k_prefix[b, :, L:] = np.nan
            v_prefix[b, :, L:] = np.nan
    return dict(q=_mk(rng, (B, N, Hq, D), dtype), k_prefix=k_prefix, v_prefix=v_prefix,
                prefix_lens=np.asarray(lens, np.int32), k_tree=_mk(rng, (B, N, Hkv, D), dtype),
                v_tree=_mk(rng, (B, N, Hkv, D), dtype), parents=par)


def _run_attention(cuda_lib, inp, dtype, H=64, V=128):
    from tree_verify_b200.step import to_device
    B, N, Hq, D = inp["q"].shape
    Hkv, Lmax = inp["k_prefix"].shape[1:3]
    shape = cuda_lib.make_shape(B, N, Hq, Hkv, D, Lmax, H, V, dtype)
    dev = {k: to_device(v, dtype) for k, v in inp.items()}
    out = torch.empty((B, N, Hq, D), dtype=torch.float32 if dtype == "f32" else torch.bfloat16,
                      device="cuda")
    ws = torch.empty(max(cuda_lib.workspace_bytes(shape), 256), dtype=torch.uint8, device="cuda")
    cuda_lib.tree_attention(shape, dev["q"], dev["k_prefix"], dev["v_prefix"], dev["prefix_lens"],
                            dev["k_tree"], dev["v_tree"], dev["parents"], out, ws)
    torch.cuda.synchronize()
    return out.float().cpu().numpy()


ATTN_CASES = [
    # B, N, Hq, Hkv, D, Lmax, lens, dtype
    (1, 6, 4, 4, 64, 64, [64], "f32"),                       # tiny chain shape, fp32
    (2, 9, 4, 2, 128, 70, [70, 3], "f32"),                   # fp32 GQA, varlen
    (2, 13, 8, 2, 128, 300, [300, 77], "bf16"),              # ragged last tile, varlen, splits
    (1, 64, 2, 2, 64, 193, [193], "bf16"),                   # max nodes, D=64
    (1, 60, 64, 8, 128, 200, [200], "bf16"),                 # G=8: 480 rows -> 8 row blocks
    (2, 7, 4, 4, 128, 50, [50, 0], "bf16"),                  # one split; an empty prefix
    (3, 21, 6, 3, 128, 1500, [1500, 640, 1], "bf16"),        # many splits, 1-key prefix
]


@pytest.mark.parametrize("case", ATTN_CASES, ids=lambda c: f"B{c[0]}N{c[1]}H{c[2]}/{c[3]}D{c[4]}L{c[5]}{c[7]}")
def test_tree_attention_matches_oracle(cuda_lib, orc, case):
    B, N, Hq, Hkv, D, Lmax, lens, dtype = case
    rng = np.random.default_rng(zlib.crc32(repr(case).encode()))
    inp = _attn_case(rng, B, N, Hq, Hkv, D, Lmax, lens, dtype)
    got = _run_attention(cuda_lib, inp, dtype)
    ref = orc.tree_attention(**inp)
    assert np.isfinite(got).all()
    err = row_rel_err(got, ref)
    assert err.max() <= TOL[dtype], f"max row error {err.max():.3e}"


def test_tree_attention_invalid_parent_is_safe(cuda_lib, orc):
    rng = np.random.default_rng(8)
    inp = _attn_case(rng, 1, 5, 2, 2, 128, 64, [64], "bf16")
    inp["parents"][0, 3] = 7  # forward link: the node keeps only itself
    got = _run_attention(cuda_lib, inp, "bf16")
    assert np.isfinite(got).all()
    inp2 = dict(inp)
    par = inp["parents"].copy()
    par[0, 3] = 0
    inp2["parents"] = par
    ok_rows = [i for i in range(5) if i != 3 and 3 not in _path(par[0], i)]
    ref = orc.tree_attention(**inp2)
    assert row_rel_err(got[0, ok_rows], ref[0, ok_rows]).max() <= TOL["bf16"]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_tree_attention_out_of_range_prefix_len_is_recorded(cuda_lib, orc, dtype):
    """A prefix length outside [0, Lmax] is a caller bug the host cannot see (the lengths
    live on the device): the kernel clamps it into range, so it stays in bounds, and
    records device error 0x205."""
    rng = np.random.default_rng(21)
    inp = _attn_case(rng, 2, 5, 4, 2, 128, 100, [100, 40], dtype)
    inp["prefix_lens"] = np.asarray([250, -3], np.int32)
    got = _run_attention(cuda_lib, inp, dtype)
    assert cuda_lib.device_error(reset=True) == 0x205
    ref = orc.tree_attention(**dict(inp, prefix_lens=np.asarray([100, 0], np.int32)))
    assert np.isfinite(got[0]).all()
    assert row_rel_err(got[0], ref[0]).max() <= TOL[dtype]
    assert row_rel_err(got[1], ref[1]).max() <= TOL[dtype]


def _path(par, i):
    out = []
    while i >= 0:
        out.append(i)
        i = par[i]
    return out


# ------------------------------------------------------------------ LM head

LM_CASES = [
    # M, H, V, dtype
    (6, 256, 512, "f32"),
    (45, 4096, 1000, "bf16"),     # ragged vocab tile
    (300, 264, 333, "bf16"),      # two row chunks, ragged K block
    (64, 128, 128, "bf16"),
    (960, 512, 700, "bf16"),      # four row chunks of 240
]


@pytest.mark.parametrize("case", LM_CASES, ids=lambda c: f"M{c[0]}H{c[1]}V{c[2]}{c[3]}")
def test_lm_head_matches_oracle(cuda_lib, orc, case):
    from tree_verify_b200.step import to_device
    M, H, V, dtype = case
    rng = np.random.default_rng(M * 7 + V)
    hidden = _mk(rng, (M, H), dtype)
    w = (rng.standard_normal((V, H)) / np.sqrt(H)).astype(np.float32)
    w = wl.round_to_bf16_bits(w) if dtype == "bf16" else w
    shape = cuda_lib.make_shape(1, 1, 1, 1, 64, 1, H, V, dtype)
    shape.batch, shape.num_nodes = M, 1
    logits = torch.full((M, V), float("nan"), dtype=torch.float32, device="cuda")
    cuda_lib.lm_head_logits(shape, to_device(hidden, dtype), to_device(w, dtype), logits)
    torch.cuda.synchronize()
    got = logits.cpu().numpy()
    ref = orc.lm_head(hidden, w)
    err = row_rel_err(got, ref)
    assert err.max() <= TOL[dtype], f"max row error {err.max():.3e}"
    if dtype == "bf16":
        # bf16 products are exact in fp32; only the fp32 accumulation rounds
        assert err.max() <= 1e-5, f"max row error {err.max():.3e}"


def test_lm_head_two_block_tiles_match_oracle(cuda_lib, orc):
    """Enough vocabulary for the persistent kernel's two-block tiles (six or more tiles of
    256 vocabulary rows per SM), with a ragged last tile whose second block lies past the
    vocabulary: every logit written, sampled rows of both row chunks against the oracle."""
    from tree_verify_b200.step import to_device
    M, H, V = 300, 256, 113_500
    rng = np.random.default_rng(2024)
    hidden = _mk(rng, (M, H), "bf16")
    w = wl.round_to_bf16_bits((rng.standard_normal((V, H)) / np.sqrt(H)).astype(np.float32))
    shape = cuda_lib.make_shape(1, 1, 1, 1, 64, 1, H, V, "bf16")
    shape.batch, shape.num_nodes = M, 1
    logits = torch.full((M, V), float("nan"), dtype=torch.float32, device="cuda")
    cuda_lib.lm_head_logits(shape, to_device(hidden, "bf16"), to_device(w, "bf16"), logits)
    torch.cuda.synchronize()
    assert cuda_lib.device_error(reset=True) == 0
    got = logits.cpu().numpy()
    assert np.isfinite(got).all()
    rows = np.array([0, 1, 77, 149, 150, 151, 159, 160, 161, 230, 298, 299], dtype=np.int32)
    ref = orc.lm_head(hidden, w, rows=rows)
    err = row_rel_err(got[rows], ref)
    assert err.max() <= 1e-5, f"max row error {err.max():.3e}"


# ------------------------------------------------------------------ accept / resample

def _accept_inputs(rng, B, N, V, T, max_depth=5, dup_draft=True):
    par = np.stack([wl.random_parents(rng, N, max_depth) for _ in range(B)]).astype(np.int32)
    logits = (rng.standard_normal((B, N, V)) * 2.0).astype(np.float32)
    draft = np.zeros((B, N, V), np.float32)
    tokens = np.zeros((B, N), np.int32)
    for b in range(B):
        ch = wl.children_lists(par[b])
        for u in range(N):
            if not ch[u]:
                continue
            # draft rows near the target's so that walks go several levels deep
            z = logits[b, u] / max(T, 1e-3) + rng.standard_normal(V) * 0.7
            z = np.exp(z - z.max())
            row = (z / z.sum()).astype(np.float32)
            if T == 0:
                order = np.argsort(-logits[b, u] + rng.standard_normal(V) * 0.3)
                picks = order[:len(ch[u])]
            else:
                r64 = row.astype(np.float64)
                picks = rng.choice(V, size=len(ch[u]), p=r64 / r64.sum())
            for c, t in zip(ch[u], picks):
                tokens[b, c] = t
                draft[b, c] = row
    return logits, draft, tokens, par


def _run_accept(cuda_lib, logits, draft, tokens, par, T, seed, offset):
    B, N, V = logits.shape
    shape = cuda_lib.make_shape(B, N, 1, 1, 64, 1, 8, V, "f32")
    d = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    acc = torch.full((B, N), -7, dtype=torch.int32, device="cuda")
    alen = torch.full((B,), -7, dtype=torch.int32, device="cuda")
    nxt = torch.full((B,), -7, dtype=torch.int32, device="cuda")
    cuda_lib.tree_accept(shape, d(logits), d(draft), d(tokens), d(par), T, seed, offset, acc, alen, nxt)
    torch.cuda.synchronize()
    return dict(accepted_nodes=acc.cpu().numpy(), accept_len=alen.cpu().numpy(),
                next_token=nxt.cpu().numpy())


@pytest.mark.parametrize("T", [0.0, 0.7, 1.0])
@pytest.mark.parametrize("V", [1000, 1001, 32000])
def test_tree_accept_matches_oracle(cuda_lib, orc, T, V):
    rng = np.random.default_rng(int(V + 10 * T))
    B, N = 24, 40
    logits, draft, tokens, par = _accept_inputs(rng, B, N, V, T)
    for seed, offset in [(0, 0), (123456789, 3), (2 ** 40 + 5, 2 ** 33 + 1)]:
        got = _run_accept(cuda_lib, logits, draft, tokens, par, T, seed, offset)
        ref = orc.tree_accept(draft, tokens, par, T, seed=seed, offset=offset, logits=logits,
                              margin=MARGIN)
        st = compare_accept(got, ref, par, exact_all=(T == 0.0))
        # identical fp32 logits on both sides: at T = 0 every decision is compared; at T > 0
        # only decisions inside the margin (rare at these sizes) are excluded
        assert st.compared >= 0.95 * st.decisions, st
        assert st.whole >= B - 2, st
    # the walks are not trivial
    assert ref["accept_len"].max() >= 2


def test_tree_accept_large_vocab(cuda_lib, orc):
    rng = np.random.default_rng(77)
    B, N, V = 4, 16, 128256
    logits, draft, tokens, par = _accept_inputs(rng, B, N, V, 1.0)
    got = _run_accept(cuda_lib, logits, draft, tokens, par, 1.0, 5, 6)
    ref = orc.tree_accept(draft, tokens, par, 1.0, seed=5, offset=6, logits=logits)
    st = compare_accept(got, ref, par)
    assert st.compared >= 0.9 * st.decisions, st


def test_tree_accept_invalid_trees(cuda_lib):
    V = 64
    rng = np.random.default_rng(1)
    logits = rng.standard_normal((4, 4, V)).astype(np.float32)
    draft = np.full((4, 4, V), 1.0 / V, np.float32)
    tokens = np.array([[0, 1, 2, 3], [0, 1, 2, 99], [0, 1, 2, 3], [0, 1, 2, 3]], np.int32)
    par = np.array([[-1, 0, 3, 0], [-1, 0, 0, 1], [0, 0, 0, 1], [-1, 0, 0, 1]], np.int32)
    got = _run_accept(cuda_lib, logits, draft, tokens, par, 1.0, 0, 0)
    assert list(got["accept_len"][:3]) == [-1, -1, -1]
    assert list(got["next_token"][:3]) == [-1, -1, -1]
    assert (got["accepted_nodes"][:3] == -1).all()
    assert got["accept_len"][3] >= 0 and 0 <= got["next_token"][3] < V


@pytest.mark.parametrize("name", ["walk_greedy_small.json", "walk_residual_small.json"])
def test_golden_walks_on_gpu(cuda_lib, name):
    g = json.load(open(os.path.join(ROOT, "tests", "golden", name)))
    V, N = g["vocab"], len(g["parents"])
    logits = np.asarray(g["logits"], np.float32)[None]
    draft = np.asarray(g.get("draft_probs", np.zeros((N, V))), np.float32)[None]
    for seed, off in [(0, 0), (99, 7)]:
        got = _run_accept(cuda_lib, logits, draft, np.asarray([g["tokens"]], np.int32),
                          np.asarray([g["parents"]], np.int32), g["temperature"], seed, off)
        assert list(got["accepted_nodes"][0]) == g["expect_accepted_nodes"]
        assert got["accept_len"][0] == g["expect_accept_len"]
        assert got["next_token"][0] == g["expect_next_token"]


# ------------------------------------------------------------------ generator pin

def test_oracle_philox_equals_curand(orc, tmp_path):
    """The oracle's Philox4x32-10 words equal cuRAND's curand_Philox4x32_10."""
    src = os.path.join(ROOT, "tests", "cuda", "philox_curand.cu")
    so = str(tmp_path / "libphilox_curand.so")
    subprocess.check_call(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O2", "-shared",
                           "-Xcompiler", "-fPIC", src, "-o", so])
    lib = ctypes.CDLL(so)
    rng = np.random.default_rng(0)
    n = 4096
    ck = rng.integers(0, 2 ** 32, size=(n, 6), dtype=np.uint64).astype(np.uint32)
    ck[0] = 0
    ck[1] = 0xFFFFFFFF
    out = np.zeros((n, 4), np.uint32)
    assert lib.philox_curand(ck.ctypes.data_as(ctypes.c_void_p), out.ctypes.data_as(ctypes.c_void_p),
                             n) == 0
    for i in range(n):
        np.testing.assert_array_equal(orc.philox(ck[i, :4], ck[i, 4:]), out[i])
