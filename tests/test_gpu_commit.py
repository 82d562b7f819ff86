"""eagle_commit_accepted on the GPU against oracle O4, bit for bit: random problems with
every degenerate case (invalid tree, root only, overflow of Lmax, a path that is not a
chain, a bad prefix length, rows and positions that must stay untouched), and the real
walk's output at full size (eagle_verify_step, then the commit)."""
import numpy as np
import pytest
import torch

import workloads as wl

pytestmark = pytest.mark.gpu


def _dev(a, dtype):
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _host(t):
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


def _run(cuda_lib, orc, shape, kp, vp, lens, kt, vt, hid, par, acc, alen, feat0):
    d = dict(kp=_dev(kp, None), vp=_dev(vp, None), lens=_dev(lens, None), kt=_dev(kt, None),
             vt=_dev(vt, None), hid=_dev(hid, None), par=_dev(par, None), acc=_dev(acc, None),
             alen=_dev(alen, None), new=torch.full(lens.shape, -7, dtype=torch.int32, device="cuda"),
             feat=_dev(feat0, None))
    cuda_lib.commit_accepted(shape, d["kp"], d["vp"], d["lens"], d["kt"], d["vt"], d["hid"], d["par"],
                             d["acc"], d["alen"], d["new"], d["feat"])
    torch.cuda.synchronize()
    assert cuda_lib.device_error(reset=True) == 0
    ref = orc.commit(kp, vp, lens, kt, vt, hid, par, acc, alen, feat=feat0)
    np.testing.assert_array_equal(_host(d["new"]), ref[2])
    np.testing.assert_array_equal(_host(d["kp"]), ref[0])
    np.testing.assert_array_equal(_host(d["vp"]), ref[1])
    np.testing.assert_array_equal(_host(d["feat"]), ref[3])


CASES = [  # dtype, B, N, Hkv, D, Lmax, H
    ("bf16", 4, 45, 8, 128, 300, 512),
    ("bf16", 3, 64, 2, 64, 90, 256),
    ("f32", 4, 12, 4, 64, 40, 101),   # H * 4 not a multiple of 16: word copies
    ("f32", 2, 7, 1, 128, 20, 64),
]


@pytest.mark.parametrize("case", CASES, ids=[f"{c[0]}-N{c[2]}-D{c[4]}" for c in CASES])
def test_commit_random_paths(cuda_lib, orc, case):
    dtype, B, N, Hkv, D, Lmax, H = case
    rng = np.random.default_rng(zlib_seed(case))

    def mk(shape):
        x = rng.standard_normal(shape).astype(np.float32)
        return wl.round_to_bf16_bits(x) if dtype == "bf16" else x
    par = np.stack([wl.random_parents(rng, N, 6) for _ in range(B)]).astype(np.int32)
    acc = np.full((B, N), -1, np.int32)
    alen = np.zeros(B, np.int32)
    for b in range(B):
        end = int(rng.integers(0, N))
        path = []
        while end > 0:
            path.append(end)
            end = int(par[b, end])
        path = path[::-1]
        acc[b, :len(path)] = path
        alen[b] = len(path)
    lens = rng.integers(0, Lmax - N, B).astype(np.int32)
    # degenerate sequences: invalid tree, root only, overflow, broken chain
    alen[0] = -1
    if B > 1:
        alen[1], acc[1] = 0, -1
    if B > 2:
        lens[2] = Lmax - alen[2]  # L + a + 1 = Lmax + 1
    if B > 3 and alen[3] >= 2:
        acc[3, 1] = acc[3, 0]  # a node repeated: not a chain
    shape = cuda_lib.make_shape(B, N, 4 * Hkv, Hkv, D, Lmax, H, 1000, dtype)
    feat0 = mk((B, N, H))
    _run(cuda_lib, orc, shape, mk((B, Hkv, Lmax, D)), mk((B, Hkv, Lmax, D)), lens, mk((B, N, Hkv, D)),
         mk((B, N, Hkv, D)), mk((B * N, H)), par, acc, alen, feat0)


def test_commit_bad_prefix_lengths(cuda_lib, orc):
    rng = np.random.default_rng(3)
    B, N, Hkv, D, Lmax, H = 3, 6, 2, 64, 32, 64

    def mk(shape):
        return wl.round_to_bf16_bits(rng.standard_normal(shape).astype(np.float32))
    par = np.tile(wl.chain_parents(N - 1), (B, 1)).astype(np.int32)
    acc = np.full((B, N), -1, np.int32)
    acc[:, :2] = [1, 2]
    alen = np.full(B, 2, np.int32)
    lens = np.array([-1, Lmax + 1, Lmax - 3], np.int32)  # negative, past Lmax, exactly full
    shape = cuda_lib.make_shape(B, N, 2, Hkv, D, Lmax, H, 1000, "bf16")
    _run(cuda_lib, orc, shape, mk((B, Hkv, Lmax, D)), mk((B, Hkv, Lmax, D)), lens, mk((B, N, Hkv, D)),
         mk((B, N, Hkv, D)), mk((B * N, H)), par, acc, alen, mk((B, N, H)))


@pytest.mark.parametrize("name,T", [("vicuna7b_static", 1.0), ("vicuna7b_static", 0.0)])
def test_commit_after_verify_step(cuda_lib, orc, name, T):
    """The commit of the real walk's output, at full size, equals the oracle's commit of the
    same accepted nodes, with the cache given room for the new rows."""
    from tree_verify_b200.step import StepInputs, VerifyStep, shape_from_workload
    w = wl.WORKLOADS[name]
    inp = wl.generate(w, T)
    x = StepInputs.from_numpy(inp, w.dtype)
    step = VerifyStep(shape_from_workload(w))
    step.run(x, T, 5, 6)
    torch.cuda.synchronize()
    acc, alen = step.accepted_nodes.cpu().numpy(), step.accept_len.cpu().numpy()
    assert (alen >= 0).all()
    # a cache with N more positions than the prefix stride
    B, N, Hkv, D, H = w.batch, w.num_nodes, w.num_kv_heads, w.head_dim, w.hidden
    L2 = w.prefix_len + N
    kp = np.zeros((B, Hkv, L2, D), inp["k_prefix"].dtype)
    vp = np.zeros_like(kp)
    kp[:, :, :w.prefix_len] = inp["k_prefix"]
    vp[:, :, :w.prefix_len] = inp["v_prefix"]
    shape = cuda_lib.make_shape(B, N, w.num_q_heads, Hkv, D, L2, H, w.vocab, w.dtype)
    _run(cuda_lib, orc, shape, kp, vp, inp["prefix_lens"], inp["k_tree"], inp["v_tree"],
         inp["hidden"].reshape(B * N, H), inp["parents"], acc, alen,
         np.zeros((B, N, H), kp.dtype))


def zlib_seed(case):
    import zlib
    return zlib.crc32(repr(case).encode())
