"""eagle_tree_attention_static: tree attention for callers that cannot allocate device
memory when they call us (a server that fixed its whole device-memory plan at start-up,
or a host that gives a kernel only its inputs and outputs).  Its split scratch is a
fixed array inside the library.

Checked through the C ABI against eagle_tree_attention (caller workspace) on two calls in
a row with different inputs, so a second call cannot pass on the first call's leftovers.
This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

import workloads as wl
from tests.parity import TOL, row_rel_err

pytestmark = pytest.mark.gpu

STATIC_SCRATCH_BYTES = 16 << 20


def _static_fn(binding):
    fn = binding.load().eagle_tree_attention_static
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.POINTER(binding.Shape)] + [ctypes.c_void_p] * 9
    return fn


def _inputs(seed, B, N, Hq, Hkv, D, Lmax, lens):
    from tree_verify_b200.step import to_device
    rng = np.random.default_rng(seed)
    mk = lambda s: to_device(wl.round_to_bf16_bits(rng.standard_normal(s).astype(np.float32)), "bf16")
    par = np.stack([wl.random_parents(rng, N, 5) for _ in range(B)]).astype(np.int32)
    return dict(q=mk((B, N, Hq, D)), k_prefix=mk((B, Hkv, Lmax, D)), v_prefix=mk((B, Hkv, Lmax, D)),
                prefix_lens=torch.tensor(lens, dtype=torch.int32, device="cuda"),
                k_tree=mk((B, N, Hkv, D)), v_tree=mk((B, N, Hkv, D)),
                parents=torch.from_numpy(par).cuda())


def test_static_scratch_matches_workspace_entry_point(cuda_lib):
    fn = _static_fn(cuda_lib)
    B, N, Hq, Hkv, D, Lmax = 2, 45, 32, 8, 128, 1500
    shape = cuda_lib.make_shape(B, N, Hq, Hkv, D, Lmax, 64, 128, "bf16")
    need = cuda_lib.workspace_bytes(shape)
    assert 0 < need <= STATIC_SCRATCH_BYTES  # this shape really uses split scratch
    stream = torch.cuda.current_stream().cuda_stream
    for call, (seed, lens) in enumerate([(1, [1500, 700]), (2, [333, 1499])]):
        x = _inputs(seed, B, N, Hq, Hkv, D, Lmax, lens)
        ref = torch.empty((B, N, Hq, D), dtype=torch.bfloat16, device="cuda")
        ws = torch.empty(need, dtype=torch.uint8, device="cuda")
        cuda_lib.tree_attention(shape, x["q"], x["k_prefix"], x["v_prefix"], x["prefix_lens"],
                                x["k_tree"], x["v_tree"], x["parents"], ref, ws)
        out = torch.full_like(ref, float("nan"))
        rc = fn(ctypes.byref(shape), x["q"].data_ptr(), x["k_prefix"].data_ptr(),
                x["v_prefix"].data_ptr(), x["prefix_lens"].data_ptr(), x["k_tree"].data_ptr(),
                x["v_tree"].data_ptr(), x["parents"].data_ptr(), out.data_ptr(), stream)
        assert rc == 0, cuda_lib.status_string(rc)
        torch.cuda.synchronize()
        got, want = out.float().cpu().numpy(), ref.float().cpu().numpy()
        assert np.isfinite(got).all(), f"call {call}"
        err = row_rel_err(got.reshape(-1, D), want.reshape(-1, D))
        assert err.max() <= TOL["bf16"], f"call {call}: max row error {err.max():.3e}"
    assert cuda_lib.device_error(reset=True) == 0


def test_static_scratch_rejects_shapes_beyond_its_size(cuda_lib):
    fn = _static_fn(cuda_lib)
    # 2 sequences, 64 query / 8 kv heads, a 64K-token prefix: split partials of ~37 MB
    shape = cuda_lib.make_shape(2, 64, 64, 8, 128, 65536, 64, 128, "bf16")
    assert cuda_lib.workspace_bytes(shape) > STATIC_SCRATCH_BYTES
    fake = 1 << 20
    rc = fn(ctypes.byref(shape), *([fake] * 8), None)
    assert rc == cuda_lib.EAGLE_ERR_UNSUPPORTED
