"""The C-ABI library on a machine without a GPU: it loads, exports every function that
include/eagle_verify.h declares, and rejects bad arguments with a status before any
CUDA call (nothing here launches work)."""
import ctypes
import os
import re

import pytest

from tree_verify_b200 import binding
from tree_verify_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build()
    return binding.load()


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            names |= set(re.findall(r"\b(eagle_[a-z_]+)\s*\(", text))
    return names


def test_every_declared_symbol_is_exported(lib):
    declared = _declared()
    assert {"eagle_tree_attention", "eagle_lm_head_logits", "eagle_tree_accept",
            "eagle_verify_step"} <= declared
    for name in declared:
        assert hasattr(lib, name), name
    assert set(binding.EXPORTED) <= declared


def test_status_strings(lib):
    for code, name in [(0, "EAGLE_OK"), (1, "EAGLE_ERR_INVALID_ARGUMENT"), (2, "EAGLE_ERR_UNSUPPORTED"),
                       (3, "EAGLE_ERR_WORKSPACE_TOO_SMALL"), (4, "EAGLE_ERR_CUDA")]:
        assert binding.status_string(code) == name


def _shape(**kw):
    base = dict(batch=1, num_nodes=45, num_q_heads=32, num_kv_heads=32, head_dim=128,
                max_prefix_len=1024, hidden=4096, vocab=32000, dtype="bf16")
    base.update(kw)
    return binding.make_shape(**base)


def test_workspace_sizing(lib):
    # bf16 with split-KV: partials of (D + 2) floats per (row, split)
    s = _shape()
    ws = binding.workspace_bytes(s)
    rows = 45 * 32
    assert ws >= rows * 2 * 130 * 4 and ws % 256 == 0
    # f32 path and invalid shapes need none
    assert binding.workspace_bytes(_shape(dtype="f32", head_dim=64)) == 0
    assert binding.workspace_bytes(_shape(num_nodes=65)) == 0
    assert binding.workspace_bytes(_shape(num_q_heads=6, num_kv_heads=4)) == 0


FAKE = 1 << 20  # 16-byte aligned fake device address; never dereferenced on these paths


@pytest.mark.parametrize("bad", [
    dict(num_nodes=0), dict(num_nodes=65), dict(batch=0), dict(batch=70000),
    dict(num_q_heads=6, num_kv_heads=4), dict(head_dim=96), dict(max_prefix_len=0),
    dict(hidden=4100), dict(vocab=0), dict(dtype=7),
])
def test_bad_shapes_rejected_before_launch(lib, bad):
    s = _shape(**bad)
    p = [FAKE] * 8
    rc = lib.eagle_tree_attention(ctypes.byref(s), *p, FAKE, 1 << 30, None)
    assert rc == binding.EAGLE_ERR_INVALID_ARGUMENT
    assert lib.eagle_lm_head_logits(ctypes.byref(s), FAKE, FAKE, FAKE, None) == binding.EAGLE_ERR_INVALID_ARGUMENT


def test_null_and_misaligned_pointers(lib):
    s = _shape()
    ws = binding.workspace_bytes(s)
    p = [FAKE] * 8
    p[0] = None
    assert lib.eagle_tree_attention(ctypes.byref(s), *p, FAKE, ws, None) == binding.EAGLE_ERR_INVALID_ARGUMENT
    p[0] = FAKE + 4  # misaligned q
    assert lib.eagle_tree_attention(ctypes.byref(s), *p, FAKE, ws, None) == binding.EAGLE_ERR_INVALID_ARGUMENT
    assert lib.eagle_lm_head_logits(ctypes.byref(s), FAKE, None, FAKE, None) == binding.EAGLE_ERR_INVALID_ARGUMENT
    assert lib.eagle_tree_attention(None, *([FAKE] * 8), FAKE, ws, None) == binding.EAGLE_ERR_INVALID_ARGUMENT


def test_workspace_too_small(lib):
    s = _shape()
    ws = binding.workspace_bytes(s)
    rc = lib.eagle_tree_attention(ctypes.byref(s), *([FAKE] * 8), FAKE, ws - 1, None)
    assert rc == binding.EAGLE_ERR_WORKSPACE_TOO_SMALL
    rc = lib.eagle_tree_attention(ctypes.byref(s), *([FAKE] * 8), FAKE + 16, ws, None)
    assert rc == binding.EAGLE_ERR_INVALID_ARGUMENT  # workspace must be 256-byte aligned


@pytest.mark.parametrize("T", [-1.0, float("nan"), float("inf")])
def test_bad_temperature(lib, T):
    s = _shape()
    rc = lib.eagle_tree_accept(ctypes.byref(s), FAKE, FAKE, FAKE, FAKE, T, 0, 0, FAKE, FAKE, FAKE,
                               None, 0, None)
    assert rc == binding.EAGLE_ERR_INVALID_ARGUMENT


def test_vocab_beyond_shared_memory_is_unsupported(lib):
    s = _shape(vocab=1 << 20)
    rc = lib.eagle_tree_accept(ctypes.byref(s), FAKE, FAKE, FAKE, FAKE, 1.0, 0, 0, FAKE, FAKE, FAKE,
                               None, 0, None)
    assert rc == binding.EAGLE_ERR_UNSUPPORTED


def test_verify_step_validates_every_stage(lib):
    s = _shape()
    ws = binding.workspace_bytes(s)
    args = [FAKE] * 11
    common = dict()
    rc = lib.eagle_verify_step(ctypes.byref(s), *args, -0.5, 0, 0, *([FAKE] * 5), FAKE, ws, None)
    assert rc == binding.EAGLE_ERR_INVALID_ARGUMENT
    args[8] = None  # hidden
    rc = lib.eagle_verify_step(ctypes.byref(s), *args, 1.0, 0, 0, *([FAKE] * 5), FAKE, ws, None)
    assert rc == binding.EAGLE_ERR_INVALID_ARGUMENT
    del common


def test_commit_checks_arguments_before_launch(lib):
    s = _shape()
    args = [FAKE, FAKE, FAKE + 4096, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE + 8192, FAKE]
    bad = list(args)
    bad[0] = None  # k_prefix
    assert lib.eagle_commit_accepted(ctypes.byref(s), *bad, None) == binding.EAGLE_ERR_INVALID_ARGUMENT
    bad = list(args)
    bad[5] = FAKE + 8  # misaligned hidden
    assert lib.eagle_commit_accepted(ctypes.byref(s), *bad, None) == binding.EAGLE_ERR_INVALID_ARGUMENT
    bad = list(args)
    bad[9] = args[2] + 2  # new_prefix_lens overlaps prefix_lens
    assert lib.eagle_commit_accepted(ctypes.byref(s), *bad, None) == binding.EAGLE_ERR_INVALID_ARGUMENT
    s_bad = _shape(num_nodes=65)
    assert lib.eagle_commit_accepted(ctypes.byref(s_bad), *args, None) == binding.EAGLE_ERR_INVALID_ARGUMENT


def test_rerank_checks_arguments_before_launch(lib):
    p = [FAKE] * 8
    ok = lambda B, M, m, masks=FAKE: lib.eagle_tree_rerank(B, M, m, *p[:6], masks, FAKE, None)
    assert ok(1, 1025, 8) == binding.EAGLE_ERR_INVALID_ARGUMENT   # more candidates than a CTA
    assert ok(1, 100, 65) == binding.EAGLE_ERR_INVALID_ARGUMENT   # more kept nodes than a mask
    assert ok(1, 100, 0) == binding.EAGLE_ERR_INVALID_ARGUMENT
    assert ok(0, 100, 8) == binding.EAGLE_ERR_INVALID_ARGUMENT
    assert ok(1, 100, 8, masks=FAKE + 4) == binding.EAGLE_ERR_INVALID_ARGUMENT
    assert lib.eagle_tree_rerank(1, 100, 8, None, *p[:5], FAKE, FAKE, None) == binding.EAGLE_ERR_INVALID_ARGUMENT


def test_draft_select_checks_arguments_before_launch(lib):
    call = lambda B, F, V, k, T=1.0, lg=FAKE: lib.eagle_draft_select(B, F, V, k, lg, T, 0, 0, FAKE,
                                                                     FAKE, None, None)
    assert call(1, 4, 1000, 17) == binding.EAGLE_ERR_INVALID_ARGUMENT   # more than 16 children
    assert call(1, 4, 8, 10) == binding.EAGLE_ERR_INVALID_ARGUMENT      # k > V
    assert call(1, 257, 1000, 4) == binding.EAGLE_ERR_INVALID_ARGUMENT  # node field is 8 bits
    assert call(0, 4, 1000, 4) == binding.EAGLE_ERR_INVALID_ARGUMENT
    assert call(1, 4, 1000, 4, T=-1.0) == binding.EAGLE_ERR_INVALID_ARGUMENT
    assert call(1, 4, 1000, 4, T=float("nan")) == binding.EAGLE_ERR_INVALID_ARGUMENT
    assert call(1, 4, 1000, 4, lg=None) == binding.EAGLE_ERR_INVALID_ARGUMENT
    assert call(1, 4, 1000, 4, lg=FAKE + 2) == binding.EAGLE_ERR_INVALID_ARGUMENT  # not a float address
    # a row is staged in the shared memory of at most 8 CTAs (192 KB each)
    assert call(1, 4, 8 * 49152 + 1, 4) == binding.EAGLE_ERR_UNSUPPORTED


def test_draft_distinct_and_child_rows_check_arguments_before_launch(lib):
    call = lambda B, F, V, k, T=1.0, lg=FAKE: lib.eagle_draft_select_distinct(B, F, V, k, lg, T, 0, 0, FAKE,
                                                                              FAKE, None, None)
    assert call(1, 4, 1000, 17) == binding.EAGLE_ERR_INVALID_ARGUMENT
    assert call(1, 4, 8, 10) == binding.EAGLE_ERR_INVALID_ARGUMENT
    assert call(1, 257, 1000, 4) == binding.EAGLE_ERR_INVALID_ARGUMENT
    assert call(1, 4, 1000, 4, T=float("inf")) == binding.EAGLE_ERR_INVALID_ARGUMENT
    assert call(1, 4, 1000, 4, lg=FAKE + 2) == binding.EAGLE_ERR_INVALID_ARGUMENT
    assert call(1, 4, 8 * 49152 + 1, 4) == binding.EAGLE_ERR_UNSUPPORTED
    rows = lambda B, F, V, k, pr=FAKE, tk=FAKE, out=FAKE: lib.eagle_draft_child_rows(B, F, V, k, pr, tk, out, None)
    assert rows(1, 4, 1000, 17) == binding.EAGLE_ERR_INVALID_ARGUMENT
    assert rows(0, 4, 1000, 4) == binding.EAGLE_ERR_INVALID_ARGUMENT
    assert rows(1, 4, 0, 4) == binding.EAGLE_ERR_INVALID_ARGUMENT
    assert rows(1, 4, 1000, 4, pr=None) == binding.EAGLE_ERR_INVALID_ARGUMENT
    assert rows(1, 4, 1000, 4, out=None) == binding.EAGLE_ERR_INVALID_ARGUMENT


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(binding, "LIB_PATH", str(tmp_path / "nope.so"))
    monkeypatch.setattr(binding, "_lib", None)
    with pytest.raises(RuntimeError, match="not built"):
        binding.load()
