"""ctypes binding of libeagle_verify.so (the C ABI in include/eagle_verify.h).

Argument marshalling only: torch tensors become device pointers and the current CUDA
stream becomes the `stream` argument; every step of the computation runs in the
library's kernels.  There is no fallback: if the library is missing, ``load()`` raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libeagle_verify.so")

EAGLE_OK = 0
EAGLE_ERR_INVALID_ARGUMENT = 1
EAGLE_ERR_UNSUPPORTED = 2
EAGLE_ERR_WORKSPACE_TOO_SMALL = 3
EAGLE_ERR_CUDA = 4
DTYPE_F32 = 0
DTYPE_BF16 = 1

EXPORTED = ("eagle_status_string", "eagle_workspace_bytes", "eagle_tree_attention",
            "eagle_lm_head_logits", "eagle_tree_accept", "eagle_verify_step",
            "eagle_commit_accepted", "eagle_tree_rerank", "eagle_draft_select",
            "eagle_draft_select_distinct", "eagle_draft_child_rows",
            "eagle_device_error")


class Shape(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("num_nodes", ctypes.c_int32),
                ("num_q_heads", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("max_prefix_len", ctypes.c_int32),
                ("hidden", ctypes.c_int32), ("vocab", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("softmax_scale", ctypes.c_float)]


def make_shape(batch, num_nodes, num_q_heads, num_kv_heads, head_dim, max_prefix_len, hidden,
               vocab, dtype, softmax_scale: float = 0.0) -> Shape:
    if isinstance(dtype, str):
        dtype = {"f32": DTYPE_F32, "bf16": DTYPE_BF16}[dtype]
    return Shape(batch, num_nodes, num_q_heads, num_kv_heads, head_dim, max_prefix_len, hidden,
                 vocab, dtype, softmax_scale)


class EagleError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} failed: {status_string(code)} ({code})")
        self.code = code


_lib: Optional[ctypes.CDLL] = None


def load() -> ctypes.CDLL:
    """Load the CUDA library (it must have been built; see tree_verify_b200/build.py)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"CUDA library not built: {LIB_PATH} is missing "
                           "(run `python -m tree_verify_b200.build`)")
    L = ctypes.CDLL(LIB_PATH)
    vp, sz, i32, u64, f32 = (ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32, ctypes.c_uint64,
                             ctypes.c_float)
    sp = ctypes.POINTER(Shape)
    L.eagle_status_string.restype = ctypes.c_char_p
    L.eagle_status_string.argtypes = [ctypes.c_int]
    L.eagle_workspace_bytes.restype = sz
    L.eagle_workspace_bytes.argtypes = [sp]
    L.eagle_tree_attention.restype = ctypes.c_int
    L.eagle_tree_attention.argtypes = [sp] + [vp] * 9 + [sz, vp]
    L.eagle_lm_head_logits.restype = ctypes.c_int
    L.eagle_lm_head_logits.argtypes = [sp, vp, vp, vp, vp]
    L.eagle_tree_accept.restype = ctypes.c_int
    L.eagle_tree_accept.argtypes = [sp, vp, vp, vp, vp, f32, u64, u64, vp, vp, vp, vp, sz, vp]
    L.eagle_verify_step.restype = ctypes.c_int
    L.eagle_verify_step.argtypes = ([sp] + [vp] * 11 + [f32, u64, u64] + [vp] * 6 + [sz, vp])
    L.eagle_commit_accepted.restype = ctypes.c_int
    L.eagle_commit_accepted.argtypes = [sp] + [vp] * 12
    L.eagle_tree_rerank.restype = ctypes.c_int
    L.eagle_tree_rerank.argtypes = [i32, i32, i32] + [vp] * 9
    L.eagle_draft_select.restype = ctypes.c_int
    L.eagle_draft_select.argtypes = [i32, i32, i32, i32, vp, f32, u64, u64, vp, vp, vp, vp]
    L.eagle_draft_select_distinct.restype = ctypes.c_int
    L.eagle_draft_select_distinct.argtypes = [i32, i32, i32, i32, vp, f32, u64, u64, vp, vp, vp, vp]
    L.eagle_draft_child_rows.restype = ctypes.c_int
    L.eagle_draft_child_rows.argtypes = [i32, i32, i32, i32, vp, vp, vp, vp]
    L.eagle_device_error.restype = ctypes.c_int
    L.eagle_device_error.argtypes = [ctypes.POINTER(i32), i32]
    _lib = L
    return L


def status_string(code: int) -> str:
    return load().eagle_status_string(code).decode()


def workspace_bytes(shape: Shape) -> int:
    return int(load().eagle_workspace_bytes(ctypes.byref(shape)))


# ---------------------------------------------------------------- tensor marshalling

def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    import torch
    assert isinstance(t, torch.Tensor)
    if not t.is_cuda:
        raise ValueError("library arguments are device tensors")
    if not t.is_contiguous():
        raise ValueError("library arguments are contiguous tensors")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is not None:
        return stream if isinstance(stream, int) else stream.cuda_stream
    import torch
    return torch.cuda.current_stream().cuda_stream


def _check(fn: str, code: int) -> None:
    if code != EAGLE_OK:
        raise EagleError(fn, code)


def _nbytes(t) -> int:
    return 0 if t is None else t.numel() * t.element_size()


def tree_attention(shape: Shape, q, k_prefix, v_prefix, prefix_lens, k_tree, v_tree, parents, out,
                   workspace=None, stream=None) -> None:
    _check("eagle_tree_attention", load().eagle_tree_attention(
        ctypes.byref(shape), _ptr(q), _ptr(k_prefix), _ptr(v_prefix), _ptr(prefix_lens),
        _ptr(k_tree), _ptr(v_tree), _ptr(parents), _ptr(out), _ptr(workspace), _nbytes(workspace),
        _stream(stream)))


def lm_head_logits(shape: Shape, hidden, w_lm, logits, stream=None) -> None:
    _check("eagle_lm_head_logits", load().eagle_lm_head_logits(
        ctypes.byref(shape), _ptr(hidden), _ptr(w_lm), _ptr(logits), _stream(stream)))


def tree_accept(shape: Shape, logits, draft_probs, tokens, parents, temperature: float, seed: int,
                offset: int, accepted_nodes, accept_len, next_token, workspace=None,
                stream=None) -> None:
    _check("eagle_tree_accept", load().eagle_tree_accept(
        ctypes.byref(shape), _ptr(logits), _ptr(draft_probs), _ptr(tokens), _ptr(parents),
        float(temperature), int(seed), int(offset), _ptr(accepted_nodes), _ptr(accept_len),
        _ptr(next_token), _ptr(workspace), _nbytes(workspace), _stream(stream)))


def verify_step(shape: Shape, q, k_prefix, v_prefix, prefix_lens, k_tree, v_tree, parents, hidden,
                w_lm, draft_probs, tokens, temperature: float, seed: int, offset: int, out, logits,
                accepted_nodes, accept_len, next_token, workspace=None, stream=None) -> None:
    _check("eagle_verify_step", load().eagle_verify_step(
        ctypes.byref(shape), _ptr(q), _ptr(k_prefix), _ptr(v_prefix), _ptr(prefix_lens),
        _ptr(k_tree), _ptr(v_tree), _ptr(parents), _ptr(hidden), _ptr(w_lm), _ptr(draft_probs),
        _ptr(tokens), float(temperature), int(seed), int(offset), _ptr(out), _ptr(logits),
        _ptr(accepted_nodes), _ptr(accept_len), _ptr(next_token), _ptr(workspace),
        _nbytes(workspace), _stream(stream)))


def commit_accepted(shape: Shape, k_prefix, v_prefix, prefix_lens, k_tree, v_tree, hidden, parents,
                    accepted_nodes, accept_len, new_prefix_lens, feat, stream=None) -> None:
    _check("eagle_commit_accepted", load().eagle_commit_accepted(
        ctypes.byref(shape), _ptr(k_prefix), _ptr(v_prefix), _ptr(prefix_lens), _ptr(k_tree),
        _ptr(v_tree), _ptr(hidden), _ptr(parents), _ptr(accepted_nodes), _ptr(accept_len),
        _ptr(new_prefix_lens), _ptr(feat), _stream(stream)))


def tree_rerank(cand_parents, cand_tokens, confidence, num_select: int, sel, parents_out,
                tokens_out, masks_out, num_selected, stream=None) -> None:
    B, M = cand_parents.shape
    _check("eagle_tree_rerank", load().eagle_tree_rerank(
        int(B), int(M), int(num_select), _ptr(cand_parents), _ptr(cand_tokens), _ptr(confidence),
        _ptr(sel), _ptr(parents_out), _ptr(tokens_out), _ptr(masks_out), _ptr(num_selected),
        _stream(stream)))


def draft_select(logits, temperature: float, k: int, seed: int, offset: int, tokens, conf,
                 probs=None, stream=None) -> None:
    B, F, V = logits.shape
    _check("eagle_draft_select", load().eagle_draft_select(
        int(B), int(F), int(V), int(k), _ptr(logits), float(temperature), int(seed), int(offset),
        _ptr(tokens), _ptr(conf), _ptr(probs), _stream(stream)))


def draft_select_distinct(logits, temperature: float, k: int, seed: int, offset: int, tokens, conf,
                          probs=None, stream=None) -> None:
    B, F, V = logits.shape
    _check("eagle_draft_select_distinct", load().eagle_draft_select_distinct(
        int(B), int(F), int(V), int(k), _ptr(logits), float(temperature), int(seed), int(offset),
        _ptr(tokens), _ptr(conf), _ptr(probs), _stream(stream)))


def draft_child_rows(probs, tokens, child_probs, stream=None) -> None:
    B, F, V = probs.shape
    k = tokens.shape[-1]
    _check("eagle_draft_child_rows", load().eagle_draft_child_rows(
        int(B), int(F), int(V), int(k), _ptr(probs), _ptr(tokens), _ptr(child_probs), _stream(stream)))


def device_error(reset: bool = True) -> int:
    code = ctypes.c_int32(0)
    _check("eagle_device_error", load().eagle_device_error(ctypes.byref(code), int(reset)))
    return code.value
