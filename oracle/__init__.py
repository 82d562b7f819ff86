"""CPU oracle for draft-tree verification -- TEST INFRASTRUCTURE ONLY.

A plain fp64 C implementation (``oracle.c``) of the three steps of one
verification pass, loaded through ctypes.  Only ``tests/``, the smoke check
and the benchmark's CPU-baseline leg may import this package; the product
path never does.  It shares no code with the CUDA library: the two meet only
in the seeded inputs of ``workloads``.

Functions (each follows the passage cited in ``oracle.c``):
  tree_attention  O1 -- attention over prefix + own ancestors (EAGLE summary, section 3)
  lm_head         O2 -- logits = hidden W^T (EAGLE summary, section 3 "Draft model")
  tree_accept     O3 -- multi-round speculative sampling walk (EAGLE summary, section 2,
                        appendix A.2 and appendix B "Algorithm 1")
  commit          O4 -- append the root and the accepted nodes to the prefix K/V cache and
                        gather their hidden rows (EAGLE summary, section 3)
  tree_rerank     O5 -- the m candidates with the highest path confidence, renumbered as a
                        tree (EAGLE-2 blog, sections 1 and 4)
  draft_select    O6 -- the children of draft nodes: top-k at T = 0, k races at T > 0
                        (EAGLE summary, appendix A.1 "Tree Structure")
  draft_select_distinct, draft_child_rows
                  O7 -- siblings drawn without replacement and the row each was drawn from
  race, uniform, philox -- the sampler and the counter-based generator it uses
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

F32, BF16 = 0, 1
OK, BAD_TREE, BAD_ARG = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc, -O2, OpenMP, IEEE semantics)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                               "-Wall", "-Wno-unknown-pragmas", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib: Optional[ctypes.CDLL] = None


def lib() -> ctypes.CDLL:
    """The compiled oracle.  EAGLE_ORACLE_LIB names another build of oracle.c to load
    instead (the mutation tests load deliberately broken copies this way)."""
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(os.environ.get("EAGLE_ORACLE_LIB") or build())
        L = _lib
        vp, i32p, f64p = ctypes.c_void_p, ctypes.POINTER(ctypes.c_int32), ctypes.c_void_p
        L.orc_uniform.restype = ctypes.c_double
        L.orc_uniform.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int32,
                                  ctypes.c_int32, ctypes.c_int32, ctypes.c_int32]
        L.orc_philox4x32_10.argtypes = [vp, vp, vp]
        L.orc_check_tree.argtypes = [ctypes.c_int32, vp]
        L.orc_tree_attention.argtypes = [ctypes.c_int] * 7 + [vp] * 7 + [
                                         ctypes.c_double, ctypes.c_int, vp, vp]
        L.orc_lm_head.argtypes = [ctypes.c_int] * 4 + [vp, vp, ctypes.c_int, vp, vp]
        L.orc_lm_head.restype = None
        L.orc_draft_select.restype = None
        L.orc_draft_select_distinct.restype = None
        L.orc_draft_select_distinct.argtypes = [ctypes.c_int] * 4 + [vp, ctypes.c_double, ctypes.c_uint64,
                                                 ctypes.c_uint64, ctypes.c_double, vp, vp, vp, vp]
        L.orc_draft_child_rows.restype = None
        L.orc_draft_child_rows.argtypes = [ctypes.c_int] * 4 + [vp, vp, vp]
        L.orc_draft_select.argtypes = [ctypes.c_int] * 4 + [vp, ctypes.c_double, ctypes.c_uint64,
                                       ctypes.c_uint64, ctypes.c_double, vp, vp, vp, vp]
        L.orc_tree_rerank.restype = None
        L.orc_tree_rerank.argtypes = [ctypes.c_int] * 3 + [vp] * 8
        L.orc_commit.restype = None
        L.orc_commit.argtypes = [ctypes.c_int] * 7 + [vp] * 11
        L.orc_race.restype = ctypes.c_int32
        L.orc_race.argtypes = [ctypes.c_int, vp, ctypes.c_uint64, ctypes.c_uint64,
                               ctypes.c_int32, ctypes.c_int32, vp]
        L.orc_tree_accept.argtypes = ([ctypes.c_int] * 4 + [vp, ctypes.c_int, ctypes.c_int,
                                      vp, vp, vp, vp, vp, ctypes.c_double, ctypes.c_uint64,
                                      ctypes.c_uint64, ctypes.c_double] + [vp] * 8)
        L.orc_num_threads.restype = ctypes.c_int
        L.orc_fill_uniforms.argtypes = [ctypes.c_uint64, ctypes.c_uint64] + [ctypes.c_int32] * 4 + [vp]
        del i32p, f64p
    return _lib


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _elem(arr: np.ndarray) -> int:
    if arr.dtype == np.uint16:
        return BF16
    if arr.dtype == np.float32:
        return F32
    raise TypeError(f"oracle inputs are float32 or bf16 bit patterns (uint16), got {arr.dtype}")


def num_threads() -> int:
    return lib().orc_num_threads()


def philox(counter, key) -> np.ndarray:
    c = np.ascontiguousarray(counter, dtype=np.uint32)
    k = np.ascontiguousarray(key, dtype=np.uint32)
    out = np.zeros(4, dtype=np.uint32)
    lib().orc_philox4x32_10(_p(c), _p(k), _p(out))
    return out


def uniform(seed: int, offset: int, b: int, node: int, v: int, purpose: int) -> float:
    return lib().orc_uniform(seed, offset, b, node, v, purpose)


def uniforms(seed: int, offset: int, b: int, node: int, purpose: int, n: int) -> np.ndarray:
    out = np.zeros(n, dtype=np.float64)
    lib().orc_fill_uniforms(seed, offset, b, node, purpose, n, _p(out))
    return out


def check_tree(parents: np.ndarray) -> bool:
    p = np.ascontiguousarray(parents, dtype=np.int32)
    return lib().orc_check_tree(len(p), _p(p)) == OK


def tree_attention(q, k_prefix, v_prefix, prefix_lens, k_tree, v_tree, parents,
                   scale: Optional[float] = None, rows: Optional[np.ndarray] = None):
    """O1.  Inputs in the library's layouts; returns float64 [B,N,Hq,D], or [len(rows), D]
    for ``rows`` = int array of (b, i, h) triples."""
    B, N, Hq, D = q.shape
    Hkv, Lmax = k_prefix.shape[1], k_prefix.shape[2]
    et = _elem(q)
    arrs = [np.ascontiguousarray(a) for a in (q, k_prefix, v_prefix, k_tree, v_tree)]
    pl = np.ascontiguousarray(prefix_lens, dtype=np.int32)
    par = np.ascontiguousarray(parents, dtype=np.int32)
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    if rows is not None:
        rr = np.ascontiguousarray(rows, dtype=np.int32).reshape(-1, 3)
        out = np.zeros((len(rr), D), dtype=np.float64)
        nrows, rp = len(rr), _p(rr)
    else:
        out = np.zeros((B, N, Hq, D), dtype=np.float64)
        nrows, rp = 0, None
    rc = lib().orc_tree_attention(B, N, Hq, Hkv, D, Lmax, et, _p(arrs[0]), _p(arrs[1]),
                                  _p(arrs[2]), _p(pl), _p(arrs[3]), _p(arrs[4]), _p(par),
                                  float(scale), nrows, rp, _p(out))
    if rc != OK:
        raise ValueError(f"oracle tree_attention rejected its inputs (code {rc})")
    return out


def lm_head(hidden, w_lm, rows: Optional[np.ndarray] = None):
    """O2.  hidden [M,H], w_lm [V,H] (float32 or bf16 bits) -> float64 [M or len(rows), V]."""
    M, H = hidden.shape
    V = w_lm.shape[0]
    et = _elem(hidden)
    h = np.ascontiguousarray(hidden)
    w = np.ascontiguousarray(w_lm)
    if rows is not None:
        rr = np.ascontiguousarray(rows, dtype=np.int32)
        out = np.zeros((len(rr), V), dtype=np.float64)
        lib().orc_lm_head(M, H, V, et, _p(h), _p(w), len(rr), _p(rr), _p(out))
    else:
        out = np.zeros((M, V), dtype=np.float64)
        lib().orc_lm_head(M, H, V, et, _p(h), _p(w), 0, None, _p(out))
    return out


def race(weights: np.ndarray, seed: int, offset: int, b: int, node: int):
    """Exponential-race sample of unnormalised ``weights``; returns (index, relative gap)."""
    w = np.ascontiguousarray(weights, dtype=np.float64)
    gap = np.zeros(1, dtype=np.float64)
    idx = lib().orc_race(len(w), _p(w), seed, offset, b, node, _p(gap))
    return int(idx), float(gap[0])


def tree_accept(draft_probs, tokens, parents, temperature: float, seed: int = 0,
                offset: int = 0, logits=None, hidden=None, w_lm=None, margin: float = 1e-4):
    """O3.  ``logits`` [B,N,V] (float32 or float64), or ``hidden``/``w_lm`` to let the
    oracle compute the rows it visits.  Returns a dict with accepted_nodes [B,N],
    accept_len [B], next_token [B] and the margin diagnostics [B]: near (decisions inside
    the margin), decisions, first_near (index of the first near decision, -1 if none),
    exact_len (accepted nodes fixed before it; accept_len when there is none) and
    near_child (the candidate tested at the first near decision; -1 when it is the final
    race or there is none, -2 when it is a greedy argmax)."""
    B, N, V = draft_probs.shape
    dp = np.ascontiguousarray(draft_probs, dtype=np.float32)
    tk = np.ascontiguousarray(tokens, dtype=np.int32)
    par = np.ascontiguousarray(parents, dtype=np.int32)
    keep = []
    if logits is not None:
        lg = np.ascontiguousarray(logits)
        mode = 0 if lg.dtype == np.float32 else 1
        if mode == 1:
            lg = np.ascontiguousarray(lg, dtype=np.float64)
        keep.append(lg)
        lp, H, et, hp, wp = _p(lg), 0, F32, None, None
    else:
        h = np.ascontiguousarray(hidden)
        w = np.ascontiguousarray(w_lm)
        keep += [h, w]
        mode, lp, H, et, hp, wp = 2, None, h.shape[1], _elem(h), _p(h), _p(w)
    acc = np.zeros((B, N), dtype=np.int32)
    alen = np.zeros(B, dtype=np.int32)
    nxt = np.zeros(B, dtype=np.int32)
    near = np.zeros(B, dtype=np.int32)
    ndec = np.zeros(B, dtype=np.int32)
    first = np.zeros(B, dtype=np.int32)
    exact_len = np.zeros(B, dtype=np.int32)
    near_child = np.zeros(B, dtype=np.int32)
    rc = lib().orc_tree_accept(B, N, V, mode, lp, H, et, hp, wp, _p(dp), _p(tk), _p(par),
                               float(temperature), seed, offset, float(margin), _p(acc),
                               _p(alen), _p(nxt), _p(near), _p(ndec), _p(first),
                               _p(exact_len), _p(near_child))
    if rc != OK:
        raise ValueError(f"oracle tree_accept rejected its inputs (code {rc})")
    return dict(accepted_nodes=acc, accept_len=alen, next_token=nxt, near=near,
                decisions=ndec, first_near=first, exact_len=exact_len, near_child=near_child)


def commit(k_prefix, v_prefix, prefix_lens, k_tree, v_tree, hidden, parents, accepted_nodes,
           accept_len, feat=None):
    """O4: the post-accept commit on copies of the cache (bit-for-bit element copies).

    k_prefix/v_prefix [B, Hkv, Lmax, D], k_tree/v_tree [B, N, Hkv, D], hidden [B, N, H]
    (all of one element type: uint16 bf16 bits or float32), parents / accepted_nodes [B, N]
    and prefix_lens / accept_len [B] int32.  feat [B, N, H] gives the rows the commit does not
    write (default zeros).  Returns (k_prefix', v_prefix', new_lens, feat')."""
    kp = np.ascontiguousarray(k_prefix).copy()
    vp = np.ascontiguousarray(v_prefix).copy()
    B, Hkv, Lmax, D = kp.shape
    N = k_tree.shape[1]
    H = hidden.shape[-1]
    kt = np.ascontiguousarray(k_tree, dtype=kp.dtype)
    vt = np.ascontiguousarray(v_tree, dtype=kp.dtype)
    hid = np.ascontiguousarray(hidden, dtype=kp.dtype)
    out = (np.zeros((B, N, H), kp.dtype) if feat is None
           else np.ascontiguousarray(feat, dtype=kp.dtype).copy())
    lens = np.ascontiguousarray(prefix_lens, np.int32)
    par = np.ascontiguousarray(parents, np.int32)
    acc = np.ascontiguousarray(accepted_nodes, np.int32)
    alen = np.ascontiguousarray(accept_len, np.int32)
    new = np.empty(B, np.int32)
    lib().orc_commit(B, N, Hkv, D, Lmax, H, kp.itemsize, _p(kp), _p(vp), _p(lens), _p(kt), _p(vt),
                     _p(hid), _p(par), _p(acc), _p(alen), _p(new), _p(out))
    return kp, vp, new, out


def tree_rerank(parents, tokens, confidence, m: int):
    """O5: keep the m candidates with the highest path confidence (product of the clamped
    confidences from the root, float32), renumbered in candidate order.  parents / tokens
    int32 [B, M], confidence float32 [B, M].  Returns dict(sel, parents, tokens, masks,
    num_selected) with [B, m] arrays (-1 / 0 padded) and num_selected [B] (-1: bad tree)."""
    par = np.ascontiguousarray(parents, np.int32)
    tok = np.ascontiguousarray(tokens, np.int32)
    conf = np.ascontiguousarray(confidence, np.float32)
    B, M = par.shape
    out = dict(sel=np.empty((B, m), np.int32), parents=np.empty((B, m), np.int32),
               tokens=np.empty((B, m), np.int32), masks=np.empty((B, m), np.uint64),
               num_selected=np.empty(B, np.int32))
    lib().orc_tree_rerank(B, M, m, _p(par), _p(tok), _p(conf), _p(out["sel"]), _p(out["parents"]),
                          _p(out["tokens"]), _p(out["masks"]), _p(out["num_selected"]))
    return out


def draft_select(logits, temperature: float, k: int, seed: int = 0, offset: int = 0,
                 margin: float = 0.0, with_probs: bool = False):
    """O6: children of draft nodes.  logits float32 [B, F, V]; returns dict(tokens [B, F, k]
    int32, conf [B, F, k] float64, near [B, F, k] int32 and, if asked, probs [B, F, V])."""
    lg = np.ascontiguousarray(logits, np.float32)
    B, F, V = lg.shape
    out = dict(tokens=np.empty((B, F, k), np.int32), conf=np.empty((B, F, k)),
               near=np.empty((B, F, k), np.int32))
    probs = np.empty((B, F, V)) if with_probs else None
    lib().orc_draft_select(B, F, V, k, _p(lg), float(temperature), int(seed), int(offset),
                           float(margin), _p(out["tokens"]), _p(out["conf"]), _p(probs),
                           _p(out["near"]))
    if with_probs:
        out["probs"] = probs
    return out


def draft_select_distinct(logits, temperature: float, k: int, seed: int = 0, offset: int = 0,
                          margin: float = 0.0, with_probs: bool = False):
    """O7: k siblings drawn without replacement (the k smallest clocks of one race, purpose 2;
    the top k logits at T = 0).  Same arguments and outputs as draft_select."""
    lg = np.ascontiguousarray(logits, np.float32)
    B, F, V = lg.shape
    out = dict(tokens=np.empty((B, F, k), np.int32), conf=np.empty((B, F, k)),
               near=np.empty((B, F, k), np.int32))
    probs = np.empty((B, F, V)) if with_probs else None
    lib().orc_draft_select_distinct(B, F, V, k, _p(lg), float(temperature), int(seed), int(offset),
                                    float(margin), _p(out["tokens"]), _p(out["conf"]), _p(probs),
                                    _p(out["near"]))
    if with_probs:
        out["probs"] = probs
    return out


def draft_child_rows(probs, tokens):
    """O7: the row each sibling was drawn from: probs [B, F, V], tokens [B, F, k] ->
    [B, F, k, V] float64, row j = probs without tokens[..., :j], renormalised."""
    pr = np.ascontiguousarray(probs, np.float64)
    tk = np.ascontiguousarray(tokens, np.int32)
    B, F, V = pr.shape
    k = tk.shape[-1]
    out = np.empty((B, F, k, V))
    lib().orc_draft_child_rows(B, F, V, k, _p(pr), _p(tk), _p(out))
    return out
