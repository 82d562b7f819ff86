"""One verification step on device tensors: the buffers of a step and the call that runs it.

``VerifyStep`` owns the outputs and the workspace of one problem shape and calls
``eagle_verify_step`` (or the three stages separately).  Inputs are torch tensors
already on the GPU in the library's layouts.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Dict, Optional

import numpy as np
import torch

from . import binding

TORCH_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16}


def to_device(arr: np.ndarray, dtype: str, device="cuda") -> torch.Tensor:
    """numpy input (float32, or bf16 bit patterns as uint16, or int32) -> device tensor."""
    if arr.dtype == np.uint16:
        return torch.from_numpy(arr.view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(arr)).to(device)


@dataclass
class StepInputs:
    q: torch.Tensor
    k_prefix: torch.Tensor
    v_prefix: torch.Tensor
    prefix_lens: torch.Tensor
    k_tree: torch.Tensor
    v_tree: torch.Tensor
    parents: torch.Tensor
    hidden: torch.Tensor
    w_lm: torch.Tensor
    draft_probs: torch.Tensor
    tokens: torch.Tensor

    @classmethod
    def from_numpy(cls, inp: Dict[str, np.ndarray], dtype: str, device="cuda") -> "StepInputs":
        names = ["q", "k_prefix", "v_prefix", "prefix_lens", "k_tree", "v_tree", "parents", "hidden",
                 "w_lm", "draft_probs", "tokens"]
        return cls(**{n: to_device(inp[n], dtype, device) for n in names})


class VerifyStep:
    def __init__(self, shape: binding.Shape, device="cuda"):
        self.shape = shape
        B, N, Hq, D = shape.batch, shape.num_nodes, shape.num_q_heads, shape.head_dim
        dt = torch.float32 if shape.dtype == binding.DTYPE_F32 else torch.bfloat16
        self.out = torch.empty((B, N, Hq, D), dtype=dt, device=device)
        self.logits = torch.empty((B * N, shape.vocab), dtype=torch.float32, device=device)
        self.accepted_nodes = torch.empty((B, N), dtype=torch.int32, device=device)
        self.accept_len = torch.empty((B,), dtype=torch.int32, device=device)
        self.next_token = torch.empty((B,), dtype=torch.int32, device=device)
        ws = binding.workspace_bytes(shape)
        # 256-byte aligned workspace (torch's caching allocator aligns to at least 512 B)
        self.workspace = torch.empty((max(ws, 256),), dtype=torch.uint8, device=device)

    def run(self, x: StepInputs, temperature: float, seed: int = 0, offset: int = 0,
            stream: Optional[torch.cuda.Stream] = None) -> None:
        binding.verify_step(self.shape, x.q, x.k_prefix, x.v_prefix, x.prefix_lens, x.k_tree,
                            x.v_tree, x.parents, x.hidden, x.w_lm, x.draft_probs, x.tokens,
                            temperature, seed, offset, self.out, self.logits, self.accepted_nodes,
                            self.accept_len, self.next_token, self.workspace, stream)

    def attention(self, x: StepInputs, stream=None) -> None:
        binding.tree_attention(self.shape, x.q, x.k_prefix, x.v_prefix, x.prefix_lens, x.k_tree,
                               x.v_tree, x.parents, self.out, self.workspace, stream)

    def lm_head(self, x: StepInputs, stream=None) -> None:
        binding.lm_head_logits(self.shape, x.hidden, x.w_lm, self.logits, stream)

    def accept(self, x: StepInputs, temperature: float, seed: int = 0, offset: int = 0,
               logits: Optional[torch.Tensor] = None, stream=None) -> None:
        binding.tree_accept(self.shape, self.logits if logits is None else logits, x.draft_probs,
                            x.tokens, x.parents, temperature, seed, offset, self.accepted_nodes,
                            self.accept_len, self.next_token, self.workspace, stream)


    def commit(self, x: StepInputs, k_cache: torch.Tensor, v_cache: torch.Tensor,
               new_prefix_lens: torch.Tensor, feat: torch.Tensor, stream=None) -> None:
        """Post-accept commit of this step's walk: the root and the accepted nodes' K/V into
        k_cache/v_cache [B, Hkv, Lcap, D] at prefix_lens.. (Lcap from the cache's shape), their
        hidden rows into feat [B, N, H], the new lengths into new_prefix_lens [B]."""
        s = self.shape
        cache_shape = binding.make_shape(s.batch, s.num_nodes, s.num_q_heads, s.num_kv_heads,
                                         s.head_dim, k_cache.shape[2], s.hidden, s.vocab, s.dtype,
                                         s.softmax_scale)
        binding.commit_accepted(cache_shape, k_cache, v_cache, x.prefix_lens, x.k_tree, x.v_tree,
                                x.hidden, x.parents, self.accepted_nodes, self.accept_len,
                                new_prefix_lens, feat, stream)


def shape_from_workload(w) -> binding.Shape:
    return binding.make_shape(w.batch, w.num_nodes, w.num_q_heads, w.num_kv_heads, w.head_dim,
                              w.prefix_len, w.hidden, w.vocab, w.dtype)
