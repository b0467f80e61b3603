"""The whole prefill attention step of one layer: score, select, attend.

This strings the C-ABI calls together on the current CUDA stream: scoring
fused with the block sums and find_blocks (xattn_score_select), then the
block-sparse attention. It holds no arithmetic of its own.
"""
from __future__ import annotations

from typing import Optional

import torch

from .xattn import (make_shape, xattn_attn_workspace_bytes, xattn_score_select,
                    xattn_score_workspace_bytes, xattn_sparse_attn)

__all__ = ["prefill_attention", "prefill_buffers"]


def prefill_buffers(Q: torch.Tensor, K: torch.Tensor, B: int, S: int, causal: bool) -> dict:
    """Every buffer one prefill_attention call writes (selection outputs, O,
    the two workspaces), allocated once so that repeated calls -- a serving
    loop, a timed loop, a CUDA-graph capture -- allocate nothing."""
    b, hq, L, d = Q.shape
    NB = -(-L // B)
    shape = make_shape(b, hq, K.shape[1], L, d, B, S, causal, Q.dtype)
    dev = Q.device
    i32 = dict(device=dev, dtype=torch.int32)
    return {
        "mask": torch.empty(b, hq, NB, (NB + 31) // 32, **i32),
        "counts": torch.empty(b, hq, NB, **i32),
        "idx": torch.empty(b, hq, NB, NB, **i32),
        "out": torch.empty_like(Q),
        "ws_score": torch.empty(max(xattn_score_workspace_bytes(shape), 1), device=dev,
                                dtype=torch.uint8),
        "ws_attn": torch.empty(max(xattn_attn_workspace_bytes(shape), 1), device=dev,
                               dtype=torch.uint8),
    }


def prefill_attention(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, B: int, S: int,
                      tau, causal: bool, return_all: bool = False,
                      buffers: Optional[dict] = None):
    """XAttention prefill attention for one layer.

    Q: [batch, hq, L, d]; K, V: [batch, hkv, L, d] (CUDA, contiguous, same
    dtype). tau: one threshold per query head (a CUDA float32 tensor, read on
    the device, or host values). ``buffers`` (from prefill_buffers) holds the
    outputs and workspaces to use instead of allocating them. Returns O, or
    (O, probs, mask, counts, idx) with return_all.
    """
    bf = buffers or {}
    sel_out = (bf["mask"], bf["counts"], bf["idx"]) if "mask" in bf else None
    if return_all:
        probs, mask, counts, idx = xattn_score_select(Q, K, B, S, causal, tau, probs=True,
                                                      out=sel_out,
                                                      workspace=bf.get("ws_score"))
    else:
        mask, counts, idx = xattn_score_select(Q, K, B, S, causal, tau, out=sel_out,
                                               workspace=bf.get("ws_score"))
    O = xattn_sparse_attn(Q, K, V, counts, idx, B, causal, out=bf.get("out"),
                          workspace=bf.get("ws_attn"))
    if return_all:
        return O, probs, mask, counts, idx
    return O
