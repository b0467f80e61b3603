"""The whole prefill attention step of one layer: score, select, attend.

This strings the C-ABI calls together on the current CUDA stream: scoring
fused with the block sums and find_blocks (xattn_score_select), then the
block-sparse attention. It holds no arithmetic of its own.
"""
from __future__ import annotations

from typing import Sequence

import torch

from .xattn import xattn_score_select, xattn_sparse_attn


def prefill_attention(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, B: int, S: int,
                      tau: Sequence[float], causal: bool, return_all: bool = False):
    """XAttention prefill attention for one layer.

    Q: [batch, hq, L, d]; K, V: [batch, hkv, L, d] (CUDA, contiguous, same
    dtype). tau: one threshold per query head. Returns O, or
    (O, probs, mask, counts, idx) with return_all.
    """
    if return_all:
        probs, mask, counts, idx = xattn_score_select(Q, K, B, S, causal, tau, probs=True)
    else:
        mask, counts, idx = xattn_score_select(Q, K, B, S, causal, tau)
    O = xattn_sparse_attn(Q, K, V, counts, idx, B, causal)
    if return_all:
        return O, probs, mask, counts, idx
    return O
