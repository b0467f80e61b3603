"""Head-sharded prefill of one layer over several GPUs, one process per GPU.

Every step of the method works per head: scoring, block sums and find_blocks
of query head h read only Q[h] and K[h // (hq/hkv)], and the attention of a
(head, query block) unit reads only that head's Q and its KV head's K and V
("XAttention: Block Sparse Attention with Antidiagonal Scoring", §2.1-§2.2
and §1 step 3 define every quantity per head). So a layer splits into
contiguous ranges of KV heads -- each with its hq/hkv query heads -- with no
exchange step: rank r of N runs KV heads [kv0, kv1) through the ordinary
calls, on views of its heads. The only collective is the optional all-gather
of O, for a caller that wants the whole output on every device.

This module holds no arithmetic: the calls run in the CUDA library, and the
functions here only cut the heads, run the calls on views and gather.
"""
from __future__ import annotations

from typing import Callable, Optional

import torch

__all__ = ["kv_head_range", "run_heads", "prefill_attention_heads", "gather_heads"]


def kv_head_range(rank: int, world: int, hkv: int) -> tuple:
    """Contiguous KV heads [kv0, kv1) of `rank` out of `world`: the first
    hkv % world ranks take one head more; ranks past hkv get an empty range."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("need 0 <= rank < world")
    base, extra = divmod(hkv, world)
    kv0 = rank * base + min(rank, extra)
    kv1 = kv0 + base + (1 if rank < extra else 0)
    return kv0, kv1


def run_heads(step: Callable, Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, tau,
              kv0: int, kv1: int, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Runs `step(Qv, Kv, Vv, tau_v, Ov)` on the heads of KV range [kv0, kv1)
    of every batch entry. Q: [batch, hq, L, d]; K, V: [batch, hkv, L, d];
    tau: hq values (a sequence or a tensor). Each call gets batch-1 views
    ([1, heads, L, d], contiguous) and writes Ov, a view of the returned
    [batch, (kv1 - kv0) * g, L, d] tensor (`out` if given)."""
    b, hq = Q.shape[0], Q.shape[1]
    hkv = K.shape[1]
    g = hq // hkv
    h0, h1 = kv0 * g, kv1 * g
    if out is None:
        out = torch.empty((b, h1 - h0) + tuple(Q.shape[2:]), dtype=Q.dtype, device=Q.device)
    if h1 == h0:
        return out
    tau_v = tau[h0:h1]
    for bb in range(b):
        step(Q[bb:bb + 1, h0:h1], K[bb:bb + 1, kv0:kv1], V[bb:bb + 1, kv0:kv1], tau_v,
             out[bb:bb + 1])
    return out


def prefill_attention_heads(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, B: int, S: int,
                            tau, causal: bool, kv0: int, kv1: int,
                            out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """The prefill step (xattn_score_select, then xattn_sparse_attn) of the
    query heads of KV heads [kv0, kv1). Returns O of those heads,
    [batch, (kv1 - kv0) * hq / hkv, L, d]; bit-identical to the same heads of
    the whole-layer call."""
    from .xattn import xattn_score_select, xattn_sparse_attn

    def step(q, k, v, t, o):
        _, counts, idx = xattn_score_select(q, k, B, S, causal, t)
        xattn_sparse_attn(q, k, v, counts, idx, B, causal, out=o)

    return run_heads(step, Q, K, V, tau, kv0, kv1, out=out)


def gather_heads(O_local: torch.Tensor, hq: int, hkv: int, group=None) -> torch.Tensor:
    """All-gathers every rank's head range into O [batch, hq, L, d] on every
    rank (torch.distributed; NCCL on GPUs). Ranges are padded to the largest
    one for the collective and cut back in head order."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    g = hq // hkv
    ranges = [kv_head_range(r, world, hkv) for r in range(world)]
    most = max(k1 - k0 for k0, k1 in ranges) * g
    b = O_local.shape[0]
    tail = tuple(O_local.shape[2:])
    pad = torch.zeros((b, most) + tail, dtype=O_local.dtype, device=O_local.device)
    pad[:, :O_local.shape[1]] = O_local
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad.contiguous(), group=group)
    full = torch.empty((b, hq) + tail, dtype=O_local.dtype, device=O_local.device)
    for (k0, k1), part in zip(ranges, parts):
        full[:, k0 * g:k1 * g] = part[:, :(k1 - k0) * g]
    return full
