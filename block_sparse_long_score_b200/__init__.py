"""XAttention prefill hot path for NVIDIA B200 (sm_100a).

Three steps, each one call into the C-ABI library ``libxattn.so``:
``xattn_score`` (strided antidiagonal block scoring), ``xattn_select``
(find_blocks threshold selection) and ``xattn_sparse_attn`` (block-sparse
attention over the selected blocks). The pages' ablation variants run
through the same kernels: ``xattn_score_pattern`` (diagonal or random
sampling) and ``xattn_select_topk`` / ``xattn_select_topratio`` (fixed
budgets). ``xattn_prefill_host`` runs the whole step on host tensors with the
host<->device copies overlapped with the compute, and ``xattn_prefill_varlen``
on a batch of sequences of different lengths; ``xattn_check_lists`` validates
block lists made elsewhere before they reach the attention; ``xattn_score_partials``
runs the scoring GEMM alone. The library loads on first
use and the calls raise if it is missing.
"""
from .xattn import (  # noqa: F401
    XattnError, xattn_score, xattn_select, xattn_sparse_attn, xattn_score_workspace_bytes,
    xattn_attn_workspace_bytes, xattn_get_device_status, xattn_strerror, make_shape,
    library_path, EXPORTED_SYMBOLS, xattn_sparse_attn_noalloc, xattn_score_pattern,
    xattn_select_topk, xattn_select_topratio, antidiagonal_perm, diagonal_perm,
    xattn_score_select, xattn_selftest_timeout, xattn_prefill_host,
    xattn_prefill_host_workspace_bytes, xattn_prefill_varlen,
    xattn_prefill_varlen_workspace_bytes, xattn_check_lists, xattn_score_partials,
)
from .pipeline import prefill_attention, prefill_buffers  # noqa: F401
