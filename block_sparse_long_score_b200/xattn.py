"""Python binding of libxattn.so: argument marshalling only.

Every function here has the name of the C entry point it calls
(``include/xattn.h``). It checks that the tensors are CUDA, contiguous and of
the right dtype, allocates outputs and workspace with torch when the caller
gives none, and passes raw pointers plus the current CUDA stream to the
library. All computation happens in the library's CUDA kernels. There is no
fallback: if the library is missing, or a call fails, this module raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

__all__ = [
    "XattnError", "xattn_score", "xattn_select", "xattn_sparse_attn",
    "xattn_score_workspace_bytes", "xattn_attn_workspace_bytes",
    "xattn_get_device_status", "xattn_strerror", "make_shape", "library_path",
    "EXPORTED_SYMBOLS", "xattn_sparse_attn_noalloc", "NOALLOC_MAX_UNITS",
    "xattn_score_pattern", "xattn_select_topk", "xattn_select_topratio",
    "antidiagonal_perm", "diagonal_perm", "xattn_score_select", "xattn_selftest_timeout",
    "xattn_prefill_host_workspace_bytes", "xattn_prefill_host",
    "xattn_prefill_varlen_workspace_bytes", "xattn_prefill_varlen", "xattn_check_lists",
    "xattn_score_partials",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIBNAME = "libxattn.so"

XATTN_F32, XATTN_BF16 = 0, 1
EXPORTED_SYMBOLS = (
    "xattn_score_workspace_bytes", "xattn_score", "xattn_select",
    "xattn_attn_workspace_bytes", "xattn_sparse_attn", "xattn_get_device_status",
    "xattn_strerror", "xattn_sparse_attn_noalloc", "xattn_score_pattern",
    "xattn_select_topk", "xattn_select_topratio", "xattn_score_select",
    "xattn_selftest_timeout", "xattn_prefill_host_workspace_bytes", "xattn_prefill_host",
    "xattn_prefill_varlen_workspace_bytes", "xattn_prefill_varlen", "xattn_check_lists",
    "xattn_score_partials",
)
# batch * hq * NB limit of xattn_sparse_attn_noalloc (XATTN_NOALLOC_MAX_UNITS)
NOALLOC_MAX_UNITS = 1 << 18


class XattnError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} failed: {xattn_strerror(code)} ({code})")
        self.code = code


class _Shape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in
                ("batch", "hq", "hkv", "L", "d", "B", "S", "causal", "dtype")]


_lib_handle = None


def library_path() -> str:
    return os.path.join(_HERE, _LIBNAME)


def _lib() -> ctypes.CDLL:
    global _lib_handle
    if _lib_handle is None:
        path = library_path()
        if not os.path.exists(path):
            raise ImportError(
                f"{path} is missing: build it with `python -m block_sparse_long_score_b200.build`")
        lib = ctypes.CDLL(path)
        vp, sz, i32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
        sp = ctypes.POINTER(_Shape)
        lib.xattn_score_workspace_bytes.argtypes = [sp]
        lib.xattn_score_workspace_bytes.restype = sz
        lib.xattn_attn_workspace_bytes.argtypes = [sp]
        lib.xattn_attn_workspace_bytes.restype = sz
        lib.xattn_score.argtypes = [vp, vp, sp, vp, vp, sz, vp]
        lib.xattn_score_partials.argtypes = [vp, vp, sp, vp, sz, vp]
        lib.xattn_score_partials.restype = i32
        lib.xattn_score.restype = i32
        lib.xattn_select.argtypes = [vp, vp, sp, vp, vp, vp, vp]
        lib.xattn_select.restype = i32
        lib.xattn_score_pattern.argtypes = [vp, vp, sp, ctypes.POINTER(ctypes.c_int32), vp, vp,
                                            sz, vp]
        lib.xattn_score_pattern.restype = i32
        lib.xattn_score_select.argtypes = [vp, vp, sp, vp, vp, vp, vp, vp, vp, sz, vp]
        lib.xattn_score_select.restype = i32
        lib.xattn_select_topk.argtypes = [vp, ctypes.POINTER(ctypes.c_int32), sp, vp, vp, vp,
                                          vp]
        lib.xattn_select_topk.restype = i32
        lib.xattn_select_topratio.argtypes = [vp, ctypes.POINTER(ctypes.c_float), sp, vp, vp,
                                              vp, vp]
        lib.xattn_select_topratio.restype = i32
        lib.xattn_sparse_attn.argtypes = [vp, vp, vp, sp, vp, vp, vp, vp, vp, sz, vp]
        lib.xattn_sparse_attn.restype = i32
        lib.xattn_sparse_attn_noalloc.argtypes = [vp, vp, vp, sp, vp, vp, vp, vp, vp]
        lib.xattn_sparse_attn_noalloc.restype = i32
        lib.xattn_prefill_host_workspace_bytes.argtypes = [sp, i32]
        lib.xattn_prefill_host_workspace_bytes.restype = sz
        lib.xattn_prefill_host.argtypes = [vp, vp, vp, sp, ctypes.POINTER(ctypes.c_float), vp,
                                           vp, i32, vp, sz, vp]
        lib.xattn_prefill_host.restype = i32
        i32p = ctypes.POINTER(ctypes.c_int32)
        lib.xattn_prefill_varlen_workspace_bytes.argtypes = [sp, i32, i32p]
        lib.xattn_prefill_varlen_workspace_bytes.restype = sz
        lib.xattn_prefill_varlen.argtypes = [vp, vp, vp, sp, i32, i32p,
                                             ctypes.POINTER(ctypes.c_float), vp, vp, vp, sz, vp]
        lib.xattn_prefill_varlen.restype = i32
        lib.xattn_check_lists.argtypes = [vp, vp, sp, vp, vp]
        lib.xattn_check_lists.restype = i32
        lib.xattn_selftest_timeout.argtypes = [vp]
        lib.xattn_selftest_timeout.restype = i32
        lib.xattn_get_device_status.argtypes = [vp]
        lib.xattn_get_device_status.restype = i32
        lib.xattn_strerror.argtypes = [i32]
        lib.xattn_strerror.restype = ctypes.c_char_p
        _lib_handle = lib
    return _lib_handle


def xattn_strerror(code: int) -> str:
    return _lib().xattn_strerror(int(code)).decode()


def make_shape(batch: int, hq: int, hkv: int, L: int, d: int, B: int, S: int, causal: bool,
               dtype) -> _Shape:
    dt = XATTN_BF16 if dtype in (torch.bfloat16, "bf16", XATTN_BF16) else XATTN_F32
    return _Shape(int(batch), int(hq), int(hkv), int(L), int(d), int(B), int(S),
                  1 if causal else 0, dt)


def _shape_of(Q: torch.Tensor, K: torch.Tensor, B: int, S: int, causal: bool) -> _Shape:
    if Q.dim() != 4 or K.dim() != 4:
        raise ValueError("Q and K must be [batch, heads, L, d]")
    b, hq, L, d = Q.shape
    if K.shape[0] != b or K.shape[2] != L or K.shape[3] != d:
        raise ValueError("K shape does not match Q")
    return make_shape(b, hq, K.shape[1], L, d, B, S, causal, Q.dtype)


def _attn_shape(Q, K, V, counts, idx, B: int, causal: bool) -> _Shape:
    """Shape of an attention call, after checking V against K and the block
    lists against the number of work units."""
    shape = _shape_of(Q, K, B, 1, causal)
    _check_shape(V, K.shape, "V")
    _check_lists(counts, idx, shape.batch, shape.hq, -(-shape.L // max(shape.B, 1)))
    return shape


def _check(t: torch.Tensor, name: str, dtype=None) -> None:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")


def _check_shape(t: torch.Tensor, shape, name: str) -> None:
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _check_lists(counts: torch.Tensor, idx: torch.Tensor, batch: int, hq: int, NB: int) -> None:
    """counts [batch, hq, NB] and idx [batch, hq, NB, NB] (the kernels index
    them by unit; a smaller buffer would be read past its end)."""
    if counts.numel() != batch * hq * NB or idx.numel() != batch * hq * NB * NB:
        raise ValueError(f"counts / idx must hold {batch}x{hq}x{NB} rows of {NB} entries, got "
                         f"{tuple(counts.shape)} / {tuple(idx.shape)}")


def _check_select_outputs(mask, counts, idx, batch: int, hq: int, NB: int) -> None:
    for t, n in ((mask, "mask"), (counts, "counts"), (idx, "idx")):
        _check(t, n, torch.int32)
    _check_shape(mask, (batch, hq, NB, (NB + 31) // 32), "mask")
    _check_shape(counts, (batch, hq, NB), "counts")
    _check_shape(idx, (batch, hq, NB, NB), "idx")


def _same_device(ref: torch.Tensor, *ts) -> None:
    for t in ts:
        if t is not None and t.device != ref.device:
            raise ValueError(f"every tensor must be on {ref.device}, got one on {t.device}")


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _raise(fn: str, rc: int) -> None:
    if rc != 0:
        raise XattnError(fn, rc)


def xattn_score_workspace_bytes(shape: _Shape) -> int:
    return int(_lib().xattn_score_workspace_bytes(ctypes.byref(shape)))


def xattn_attn_workspace_bytes(shape: _Shape) -> int:
    return int(_lib().xattn_attn_workspace_bytes(ctypes.byref(shape)))


def antidiagonal_perm(S: int) -> list:
    """Sampling pattern of xattn_score: chunk i reads query sub-row S-1-i."""
    return [S - 1 - i for i in range(S)]


def diagonal_perm(S: int) -> list:
    """Main-diagonal sampling pattern: chunk i reads query sub-row i."""
    return list(range(S))


def xattn_score(Q: torch.Tensor, K: torch.Tensor, B: int, S: int, causal: bool,
                probs: Optional[torch.Tensor] = None,
                workspace: Optional[torch.Tensor] = None,
                perm: Optional[Sequence[int]] = None) -> torch.Tensor:
    """Block probabilities P [batch, hq, NB, NB] (fp32, NB = ceil(L/B)) of antidiagonal
    scoring.

    With ``perm`` (a permutation of 0..S-1) the call is xattn_score_pattern:
    chunk i pairs query sub-row perm[i] with key sub-row i."""
    _check(Q, "Q")
    _check(K, "K", Q.dtype)
    shape = _shape_of(Q, K, B, S, causal)
    NB = -(-shape.L // max(shape.B, 1))
    if probs is None:
        probs = torch.empty(shape.batch, shape.hq, NB, NB, device=Q.device, dtype=torch.float32)
    _check(probs, "probs", torch.float32)
    _check_shape(probs, (shape.batch, shape.hq, NB, NB), "probs")
    need = xattn_score_workspace_bytes(shape)
    if workspace is None:
        workspace = torch.empty(max(need, 1), device=Q.device, dtype=torch.uint8)
    _check(workspace, "workspace")
    _same_device(Q, K, probs, workspace)
    with torch.cuda.device(Q.device):
        return _score_call(Q, K, S, shape, probs, workspace, perm)


def xattn_score_partials(Q: torch.Tensor, K: torch.Tensor, B: int, S: int, causal: bool,
                         workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """The scoring GEMM alone: the per-key-block partial log2-sum-exp sums of
    every reshaped query row, written to (and returned as) the uint8 scoring
    workspace; the sums are its first fp32 entries, laid out as the header
    states."""
    _check(Q, "Q")
    _check(K, "K", Q.dtype)
    shape = _shape_of(Q, K, B, S, causal)
    need = xattn_score_workspace_bytes(shape)
    if workspace is None:
        workspace = torch.empty(max(need, 1), device=Q.device, dtype=torch.uint8)
    _check(workspace, "workspace")
    _same_device(Q, K, workspace)
    with torch.cuda.device(Q.device):
        rc = _lib().xattn_score_partials(Q.data_ptr(), K.data_ptr(), ctypes.byref(shape),
                                         workspace.data_ptr(),
                                         workspace.numel() * workspace.element_size(),
                                         _stream(Q.device))
    _raise("xattn_score_partials", rc)
    return workspace


def _score_call(Q, K, S, shape, probs, workspace, perm):
    if perm is None:
        rc = _lib().xattn_score(Q.data_ptr(), K.data_ptr(), ctypes.byref(shape),
                                probs.data_ptr(), workspace.data_ptr(),
                                workspace.numel() * workspace.element_size(), _stream(Q.device))
        _raise("xattn_score", rc)
    else:
        perm = [int(x) for x in perm]
        if len(perm) != S:
            raise ValueError("perm needs S entries")
        parr = (ctypes.c_int32 * S)(*perm)
        rc = _lib().xattn_score_pattern(Q.data_ptr(), K.data_ptr(), ctypes.byref(shape), parr,
                                        probs.data_ptr(), workspace.data_ptr(),
                                        workspace.numel() * workspace.element_size(),
                                        _stream(Q.device))
        _raise("xattn_score_pattern", rc)
    return probs


def xattn_score_pattern(Q: torch.Tensor, K: torch.Tensor, B: int, S: int, causal: bool,
                        perm: Sequence[int], probs: Optional[torch.Tensor] = None,
                        workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Scoring with the sampling pattern ``perm`` (see xattn_score)."""
    return xattn_score(Q, K, B, S, causal, probs=probs, workspace=workspace, perm=perm)


def _select_outputs(probs: torch.Tensor, causal: bool, out: Optional[tuple]):
    _check(probs, "probs", torch.float32)
    b, hq, NB, NB2 = probs.shape
    if NB != NB2:
        raise ValueError("probs must be [batch, hq, NB, NB]")
    shape = make_shape(b, hq, hq, NB, 128, 1, 1, causal, XATTN_F32)
    W = (NB + 31) // 32
    if out is None:
        mask = torch.empty(b, hq, NB, W, device=probs.device, dtype=torch.int32)
        counts = torch.empty(b, hq, NB, device=probs.device, dtype=torch.int32)
        idx = torch.empty(b, hq, NB, NB, device=probs.device, dtype=torch.int32)
    else:
        mask, counts, idx = out
    _check_select_outputs(mask, counts, idx, b, hq, NB)
    _same_device(probs, mask, counts, idx)
    return shape, mask, counts, idx


def _tau_device(tau, hq: int, device) -> torch.Tensor:
    """Per-head thresholds as the device array the C ABI reads: a CUDA float32
    tensor of hq values is used as it is (the kernels check each value and
    report one outside (0, 1] through xattn_get_device_status); host values
    are checked here and copied to the device (a synchronous copy, so pass a
    CUDA tensor inside a CUDA-graph capture)."""
    if isinstance(tau, torch.Tensor) and tau.is_cuda:
        _check(tau, "tau", torch.float32)
        if tau.numel() != hq:
            raise ValueError("tau needs one value per query head")
        if tau.device != torch.device(device):
            raise ValueError(f"tau must be on {device}, got {tau.device}")
        return tau
    vals = [float(v) for v in (tau.tolist() if hasattr(tau, "tolist") else tau)]
    if len(vals) != hq:
        raise ValueError("tau needs one value per query head")
    if not all(0.0 < v <= 1.0 for v in vals):
        raise ValueError("every tau must lie in (0, 1]")
    return torch.tensor(vals, dtype=torch.float32).to(device)


def _per_head(values, hq: int, name: str, kind):
    vals = [kind(v) for v in values]
    if len(vals) != hq:
        raise ValueError(f"{name} needs one value per query head")
    return vals


def xattn_select(probs: torch.Tensor, tau, causal: bool, out: Optional[tuple] = None):
    """find_blocks on every row of P with per-head thresholds ``tau`` (a CUDA
    float32 tensor [hq], read on the device, or host values). Returns (mask
    uint32 [.., NB, ceil(NB/32)] as int32, counts int32 [.., NB], idx int32
    [.., NB, NB])."""
    shape, mask, counts, idx = _select_outputs(probs, causal, out)
    with torch.cuda.device(probs.device):
        tdev = _tau_device(tau, shape.hq, probs.device)
        rc = _lib().xattn_select(probs.data_ptr(), tdev.data_ptr(), ctypes.byref(shape),
                                 mask.data_ptr(), counts.data_ptr(), idx.data_ptr(),
                                 _stream(probs.device))
    _raise("xattn_select", rc)
    return mask, counts, idx


def xattn_score_select(Q: torch.Tensor, K: torch.Tensor, B: int, S: int, causal: bool,
                       tau, probs: Optional[torch.Tensor] | bool = None,
                       out: Optional[tuple] = None, workspace: Optional[torch.Tensor] = None):
    """Scoring and find_blocks in one call (P stays on chip); ``tau`` as for
    xattn_select. Returns (mask, counts, idx), or (probs, mask, counts, idx)
    when probs is True or a tensor."""
    _check(Q, "Q")
    _check(K, "K", Q.dtype)
    shape = _shape_of(Q, K, B, S, causal)
    NB = -(-shape.L // max(shape.B, 1))
    want_p = probs is not None and probs is not False
    if probs is True:
        probs = torch.empty(shape.batch, shape.hq, NB, NB, device=Q.device, dtype=torch.float32)
    if want_p:
        _check(probs, "probs", torch.float32)
        _check_shape(probs, (shape.batch, shape.hq, NB, NB), "probs")
    W = (NB + 31) // 32
    if out is None:
        mask = torch.empty(shape.batch, shape.hq, NB, W, device=Q.device, dtype=torch.int32)
        counts = torch.empty(shape.batch, shape.hq, NB, device=Q.device, dtype=torch.int32)
        idx = torch.empty(shape.batch, shape.hq, NB, NB, device=Q.device, dtype=torch.int32)
    else:
        mask, counts, idx = out
    _check_select_outputs(mask, counts, idx, shape.batch, shape.hq, NB)
    need = xattn_score_workspace_bytes(shape)
    if workspace is None:
        workspace = torch.empty(max(need, 1), device=Q.device, dtype=torch.uint8)
    _check(workspace, "workspace")
    _same_device(Q, K, probs if want_p else None, mask, counts, idx, workspace)
    with torch.cuda.device(Q.device):
        tdev = _tau_device(tau, shape.hq, Q.device)
        rc = _lib().xattn_score_select(Q.data_ptr(), K.data_ptr(), ctypes.byref(shape),
                                       tdev.data_ptr(), probs.data_ptr() if want_p else None,
                                       mask.data_ptr(), counts.data_ptr(), idx.data_ptr(),
                                       workspace.data_ptr(),
                                       workspace.numel() * workspace.element_size(),
                                       _stream(Q.device))
    _raise("xattn_score_select", rc)
    return (probs, mask, counts, idx) if want_p else (mask, counts, idx)


def xattn_select_topk(probs: torch.Tensor, k: Sequence[int], causal: bool,
                      out: Optional[tuple] = None):
    """Top-K: the k[h] best allowed blocks of every row (outputs as xattn_select)."""
    shape, mask, counts, idx = _select_outputs(probs, causal, out)
    ks = _per_head(k, shape.hq, "k", int)
    karr = (ctypes.c_int32 * shape.hq)(*ks)
    with torch.cuda.device(probs.device):
        rc = _lib().xattn_select_topk(probs.data_ptr(), karr, ctypes.byref(shape),
                                      mask.data_ptr(), counts.data_ptr(), idx.data_ptr(),
                                      _stream(probs.device))
    _raise("xattn_select_topk", rc)
    return mask, counts, idx


def xattn_select_topratio(probs: torch.Tensor, ratio: Sequence[float], causal: bool,
                          out: Optional[tuple] = None):
    """Top-Ratio: round(ratio[h] * allowed) best blocks of every row (at least one)."""
    shape, mask, counts, idx = _select_outputs(probs, causal, out)
    rs = _per_head(ratio, shape.hq, "ratio", float)
    rarr = (ctypes.c_float * shape.hq)(*rs)
    with torch.cuda.device(probs.device):
        rc = _lib().xattn_select_topratio(probs.data_ptr(), rarr, ctypes.byref(shape),
                                          mask.data_ptr(), counts.data_ptr(), idx.data_ptr(),
                                          _stream(probs.device))
    _raise("xattn_select_topratio", rc)
    return mask, counts, idx


def xattn_sparse_attn(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, counts: torch.Tensor,
                      idx: torch.Tensor, B: int, causal: bool, out: Optional[torch.Tensor] = None,
                      lse: Optional[torch.Tensor] | bool = None,
                      workspace: Optional[torch.Tensor] = None):
    """Attention over the listed key blocks. Returns O, or (O, lse) if lse is
    True or a tensor."""
    _check(Q, "Q")
    _check(K, "K", Q.dtype)
    _check(V, "V", Q.dtype)
    _check(counts, "counts", torch.int32)
    _check(idx, "idx", torch.int32)
    shape = _attn_shape(Q, K, V, counts, idx, B, causal)
    if out is None:
        out = torch.empty_like(Q)
    _check(out, "O", Q.dtype)
    _check_shape(out, Q.shape, "O")
    want_lse = lse is not None and lse is not False
    if lse is True:
        lse = torch.empty(Q.shape[:3], device=Q.device, dtype=torch.float32)
    if want_lse:
        _check(lse, "lse", torch.float32)
        _check_shape(lse, Q.shape[:3], "lse")
    need = xattn_attn_workspace_bytes(shape)
    if workspace is None:
        workspace = torch.empty(max(need, 1), device=Q.device, dtype=torch.uint8)
    _check(workspace, "workspace")
    _same_device(Q, K, V, counts, idx, out, lse if want_lse else None, workspace)
    with torch.cuda.device(Q.device):
        rc = _lib().xattn_sparse_attn(Q.data_ptr(), K.data_ptr(), V.data_ptr(),
                                      ctypes.byref(shape), counts.data_ptr(), idx.data_ptr(),
                                      out.data_ptr(), lse.data_ptr() if want_lse else None,
                                      workspace.data_ptr(),
                                      workspace.numel() * workspace.element_size(),
                                      _stream(Q.device))
    _raise("xattn_sparse_attn", rc)
    return (out, lse) if want_lse else out


def xattn_sparse_attn_noalloc(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor,
                              counts: torch.Tensor, idx: torch.Tensor, B: int, causal: bool,
                              out: torch.Tensor, lse: Optional[torch.Tensor] = None):
    """xattn_sparse_attn for callers that cannot allocate: the library keeps the
    work order in its own device array, and the caller passes every output
    buffer (``out``, and ``lse`` if wanted). Nothing is allocated here."""
    _check(Q, "Q")
    _check(K, "K", Q.dtype)
    _check(V, "V", Q.dtype)
    _check(counts, "counts", torch.int32)
    _check(idx, "idx", torch.int32)
    _check(out, "O", Q.dtype)
    shape = _attn_shape(Q, K, V, counts, idx, B, causal)
    _check_shape(out, Q.shape, "O")
    if lse is not None:
        _check(lse, "lse", torch.float32)
        _check_shape(lse, Q.shape[:3], "lse")
    _same_device(Q, K, V, counts, idx, out, lse)
    with torch.cuda.device(Q.device):
        rc = _lib().xattn_sparse_attn_noalloc(Q.data_ptr(), K.data_ptr(), V.data_ptr(),
                                              ctypes.byref(shape), counts.data_ptr(),
                                              idx.data_ptr(), out.data_ptr(),
                                              lse.data_ptr() if lse is not None else None,
                                              _stream(Q.device))
    _raise("xattn_sparse_attn_noalloc", rc)
    return out


def xattn_check_lists(Q: torch.Tensor, K: torch.Tensor, counts: torch.Tensor, idx: torch.Tensor,
                      B: int, causal: bool, bad: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Counts the rows of (counts, idx) that break the list layout
    xattn_sparse_attn expects (counts in [0, NB], entries strictly ascending
    in [0, NB)). Q and K give the shape only. Returns a one-element int32
    device tensor (``bad`` if given), written on the current stream."""
    _check(Q, "Q")
    _check(K, "K", Q.dtype)
    _check(counts, "counts", torch.int32)
    _check(idx, "idx", torch.int32)
    shape = _shape_of(Q, K, B, 1, causal)
    rows = shape.batch * shape.hq * -(-shape.L // shape.B)
    if counts.numel() != rows or idx.numel() != rows * -(-shape.L // shape.B):
        raise ValueError("counts / idx do not match the shape")
    if bad is None:
        bad = torch.empty(1, device=Q.device, dtype=torch.int32)
    _check(bad, "bad", torch.int32)
    _same_device(Q, counts, idx, bad)
    with torch.cuda.device(Q.device):
        rc = _lib().xattn_check_lists(counts.data_ptr(), idx.data_ptr(), ctypes.byref(shape),
                                      bad.data_ptr(), _stream(Q.device))
    _raise("xattn_check_lists", rc)
    return bad


def xattn_prefill_host_workspace_bytes(shape: _Shape, kv_heads_per_chunk: int = 0) -> int:
    return int(_lib().xattn_prefill_host_workspace_bytes(ctypes.byref(shape),
                                                         int(kv_heads_per_chunk)))


def _check_any(t: torch.Tensor, name: str, dtype=None) -> None:
    """Layout and type check of a tensor that may live in host or device memory."""
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")


def xattn_prefill_host(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, B: int, S: int,
                       causal: bool, tau: Sequence[float], out: Optional[torch.Tensor] = None,
                       lse: Optional[torch.Tensor] | bool = None, kv_heads_per_chunk: int = 0,
                       workspace: Optional[torch.Tensor] = None, device=None):
    """The whole prefill step (score + select with threshold tau, then sparse
    attention) on Q, K, V in host memory -- pinned for the copies to overlap
    the compute -- with O (and lse) written to host memory. Runs on the current
    stream of ``device`` (the current CUDA device by default); synchronise it
    before reading ``out``. Returns O, or (O, lse) if lse is True or a tensor."""
    _check_any(Q, "Q")
    _check_any(K, "K", Q.dtype)
    _check_any(V, "V", Q.dtype)
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None \
        else torch.device(device)
    shape = _shape_of(Q, K, B, S, causal)
    if out is None:
        out = torch.empty(Q.shape, dtype=Q.dtype, pin_memory=not Q.is_cuda,
                          device=Q.device)
    _check_any(out, "O", Q.dtype)
    _check_shape(V, K.shape, "V")
    _check_shape(out, Q.shape, "O")
    want_lse = lse is not None and lse is not False
    if lse is True:
        lse = torch.empty(Q.shape[:3], dtype=torch.float32, pin_memory=not Q.is_cuda,
                          device=Q.device)
    if want_lse:
        _check_any(lse, "lse", torch.float32)
        _check_shape(lse, Q.shape[:3], "lse")
    taus = _per_head(tau, shape.hq, "tau", float)
    tarr = (ctypes.c_float * shape.hq)(*taus)
    need = xattn_prefill_host_workspace_bytes(shape, kv_heads_per_chunk)
    if workspace is None:
        workspace = torch.empty(max(need, 1), device=dev, dtype=torch.uint8)
    _check(workspace, "workspace")
    rc = _lib().xattn_prefill_host(Q.data_ptr(), K.data_ptr(), V.data_ptr(), ctypes.byref(shape),
                                   tarr, out.data_ptr(), lse.data_ptr() if want_lse else None,
                                   int(kv_heads_per_chunk), workspace.data_ptr(),
                                   workspace.numel() * workspace.element_size(), _stream(dev))
    _raise("xattn_prefill_host", rc)
    return (out, lse) if want_lse else out


def xattn_prefill_varlen_workspace_bytes(shape: _Shape, seqlens: Sequence[int]) -> int:
    arr = (ctypes.c_int32 * len(seqlens))(*[int(x) for x in seqlens])
    return int(_lib().xattn_prefill_varlen_workspace_bytes(ctypes.byref(shape), len(seqlens),
                                                           arr))


def xattn_prefill_varlen(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor,
                         seqlens: Sequence[int], hq: int, hkv: int, B: int, S: int,
                         causal: bool, tau: Sequence[float], out: Optional[torch.Tensor] = None,
                         lse: Optional[torch.Tensor] | bool = None,
                         workspace: Optional[torch.Tensor] = None):
    """The whole step on sequences of different lengths, packed one after
    another: Q is [hq * T, d] with sequence i's [hq, L_i, d] block after the
    previous ones (T = sum of the lengths); K and V are [hkv * T, d]. Returns O
    packed like Q, or (O, lse) with lse [hq * T] when lse is True or a tensor."""
    _check(Q, "Q")
    _check(K, "K", Q.dtype)
    _check(V, "V", Q.dtype)
    lens = [int(x) for x in seqlens]
    T = sum(lens)
    if Q.dim() != 2 or Q.shape[0] != hq * T or K.shape != (hkv * T, Q.shape[1]) \
            or V.shape != K.shape:
        raise ValueError("expected Q [hq*T, d] and K, V [hkv*T, d] for T = sum(seqlens)")
    shape = make_shape(1, hq, hkv, max(max(lens), 1), Q.shape[1], B, S, causal, Q.dtype)
    if out is None:
        out = torch.empty_like(Q)
    _check(out, "O", Q.dtype)
    _check_shape(out, Q.shape, "O")
    want_lse = lse is not None and lse is not False
    if lse is True:
        lse = torch.empty(hq * T, device=Q.device, dtype=torch.float32)
    if want_lse:
        _check(lse, "lse", torch.float32)
        _check_shape(lse, (hq * T,), "lse")
    taus = _per_head(tau, hq, "tau", float)
    tarr = (ctypes.c_float * hq)(*taus)
    larr = (ctypes.c_int32 * len(lens))(*lens)
    need = int(_lib().xattn_prefill_varlen_workspace_bytes(ctypes.byref(shape), len(lens), larr))
    if workspace is None:
        workspace = torch.empty(max(need, 1), device=Q.device, dtype=torch.uint8)
    _check(workspace, "workspace")
    _same_device(Q, K, V, out, lse if want_lse else None, workspace)
    with torch.cuda.device(Q.device):
        rc = _lib().xattn_prefill_varlen(Q.data_ptr(), K.data_ptr(), V.data_ptr(),
                                         ctypes.byref(shape), len(lens), larr, tarr,
                                         out.data_ptr(), lse.data_ptr() if want_lse else None,
                                         workspace.data_ptr(),
                                         workspace.numel() * workspace.element_size(),
                                         _stream(Q.device))
    _raise("xattn_prefill_varlen", rc)
    return (out, lse) if want_lse else out


def xattn_selftest_timeout(device=None) -> None:
    """Launches the failure-detection self-test (see include/xattn.h): the next
    xattn_get_device_status on this stream returns XATTN_ERR_TIMEOUT."""
    _raise("xattn_selftest_timeout", _lib().xattn_selftest_timeout(_stream(device)))


def xattn_get_device_status(device=None) -> int:
    """Synchronises the current stream; returns the device status (0 = ok)."""
    return int(_lib().xattn_get_device_status(_stream(device)))
