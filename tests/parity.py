"""Comparison helpers for the GPU-vs-oracle parity tests.

Tolerances:
* P (block probabilities): |P_gpu - P_oracle| <= 1e-3 * P_oracle + 1e-9.
  The 1e-9 floor covers fp32 underflow of blocks whose probability is
  negligible.
* Masks: exact, except blocks whose oracle cumulative sum (fp64, in the
  oracle's ranked order) lies within 1e-4 of tau. The block at ranked
  position t is exempt if |C_{t-1} - tau| <= 1e-4 or |C_t - tau| <= 1e-4.
* Outputs, given the GPU's own mask: max |O_gpu - O_oracle| <= 2e-2 for bf16
  and <= 1e-4 for fp32.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle.xattn_oracle as O

P_RTOL, P_ATOL = 1e-3, 1e-9
TAU_BAND = 1e-4
O_TOL = {"bf16": 2e-2, "f32": 1e-4}
LSE_TOL = {"bf16": 2e-3, "f32": 1e-5}


def mask_to_bool(mask_words: np.ndarray, NB: int) -> np.ndarray:
    """uint32 words [..., ceil(NB/32)] -> bool [..., NB]."""
    w = mask_words.astype(np.int64) & 0xFFFFFFFF
    bits = (w[..., :, None] >> np.arange(32)[None, :]) & 1
    return bits.reshape(*w.shape[:-1], -1)[..., :NB].astype(bool)


def lists_from(counts: np.ndarray, idx: np.ndarray, bb: int, h: int, blocks) -> dict:
    return {b: [int(x) for x in idx[bb, h, b, : counts[bb, h, b]]] for b in blocks}


def check_probs(P_gpu: np.ndarray, P_ref: np.ndarray) -> float:
    """Returns the worst ratio of |error| to the allowed bound (<= 1 passes)."""
    if not np.all(np.isfinite(P_gpu)):
        return float("inf")
    err = np.abs(P_gpu.astype(np.float64) - P_ref)
    bound = P_RTOL * np.abs(P_ref) + P_ATOL
    return float(np.max(err / bound))


def compare_row_masks(p_ref: np.ndarray, tau: float, n_allowed: int, sel_gpu: np.ndarray):
    """(mismatches not exempt, exempt blocks, mismatches total) for one row."""
    p = p_ref[:n_allowed]
    want = np.zeros(n_allowed, bool)
    want[O.find_blocks(p, tau)] = True
    got = sel_gpu[:n_allowed]
    extra = sel_gpu[n_allowed:].any()
    order = np.lexsort((np.arange(n_allowed), -p))
    csum = np.cumsum(p[order])
    before = np.concatenate([[0.0], csum[:-1]])
    exempt_pos = (np.abs(before - tau) <= TAU_BAND) | (np.abs(csum - tau) <= TAU_BAND)
    exempt = np.zeros(n_allowed, bool)
    exempt[order[exempt_pos]] = True
    if tau >= 1.0:
        exempt[:] = False
    diff = got != want
    bad = int(np.sum(diff & ~exempt)) + (1 if extra else 0)
    return bad, int(np.sum(exempt)), int(np.sum(diff))


def check_lists(mask_bool: np.ndarray, counts: np.ndarray, idx: np.ndarray) -> None:
    """counts and idx must describe exactly the set bits, ascending."""
    it = np.ndindex(*counts.shape)
    for key in it:
        c = int(counts[key])
        got = idx[key][:c]
        want = np.nonzero(mask_bool[key])[0]
        assert c == want.size, (key, c, want.size)
        assert np.array_equal(got, want), key


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").numpy()
