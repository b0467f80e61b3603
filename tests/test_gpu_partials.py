"""xattn_score_partials (the scoring GEMM alone) against the oracle.

The oracle gives the raw reshaped logits Q_r K_r^T; scaled by 1/sqrt(d S), the
partial of reshaped row rho and key block j is log2 of the sum of 2^(x log2 e)
over the block's visible columns, as the header defines it. The test unpacks
the GPU's workspace with the header's layout and compares every partial. It
then forms P from the partials with the header's formula in float64 and checks
it against the oracle's P (the tolerance of the other P parity tests), and
against xattn_score's P, which the reduce kernel forms from the same partials.
"""
import math

import numpy as np
import pytest
import torch

import oracle.xattn_oracle as O
from block_sparse_long_score_b200 import (xattn_get_device_status, xattn_score,
                                          xattn_score_partials)
from block_sparse_long_score_b200.synth import make_problem
from tests import parity as PT

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
L_ATOL = 2e-3   # log2 units: bf16 products summed in fp32, and the approximate exp2 / log2


def _row_offset(rho, r, NB, causal):
    if not causal:
        return rho * NB
    b, t = divmod(rho, r)
    return r * b * (b + 1) // 2 + t * (b + 1)


def _oracle_partials(q, k, B, S, causal):
    """[R, NB] partials of one head from the oracle's reshaped logits (NaN where
    a block is not allowed)."""
    d = q.shape[1]
    x = O.reshaped_logits(q, k, S) / math.sqrt(d * S)
    R = x.shape[0]
    r = B // S
    NB = -(-R // r)
    out = np.full((R, NB), np.nan)
    for rho in range(R):
        for j in range(NB if not causal else rho // r + 1):
            c0, c1 = j * r, min((j + 1) * r, R)
            cols = x[rho, c0:c1]
            if causal:
                cols = cols[: max(0, min(c1, rho + 1) - c0)]
            m = cols.max()
            out[rho, j] = (m + math.log(np.exp(cols - m).sum())) / math.log(2.0)
    return out


@pytest.mark.parametrize("case", [
    dict(name="c1", L=1024, hq=2, hkv=1, causal=None),        # pair kernel (S = 16), causal
    dict(name="c1", L=1000, hq=2, hkv=1, S=8, causal=None),   # ragged last block
    dict(name="c4", frames=2, frame_tokens=512, hq=2, S=8, causal=None),  # non-causal
    dict(name="c4", frames=2, frame_tokens=512, hq=2, S=4, causal=None),  # one-CTA kernel
    dict(name="c0", causal=None),                             # fp32 CUDA-core path
])
def test_partials_match_oracle(case):
    kw = {k: v for k, v in case.items() if k not in ("name", "causal") and v is not None}
    prob = make_problem(case["name"], **kw)
    Q, K = prob.Q.to(DEV), prob.K.to(DEV)
    ws = xattn_score_partials(Q, K, prob.B, prob.S, prob.causal)
    P_gpu = xattn_score(Q, K, prob.B, prob.S, prob.causal).cpu().numpy()
    torch.cuda.synchronize()
    assert xattn_get_device_status() == 0
    r = prob.B // prob.S
    R = prob.L // prob.S
    NB = prob.NB
    per_head = r * NB * (NB + 1) // 2 if prob.causal else R * NB
    flat = ws[: prob.batch * prob.hq * per_head * 4].view(torch.float32).cpu().numpy()
    for bb in range(prob.batch):
        for h in range(prob.hq):
            bh = bb * prob.hq + h
            kv = O.kv_head(h, prob.hq, prob.hkv)
            q, k = O.to_f64(prob.Q[bb, h]), O.to_f64(prob.K[bb, kv])
            ref = _oracle_partials(q, k, prob.B, prob.S, prob.causal)
            head = flat[bh * per_head:(bh + 1) * per_head].astype(np.float64)
            Lp = np.full((R, NB), np.nan)
            for rho in range(R):
                n = rho // r + 1 if prob.causal else NB
                o = _row_offset(rho, r, NB, prob.causal)
                Lp[rho, :n] = head[o:o + n]
            allowed = ~np.isnan(ref)
            assert np.array_equal(allowed, ~np.isnan(Lp))
            err = np.abs(Lp[allowed] - ref[allowed])
            assert err.max() <= L_ATOL, (case, bh, float(err.max()))
            # P from the partials, by the header's formula, in float64
            m = np.nanmax(Lp, axis=1)
            lse = m + np.log2(np.nansum(np.exp2(Lp - m[:, None]), axis=1))
            P = np.zeros((NB, NB))
            for b in range(NB):
                rows = range(b * r, min((b + 1) * r, R))
                acc = np.zeros(NB)
                for rho in rows:
                    acc += np.nan_to_num(np.exp2(Lp[rho] - lse[rho]), nan=0.0)
                P[b] = acc / len(rows)
            P_ref = O.block_probs_head(q, k, prob.B, prob.S, prob.causal)
            assert PT.check_probs(P, P_ref) <= 1.0, case
            assert PT.check_probs(P_gpu[bb, h], P) <= 1.0, case
