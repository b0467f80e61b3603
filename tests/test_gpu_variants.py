"""GPU parity of the ablation variants against the fp64 CPU oracle.

* Sampling patterns (xattn_score_pattern): the diagonal and random-permutation
  patterns of the sparsity-pattern ablation. P is compared element by element
  with the oracle's block probabilities under the same permutation, within the
  P tolerance of the antidiagonal path.
* Fixed budgets (xattn_select_topk / xattn_select_topratio): selection turns
  fp32 values into integers, so on the same fp32 rows the GPU must keep
  exactly the oracle's blocks (mask, counts and index lists). The rows reach
  every path of the kernel: early cuts at a bucket boundary, cuts inside
  groups of more than 32 equal values, zeros, subnormals, k >= allowed.
"""
import numpy as np
import pytest
import torch

import oracle.xattn_oracle as O
from block_sparse_long_score_b200 import (antidiagonal_perm, diagonal_perm,
                                          xattn_get_device_status, xattn_score,
                                          xattn_score_pattern, xattn_select_topk,
                                          xattn_select_topratio)
from block_sparse_long_score_b200.synth import make_problem
from tests import parity as PT

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _perm(kind, S, seed=0):
    if kind == "diagonal":
        return diagonal_perm(S)
    if kind == "antidiagonal":
        return antidiagonal_perm(S)
    return [int(x) for x in np.random.default_rng(1000 + S + seed).permutation(S)]


# ------------------------------------------------------------ patterns ----
@pytest.mark.parametrize("name,kw", [
    ("c0", {}),                                              # fp32 CUDA-core path
    ("c1", dict(L=4096, hq=4, hkv=2)),
    ("c4", dict(frames=3, frame_tokens=640, hq=2, S=16)),    # non-causal, ragged tiles
    ("c4", dict(frames=3, frame_tokens=640, hq=2, S=4)),
])
@pytest.mark.parametrize("kind", ["diagonal", "random"])
def test_pattern_probs_small(name, kw, kind):
    prob = make_problem(name, **kw)
    perm = _perm(kind, prob.S)
    Q, K = prob.Q.to(DEV), prob.K.to(DEV)
    P = xattn_score_pattern(Q, K, prob.B, prob.S, prob.causal, perm)
    torch.cuda.synchronize()
    assert xattn_get_device_status() == 0
    P_ref = O.block_probs(prob.Q, prob.K, prob.B, prob.S, prob.causal, perm=perm)
    worst = PT.check_probs(PT.to_np(P), P_ref)
    assert worst <= 1.0, f"P error {worst:.3g} x tolerance"


@pytest.mark.parametrize("name,kw", [("c0", {}), ("c1", dict(L=2048, hq=2, hkv=1))])
def test_antidiagonal_pattern_is_xattn_score(name, kw):
    """The antidiagonal permutation reproduces xattn_score bit for bit."""
    prob = make_problem(name, **kw)
    Q, K = prob.Q.to(DEV), prob.K.to(DEV)
    P1 = xattn_score(Q, K, prob.B, prob.S, prob.causal)
    P2 = xattn_score_pattern(Q, K, prob.B, prob.S, prob.causal, antidiagonal_perm(prob.S))
    torch.cuda.synchronize()
    assert torch.equal(P1, P2)


def test_pattern_changes_the_scores():
    """The diagonal pattern is a different function (guards against a kernel
    that ignores the permutation)."""
    prob = make_problem("c1", L=2048, hq=2, hkv=1)
    Q, K = prob.Q.to(DEV), prob.K.to(DEV)
    P1 = xattn_score(Q, K, prob.B, prob.S, prob.causal)
    P2 = xattn_score_pattern(Q, K, prob.B, prob.S, prob.causal, diagonal_perm(prob.S))
    torch.cuda.synchronize()
    assert (P1 - P2).abs().max().item() > 1e-4


def test_pattern_full_size_sampled():
    """The 128K Llama layer with the diagonal and a random pattern, checked on
    sampled heads and query blocks (first and last included)."""
    prob = make_problem("c2")
    Q, K = prob.Q.to(DEV), prob.K.to(DEV)
    heads = [0, 13, 31]
    rng = np.random.default_rng(3)
    qblocks = sorted(set([0, prob.NB - 1] + rng.choice(prob.NB, 10, replace=False).tolist()))
    for kind in ("diagonal", "random"):
        perm = _perm(kind, prob.S, seed=7)
        P = PT.to_np(xattn_score_pattern(Q, K, prob.B, prob.S, prob.causal, perm))
        assert xattn_get_device_status() == 0
        P_ref = O.block_probs(prob.Q, prob.K, prob.B, prob.S, prob.causal, heads=heads,
                              q_blocks=qblocks, perm=perm)
        for h in heads:
            worst = PT.check_probs(P[0, h, qblocks], P_ref[0, h, qblocks])
            assert worst <= 1.0, (kind, h, worst)


# ------------------------------------------------------------- budgets ----
def _budget_rows(NB, kind, rng, causal):
    P = np.zeros((NB, NB))
    for b in range(NB):
        n = b + 1 if causal else NB
        if kind == "dirichlet":
            p = rng.dirichlet(np.ones(n) * rng.choice([0.05, 0.3, 1.0, 5.0]))
        elif kind == "flat":
            p = np.full(n, 1.0 / n)
        elif kind == "ties":        # > 32 equal values above and at the cut
            p = np.full(n, 1e-4)
            m = min(n, 40)
            p[rng.choice(n, size=m, replace=False)] = 0.5 / m
        elif kind == "zeros":
            p = rng.dirichlet(np.ones(n) * 0.2)
            p[rng.random(n) < 0.5] = 0.0
        elif kind == "subnormal":   # exponents over the whole fp32 range
            p = 2.0 ** -rng.uniform(0, 149, size=n)
            p[rng.random(n) < 0.1] = 2.0 ** -140
        elif kind == "bucket":      # values on a few exact levels: cuts at bucket edges
            p = rng.choice([0.5, 0.25, 0.125, 2.0 ** -20], size=n)
        P[b, :n] = p
    return P


def _run_budget(P, arg, causal, mode):
    Pt = torch.from_numpy(P.astype(np.float32)).to(DEV)
    if mode == "topk":
        mask, counts, idx = xattn_select_topk(Pt, arg, causal)
    else:
        mask, counts, idx = xattn_select_topratio(Pt, arg, causal)
    torch.cuda.synchronize()
    NB = P.shape[-1]
    return PT.mask_to_bool(PT.to_np(mask), NB), PT.to_np(counts), PT.to_np(idx)


def _check_budget(P, arg, causal, mode, rows=None):
    m, c, ix = _run_budget(P, arg, causal, mode)
    P32 = P.astype(np.float32).astype(np.float64)
    _, hq, NB, _ = P.shape
    for h in range(hq):
        for b in (range(NB) if rows is None else rows):
            n = b + 1 if causal else NB
            k = int(arg[h]) if mode == "topk" else O.top_ratio_count(float(arg[h]), n)
            want = np.zeros(NB, bool)
            want[O.top_k_blocks(P32[0, h, b, :n], k)] = True
            assert np.array_equal(m[0, h, b], want), (mode, h, b, np.nonzero(m[0, h, b] != want))
            assert c[0, h, b] == want.sum()
            assert np.array_equal(ix[0, h, b, : c[0, h, b]], np.nonzero(want)[0])


@pytest.mark.parametrize("NB", [1, 7, 33, 100, 600, 2048])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("kind", ["dirichlet", "flat", "ties", "zeros", "subnormal", "bucket"])
@pytest.mark.parametrize("mode", ["topk", "topratio"])
def test_budget_exact(NB, causal, kind, mode):
    if NB == 2048 and not causal and kind not in ("dirichlet", "ties"):
        pytest.skip("covered by the causal case")
    rng = np.random.default_rng(NB * 13 + causal * 5 + len(kind) + len(mode))
    hq = 4
    P = np.stack([_budget_rows(NB, kind, rng, causal) for _ in range(hq)])[None]
    arg = [1, 5, 64, 4096] if mode == "topk" else [0.27, 0.5, 0.01, 1.0]
    _check_budget(P, arg, causal, mode)


def test_budget_full_size():
    """Top-K (8192 tokens = 64 blocks) and Top-Ratio (27 %), the ablation's
    settings, on the GPU's own P of the 128K Llama layer: every row of two
    heads, checked exactly."""
    prob = make_problem("c2")
    Q, K = prob.Q.to(DEV), prob.K.to(DEV)
    P = xattn_score(Q, K, prob.B, prob.S, prob.causal)
    for mode, arg in (("topk", [64] * prob.hq), ("topratio", [0.27] * prob.hq)):
        fn = xattn_select_topk if mode == "topk" else xattn_select_topratio
        mask, counts, idx = fn(P, arg, prob.causal)
        torch.cuda.synchronize()
        assert xattn_get_device_status() == 0
        Pn = PT.to_np(P[:, [0, 31]]).astype(np.float64)
        mb = PT.mask_to_bool(PT.to_np(mask[:, [0, 31]]), prob.NB)
        cn = PT.to_np(counts[:, [0, 31]])
        ixn = PT.to_np(idx[:, [0, 31]])
        for hh in range(2):
            for b in range(prob.NB):
                n = b + 1
                k = arg[0] if mode == "topk" else O.top_ratio_count(arg[0], n)
                want = O.top_k_blocks(Pn[0, hh, b, :n], k)
                assert cn[0, hh, b] == len(want), (mode, hh, b)
                assert np.array_equal(ixn[0, hh, b, : len(want)], want), (mode, hh, b)
                assert mb[0, hh, b].sum() == len(want)
