"""xattn_score_select (scoring, block sums and find_blocks in one call)
against xattn_score followed by xattn_select.

The fused kernel computes each row of P with the reduce kernel's arithmetic,
so P is bit-identical. Its cut comes from the histogram search, while the
two-call path first walks the ranking in order; both add the probabilities
in fp64, so they can differ only where a running sum lies within a rounding
step of tau, which no row of these inputs does. Masks, counts and lists must
therefore agree bit for bit. The two-call path is itself checked against the
oracle in the parity tests.
"""
import numpy as np
import pytest
import torch

import oracle.xattn_oracle as O
from block_sparse_long_score_b200 import (xattn_get_device_status, xattn_score,
                                          xattn_score_select, xattn_select)
from block_sparse_long_score_b200.synth import make_problem
from tests import parity as PT

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _both(prob, tau=None):
    Q, K = prob.Q.to(DEV), prob.K.to(DEV)
    taus = prob.tau.tolist() if tau is None else tau
    P = xattn_score(Q, K, prob.B, prob.S, prob.causal)
    m1, c1, i1 = xattn_select(P, taus, prob.causal)
    P2, m2, c2, i2 = xattn_score_select(Q, K, prob.B, prob.S, prob.causal, taus, probs=True)
    m3, c3, i3 = xattn_score_select(Q, K, prob.B, prob.S, prob.causal, taus)
    torch.cuda.synchronize()
    assert xattn_get_device_status() == 0
    return (P, m1, c1, i1), (P2, m2, c2, i2), (m3, c3, i3)


def _assert_same_lists(c1, i1, c2, i2):
    assert torch.equal(c1, c2)
    NB = i1.shape[-1]
    ar = torch.arange(NB, device=i1.device)
    valid = ar[None, None, None, :] < c1[..., None]
    assert torch.equal(torch.where(valid, i1, 0), torch.where(valid, i2, 0))


@pytest.mark.parametrize("name,kw", [
    ("c0", {}),
    ("c1", dict(L=4096, hq=4, hkv=2)),
    ("c2", dict(L=8192, hq=4, hkv=1)),
    ("c4", dict(frames=3, frame_tokens=640, hq=2, S=16)),
    ("c4", dict(frames=3, frame_tokens=640, hq=2, S=4)),
    ("c1", dict(L=76800, hq=2, hkv=1)),          # rows of 513..600 blocks: two passes (r = 16)
    ("c4", dict(frames=3, frame_tokens=12800, hq=1, S=4)),  # 300-block rows, r = 32
])
def test_fused_equals_two_calls(name, kw):
    prob = make_problem(name, **kw)
    (P, m1, c1, i1), (P2, m2, c2, i2), (m3, c3, i3) = _both(prob)
    assert torch.equal(P, P2)
    assert torch.equal(m1, m2) and torch.equal(m1, m3)
    _assert_same_lists(c1, i1, c2, i2)
    _assert_same_lists(c1, i1, c3, i3)


@pytest.mark.parametrize("tau", [0.5, 0.99, 1.0])
def test_fused_thresholds(tau):
    """Peaked and flat selections (ranked walk and histogram search), and the
    full mask at tau = 1."""
    prob = make_problem("c1", L=4096, hq=2, hkv=1)
    (P, m1, c1, i1), (P2, m2, c2, i2), _ = _both(prob, [tau] * prob.hq)
    assert torch.equal(m1, m2)
    _assert_same_lists(c1, i1, c2, i2)
    if tau == 1.0:
        NB = prob.NB
        assert torch.equal(c2[0, 0].cpu(), torch.arange(1, NB + 1, dtype=torch.int32))


def test_fused_matches_oracle_selection():
    """find_blocks of the oracle on the fused call's own P gives its mask."""
    prob = make_problem("c1", L=4096, hq=4, hkv=2)
    Q, K = prob.Q.to(DEV), prob.K.to(DEV)
    P, mask, counts, idx = xattn_score_select(Q, K, prob.B, prob.S, prob.causal,
                                              prob.tau.tolist(), probs=True)
    Pn = PT.to_np(P).astype(np.float64)
    mb = PT.mask_to_bool(PT.to_np(mask), prob.NB)
    for h in range(prob.hq):
        for b in range(prob.NB):
            want = np.zeros(prob.NB, bool)
            want[O.find_blocks(Pn[0, h, b, : b + 1], float(prob.tau[h]))] = True
            assert np.array_equal(mb[0, h, b], want), (h, b)


def test_fused_full_size():
    """The 128K Llama layer, as bench.py runs it."""
    prob = make_problem("c2")
    (P, m1, c1, i1), (P2, m2, c2, i2), (m3, c3, i3) = _both(prob)
    assert torch.equal(P, P2)
    assert torch.equal(m1, m2) and torch.equal(m1, m3)
    _assert_same_lists(c1, i1, c2, i2)


@pytest.mark.parametrize("name,kw,blocks", [
    ("c4", dict(frames=3, frame_tokens=12800, hq=1, S=4), [0, 150, 299]),
    ("c1", dict(L=76800, hq=1, hkv=1), [0, 511, 512, 599]),
])
def test_long_rows_match_oracle(name, kw, blocks):
    """Rows longer than one register pass of the reduction (two passes over the
    partials) against the oracle's P, and its find_blocks on the GPU's P."""
    prob = make_problem(name, **kw)
    Q, K = prob.Q.to(DEV), prob.K.to(DEV)
    P, mask, counts, idx = xattn_score_select(Q, K, prob.B, prob.S, prob.causal,
                                              prob.tau.tolist(), probs=True)
    torch.cuda.synchronize()
    Pg = PT.to_np(P).astype(np.float64)
    Pref = O.block_probs(prob.Q, prob.K, prob.B, prob.S, prob.causal, heads=[0],
                         q_blocks=blocks)
    assert PT.check_probs(Pg[0, 0, blocks], Pref[0, 0, blocks]) <= 1.0
    mb = PT.mask_to_bool(PT.to_np(mask), prob.NB)
    for b in blocks:
        n = b + 1 if prob.causal else prob.NB
        want = np.zeros(prob.NB, bool)
        want[O.find_blocks(Pg[0, 0, b, :n], float(prob.tau[0]))] = True
        assert np.array_equal(mb[0, 0, b], want), b
