"""xattn_prefill_varlen: sequences of different lengths, packed one after
another, through one call.

Each sequence must come out exactly as the batch-1 calls on that sequence
alone give it (torch.equal on O and lse); those calls are checked against
the oracle elsewhere, and one short sequence here is checked against the
oracle directly. Lengths cover a whole number of blocks, a short last
block, a sequence shorter than one block, and an empty sequence.
"""
import numpy as np
import pytest
import torch

import oracle.xattn_oracle as O
from block_sparse_long_score_b200 import (xattn_get_device_status, xattn_prefill_varlen,
                                          xattn_score_select, xattn_sparse_attn)
from block_sparse_long_score_b200.synth import make_problem
from tests import parity as PT

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _problems(name, lens, **kw):
    return [make_problem(name, L=L, seed=100 + i, **kw) if L else None
            for i, L in enumerate(lens)]


def _pack(probs, attr, heads):
    parts = [getattr(p, attr)[0].reshape(-1, p.d) for p in probs if p is not None]
    return torch.cat(parts).contiguous().to(DEV)


def _alone(p):
    Q, K, V = p.Q.to(DEV), p.K.to(DEV), p.V.to(DEV)
    _, counts, idx = xattn_score_select(Q, K, p.B, p.S, p.causal, p.tau.tolist())
    out, lse = xattn_sparse_attn(Q, K, V, counts, idx, p.B, p.causal, lse=True)
    return out[0].reshape(-1, p.d), lse[0].reshape(-1), counts, idx


@pytest.mark.parametrize("name,lens,kw", [
    ("c1", [2048, 1040, 48, 0, 4160, 128], dict(hq=4, hkv=2)),
    ("c4", [1280, 592, 1776], dict(hq=2, S=8)),          # non-causal, ragged lengths
    ("c0", [1024, 992, 40], {}),                         # fp32
])
def test_varlen_equals_each_sequence_alone(name, lens, kw):
    probs = _problems(name, lens, **kw)
    ref = next(p for p in probs if p is not None)
    hq, hkv = ref.hq, ref.hkv
    Q, K, V = _pack(probs, "Q", hq), _pack(probs, "K", hkv), _pack(probs, "V", hkv)
    out, lse = xattn_prefill_varlen(Q, K, V, lens, hq, hkv, ref.B, ref.S, ref.causal,
                                    ref.tau.tolist(), lse=True)
    torch.cuda.synchronize()
    assert xattn_get_device_status() == 0
    row = 0
    for p in probs:
        if p is None:
            continue
        o1, l1, _, _ = _alone(p)
        n = hq * p.L
        assert torch.equal(out[row:row + n], o1), p.L
        assert torch.equal(lse[row:row + n], l1), p.L
        row += n
    assert row == out.shape[0]


def test_varlen_short_sequence_against_the_oracle():
    """A 48-token sequence (less than one 128-token block) between two longer
    ones: its selection and output against the oracle."""
    lens = [256, 48, 384]
    probs = _problems("c1", lens, hq=2, hkv=1)
    Q, K, V = _pack(probs, "Q", 2), _pack(probs, "K", 1), _pack(probs, "V", 1)
    p = probs[1]
    out = xattn_prefill_varlen(Q, K, V, lens, 2, 1, p.B, p.S, p.causal, p.tau.tolist())
    torch.cuda.synchronize()
    o = PT.to_np(out[2 * 256: 2 * 256 + 2 * 48].float()).reshape(1, 2, 48, p.d)
    # one block of 48 tokens: P = [[1]], so the list is block 0 and the
    # output is plain causal attention over the 48 tokens
    P = O.block_probs(p.Q, p.K, p.B, p.S, p.causal)
    assert P.shape == (1, 2, 1, 1) and np.allclose(P, 1.0)
    lists = {(0, h, 0): [0] for h in range(2)}
    Oref, _ = O.sparse_attention(p.Q, p.K, p.V, p.B, p.causal, lists)
    assert np.max(np.abs(o - Oref)) <= PT.O_TOL["bf16"]
