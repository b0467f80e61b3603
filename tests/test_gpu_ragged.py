"""GPU parity for lengths that B does not divide: the last query and key
block is shorter (NB = ceil(L / B); L stays a multiple of S).

Every path is checked against the oracle: P (the short last row divides by
its own reshaped-row count), the selection, and the attention, whose last
block has fewer queries (rows past L are never written) and fewer keys
(non-causal lists mask the missing columns). The fused call, the no-alloc
attention and the host-buffer call must agree with the plain calls bit for
bit.
"""
import numpy as np
import pytest
import torch

from block_sparse_long_score_b200 import (xattn_get_device_status, xattn_prefill_host,
                                          xattn_score, xattn_score_select, xattn_select,
                                          xattn_sparse_attn, xattn_sparse_attn_noalloc)
from block_sparse_long_score_b200.synth import make_problem
from tests.test_gpu_parity import check_problem, run_gpu, sample_blocks

pytestmark = pytest.mark.gpu

DEV = "cuda:0"

RAGGED = [
    ("c0", dict(L=992)),                                         # fp32, 32-token last block
    ("c1", dict(L=2496, hq=4, hkv=2)),                           # S = 8: 8 of 16 reshaped rows
    ("c1", dict(L=1088, hq=2, hkv=1, S=2)),                      # r = 64: a block spans 2 chunks
    ("c1", dict(L=1040, hq=2, hkv=1, S=1)),                      # r = 128, 16-token last block
    ("c2", dict(L=9296, hq=4, hkv=1)),                           # S = 16: 5 of 8 reshaped rows
    ("c4", dict(frames=3, frame_tokens=592, hq=2, S=4)),         # non-causal, 112-token last block
    ("c4", dict(frames=3, frame_tokens=592, hq=2, S=16)),
]


@pytest.mark.parametrize("name,kw", RAGGED)
def test_ragged_full_parity(name, kw):
    prob = make_problem(name, **kw)
    assert prob.L % prob.B != 0 and prob.L % prob.S == 0
    res = run_gpu(prob)
    assert res["P"].shape[-1] == prob.NB
    np.testing.assert_allclose(res["P"].sum(axis=-1), 1.0, atol=1e-4)
    check_problem(prob, list(range(prob.hq)), list(range(prob.NB)), res)


def test_ragged_rows_past_L_are_not_written():
    """O and lse have exactly L rows; the canary past the end of a larger
    buffer view stays untouched (the kernel stores no row past L)."""
    prob = make_problem("c4", frames=3, frame_tokens=592, hq=2, S=8)
    Q, K, V = prob.Q.to(DEV), prob.K.to(DEV), prob.V.to(DEV)
    _, counts, idx = xattn_score_select(Q, K, prob.B, prob.S, prob.causal, prob.tau.tolist())
    # O for head h lives at rows [h*L, (h+1)*L) of one buffer with a tail guard
    buf = torch.full((prob.hq * prob.L + 256, prob.d), float("nan"), device=DEV,
                     dtype=torch.bfloat16)
    out = buf[: prob.hq * prob.L].view(1, prob.hq, prob.L, prob.d)
    xattn_sparse_attn(Q, K, V, counts, idx, prob.B, prob.causal, out=out)
    torch.cuda.synchronize()
    assert xattn_get_device_status() == 0
    assert torch.isfinite(out.float()).all()
    assert torch.isnan(buf[prob.hq * prob.L:].float()).all()


@pytest.mark.parametrize("name,kw", [("c1", dict(L=2496, hq=4, hkv=2)),
                                     ("c4", dict(frames=3, frame_tokens=592, hq=2, S=8))])
def test_ragged_every_path_bit_exact(name, kw):
    prob = make_problem(name, **kw)
    Q, K, V = prob.Q.to(DEV), prob.K.to(DEV), prob.V.to(DEV)
    taus = prob.tau.tolist()
    P = xattn_score(Q, K, prob.B, prob.S, prob.causal)
    mask, counts, idx = xattn_select(P, taus, prob.causal)
    out, lse = xattn_sparse_attn(Q, K, V, counts, idx, prob.B, prob.causal, lse=True)
    P2, mask2, counts2, idx2 = xattn_score_select(Q, K, prob.B, prob.S, prob.causal, taus,
                                                  probs=True)
    out2 = torch.empty_like(Q)
    xattn_sparse_attn_noalloc(Q, K, V, counts, idx, prob.B, prob.causal, out2)
    torch.cuda.synchronize()
    assert torch.equal(P, P2) and torch.equal(mask, mask2) and torch.equal(counts, counts2)
    assert torch.equal(out, out2)
    out3, lse3 = xattn_prefill_host(prob.Q.contiguous().pin_memory(),
                                    prob.K.contiguous().pin_memory(),
                                    prob.V.contiguous().pin_memory(), prob.B, prob.S,
                                    prob.causal, taus, lse=True)
    torch.cuda.synchronize()
    assert xattn_get_device_status() == 0
    assert torch.equal(out3, out.cpu()) and torch.equal(lse3, lse.cpu())


def test_ragged_large_sampled():
    """A 32K-class Llama layer (all 32 heads) whose length ends 88 tokens
    into a block, checked on sampled heads and query blocks, the short last
    block included."""
    prob = make_problem("c1", L=32728)
    assert prob.L % prob.B == 88
    res = run_gpu(prob)
    check_problem(prob, [0, 17, 31], sample_blocks(prob.NB, k=24, seed=5), res)
