"""Failure detection and output coverage on the GPU, without any GPU fault.

* Time-out path: a self-test kernel waits, with the library's bounded wait, on
  a barrier nothing completes. The device status must report the time-out,
  and the context must stay usable (a following call runs and is correct).
* Canary fills: every output is pre-filled with a sentinel. After a call,
  every element the header says is written must be written (no sentinel
  left), and nothing past a row's count in the index lists may be touched.
"""
import time

import numpy as np
import pytest
import torch

from block_sparse_long_score_b200 import (xattn_get_device_status, xattn_score,
                                          xattn_score_select, xattn_select,
                                          xattn_selftest_timeout, xattn_sparse_attn)
from block_sparse_long_score_b200.synth import make_problem

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
SENT = 0x7F7F7F7F   # sentinel of the integer outputs; floating outputs start as NaN


def _small():
    prob = make_problem("c1", L=2048, hq=2, hkv=1)
    return prob, prob.Q.to(DEV), prob.K.to(DEV), prob.V.to(DEV)


def test_timeout_is_reported_and_context_survives():
    assert xattn_get_device_status() == 0  # clears anything left over
    prob, Q, K, V = _small()
    taus = prob.tau.tolist()
    P = xattn_score(Q, K, prob.B, prob.S, prob.causal)
    _, counts, idx = xattn_select(P, taus, prob.causal)
    before = xattn_sparse_attn(Q, K, V, counts, idx, prob.B, prob.causal).clone()
    assert xattn_get_device_status() == 0

    t0 = time.time()
    xattn_selftest_timeout()
    status = xattn_get_device_status()
    waited = time.time() - t0
    assert status == -5, status            # XATTN_ERR_TIMEOUT
    assert waited > 1.0                    # the bounded wait really ran out
    assert xattn_get_device_status() == 0  # reading clears it

    after = xattn_sparse_attn(Q, K, V, counts, idx, prob.B, prob.causal)
    assert xattn_get_device_status() == 0
    assert torch.equal(before, after)


def _filled(shape, dtype):
    if dtype == torch.int32:
        return torch.full(shape, SENT, device=DEV, dtype=torch.int32)
    return torch.full(shape, float("nan"), device=DEV, dtype=dtype)


@pytest.mark.parametrize("causal_case", ["c1", "c4"])
def test_canary_every_output_written(causal_case):
    if causal_case == "c1":
        prob = make_problem("c1", L=2048, hq=2, hkv=1)
    else:
        prob = make_problem("c4", frames=2, frame_tokens=640, hq=2, S=16)
    Q, K, V = prob.Q.to(DEV), prob.K.to(DEV), prob.V.to(DEV)
    NB, W = prob.NB, (prob.NB + 31) // 32
    b, hq = 1, prob.hq
    taus = prob.tau.tolist()

    probs = _filled((b, hq, NB, NB), torch.float32)
    xattn_score(Q, K, prob.B, prob.S, prob.causal, probs=probs)
    mask = _filled((b, hq, NB, W), torch.int32)
    counts = _filled((b, hq, NB), torch.int32)
    idx = _filled((b, hq, NB, NB), torch.int32)
    xattn_select(probs, taus, prob.causal, out=(mask, counts, idx))
    out = torch.full_like(Q, float("nan"))
    lse = _filled((b, hq, prob.L), torch.float32)
    xattn_sparse_attn(Q, K, V, counts, idx, prob.B, prob.causal, out=out, lse=lse)
    m2 = _filled((b, hq, NB, W), torch.int32)
    c2 = _filled((b, hq, NB), torch.int32)
    i2 = _filled((b, hq, NB, NB), torch.int32)
    p2 = _filled((b, hq, NB, NB), torch.float32)
    xattn_score_select(Q, K, prob.B, prob.S, prob.causal, taus, probs=p2, out=(m2, c2, i2))
    torch.cuda.synchronize()
    assert xattn_get_device_status() == 0

    for P in (probs, p2):
        assert torch.all(torch.isfinite(P))      # every entry written (no NaN left)
        if prob.causal:
            assert torch.all(torch.triu(P[0, 0], 1) == 0)
    for m, c, ix in ((mask, counts, idx), (m2, c2, i2)):
        assert not torch.any(c == SENT)
        cn = c.cpu().numpy()
        ixn = ix.cpu().numpy()
        mn = m.cpu().numpy().view(np.uint32)
        # bits past NB in the last mask word are zero, every word written
        if NB % 32:
            assert np.all((mn[..., -1] >> (NB % 32)) == 0)
        for h in range(hq):
            for qb in range(NB):
                n = int(cn[0, h, qb])
                assert 1 <= n <= (qb + 1 if prob.causal else NB)
                assert np.all(ixn[0, h, qb, :n] != SENT)
                assert np.all(ixn[0, h, qb, n:] == SENT)   # nothing written past the count
    assert torch.all(torch.isfinite(out.float()))   # every row of O written
    assert torch.all(torch.isfinite(lse))           # every row has a visible key here


def test_binding_rejects_buffers_of_the_wrong_shape():
    """The binding checks every caller-passed buffer against the shape before
    the call: a buffer too small for what the kernels write or read raises
    here instead of reaching the GPU."""
    from block_sparse_long_score_b200 import xattn_sparse_attn_noalloc
    prob, Q, K, V = _small()
    taus = prob.tau.tolist()
    P = xattn_score(Q, K, prob.B, prob.S, prob.causal)
    mask, counts, idx = xattn_select(P, taus, prob.causal)
    torch.cuda.synchronize()
    bad_calls = [
        lambda: xattn_sparse_attn(Q, K, V[:, :, :-128], counts, idx, prob.B, prob.causal),
        lambda: xattn_sparse_attn(Q, K, V, counts[..., :-1], idx, prob.B, prob.causal),
        lambda: xattn_sparse_attn(Q, K, V, counts, idx[..., :-1], prob.B, prob.causal),
        lambda: xattn_sparse_attn(Q, K, V, counts, idx, prob.B, prob.causal,
                                  out=torch.empty_like(Q)[:, :, :-1]),
        lambda: xattn_sparse_attn(Q, K, V, counts, idx, prob.B, prob.causal,
                                  lse=torch.empty(Q.shape[:2], device=DEV)),
        lambda: xattn_sparse_attn_noalloc(Q, K, V, counts, idx, prob.B, prob.causal,
                                          torch.empty_like(Q)[:, :1]),
        lambda: xattn_sparse_attn_noalloc(Q, K, V, counts, idx, prob.B, prob.causal,
                                          torch.empty_like(Q),
                                          torch.empty(Q.shape[:3][:-1] + (7,), device=DEV)),
        lambda: xattn_sparse_attn_noalloc(Q, K, V[:, :, :-128], counts, idx, prob.B,
                                          prob.causal, torch.empty_like(Q)),
        lambda: xattn_score(Q, K, prob.B, prob.S, prob.causal, probs=P[..., :-1]),
        lambda: xattn_select(P, taus, prob.causal, out=(mask[..., :-1], counts, idx)),
        lambda: xattn_score_select(Q, K, prob.B, prob.S, prob.causal, taus,
                                   out=(mask, counts[:, :1], idx)),
    ]
    for i, call in enumerate(bad_calls):
        with pytest.raises(ValueError):
            call()
            pytest.fail(f"bad call {i} was accepted")
    assert xattn_get_device_status() == 0
