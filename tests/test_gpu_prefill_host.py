"""xattn_prefill_host: the whole step on host tensors, with the copies
overlapped with the compute chunk by chunk.

Every step of the method is independent across KV heads, so cutting the layer
into KV-head chunks must not change a single bit: O and lse are compared with
torch.equal against xattn_score_select + xattn_sparse_attn on device copies,
for every chunk size (ragged last chunks included), a batch of two, the fp32
path, and the full 128K Llama layer. One case also goes to the oracle
directly.
"""
import numpy as np
import pytest
import torch

import oracle.xattn_oracle as O
from block_sparse_long_score_b200 import (xattn_get_device_status, xattn_prefill_host,
                                          xattn_score_select, xattn_sparse_attn)
from block_sparse_long_score_b200.synth import make_problem
from tests import parity as PT

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _device_reference(prob):
    Q, K, V = prob.Q.to(DEV), prob.K.to(DEV), prob.V.to(DEV)
    mask, counts, idx = xattn_score_select(Q, K, prob.B, prob.S, prob.causal, prob.tau.tolist())
    out, lse = xattn_sparse_attn(Q, K, V, counts, idx, prob.B, prob.causal, lse=True)
    torch.cuda.synchronize()
    return out.cpu(), lse.cpu(), counts.cpu(), idx.cpu()


def _pinned(t):
    return t.contiguous().pin_memory()


def _host_run(prob, ck, lse=True):
    Qh, Kh, Vh = _pinned(prob.Q), _pinned(prob.K), _pinned(prob.V)
    res = xattn_prefill_host(Qh, Kh, Vh, prob.B, prob.S, prob.causal, prob.tau.tolist(),
                             lse=lse, kv_heads_per_chunk=ck)
    torch.cuda.synchronize()
    assert xattn_get_device_status() == 0
    return res


@pytest.mark.parametrize("ck", [0, 1, 3, 8])
def test_chunking_is_bit_exact(ck):
    """8 KV heads in chunks of 1, 3 (3 + 3 + 2: a ragged last chunk) and 8."""
    prob = make_problem("c1", L=2048, hq=16, hkv=8)
    O_ref, l_ref, _, _ = _device_reference(prob)
    out, lse = _host_run(prob, ck)
    assert not out.is_cuda and out.is_pinned()
    assert torch.equal(out, O_ref)
    assert torch.equal(lse, l_ref)


def test_batch_of_two_and_no_lse():
    prob = make_problem("c1", L=2048, hq=4, hkv=2, batch=2)
    O_ref, _, _, _ = _device_reference(prob)
    out = _host_run(prob, 1, lse=None)
    assert torch.equal(out, O_ref)
    assert (out[0].float() - out[1].float()).abs().max().item() > 0.1


def test_fp32_path():
    prob = make_problem("c0")
    O_ref, l_ref, _, _ = _device_reference(prob)
    out, lse = _host_run(prob, 0)
    assert torch.equal(out, O_ref) and torch.equal(lse, l_ref)


def test_device_tensors_and_stream_order():
    """Device pointers are accepted as well, and the call is ordered after the
    work queued before it on the stream: Q is produced by a kernel queued just
    before the call."""
    prob = make_problem("c1", L=1024, hq=4, hkv=2)
    O_ref, _, _, _ = _device_reference(prob)
    Qs = prob.Q.to(DEV)
    K, V = prob.K.to(DEV), prob.V.to(DEV)
    torch.cuda.synchronize()
    Q = torch.empty_like(Qs)
    Q.copy_(Qs)               # queued on the current stream, not yet synchronised
    out = xattn_prefill_host(Q, K, V, prob.B, prob.S, prob.causal, prob.tau.tolist())
    torch.cuda.synchronize()
    assert out.is_cuda
    assert torch.equal(out.cpu(), O_ref)


def test_against_the_oracle():
    """O of every head and block against the oracle's attention over the
    GPU's own block lists, and the lists against the oracle's find_blocks."""
    prob = make_problem("c1", L=2048, hq=4, hkv=2)
    out, lse = _host_run(prob, 1)
    _, _, counts, idx = _device_reference(prob)
    cn, ixn = counts.numpy(), idx.numpy()
    lists = {(0, h, b): [int(x) for x in ixn[0, h, b, : cn[0, h, b]]]
             for h in range(prob.hq) for b in range(prob.NB)}
    P_ref = O.block_probs(prob.Q, prob.K, prob.B, prob.S, prob.causal)
    for h in range(prob.hq):
        for b in range(prob.NB):
            sel = np.zeros(prob.NB, bool)
            sel[lists[(0, h, b)]] = True
            bd, _, _ = PT.compare_row_masks(P_ref[0, h, b], float(prob.tau[h]), b + 1, sel)
            assert bd == 0, (h, b)
    Oref, lref = O.sparse_attention(prob.Q, prob.K, prob.V, prob.B, prob.causal, lists)
    assert np.max(np.abs(out.float().numpy() - Oref)) <= PT.O_TOL["bf16"]
    assert np.max(np.abs(lse.numpy() - lref)) <= PT.LSE_TOL["bf16"]


def test_full_size_llama_layer():
    """The 128K Llama layer (32 query heads, 8 KV heads) through the host call,
    bit for bit against the device calls."""
    prob = make_problem("c2")
    O_ref, l_ref, _, _ = _device_reference(prob)
    out, lse = _host_run(prob, 0)
    assert torch.equal(out, O_ref)
    assert torch.equal(lse, l_ref)


def test_pageable_host_memory():
    """Pageable (not page-locked) host tensors give the same results; the
    copies then only lose their overlap."""
    prob = make_problem("c1", L=1024, hq=4, hkv=2)
    O_ref, l_ref, _, _ = _device_reference(prob)
    Qh, Kh, Vh = prob.Q.contiguous(), prob.K.contiguous(), prob.V.contiguous()
    assert not Qh.is_pinned()
    out = torch.empty_like(Qh)
    lse = torch.empty(Qh.shape[:3], dtype=torch.float32)
    xattn_prefill_host(Qh, Kh, Vh, prob.B, prob.S, prob.causal, prob.tau.tolist(), out=out,
                       lse=lse)
    torch.cuda.synchronize()
    assert xattn_get_device_status() == 0
    assert torch.equal(out, O_ref) and torch.equal(lse, l_ref)
