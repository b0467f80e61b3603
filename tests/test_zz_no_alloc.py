"""xattn_sparse_attn_noalloc: the attention entry point that allocates nothing.

It serves callers that cannot call cudaMalloc (all device memory owned by
another allocator, or a serving loop that must not allocate once running).
The test calls it through the C ABI twice in a row and compares each output
with the ordinary entry point's, which takes a caller-allocated workspace.
This file is collected last on purpose, so a stop-at-first-failure run has
already run every other test.
"""
import pytest
import torch

from block_sparse_long_score_b200 import (xattn_score,
                                          xattn_select, xattn_sparse_attn,
                                          xattn_sparse_attn_noalloc, xattn_get_device_status,
                                          make_shape)
from block_sparse_long_score_b200 import xattn as X
from block_sparse_long_score_b200.synth import make_problem
from tests import parity as PT

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,kw", [
    ("c1", dict(L=4096, hq=4, hkv=2)),
    ("c4", dict(frames=3, frame_tokens=640, hq=2, S=16)),
    ("c0", dict()),
])
def test_noalloc_matches_workspace_entry_point(name, kw):
    prob = make_problem(name, **kw)
    dev = torch.device("cuda", 0)
    Q, K, V = prob.Q.to(dev), prob.K.to(dev), prob.V.to(dev)
    P = xattn_score(Q, K, prob.B, prob.S, prob.causal)
    _, counts, idx = xattn_select(P, prob.tau, prob.causal)
    ref, ref_lse = xattn_sparse_attn(Q, K, V, counts, idx, prob.B, prob.causal, lse=True)
    tol = PT.O_TOL[prob.dtype]
    for _ in range(2):   # two calls in a row share the library's scratch array
        out = torch.full_like(Q, float("nan"))
        lse = torch.full(Q.shape[:3], float("nan"), device=dev, dtype=torch.float32)
        xattn_sparse_attn_noalloc(Q, K, V, counts, idx, prob.B, prob.causal, out, lse)
        torch.cuda.synchronize()
        assert xattn_get_device_status() == 0
        err = (out.float() - ref.float()).abs().max().item()
        assert err <= tol, err
        assert torch.allclose(lse, ref_lse, atol=PT.LSE_TOL[prob.dtype], rtol=0)


def test_noalloc_rejects_too_many_units():
    """More work units than the scratch array holds: a clear error, no launch."""
    units = X.NOALLOC_MAX_UNITS
    hq = 256
    L = 128 * (units // hq + 1)      # batch * hq * (L/B) just above the limit
    shape = make_shape(1, hq, 1, L, 128, 128, 8, True, "bf16")
    fake = X.ctypes.c_void_p(0x10000)
    import ctypes
    rc = X._lib().xattn_sparse_attn_noalloc(fake, fake, fake, ctypes.byref(shape), fake, fake,
                                            fake, None, None)
    assert rc == -4
