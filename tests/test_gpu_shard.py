"""The head-sharded split on one GPU: the ranges of KV heads that the ranks
of a head-sharded run would take, run one after another here, give exactly the
whole-layer output when put side by side (every step works per head)."""
import pytest
import torch

from block_sparse_long_score_b200 import prefill_attention, xattn_get_device_status
from block_sparse_long_score_b200.shard import kv_head_range, prefill_attention_heads
from block_sparse_long_score_b200.synth import make_problem

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.mark.parametrize("name,kw,world", [
    ("c1", dict(L=4096, hq=8, hkv=4), 2),
    ("c1", dict(L=4096, hq=12, hkv=3, batch=2), 2),      # uneven ranges, batch of two
    ("c2", dict(L=8192, hq=32, hkv=8), 4),
    ("c4", dict(frames=3, frame_tokens=640, hq=4, S=8), 3),
])
def test_head_ranges_reassemble_the_whole_layer(name, kw, world):
    prob = make_problem(name, **kw)
    Q, K, V = prob.Q.to(DEV), prob.K.to(DEV), prob.V.to(DEV)
    tau = torch.tensor(prob.tau.tolist(), dtype=torch.float32, device=DEV)
    whole = prefill_attention(Q, K, V, prob.B, prob.S, tau, prob.causal)
    g = prob.hq // prob.hkv
    parts = []
    for r in range(world):
        kv0, kv1 = kv_head_range(r, world, prob.hkv)
        parts.append(prefill_attention_heads(Q, K, V, prob.B, prob.S, tau, prob.causal,
                                             kv0, kv1))
        assert parts[-1].shape[1] == (kv1 - kv0) * g
    torch.cuda.synchronize()
    assert xattn_get_device_status() == 0
    assert torch.equal(torch.cat(parts, dim=1), whole)
