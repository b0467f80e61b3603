"""The seeded generators: deterministic, right shapes and dtypes, and the
planted structure is where the recipe puts it."""
import numpy as np
import torch

from block_sparse_long_score_b200.synth import make_problem, CONFIGS


def test_tiny_full_size_deterministic():
    a = make_problem("c0")
    b = make_problem("c0")
    assert a.Q.shape == (1, 1, 1024, 64) and a.Q.dtype == torch.float32
    assert torch.equal(a.Q, b.Q) and torch.equal(a.K, b.K) and torch.equal(a.V, b.V)
    assert a.B == 64 and a.S == 8 and a.causal and np.allclose(a.tau, 0.9)


def test_llama_small_variant():
    p = make_problem("c1", L=2048, hq=4, hkv=2)
    assert p.Q.shape == (1, 4, 2048, 128) and p.K.shape == (1, 2, 2048, 128)
    assert p.Q.dtype == torch.bfloat16 and p.B == 128 and p.S == 8
    # sink keys carry ~4x the norm of an ordinary key
    kn = p.K[0, 0].float().norm(dim=1)
    assert kn[:4].min() > 3.0 * kn[4:].median()


def test_llama_c2_taus_and_offsets():
    p = make_problem("c2", L=4096, hq=8, hkv=2)
    assert set(np.round(p.tau.astype(np.float64), 2).tolist()) <= {0.8, 0.85, 0.9, 0.95}
    assert p.S == 16
    offs = p.recipe["band_offsets"]
    assert len(offs) == 2 and all(len(o) == 3 for o in offs)
    assert all(0 <= x < 2048 for o in offs for x in o)


def test_video_small_variant():
    p = make_problem("c4", frames=3, frame_tokens=256, hq=2, S=16)
    assert p.Q.shape == (1, 2, 768, 128) and not p.causal and p.S == 16
    assert np.allclose(p.tau, 0.95) and p.hkv == 2
    # same-position tokens of different frames correlate through p[pos]
    q = p.Q[0, 0].float()
    same = (q[5] * q[256 + 5]).sum()
    other = (q[5] * q[256 + 77]).sum()
    assert same > other


def test_config_table():
    assert CONFIGS["c2"]["L"] == 131072 and CONFIGS["c3"]["L"] == 262144
    assert CONFIGS["c4"]["S"] == [4, 8, 16, 64]
