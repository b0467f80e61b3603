"""GPU parity: the CUDA path through the C ABI against the fp64 CPU oracle.

Small problems are checked element by element (every head, every query
block). Full-size workloads run exactly as bench.py launches them and are
checked on sampled heads and query blocks (always including the first and the
last), which the oracle can compute one by one.
"""
import numpy as np
import pytest
import torch

import oracle.xattn_oracle as O
from block_sparse_long_score_b200 import (xattn_get_device_status, xattn_score, xattn_select,
                                          xattn_sparse_attn)
from block_sparse_long_score_b200.synth import make_problem
from tests import parity as PT

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def run_gpu(prob, tau=None):
    Q, K, V = prob.Q.to(DEV), prob.K.to(DEV), prob.V.to(DEV)
    taus = prob.tau if tau is None else tau
    P = xattn_score(Q, K, prob.B, prob.S, prob.causal)
    mask, counts, idx = xattn_select(P, taus, prob.causal)
    out, lse = xattn_sparse_attn(Q, K, V, counts, idx, prob.B, prob.causal, lse=True)
    torch.cuda.synchronize()
    assert xattn_get_device_status() == 0
    return dict(P=PT.to_np(P), mask=PT.mask_to_bool(PT.to_np(mask), prob.NB),
                counts=PT.to_np(counts), idx=PT.to_np(idx), O=PT.to_np(out.float()),
                lse=PT.to_np(lse))


def check_problem(prob, heads, qblocks, res, require_no_exempt=False):
    """P, masks and outputs on the sampled heads / query blocks."""
    taus = prob.tau
    NB = prob.NB
    P_ref = O.block_probs(prob.Q, prob.K, prob.B, prob.S, prob.causal, heads=heads,
                          q_blocks=qblocks)
    worst = 0.0
    bad = exempt = 0
    for h in heads:
        worst = max(worst, PT.check_probs(res["P"][0, h, qblocks], P_ref[0, h, qblocks]))
        for b in qblocks:
            n = b + 1 if prob.causal else NB
            bd, ex, _ = PT.compare_row_masks(P_ref[0, h, b], float(taus[h]), n, res["mask"][0, h, b])
            bad += bd
            exempt += ex
    assert worst <= 1.0, f"P error {worst:.3g} x tolerance"
    assert bad == 0, f"{bad} mask mismatches outside the tau band"
    if require_no_exempt:
        assert exempt == 0
    PT.check_lists(res["mask"][0][np.ix_(heads, qblocks)], res["counts"][0][np.ix_(heads, qblocks)],
                   res["idx"][0][np.ix_(heads, qblocks)])
    # attention given the GPU's own lists
    lists = {}
    for h in heads:
        for b in qblocks:
            lists[(0, h, b)] = [int(x) for x in res["idx"][0, h, b, : res["counts"][0, h, b]]]
    Oref, lref = O.sparse_attention(prob.Q, prob.K, prob.V, prob.B, prob.causal, lists,
                                    heads=heads, q_blocks=qblocks)
    rows = np.concatenate([np.arange(b * prob.B, min((b + 1) * prob.B, prob.L)) for b in qblocks])
    for h in heads:
        err = np.max(np.abs(res["O"][0, h, rows] - Oref[0, h, rows]))
        assert err <= PT.O_TOL[prob.dtype], f"head {h}: max |dO| = {err:.3g}"
        lerr = np.max(np.abs(res["lse"][0, h, rows] - lref[0, h, rows]))
        assert lerr <= PT.LSE_TOL[prob.dtype], f"head {h}: max |dlse| = {lerr:.3g}"
    return exempt


def sample_blocks(NB, k=48, seed=0):
    rng = np.random.default_rng(seed)
    mid = rng.choice(np.arange(1, NB - 1), size=min(k - 2, NB - 2), replace=False)
    return sorted(set([0, NB - 1] + mid.tolist()))


# ------------------------------------------------------------ tiny fp32 ----
def test_tiny_fp32_full_parity():
    """The 1-head fp32 workload, element by element. No block may sit in the
    tau band, and no mask may differ."""
    prob = make_problem("c0")
    res = run_gpu(prob)
    exempt = check_problem(prob, [0], list(range(prob.NB)), res, require_no_exempt=True)
    assert exempt == 0


def test_select_matches_oracle_on_same_probs():
    """xattn_select on the GPU's own P equals find_blocks on those values."""
    prob = make_problem("c1", L=4096, hq=4, hkv=2)
    res = run_gpu(prob)
    for h in range(prob.hq):
        for b in range(prob.NB):
            p = res["P"][0, h, b, : b + 1].astype(np.float64)
            want = np.zeros(prob.NB, bool)
            want[O.find_blocks(p, float(prob.tau[h]))] = True
            assert np.array_equal(res["mask"][0, h, b], want), (h, b)


# ------------------------------------------------------- small bf16 ----
@pytest.mark.parametrize("name,kw", [
    ("c1", dict(L=4096, hq=4, hkv=2)),
    ("c2", dict(L=8192, hq=4, hkv=1)),
    ("c3", dict(L=2048, hq=8, hkv=2)),
    ("c4", dict(frames=3, frame_tokens=640, hq=2, S=4)),
    ("c4", dict(frames=3, frame_tokens=640, hq=2, S=8)),
    ("c4", dict(frames=3, frame_tokens=640, hq=2, S=16)),   # L/S = 120: ragged M and N tiles
    ("c4", dict(frames=3, frame_tokens=640, hq=2, S=64)),   # r = 2
])
def test_small_bf16_full_parity(name, kw):
    prob = make_problem(name, **kw)
    res = run_gpu(prob)
    check_problem(prob, list(range(prob.hq)), list(range(prob.NB)), res)


@pytest.mark.parametrize("S", [1, 2, 32])
def test_unusual_strides(S):
    prob = make_problem("c1", L=1024, hq=2, hkv=1)
    prob.S = S
    res = run_gpu(prob)
    check_problem(prob, [0, 1], list(range(prob.NB)), res)


def test_single_block_sequence():
    prob = make_problem("c1", L=128, hq=2, hkv=2)
    res = run_gpu(prob)
    assert np.allclose(res["P"][0, :, 0, 0], 1.0, atol=1e-6)
    check_problem(prob, [0, 1], [0], res)


# ---------------------------------------------------------- edge cases ----
@pytest.mark.parametrize("causal", [True, False])
def test_tau_one_is_dense_attention(causal):
    """tau = 1 selects every allowed block; the output is then plain
    (causal) attention, checked against the naive oracle."""
    prob = make_problem("c1", L=1024, hq=2, hkv=1)
    prob.causal = causal
    res = run_gpu(prob, tau=np.ones(2, np.float32))
    NB = prob.NB
    for h in range(2):
        for b in range(NB):
            n = b + 1 if causal else NB
            assert res["counts"][0, h, b] == n
    q = O.to_f64(prob.Q)[0, 1, :256]
    k = O.to_f64(prob.K)[0, 0]
    v = O.to_f64(prob.V)[0, 0]
    logits = q @ k.T / np.sqrt(128)
    if causal:
        logits[np.arange(256)[:, None] < np.arange(1024)[None, :]] = -np.inf
    w = np.exp(logits - logits.max(1, keepdims=True))
    want = (w / w.sum(1, keepdims=True)) @ v
    assert np.max(np.abs(res["O"][0, 1, :256] - want)) <= PT.O_TOL["bf16"]


def test_empty_and_trailing_lists():
    """A row with no block gives O = 0 and lse = -inf. In causal mode listed
    blocks above the diagonal are skipped."""
    prob = make_problem("c1", L=1024, hq=1, hkv=1)
    Q, K, V = prob.Q.to(DEV), prob.K.to(DEV), prob.V.to(DEV)
    NB = prob.NB
    counts = torch.zeros(1, 1, NB, dtype=torch.int32)
    idx = torch.zeros(1, 1, NB, NB, dtype=torch.int32)
    lists = {}
    for b in range(NB):
        if b == 3:
            lists[b] = []
            continue
        lst = sorted(set([0, b]))
        lists[b] = lst
        full = lst + list(range(b + 1, min(b + 3, NB)))   # trailing blocks above the diagonal
        counts[0, 0, b] = len(full)
        idx[0, 0, b, : len(full)] = torch.tensor(full, dtype=torch.int32)
    out, lse = xattn_sparse_attn(Q, K, V, counts.to(DEV), idx.to(DEV), 128, True, lse=True)
    torch.cuda.synchronize()
    o = PT.to_np(out.float())
    l = PT.to_np(lse)
    assert np.all(o[0, 0, 384:512] == 0) and np.all(np.isneginf(l[0, 0, 384:512]))
    Oref, lref = O.sparse_attention(prob.Q, prob.K, prob.V, 128, True,
                                    {(0, 0, b): lists[b] for b in range(NB)})
    assert np.max(np.abs(o - Oref)) <= PT.O_TOL["bf16"]


def test_gqa_mapping_on_gpu():
    """Heads 0..3 read KV head 0, heads 4..7 KV head 1."""
    prob = make_problem("c1", L=1024, hq=8, hkv=2)
    res = run_gpu(prob)
    check_problem(prob, [0, 3, 4, 7], list(range(prob.NB)), res)


def test_deterministic():
    prob = make_problem("c1", L=2048, hq=4, hkv=2)
    a = run_gpu(prob)
    b = run_gpu(prob)
    for k in ("P", "mask", "counts", "O", "lse"):
        assert np.array_equal(a[k], b[k]), k


# ------------------------------------------------------ full-size workloads ----
FULL = [
    ("c1", dict(), [0, 13, 31]),
    ("c2", dict(), [5]),
    ("c3", dict(), [9]),
    ("c4", dict(S=4), [2]),
    ("c4", dict(S=8), [2]),
    ("c4", dict(S=16), [11]),
    ("c4", dict(S=64), [23]),
]


@pytest.mark.parametrize("name,kw,heads", FULL)
def test_full_size_sampled(name, kw, heads):
    prob = make_problem(name, **kw)
    res = run_gpu(prob)
    # every row of P sums to 1 and causal rows are 0 above the diagonal
    sums = res["P"].sum(axis=-1)
    assert np.max(np.abs(sums - 1.0)) < 1e-3
    if prob.causal:
        assert np.all(res["P"][0, :, np.triu_indices(prob.NB, 1)[0], np.triu_indices(prob.NB, 1)[1]] == 0)
    check_problem(prob, heads, sample_blocks(prob.NB), res)


# ------------------------------------------------------------- batch > 1 ----
def test_batch_of_two_every_path():
    """Two sequences in one call: every batch element checked against the
    oracle (P, masks, outputs), through the three calls, the fused call and
    the no-alloc attention."""
    from block_sparse_long_score_b200 import xattn_score_select, xattn_sparse_attn_noalloc
    prob = make_problem("c1", L=2048, hq=4, hkv=2, batch=2)
    assert prob.Q.shape[0] == 2
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
    assert xattn_get_device_status() == 0
    assert torch.equal(P, P2) and torch.equal(mask, mask2) and torch.equal(counts, counts2)
    assert torch.equal(out, out2)
    Pn, mb = PT.to_np(P), PT.mask_to_bool(PT.to_np(mask), prob.NB)
    cn, ixn = PT.to_np(counts), PT.to_np(idx)
    On, ln = PT.to_np(out.float()), PT.to_np(lse)
    P_ref = O.block_probs(prob.Q, prob.K, prob.B, prob.S, prob.causal)
    lists = {}
    for bb in range(2):
        for h in range(prob.hq):
            assert PT.check_probs(Pn[bb, h], P_ref[bb, h]) <= 1.0
            for b in range(prob.NB):
                bd, _, _ = PT.compare_row_masks(P_ref[bb, h, b], float(taus[h]), b + 1, mb[bb, h, b])
                assert bd == 0, (bb, h, b)
                lists[(bb, h, b)] = [int(x) for x in ixn[bb, h, b, : cn[bb, h, b]]]
    Oref, lref = O.sparse_attention(prob.Q, prob.K, prob.V, prob.B, prob.causal, lists)
    assert np.max(np.abs(On - Oref)) <= PT.O_TOL["bf16"]
    assert np.max(np.abs(ln - lref)) <= PT.LSE_TOL["bf16"]
    # the two sequences differ, so a batch-index mix-up would show
    assert np.max(np.abs(On[0] - On[1])) > 0.1


# -------------------------------------------------------- maximum size ----
def test_maximum_block_count():
    """NB = 4096 query / key blocks (L = 512K tokens, the largest NB the calls
    accept), one head: sampled query blocks against the oracle."""
    prob = make_problem("c1", L=4096 * 128, hq=1, hkv=1)
    assert prob.NB == 4096
    res = run_gpu(prob)
    qblocks = [0, 1, 2047, 3000, 4094, 4095]
    check_problem(prob, [0], qblocks, res)


def test_output_only_16_byte_aligned():
    """O at a 16-byte but not 32-byte aligned address takes the 16-byte store
    path and gives the same result as an aligned O."""
    prob = make_problem("c1", L=2048, hq=2, hkv=1)
    Q, K, V = prob.Q.to(DEV), prob.K.to(DEV), prob.V.to(DEV)
    P = xattn_score(Q, K, prob.B, prob.S, prob.causal)
    _, counts, idx = xattn_select(P, prob.tau.tolist(), prob.causal)
    ref = xattn_sparse_attn(Q, K, V, counts, idx, prob.B, prob.causal)
    flat = torch.empty(Q.numel() + 16, device=DEV, dtype=Q.dtype)
    out = flat[8:8 + Q.numel()].view(Q.shape)   # 8 bf16 = 16 bytes past a 256-byte base
    assert out.data_ptr() % 32 == 16
    xattn_sparse_attn(Q, K, V, counts, idx, prob.B, prob.causal, out=out)
    torch.cuda.synchronize()
    assert xattn_get_device_status() == 0
    assert torch.equal(out, ref)
