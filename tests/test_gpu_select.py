"""xattn_select against the oracle's find_blocks on the same fp32 rows.

Selection turns floating-point sums into integers, so on identical inputs the
GPU must choose exactly the oracle's blocks. The rows here are built to reach
every path of the kernel: ordinary rows, exact ties (more than 32 equal
values), flat rows, zeros, tau = 1, and a cut that lies more than 31 octaves
below the row maximum.
"""
import numpy as np
import pytest
import torch

import oracle.xattn_oracle as O
from block_sparse_long_score_b200 import xattn_select
from tests import parity as PT

pytestmark = pytest.mark.gpu


def _run(P: np.ndarray, taus, causal: bool):
    Pt = torch.from_numpy(P.astype(np.float32)).cuda()
    mask, counts, idx = xattn_select(Pt, list(taus), causal)
    torch.cuda.synchronize()
    NB = P.shape[-1]
    return (PT.mask_to_bool(PT.to_np(mask), NB), PT.to_np(counts), PT.to_np(idx))


def _check(P, taus, causal):
    m, c, ix = _run(P, taus, causal)
    P32 = P.astype(np.float32).astype(np.float64)
    b_, hq, NB, _ = P.shape
    for h in range(hq):
        for b in range(NB):
            n = b + 1 if causal else NB
            want = np.zeros(NB, bool)
            want[O.find_blocks(P32[0, h, b, :n], float(np.float32(taus[h])))] = True
            assert np.array_equal(m[0, h, b], want), (h, b, np.nonzero(m[0, h, b])[0][:10],
                                                      np.nonzero(want)[0][:10])
            assert c[0, h, b] == want.sum()
            assert np.array_equal(ix[0, h, b, : c[0, h, b]], np.nonzero(want)[0])


def _rows(NB, kind, rng, causal):
    P = np.zeros((NB, NB))
    for b in range(NB):
        n = b + 1 if causal else NB
        if kind == "dirichlet":
            a = rng.choice([0.05, 0.3, 1.0, 5.0])
            p = rng.dirichlet(np.ones(n) * a)
        elif kind == "flat":
            p = np.full(n, 1.0 / n)
        elif kind == "ties":
            p = np.full(n, 1e-4)
            k = min(n, 40)
            p[rng.choice(n, size=k, replace=False)] = 0.5 / k
        elif kind == "zeros":
            p = rng.dirichlet(np.ones(n) * 0.2)
            p[rng.random(n) < 0.5] = 0.0
            if p.sum() == 0:
                p[0] = 1.0
        P[b, :n] = p / max(p.sum(), 1e-300) if kind != "ties" else p
    return P


@pytest.mark.parametrize("NB", [1, 7, 33, 100, 600, 2048])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("kind", ["dirichlet", "flat", "ties", "zeros"])
def test_select_exact(NB, causal, kind):
    if NB == 2048 and not causal and kind != "dirichlet":
        pytest.skip("covered by the causal case")
    rng = np.random.default_rng(NB * 7 + causal * 3 + len(kind))
    hq = 4
    P = np.stack([_rows(NB, kind, rng, causal) for _ in range(hq)])[None]
    taus = [0.5, 0.8, 0.95, 1.0]
    _check(P, taus, causal)


def test_cut_far_below_the_maximum():
    """tau one fp32 step above the largest block (0.75), so the cut lies
    among ~500 blocks 32 octaves below it."""
    NB = 1024
    P = np.zeros((1, 1, NB, NB))
    tiny = 2.0 ** -33
    for b in range(NB):
        P[0, 0, b, :] = tiny * (1.0 + (np.arange(NB) % 5) / 8.0)
        P[0, 0, b, b % 7] = 0.75
    tau = float(np.nextafter(np.float32(0.75), np.float32(1.0)))
    assert tau > 0.75
    _check(P, [tau], False)


def test_many_equal_values_at_the_cut():
    """100 blocks share the cut value exactly: ties go to the lower index."""
    NB = 300
    P = np.zeros((1, 2, NB, NB))
    for h in range(2):
        for b in range(NB):
            P[0, h, b, :] = 1.0 / 1024
            P[0, h, b, 200:] = 1.0 / 8192
            P[0, h, b, 7] = 0.25
    _check(P, [0.3, 0.45], False)


def test_cut_below_the_first_thresholds_and_zero_rows():
    """Rows whose cut lies 9 and 15 octaves below the maximum (the filter's
    first thresholds hold too little mass, so lower ones are tried), rows with
    more candidates than the filter sorts (left to the histogram search), and
    all-zero rows (the sum never reaches tau: every allowed block)."""
    NB = 700
    rng = np.random.default_rng(5)
    P = np.zeros((1, 4, NB, NB))
    for h in range(4):
        for b in range(NB):
            n = b + 1
            row = np.full(n, 1e-9)
            row[rng.integers(0, n)] = 0.5
            k = min(n, [20, 20, 200, 0][h])
            if k:
                pos = rng.choice(n, size=k, replace=False)
                row[pos] = 0.5 * 2.0 ** -(9 if h == 0 else (15 if h == 1 else 10))
            if h == 3 and b % 3 == 0:
                row[:] = 0.0
            P[0, h, b, :n] = row
    _check(P, [0.5 + 0.5 * 2.0 ** -9 * 7.5, 0.5 + 0.5 * 2.0 ** -15 * 12.5, 0.6, 0.9], True)


@pytest.mark.parametrize("k", [32, 33, 64, 65, 128, 129, 200, 256, 257, 400])
def test_candidate_counts_around_the_filter_sizes(k):
    """Rows whose threshold that first reaches tau holds exactly k candidates:
    one to eight keys a lane in the filter's sort (k <= 256), the histogram
    search above that. The candidates take a few distinct values within a
    factor of 8, and many tie, so both the ranked order and the exact prefix
    scan of the walk are exercised; tau falls between and exactly on ranked
    sums."""
    NB = 512
    rng = np.random.default_rng(k)
    P = np.zeros((1, 3, NB, NB))
    for h in range(3):
        for b in range(NB):
            row = np.full(NB, 2.0 ** -30)
            pos = rng.choice(NB, size=k, replace=False)
            row[pos] = rng.choice([1.0, 1.0, 0.5, 0.25, 0.125], size=k)
            row /= row.sum()
            P[0, h, b] = row
    P32 = P.astype(np.float32).astype(np.float64)
    # head 2: tau exactly equal to a ranked fp64 partial sum (cut on the boundary)
    ranked = np.sort(P32[0, 2, 0])[::-1]
    tau2 = float(np.float32(np.cumsum(ranked)[k // 2]))
    _check(P, [0.5, 0.9, tau2], False)
