"""xattn_check_lists: the validation of block lists made outside xattn_select.

Lists written by xattn_select must pass (causal, non-causal with a short last
block, tau = 1 where rows hold every block). Then mistakes are planted on the
host in copies of those lists -- a count out of range, an entry out of range,
a repeated entry, two entries swapped, a mistake on either side of a 32-entry
chunk boundary -- and the kernel must count exactly the rows a plain Python
check of the same layout rule finds. Entries past a row's count are never
looked at.
"""
import numpy as np
import pytest
import torch

from block_sparse_long_score_b200 import (xattn_check_lists, xattn_get_device_status,
                                          xattn_score_select)
from block_sparse_long_score_b200.synth import make_problem

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _lists(prob, tau=None):
    Q, K = prob.Q.to(DEV), prob.K.to(DEV)
    taus = prob.tau.tolist() if tau is None else [tau] * prob.hq
    _, counts, idx = xattn_score_select(Q, K, prob.B, prob.S, prob.causal, taus)
    torch.cuda.synchronize()
    return Q, K, counts.cpu(), idx.cpu()


def _bad_rows_host(counts, idx, NB):
    """The layout rule, row by row in Python."""
    c = counts.reshape(-1).numpy()
    ix = idx.reshape(-1, NB).numpy()
    bad = 0
    for r in range(c.size):
        n = int(c[r])
        if n < 0 or n > NB:
            bad += 1
            continue
        row = ix[r, :n].astype(np.int64)
        ok = all(0 <= v < NB for v in row) and all(row[i] < row[i + 1] for i in range(n - 1))
        bad += 0 if ok else 1
    return bad


def _check(prob, Q, K, counts, idx):
    bad = xattn_check_lists(Q, K, counts.to(DEV), idx.to(DEV), prob.B, prob.causal)
    torch.cuda.synchronize()
    assert xattn_get_device_status() == 0
    return int(bad.item())


@pytest.mark.parametrize("name,kw,tau", [
    ("c1", dict(L=4096, hq=4, hkv=2), None),
    ("c1", dict(L=2496, hq=4, hkv=2), None),                      # short last block
    ("c4", dict(frames=3, frame_tokens=592, hq=2, S=8), None),    # non-causal, ragged
    ("c1", dict(L=8192, hq=2, hkv=1), 1.0),                       # every block: 64-entry rows
])
def test_select_lists_pass(name, kw, tau):
    prob = make_problem(name, **kw)
    Q, K, counts, idx = _lists(prob, tau)
    assert _bad_rows_host(counts, idx, prob.NB) == 0
    assert _check(prob, Q, K, counts, idx) == 0


def test_planted_mistakes_are_counted():
    prob = make_problem("c1", L=8192, hq=2, hkv=1)
    NB = prob.NB
    Q, K, counts, idx = _lists(prob, 1.0)   # row (h, b) lists blocks 0..b
    c = counts.clone()
    ix = idx.clone()
    planted = {
        (0, 5): lambda: c.__setitem__((0, 0, 5), NB + 1),          # count above NB
        (0, 6): lambda: c.__setitem__((0, 0, 6), -1),              # negative count
        (0, 7): lambda: ix.__setitem__((0, 0, 7, 3), NB),          # entry past the last block
        (0, 8): lambda: ix.__setitem__((0, 0, 8, 0), -2),          # negative entry
        (0, 9): lambda: ix.__setitem__((0, 0, 9, 4), 3),           # repeated entry
        (1, 40): lambda: ix.__setitem__((0, 1, 40, slice(31, 33)),
                                        torch.tensor([32, 31], dtype=torch.int32)),  # swap across chunks
        (1, 50): lambda: ix.__setitem__((0, 1, 50, 32), 31),       # first entry of chunk 2 repeats
        (1, 63): lambda: ix.__setitem__((0, 1, 63, 63), 62),       # last entry of a full row
    }
    for fn in planted.values():
        fn()
    # not mistakes: junk past a row's count, and an empty row
    ix[0, 1, 10, 11:] = -7
    c[0, 1, 11] = 0
    ix[0, 1, 11, :] = 999
    expect = _bad_rows_host(c, ix, NB)
    assert expect == len(planted)
    assert _check(prob, Q, K, c, ix) == expect


def test_one_mistake_in_many_rows():
    """Every row of a head broken: the count equals the number of rows."""
    prob = make_problem("c1", L=4096, hq=4, hkv=2)
    Q, K, counts, idx = _lists(prob, 1.0)
    c = counts.clone()
    c[0, 2] = prob.NB + 5
    assert _check(prob, Q, K, c, idx) == prob.NB
