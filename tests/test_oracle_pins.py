"""Pins for the CPU oracle, against facts that come from outside the oracle.

Every check compares the oracle with something it does not share code with:
brute-force sums written as loops, closed forms, special cases that reduce
to plain attention, brute force over subsets, and the worked example printed
on "XAttention 计算步骤详解及示例" (§2). A few tests plant a plausible mistake
in a copy of the oracle and check that a pin catches it.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest

import oracle.xattn_oracle as O

GOLD = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(1234)


def _rand(*shape, scale=1.0):
    return rng.standard_normal(shape) * scale


# ---------------------------------------------------------------- P1 --------
@pytest.mark.parametrize("S", [1, 2, 4, 8])
def test_reshape_equals_bruteforce_antidiagonal(S):
    """Alg. 1's reshaped product equals the antidiagonal sum of every S x S
    tile of Q K^T (§2.1: lower-left to upper-right)."""
    q, k = _rand(32, 4), _rand(32, 4)
    got = O.reshaped_logits(q, k, S)
    want = O.antidiagonal_sums_bruteforce(q, k, S)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_main_diagonal_mistake_is_caught():
    """Planted mistake: stacking query slices in increasing order gives the
    main diagonal, which the brute-force pin rejects."""
    q, k = _rand(32, 4), _rand(32, 4)
    S = 4
    wrong = np.concatenate([q[i::S] for i in range(S)], axis=1) @ O.reshape_keys(k, S).T
    want = O.antidiagonal_sums_bruteforce(q, k, S)
    assert np.max(np.abs(wrong - want)) > 1e-3


# ---------------------------------------------------------------- scale -----
def _group_constant(nt, d, S, scale=1.0):
    base = _rand(nt, d, scale=scale)
    return base, np.repeat(base, S, axis=0)


@pytest.mark.parametrize("causal", [True, False])
def test_scale_sqrt_dS_closed_form(causal):
    """Queries and keys constant within each S-group turn A_approx into plain
    attention of (sqrt(S) q_hat, k_hat). So the scale 1/sqrt(d_h S) is pinned
    against the independent naive attention routine."""
    S, d, B = 4, 8, 16
    r = B // S
    qh, q = _group_constant(16, d, S, 0.7)
    kh, k = _group_constant(16, d, S, 0.7)
    P = O.block_probs_head(q, k, B, S, causal)
    _, probs = O.dense_attention_naive(math.sqrt(S) * qh, kh, np.zeros((16, 1)), causal)
    NB = q.shape[0] // B
    want = probs.reshape(NB, r, NB, r).sum(axis=(1, 3)) / r
    np.testing.assert_allclose(P, want, rtol=0, atol=1e-12)


def test_wrong_scale_is_caught():
    """Planted mistake: scaling by 1/sqrt(d) alone changes P beyond 1e-6."""
    S, d, B = 4, 8, 16
    qh, q = _group_constant(16, d, S, 0.7)
    kh, k = _group_constant(16, d, S, 0.7)
    good = O.block_probs_head(q, k, B, S, True)
    bad = O.block_probs_head(q * math.sqrt(S), k, B, S, True)
    assert np.max(np.abs(good - bad)) > 1e-6


# ---------------------------------------------------------------- P2 --------
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("S", [2, 4, 8])
def test_rows_are_distributions(causal, S):
    """Each softmax row sums to 1, so each P row sums to 1 (tau in (0, 1]).
    Causal rows are 0 above the diagonal."""
    q, k = _rand(256, 16), _rand(256, 16)
    P = O.block_probs_head(q, k, 32, S, causal)
    np.testing.assert_allclose(P.sum(axis=1), 1.0, rtol=0, atol=1e-12)
    assert (P >= 0).all()
    if causal:
        assert np.all(P[np.triu_indices(P.shape[0], 1)] == 0.0)
    x = O.reshaped_logits(q, k, S) / math.sqrt(16 * S)
    A = O.approx_attention_rows(x, 0, causal)
    np.testing.assert_allclose(A.sum(axis=1), 1.0, rtol=0, atol=1e-12)
    if causal:
        assert A[0, 0] == 1.0   # reshaped row 0 sees only reshaped column 0


# ---------------------------------------------------------------- P3 --------
@pytest.mark.parametrize("causal", [True, False])
def test_stride_one_is_exact_attention(causal):
    """With S = 1 the reshape is the identity and A_approx is exact attention,
    so P is the block mean of the naive attention probabilities."""
    q, k = _rand(48, 4), _rand(48, 4)
    B = 8
    P = O.block_probs_head(q, k, B, 1, causal)
    _, probs = O.dense_attention_naive(q, k, np.zeros((48, 1)), causal)
    NB = 48 // B
    want = probs.reshape(NB, B, NB, B).sum(axis=(1, 3)) / B
    np.testing.assert_allclose(P, want, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- P4 --------
@pytest.mark.parametrize("causal", [True, False])
def test_tau_one_selects_everything_allowed(causal):
    q, k = _rand(256, 8), _rand(256, 8)
    P = O.block_probs_head(q, k, 32, 4, causal)[None, None]
    mask, lists = O.select_blocks(P, [1.0], causal)
    NB = P.shape[-1]
    want = np.tril(np.ones((NB, NB), bool)) if causal else np.ones((NB, NB), bool)
    assert (mask[0, 0] == want).all()


# ---------------------------------------------------------------- P5 --------
@pytest.mark.parametrize("causal", [True, False])
def test_dense_mask_sparse_attention_is_naive_attention(causal):
    q, k, v = _rand(32, 4), _rand(32, 4), _rand(32, 3)
    B = 8
    NB = 4
    lists = {b: list(range(b + 1 if causal else NB)) for b in range(NB)}
    Os, lse = O.sparse_attention_head(q, k, v, B, causal, lists)
    On, _ = O.dense_attention_naive(q, k, v, causal)
    np.testing.assert_allclose(Os, On, rtol=0, atol=1e-12)
    raw = O.dense_scores(q, k) / math.sqrt(4)
    for i in range(32):
        n = i + 1 if causal else 32
        want = math.log(math.fsum(math.exp(x) for x in raw[i, :n]))
        assert abs(lse[i] - want) < 1e-12


@pytest.mark.parametrize("causal", [True, False])
def test_sparse_lists_match_filtered_naive_attention(causal):
    """Any block list equals naive attention with the unlisted blocks
    filtered out (block 0 is in every list, so no row is empty)."""
    q, k, v = _rand(64, 4), _rand(64, 4), _rand(64, 5)
    B, NB = 8, 8
    lists = {}
    for b in range(NB):
        n = b + 1 if causal else NB
        pick = {0} | {j for j in range(n) if rng.random() < 0.5}
        lists[b] = sorted(pick)
    Os, _ = O.sparse_attention_head(q, k, v, B, causal, lists)
    On, _ = O.dense_attention_naive(q, k, v, causal,
                                    allowed=lambda i, j: (j // B) in lists[i // B])
    np.testing.assert_allclose(Os, On, rtol=0, atol=1e-12)


def test_empty_list_gives_zero_row():
    q, k, v = _rand(16, 4), _rand(16, 4), _rand(16, 2)
    Os, lse = O.sparse_attention_head(q, k, v, 8, True, {0: [0], 1: []})
    assert np.all(Os[8:] == 0.0) and np.all(np.isneginf(lse[8:]))


# ---------------------------------------------------------------- P6 --------
def _brute_minimal(p, tau):
    n = len(p)
    for size in range(1, n + 1):
        best = None
        for sub in itertools.combinations(range(n), size):
            s = math.fsum(p[i] for i in sub)
            if s >= tau:
                key = (-s, sub)
                if best is None or key < best:
                    best = key
        if best is not None:
            return list(best[1])
    return list(range(n))


@pytest.mark.parametrize("trial", range(40))
def test_find_blocks_minimal_and_tie_break(trial):
    """Brute force over all subsets: the chosen set has the smallest size that
    reaches tau. Among the sets of that size with the largest sum it is the
    one with the lowest indices (ties go to the lower block index)."""
    n = int(rng.integers(1, 11))
    p = rng.dirichlet(np.ones(n) * 0.5)
    if trial % 3 == 0:           # plant exact ties
        p = np.round(p * 8) / 8
        p = p / p.sum() if p.sum() > 0 else np.full(n, 1.0 / n)
    cs = np.cumsum(np.sort(p)[::-1])
    while True:
        tau = float(rng.uniform(0.05, 0.999))
        if np.min(np.abs(cs - tau)) > 1e-9:
            break
    got = list(O.find_blocks(p, tau))
    want = sorted(_brute_minimal(list(p), tau))
    assert got == want
    order = np.lexsort((np.arange(n), -p))
    csum = np.cumsum(p[order])
    k = len(got)
    if csum[-1] >= tau:
        assert csum[k - 1] >= tau and (k == 1 or csum[k - 2] < tau)


def test_find_blocks_unreached_takes_all():
    assert list(O.find_blocks(np.array([0.3, 0.3]), 0.9)) == [0, 1]


# ---------------------------------------------------------------- P7 --------
def test_worked_example_selection():
    with open(os.path.join(GOLD, "find_blocks_worked_example.json")) as f:
        g = json.load(f)
    assert list(O.find_blocks(np.array(g["p"]), g["tau"])) == g["selected"]


def test_worked_example_raw_scores():
    with open(os.path.join(GOLD, "raw_scores_worked_example.json")) as f:
        g = json.load(f)
    q, k = np.array(g["Q"]), np.array(g["K"])
    assert (O.dense_scores(q, k) == np.array(g["QKt"])).all()
    assert (O.reshaped_logits(q, np.vstack([k, k[:1]])[:3], 1) == np.array(g["QKt"])).all()


# ---------------------------------------------------------------- P8 --------
def test_vertical_line_is_detected():
    """§2.1: every key meets the antidiagonal of every tile in its column. A
    single dominant key k* makes every later block row put almost all its mass
    on k*'s block, and tau = 0.9 keeps only that block."""
    L, d, B, S = 256, 32, 32, 4
    q, k = _rand(L, d, scale=0.1), _rand(L, d, scale=0.1)
    u = _rand(d)
    u /= np.linalg.norm(u)
    kstar = 77
    q += u
    k[kstar] += 400.0 * u
    P = O.block_probs_head(q, k, B, S, True)
    jb = kstar // B
    r = B // S
    first_full = -(-(kstar // S) // r)      # first block whose rows all see k*
    for b in range(max(first_full, jb + 1), L // B):
        assert P[b, jb] >= 0.99
        assert list(O.find_blocks(P[b, : b + 1], 0.9)) == [jb]


# ---------------------------------------------------------------- P9 --------
@pytest.mark.parametrize("delta,seen", [(2, False), (4, False), (3, True), (1, True)])
def test_antidiagonal_parity_orientation(delta, seen):
    """For even S, antidiagonal cells have q - k odd. A slash at an even
    offset is invisible, one at an odd offset is seen. A main-diagonal scorer
    (the wrong orientation) shows the opposite parity, so this pins it."""
    L, S = 32, 4
    q = np.eye(L)
    k = np.zeros((L, L))
    for j in range(L - delta):
        k[j, j + delta] = 1.0           # q_i . k_j = 1 iff i - j = delta
    x = O.reshaped_logits(q, k, S)
    assert (np.abs(x).sum() > 0) == seen
    for t in range(L // S):
        for c in range(L // S):
            want = sum(1 for i in range(S) if t * S + S - 1 - i == c * S + i + delta)
            assert x[t, c] == want
    main = np.concatenate([q[i::S] for i in range(S)], axis=1) @ O.reshape_keys(k, S).T
    assert (np.abs(main).sum() > 0) == (delta % S == 0)


# ---------------------------------------------------------------- GQA -------
def test_gqa_head_mapping():
    """Query head h reads KV head h // (Hq / Hkv), not h % Hkv."""
    hq, hkv, L, d = 4, 2, 64, 8
    Q = _rand(1, hq, L, d)
    K = _rand(1, hkv, L, d)
    K[0, 1] *= 3.0
    P = O.block_probs(Q, K, 16, 4, True)
    for h in range(hq):
        want = O.block_probs_head(Q[0, h], K[0, h // 2], 16, 4, True)
        np.testing.assert_allclose(P[0, h], want, rtol=0, atol=0)
    wrong = O.block_probs_head(Q[0, 1], K[0, 1], 16, 4, True)
    assert np.max(np.abs(wrong - P[0, 1])) > 1e-6


def test_q_block_subset_equals_full():
    """Filling only some query blocks gives the same rows as the full run."""
    q, k = _rand(512, 8), _rand(512, 8)
    full = O.block_probs_head(q, k, 64, 8, True, chunk_rows=16)
    part = O.block_probs_head(q, k, 64, 8, True, q_blocks=[0, 3, 7])
    for b in (0, 3, 7):
        np.testing.assert_allclose(part[b], full[b], rtol=0, atol=1e-14)


# ------------------------------------------------- sampling patterns --------
def _random_perm(S, seed):
    return [int(x) for x in np.random.default_rng(seed).permutation(S)]


@pytest.mark.parametrize("S", [1, 2, 4, 8])
@pytest.mark.parametrize("kind", ["antidiagonal", "diagonal", "random"])
def test_pattern_reshape_equals_bruteforce(S, kind):
    """The generalised reshape samples exactly the cells a == perm[b] of every
    S x S tile (query offset a, key offset b), checked cell by cell."""
    perm = {"antidiagonal": O.antidiagonal_perm(S), "diagonal": O.diagonal_perm(S),
            "random": _random_perm(S, S)}[kind]
    q, k = _rand(32, 4), _rand(32, 4)
    got = O.reshaped_logits(q, k, S, perm)
    want = O.pattern_sums_bruteforce(q, k, S, perm)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_default_pattern_is_the_antidiagonal():
    """No permutation means the antidiagonal (lower-left to upper-right)."""
    q, k = _rand(32, 4), _rand(32, 4)
    np.testing.assert_array_equal(O.reshaped_logits(q, k, 4),
                                  O.reshaped_logits(q, k, 4, [3, 2, 1, 0]))
    np.testing.assert_allclose(O.reshaped_logits(q, k, 4),
                               O.antidiagonal_sums_bruteforce(q, k, 4), rtol=0, atol=1e-12)


@pytest.mark.parametrize("delta,seen", [(0, True), (4, True), (1, False), (3, False)])
def test_diagonal_pattern_parity(delta, seen):
    """The main-diagonal pattern only pairs q, k with q - k = 0 (mod S): a
    planted slash at an offset that is a multiple of S is seen, any other is
    not (the opposite of the antidiagonal's odd-offset rule for S = 4)."""
    S, L, d = 4, 64, 16
    q = np.zeros((L, d))
    k = np.zeros((L, d))
    for i in range(L):
        q[i, i % d] = 1.0
    for j in range(L):
        if j + delta < L:
            k[j, (j + delta) % d] = 1.0
    x = O.reshaped_logits(q, k, S, O.diagonal_perm(S))
    assert (np.abs(x).sum() > 0) == seen


def test_perm_must_be_a_permutation():
    with pytest.raises(ValueError):
        O.reshape_queries(_rand(8, 2), 4, [0, 0, 1, 2])
    with pytest.raises(ValueError):
        O.reshape_queries(_rand(8, 2), 4, [0, 1, 2])


@pytest.mark.parametrize("causal", [True, False])
def test_pattern_rows_are_distributions(causal):
    """Any sampling pattern still gives rows of P that sum to 1, and causal P
    is 0 above the diagonal."""
    q, k = _rand(256, 8), _rand(256, 8)
    P = O.block_probs_head(q, k, 32, 8, causal, perm=_random_perm(8, 7))
    np.testing.assert_allclose(P.sum(axis=1), 1.0, rtol=0, atol=1e-12)
    if causal:
        assert np.all(np.triu(P, 1) == 0)


# --------------------------------------------- Top-K and Top-Ratio ----------
def _dyadic_row(n, r):
    """Probabilities that are multiples of 1/64 (sums are exact), with ties."""
    return r.integers(0, 6, size=n) / 64.0


@pytest.mark.parametrize("trial", range(30))
def test_top_k_bruteforce(trial):
    """Top-K keeps the k-subset with the largest sum; among those, the one
    whose ascending index tuple is smallest (ties go to the lower index).
    Checked against every k-subset of a small row."""
    r = np.random.default_rng(100 + trial)
    n = int(r.integers(1, 10))
    p = _dyadic_row(n, r)
    k = int(r.integers(1, n + 2))
    got = tuple(int(x) for x in O.top_k_blocks(p, k))
    if k >= n:
        assert got == tuple(range(n))
        return
    best = None
    for sub in itertools.combinations(range(n), k):
        key = (-sum(p[list(sub)]), sub)
        if best is None or key < best:
            best = key
    assert got == best[1]


def test_top_k_is_the_threshold_set_of_the_same_size():
    """For any tau, find_blocks keeps exactly the Top-K set with k = its size
    (both rank by probability, then index)."""
    r = np.random.default_rng(5)
    for _ in range(50):
        p = r.dirichlet(np.ones(40) * 0.3)
        p[r.integers(0, 40, 5)] = p[3]  # ties
        tau = float(r.uniform(0.1, 0.99))
        sel = O.find_blocks(p, tau)
        np.testing.assert_array_equal(O.top_k_blocks(p, len(sel)), sel)


def test_top_k_rejects_nonpositive_k():
    with pytest.raises(ValueError):
        O.top_k_blocks(np.ones(4) / 4, 0)


def test_top_ratio_count_exact():
    """The rounded count equals round-half-up of the exact rational product
    of the fp32 ratio and n (Fraction arithmetic), clamped to [1, n]."""
    from fractions import Fraction
    ratios = [0.27, 0.5, 0.1, 0.3, 1.0, 0.999, 1e-9, 0.0625, 0.7, 1 / 3, 0.25, 0.125]
    for ratio in ratios:
        fr = Fraction(float(np.float32(ratio)))
        for n in list(range(1, 70)) + [127, 128, 255, 1000, 1024, 2048, 4095, 4096]:
            x = fr * n
            want = int((x + Fraction(1, 2)).__floor__())
            want = max(1, min(n, want))
            assert O.top_ratio_count(ratio, n) == want, (ratio, n)
    # halves go up: 0.5 * 3 = 1.5 -> 2; 0.25 * 2 = 0.5 -> 1
    assert O.top_ratio_count(0.5, 3) == 2
    assert O.top_ratio_count(0.25, 2) == 1
    assert O.top_ratio_count(0.27, 100) == 27


@pytest.mark.parametrize("causal", [True, False])
def test_select_topk_and_topratio_rows(causal):
    """Row counts follow min(k, allowed) and the rounded ratio; the kept
    blocks are allowed ones and outrank every dropped allowed block."""
    r = np.random.default_rng(11)
    NB = 20
    P = np.zeros((1, 2, NB, NB))
    for h in range(2):
        for b in range(NB):
            n = b + 1 if causal else NB
            P[0, h, b, :n] = r.dirichlet(np.ones(n))
    for kind, arg in (("k", [3, 7]), ("ratio", [0.27, 0.6])):
        if kind == "k":
            mask, lists = O.select_blocks_topk(P, arg, causal)
        else:
            mask, lists = O.select_blocks_topratio(P, arg, causal)
        for h in range(2):
            for b in range(NB):
                n = b + 1 if causal else NB
                want_n = min(arg[h], n) if kind == "k" else O.top_ratio_count(arg[h], n)
                sel = lists[(0, h, b)]
                assert len(sel) == want_n and mask[0, h, b].sum() == want_n
                assert np.all(sel < n)
                dropped = np.setdiff1d(np.arange(n), sel)
                if len(dropped):
                    assert P[0, h, b, sel].min() >= P[0, h, b, dropped].max()


# ------------------------------------------------- short last block (L % B) --
# A length that is not a multiple of B ends in a shorter last block. These pins
# check the oracle's reading of that case against facts from outside it.

@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("S", [2, 4, 8])
def test_short_last_block_rows_are_distributions(causal, S):
    """L = 232 with B = 32: NB = 8 and the last block has 8 tokens. Every row
    of P, the short one included, still sums to 1 (a divisor of r instead of
    the block's own row count would give 8/32 on the last row)."""
    q, k = _rand(232, 16), _rand(232, 16)
    P = O.block_probs_head(q, k, 32, S, causal)
    assert P.shape == (8, 8)
    np.testing.assert_allclose(P.sum(axis=1), 1.0, rtol=0, atol=1e-12)
    assert (P >= 0).all()
    if causal:
        assert np.all(P[np.triu_indices(8, 1)] == 0.0)


@pytest.mark.parametrize("causal", [True, False])
def test_short_last_block_stride_one_is_exact_attention(causal):
    """S = 1, L = 44, B = 8: the last block has 4 tokens. P[b, j] is the mean
    over block b's queries of the naive attention mass on block j's keys."""
    L, B = 44, 8
    q, k = _rand(L, 4), _rand(L, 4)
    P = O.block_probs_head(q, k, B, 1, causal)
    _, probs = O.dense_attention_naive(q, k, np.zeros((L, 1)), causal)
    NB = 6
    want = np.zeros((NB, NB))
    for i in range(L):
        for j in range(L):
            want[i // B, j // B] += probs[i, j]
    for b in range(NB):
        want[b] /= min(B, L - b * B)
    np.testing.assert_allclose(P, want, rtol=0, atol=1e-12)


@pytest.mark.parametrize("S", [2, 4])
def test_short_last_block_causal_rows_ignore_the_tail(S):
    """Causal: the rows of the whole blocks see no token after their block, so
    they equal the P of the sequence cut after its last whole block."""
    q, k = _rand(232, 8), _rand(232, 8)
    P = O.block_probs_head(q, k, 32, S, True)
    Pc = O.block_probs_head(q[:224], k[:224], 32, S, True)
    np.testing.assert_allclose(P[:7, :7], Pc, rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [True, False])
def test_short_last_block_dense_mask_is_naive_attention(causal):
    """L = 28, B = 8 (last block: 4 tokens): attention over every allowed
    block equals the naive triple loop over the 28 keys."""
    L, B, NB = 28, 8, 4
    q, k, v = _rand(L, 4), _rand(L, 4), _rand(L, 3)
    lists = {b: list(range(b + 1 if causal else NB)) for b in range(NB)}
    Os, lse = O.sparse_attention_head(q, k, v, B, causal, lists)
    On, _ = O.dense_attention_naive(q, k, v, causal)
    np.testing.assert_allclose(Os, On, rtol=0, atol=1e-12)
    raw = O.dense_scores(q, k) / math.sqrt(4)
    for i in range(L):
        n = i + 1 if causal else L
        want = math.log(math.fsum(math.exp(x) for x in raw[i, :n]))
        assert abs(lse[i] - want) < 1e-12


@pytest.mark.parametrize("causal", [True, False])
def test_short_last_block_lists_match_filtered_naive_attention(causal):
    L, B, NB = 60, 8, 8
    q, k, v = _rand(L, 4), _rand(L, 4), _rand(L, 5)
    lists = {}
    for b in range(NB):
        n = b + 1 if causal else NB
        lists[b] = sorted({0} | {j for j in range(n) if rng.random() < 0.5})
    Os, _ = O.sparse_attention_head(q, k, v, B, causal, lists)
    On, _ = O.dense_attention_naive(q, k, v, causal,
                                    allowed=lambda i, j: (j // B) in lists[i // B])
    np.testing.assert_allclose(Os, On, rtol=0, atol=1e-12)


def test_short_last_block_batched_shapes():
    """The batched wrappers size P and O by ceil(L / B) blocks."""
    Q, K, V = _rand(1, 2, 40, 4), _rand(1, 1, 40, 4), _rand(1, 1, 40, 4)
    P = O.block_probs(Q, K, 16, 4, True)
    assert P.shape == (1, 2, 3, 3)
    _, lists = O.select_blocks(P, [0.9, 1.0], True)
    Os, lse = O.sparse_attention(Q, K, V, 16, True, lists)
    assert Os.shape == (1, 2, 40, 4) and np.isfinite(Os).all() and np.isfinite(lse).all()


# ------------------------------------------- batched wrappers (GQA, tau) ----
def _gqa_inputs():
    """hq = 4 query heads over hkv = 2 KV heads, batch 2, with K and V of each
    KV head and batch entry drawn apart (V scaled so it can never pass for K)."""
    b, hq, hkv, L, d = 2, 4, 2, 48, 4
    Q = _rand(b, hq, L, d)
    K = _rand(b, hkv, L, d)
    V = _rand(b, hkv, L, d, scale=5.0)
    K[:, 1] += 2.0
    V[1] -= 3.0
    return Q, K, V


def _random_lists(b, hq, NB, causal):
    lists = {}
    for bb in range(b):
        for h in range(hq):
            for qb in range(NB):
                n = qb + 1 if causal else NB
                lists[(bb, h, qb)] = sorted({0} | {j for j in range(n) if rng.random() < 0.5})
    return lists


@pytest.mark.parametrize("causal", [True, False])
def test_batched_sparse_attention_reads_the_gqa_kv_head(causal):
    """The batched attention wrapper gives query head h of batch entry bb the
    keys and values of KV head h // (hq / hkv) of the same entry (GQA, the
    mapping read into the pages). Pinned against the triple-loop attention on
    hand-picked operands, so a K/V swap, the h % hkv mapping or a batch mix-up
    in the wrapper fails here."""
    Q, K, V = _gqa_inputs()
    b, hq, L, _ = Q.shape
    hkv, B = K.shape[1], 16
    NB = L // B
    lists = _random_lists(b, hq, NB, causal)
    Os, lse = O.sparse_attention(Q, K, V, B, causal, lists)
    for bb in range(b):
        for h in range(hq):
            kv = h // (hq // hkv)
            want, _ = O.dense_attention_naive(
                Q[bb, h], K[bb, kv], V[bb, kv], causal,
                allowed=lambda i, j, bb=bb, h=h: (j // B) in lists[(bb, h, i // B)])
            np.testing.assert_allclose(Os[bb, h], want, rtol=0, atol=1e-12)
    # planted mistakes: each gives a different answer on these inputs
    h = 1
    for kk, vv in ((V[0, 0], K[0, 0]),             # K and V swapped
                   (K[0, h % hkv], V[0, h % hkv]),  # h % hkv instead of h // g
                   (K[1, 0], V[1, 0])):            # the other batch entry's KV head
        wrong, _ = O.dense_attention_naive(
            Q[0, h], kk, vv, causal,
            allowed=lambda i, j: (j // B) in lists[(0, h, i // B)])
        assert np.max(np.abs(wrong - Os[0, h])) > 1e-3


@pytest.mark.parametrize("causal", [True, False])
def test_batched_select_uses_each_heads_tau(causal):
    """The batched selection applies head h's own threshold tau[h] (per-head
    tau, §2.3 of the pages; an input of the hot path). Every row is checked
    against brute force over all subsets with that head's tau, and the rows
    of heads 1..3 would differ under tau[0]."""
    b, hq, NB = 2, 4, 7
    taus = [0.5, 0.7, 0.85, 0.97]
    P = np.zeros((b, hq, NB, NB))
    for bb in range(b):
        for h in range(hq):
            for qb in range(NB):
                n = qb + 1 if causal else NB
                P[bb, h, qb, :n] = rng.dirichlet(np.ones(n) * 0.7)
    mask, lists = O.select_blocks(P, taus, causal)
    differs = 0
    for bb in range(b):
        for h in range(hq):
            for qb in range(NB):
                n = qb + 1 if causal else NB
                row = list(P[bb, h, qb, :n])
                want = sorted(_brute_minimal(row, taus[h]))
                assert list(lists[(bb, h, qb)]) == want, (bb, h, qb)
                assert list(np.nonzero(mask[bb, h, qb])[0]) == want
                if h > 0 and sorted(_brute_minimal(row, taus[0])) != want:
                    differs += 1
    assert differs > 0   # tau[0] for every head would fail the rows above
