"""Plain fp64 CPU oracle for the XAttention prefill path.

TEST INFRASTRUCTURE. Only the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module. The product path (the CUDA library and its Python binding) never calls
it. The two share no code.

What it computes, step by step, following "XAttention: Block Sparse Attention
with Antidiagonal Scoring" (§2.1 Importance Prediction, §2.2 Threshold Block
Selection, Algorithm 1 "Block Selection"):

1. Reshape each query block and the keys by the stride S along the
   antidiagonal. Query rows i::S are stacked for i = S-1 down to 0; key rows
   i::S for i = 0 up to S-1. "Append" joins along the feature axis, so a
   reshaped row has length S*d.
2. A_approx = softmax(Q_r K_r^T / sqrt(d_h * S)) over the reshaped key axis,
   with the causal mask applied in the reshaped index space.
3. Block probabilities: A_approx summed over each (B/S) x (B/S) sub-block,
   divided by B/S so that each row of P sums to 1. This is the normalisation
   under which the threshold tau in (0, 1] makes sense.
4. find_blocks: the smallest set of blocks whose probabilities sum to at least
   tau, with ties broken toward the lower block index.
5. Block-sparse attention: softmax(q . k / sqrt(d)) v over the keys of the
   selected blocks only (token-causal inside the diagonal block).

Readings where the pages are silent or garbled:
* "append" joins features, not rows (the sqrt(d_h * S) scale only fits a
  length S*d dot product).
* Causal in the reshaped space keeps reshaped key column c for reshaped query
  row rho when c <= rho. The diagonal S x S tile is kept whole.
* The comparison is ">= tau" (the find_blocks formula in §2.2); the "> tau"
  in two secondary pages is not used.
* tau >= 1, or a cumulative sum that never reaches tau, selects every allowed
  block.
* GQA: query head h reads KV head h // (Hq / Hkv).
* A sequence whose length L is not a multiple of B (Algorithm 1 only walks
  floor(L/B) whole blocks) ends in a shorter last block: NB = ceil(L/B), and
  the last query / key block holds the L - (NB-1)B remaining tokens. L must be
  a multiple of S, so every reshaped row and column is whole. The softmax rows
  run over the L/S reshaped columns that exist, and P[b, j] divides by the
  number of reshaped rows block b actually has (r for a whole block), so every
  row of P still sums to 1.

Everything runs in float64. bf16 and fp32 inputs convert to float64 exactly.
Matrix products go through numpy's matmul (a library primitive); everything
else is written out.
"""
from __future__ import annotations

import math
from typing import Iterable, Sequence

import numpy as np

__all__ = [
    "to_f64", "reshape_queries", "reshape_keys", "reshaped_logits",
    "approx_attention_rows", "block_probs_head", "block_probs",
    "find_blocks", "select_blocks", "sparse_attention_head",
    "sparse_attention", "dense_attention_naive", "dense_scores",
    "antidiagonal_sums_bruteforce", "kv_head",
    "antidiagonal_perm", "diagonal_perm", "check_perm", "top_k_blocks",
    "top_ratio_count", "select_blocks_topk", "select_blocks_topratio",
    "pattern_sums_bruteforce",
]


def to_f64(x) -> np.ndarray:
    """Exact conversion of a torch tensor (fp32 / bf16) or array to float64."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


def kv_head(h: int, hq: int, hkv: int) -> int:
    """GQA head mapping: query head h reads KV head h // (hq / hkv)."""
    return h // (hq // hkv)


# --------------------------------------------------------------------------
# Step 1: strided antidiagonal reshape (§2.1; Algorithm 1, reshape loops)
# --------------------------------------------------------------------------

def antidiagonal_perm(S: int) -> list:
    """Query sub-row of each feature chunk for the antidiagonal pattern.

    Chunk i pairs query sub-row S-1-i with key sub-row i: the cells (a, b) of
    an S x S tile with a + b = S - 1 (§2.1, lower-left to upper-right).
    """
    return [S - 1 - i for i in range(S)]


def diagonal_perm(S: int) -> list:
    """Chunk i pairs query sub-row i with key sub-row i: the main diagonal of
    every S x S tile (the "diagonal" pattern of the sparsity-pattern ablation,
    Knowl 9 of the chapterpal page, §3.4 Ablation Study)."""
    return list(range(S))


def check_perm(perm: Sequence[int], S: int) -> list:
    """perm as a list, after checking that it is a permutation of 0..S-1."""
    perm = [int(x) for x in perm]
    if sorted(perm) != list(range(S)):
        raise ValueError(f"not a permutation of 0..{S - 1}: {perm}")
    return perm


def reshape_queries(q: np.ndarray, S: int, perm: Sequence[int] | None = None) -> np.ndarray:
    """Q_reshaped for a slab of queries whose length is a multiple of S.

    The slices q[i::S] are joined along the features for i = S-1 down to 0,
    so reshaped row t is [q[tS+S-1], q[tS+S-2], ..., q[tS]].

    ``perm`` generalises the order: feature chunk i holds the slice
    q[perm[i]::S]. The default is the antidiagonal order perm[i] = S-1-i;
    perm[i] = i gives the main diagonal, and any other permutation one cell
    per row and per column of every S x S tile (a "random" pattern when the
    permutation is drawn at random).
    """
    n, d = q.shape
    assert n % S == 0
    perm = antidiagonal_perm(S) if perm is None else check_perm(perm, S)
    parts = [q[perm[i]::S, :] for i in range(S)]
    return np.concatenate(parts, axis=1)


def reshape_keys(k: np.ndarray, S: int) -> np.ndarray:
    """K_reshaped: the slices k[i::S] joined along features for i = 0..S-1.

    Reshaped row c is [k[cS], k[cS+1], ..., k[cS+S-1]].
    """
    n, d = k.shape
    assert n % S == 0
    parts = [k[i::S, :] for i in range(0, S)]
    return np.concatenate(parts, axis=1)


def reshaped_logits(q: np.ndarray, k: np.ndarray, S: int,
                    perm: Sequence[int] | None = None) -> np.ndarray:
    """Q_r K_r^T without the 1/sqrt(d_h S) scale (the raw antidiagonal sums,
    or the sums of the pattern ``perm`` selects)."""
    return reshape_queries(q, S, perm) @ reshape_keys(k, S).T


# --------------------------------------------------------------------------
# Step 2: A_approx (§2.2, the softmax of Algorithm 1)
# --------------------------------------------------------------------------

def approx_attention_rows(x_scaled: np.ndarray, row0: int, causal: bool) -> np.ndarray:
    """Row softmax of scaled reshaped logits.

    x_scaled[t, c] belongs to global reshaped query row row0 + t. With the
    causal mask, column c is kept only when c <= row0 + t.
    """
    x = np.array(x_scaled, dtype=np.float64, copy=True)
    if causal:
        rows = row0 + np.arange(x.shape[0])[:, None]
        cols = np.arange(x.shape[1])[None, :]
        x[cols > rows] = -np.inf
    m = np.max(x, axis=1, keepdims=True)
    e = np.exp(x - m)
    return e / np.sum(e, axis=1, keepdims=True)


# --------------------------------------------------------------------------
# Step 3: block probabilities (§2.2 block sums; tau in (0, 1])
# --------------------------------------------------------------------------

def block_probs_head(q: np.ndarray, k: np.ndarray, B: int, S: int, causal: bool,
                     q_blocks: Iterable[int] | None = None,
                     chunk_rows: int = 1024,
                     perm: Sequence[int] | None = None) -> np.ndarray:
    """P[b, j] for one head: the normalised block sums of A_approx.

    q, k: [L, d] float64. Returns an [NB, NB] array. With ``q_blocks`` given,
    only those rows are filled (the others stay NaN). Causal rows are 0 above
    the diagonal.

    Per query block b (Algorithm 1's loop), the reshaped query rows are
    rows [b*r, (b+1)*r) of the reshaped whole Q, where r = B/S (B is a
    multiple of S). So several blocks' reshaped logits can come from one
    matmul call. Every row is then masked, normalised and block-summed on its
    own, exactly as the per-block loop does.

    ``perm`` selects the sampling pattern inside each S x S tile (see
    reshape_queries); the default is the antidiagonal.
    """
    L, d = q.shape
    assert L % S == 0 and B % S == 0
    NB, r, R = -(-L // B), B // S, L // S
    scale = 1.0 / math.sqrt(d * S)
    Qr = reshape_queries(q, S, perm)
    Kr = reshape_keys(k, S)
    P = np.full((NB, NB), np.nan)
    blocks = list(range(NB)) if q_blocks is None else sorted(set(int(b) for b in q_blocks))
    per_chunk = max(1, chunk_rows // r)
    for i0 in range(0, len(blocks), per_chunk):
        group = blocks[i0:i0 + per_chunk]
        # reshaped rows of block b: [b*r, min((b+1)*r, R)); the last block may be short
        spans = [(b * r, min((b + 1) * r, R)) for b in group]
        rows = np.concatenate([np.arange(a, e) for a, e in spans])
        ncols = min((max(group) + 1) * r, R) if causal else R
        x = (Qr[rows] @ Kr[:ncols].T) * scale
        o = 0
        for (a, e), b in zip(spans, group):
            rb = e - a
            xb = x[o:o + rb]
            o += rb
            A = approx_attention_rows(xb, a, causal)
            nj = b + 1 if causal else NB
            # columns of key block j: [j*r, min((j+1)*r, R)); pad the missing
            # columns of a short last block with zeros, sum each sub-block,
            # then divide by the block's number of rows
            Ap = np.zeros((rb, nj * r))
            w = min(nj * r, A.shape[1])
            Ap[:, :w] = A[:, :w]
            blk = Ap.reshape(rb, nj, r).sum(axis=(0, 2)) / rb
            P[b, :] = 0.0
            P[b, :nj] = blk
    return P


def block_probs(Q, K, B: int, S: int, causal: bool, heads: Sequence[int] | None = None,
                q_blocks: Iterable[int] | None = None,
                perm: Sequence[int] | None = None) -> np.ndarray:
    """P for [batch, hq, L, d] queries and [batch, hkv, L, d] keys.

    Returns [batch, hq, NB, NB]. Heads outside ``heads`` are NaN.
    """
    Qf, Kf = to_f64(Q), to_f64(K)
    b_, hq, L, d = Qf.shape
    hkv = Kf.shape[1]
    NB = -(-L // B)
    out = np.full((b_, hq, NB, NB), np.nan)
    hs = range(hq) if heads is None else heads
    for bb in range(b_):
        for h in hs:
            out[bb, h] = block_probs_head(Qf[bb, h], Kf[bb, kv_head(h, hq, hkv)], B, S,
                                          causal, q_blocks, perm=perm)
    return out


# --------------------------------------------------------------------------
# Step 4: find_blocks (§2.2 formula; Algorithm 1's per-block selection)
# --------------------------------------------------------------------------

def find_blocks(p: np.ndarray, tau: float) -> np.ndarray:
    """Smallest set of blocks whose probabilities sum to at least tau.

    p holds the probabilities of the allowed blocks (index = block index).
    Blocks are taken in the order (probability descending, index ascending),
    and a block is taken while the sum of those already taken is below tau.
    If tau >= 1, or the sum never reaches tau, every allowed block is taken.
    Returns the chosen indices in ascending order.
    """
    p = np.asarray(p, dtype=np.float64)
    n = p.shape[0]
    if tau >= 1.0:
        return np.arange(n)
    order = np.lexsort((np.arange(n), -p))     # primary: -p, secondary: index
    csum = np.cumsum(p[order])                 # sequential fp64 accumulation
    reached = np.nonzero(csum >= tau)[0]
    if reached.size == 0:
        return np.arange(n)
    k = int(reached[0]) + 1
    return np.sort(order[:k])


def select_blocks(P: np.ndarray, tau: Sequence[float], causal: bool,
                  heads: Sequence[int] | None = None,
                  q_blocks: Iterable[int] | None = None):
    """Apply find_blocks to every (batch, head, query-block) row of P.

    P: [batch, hq, NB, NB]; tau: per query head. Causal row b allows blocks
    0..b, non-causal rows allow all NB. Returns (mask bool [batch, hq, NB, NB],
    lists dict (bb, h, b) -> ascending block indices).
    """
    P = np.asarray(P, dtype=np.float64)
    b_, hq, NB, _ = P.shape
    mask = np.zeros(P.shape, dtype=bool)
    lists = {}
    hs = range(hq) if heads is None else heads
    bs = range(NB) if q_blocks is None else q_blocks
    for bb in range(b_):
        for h in hs:
            for b in bs:
                n = b + 1 if causal else NB
                sel = find_blocks(P[bb, h, b, :n], float(tau[h]))
                mask[bb, h, b, sel] = True
                lists[(bb, h, b)] = sel
    return mask, lists


# --------------------------------------------------------------------------
# Step 4b: fixed-budget selection, the Top-K and Top-Ratio strategies of the
# selection-strategy ablation (Knowl 9 of the chapterpal page; §3.4 Ablation
# Study). The pages name them only; the readings used here:
# * both rank a row's allowed blocks like find_blocks (probability
#   descending, ties to the lower index) and keep a fixed number of them;
# * Top-K keeps k blocks per row (k counted in blocks; a token budget such as
#   K = 8192 is K / B blocks), or every allowed block when fewer are allowed;
# * Top-Ratio keeps ratio * n blocks of a row with n allowed blocks, rounded
#   to the nearest integer (halves up), and at least one block.
# --------------------------------------------------------------------------

def top_k_blocks(p: np.ndarray, k: int) -> np.ndarray:
    """The k allowed blocks of highest probability (ties: lower index first).

    Returns ascending indices; every allowed block when k >= len(p).
    """
    p = np.asarray(p, dtype=np.float64)
    n = p.shape[0]
    if k < 1:
        raise ValueError("k must be at least 1")
    order = np.lexsort((np.arange(n), -p))     # primary: -p, secondary: index
    return np.sort(order[:min(k, n)])


def top_ratio_count(ratio: float, n: int) -> int:
    """Blocks kept by Top-Ratio in a row with n allowed blocks.

    ratio is taken as an fp32 value (the type the boundary passes). The
    product ratio * n is exact in float64 (a 24-bit significand times an
    integer below 2^13), and so is adding 1/2 for every ratio the count can
    depend on, so floor(ratio * n + 1/2) is the exactly rounded count.
    """
    r = float(np.float32(ratio))
    if not (0.0 < r <= 1.0):
        raise ValueError("ratio must lie in (0, 1]")
    k = int(math.floor(r * n + 0.5))
    return max(1, min(n, k))


def _select_rows(P: np.ndarray, causal: bool, heads, q_blocks, choose):
    P = np.asarray(P, dtype=np.float64)
    b_, hq, NB, _ = P.shape
    mask = np.zeros(P.shape, dtype=bool)
    lists = {}
    hs = range(hq) if heads is None else heads
    bs = range(NB) if q_blocks is None else q_blocks
    for bb in range(b_):
        for h in hs:
            for b in bs:
                n = b + 1 if causal else NB
                sel = choose(P[bb, h, b, :n], h)
                mask[bb, h, b, sel] = True
                lists[(bb, h, b)] = sel
    return mask, lists


def select_blocks_topk(P: np.ndarray, k: Sequence[int], causal: bool,
                       heads: Sequence[int] | None = None,
                       q_blocks: Iterable[int] | None = None):
    """Top-K on every row of P ([batch, hq, NB, NB]); k is per query head.

    Returns (mask, lists) like select_blocks.
    """
    return _select_rows(P, causal, heads, q_blocks,
                        lambda row, h: top_k_blocks(row, int(k[h])))


def select_blocks_topratio(P: np.ndarray, ratio: Sequence[float], causal: bool,
                           heads: Sequence[int] | None = None,
                           q_blocks: Iterable[int] | None = None):
    """Top-Ratio on every row of P; ratio is per query head, in (0, 1]."""
    return _select_rows(
        P, causal, heads, q_blocks,
        lambda row, h: top_k_blocks(row, top_ratio_count(float(ratio[h]), row.shape[0])))


# --------------------------------------------------------------------------
# Step 5: block-sparse attention over the selected blocks
# --------------------------------------------------------------------------

def sparse_attention_head(q: np.ndarray, k: np.ndarray, v: np.ndarray, B: int,
                          causal: bool, block_lists: dict,
                          q_blocks: Iterable[int] | None = None):
    """softmax(q k^T / sqrt(d)) v over the keys of each query block's list.

    q, k, v: [L, d] float64; block_lists[b] = key-block indices for query
    block b. Inside a kept block, causal attention keeps keys k <= q. Returns
    (O [L, d], lse [L]) with NaN rows for query blocks not computed. A row
    with no visible key gets O = 0 and lse = -inf.
    """
    L, d = q.shape
    NB = -(-L // B)
    O = np.full((L, v.shape[1]), np.nan)
    lse = np.full(L, np.nan)
    blocks = range(NB) if q_blocks is None else q_blocks
    for b in blocks:
        kb = np.asarray(block_lists[b], dtype=np.int64)
        qi = np.arange(b * B, min((b + 1) * B, L))   # the last block may be short
        if kb.size == 0:
            O[qi] = 0.0
            lse[qi] = -np.inf
            continue
        keys = np.concatenate([np.arange(j * B, min((j + 1) * B, L)) for j in kb])
        logits = (q[qi] @ k[keys].T) / math.sqrt(d)
        if causal:
            logits[keys[None, :] > qi[:, None]] = -np.inf
        m = np.max(logits, axis=1, keepdims=True)
        empty = ~np.isfinite(m[:, 0])
        m[empty] = 0.0
        e = np.exp(logits - m)
        s = np.sum(e, axis=1, keepdims=True)
        with np.errstate(invalid="ignore", divide="ignore"):
            O[qi] = (e @ v[keys]) / s
            lse[qi] = (m + np.log(s))[:, 0]
        O[qi[empty]] = 0.0
        lse[qi[empty]] = -np.inf
    return O, lse


def sparse_attention(Q, K, V, B: int, causal: bool, lists: dict,
                     heads: Sequence[int] | None = None,
                     q_blocks: Iterable[int] | None = None):
    """Batched wrapper: lists[(bb, h, b)] = key blocks. Returns (O, lse)."""
    Qf, Kf, Vf = to_f64(Q), to_f64(K), to_f64(V)
    b_, hq, L, d = Qf.shape
    hkv = Kf.shape[1]
    O = np.full(Qf.shape[:3] + (Vf.shape[3],), np.nan)
    lse = np.full((b_, hq, L), np.nan)
    hs = range(hq) if heads is None else heads
    NB = -(-L // B)
    for bb in range(b_):
        for h in hs:
            kv = kv_head(h, hq, hkv)
            bl = {b: lists[(bb, h, b)] for b in (range(NB) if q_blocks is None else q_blocks)}
            O[bb, h], lse[bb, h] = sparse_attention_head(Qf[bb, h], Kf[bb, kv], Vf[bb, kv],
                                                         B, causal, bl, q_blocks)
    return O, lse


# --------------------------------------------------------------------------
# Independent plain routines used only to pin the above
# --------------------------------------------------------------------------

def dense_scores(q: np.ndarray, k: np.ndarray) -> np.ndarray:
    """Raw Q K^T written as explicit dot products (no matmul)."""
    n, m = q.shape[0], k.shape[0]
    out = np.zeros((n, m))
    for i in range(n):
        for j in range(m):
            out[i, j] = float(np.dot(q[i], k[j]))
    return out


def dense_attention_naive(q: np.ndarray, k: np.ndarray, v: np.ndarray, causal: bool,
                          allowed=None):
    """Triple-loop softmax(q k^T / sqrt(d)) v for small inputs.

    ``allowed(i, j)``, if given, is an extra key filter. Returns (O, probs),
    where probs is the full attention-probability matrix.
    """
    n, d = q.shape
    m = k.shape[0]
    probs = np.zeros((n, m))
    O = np.zeros((n, v.shape[1]))
    for i in range(n):
        logits = []
        for j in range(m):
            ok = (not causal or j <= i) and (allowed is None or allowed(i, j))
            logits.append(sum(q[i, t] * k[j, t] for t in range(d)) / math.sqrt(d) if ok else None)
        mx = max(x for x in logits if x is not None)
        w = [math.exp(x - mx) if x is not None else 0.0 for x in logits]
        s = sum(w)
        for j in range(m):
            probs[i, j] = w[j] / s
            O[i] += probs[i, j] * v[j]
    return O, probs


def antidiagonal_sums_bruteforce(q: np.ndarray, k: np.ndarray, S: int) -> np.ndarray:
    """Sum of q_a . k_b over the antidiagonal cells of every S x S tile.

    Tile (t, c) covers queries tS..tS+S-1 and keys cS..cS+S-1. Its
    antidiagonal runs from the lower-left cell to the upper-right one: local
    offsets (a, b) with a + b = S - 1.
    """
    n, m = q.shape[0], k.shape[0]
    out = np.zeros((n // S, m // S))
    for t in range(n // S):
        for c in range(m // S):
            acc = 0.0
            for a in range(S):
                for b in range(S):
                    if a + b == S - 1:
                        acc += float(np.dot(q[t * S + a], k[c * S + b]))
            out[t, c] = acc
    return out


def pattern_sums_bruteforce(q: np.ndarray, k: np.ndarray, S: int,
                            perm: Sequence[int]) -> np.ndarray:
    """Sum of q_a . k_b over the cells of every S x S tile that a pattern
    samples: local offsets (a, b) with a == perm[b] (b = key offset)."""
    n, m = q.shape[0], k.shape[0]
    out = np.zeros((n // S, m // S))
    for t in range(n // S):
        for c in range(m // S):
            acc = 0.0
            for a in range(S):
                for b in range(S):
                    if a == perm[b]:
                        acc += float(np.dot(q[t * S + a], k[c * S + b]))
            out[t, c] = acc
    return out
