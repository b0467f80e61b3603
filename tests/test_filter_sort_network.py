"""The selection filter sorts up to 256 rank keys across a warp with a bitonic
network: KPL keys a lane, k[q] at position lane + 32 q. Partners closer than 32
positions are exchanged with warp shuffles (lane ^ stride), farther ones sit in
the same lane (q ^ stride / 32). This test runs that network stage by stage,
with the same index rules, on the host, and checks that it sorts any input
descending, duplicates and padding zeros included, for 1, 2, 4 and 8 keys a
lane. (The device network is also exercised end to end by the GPU selection
tests; this pins its structure for every size on inputs the GPU tests do not
reach.)
"""
import numpy as np
import pytest


def bitonic_desc(keys: np.ndarray, kpl: int) -> np.ndarray:
    """keys[lane, q] = the key at position lane + 32 q; returns the same layout
    after the network."""
    k = keys.copy()
    n = 32 * kpl
    lanes = np.arange(32)
    size = 2
    while size <= n:
        stride = size >> 1
        while stride > 0:
            if stride >= 32:
                qs = stride // 32
                for q in range(kpl):
                    if q & qs:
                        continue
                    up = ((lanes + 32 * q) & size) == 0
                    x, y = k[:, q].copy(), k[:, q | qs].copy()
                    hi, lo = np.maximum(x, y), np.minimum(x, y)
                    k[:, q] = np.where(up, hi, lo)
                    k[:, q | qs] = np.where(up, lo, hi)
            else:
                lower = (lanes & stride) == 0
                for q in range(kpl):
                    o = k[lanes ^ stride, q]        # __shfl_xor_sync(k[q], stride)
                    up = ((lanes + 32 * q) & size) == 0
                    take_max = up == lower
                    k[:, q] = np.where(take_max, np.maximum(o, k[:, q]), np.minimum(o, k[:, q]))
            stride >>= 1
        size <<= 1
    return k


def _positions(k):
    """Flatten [lane, q] into position order lane + 32 q."""
    return k.T.reshape(-1)


@pytest.mark.parametrize("kpl", [1, 2, 4, 8])
@pytest.mark.parametrize("seed", range(25))
def test_network_sorts_descending(kpl, seed):
    rng = np.random.default_rng(seed * 10 + kpl)
    n = 32 * kpl
    c = int(rng.integers(1, n + 1))          # candidates; the rest are padding zeros
    vals = rng.integers(1, 1 << 20, size=c, dtype=np.uint64)
    if seed % 3 == 0:
        vals = rng.integers(1, 6, size=c, dtype=np.uint64)   # many duplicates
    flat = np.zeros(n, dtype=np.uint64)
    flat[:c] = vals
    keys = flat.reshape(kpl, 32).T            # position lane + 32 q -> keys[lane, q]
    out = _positions(bitonic_desc(keys, kpl))
    assert np.array_equal(out, np.sort(flat)[::-1])


def test_layout_round_trip():
    kpl = 4
    flat = np.arange(32 * kpl, dtype=np.uint64)
    assert np.array_equal(_positions(flat.reshape(kpl, 32).T), flat)
