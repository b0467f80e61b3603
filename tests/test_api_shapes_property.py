"""Shape validation of the C ABI, checked with random shapes on the CPU.

For any shape, every entry point must agree: a shape the rules reject is
refused with the same status by each call (before anything is launched, so
no GPU is needed), and a shape the rules accept gets workspace sizes that
match their definition. The rules are restated here independently of the
library: L and B multiples of S, hq a multiple of hkv, bf16 only with d = 128
and B = 128, at most 256 query heads and 4096 blocks.
"""
import ctypes

import pytest
from hypothesis import given, settings
from hypothesis import strategies as st

from block_sparse_long_score_b200 import build as xbuild
from block_sparse_long_score_b200 import xattn as X

FAKE = ctypes.c_void_p(0x10000)   # never dereferenced: only host checks run


@pytest.fixture(scope="module")
def lib():
    xbuild.build()
    return X._lib()


def expected_status(batch, hq, hkv, L, d, B, S, dtype):
    """The shape rules, written out on their own."""
    if min(batch, hq, hkv, L, d, B, S) < 1 or hq % hkv or L % S or B % S:
        return -1
    if hq > 256:
        return -2
    NB = -(-L // B)
    if NB > 4096 or batch * hq * L > 2**31 - 1 or batch * hq * NB > 2**24:
        return -2
    if dtype == "bf16":
        return 0 if (d == 128 and B == 128) else -2
    if d not in (32, 64, 128) or B > 256 or S * d * 4 > 48 * 1024:
        return -2
    return 0


shapes = st.tuples(
    st.integers(1, 3),                                   # batch
    st.sampled_from([1, 2, 3, 4, 8, 32, 300]),           # hq
    st.sampled_from([1, 2, 3, 4, 8]),                    # hkv
    st.integers(1, 70000),                               # L
    st.sampled_from([32, 64, 96, 128]),                  # d
    st.sampled_from([16, 64, 100, 128, 256, 512]),       # B
    st.sampled_from([1, 2, 3, 4, 8, 16, 64]),            # S
    st.booleans(),                                       # causal
    st.sampled_from(["bf16", "f32"]),
)


@settings(max_examples=300, deadline=None)
@given(shapes)
def test_every_entry_point_applies_the_same_rules(lib, shp):
    batch, hq, hkv, L, d, B, S, causal, dtype = shp
    s = X.make_shape(batch, hq, hkv, L, d, B, S, causal, dtype)
    want = expected_status(batch, hq, hkv, L, d, B, S, dtype)
    tau = (ctypes.c_float * max(hq, 1))(*([0.9] * max(hq, 1)))
    sref = ctypes.byref(s)
    if want == 0:
        NB = -(-L // B)
        r = B // S
        part = r * NB * (NB + 1) // 2 if causal else (L // S) * NB
        assert X.xattn_score_workspace_bytes(s) == batch * hq * part * 4 + 256
        assert X.xattn_attn_workspace_bytes(s) == 8 * (batch * hq * NB + 32)
        return
    assert X.xattn_score_workspace_bytes(s) == 0
    assert X.xattn_attn_workspace_bytes(s) == 0
    assert X.xattn_prefill_host_workspace_bytes(s, 0) == 0
    calls = [
        lib.xattn_score(FAKE, FAKE, sref, FAKE, FAKE, 1 << 40, None),
        lib.xattn_score_partials(FAKE, FAKE, sref, FAKE, 1 << 40, None),
        lib.xattn_score_select(FAKE, FAKE, sref, tau, None, FAKE, FAKE, FAKE, FAKE, 1 << 40,
                               None),
        lib.xattn_select(FAKE, tau, sref, FAKE, FAKE, FAKE, None),
        lib.xattn_sparse_attn(FAKE, FAKE, FAKE, sref, FAKE, FAKE, FAKE, None, FAKE, 1 << 40,
                              None),
        lib.xattn_sparse_attn_noalloc(FAKE, FAKE, FAKE, sref, FAKE, FAKE, FAKE, None, None),
        lib.xattn_prefill_host(FAKE, FAKE, FAKE, sref, tau, FAKE, None, 0, FAKE, 1 << 40, None),
    ]
    assert calls == [want] * len(calls), (shp, calls)
