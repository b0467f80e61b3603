"""C-ABI checks that need no GPU: the library loads, exports every entry point
that include/xattn.h declares, sizes its workspaces, and rejects bad
arguments on the host before launching anything."""
import ctypes
import os
import re

import pytest

from block_sparse_long_score_b200 import build as xbuild
from block_sparse_long_score_b200 import xattn as X

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FAKE = ctypes.c_void_p(0x10000)   # never dereferenced: every call below fails its host checks


@pytest.fixture(scope="module")
def lib():
    xbuild.build()
    return X._lib()


def _declared():
    src = open(os.path.join(ROOT, "include", "xattn.h")).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\*?\s+\*?(xattn_\w+)\s*\(", src, re.M)))


def test_exports_every_declared_symbol(lib):
    names = _declared()
    assert len(names) >= 7
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(X.EXPORTED_SYMBOLS)


def test_workspace_sizes(lib):
    s = X.make_shape(1, 32, 8, 131072, 128, 128, 16, True, "bf16")
    NB, r = 1024, 8
    assert X.xattn_score_workspace_bytes(s) == 32 * r * NB * (NB + 1) // 2 * 4 + 256
    assert X.xattn_attn_workspace_bytes(s) == 8 * (32 * NB + 32)
    nc = X.make_shape(1, 24, 24, 76800, 128, 128, 4, False, "bf16")
    assert X.xattn_score_workspace_bytes(nc) == 24 * (76800 // 4) * 600 * 4 + 256
    bad = X.make_shape(1, 32, 8, 1000, 128, 128, 16, True, "bf16")
    assert X.xattn_score_workspace_bytes(bad) == 0


@pytest.mark.parametrize("kw,code", [
    (dict(L=1004), -1),             # L % S != 0 (L % B != 0 alone is allowed)
    (dict(S=3), -1),                # B % S != 0
    (dict(hkv=3), -1),              # hq % hkv != 0
    (dict(d=64), -2),               # bf16 needs d = 128
    (dict(B=64, S=8), -2),          # bf16 needs B = 128
    (dict(hq=512, hkv=8), -2),      # too many heads
    (dict(L=128 * 8192), -2),       # NB above the maximum
])
def test_bad_shapes_rejected(lib, kw, code):
    a = dict(batch=1, hq=32, hkv=8, L=4096, d=128, B=128, S=8, causal=True, dtype="bf16")
    a.update(kw)
    s = X.make_shape(**a)
    rc = lib.xattn_score(FAKE, FAKE, ctypes.byref(s), FAKE, FAKE, 1 << 40, None)
    assert rc == code
    rc = lib.xattn_sparse_attn(FAKE, FAKE, FAKE, ctypes.byref(s), FAKE, FAKE, FAKE, None,
                               FAKE, 1 << 40, None)
    assert rc == code


def test_null_pointers_and_workspace(lib):
    s = X.make_shape(1, 4, 2, 1024, 128, 128, 8, True, "bf16")
    assert lib.xattn_score(None, FAKE, ctypes.byref(s), FAKE, FAKE, 1 << 40, None) == -1
    assert lib.xattn_score(FAKE, FAKE, ctypes.byref(s), FAKE, None, 1 << 40, None) == -4
    assert lib.xattn_score(FAKE, FAKE, ctypes.byref(s), FAKE, FAKE, 16, None) == -4
    assert lib.xattn_sparse_attn(FAKE, FAKE, FAKE, ctypes.byref(s), FAKE, FAKE, FAKE, None,
                                 FAKE, 8, None) == -4
    assert lib.xattn_score(FAKE, FAKE, None, FAKE, FAKE, 1 << 40, None) == -1


@pytest.mark.parametrize("tau", [0.0, -0.5, 1.5, float("nan")])
def test_tau_out_of_range(lib, tau):
    """The whole-step calls take tau in host memory and check it before any
    launch. (xattn_select and xattn_score_select read tau from device memory;
    the kernels check it there, which the GPU tests cover.)"""
    s = X.make_shape(1, 2, 2, 1024, 128, 128, 8, True, "bf16")
    t = (ctypes.c_float * 2)(0.9, tau)
    assert lib.xattn_prefill_host(FAKE, FAKE, FAKE, ctypes.byref(s), t, FAKE, None, 0, FAKE,
                                  1 << 40, None) == -1
    lens = (ctypes.c_int32 * 1)(1024)
    assert lib.xattn_prefill_varlen(FAKE, FAKE, FAKE, ctypes.byref(s), 1, lens, t, FAKE, None,
                                    FAKE, 1 << 40, None) == -1


def test_null_tau_refused(lib):
    s = X.make_shape(1, 2, 2, 1024, 128, 128, 8, True, "bf16")
    assert lib.xattn_select(FAKE, None, ctypes.byref(s), FAKE, FAKE, FAKE, None) == -1
    assert lib.xattn_score_select(FAKE, FAKE, ctypes.byref(s), None, None, FAKE, FAKE, FAKE,
                                  FAKE, 1 << 40, None) == -1


def test_misaligned_bf16_pointer(lib):
    s = X.make_shape(1, 4, 2, 1024, 128, 128, 8, True, "bf16")
    odd = ctypes.c_void_p(0x10008)
    assert lib.xattn_score(odd, FAKE, ctypes.byref(s), FAKE, FAKE, 1 << 40, None) == -1


def test_strerror(lib):
    assert X.xattn_strerror(0) == "ok"
    assert "timed out" in X.xattn_strerror(-5)
    assert X.xattn_strerror(42) == "unknown status"


@pytest.mark.parametrize("perm", [[0, 0, 1, 2, 3, 4, 5, 6], [0, 1, 2, 3, 4, 5, 6, 8],
                                  [-1, 1, 2, 3, 4, 5, 6, 7], None])
def test_bad_pattern_rejected(lib, perm):
    s = X.make_shape(1, 4, 2, 1024, 128, 128, 8, True, "bf16")
    arr = None if perm is None else (ctypes.c_int32 * 8)(*perm)
    assert lib.xattn_score_pattern(FAKE, FAKE, ctypes.byref(s), arr, FAKE, FAKE, 1 << 40,
                                   None) == -1


def test_pattern_checks_shape_and_workspace_first(lib):
    ok = (ctypes.c_int32 * 8)(*range(8))
    bad = X.make_shape(1, 4, 2, 1004, 128, 128, 8, True, "bf16")   # L % S != 0
    assert lib.xattn_score_pattern(FAKE, FAKE, ctypes.byref(bad), ok, FAKE, FAKE, 1 << 40,
                                   None) == -1
    s = X.make_shape(1, 4, 2, 1024, 128, 128, 8, True, "bf16")
    assert lib.xattn_score_pattern(FAKE, FAKE, ctypes.byref(s), ok, FAKE, FAKE, 16, None) == -4


@pytest.mark.parametrize("k", [0, -3])
def test_topk_out_of_range(lib, k):
    s = X.make_shape(1, 2, 2, 1024, 128, 128, 8, True, "bf16")
    arr = (ctypes.c_int32 * 2)(4, k)
    assert lib.xattn_select_topk(FAKE, arr, ctypes.byref(s), FAKE, FAKE, FAKE, None) == -1


@pytest.mark.parametrize("ratio", [0.0, -0.1, 1.5, float("nan")])
def test_topratio_out_of_range(lib, ratio):
    s = X.make_shape(1, 2, 2, 1024, 128, 128, 8, True, "bf16")
    arr = (ctypes.c_float * 2)(0.25, ratio)
    assert lib.xattn_select_topratio(FAKE, arr, ctypes.byref(s), FAKE, FAKE, FAKE, None) == -1


def test_budget_null_pointers(lib):
    s = X.make_shape(1, 2, 2, 1024, 128, 128, 8, True, "bf16")
    k = (ctypes.c_int32 * 2)(4, 4)
    r = (ctypes.c_float * 2)(0.5, 0.5)
    assert lib.xattn_select_topk(None, k, ctypes.byref(s), FAKE, FAKE, FAKE, None) == -1
    assert lib.xattn_select_topk(FAKE, None, ctypes.byref(s), FAKE, FAKE, FAKE, None) == -1
    assert lib.xattn_select_topratio(FAKE, r, ctypes.byref(s), FAKE, None, FAKE, None) == -1


def test_score_select_host_checks(lib):
    s = X.make_shape(1, 2, 2, 1024, 128, 128, 8, True, "bf16")
    good = FAKE   # tau is a device pointer here: its values are checked by the kernels
    f = lib.xattn_score_select
    assert f(FAKE, FAKE, ctypes.byref(s), None, None, FAKE, FAKE, FAKE, FAKE, 1 << 40, None) == -1
    assert f(FAKE, FAKE, ctypes.byref(s), good, None, None, FAKE, FAKE, FAKE, 1 << 40, None) == -1
    assert f(None, FAKE, ctypes.byref(s), good, None, FAKE, FAKE, FAKE, FAKE, 1 << 40, None) == -1
    assert f(FAKE, FAKE, ctypes.byref(s), good, None, FAKE, FAKE, FAKE, FAKE, 16, None) == -4
    odd = ctypes.c_void_p(0x10008)
    assert f(odd, FAKE, ctypes.byref(s), good, None, FAKE, FAKE, FAKE, FAKE, 1 << 40, None) == -1


def _r256(x):
    return (x + 255) // 256 * 256


@pytest.mark.parametrize("ck", [0, 1, 3, 8])
def test_prefill_host_workspace_size(lib, ck):
    """Two slots of one chunk's Q, K, V, O and lse, plus one chunk's selection
    outputs and the two steps' workspaces."""
    s = X.make_shape(1, 32, 8, 131072, 128, 128, 16, True, "bf16")
    c = max(ck, 1)
    hq_c, L, NB = 4 * c, 131072, 1024
    row = L * 128 * 2
    cs = X.make_shape(1, hq_c, c, L, 128, 128, 16, True, "bf16")
    slot = _r256(hq_c * row) * 2 + _r256(c * row) * 2 + _r256(hq_c * L * 4)
    want = 2 * slot + _r256(hq_c * NB * 32 * 4) + _r256(hq_c * NB * 4) + \
        _r256(hq_c * NB * NB * 4) + _r256(X.xattn_score_workspace_bytes(cs)) + \
        _r256(X.xattn_attn_workspace_bytes(cs))
    assert X.xattn_prefill_host_workspace_bytes(s, ck) == want


def test_prefill_host_checks(lib):
    s = X.make_shape(2, 4, 2, 1024, 128, 128, 8, True, "bf16")
    good = (ctypes.c_float * 4)(0.9, 0.9, 0.9, 0.9)
    bad = (ctypes.c_float * 4)(0.9, 0.0, 0.9, 0.9)
    f = lib.xattn_prefill_host
    big = 1 << 40
    assert X.xattn_prefill_host_workspace_bytes(s, -1) == 0
    assert X.xattn_prefill_host_workspace_bytes(s, 3) == 0      # more than hkv
    assert f(None, FAKE, FAKE, ctypes.byref(s), good, FAKE, None, 0, FAKE, big, None) == -1
    assert f(FAKE, FAKE, FAKE, ctypes.byref(s), good, None, None, 0, FAKE, big, None) == -1
    assert f(FAKE, FAKE, FAKE, ctypes.byref(s), None, FAKE, None, 0, FAKE, big, None) == -1
    assert f(FAKE, FAKE, FAKE, ctypes.byref(s), bad, FAKE, None, 0, FAKE, big, None) == -1
    assert f(FAKE, FAKE, FAKE, ctypes.byref(s), good, FAKE, None, -1, FAKE, big, None) == -1
    assert f(FAKE, FAKE, FAKE, ctypes.byref(s), good, FAKE, None, 3, FAKE, big, None) == -1
    assert f(FAKE, FAKE, FAKE, None, good, FAKE, None, 0, FAKE, big, None) == -1
    need = X.xattn_prefill_host_workspace_bytes(s, 0)
    assert f(FAKE, FAKE, FAKE, ctypes.byref(s), good, FAKE, None, 0, None, big, None) == -4
    assert f(FAKE, FAKE, FAKE, ctypes.byref(s), good, FAKE, None, 0, FAKE, need - 1, None) == -4
    odd = ctypes.c_void_p(0x10080)                               # not 256-byte aligned
    assert f(FAKE, FAKE, FAKE, ctypes.byref(s), good, FAKE, None, 0, odd, big, None) == -4
    wide = X.make_shape(1, 4, 2, 1024, 64, 128, 8, True, "bf16")  # bf16 needs d = 128
    assert f(FAKE, FAKE, FAKE, ctypes.byref(wide), good, FAKE, None, 0, FAKE, big, None) == -2


def test_misaligned_score_workspace_rejected(lib):
    """The scoring workspace holds fp32 partials: a workspace pointer that is
    not 4-byte aligned is refused on the host (INVALID_ARG), by both scoring
    calls, before any device work."""
    s = X.make_shape(1, 4, 2, 1024, 128, 128, 8, True, "bf16")
    need = X.xattn_score_workspace_bytes(s)
    bad_ws = ctypes.c_void_p(0x10002)
    assert lib.xattn_score(FAKE, FAKE, ctypes.byref(s), FAKE, bad_ws, need, None) == -1
    assert lib.xattn_score_select(FAKE, FAKE, ctypes.byref(s), FAKE, None, FAKE, FAKE, FAKE,
                                  bad_ws, need, None) == -1
    assert lib.xattn_score_partials(FAKE, FAKE, ctypes.byref(s), bad_ws, need, None) == -1


def test_score_partials_host_checks(lib):
    """xattn_score_partials applies xattn_score's host checks: NULL inputs are
    INVALID_ARG, a missing or short workspace is WORKSPACE, all before any
    device work."""
    s = X.make_shape(1, 4, 2, 1024, 128, 128, 8, True, "bf16")
    need = X.xattn_score_workspace_bytes(s)
    assert lib.xattn_score_partials(None, FAKE, ctypes.byref(s), FAKE, need, None) == -1
    assert lib.xattn_score_partials(FAKE, None, ctypes.byref(s), FAKE, need, None) == -1
    assert lib.xattn_score_partials(FAKE, FAKE, ctypes.byref(s), None, need, None) == -4
    assert lib.xattn_score_partials(FAKE, FAKE, ctypes.byref(s), FAKE, need - 1, None) == -4
    assert lib.xattn_score_partials(FAKE, FAKE, None, FAKE, need, None) == -1


def test_ragged_length_accepted(lib):
    """L = 1000 (not a multiple of B = 128, a multiple of S = 8): 8 blocks,
    the last of 104 tokens. The host checks pass (the call then fails only on
    the missing workspace)."""
    s = X.make_shape(1, 4, 2, 1000, 128, 128, 8, True, "bf16")
    NB, r = 8, 16
    assert X.xattn_score_workspace_bytes(s) == 4 * r * NB * (NB + 1) // 2 * 4 + 256
    assert X.xattn_attn_workspace_bytes(s) == 8 * (4 * NB + 32)
    assert lib.xattn_score(FAKE, FAKE, ctypes.byref(s), FAKE, None, 0, None) == -4


def _varlen(lib, shape, lens):
    arr = (ctypes.c_int32 * len(lens))(*lens)
    return lib.xattn_prefill_varlen_workspace_bytes(ctypes.byref(shape), len(lens), arr), arr


def test_varlen_workspace_is_the_longest_sequences_per_lane(lib):
    s = X.make_shape(7, 4, 2, 1, 128, 128, 8, True, "bf16")   # batch and L are ignored
    got, _ = _varlen(lib, s, [1000, 4096, 0, 512])
    one = X.make_shape(1, 4, 2, 4096, 128, 128, 8, True, "bf16")
    NB = 32
    lane = _r256(4 * NB * 1 * 4) + _r256(4 * NB * 4) + _r256(4 * NB * NB * 4) + \
        _r256(X.xattn_score_workspace_bytes(one)) + _r256(X.xattn_attn_workspace_bytes(one))
    assert got == 3 * lane                       # three non-empty sequences: three lanes
    many, _ = _varlen(lib, s, [4096] + [128] * 9)
    assert many == 4 * lane                      # at most four lanes


@pytest.mark.parametrize("lens,code", [
    ([], -1), ([0, 0], -1), ([128, -8], -1), ([128, 100], -1),   # 100 % S != 0
    ([128, 128 * 4097], -2),                                    # too many blocks
])
def test_varlen_bad_lengths(lib, lens, code):
    s = X.make_shape(1, 4, 2, 1, 128, 128, 8, True, "bf16")
    arr = (ctypes.c_int32 * max(len(lens), 1))(*lens)
    assert lib.xattn_prefill_varlen_workspace_bytes(ctypes.byref(s), len(lens), arr) == 0
    t = (ctypes.c_float * 4)(0.9, 0.9, 0.9, 0.9)
    rc = lib.xattn_prefill_varlen(FAKE, FAKE, FAKE, ctypes.byref(s), len(lens), arr, t, FAKE,
                                  None, FAKE, 1 << 40, None)
    assert rc == code


def test_varlen_host_checks(lib):
    s = X.make_shape(1, 4, 2, 1, 128, 128, 8, True, "bf16")
    need, arr = _varlen(lib, s, [128, 1000])
    good = (ctypes.c_float * 4)(0.9, 0.9, 0.9, 0.9)
    bad = (ctypes.c_float * 4)(0.9, 0.9, 1.5, 0.9)
    f = lib.xattn_prefill_varlen
    big = 1 << 40
    assert f(None, FAKE, FAKE, ctypes.byref(s), 2, arr, good, FAKE, None, FAKE, big, None) == -1
    assert f(FAKE, FAKE, FAKE, ctypes.byref(s), 2, arr, good, None, None, FAKE, big, None) == -1
    assert f(FAKE, FAKE, FAKE, ctypes.byref(s), 2, arr, None, FAKE, None, FAKE, big, None) == -1
    assert f(FAKE, FAKE, FAKE, ctypes.byref(s), 2, arr, bad, FAKE, None, FAKE, big, None) == -1
    assert f(FAKE, FAKE, FAKE, ctypes.byref(s), 2, None, good, FAKE, None, FAKE, big, None) == -1
    assert f(FAKE, FAKE, FAKE, ctypes.byref(s), 2, arr, good, FAKE, None, None, big, None) == -4
    assert f(FAKE, FAKE, FAKE, ctypes.byref(s), 2, arr, good, FAKE, None, FAKE, need - 1,
             None) == -4
    odd = ctypes.c_void_p(0x10080)
    assert f(FAKE, FAKE, FAKE, ctypes.byref(s), 2, arr, good, FAKE, None, odd, big, None) == -4


def test_check_lists_host_checks(lib):
    """xattn_check_lists rejects a bad shape or a NULL pointer before any CUDA call."""
    s = X.make_shape(1, 2, 2, 1024, 128, 128, 1, True, "bf16")
    bad = X.make_shape(1, 2, 2, 1004, 128, 128, 8, True, "bf16")   # L not a multiple of S
    assert lib.xattn_check_lists(FAKE, FAKE, ctypes.byref(bad), FAKE, None) == -1
    assert lib.xattn_check_lists(None, FAKE, ctypes.byref(s), FAKE, None) == -1
    assert lib.xattn_check_lists(FAKE, None, ctypes.byref(s), FAKE, None) == -1
    assert lib.xattn_check_lists(FAKE, FAKE, ctypes.byref(s), None, None) == -1
    assert lib.xattn_check_lists(FAKE, FAKE, None, FAKE, None) == -1
