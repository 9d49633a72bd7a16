"""The C-ABI library builds for sm_100a, loads, and exports every call include/dsa.h
declares.  No compute call is made (no GPU here); only host-side argument checks that
return before any device access are exercised."""
import ctypes
import os
import re

import pytest

from sparse_long_context_dsa_b200 import build as B
from sparse_long_context_dsa_b200 import dsa

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "dsa.h")


def declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(dsa_[a-z_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    B.build()
    return dsa.lib()


def test_every_declared_symbol_is_exported(lib):
    names = declared()
    assert len(names) >= 11
    raw = ctypes.CDLL(dsa.LIB_PATH)
    for n in names:
        assert hasattr(raw, n), n
    assert sorted(dsa.exported_symbols()) == names


def test_version(lib):
    assert lib.dsa_version() == 100


def test_workspace_sizes_are_host_only(lib):
    assert lib.dsa_topk_workspace_size(0, 10, 4) == 0
    a = lib.dsa_topk_workspace_size(1, 131072, 512)
    b = lib.dsa_topk_workspace_size(2, 131072, 512)
    assert a > 4 * 131072 * 8 and b > a and a % 256 == 0
    assert lib.dsa_indexer_workspace_size(8, 16384) == 0


@pytest.mark.parametrize("call", [
    lambda L: L.dsa_topk_regions(None, 16, None, 1, 0, None, None, None, 0, None),        # k = 0
    lambda L: L.dsa_topk_regions(None, 16, None, 1, 4096, None, None, None, 0, None),     # k too large
    lambda L: L.dsa_topk_regions(None, 1 << 21, None, 1, 8, None, None, None, 0, None),   # ld too large
    lambda L: L.dsa_compress_regions(None, 1024, 8, None, None, -1, None, None, 1, None),  # n < 0
    lambda L: L.dsa_compress_regions(None, 1000, 8, None, None, 1, None, None, 1, None),  # NULL / stride
    lambda L: L.dsa_indexer_scores(None, None, None, None, 1, None, None, 4, None, 1, None, 8, 2, None, 0, None),
    lambda L: L.dsa_sparse_attn_decode(None, None, None, 1, None, 1, None, 1, None, None, 0, None, None, None, 0,
                                       None),
])
def test_bad_arguments_are_rejected_on_the_host(lib, call):
    assert call(lib) == dsa.ERR_INVALID_ARG
    assert lib.dsa_last_error().decode()


def test_last_error_copied_into_a_caller_buffer(lib):
    assert lib.dsa_topk_regions(None, 16, None, 1, 0, None, None, None, 0, None) == dsa.ERR_INVALID_ARG
    msg = lib.dsa_last_error()
    n = len(msg)
    assert n > 8
    assert lib.dsa_get_last_error(None, 0) == n                   # length only, nothing written
    buf = ctypes.create_string_buffer(b"x" * 8)                   # 9 bytes with its own NUL
    assert lib.dsa_get_last_error(buf, 5) == n                    # cut short: 4 bytes and a NUL
    assert buf.raw[:5] == msg[:4] + b"\0" and buf.raw[5:8] == b"xxx"
    big = ctypes.create_string_buffer(n + 1)
    assert lib.dsa_get_last_error(big, n + 1) == n and big.value == msg


def test_zero_sized_calls_are_noops(lib):
    assert lib.dsa_compress_regions(None, 1024, 8, None, None, 0, None, None, 1, None) == dsa.OK
    assert lib.dsa_topk_regions(None, 16, None, 0, 8, None, None, None, 0, None) == dsa.OK


def test_group_ranges_are_checked_on_the_host(lib):
    # a KV group shard is 1, 2 or 4 consecutive groups of 0 .. 3
    for g0, ng in ((0, 3), (3, 2), (-1, 1), (2, 4), (0, 0)):
        assert lib.dsa_decode_select_groups(None, None, None, None, 1, g0, ng, None, None, 1, None, 1, None, 8, 0, 8,
                                            None, None, None, 0, None) == dsa.ERR_INVALID_ARG
        assert lib.dsa_sparse_attn_decode_groups(None, None, None, 1, None, 1, None, 1, g0, ng, None, None, 8, None,
                                                 None, None, 0, None) == dsa.ERR_INVALID_ARG
        assert lib.dsa_compress_regions_groups(None, 1024, 8, None, None, 1, g0, ng, None, None, 1, None) == \
            dsa.ERR_INVALID_ARG
        assert "g0" in lib.dsa_last_error().decode() or "ng" in lib.dsa_last_error().decode()
    assert lib.dsa_attn_groups_workspace_size(4, 512, 3) == 0


def test_selftest_bound_is_checked_on_the_host(lib):
    assert lib.dsa_selftest_wait_timeout(0, None) == dsa.ERR_INVALID_ARG
    assert lib.dsa_selftest_wait_timeout((1 << 31) + 1, None) == dsa.ERR_INVALID_ARG
