"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every symbol include/csa2.h declares, reports sizes, and rejects invalid
arguments before enqueuing anything."""
import ctypes as C
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def csa2():
    from csa2_sparse_attention_decode_b200 import build
    build.build()
    import csa2_sparse_attention_decode_b200 as m
    return m


def _declared():
    names = set()
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            src = open(os.path.join(ROOT, "include", f)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(csa2_[a-z0-9_]+)\s*\(", src))
    return names


def test_every_declared_symbol_is_exported(csa2):
    decl = _declared()
    assert {"csa2_prefill", "csa2_append", "csa2_index", "csa2_attend", "csa2_get_device_error"} <= decl
    lib = C.CDLL(csa2.LIB_PATH)
    for n in decl:
        assert hasattr(lib, n), n
    assert decl >= set(csa2.EXPORTS)


def test_sizes(csa2):
    assert csa2.csa2_page_bytes() == 64 * 256 + 64 * 32 + 64 * 128 + 8 * 128 == 27648
    assert csa2.csa2_swa_bytes() == 128 * 512 + 128 * 4
    ws = csa2.csa2_workspace_bytes(4, 1 << 20)
    # scan scores + selected blocks + the scan's key range per request
    need = 4 * (1 << 20) * 4 + 4 * 2048 * 4 + 4 * 512
    assert need <= ws <= need + 3 * 256
    assert csa2.csa2_workspace_bytes(0, 10) == 0


def _fake_cache(csa2, **kw):
    c = csa2.csa2_cache(256 * 1000, 10, 256 * 2000, 4, 256 * 3000, 256 * 4000, 256 * 5000, 256 * 6000, 256 * 7000, 2)
    for k, v in kw.items():
        setattr(c, k, v)
    return c


def test_invalid_arguments_rejected_before_launch(csa2):
    L = csa2.lib
    P = C.c_void_p
    good = P(256 * 100)
    # null cache
    assert L.csa2_index(None, 0, good, good, good, good, good, good, 1 << 30, None) == 1
    # cache with a null field / zero batch
    for kw in ({"pool": None}, {"batch": 0}, {"n_pages": 0}, {"max_pages": 0}, {"pool": 256 * 1000 + 8}):
        c = _fake_cache(csa2, **kw)
        assert L.csa2_attend(C.byref(c), 64, good, good, 0.1, good, 0, 0, good, 1 << 30, None) == 1, kw
    c = _fake_cache(csa2)
    # bad mode, bad heads, missing pool in FULL mode, workspace too small
    assert L.csa2_index(C.byref(c), 7, good, good, good, good, good, good, 1 << 30, None) == 1
    assert L.csa2_attend(C.byref(c), 0, good, good, 0.1, good, 0, 0, good, 1 << 30, None) == 1
    assert L.csa2_attend(C.byref(c), 129, good, good, 0.1, good, 0, 0, good, 1 << 30, None) == 1
    assert L.csa2_index(C.byref(c), 1, good, good, None, None, good, good, 1 << 30, None) == 1
    assert L.csa2_index(C.byref(c), 0, good, good, None, None, good, good, 16, None) == 1
    assert L.csa2_attend(C.byref(c), 64, good, good, 0.1, good, 0, 0, good, 16, None) == 1
    # prefill: bad request, m, alignment, range, capacity
    assert L.csa2_prefill(C.byref(c), 5, 1, 0, 10, 10, good, good, good, None) == 1
    assert L.csa2_prefill(C.byref(c), 0, 3, 0, 10, 10, good, good, good, None) == 1
    assert L.csa2_prefill(C.byref(c), 0, 2, 1, 10, 20, good, good, good, None) == 1
    assert L.csa2_prefill(C.byref(c), 0, 1, 0, 10, 5, good, good, good, None) == 1
    assert L.csa2_prefill(C.byref(c), 0, 1, 0, 300, 300, good, good, good, None) == 1   # 4 pages = 256 entries
    assert L.csa2_attend(C.byref(c), 64, good, good, 0.1, good, 0, 6, good, 1 << 30, None) == 1   # unknown flag
    assert L.csa2_append(C.byref(c), None, good, good, good, None) == 1
    # top-k: k out of 1..2048, null pointers, empty batch, zero stride
    assert L.csa2_topk(good, 100, good, 4, 0, good, None) == 1
    assert L.csa2_topk(good, 100, good, 4, 2049, good, None) == 1
    assert L.csa2_topk(None, 100, good, 4, 512, good, None) == 1
    assert L.csa2_topk(good, 100, None, 4, 512, good, None) == 1
    assert L.csa2_topk(good, 100, good, 0, 512, good, None) == 1
    assert L.csa2_topk(good, 0, good, 4, 512, good, None) == 1
    assert L.csa2_get_device_error(None, None, None) == 1
    assert csa2.status_string(1) == "invalid argument"


def test_sharded_calls_reject_invalid_arguments_before_launch(csa2):
    L = csa2.lib
    P = C.c_void_p
    good = P(256 * 100)
    c = _fake_cache(csa2)
    lists = (C.c_void_p * 9)(*([256 * 200] * 9))
    lp = C.cast(lists, C.c_void_p)
    holes = (C.c_void_p * 2)(256 * 200, None)
    hp = C.cast(holes, C.c_void_p)
    # shard counts outside 1..8, a null list entry, null outputs
    for n in (0, 9):
        assert L.csa2_shard_pool(C.byref(c), good, n, lp, lp, good, good, None) == 1, n
        assert L.csa2_shard_topk(C.byref(c), good, n, lp, lp, good, None) == 1, n
        assert L.csa2_combine(n, lp, lp, 2, 64, good, 0, None) == 1, n
    assert L.csa2_shard_pool(C.byref(c), good, 2, hp, lp, good, good, None) == 1
    assert L.csa2_shard_topk(C.byref(c), good, 2, lp, hp, good, None) == 1
    assert L.csa2_shard_pool(C.byref(c), None, 2, lp, lp, good, good, None) == 1
    assert L.csa2_shard_topk(C.byref(c), good, 2, lp, lp, None, None) == 1
    assert L.csa2_shard_blocks(C.byref(c), good, good, good, good, good, good, 16, None) == 1   # workspace
    assert L.csa2_shard_blocks(C.byref(c), None, good, good, good, good, good, 1 << 30, None) == 1
    assert L.csa2_shard_rescore(C.byref(c), good, good, good, good, good, good, None, None) == 1
    assert L.csa2_shard_rescore(None, good, good, good, good, good, good, good, None) == 1
    # partial attention: heads, null lse, unknown flag
    assert L.csa2_attend_partial(C.byref(c), 0, good, good, 0.1, 1, good, good, 0, None) == 1
    assert L.csa2_attend_partial(C.byref(c), 64, good, good, 0.1, 1, good, None, 0, None) == 1
    assert L.csa2_attend_partial(C.byref(c), 64, good, good, 0.1, 1, good, good, 2, None) == 1
    # combine: batch, heads, misaligned part
    mis = (C.c_void_p * 2)(256 * 200, 256 * 200 + 4)
    assert L.csa2_combine(2, lp, lp, 0, 64, good, 0, None) == 1
    assert L.csa2_combine(2, lp, lp, 2, 129, good, 0, None) == 1
    assert L.csa2_combine(2, C.cast(mis, C.c_void_p), lp, 2, 64, good, 0, None) == 1


def test_selftest_wait_timeout_rejects_invalid_arguments(csa2):
    L = csa2.lib
    assert L.csa2_selftest_wait_timeout(None, 100, None) == 1
    assert L.csa2_selftest_wait_timeout(C.c_void_p(256 * 100), 0, None) == 1
    assert L.csa2_selftest_wait_timeout(C.c_void_p(256 * 100), (1 << 16) + 1, None) == 1
