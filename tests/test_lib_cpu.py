"""The C-ABI library without a GPU: it loads, exports every function that
include/st.h declares, and rejects bad arguments on the host before touching
CUDA."""
import ctypes
import os
import re

import pytest

import filtered_int8_ann_b200 as st
from filtered_int8_ann_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return st.lib()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "st.h")).read()
    return sorted(set(re.findall(r"^\s*(?:st_status|void|const char\*)\s+(st_\w+)\s*\(", text, re.M)))


def test_header_declares_the_binding_exports():
    assert declared_functions() == sorted(st.EXPORTS)


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for s in range(7):
        assert st.status_string(s)
    assert st.status_string(3) == "out of device memory"


def test_create_rejects_bad_arguments_on_host(lib):
    h = ctypes.c_void_p()
    P = ctypes.c_void_p
    fake = P(16)
    # null pointers
    assert lib.st_index_create(None, fake, fake, fake, 10, 64, 2, 2, None, ctypes.byref(h)) == st.ST_ERR_INVALID_ARG
    # n < 1, nlist < 1
    assert lib.st_index_create(fake, fake, fake, fake, 0, 64, 2, 2, None, ctypes.byref(h)) == st.ST_ERR_INVALID_ARG
    assert lib.st_index_create(fake, fake, fake, fake, 10, 64, 0, 2, None, ctypes.byref(h)) == st.ST_ERR_INVALID_ARG
    # unsupported d, signature width, n
    assert lib.st_index_create(fake, fake, fake, fake, 10, 40, 2, 2, None, ctypes.byref(h)) == st.ST_ERR_UNSUPPORTED
    assert lib.st_index_create(fake, fake, fake, fake, 10, 1024, 2, 2, None, ctypes.byref(h)) == st.ST_ERR_UNSUPPORTED
    assert lib.st_index_create(fake, fake, fake, fake, 10, 64, 2, 3, None, ctypes.byref(h)) == st.ST_ERR_UNSUPPORTED
    assert lib.st_index_create(fake, fake, fake, fake, 2**31, 64, 2, 2, None, ctypes.byref(h)) == st.ST_ERR_UNSUPPORTED
    assert h.value is None
    # null out
    assert lib.st_index_create(fake, fake, fake, fake, 10, 64, 2, 2, None, None) == st.ST_ERR_INVALID_ARG


def test_search_rejects_null_index(lib):
    fake = ctypes.c_void_p(16)
    assert lib.st_search(None, fake, fake, 1, 1, 1, fake, fake, None) == st.ST_ERR_INVALID_ARG
    assert lib.st_search_host(None, fake, fake, 1, 1, 1, fake, fake, None) == st.ST_ERR_INVALID_ARG
    assert lib.st_index_check(None, None) == st.ST_ERR_INVALID_ARG
    assert lib.st_probe_noalloc(None, fake, 1, 1, fake, None) == st.ST_ERR_INVALID_ARG
    assert lib.st_merge_topk(fake, fake, 0, 1, 1, fake, fake, None) == st.ST_ERR_INVALID_ARG
    assert lib.st_merge_topk(fake, fake, 1, 1, 0, fake, fake, None) == st.ST_ERR_INVALID_ARG
    assert lib.st_merge_topk(fake, fake, 2, 1, 8192, fake, fake, None) == st.ST_ERR_UNSUPPORTED
    assert lib.st_index_set_option(None, 1, 5) == st.ST_ERR_INVALID_ARG
    lib.st_index_destroy(None)  # NULL-safe


def test_freshness_and_host_calls_reject_null_index(lib):
    fake = ctypes.c_void_p(16)
    lists = (ctypes.c_int32 * 2)(0, 1)
    ids = (ctypes.c_int64 * 2)()
    L = lib  # argument types as the binding declares them
    assert L.st_index_insert(None, ctypes.cast(lists, ctypes.c_void_p), fake, fake, 2,
                             ctypes.cast(ids, ctypes.c_void_p), None) == st.ST_ERR_INVALID_ARG
    assert L.st_index_update(None, fake, fake, fake, 2, None) == st.ST_ERR_INVALID_ARG
    assert L.st_index_delete(None, fake, 2, None) == st.ST_ERR_INVALID_ARG
    assert L.st_search_host_async(None, fake, fake, 1, 1, 1, fake, fake, None) == st.ST_ERR_INVALID_ARG
    assert L.st_merge_topk_union(fake, fake, 0, 1, 1, fake, fake, None) == st.ST_ERR_INVALID_ARG
    assert L.st_merge_topk_union(fake, fake, 4, 1, 8192, fake, fake, None) == st.ST_ERR_UNSUPPORTED
