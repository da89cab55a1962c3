"""The C ABI without a GPU: libkvq.so loads, exports every function that
include/kvq.h declares, and rejects bad arguments on the host before touching
the device."""
import ctypes
import os
import re

import pytest

import fp8_kv_paged_kvq_b200 as kvq
from fp8_kv_paged_kvq_b200 import build as kvq_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kvq.h")


@pytest.fixture(scope="module")
def lib():
    kvq_build.build()
    return kvq.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(kvq_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_path(lib):
    names = declared_functions()
    for must in ("kvq_append", "kvq_validate", "kvq_decode", "kvq_decode_bf16",
                 "kvq_decode_workspace_size", "kvq_status_string"):
        assert must in names


def test_every_declared_symbol_is_exported(lib):
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_status_strings(lib):
    for code, name in enumerate(["KVQ_OK", "KVQ_ERR_INVALID_ARG", "KVQ_ERR_UNSUPPORTED",
                                 "KVQ_ERR_WORKSPACE", "KVQ_ERR_CUDA"]):
        assert lib.kvq_status_string(code).decode() == name
    assert lib.kvq_status_string(99).decode() == "KVQ_ERR_UNKNOWN"


def test_host_checks_reject_bad_arguments_without_a_device(lib):
    E = kvq.KVQ_ERR_INVALID_ARG
    assert lib.kvq_append(None, None, None, None, 0, None, 0, None) == E
    assert lib.kvq_validate(None, 1, None, None, None, 16, -1, 1, None, None, None, None) == E
    assert lib.kvq_validate(None, 0, None, None, None, 16, 1, 1, None, None, None, None) == E
    assert lib.kvq_validate(None, 4, None, None, None, 16, 1, 1, None, None, None, None) == E
    assert lib.kvq_amax(None, 4, 1, 12, 0, None, None) == E           # D % 8 != 0, null out
    assert lib.kvq_scale_from_amax(None, None, -1, None) == E
    assert lib.kvq_e4m3_encode_bits(0, 16, None, None) == E
    assert lib.kvq_device_error(None) == E
    assert lib.kvq_decode_workspace_size(None, 1, 8, 0) == 0
    d = kvq.KvqCacheDesc(0, 1, 4, 16, 1, 100, 128, 16, 16, 16, 16, 16)   # Dk not a multiple of 16
    assert lib.kvq_decode(ctypes.byref(d), None, 8, None, 1, None, 1, None, ctypes.c_float(1.0),
                          None, None, None, 0, 0, None) == E
    d2 = kvq.KvqCacheDesc(0, 1, 4, 16, 1, 128, 128, 16, 16, 16, 16, 16)
    assert lib.kvq_decode(ctypes.byref(d2), None, 7, None, 1, None, 1, None, ctypes.c_float(1.0),
                          None, None, None, 0, 0, None) == E          # 7 query heads on 1 KV head? ok
    assert lib.kvq_decode_bf16(ctypes.byref(d2), None, 8, None, 1, None, 1, None,
                               ctypes.c_float(1.0), None, None, None, 0, 0, None) == E  # dtype mismatch
