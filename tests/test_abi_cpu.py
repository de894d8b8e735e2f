"""The C-ABI library loads on a machine without a GPU, exports every symbol that
include/fs_stream.h declares, and rejects bad arguments before touching CUDA."""
from __future__ import annotations

import ctypes
import os
import re

import pytest

from streaming_kv_cache_stream_b200 import abi

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "fs_stream.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fs_[a-z_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(abi.LIB_PATH):
        from streaming_kv_cache_stream_b200.build import build

        build()
    return abi.load()


def test_every_declared_symbol_is_exported_and_bound(lib):
    names = _declared()
    assert "fs_stream_create" in names and "fs_stream_attend" in names
    for n in names:
        assert hasattr(lib, n), f"{n} missing from the library"
        assert n in abi.SIGNATURES, f"{n} has no binding"
    assert set(abi.SIGNATURES) == set(names)


def test_status_codes_match_header():
    text = open(HEADER).read()
    for name in ("FS_OK", "FS_ERR_ARG", "FS_ERR_STATE", "FS_ERR_CUDA", "FS_ERR_DEVICE_TIMEOUT", "FS_ERR_OOM",
                 "FS_ERR_RANGE", "FS_STATE_EXPECT_PREFILL", "FS_STATE_PREFILLED", "FS_STATE_STREAMING",
                 "FS_MAX_VERIFY_TOKENS", "FS_MAX_TAIL_TOKENS"):
        m = re.search(rf"#define {name}\s+(-?\d+)", text)
        assert m and int(m.group(1)) == getattr(abi, name), name


@pytest.mark.parametrize("args", [
    (0, 4, 16, 8, 32, 8, 128),      # no views
    (4, 0, 16, 8, 32, 8, 128),      # no frames
    (4, 4, 0, 8, 32, 8, 128),       # empty frames
    (4, 4, 16, -1, 32, 8, 128),     # negative text
    (4, 4, 16, 8, 30, 8, 128),      # H not a multiple of Hkv
    (4, 4, 16, 8, 24, 8, 128),      # G = 3 does not divide 128
    (4, 4, 16, 8, 32, 8, 96),       # unsupported head dim
    (64, 64, 64, 0, 32, 8, 128),    # window longer than the kernel's key-tile table
])
def test_create_rejects_bad_shapes_without_cuda(lib, args):
    h = ctypes.c_void_p()
    rc = lib.fs_stream_create(ctypes.byref(h), *args, 10000.0)
    assert rc == abi.FS_ERR_ARG
    assert not h.value
    assert lib.fs_last_error()


def test_null_handle_calls_fail_cleanly(lib):
    assert lib.fs_stream_insert(None, None, None) == abi.FS_ERR_ARG
    assert lib.fs_stream_attend(None, None, None) == abi.FS_ERR_ARG
    assert lib.fs_stream_destroy(None) == abi.FS_OK
    assert lib.fs_stream_create(None, 1, 1, 1, 0, 1, 1, 64, 1.0) == abi.FS_ERR_ARG
    assert lib.fs_stream_attend_ext(None, None, None, None, 8, None) == abi.FS_ERR_ARG
    assert lib.fs_stream_append(None, None, None, 1) == abi.FS_ERR_ARG
    assert lib.fs_stream_insert_batch(None, 1, None, None) == abi.FS_ERR_ARG
    assert lib.fs_stream_insert_batch(None, 0, None, None) == abi.FS_ERR_ARG
    assert lib.fs_stream_insert_proj(None, None, None, 4096) == abi.FS_ERR_ARG
    assert lib.fs_frame_attend(None, None, None, None, 16, 16, 64, None) == abi.FS_ERR_ARG
    assert lib.fs_stream_attend_ext_static(None, None, None, None, 8, None) == abi.FS_ERR_ARG
    assert lib.fs_stream_step_host(None, None, None, None, None) == abi.FS_ERR_ARG
