"""The C-ABI library loads and exports every symbol include/pa.h declares;
host-side validation answers without touching a GPU."""
import ctypes
import glob
import os
import re

import pytest

from paged_kv_cache_481_b200 import binding, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pa.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return binding.load()


def _declared_functions():
    names = set()
    for path in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = re.sub(r"/\*.*?\*/", "", open(path).read(), flags=re.S)
        names |= set(re.findall(r"\b(pa_[a-z0-9_]+)\s*\(", text))
    return sorted(names)


def test_header_declares_the_binding_names():
    assert _declared_functions() == sorted(binding.EXPORTED)


def test_every_declared_symbol_is_exported(lib):
    for name in _declared_functions():
        assert hasattr(lib, name), name


def test_only_declared_symbols_are_exported():
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", binding.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    pa_syms = sorted({line.split()[-1] for line in out.splitlines()
                      if line.split()[-1].startswith("pa_")})
    assert pa_syms == sorted(binding.EXPORTED)


def test_status_strings(lib):
    assert binding.status_string(0) == "ok"
    assert "workspace" in binding.status_string(4)
    assert binding.status_string(99) == "unknown status"
    assert "free blocks" in binding.status_string(binding.PA_ERR_OUT_OF_BLOCKS)


def test_workspace_size_covers_partials_and_tickets(lib):
    small = binding.pa_decode_workspace_size(1, 1, 128, 512)
    big = binding.pa_decode_workspace_size(256, 40, 128, 4096)
    assert small > 0 and big > small
    # two partial slots of (D + 2) floats per worker, one ticket per (seq, head)
    assert small >= 2 * 4096 * (128 + 2) * 4
    assert big - small >= (256 * 40 - 1) * 4 - 256
    assert binding.pa_decode_workspace_size(256, 40, 128, 4096) == \
        binding.pa_decode_workspace_size(256, 40, 128, 16)


NULL = ctypes.c_void_p(None)


def test_decode_rejects_unsupported_shapes_before_any_launch(lib):
    args = lambda d, bs, mctx=16, mb=1: (NULL, NULL, NULL, NULL, NULL, mb, NULL, mctx, 1, 1, d, bs,
                                         1, ctypes.c_float(1.0), NULL, 0, NULL)
    assert lib.pa_decode(*args(96, 16)) == binding.PA_ERR_UNSUPPORTED
    assert lib.pa_decode(*args(128, 24)) == binding.PA_ERR_UNSUPPORTED
    # context longer than the table can address
    assert lib.pa_decode(*args(128, 16, 17, 1)) == binding.PA_ERR_INVALID_ARG
    # null pointers
    assert lib.pa_decode(*args(128, 16)) == binding.PA_ERR_INVALID_ARG
    # nothing to do
    z = list(args(128, 16))
    z[8] = 0
    assert lib.pa_decode(*z) == binding.PA_OK


def test_cache_ops_reject_bad_arguments_before_any_launch(lib):
    assert lib.pa_reshape_and_cache(NULL, NULL, NULL, NULL, NULL, 0, 4, 64, 16, 8,
                                    NULL) == binding.PA_OK
    assert lib.pa_reshape_and_cache(NULL, NULL, NULL, NULL, NULL, 3, 4, 64, 16, 8,
                                    NULL) == binding.PA_ERR_INVALID_ARG
    assert lib.pa_reshape_and_cache(NULL, NULL, NULL, NULL, NULL, 3, 4, 80, 16, 8,
                                    NULL) == binding.PA_ERR_UNSUPPORTED
    assert lib.pa_copy_blocks(NULL, NULL, NULL, 0, 4, 64, 16, 8, NULL) == binding.PA_OK
    assert lib.pa_copy_blocks(NULL, NULL, NULL, 2, 4, 64, 16, 8, NULL) == binding.PA_ERR_INVALID_ARG
    assert lib.pa_copy_blocks(NULL, NULL, NULL, 2, 4, 64, 12, 8, NULL) == binding.PA_ERR_UNSUPPORTED
    misaligned = ctypes.c_void_p(0x1008)
    assert lib.pa_copy_blocks(misaligned, misaligned, misaligned, 1, 4, 64, 16, 8,
                              NULL) == binding.PA_ERR_INVALID_ARG


def test_device_error_read_rejects_null(lib):
    assert lib.pa_get_last_device_error(None) == binding.PA_ERR_INVALID_ARG
