"""The C ABI library on the CPU: it loads, exports every symbol include/clha.h declares, and its pure
host functions behave (no compute call needs a GPU here)."""
import ctypes as C
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "clha.h")).read()
    return sorted(set(re.findall(r"^CLHA_API\s+[\w\s\*]+?\b(clha_\w+)\(", src, flags=re.M)))


@pytest.fixture(scope="module")
def lib():
    from post_quantization_expert_b200 import build, clha
    build.build()
    return clha.load()


def test_every_declared_symbol_is_exported(lib):
    from post_quantization_expert_b200 import clha
    names = _declared()
    assert len(names) >= 20
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(clha.SYMBOLS) == names


def test_host_only_calls(lib):
    assert lib.clha_version() == 100
    assert lib.clha_packed_rows(8192, 2, 16) == 8192 * 2 + 128 * 16
    assert lib.clha_packed_rows(0, 1, 1) == 128
    assert lib.clha_packed_rows(-1, 1, 1) == 0
    assert lib.clha_last_error(None) == b"null context"


def test_null_context_is_rejected(lib):
    from post_quantization_expert_b200 import clha
    assert lib.clha_route_topk(None, None, 0, 4, 2, None, None) == clha.ERR_INVALID_ARG
    assert lib.clha_factor(None, None, 1, 128, None) == clha.ERR_INVALID_ARG
    assert lib.clha_check(None) == clha.ERR_INVALID_ARG
    lib.clha_destroy(None)


def test_create_without_a_gpu_fails_cleanly(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    h = C.c_void_p()
    assert lib.clha_create(0, None, C.byref(h)) != 0
    assert not h.value
