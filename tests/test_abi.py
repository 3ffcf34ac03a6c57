"""The C-ABI library loads on a machine without a GPU, exports every symbol that
include/adamas.h declares, and rejects bad arguments on the host before any CUDA
call is made."""
import ctypes
import os
import re

import pytest

from compressed_sparse_kv_fp32_b200 import adamas, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    text = open(os.path.join(ROOT, "include", "adamas.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(adamas_[a-z_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return adamas.load()


def test_every_declared_symbol_is_exported(lib):
    names = header_functions()
    assert len(names) >= 8
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(adamas.SYMBOLS)


def test_status_strings(lib):
    for rc, text in [(0, "ok"), (-1, "invalid argument"), (-3, "workspace missing or too small")]:
        assert adamas.status_string(rc) == text
    assert adamas.status_string(12345) == "unknown status"
    assert lib.adamas_version() >= 100


def test_host_side_argument_errors(lib):
    P = ctypes.c_void_p
    fake = P(4096)          # never dereferenced: every call below fails its checks first
    # unsupported head dimension
    assert lib.adamas_decode_step(fake, fake, fake, fake, fake, 1, 4, 4, 64, 64, 8, fake, fake,
                                  fake, 1 << 20, None) == -2
    # Hq not a multiple of Hkv
    assert lib.adamas_decode_step(fake, fake, fake, fake, fake, 1, 6, 4, 64, 128, 8, fake, fake,
                                  fake, 1 << 20, None) == -1
    # negative budget, group too large, batch too large
    assert lib.adamas_workspace_bytes(1, 4, 4, 64, 128, -1) == 0
    assert lib.adamas_workspace_bytes(1, 32, 2, 64, 128, 8) == 0
    assert lib.adamas_workspace_bytes(2000, 4, 4, 64, 128, 8) == 0
    # null pointers and misalignment
    assert lib.adamas_decode_step(None, fake, fake, fake, fake, 1, 4, 4, 64, 128, 8, fake, fake,
                                  fake, 1 << 20, None) == -1
    assert lib.adamas_decode_step(P(4098), fake, fake, fake, fake, 1, 4, 4, 64, 128, 8, fake, fake,
                                  fake, 1 << 20, None) == -1
    assert lib.adamas_encode_keys(fake, None, None, 4, 1, 4, 64, 128, None) == -1
    assert lib.adamas_encode_keys(fake, fake, None, -1, 1, 4, 64, 128, None) == -1
    assert lib.adamas_score(fake, fake, fake, 1, 4, 4, 64, 96, fake, None) == -2
    assert lib.adamas_workspace_init(None, 16, None) == -1
    # fused append step: missing or misaligned positions, and the decode step's own checks
    assert lib.adamas_decode_step_append(fake, fake, fake, fake, fake, None, 1, 4, 4, 64, 128, 8, fake, fake,
                                         fake, 1 << 20, None) == -1
    assert lib.adamas_decode_step_append(fake, fake, fake, fake, fake, P(4098), 1, 4, 4, 64, 128, 8, fake,
                                         fake, fake, 1 << 20, None) == -1
    assert lib.adamas_decode_step_append(fake, fake, fake, fake, fake, fake, 1, 4, 4, 64, 64, 8, fake, fake,
                                         fake, 1 << 20, None) == -2
    # empty batch: nothing to do, nothing touched, no CUDA call
    assert lib.adamas_decode_step(None, None, None, None, None, 0, 4, 4, 64, 128, 8, None, None,
                                  None, 0, None) == 0
    assert lib.adamas_encode_keys(None, None, None, 0, 1, 4, 64, 128, None) == 0
