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


def test_decode_args_layout_matches_the_header(tmp_path):
    # the ctypes mirror of adamas_decode_args must agree with the C compiler's layout
    fields = [f for f, _ in adamas.DecodeArgs._fields_]
    prog = tmp_path / "layout.c"
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "adamas.h"', 'int main(void) {',
             '  printf("%zu\\n", sizeof(adamas_decode_args));']
    lines += [f'  printf("%zu\\n", offsetof(adamas_decode_args, {f}));' for f in fields]
    lines += ['  return 0;', '}']
    prog.write_text("\n".join(lines))
    exe = tmp_path / "layout"
    import subprocess
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), "-o", str(exe), str(prog)], check=True)
    got = [int(x) for x in subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()]
    assert got[0] == ctypes.sizeof(adamas.DecodeArgs)
    assert got[1:] == [getattr(adamas.DecodeArgs, f).offset for f in fields]


def test_decode_ex_rejects_bad_options_before_any_launch(lib):
    fake = 1 << 20                                   # never dereferenced: the checks come first
    base = dict(q=fake, codes=fake, K=fake, V=fake, seq_lens=fake, B=1, Hq=4, Hkv=1, Nmax=4096, d=128, budget=64,
                out=fake, idx=fake, workspace=fake, workspace_bytes=1 << 20, policy=0)
    def call(**kw):
        a = adamas.DecodeArgs(**dict(base, **kw))
        return lib.adamas_decode_step_ex(ctypes.byref(a), None)
    assert call(policy=7) == -1                      # unknown policy
    assert call(policy=1, budget=5000) == -2         # group-shared budget above 4096
    assert call(n_sink=-1) == -1
    assert call(k_new=fake) == -1                    # k_new without v_new
    assert call(k_new=fake, v_new=fake) == -1        # rows without append positions
    assert call(block_table=fake, page_size=0, max_pages=4, n_pages=8) == -1
    assert call(block_table=fake + 2, page_size=16, max_pages=4, n_pages=8) == -1   # misaligned table
    assert lib.adamas_decode_step_ex(None, None) == -1


def test_sharded_and_static_calls_reject_bad_arguments_before_any_launch(lib):
    fake = ctypes.c_void_p(1 << 20)                  # never dereferenced: the checks come first
    # adamas_shard_score: a null histogram buffer, a misaligned q
    assert lib.adamas_shard_score(fake, fake, fake, 1, 4, 1, 4096, 128, 64, None, fake, 1 << 20, None) == -1
    assert lib.adamas_shard_score(ctypes.c_void_p((1 << 20) + 2), fake, fake, 1, 4, 1, 4096, 128, 64, fake, fake,
                                  1 << 20, None) == -1
    assert lib.adamas_shard_score(fake, fake, fake, 1, 4, 1, 4096, 64, 64, fake, fake, 1 << 20, None) == -2  # d != 128
    # adamas_shard_attend: world < 1, rank outside [0, world), a null state buffer
    def attend(world, rank, partial=fake):
        return lib.adamas_shard_attend(fake, fake, fake, fake, 1, 4, 1, 4096, 128, 64, fake, world, rank, partial,
                                       fake, fake, 1 << 20, None)
    assert attend(0, 0) == -1
    assert attend(2, 2) == -1
    assert attend(2, -1) == -1
    assert attend(2, 1, partial=None) == -1
    # adamas_merge_partials: no state, a null output, nothing to merge
    assert lib.adamas_merge_partials(fake, 0, 1, 4, fake, None) == -1
    assert lib.adamas_merge_partials(fake, 2, 1, 4, None, None) == -1
    assert lib.adamas_merge_partials(fake, 2, 0, 4, fake, None) == 0
    # adamas_static_device_error: a null word pointer
    assert lib.adamas_static_device_error(None, None) == -1
