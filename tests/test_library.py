"""CPU-side checks of the C-ABI library: it builds, loads without a GPU, and
exports every function include/attn.h declares; host-side validation."""

import ctypes
import os
import re
import subprocess

import pytest

from online_softmax_attention_flash_b200 import binding as B
from online_softmax_attention_flash_b200 import build as build_mod

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "attn.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(attn_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return B.load_library()


def test_header_declares_the_three_entry_points():
    names = _declared_functions()
    for n in ("attn_encoder_fwd", "attn_gqa_decode", "attn_paged_history", "attn_check",
              "attn_gqa_decode_workspace_size"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", B.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for n in _declared_functions():
        assert n in exported, n
        assert hasattr(lib, n)


def test_binding_signatures_cover_the_header():
    assert sorted(n for n, _, _ in B.SIGNATURES) == _declared_functions()


def test_nothing_else_is_exported(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", B.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    ours = {line.split()[-1] for line in out.splitlines() if " T " in line}
    assert ours == set(_declared_functions())


def test_version_and_status_strings(lib):
    assert lib.attn_version() == 10000
    assert lib.attn_status_string(-8) == b"ATTN_ERR_BLOCK_TABLE"
    assert lib.attn_status_string(0) == b"ATTN_OK"


def test_host_validation_rejects_before_any_launch(lib):
    P = ctypes.c_void_p
    fake = P(4096)   # never dereferenced: validation fails first
    # null pointers
    assert lib.attn_encoder_fwd(None, fake, fake, fake, 1, 1, 128, 64, 0.125, None, None) == -1
    # bad head_dim / shape / scale / alignment
    assert lib.attn_encoder_fwd(fake, fake, fake, fake, 1, 1, 128, 96, 0.125, None, None) == -3
    assert lib.attn_encoder_fwd(fake, fake, fake, fake, 0, 1, 128, 64, 0.125, None, None) == -2
    assert lib.attn_encoder_fwd(fake, fake, fake, fake, 1, 1, 128, 64, -1.0, None, None) == -2
    assert lib.attn_encoder_fwd(fake, fake, fake, P(4098), 1, 1, 128, 64, 0.1, None, None) == -4
    # decode: group mismatch, head_dim, workspace
    assert lib.attn_gqa_decode(fake, fake, fake, None, fake, 2, 16, 8, 3, 64, 256, 1.0, fake,
                               1 << 20, None) == -2
    assert lib.attn_gqa_decode(fake, fake, fake, None, fake, 2, 16, 8, 2, 64, 96, 1.0, fake,
                               1 << 20, None) == -3
    assert lib.attn_gqa_decode(fake, fake, fake, None, fake, 2, 16, 8, 2, 64, 256, 1.0, fake,
                               16, None) == -5
    # paged: block size, history length beyond the table, head_dim
    args = dict(n_table=4, nb=4, bs=512, L=100, D=256)
    def paged(bs=512, L=100, D=256, n_table=4):
        return lib.attn_paged_history(fake, fake, fake, fake, n_table, 4, bs, L, 1.0, 1.0, 0.0625,
                                      32, 2, 16, 64, D, fake, None)
    assert paged(bs=500) == -2
    assert paged(bs=640) == -2
    assert paged(L=4 * 512 + 1) == -2
    assert paged(D=192) == -3


def test_workspace_size_query(lib):
    n = lib.attn_gqa_decode_workspace_size(8, 16, 8, 4096, 256)
    # at least one fp32 partial row [D] plus (m, l) per (batch, query head), growing with S_ctx
    assert n >= 8 * 16 * (256 + 2) * 4
    assert lib.attn_gqa_decode_workspace_size(8, 16, 8, 65536, 256) > n
    assert lib.attn_gqa_decode_workspace_size(8, 15, 8, 4096, 256) == 0


def test_noalloc_size_limit_is_checked_on_the_host(lib):
    fake = ctypes.c_void_p(4096)
    assert lib.attn_gqa_decode_noalloc(fake, fake, fake, None, fake, 64, 64, 8, 8, 65536, 512,
                                       1.0, None) == -5
    assert lib.attn_gqa_decode_noalloc(fake, fake, fake, None, fake, 0, 16, 8, 2, 64, 256,
                                       1.0, None) == -2


def test_rope_validation_rejects_before_any_launch(lib):
    fake = [ctypes.c_void_p(4096 * (i + 1) * 1024 * 1024) for i in range(6)]   # never dereferenced
    q, k, qo, ko, c, s = fake
    f = lib.attn_rope_qk
    assert f(None, k, qo, ko, c, s, 1, 1, 8, 64, 0, None) == -1                 # NULL
    assert f(q, k, qo, ko, c, s, 0, 1, 8, 64, 0, None) == -2                    # B < 1
    assert f(q, k, qo, ko, c, s, 1, 1, 8, 64, 2, None) == -2                    # pairing flag
    assert f(q, k, qo, ko, c, s, 1, 1, 8, 72, 0, None) == -3                    # D % 16
    assert f(q, k, qo, ko, c, s, 1, 1, 8, 1024, 0, None) == -3                  # D > 512
    assert f(ctypes.c_void_p(4096 + 8), k, qo, ko, c, s, 1, 1, 8, 64, 0, None) == -4
    assert f(q, k, ctypes.c_void_p(q.value + 256), ko, c, s, 1, 1, 8, 64, 0, None) == -2  # overlap
    assert f(q, k, ko, ko, c, s, 1, 1, 8, 64, 0, None) == -2                    # q_out == k_out


def test_source_digest_ignores_comments_and_covers_every_benched_kernel():
    import bench
    src = 'int a; // note\n/* block\n comment */ const char* s = "x // y /* z */";\n\n'
    assert build_mod._strip_comments(src) == 'int a;\n const char* s = "x // y /* z */";'
    assert build_mod._strip_comments(src) == build_mod._strip_comments(src.replace("note", "other"))
    benched = set(re.findall(r'self\.kernel_regex = "(\w+)"', open(bench.__file__).read()))
    assert benched and benched <= set(build_mod.KERNEL_SOURCES)   # each has its own digest
    for name in benched:
        assert len(build_mod.source_digest(name)) == 16
