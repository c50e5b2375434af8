"""Host-side checks of the C ABI: the library loads, exports every symbol that
include/csa.h declares, and rejects bad arguments before any launch (no GPU needed)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "csa.h")


@pytest.fixture(scope="module")
def lib():
    from long_context_compressed_csa_b200 import build
    build.build()
    from long_context_compressed_csa_b200._binding import library
    return library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s+\*?([a-z_0-9]+)\s*\(",
                       text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_five_exports():
    names = declared_functions()
    for n in ("csa_compress", "hca_compress", "csa_indexer_topk", "csa_sparse_attn",
              "hca_dense_attn"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings_and_version(lib):
    from long_context_compressed_csa_b200 import csa_status_string, csa_version
    assert csa_status_string(0) == "CSA_OK"
    for code in range(-1, -8, -1):
        assert csa_status_string(code).startswith("CSA_ERR_")
    assert csa_status_string(-99) == "CSA_ERR_UNKNOWN"
    assert csa_version() >= 100


def test_workspace_sizes_are_host_arithmetic(lib):
    from long_context_compressed_csa_b200 import (csa_attn_workspace_size,
                                                  csa_indexer_topk_workspace_size)
    s1 = csa_indexer_topk_workspace_size(1, 1, 262144, 1024)
    assert s1 >= 262144 * (4 + 16)
    assert csa_indexer_topk_workspace_size(4, 1, 65536, 1024) > s1 / 2
    assert csa_indexer_topk_workspace_size(0, 1, 10, 1) == 0
    a = csa_attn_workspace_size(1, 1, 128, 512, 1024)
    assert a >= 128 * 512 * 4
    assert csa_attn_workspace_size(16, 1, 128, 512, 1024) >= a


def test_host_validation_rejects_bad_arguments_without_launching(lib):
    vp = ctypes.c_void_p
    fake = vp(0x10000)  # never dereferenced: every call below fails validation first
    # unknown dtype
    assert lib.csa_compress(fake, fake, fake, fake, 8, 64, 0, 8, None, None, fake, 64, 1, 8, 4,
                            0, 2, 7, None) == -3
    # m * entry_end > n
    assert lib.csa_compress(fake, fake, fake, fake, 8, 64, 0, 8, None, None, fake, 64, 1, 8, 4,
                            0, 3, 0, None) == -1
    # null stream pointer
    assert lib.csa_compress(None, fake, fake, fake, 8, 64, 0, 8, None, None, fake, 64, 1, 8, 4,
                            0, 2, 0, None) == -1
    # rows before tok0 requested
    assert lib.hca_compress(fake, fake, 8, 1024, 128, 256, None, fake, 16, 1, 8, 128, 0, 2, 0,
                            None) == -1
    # misaligned pointer (bf16 needs 2-byte alignment)
    odd = vp(0x10001)
    assert lib.hca_compress(odd, fake, 8, 1024, 0, 256, None, fake, 16, 1, 8, 128, 0, 2, 0,
                            None) == -2
    # indexer: k = 0, workspace too small, bad dtype
    assert lib.csa_indexer_topk(fake, fake, fake, fake, 1, 1, 100, 4, 8, 4, 0, fake, None,
                                fake, 1 << 30, 0, None) == -1
    assert lib.csa_indexer_topk(fake, fake, fake, fake, 1, 1, 100, 4, 8, 4, 5, fake, None,
                                fake, 16, 0, None) == -4
    assert lib.csa_indexer_topk(fake, fake, fake, fake, 1, 1, 100, 4, 8, 4, 5, fake, None,
                                fake, 1 << 30, 5, None) == -3
    # more queries than one grid row per query allows (B * nq > 65535)
    assert lib.csa_indexer_topk(fake, fake, fake, fake, 2, 40000, 100, 64, 128, 4, 5, fake, None,
                                fake, 1 << 62, 0, None) == -6
    assert lib.csa_indexer_topk_e4m3(fake, fake, fake, fake, fake, 2, 40000, 100, 64, 128, 4, 8, fake,
                                     None, fake, 1 << 62, None) == -6
    # the no-allocation variant: B * nq above the limit (checked before any size
    # arithmetic, which would overflow), and a problem larger than its fixed scratch
    assert lib.csa_indexer_topk_noalloc(fake, fake, fake, fake, 40000, 40000, 100, 64, 128, 4, 5, fake,
                                        None, 0, None) == -6
    assert lib.csa_indexer_topk_noalloc(fake, fake, fake, fake, 1, 1, 1 << 20, 64, 128, 4, 5, fake,
                                        None, 0, None) == -4
    assert lib.csa_indexer_topk_workspace_size(40000, 40000, 100, 5) == 0
    # attention: out_bf16 with fp32, c too wide, workspace too small
    assert lib.csa_sparse_attn(fake, fake, fake, 1, 1, 4, 64, 100, 8, 0.0, fake, None, fake,
                               1 << 30, 1, 1, None) == -3
    assert lib.csa_sparse_attn(fake, fake, fake, 1, 1, 4, 1024, 100, 8, 0.0, fake, None, fake,
                               1 << 30, 0, 0, None) == -6
    assert lib.hca_dense_attn(fake, fake, fake, 1, 1, 4, 64, 100, 128, 0.0, fake, None, fake,
                              8, 0, 0, None) == -4
    assert lib.hca_dense_attn(fake, fake, fake, 1, 1, 4, 64, 100, 0, 0.0, fake, None, fake,
                              1 << 30, 0, 0, None) == -1
    # sliding window: n_win < 1, ring smaller than the window, no window buffer, misaligned t
    assert lib.csa_sparse_attn_window(fake, fake, fake, fake, fake, 1, 1, 4, 64, 100, 8, 0, 16, 0.0,
                                      fake, None, fake, 1 << 30, 0, 0, None) == -1
    assert lib.csa_sparse_attn_window(fake, fake, fake, fake, fake, 1, 1, 4, 64, 100, 8, 32, 16, 0.0,
                                      fake, None, fake, 1 << 30, 0, 0, None) == -1
    assert lib.hca_dense_attn_window(fake, fake, fake, None, 1, 1, 4, 64, 100, 128, 8, 16, 0.0,
                                     fake, None, fake, 1 << 30, 0, 0, None) == -1
    assert lib.hca_dense_attn_window(fake, fake, vp(0x10004), fake, 1, 1, 4, 64, 100, 128, 8, 16, 0.0,
                                     fake, None, fake, 1 << 30, 0, 0, None) == -2
    # E4M3: cols not a multiple of 4, bad dtype; indexer with an unsupported cI
    assert lib.csa_quantize_e4m3(fake, 10, 6, 6, fake, fake, 0, None) == -1
    assert lib.csa_quantize_e4m3(fake, 10, 8, 8, fake, fake, 9, None) == -3
    assert lib.csa_indexer_topk_e4m3(fake, fake, fake, fake, fake, 1, 1, 100, 64, 64, 4, 8, fake, None,
                                     fake, 1 << 30, None) == -6
    # E2M1: cols not a multiple of 8, bad dtype; indexer with an unsupported cI, codes not
    # 32-byte aligned, more queries than grid rows
    assert lib.csa_quantize_e2m1(fake, 10, 12, 12, fake, fake, 0, None) == -1
    assert lib.csa_quantize_e2m1(fake, 10, 16, 16, fake, fake, 9, None) == -3
    assert lib.csa_indexer_topk_e2m1(fake, fake, fake, fake, fake, 1, 1, 100, 64, 64, 4, 8, fake, None,
                                     fake, 1 << 30, None) == -6
    assert lib.csa_indexer_topk_e2m1(fake, fake, vp(0x10010), fake, fake, 1, 1, 100, 64, 128, 4, 8, fake, None,
                                     fake, 1 << 30, None) == -2
    assert lib.csa_indexer_topk_e2m1(fake, fake, fake, fake, fake, 2, 40000, 100, 64, 128, 4, 8, fake,
                                     None, fake, 1 << 62, None) == -6
    # fused projection + HCA compression: m' other than 128, d not a multiple of 64,
    # no workspace, a workspace too small
    assert lib.hca_project_compress(fake, 64, 64 * 256, 0, 256, fake, fake, 64, None, fake, 1024, 1, 128, 64,
                                    0, 4, fake, 256, None) == -6
    assert lib.hca_project_compress(fake, 96, 96 * 256, 0, 256, fake, fake, 96, None, fake, 1024, 1, 128, 128,
                                    0, 2, fake, 256, None) == -6
    assert lib.hca_project_compress(fake, 64, 64 * 256, 0, 256, fake, fake, 64, None, fake, 1024, 1, 128, 128,
                                    0, 2, None, 256, None) == -1
    assert lib.hca_project_compress(fake, 64, 64 * 256, 0, 256, fake, fake, 64, None, fake, 1024, 1, 128, 128,
                                    0, 2, fake, 16, None) == -4
    # fused CSA projections + compression: m other than 4, tok0 after the first row read
    assert lib.csa_project_compress(fake, 64, 64 * 256, 0, 256, fake, fake, fake, fake, 64, None, None, fake,
                                    1024, 1, 128, 8, 0, 4, fake, 256, None) == -6
    assert lib.csa_project_compress(fake, 64, 64 * 256, 16, 256, fake, fake, fake, fake, 64, None, None, fake,
                                    1024, 1, 128, 4, 2, 8, fake, 256, None) == -1
    # empty problems succeed without touching memory
    assert lib.csa_compress(fake, fake, fake, fake, 8, 64, 0, 8, None, None, fake, 64, 0, 8, 4,
                            0, 2, 0, None) == 0
    assert lib.csa_compress(fake, fake, fake, fake, 8, 64, 0, 8, None, None, fake, 64, 1, 8, 4,
                            1, 1, 0, None) == 0


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    import long_context_compressed_csa_b200._binding as b
    monkeypatch.setattr(b, "_lib", None)
    monkeypatch.setattr(b, "library_path", str(tmp_path / "missing.so"))
    with pytest.raises(ImportError):
        b.library()
