"""The C ABI library builds for sm_100a, loads, and exports every entry point that
include/dsa.h declares; host-side validation answers without a GPU."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "dsa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(dsa_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    import sparse_attention_tcgen05_b200 as dsa
    return dsa.load()


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert "dsa_indexer" in names and "dsa_sparse_mla_fwd" in names
    for n in names:
        assert hasattr(lib, n), n
    import sparse_attention_tcgen05_b200 as dsa
    assert sorted(dsa.EXPORTED) == names


def test_status_strings_and_version(lib):
    import sparse_attention_tcgen05_b200 as dsa
    assert dsa.dsa_status_str(0) == "DSA_OK"
    assert dsa.dsa_status_str(5) == "DSA_ERR_TIMEOUT"
    assert dsa.dsa_version() >= 100


def test_host_validation_rejects_without_touching_a_device(lib):
    P = ctypes.c_void_p
    fake = P(0x10000)  # never dereferenced: validation fails first
    assert lib.dsa_indexer(None, fake, fake, fake, 1, 1, 8, 64, 128, None, 0, None) == 1
    assert lib.dsa_indexer(fake, fake, fake, fake, 1, 9, 8, 64, 128, None, 0, None) == 1
    assert lib.dsa_topk(fake, fake, 1, 1, 8, 0, None, 0, None) == 1
    assert lib.dsa_sparse_mla_fwd(fake, fake, fake, 1, 1, 8, 128, 576, 512, 16, float("nan"), fake,
                                  None, None, None, 0, None) == 1
    assert lib.dsa_sparse_mla_fwd(fake, fake, fake, 1, 1, 8, 128, 576, 512, 16, -1.0, fake,
                                  None, None, None, 0, None) == 1
    assert lib.dsa_indexer_kl(fake, fake, None, 1, 1, 8, 4, fake, None, None, 0, None) == 1
    assert lib.dsa_indexer_kl_noalloc(fake, fake, fake, 1, 4, 2, 4, fake, None, None) == 1
    # a misaligned per-row output or workspace is refused before any launch
    odd = P(0x10004)
    assert lib.dsa_indexer_kl(fake, fake, fake, 1, 4, 8, 4, fake, odd, None, 0, None) == 1
    assert lib.dsa_indexer_kl(fake, fake, fake, 1, 4, 8, 4, fake, None, odd, 64, None) == 1
    assert lib.dsa_indexer_kl_noalloc(fake, fake, fake, 1, 4, 8, 4, fake, odd, None) == 1



def test_host_validation_of_the_variant_entry_points(lib):
    # bad arguments and unsupported shapes of the dense, backward, paged, HISA and masked-MHA calls
    # answer before any device work (1 = DSA_ERR_INVALID_ARG, 2 = DSA_ERR_UNSUPPORTED)
    P = ctypes.c_void_p
    fake, odd = P(0x10000), P(0x10004)
    nan = float("nan")
    # dense warm-up: null output, Lq > Lk, non-finite scale, more than 128 heads
    assert lib.dsa_dense_mla_fwd(fake, fake, 1, 8, 8, 128, 576, 512, 0.1, None, None, None, None, 0, None) == 1
    assert lib.dsa_dense_mla_fwd(fake, fake, 1, 9, 8, 128, 576, 512, 0.1, fake, None, None, None, 0, None) == 1
    assert lib.dsa_dense_mla_fwd(fake, fake, 1, 8, 8, 128, 576, 512, nan, fake, None, None, None, 0, None) == 1
    assert lib.dsa_dense_mla_fwd(fake, fake, 1, 8, 8, 129, 576, 512, 0.1, fake, None, None, None, 0, None) == 2
    # dense KL: no per-row output and no workspace; misaligned per-row output
    assert lib.dsa_indexer_kl_dense(fake, fake, 1, 8, 8, fake, None, None, 0, None) == 1
    assert lib.dsa_indexer_kl_dense(fake, fake, 1, 8, 8, fake, odd, None, 0, None) == 1
    # backward: a dense call (idx = NULL) must take every position; other head shapes
    assert lib.dsa_indexer_bwd(fake, fake, fake, fake, None, fake, 1, 4, 8, 64, 128, 4, fake, fake, fake, None) == 1
    assert lib.dsa_indexer_bwd(fake, fake, fake, fake, fake, fake, 1, 4, 8, 32, 128, 4, fake, fake, fake, None) == 2
    # paged decode: pages must hold a multiple of 64 entries; the table must be given
    assert lib.dsa_indexer_topk_paged(fake, fake, fake, fake, fake, fake, fake, 2, 4096, 100, 48, 64, 128, 256,
                                      fake, 1 << 20, None) == 2
    assert lib.dsa_indexer_topk_paged(fake, fake, fake, None, fake, fake, fake, 2, 4096, 100, 64, 64, 128, 256,
                                      fake, 1 << 20, None) == 1
    assert lib.dsa_sparse_mla_fwd_paged(fake, fake, fake, fake, fake, 2, 4096, 100, 64, 128, 576, 256, 256, 0.1,
                                        fake, None, fake, 1 << 20, None) == 2
    # HISA: whole blocks of a multiple of 64 keys; d_I = 128 for the block sums
    assert lib.dsa_hisa_block_sums(fake, 2, 4096, 64, 64, fake, None) == 2
    assert lib.dsa_hisa_topk(fake, fake, fake, fake, 2, 4096, 64, 128, 96, 8, 256, fake, None, fake, 1 << 20,
                             None) == 2
    assert lib.dsa_hisa_topk(fake, fake, fake, fake, 2, 4096, 64, 128, 64, 8, 256, fake, None, None, 0,
                             None) == 1
    # masked MHA: 192/128-dim heads only; the workspace is required
    assert lib.dsa_masked_mha_fwd(fake, fake, fake, fake, 1, 256, 8, 128, 128, 32, 0.1, fake, None, fake,
                                  1 << 20, None) == 2
    assert lib.dsa_masked_mha_fwd(fake, fake, fake, fake, 1, 256, 8, 192, 128, 32, 0.1, fake, None, None, 0,
                                  None) == 1


def test_workspace_sizes(lib):
    import sparse_attention_tcgen05_b200 as dsa
    assert dsa.dsa_workspace_bytes(dsa.DSA_OP_INDEXER, 1, 1, 8, 4, 8) == 0
    assert dsa.dsa_workspace_bytes(dsa.DSA_OP_INDEXER_KL, 2, 100, 100, 8, 0) == 800
    # decode: few rows -> split-KV partials need scratch; prefill: none
    assert dsa.dsa_workspace_bytes(dsa.DSA_OP_SPARSE_MLA_FWD, 32, 1, 32768, 2048, 128) > 0
    assert dsa.dsa_workspace_bytes(dsa.DSA_OP_SPARSE_MLA_FWD, 1, 16384, 16384, 2048, 128) == 0


def test_traffic_hash_ignores_comments_but_not_code():
    import importlib.util
    import os

    spec = importlib.util.spec_from_file_location(
        "bench", os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    import sys
    bench = sys.modules.setdefault("bench", bench)  # dataclasses look their module up by name
    spec.loader.exec_module(bench)
    src = "int a = 1; // one\n/* block\n comment */ int b = a + 2;\n"
    same = "int a = 1;\n\n   int b = a + 2; // other words\n"
    changed = "int a = 1; int b = a + 3;\n"
    assert bench._code_only(src) == bench._code_only(same)
    assert bench._code_only(src) != bench._code_only(changed)
