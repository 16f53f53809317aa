"""The C-ABI library builds, loads without a GPU and exports every entry point
that include/msa.h declares; the binding's struct matches the header's layout."""
import ctypes
import os
import re

import block_sparse_gqa_mean_b200 as msa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "msa.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(msa_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_four_operations():
    names = declared_functions()
    for op in ("msa_build_block_cache", "msa_select_topk", "msa_sparse_attn_prefill",
               "msa_sparse_attn_decode"):
        assert op in names


def test_library_exports_every_declared_symbol():
    lib = msa.load_library()
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(declared_functions()) <= set(msa.EXPORTS) | {"msa_status_string", "msa_version"}


def test_status_strings_and_version():
    assert msa.status_string(msa.MSA_OK) == "ok"
    assert "workspace" in msa.status_string(msa.MSA_ERR_WORKSPACE)
    assert msa.load_library().msa_version() == 1000


def test_struct_layout_matches_header():
    # 8 int32 fields, then 6 pointers
    assert ctypes.sizeof(msa._PagedKV) == 8 * 4 + 6 * 8
    assert msa._PagedKV.k_pages.offset == 32
    assert msa._PagedKV.status_word.offset == 32 + 5 * 8


def test_null_cache_is_rejected_without_a_gpu():
    lib = msa.load_library()
    assert lib.msa_select_topk(None, None, None, 1, 1, 4, None, None, None, 0, None) == \
        msa.MSA_ERR_INVALID_ARG
    assert lib.msa_workspace_size(msa.MSA_OP_DECODE, None, 1, 1, 4) == 0
