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


def test_selftest_rejects_bad_arguments_without_a_gpu():
    lib = msa.load_library()
    assert lib.msa_selftest_bounded_wait(0, None, None) == msa.MSA_ERR_INVALID_ARG
    assert lib.msa_selftest_bounded_wait(2, 4096, None) == msa.MSA_ERR_INVALID_ARG
    assert lib.msa_selftest_bounded_wait(1, 4098, None) == msa.MSA_ERR_INVALID_ARG  # misaligned


def test_null_cache_is_rejected_without_a_gpu():
    lib = msa.load_library()
    assert lib.msa_select_topk(None, None, None, 1, 1, 4, None, None, None, 0, None) == \
        msa.MSA_ERR_INVALID_ARG
    assert lib.msa_workspace_size(msa.MSA_OP_DECODE, None, 1, 1, 4) == 0


def _fake_kv(batch=2, num_pages=64, max_blocks=16, hq=32, hkv=8, d=128, B=64):
    """A cache descriptor with aligned placeholder pointers: host-side checks
    only (nothing here reaches a kernel)."""
    kv = msa._PagedKV()
    kv.batch, kv.num_pages, kv.max_blocks_per_seq = batch, num_pages, max_blocks
    kv.num_q_heads, kv.num_kv_heads, kv.head_dim, kv.block_size = hq, hkv, d, B
    kv.dtype = 0  # bf16
    for name in ("k_pages", "v_pages", "centroids", "page_table", "seq_lens", "status_word"):
        setattr(kv, name, 0x10000)
    return kv


def test_token_workspace_and_argument_checks_without_a_gpu():
    """The token selection's scratch is one fp32 score per cache position of
    every sequence, whatever top_k (top-K 2048 and beyond is the point of the
    token variant); bad arguments are refused before any launch."""
    lib = msa.load_library()
    kv = _fake_kv()
    for top_k in (1, 256, 2048, 6000):
        assert lib.msa_workspace_size(msa.MSA_OP_SELECT_TOKENS, ctypes.byref(kv), 2, 1, top_k) == \
            2 * 16 * 64 * 4
    assert lib.msa_workspace_size(msa.MSA_OP_DECODE, ctypes.byref(kv), 2, 1, 300) == 0
    P = ctypes.c_void_p
    ok = P(0x20000)
    # zero indexer heads, a null output, an unaligned query, a short workspace
    assert lib.msa_select_tokens(ctypes.byref(kv), ok, ok, 0, 16, ok, ok, 1 << 20, None) == \
        msa.MSA_ERR_INVALID_ARG
    assert lib.msa_select_tokens(ctypes.byref(kv), ok, ok, 4, 16, None, ok, 1 << 20, None) == \
        msa.MSA_ERR_INVALID_ARG
    assert lib.msa_select_tokens(ctypes.byref(kv), ok, P(0x20002), 4, 16, ok, ok, 1 << 20,
                                 None) == msa.MSA_ERR_INVALID_ARG
    assert lib.msa_select_tokens(ctypes.byref(kv), ok, ok, 4, 16, ok, ok, 100, None) == \
        msa.MSA_ERR_WORKSPACE
    assert lib.msa_sparse_attn_decode_tokens(ctypes.byref(kv), ok, ok, 0, 0.1, ok, None, None) == \
        msa.MSA_ERR_INVALID_ARG
    assert lib.msa_sparse_attn_decode_tokens(ctypes.byref(kv), ok, ok, 16, -1.0, ok, None,
                                             None) == msa.MSA_ERR_INVALID_ARG
