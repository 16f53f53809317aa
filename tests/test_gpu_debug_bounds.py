"""The bounds-checked library (libmsa_debug.so) on the GPU.

test_debug_library_parity_and_checks starts a child process whose binding
loads libmsa_debug.so (MSA_LIBRARY) and runs there:
  * parity cases against the oracle that reach every kernel family (append
    and pooling, prefill selection, decode pass 1 and merge, the tcgen05
    prefill attention with its clustering and plan kernels, the SIMT path,
    decode attention, the token variant, the context-sharded decode), each of
    which also asserts a clean status word: no check fires on valid input;
  * the two tests below, which break a launch-size precondition that the
    regular build cannot see (the caller's max rows / max new tokens per
    sequence smaller than a sequence's rows). The grid then covers only part
    of the rows, so no access leaves its buffer in either build; the regular
    build silently leaves the uncovered rows alone, the bounds-checked build
    reports MSA_DEV_BOUNDS. They skip under the regular library.
"""
import os
import subprocess
import sys

import pytest
import torch

import block_sparse_gqa_mean_b200 as msa
import workloads
from block_sparse_gqa_mean_b200 import build as libbuild

pytestmark = pytest.mark.gpu
DEV = "cuda"
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
TESTS = os.path.join(ROOT, "tests")

CASES = [
    "test_gpu_parity.py::test_append_pool_matches_oracle_and_rebuild",
    "test_gpu_parity.py::test_prefill_end_to_end",
    "test_gpu_parity.py::test_tiny_f32_prefill_and_decode",
    "test_gpu_parity.py::test_prefill_batch_varlen_chunked_and_index_edges",
    "test_gpu_parity.py::test_rows_without_blocks",
    "test_gpu_parity.py::test_decode_end_to_end",
    "test_gpu_parity.py::test_decode_repeated_and_empty_block_lists",
    "test_gpu_parity.py::test_device_status_on_bad_page_and_length",
    "test_gpu_tokens.py::test_token_decode_selection_and_attention",
    "test_gpu_tokens.py::test_token_prefill_selection_and_attention",
    "test_gpu_sharded.py::test_sharded_decode_matches_unsharded",
    "test_gpu_gate.py::test_decode_gated_splitk",
    "test_gpu_debug_bounds.py::test_rows_beyond_the_grid_are_reported",
    "test_gpu_debug_bounds.py::test_new_tokens_beyond_the_grid_are_reported",
]

CHILD = r"""
import sys
sys.path.insert(0, sys.argv[1])
sys.path.insert(0, sys.argv[2])
import block_sparse_gqa_mean_b200 as msa
assert msa.build_flags() == msa.MSA_BUILD_DEBUG_BOUNDS, "not the bounds-checked library"
import pytest
sys.exit(pytest.main(["-q", "-x", "-m", "gpu", "-p", "no:cacheprovider", "--rootdir", sys.argv[2]]
                     + [sys.argv[2] + "/" + c for c in sys.argv[3:]]))
"""


def _debug_library():
    return msa.build_flags() & msa.MSA_BUILD_DEBUG_BOUNDS


def test_debug_library_parity_and_checks():
    if _debug_library():
        pytest.skip("already running under the bounds-checked library")
    assert os.path.exists(libbuild.DEBUG_LIB), "build it: python -m block_sparse_gqa_mean_b200.build --debug-bounds"
    env = dict(os.environ, MSA_LIBRARY=libbuild.DEBUG_LIB)
    r = subprocess.run([sys.executable, "-c", CHILD, ROOT, TESTS, *CASES], env=env,
                       capture_output=True, text=True, timeout=1800, cwd=ROOT)
    tail = (r.stdout + r.stderr)[-4000:]
    assert r.returncode == 0, tail
    assert " passed" in r.stdout and " failed" not in r.stdout, tail


def _prefill_cache(T=700, top_k=4):
    w = workloads.prefill_bf16(ctx=(T,), top_k=top_k, steps=0)
    p = workloads.paging(w)
    cache = msa.PagedKVCache.allocate(1, p.num_pages, p.max_blocks, w.hq, w.hkv, w.d, w.block,
                                      torch.bfloat16, DEV)
    cache.page_table.copy_(p.table.to(DEV))
    return w, cache


def test_rows_beyond_the_grid_are_reported():
    if not _debug_library():
        pytest.skip("needs the bounds-checked library")
    T = 700
    w, cache = _prefill_cache(T)
    K = workloads.keys(w, 0, 0, T, DEV)
    V = workloads.values(w, 0, 0, T, DEV)
    cache.seq_lens.fill_(T)
    msa.build_block_cache(cache, K, V, msa.cu_seqlens([T], DEV), T)
    torch.cuda.synchronize()
    assert cache.device_status() == 0
    q = workloads.queries_prefill(w, 0, 0, T, DEV)
    cu = msa.cu_seqlens([T], DEV)
    # the caller promises at most T - 40 rows per sequence; the offsets say T
    idx, _ = msa.select_topk(cache, q, w.top_k, cu_q=cu, max_rows_per_seq=T - 40)
    torch.cuda.synchronize()
    assert cache.device_status() == msa.MSA_DEV_BOUNDS
    cache.clear_status()
    idx, _ = msa.select_topk(cache, q, w.top_k, cu_q=cu, max_rows_per_seq=T)
    msa.sparse_attn_prefill(cache, q, idx, cu_q=cu, max_rows_per_seq=T - 40)
    torch.cuda.synchronize()
    assert cache.device_status() == msa.MSA_DEV_BOUNDS
    cache.clear_status()
    msa.sparse_attn_prefill(cache, q, idx, cu_q=cu, max_rows_per_seq=T)
    torch.cuda.synchronize()
    assert cache.device_status() == 0


def test_new_tokens_beyond_the_grid_are_reported():
    if not _debug_library():
        pytest.skip("needs the bounds-checked library")
    T = 700
    w, cache = _prefill_cache(T)
    K = workloads.keys(w, 0, 0, T, DEV)
    V = workloads.values(w, 0, 0, T, DEV)
    cache.seq_lens.fill_(T)
    # T new tokens span six 128-token blocks; max_new = T // 2 sizes the grid for four
    msa.build_block_cache(cache, K, V, msa.cu_seqlens([T], DEV), T // 2)
    torch.cuda.synchronize()
    assert cache.device_status() == msa.MSA_DEV_BOUNDS
    cache.clear_status()
    msa.build_block_cache(cache, K, V, msa.cu_seqlens([T], DEV), T)
    torch.cuda.synchronize()
    assert cache.device_status() == 0
