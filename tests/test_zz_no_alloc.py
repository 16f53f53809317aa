"""The allocation-free decode entry point against the regular one.

msa_sparse_attn_decode_noalloc serves callers that cannot allocate device
memory at the call (a plugin inside a framework that owns the memory pool, an
allocator-free latency loop): it keeps its split-k scratch in a fixed 8 MiB
device array inside the library. This file is collected last on purpose, so a
run that stops at the first failure has run every other test first; it also
passes on its own in a fresh process (the first call sets up the array's
device address).
"""
import ctypes

import pytest
import torch

import block_sparse_gqa_mean_b200 as msa
import workloads
from msa_harness import TOL, append, fill_context, new_cache

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _decode_case():
    w = workloads.paged_decode_bf16(batch=4, ctx=(3000, 4095, 4096, 5000))
    p = workloads.paging(w)
    cache = new_cache(w, p)
    lens = fill_context(cache, w)
    append(cache, w, lens, [L + 1 for L in lens])
    q = workloads.queries_decode(w, 0, DEV)
    idx, _ = msa.select_topk(cache, q, w.top_k)
    return w, cache, q, idx


def test_noalloc_decode_matches_regular_entry_point_twice():
    w, cache, q, idx = _decode_case()
    ref, ref_lse = msa.sparse_attn_decode(cache, q, idx)
    torch.cuda.synchronize()
    for _ in range(2):  # two calls in a row share the library's scratch array
        out = torch.full_like(q, float("nan"))
        lse = torch.full((q.shape[0], q.shape[1]), float("nan"), device=DEV)
        msa.sparse_attn_decode_noalloc(cache, q, idx, out, lse)
        torch.cuda.synchronize()
        err = (out.float() - ref.float()).abs().max().item()
        rel = ((out.float() - ref.float()).norm() / ref.float().norm()).item()
        assert err <= TOL["bf16"]["max_abs"] and rel <= TOL["bf16"]["rel_l2"], (err, rel)
        assert (lse - ref_lse).abs().max().item() <= 1e-4
    assert cache.device_status() == 0


def test_noalloc_rejects_problems_beyond_its_scratch():
    w, cache, q, idx = _decode_case()
    kv = cache.struct()
    kv.batch = 100000  # split-k partials would need far more than 8 MiB
    lib = msa.load_library()
    st = lib.msa_sparse_attn_decode_noalloc(ctypes.byref(kv), q.data_ptr(), idx.data_ptr(),
                                            w.top_k, 0.0884, q.data_ptr(), None, None)
    assert st == msa.MSA_ERR_WORKSPACE
