"""The allocation-free decode entry point against the regular one.

msa_sparse_attn_decode_noalloc serves callers that cannot allocate device
memory at the call (a plugin inside a framework that owns the memory pool, an
allocator-free latency loop): it keeps its attention scratch in a fixed 8 MiB
device array inside the library. It runs the same kernels as
msa_sparse_attn_decode, so its outputs must equal the regular entry point's
bit for bit, call after call, and a call must not change the device's free
memory. This file is collected last on purpose, so a run that stops at the
first failure has run every other test first; it also passes on its own in a
fresh process (the first call sets up the array's device address).
"""
import ctypes

import numpy as np
import pytest
import torch

import block_sparse_gqa_mean_b200 as msa
import workloads
from msa_harness import append, fill_context, new_cache

pytestmark = pytest.mark.gpu
DEV = "cuda"
SCRATCH_BYTES = 8 << 20


def _decode_case(batch=4, ctx=(3000, 4095, 4096, 5000)):
    w = workloads.paged_decode_bf16(batch=batch, ctx=ctx)
    p = workloads.paging(w)
    cache = new_cache(w, p)
    lens = fill_context(cache, w) if batch <= 8 else _fill_all(cache, w)
    append(cache, w, lens, [L + 1 for L in lens])
    q = workloads.queries_decode(w, 0, DEV)
    idx, _ = msa.select_topk(cache, q, w.top_k)
    return w, cache, q, idx


def _fill_all(cache, w):
    append(cache, w, [0] * w.batch, list(w.ctx))
    return list(w.ctx)


def _noalloc(cache, q, idx, top_k, out, lse):
    lib = msa.load_library()
    kv = cache.struct()
    return lib.msa_sparse_attn_decode_noalloc(ctypes.byref(kv), q.data_ptr(), idx.data_ptr(),
                                              top_k, 1.0 / 128 ** 0.5, out.data_ptr(),
                                              lse.data_ptr(), None)


def _same_bits(a, b):
    return torch.equal(a.view(torch.int16) if a.dtype == torch.bfloat16 else a.view(torch.int32),
                       b.view(torch.int16) if b.dtype == torch.bfloat16 else b.view(torch.int32))


def _check_twice_against_regular(w, cache, q, idx):
    ref, ref_lse = msa.sparse_attn_decode(cache, q, idx)
    torch.cuda.synchronize()
    for _ in range(2):  # two calls in a row share the library's scratch array
        out = torch.full_like(q, float("nan"))
        lse = torch.full((q.shape[0], q.shape[1]), float("nan"), device=DEV)
        assert _noalloc(cache, q, idx, w.top_k, out, lse) == msa.MSA_OK
        torch.cuda.synchronize()
        assert _same_bits(out, ref) and _same_bits(lse, ref_lse)
    assert cache.device_status() == 0


def test_noalloc_decode_matches_regular_entry_point_twice():
    w, cache, q, idx = _decode_case()
    _check_twice_against_regular(w, cache, q, idx)


def test_noalloc_allocates_nothing():
    w, cache, q, idx = _decode_case()
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[0], q.shape[1], device=DEV)
    assert _noalloc(cache, q, idx, w.top_k, out, lse) == msa.MSA_OK  # address set-up done
    torch.cuda.synchronize()
    alloc0 = torch.cuda.memory_allocated()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        assert _noalloc(cache, q, idx, w.top_k, out, lse) == msa.MSA_OK
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert torch.cuda.memory_allocated() == alloc0
    assert free1 == free0


def _decode_need(cache, top_k, batch, hq=None, hkv=None):
    """msa_workspace_size(MSA_OP_DECODE) for a copy of the descriptor."""
    lib = msa.load_library()
    kv = cache.struct()
    kv.batch = batch
    if hq is not None:
        kv.num_q_heads, kv.num_kv_heads = hq, hkv
    return int(lib.msa_workspace_size(msa.MSA_OP_DECODE, ctypes.byref(kv), batch, 1, top_k))


def test_noalloc_scratch_covers_every_batch():
    """The decode workspace holds one part per resident CTA: it does not grow
    with the batch, and at 16 query heads per group (the most the kernels
    take) it stays under the 8 MiB array."""
    probe = new_cache(workloads.paged_decode_bf16(batch=1, ctx=(64,)),
                      workloads.paging(workloads.paged_decode_bf16(batch=1, ctx=(64,))))
    needs = {b: _decode_need(probe, 32, b) for b in (1, 7, 64, 1000, 65535)}
    assert len(set(needs.values())) == 1, needs
    assert _decode_need(probe, 256, 65535, hq=128, hkv=8) <= SCRATCH_BYTES


def test_noalloc_large_batch_matches_regular():
    rng = np.random.default_rng(3)
    ctx = tuple(int(x) for x in rng.integers(100, 700, 160))
    w, cache, q, idx = _decode_case(batch=160, ctx=ctx)
    _check_twice_against_regular(w, cache, q, idx)


def test_noalloc_rejects_bad_arguments_first():
    w, cache, q, idx = _decode_case()
    lib = msa.load_library()
    kv = cache.struct()
    out = torch.empty_like(q)
    # a null query or a zero scale is an argument error, not a scratch problem
    assert lib.msa_sparse_attn_decode_noalloc(ctypes.byref(kv), None, idx.data_ptr(), w.top_k,
                                              0.0884, out.data_ptr(), None, None) == \
        msa.MSA_ERR_INVALID_ARG
    assert lib.msa_sparse_attn_decode_noalloc(ctypes.byref(kv), q.data_ptr(), idx.data_ptr(),
                                              w.top_k, 0.0, out.data_ptr(), None, None) == \
        msa.MSA_ERR_INVALID_ARG
    assert lib.msa_sparse_attn_decode_noalloc(ctypes.byref(kv), q.data_ptr(), idx.data_ptr(),
                                              0, 0.0884, out.data_ptr(), None, None) == \
        msa.MSA_ERR_UNSUPPORTED
