"""Fused output gate O = g * A + (1 - g) * X against the oracle.

"Sparse Attention for Long-Context LLMs: Evolution and Practical Deployment",
section 4.3: the gate weights the sparse attention output against the other
branch and may be a scalar per head or vary with the dimension. A is checked
on the GPU's own block indices (the oracle attends the same blocks), so the
test isolates the gate and the epilogue it is fused into.
"""
import ctypes

import numpy as np
import pytest
import torch

import block_sparse_gqa_mean_b200 as msa
import oracle
import workloads
from msa_harness import append, compare, fill_context, new_cache

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _gates(shape, seed):
    g = torch.Generator().manual_seed(seed)
    per_head = torch.rand(shape[:2], generator=g)
    per_dim = torch.rand(shape, generator=g)
    # the other branch at the scale of attention outputs: the bf16 bound
    # (max-abs 1e-2) includes the output's own rounding, 2^-9 of its magnitude
    x = torch.randn(shape, generator=g) * 0.5
    return per_head.to(DEV), per_dim.to(DEV), x


@pytest.mark.parametrize("over", [dict(ctx=(1200,), top_k=4),                 # tcgen05 path
                                  dict(ctx=(500,), hq=16, hkv=4, top_k=3)],   # SIMT path
                         ids=["tc", "simt"])
def test_prefill_gated(over):
    w = workloads.prefill_bf16(**over)
    p = workloads.paging(w)
    cache = new_cache(w, p)
    T = w.ctx[0]
    append(cache, w, [0], [T])
    q = workloads.queries_prefill(w, 0, 0, T, DEV)
    cu = msa.cu_seqlens([T], DEV)
    idx, _ = msa.select_topk(cache, q, w.top_k, cu_q=cu, max_rows_per_seq=T)
    gh, gd, x = _gates(tuple(q.shape), 3)
    xq = x.to(q.dtype).to(DEV)
    outs = {}
    for name, g in (("head", gh), ("dim", gd)):
        outs[name], _ = msa.sparse_attn_prefill(cache, q, idx, cu_q=cu, max_rows_per_seq=T,
                                                gate=g, x=xq)
    plain, _ = msa.sparse_attn_prefill(cache, q, idx, cu_q=cu, max_rows_per_seq=T)
    torch.cuda.synchronize()
    assert cache.device_status() == 0
    K, V = workloads.keys(w, 0, 0, T), workloads.values(w, 0, 0, T)
    A, _ = oracle.attend(q.cpu(), K, V, np.arange(T), idx.cpu().numpy(), w.block, w.softmax_scale)
    compare(plain, A, w.dtype)
    compare(outs["head"], oracle.gate(A, gh.cpu().numpy(), xq.cpu()), w.dtype)
    compare(outs["dim"], oracle.gate(A, gd.cpu().numpy(), xq.cpu()), w.dtype)


def test_tiny_f32_gated_prefill_and_decode():
    w = workloads.tiny_f32()
    T = w.ctx[0]
    p = workloads.paging(w)
    cache = new_cache(w, p)
    append(cache, w, [0], [T - 1])
    q = workloads.queries_prefill(w, 0, 0, T - 1, DEV)
    cu = msa.cu_seqlens([T - 1], DEV)
    idx, _ = msa.select_topk(cache, q, w.top_k, cu_q=cu, max_rows_per_seq=T - 1)
    gh, _, x = _gates(tuple(q.shape), 4)
    x = x.to(DEV)
    out, _ = msa.sparse_attn_prefill(cache, q, idx, cu_q=cu, max_rows_per_seq=T - 1, gate=gh, x=x)
    # decode of the last token, per-coordinate gate
    append(cache, w, [T - 1], [T])
    qd = workloads.queries_prefill(w, 0, T - 1, T, DEV)
    idd, _ = msa.select_topk(cache, qd, w.top_k)
    _, gdd, xd = _gates(tuple(qd.shape), 5)
    xd = xd.to(DEV)
    outd, _ = msa.sparse_attn_decode(cache, qd, idd, gate=gdd, x=xd)
    torch.cuda.synchronize()
    assert cache.device_status() == 0
    K, V = workloads.keys(w, 0, 0, T), workloads.values(w, 0, 0, T)
    A, _ = oracle.attend(q.cpu(), K[:T - 1], V[:T - 1], np.arange(T - 1), idx.cpu().numpy(),
                         w.block, w.softmax_scale)
    compare(out, oracle.gate(A, gh.cpu().numpy(), x.cpu()), "f32")
    Ad, _ = oracle.attend(qd.cpu(), K, V, np.array([T - 1]), idd.cpu().numpy(), w.block,
                          w.softmax_scale)
    compare(outd, oracle.gate(Ad, gdd.cpu().numpy(), xd.cpu()), "f32")


def test_decode_gated_splitk():
    w = workloads.paged_decode_bf16(batch=3, ctx=(3000, 5000, 4096))
    p = workloads.paging(w)
    cache = new_cache(w, p)
    lens = fill_context(cache, w)
    after = [L + 1 for L in lens]
    append(cache, w, lens, after)
    q = workloads.queries_decode(w, 0, DEV)
    idx, _ = msa.select_topk(cache, q, w.top_k)
    gh, gd, x = _gates(tuple(q.shape), 6)
    # the other branch may be the query itself (the page's form)
    out_q, _ = msa.sparse_attn_decode(cache, q, idx, gate=gh, x=q)
    out_d, _ = msa.sparse_attn_decode(cache, q, idx, gate=gd, x=x.to(q.dtype).to(DEV))
    torch.cuda.synchronize()
    assert cache.device_status() == 0
    for b in range(w.batch):
        L = after[b]
        K, V = workloads.keys(w, b, 0, L), workloads.values(w, b, 0, L)
        A, _ = oracle.attend(q[b:b + 1].cpu(), K, V, np.array([L - 1]),
                             idx[b:b + 1].cpu().numpy(), w.block, w.softmax_scale)
        compare(out_q[b:b + 1], oracle.gate(A, gh[b:b + 1].cpu().numpy(), q[b:b + 1].cpu()),
                w.dtype)
        compare(out_d[b:b + 1], oracle.gate(A, gd[b:b + 1].cpu().numpy(),
                                            x[b:b + 1].to(q.dtype)), w.dtype)


def test_gated_argument_errors():
    w = workloads.paged_decode_bf16(batch=1, ctx=(1000,))
    cache = new_cache(w, workloads.paging(w))
    q = torch.zeros(1, w.hq, w.d, dtype=torch.bfloat16, device=DEV)
    idx = torch.zeros(1, w.hkv, w.top_k, dtype=torch.int32, device=DEV)
    out = torch.empty_like(q)
    g = torch.zeros(1, w.hq, device=DEV)
    lib = msa.load_library()
    kv = cache.struct()
    P = ctypes.c_void_p
    for gate, per_dim, x in ((None, 0, q), (g, 0, None), (g, 2, q)):
        st = lib.msa_sparse_attn_decode_gated(
            ctypes.byref(kv), P(q.data_ptr()), P(idx.data_ptr()), w.top_k, 0.1,
            None if gate is None else P(gate.data_ptr()), per_dim,
            None if x is None else P(x.data_ptr()), P(out.data_ptr()), None, None, 0, None)
        assert st == msa.MSA_ERR_INVALID_ARG
    with pytest.raises(ValueError):
        msa.sparse_attn_decode(cache, q, idx, gate=torch.zeros(1, 3, device=DEV), x=q)
