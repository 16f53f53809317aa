"""Parity at the full workload sizes, in the launch configuration bench.py times.

The oracle checks sampled outputs it can compute one by one:
  * prefill (batch 1, 32768 tokens, 32/4 heads, d 128, block 128, top-k 16):
    288 rows spread across the sequence, most of them at block edges (the
    first, second and last token of a block) and the rest at random;
  * paged decode (batch 32 x 131072 cached tokens, block 64, top-k 32; 8 of
    the 32 sequences) and varlen decode (64 sequences of 4K-512K tokens,
    block 64, top-k 64; the shortest, the longest and four lengths between):
    whole sampled sequences;
  * 1M-context decode (1048576 cached tokens, block 128, top-k 16): all 256
    consecutive decode steps run, each appending one token; at steps 0, 127,
    128 (the first token of a new block) and 255 the oracle rebuilds every
    block's representation from the full key history and checks the whole
    selection (bit-exact on groups whose top-k gap is >= 1e-2) and the output.
    The keys are drawn on the GPU and copied to the host: the generator gives
    the same bits on both devices.
"""
import numpy as np
import pytest
import torch

import block_sparse_gqa_mean_b200 as msa
import oracle
import workloads
from msa_harness import append, check_selection, compare, fill_context, new_cache

pytestmark = [pytest.mark.gpu, pytest.mark.slow]
DEV = "cuda"


def test_full_prefill_sampled_rows():
    w = workloads.prefill_bf16()
    T = w.ctx[0]
    p = workloads.paging(w)
    cache = new_cache(w, p)
    append(cache, w, [0], [T])
    q = workloads.queries_prefill(w, 0, 0, T, DEV)
    cu = msa.cu_seqlens([T], DEV)
    idx, _ = msa.select_topk(cache, q, w.top_k, cu_q=cu, max_rows_per_seq=T)
    out, lse = msa.sparse_attn_prefill(cache, q, idx, cu_q=cu, max_rows_per_seq=T)
    torch.cuda.synchronize()
    assert cache.device_status() == 0
    rng = np.random.default_rng(7)
    blocks = rng.choice(T // w.block, 64, replace=False)
    edges = np.concatenate([blocks * w.block, blocks * w.block + 1, blocks * w.block + w.block - 1])
    rows = np.unique(np.concatenate([[0, 1, 127, 128, 129, 2047, 2048, T - 1], edges,
                                     rng.integers(0, T, 96)]))
    assert len(rows) >= 256
    K, V = workloads.keys(w, 0, 0, T), workloads.values(w, 0, 0, T)
    Q = workloads.queries_prefill(w, 0, 0, T)[torch.from_numpy(rows)]
    orc = oracle.forward(Q, K, V, rows, w.block, w.top_k, w.softmax_scale)
    gi = idx.cpu().numpy()[rows]
    check_selection(gi, orc, rows, w.top_k, w.block)
    same = (gi == orc["idx"]).all(-1).all(-1)
    assert same.mean() > 0.5
    compare(out[torch.from_numpy(rows[same]).to(DEV)], orc["out"][same], "bf16")
    # rows whose selection differs within fp32 ties: attention on the oracle's indices
    if not same.all():
        idx2 = idx.clone()
        idx2[torch.from_numpy(rows).to(DEV)] = torch.from_numpy(orc["idx"]).to(DEV)
        out2, _ = msa.sparse_attn_prefill(cache, q, idx2, cu_q=cu, max_rows_per_seq=T)
        torch.cuda.synchronize()
        compare(out2[torch.from_numpy(rows).to(DEV)], orc["out"], "bf16")


def _decode_step(w, cache):
    lens = fill_context(cache, w)
    after = [L + 1 for L in lens]
    append(cache, w, lens, after)
    q = workloads.queries_decode(w, 0, DEV)
    idx, _ = msa.select_topk(cache, q, w.top_k)
    out, lse = msa.sparse_attn_decode(cache, q, idx)
    torch.cuda.synchronize()
    assert cache.device_status() == 0
    return after, q, idx, out


@pytest.mark.parametrize("make,seqs", [
    (workloads.paged_decode_bf16, (0, 5, 11, 15, 19, 23, 27, 31)),
    (workloads.varlen_decode_bf16, None),
], ids=["paged_decode", "varlen_decode"])
def test_full_decode_sampled_sequences(make, seqs):
    w = make()
    if seqs is None:  # the shortest, the longest and four lengths between, by rank
        order = np.argsort(np.array(w.ctx))
        n = len(order)
        seqs = tuple(int(order[i]) for i in (0, n // 5, 2 * n // 5, 3 * n // 5, 4 * n // 5, n - 1))
    p = workloads.paging(w)
    cache = new_cache(w, p)
    lens, q, idx, out = _decode_step(w, cache)
    for b in seqs:
        L = lens[b]
        K, V = workloads.keys(w, b, 0, L), workloads.values(w, b, 0, L)
        orc = oracle.forward(q[b:b + 1].cpu(), K, V, np.array([L - 1]), w.block, w.top_k,
                             w.softmax_scale)
        check_selection(idx[b:b + 1].cpu().numpy(), orc, np.array([L - 1]), w.top_k, w.block)
        O, _ = oracle.attend(q[b:b + 1].cpu(), K, V, np.array([L - 1]),
                             idx[b:b + 1].cpu().numpy(), w.block, w.softmax_scale)
        compare(out[b:b + 1], O, "bf16")


def test_full_1m_decode_against_oracle():
    w = workloads.decode_1m_bf16()
    assert w.steps == 256
    p = workloads.paging(w)
    cache = new_cache(w, p)
    L0, Lf, B = w.ctx[0], w.ctx[0] + w.steps, w.block
    Kd = workloads.keys(w, 0, 0, Lf, DEV)      # every key the run will ever hold
    Vd = workloads.values(w, 0, 0, Lf, DEV)
    chunk = 1 << 16
    for u0 in range(0, L0, chunk):
        u1 = min(L0, u0 + chunk)
        append(cache, w, [u0], [u1], k_rows=Kd[u0:u1], v_rows=Vd[u0:u1])
    checked = {0: None, 127: None, 128: None, 255: None}
    for step in range(w.steps):
        L = L0 + step + 1
        append(cache, w, [L - 1], [L], k_rows=Kd[L - 1:L], v_rows=Vd[L - 1:L])
        q = workloads.queries_decode(w, step, DEV)
        idx, _ = msa.select_topk(cache, q, w.top_k)
        out, lse = msa.sparse_attn_decode(cache, q, idx)
        if step in checked:
            checked[step] = (q.cpu(), idx.cpu().numpy(), out.clone(), lse.cpu().double().numpy())
    torch.cuda.synchronize()
    assert cache.device_status() == 0
    K, V = Kd.cpu(), Vd.cpu()
    del Kd, Vd
    protected = []
    for step, (qc, gi, out, lse) in checked.items():
        L = L0 + step + 1
        pos = np.array([L - 1])
        orc = oracle.forward(qc, K[:L], V[:L], pos, B, w.top_k, w.softmax_scale)
        stats = check_selection(gi, orc, pos, w.top_k, B)
        protected.append(stats["protected_frac"])
        O, ls = oracle.attend(qc, K[:L], V[:L], pos, gi, B, w.softmax_scale)
        compare(out, O, "bf16")
        assert np.abs(lse - ls).max() < 2e-3
        if np.array_equal(gi, orc["idx"]):
            compare(out, orc["out"], "bf16")
    assert np.mean(protected) > 0.8, protected
