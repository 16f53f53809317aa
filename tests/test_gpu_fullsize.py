"""Parity at the full workload sizes, in the launch configuration bench.py times.

The oracle checks sampled outputs it can compute one by one:
  * prefill (batch 1, 32768 tokens, 32/4 heads, d 128, block 128, top-k 16):
    rows sampled across the sequence (first tokens, block edges, the end);
  * paged decode (batch 32 x 131072 cached tokens, block 64, top-k 32) and
    varlen decode (64 sequences of 4K-512K tokens, block 64, top-k 64): whole
    sampled sequences;
  * 1M-context decode (1048576 cached tokens, block 128, top-k 16): the oracle
    cannot rebuild every block's representation on the host in test time, so it
    checks what holds at any size from the blocks it does rebuild: attention over
    the GPU-selected blocks exactly, every selected block's centroid, and that
    no sampled rejected block outscores a selected one by more than 1e-3.
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
    rows = np.unique(np.concatenate([[0, 1, 127, 128, 129, 2047, 2048, T - 1],
                                     rng.integers(0, T, 40)]))
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
    (workloads.paged_decode_bf16, (0, 31)),
    (workloads.varlen_decode_bf16, None),
], ids=["paged_decode", "varlen_decode"])
def test_full_decode_sampled_sequences(make, seqs):
    w = make()
    if seqs is None:  # the shortest and a middle-length sequence
        order = np.argsort(np.array(w.ctx))
        seqs = (int(order[0]), int(order[len(order) // 2]))
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


def test_full_1m_decode_properties():
    w = workloads.decode_1m_bf16(steps=2)
    p = workloads.paging(w)
    cache = new_cache(w, p)
    lens = fill_context(cache, w)
    rng = np.random.default_rng(11)
    for step in range(w.steps):
        after = [w.ctx[0] + step + 1]
        append(cache, w, lens, after)
        lens = after
        q = workloads.queries_decode(w, step, DEV)
        idx, _ = msa.select_topk(cache, q, w.top_k)
        out, _ = msa.sparse_attn_decode(cache, q, idx)
        torch.cuda.synchronize()
        assert cache.device_status() == 0
        L, B = lens[0], w.block
        own = (L - 1) // B
        sel = idx[0].cpu().numpy()                                # [Hkv, k]
        for g in range(w.hkv):
            assert sel[g, -1] == own and np.all(np.diff(sel[g]) > 0) and sel[g, 0] >= 0
        # compact copy of the selected blocks (union over groups), renumbered, for
        # an exact oracle attention over them; the own block keeps its position
        blocks = sorted(set(int(j) for j in sel.ravel()))
        remap = {j: n for n, j in enumerate(blocks)}
        Kc = torch.cat([workloads.keys(w, 0, j * B, min((j + 1) * B, L)) for j in blocks])
        Vc = torch.cat([workloads.values(w, 0, j * B, min((j + 1) * B, L)) for j in blocks])
        t_c = (len(blocks) - 1) * B + (L - 1 - own * B)
        idx_c = np.vectorize(remap.get)(sel)[None].astype(np.int32)
        O, _ = oracle.attend(q.cpu(), Kc, Vc, np.array([t_c]), idx_c, B, w.softmax_scale)
        compare(out, O, "bf16")
        # centroids of the selected blocks and of sampled rejected blocks, from the keys
        chosen = set(blocks)
        rejected = [int(j) for j in rng.choice(own, 96, replace=False) if int(j) not in chosen]
        qb = q.cpu().double().view(w.hkv, w.group, w.d).sum(1)       # [Hkv, d]
        score = {}
        for j in blocks[:-1] + rejected:
            kj = workloads.keys(w, 0, j * B, (j + 1) * B).double()    # [B, Hkv, d]
            cj = kj.mean(0)                                           # [Hkv, d]
            got = cache.centroids[int(p.table[0, j])].cpu().double()
            assert torch.all((got - cj).abs() <= 1e-6 * torch.maximum(cj.abs(), kj.abs().mean(0)))
            score[j] = (qb * cj).sum(-1)                              # [Hkv]
        for g in range(w.hkv):
            worst = min(float(score[int(c)][g]) for c in sel[g] if c != own)
            best_rejected = max(float(score[j][g]) for j in rejected)
            assert best_rejected <= worst + 1e-3, (g, best_rejected, worst)
