"""Context-sharded decode on one GPU: the shards of each sequence's blocks are
emulated in one process (caches that share the page pool, each page table
holding only its range), so every per-rank library call runs as it would on
its own GPU and the exchanges are plain stacks.

"Sparse Attention for Long-Context LLMs: Evolution and Practical Deployment",
section 8 (future directions): sharing index results across devices and
layers. The sharded selection must equal the unsharded one bit for bit (the
same scores, the same keys); the merged attention must match the unsharded
call and the oracle within the bf16 tolerance.
"""
import numpy as np
import pytest
import torch

import block_sparse_gqa_mean_b200 as msa
import oracle
import workloads
from msa_harness import append, check_selection, compare, fill_context, new_cache

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _shard(cache, lo, hi):
    """A rank's view: the same pages, page-table entries outside [lo, hi) cleared."""
    pt = cache.page_table.clone()
    cols = torch.arange(pt.shape[1], device=pt.device)
    pt[:, (cols < lo) | (cols >= hi)] = -1
    return msa.PagedKVCache(cache.k_pages, cache.v_pages, cache.centroids, pt, cache.seq_lens,
                            cache.status_word, cache.num_q_heads)


@pytest.mark.parametrize("bounds", [(0, 50, 130), (0, 1, 2, 150), (0, 200)],
                         ids=["three_ranks", "four_ranks_tiny_first", "two_ranks_one_empty"])
def test_sharded_decode_matches_unsharded(bounds):
    w = workloads.paged_decode_bf16(batch=3, ctx=(9000, 13000, 20000))
    p = workloads.paging(w)
    cache = new_cache(w, p)
    lens = fill_context(cache, w)
    after = [L + 1 for L in lens]
    append(cache, w, lens, after)
    q = workloads.queries_decode(w, 0, DEV)
    ref_idx, ref_sc = msa.select_topk(cache, q, w.top_k, want_scores=True)
    ref_out, ref_lse = msa.sparse_attn_decode(cache, q, ref_idx)
    ranges = list(zip(bounds, list(bounds[1:]) + [1 << 30]))
    shards = [_shard(cache, lo, hi) for lo, hi in ranges]
    keys = torch.stack([msa.select_topk_range(s, q, w.top_k, lo, hi)
                        for s, (lo, hi) in zip(shards, ranges)])
    idx, sc = msa.select_merge(cache, keys, w.top_k, want_scores=True)
    parts = [msa.sparse_attn_decode_range(s, q, idx, lo, hi) for s, (lo, hi) in zip(shards, ranges)]
    out, lse = msa.lse_merge(torch.stack([o for o, _ in parts]), torch.stack([l for _, l in parts]))
    torch.cuda.synchronize()
    assert cache.device_status() == 0            # no rank touched a page outside its range
    assert torch.equal(idx, ref_idx)
    assert torch.equal(sc.view(torch.int32), ref_sc.view(torch.int32))
    assert (out.float() - ref_out.float()).abs().max().item() <= 1e-2
    assert (lse - ref_lse).abs().max().item() <= 1e-4
    for b in range(w.batch):
        L = after[b]
        K, V = workloads.keys(w, b, 0, L), workloads.values(w, b, 0, L)
        pos = np.array([L - 1])
        orc = oracle.forward(q[b:b + 1].cpu(), K, V, pos, w.block, w.top_k, w.softmax_scale)
        check_selection(idx[b:b + 1].cpu().numpy(), orc, pos, w.top_k, w.block)
        O, _ = oracle.attend(q[b:b + 1].cpu(), K, V, pos, idx[b:b + 1].cpu().numpy(), w.block,
                             w.softmax_scale)
        compare(out[b:b + 1], O, "bf16")


def test_selection_reused_by_another_layer():
    """Cross-layer reuse of index results: the blocks chosen with one layer's
    queries and block cache drive another layer's attention (its own q, K, V)."""
    w1 = workloads.paged_decode_bf16(batch=2, ctx=(6000, 9000))
    w2 = workloads.paged_decode_bf16(batch=2, ctx=(6000, 9000), seed=workloads.SEED_BASE + 77)
    p = workloads.paging(w1)
    c1, c2 = new_cache(w1, p), new_cache(w2, p)
    lens = fill_context(c1, w1)
    fill_context(c2, w2)
    after = [L + 1 for L in lens]
    append(c1, w1, lens, after)
    append(c2, w2, lens, after)
    idx, _ = msa.select_topk(c1, workloads.queries_decode(w1, 0, DEV), w1.top_k)
    q2 = workloads.queries_decode(w2, 0, DEV)
    out, _ = msa.sparse_attn_decode(c2, q2, idx)
    torch.cuda.synchronize()
    assert c1.device_status() == 0 and c2.device_status() == 0
    for b in range(2):
        L = after[b]
        O, _ = oracle.attend(q2[b:b + 1].cpu(), workloads.keys(w2, b, 0, L),
                             workloads.values(w2, b, 0, L), np.array([L - 1]),
                             idx[b:b + 1].cpu().numpy(), w2.block, w2.softmax_scale)
        compare(out[b:b + 1], O, "bf16")


def test_range_arguments_rejected_on_the_host():
    w = workloads.paged_decode_bf16(batch=1, ctx=(3000,))
    cache = new_cache(w, workloads.paging(w))
    q = workloads.queries_decode(w, 0, DEV)
    with pytest.raises(msa.MsaError):
        msa.select_topk_range(cache, q, 100, 0, 10)      # top_k - 1 > 64
    with pytest.raises(msa.MsaError):
        msa.select_topk_range(cache, q, 8, 10, 5)        # empty, reversed range
