"""The exchange of context-sharded decode on CPU: two gloo ranks run
block_sparse_gqa_mean_b200.sharded_decode, each holding half of every
sequence's blocks.

The per-rank steps are stood in for by the fp64 oracle (no GPU here): a rank
keeps the best k-1 candidate blocks of its range, the lists are all-gathered
and merged into the global selection, each rank attends over the selected
blocks it holds, and the partials are all-gathered and merged by log-sum-exp.
The result must equal the oracle on the unsharded sequences: the selection
exactly, the output to fp64 rounding. This checks the exchange (what is
gathered, in which order, and the two merges), not the kernels; the GPU test
of the same path runs the library's kernels for every rank.
"""
import os
import socket
import sys

import numpy as np
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
BLOCK, TOP_K, HKV, HQ, D = 16, 5, 2, 4, 32
LENS = (300, 161, 97)      # tokens per sequence (the last one is the decode row)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs():
    g = torch.Generator().manual_seed(5)
    seqs = []
    for L in LENS:
        K = torch.randn(L, HKV, D, generator=g)
        V = torch.randn(L, HKV, D, generator=g)
        Q = torch.randn(1, HQ, D, generator=g)
        seqs.append((Q, K, V))
    return seqs


def _oracle_ops(seqs):
    import oracle
    scale = 1.0 / np.sqrt(D)

    def scores(b):
        Q, K, V = seqs[b]
        L = K.shape[0]
        return oracle.scores(Q, np.array([L - 1]), oracle.centroids(K, BLOCK), BLOCK)[0]  # [HKV, nblk]

    def select(cache, q, top_k, lo, hi):  # local candidates: block ids, best first, -1 padded
        out = torch.full((len(seqs), HKV, top_k - 1), -1, dtype=torch.int64)
        for b in range(len(seqs)):
            S = scores(b)
            own = (seqs[b][1].shape[0] - 1) // BLOCK
            cand = np.arange(max(lo, 0), min(hi, own))
            for g in range(HKV):
                order = cand[np.lexsort((cand, -S[g, cand]))][:top_k - 1] if len(cand) else cand
                out[b, g, :len(order)] = torch.from_numpy(order)
        return out

    def merge(cache, gathered, top_k):    # [world, batch, HKV, k-1] -> [batch, HKV, k]
        idx = np.full((len(seqs), HKV, top_k), -1, dtype=np.int32)
        for b in range(len(seqs)):
            S = scores(b)
            own = (seqs[b][1].shape[0] - 1) // BLOCK
            for g in range(HKV):
                cand = np.unique(gathered[:, b, g].numpy())
                cand = cand[cand >= 0]
                order = cand[np.lexsort((cand, -S[g, cand]))][:top_k - 1] if len(cand) else cand
                sel = np.sort(np.concatenate([order, [own]]))
                idx[b, g, :len(sel)] = sel
        return torch.from_numpy(idx), None

    def attend(cache, q, block_idx, lo, hi):  # this rank's blocks only
        o = torch.zeros(len(seqs), HQ, D, dtype=torch.float64)
        lse = torch.full((len(seqs), HQ), -np.inf, dtype=torch.float64)
        for b in range(len(seqs)):
            Q, K, V = seqs[b]
            L = K.shape[0]
            mine = block_idx[b:b + 1].numpy().copy()
            mine[(mine < lo) | (mine >= hi)] = -1
            if (mine >= 0).any():
                O, ls = oracle.attend(Q, K, V, np.array([L - 1]), mine, BLOCK, scale)
                o[b], lse[b] = torch.from_numpy(O[0]), torch.from_numpy(ls[0])
        return o, lse

    def combine(o_all, l_all, dtype=None):
        M = l_all.max(0).values
        w = torch.where(torch.isfinite(l_all), torch.exp(l_all - M), torch.zeros_like(l_all))
        out = (w[..., None] * o_all).sum(0) / w.sum(0)[..., None]
        return out, M + torch.log(w.sum(0))

    return {"select": select, "merge": merge, "attend": attend, "combine": combine}


def _rank_main(rank, world, port, out_dir):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import block_sparse_gqa_mean_b200 as msa
    dist.init_process_group("gloo", rank=rank, world_size=world)
    seqs = _inputs()
    nblk = max((L + BLOCK - 1) // BLOCK for L in LENS)
    per = (nblk + world - 1) // world
    lo, hi = rank * per, (rank + 1) * per if rank < world - 1 else 1 << 30
    q = torch.cat([s[0] for s in seqs])
    out, lse, idx = msa.sharded_decode(None, q, TOP_K, lo, hi, ops=_oracle_ops(seqs))
    torch.save({"out": out, "lse": lse, "idx": idx}, os.path.join(out_dir, f"rank{rank}.pt"))
    dist.destroy_process_group()


def test_two_gloo_ranks_match_the_unsharded_oracle(tmp_path):
    sys.path.insert(0, ROOT)
    import oracle
    world = 2
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    res = [torch.load(tmp_path / f"rank{r}.pt") for r in range(world)]
    assert torch.equal(res[0]["idx"], res[1]["idx"]) and torch.equal(res[0]["out"], res[1]["out"])
    for b, (Q, K, V) in enumerate(_inputs()):
        L = K.shape[0]
        ref = oracle.forward(Q, K, V, np.array([L - 1]), BLOCK, TOP_K, 1.0 / np.sqrt(D))
        assert np.array_equal(res[0]["idx"][b].numpy(), ref["idx"][0])
        assert np.abs(res[0]["out"][b].numpy() - ref["out"][0]).max() < 1e-12
        assert np.abs(res[0]["lse"][b].numpy() - ref["lse"][0]).max() < 1e-12
